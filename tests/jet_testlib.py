"""Helpers shared by the parity tests: moving the seeded inputs to the GPU,
running the library through its C ABI, and the error measures of the pass
criteria (relative L2 and max-abs against the float64 oracle)."""
from __future__ import annotations

import numpy as np
import torch

from synth import to_f64

# pass criteria: bf16 inputs -> rel-L2 <= 1e-2 and max-abs <= 5e-2; float32 -> rel-L2 <= 1e-4
TOL = {"bf16": dict(rel_l2=1e-2, max_abs=5e-2), "f32": dict(rel_l2=1e-4, max_abs=None)}


def dev(a: np.ndarray, dtype: str, device="cuda") -> torch.Tensor:
    """Stored array (bf16 bits as uint16, or float32) -> CUDA tensor of the same bits."""
    if a.dtype == np.uint16:
        return torch.from_numpy(a.view(np.int16)).to(device).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(device)


def host64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to("cpu", torch.float64).numpy()


def errors(got: np.ndarray, ref: np.ndarray) -> dict:
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.all(np.isfinite(got)), "non-finite values in GPU output"
    diff = got - ref
    den = np.linalg.norm(ref.ravel())
    return dict(rel_l2=float(np.linalg.norm(diff.ravel()) / max(den, 1e-300)),
                max_abs=float(np.max(np.abs(diff))) if diff.size else 0.0)


def assert_close(got, ref, dtype: str, what: str = "", tol: dict | None = None) -> dict:
    tol = tol or TOL[dtype]
    e = errors(got, ref)
    assert e["rel_l2"] <= tol["rel_l2"], f"{what}: rel-L2 {e['rel_l2']:.3e} > {tol['rel_l2']}"
    if tol.get("max_abs") is not None:
        assert e["max_abs"] <= tol["max_abs"], f"{what}: max-abs {e['max_abs']:.3e} > {tol['max_abs']}"
    return e


def to_oracle(inp: dict, keys=("x", "W1", "W2", "q", "k", "v", "g", "beta")) -> dict:
    """Exact float64 values of the stored inputs, for the oracle."""
    dt = inp["dtype"]
    return {key: to_f64(inp[key], dt) for key in keys if key in inp}


def gpu_inputs(inp: dict) -> dict:
    dt = inp["dtype"]
    return {key: dev(val, dt) for key, val in inp.items() if isinstance(val, np.ndarray)}
