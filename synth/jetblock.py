"""Workload shapes and the seeded input recipe for the JetBlock token mixer.

Shapes follow the Jet-Nemotron explainer (xugj520.cn, section 2.2 "JetBlock"):
q/k head dim 96 (2B) or 128 (4B), v head dim 256, 12 or 16 heads, conv kernel
size 4, generator hidden width 32. d_model is that of the base models the
paper builds on (Jet-Nemotron paper, section 3.1: 1536 for the 2B model, 2048
for the 4B model).

Recipe (numpy PCG64, one generator per call, all draws float64, in this order):
x, q, k, v, beta_raw, g_raw, W1, W2, then (decode only) the state and the conv
history.
  x, q, k, v ~ N(0, 1); q and k divided by their per-head L2 norm
  beta = sigmoid(beta_raw), g = -gate_scale * softplus(g_raw), beta_raw, g_raw ~ N(0, 1)
  W1 ~ N(0, 1/D), W2 ~ N(0, 1/32)                      (variance 1/fan_in)
  decode state ~ N(0, 0.02^2) float32, history ~ N(0, 1) in the bulk dtype
Bulk tensors (x, q, k, v, W1, W2, history) are stored in the config dtype:
bf16 (as uint16 bit patterns, round-to-nearest-even from float32) or float32.
g, beta and states are always float32.
"""
from __future__ import annotations

from dataclasses import dataclass, replace
import numpy as np

GEN_HIDDEN = 32      # kernel-generator hidden width (explainer, section 2.2)
CONV_WIDTH = 4       # dynamic causal conv kernel size (explainer, section 2.2)
CHUNK = 64           # prefill chunk length


@dataclass(frozen=True)
class JetShape:
    name: str
    B: int
    T: int            # prefill tokens per sequence (0 for pure decode workloads)
    H: int
    dk: int
    dv: int
    D: int
    dtype: str = "bf16"   # "bf16" or "f32": dtype of x, q, k, v, v', o, W1, W2
    steps: int = 0        # decode steps (one token per sequence per step)
    R: int = GEN_HIDDEN
    W: int = CONV_WIDTH

    def with_(self, **kw) -> "JetShape":
        return replace(self, **kw)


_2B = dict(H=12, dk=96, dv=256, D=1536)
_4B = dict(H=16, dk=128, dv=256, D=2048)

CONFIGS = {
    # tiny float32 case, small enough for every oracle check
    "tiny_f32": JetShape("tiny_f32", B=1, T=64, H=2, dk=16, dv=32, D=64, dtype="f32"),
    # 2B-shape prefill, 4096 tokens
    "prefill_2b_t4096": JetShape("prefill_2b_t4096", B=1, T=4096, **_2B),
    # 2B-shape decode, 256 sequences, 64 successive steps
    "decode_2b_b256": JetShape("decode_2b_b256", B=256, T=0, steps=64, **_2B),
    # 4B-shape long prefill, 65536 tokens
    "prefill_4b_t65536": JetShape("prefill_4b_t65536", B=1, T=65536, **_4B),
    # 2B-shape long-context pipeline: 262144-token prefill, then 256 decode steps
    "prefill_2b_t262144": JetShape("prefill_2b_t262144", B=1, T=262144, steps=256, **_2B),
}
for _b in (1, 16, 64, 256, 1024):
    CONFIGS[f"decode_4b_b{_b}"] = JetShape(f"decode_4b_b{_b}", B=_b, T=0, steps=64, **_4B)


# --------------------------------------------------------------------------
# storage-dtype rounding (input preparation, not mixer arithmetic)
# --------------------------------------------------------------------------
def bf16_bits_from_f64(a: np.ndarray) -> np.ndarray:
    """float64 -> float32 (RNE) -> bf16 bit pattern (RNE on the low 16 bits)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return u.astype(np.uint16)


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def to_f64(a: np.ndarray, dtype: str) -> np.ndarray:
    """Exact float64 value of a stored array (bf16 bits or float32)."""
    if dtype == "bf16" and a.dtype == np.uint16:
        return bf16_bits_to_f64(a)
    return np.asarray(a, dtype=np.float64)


def _store(a64: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_from_f64(a64) if dtype == "bf16" else a64.astype(np.float32)


def _out_dtype(dtype: str):
    return np.uint16 if dtype == "bf16" else np.float32


_BLOCK_ELEMS = 1 << 24   # draw big arrays in blocks of about 16M values


def _draw(rng, shape, dtype: str, scale: float = 1.0, unit_last: bool = False):
    """N(0, scale^2) draws of `shape`, stored in `dtype`; drawn block by block
    along the flattened leading axes (the stream equals one full draw)."""
    shape = tuple(int(s) for s in shape)
    last = shape[-1]
    rows = int(np.prod(shape[:-1])) if len(shape) > 1 else 1
    out = np.empty((rows, last), dtype=_out_dtype(dtype))
    step = max(1, _BLOCK_ELEMS // max(1, last))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        a = rng.standard_normal((r1 - r0, last))
        if unit_last:
            a /= np.sqrt(np.sum(a * a, axis=-1, keepdims=True))
        if scale != 1.0:
            a *= scale
        out[r0:r1] = _store(a, dtype)
    return out.reshape(shape)


def spread_qk_norms(a: np.ndarray, dtype: str, seed: int, zero_rows=()) -> np.ndarray:
    """Rescale every row (last axis) of a stored q or k array by 10**U(-1, 1),
    drawn from a generator of its own (PCG64 seeded with [seed, 7]), so the
    main input stream is unchanged; then set the rows at the index tuples
    `zero_rows` (over the leading axes) to exactly zero. Returns a new array
    in the same storage dtype. These inputs exercise the in-kernel L2
    normalisation, including the eps under the square root."""
    rng = np.random.Generator(np.random.PCG64([seed, 7]))
    lead = a.shape[:-1]
    s = 10.0 ** rng.uniform(-1.0, 1.0, size=lead + (1,))
    b = to_f64(a, dtype) * s
    for idx in zero_rows:
        b[tuple(idx)] = 0.0
    return _store(b, dtype)


def _gates(rng, shape, gate_scale: float):
    beta_raw = rng.standard_normal(shape)
    g_raw = rng.standard_normal(shape)
    beta = (1.0 / (1.0 + np.exp(-beta_raw))).astype(np.float32)
    g = (-gate_scale * np.logaddexp(0.0, g_raw)).astype(np.float32)
    return beta, g


def prefill_inputs(shape: JetShape, seed: int = 0, T: int | None = None,
                   gate_scale: float = 1.0, s0_std: float | None = None) -> dict:
    """Inputs of a prefill over `T` (default shape.T) tokens per sequence.

    Returns x [B,T,D], q/k [B,T,H,dk], v [B,T,H,dv] in the bulk dtype; beta, g
    [B,T,H] float32; W1 [D,32], W2 [32,H*4] in the bulk dtype; and, when
    s0_std is given, an initial state S0 [B,H,dv,dk] float32 drawn last.
    """
    T = shape.T if T is None else T
    B, H, dk, dv, D, dt = shape.B, shape.H, shape.dk, shape.dv, shape.D, shape.dtype
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    out["x"] = _draw(rng, (B, T, D), dt)
    out["q"] = _draw(rng, (B, T, H, dk), dt, unit_last=True)
    out["k"] = _draw(rng, (B, T, H, dk), dt, unit_last=True)
    out["v"] = _draw(rng, (B, T, H, dv), dt)
    out["beta"], out["g"] = _gates(rng, (B, T, H), gate_scale)
    out["W1"] = _draw(rng, (D, shape.R), dt, scale=1.0 / np.sqrt(D))
    out["W2"] = _draw(rng, (shape.R, H * shape.W), dt, scale=1.0 / np.sqrt(shape.R))
    if s0_std is not None:
        out["S0"] = _draw(rng, (B, H, dv, dk), "f32", scale=s0_std)
    out["dtype"] = dt
    return out


def decode_inputs(shape: JetShape, seed: int = 0, steps: int | None = None,
                  state_std: float = 0.02, gate_scale: float = 1.0) -> dict:
    """Inputs of `steps` decode steps for B sequences (one token each per step).

    Token tensors carry a leading step axis: x [n,B,D], q/k [n,B,H,dk],
    v [n,B,H,dv], beta/g [n,B,H]. Then W1, W2, the incoming state
    S0 [B,H,dv,dk] float32 and the conv history hist [B,3,H,dv] (oldest first).
    """
    n = shape.steps if steps is None else steps
    B, H, dk, dv, D, dt = shape.B, shape.H, shape.dk, shape.dv, shape.D, shape.dtype
    rng = np.random.Generator(np.random.PCG64(seed))
    out = {}
    out["x"] = _draw(rng, (n, B, D), dt)
    out["q"] = _draw(rng, (n, B, H, dk), dt, unit_last=True)
    out["k"] = _draw(rng, (n, B, H, dk), dt, unit_last=True)
    out["v"] = _draw(rng, (n, B, H, dv), dt)
    out["beta"], out["g"] = _gates(rng, (n, B, H), gate_scale)
    out["W1"] = _draw(rng, (D, shape.R), dt, scale=1.0 / np.sqrt(D))
    out["W2"] = _draw(rng, (shape.R, H * shape.W), dt, scale=1.0 / np.sqrt(shape.R))
    out["S0"] = _draw(rng, (B, H, dv, dk), "f32", scale=state_std)
    out["hist"] = _draw(rng, (B, shape.W - 1, H, dv), dt)
    out["dtype"] = dt
    return out


# --------------------------------------------------------------------------
# block-seeded variant (benchmark inputs of the long configurations)
# --------------------------------------------------------------------------
def _pool_map(fn, n: int, threads: int | None):
    import os
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or max(1, min(32, len(os.sched_getaffinity(0))))
    with ThreadPoolExecutor(threads) as ex:
        list(ex.map(fn, range(n)))


def prefill_inputs_blocked(shape: JetShape, seed: int = 0, T: int | None = None, block: int = 4096,
                           threads: int | None = None, gate_scale: float = 1.0) -> dict:
    """The prefill recipe of prefill_inputs (same arrays, layouts and
    distributions), with the token axis drawn in blocks of `block` tokens:
    block i of every token tensor comes from PCG64([seed, 1, i]), in the order
    x, q, k, v, beta_raw, g_raw; the weights come from PCG64([seed, 2]).
    Blocks are drawn in parallel threads (numpy releases the GIL while it
    draws), so multi-GB inputs take seconds. A different stream from
    prefill_inputs: the two are not interchangeable for stored values."""
    T = shape.T if T is None else T
    B, H, dk, dv, D, dt = shape.B, shape.H, shape.dk, shape.dv, shape.D, shape.dtype
    od = _out_dtype(dt)
    out = {"x": np.empty((B, T, D), od), "q": np.empty((B, T, H, dk), od), "k": np.empty((B, T, H, dk), od),
           "v": np.empty((B, T, H, dv), od), "beta": np.empty((B, T, H), np.float32),
           "g": np.empty((B, T, H), np.float32)}
    nblk = (T + block - 1) // block

    def one(j):
        b, i = divmod(j, nblk)
        t0, t1 = i * block, min(T, (i + 1) * block)
        rng = np.random.Generator(np.random.PCG64([seed, 1, b, i]))
        n = t1 - t0
        out["x"][b, t0:t1] = _draw(rng, (n, D), dt)
        out["q"][b, t0:t1] = _draw(rng, (n, H, dk), dt, unit_last=True)
        out["k"][b, t0:t1] = _draw(rng, (n, H, dk), dt, unit_last=True)
        out["v"][b, t0:t1] = _draw(rng, (n, H, dv), dt)
        out["beta"][b, t0:t1], out["g"][b, t0:t1] = _gates(rng, (n, H), gate_scale)

    _pool_map(one, B * nblk, threads)
    rng = np.random.Generator(np.random.PCG64([seed, 2]))
    out["W1"] = _draw(rng, (D, shape.R), dt, scale=1.0 / np.sqrt(D))
    out["W2"] = _draw(rng, (shape.R, H * shape.W), dt, scale=1.0 / np.sqrt(shape.R))
    out["dtype"] = dt
    return out


def decode_inputs_blocked(shape: JetShape, seed: int = 0, steps: int | None = None, state_std: float = 0.02,
                          block: int = 16, threads: int | None = None, gate_scale: float = 1.0) -> dict:
    """The decode recipe of decode_inputs (same arrays and distributions),
    drawn in parallel: the token tensors of step s from PCG64([seed, 3, s]);
    the state and history of sequences [i*block, (i+1)*block) from
    PCG64([seed, 4, i]); the weights from PCG64([seed, 2])."""
    n = shape.steps if steps is None else steps
    B, H, dk, dv, D, dt = shape.B, shape.H, shape.dk, shape.dv, shape.D, shape.dtype
    od = _out_dtype(dt)
    out = {"x": np.empty((n, B, D), od), "q": np.empty((n, B, H, dk), od), "k": np.empty((n, B, H, dk), od),
           "v": np.empty((n, B, H, dv), od), "beta": np.empty((n, B, H), np.float32),
           "g": np.empty((n, B, H), np.float32), "S0": np.empty((B, H, dv, dk), np.float32),
           "hist": np.empty((B, shape.W - 1, H, dv), od)}

    def tok(s):
        rng = np.random.Generator(np.random.PCG64([seed, 3, s]))
        out["x"][s] = _draw(rng, (B, D), dt)
        out["q"][s] = _draw(rng, (B, H, dk), dt, unit_last=True)
        out["k"][s] = _draw(rng, (B, H, dk), dt, unit_last=True)
        out["v"][s] = _draw(rng, (B, H, dv), dt)
        out["beta"][s], out["g"][s] = _gates(rng, (B, H), gate_scale)

    nsb = (B + block - 1) // block

    def st(i):
        b0, b1 = i * block, min(B, (i + 1) * block)
        rng = np.random.Generator(np.random.PCG64([seed, 4, i]))
        out["S0"][b0:b1] = _draw(rng, (b1 - b0, H, dv, dk), "f32", scale=state_std)
        out["hist"][b0:b1] = _draw(rng, (b1 - b0, shape.W - 1, H, dv), dt)

    _pool_map(tok, n, threads)
    _pool_map(st, nsb, threads)
    rng = np.random.Generator(np.random.PCG64([seed, 2]))
    out["W1"] = _draw(rng, (D, shape.R), dt, scale=1.0 / np.sqrt(D))
    out["W2"] = _draw(rng, (shape.R, H * shape.W), dt, scale=1.0 / np.sqrt(shape.R))
    out["dtype"] = dt
    return out
