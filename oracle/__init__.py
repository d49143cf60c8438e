"""Float64 CPU oracle of the JetBlock token mixer.

TEST INFRASTRUCTURE ONLY: imported by the tests, by the smoke check and by the
CPU-baseline leg of the benchmark. The CUDA library never imports, links or
calls anything here, and nothing here imports the CUDA library.

The arithmetic lives in ``jet_oracle.c`` (plain loops, float64, OpenMP over
independent items only); this module compiles it with gcc, loads it with
ctypes and composes the stages of the mixer:

  generator  w_t = SiLU(x_t W1) W2                 (paper section 2.4)
  conv       v'_t = sum_j w_t[h, j] v_{t-j}          (paper section 2.4)
  GDN        S_t = a_t (S_{t-1} - b_t (S_{t-1} k_t) k_t^T) + b_t v'_t k_t^T,
             o_t = S_t q_t on L2-normalised q, k     (paper section 2.3)

Every function takes float64 arrays (upcast by the caller from the stored
bf16 / float32 values) and returns float64 arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "jet_oracle.c")
LIB = os.path.join(HERE, "liboracle.so")
L2_EPS = 1e-6
_lock = threading.Lock()


def build(src: str = SRC, out: str = LIB, force: bool = False) -> str:
    """Compile the oracle into a shared library (gcc, float64, OpenMP)."""
    if force or not os.path.exists(out) or os.path.getmtime(out) < os.path.getmtime(src):
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", out, src, "-lm"]
        subprocess.run(cmd, check=True)
    return out


_D = ctypes.POINTER(ctypes.c_double)


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(_D)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


class Oracle:
    """ctypes front end of one compiled oracle library."""

    def __init__(self, lib_path: str | None = None):
        path = lib_path or build()
        self.lib = ctypes.CDLL(path)
        L, i, l, d = self.lib, ctypes.c_int, ctypes.c_long, ctypes.c_double
        L.oracle_num_threads.restype = i
        L.oracle_kernel_gen.argtypes = [_D, _D, _D, _D, l, i, i, i]
        L.oracle_dyn_conv.argtypes = [_D, _D, _D, _D, _D, i, l, i, i, i]
        L.oracle_gdn_sequential.argtypes = [_D] * 8 + [i, l, i, i, i, d]
        L.oracle_gdn_decode_step.argtypes = [_D] * 7 + [i, i, i, i, d]
        L.oracle_gdn_chunked.argtypes = [_D] * 8 + [i, l, i, i, i, i, d]
        for f in ("oracle_kernel_gen", "oracle_dyn_conv", "oracle_gdn_sequential",
                  "oracle_gdn_decode_step", "oracle_gdn_chunked"):
            getattr(L, f).restype = None

    def num_threads(self) -> int:
        return int(self.lib.oracle_num_threads())

    # ---- stages -----------------------------------------------------------
    def kernel_gen(self, x, W1, W2, H: int, W: int = 4):
        """x [..., D] -> conv taps w [..., H, W]."""
        x, W1, W2 = _f64(x), _f64(W1), _f64(W2)
        D, R = W1.shape
        lead = x.shape[:-1]
        N = int(np.prod(lead)) if lead else 1
        assert W2.shape == (R, H * W) and x.shape[-1] == D
        w = np.empty(lead + (H, W), dtype=np.float64)
        self.lib.oracle_kernel_gen(_p(x), _p(W1), _p(W2), _p(w), N, D, R, H * W)
        return w

    def dyn_conv(self, v, w, hist=None):
        """v [B,T,H,dv], w [B,T,H,W], hist [B,W-1,H,dv] or None ->
        (v' [B,T,H,dv], hist_out [B,W-1,H,dv])."""
        v, w, hist = _f64(v), _f64(w), _f64(hist)
        B, T, H, dv = v.shape
        W = w.shape[-1]
        out = np.empty_like(v)
        hist_out = np.empty((B, W - 1, H, dv), dtype=np.float64)
        self.lib.oracle_dyn_conv(_p(v), _p(w), _p(hist), _p(out), _p(hist_out), B, T, H, dv, W)
        return out, hist_out

    def gdn_sequential(self, q, k, v, g, beta, S0=None):
        """Token-by-token Gated DeltaNet. Returns (o [B,T,H,dv], S [B,H,dv,dk])."""
        q, k, v, g, beta, S0 = map(_f64, (q, k, v, g, beta, S0))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        o = np.empty((B, T, H, dv), dtype=np.float64)
        S = np.empty((B, H, dv, dk), dtype=np.float64)
        self.lib.oracle_gdn_sequential(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(S0), _p(o), _p(S),
                                       B, T, H, dk, dv, L2_EPS)
        return o, S

    def gdn_chunked(self, q, k, v, g, beta, S0=None, C: int = 64):
        """Chunked (WY / UT) form of the same recurrence; identity check only."""
        q, k, v, g, beta, S0 = map(_f64, (q, k, v, g, beta, S0))
        B, T, H, dk = q.shape
        dv = v.shape[-1]
        o = np.empty((B, T, H, dv), dtype=np.float64)
        S = np.empty((B, H, dv, dk), dtype=np.float64)
        self.lib.oracle_gdn_chunked(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(S0), _p(o), _p(S),
                                    B, T, H, dk, dv, C, L2_EPS)
        return o, S

    def gdn_decode_step(self, q, k, v, g, beta, S):
        """One token per sequence: q,k [B,H,dk], v [B,H,dv], g,beta [B,H],
        S [B,H,dv,dk]. Returns (o [B,H,dv], S_new)."""
        q, k, v, g, beta = map(_f64, (q, k, v, g, beta))
        S = np.array(S, dtype=np.float64, copy=True, order="C")
        B, H, dk = q.shape
        dv = v.shape[-1]
        o = np.empty((B, H, dv), dtype=np.float64)
        self.lib.oracle_gdn_decode_step(_p(q), _p(k), _p(v), _p(g), _p(beta), _p(S), _p(o),
                                        B, H, dk, dv, L2_EPS)
        return o, S

    # ---- the whole mixer ----------------------------------------------------
    def jetblock_prefill(self, x, W1, W2, q, k, v, g, beta, S0=None, hist=None,
                         W: int = 4, chunked: bool = False):
        """Generator -> conv on V -> GDN, no intermediate rounding.
        Returns dict(w, v_conv, o, S, hist)."""
        H = q.shape[2]
        w = self.kernel_gen(x, W1, W2, H, W)
        vc, hist_out = self.dyn_conv(v, w, hist)
        if chunked:
            o, S = self.gdn_chunked(q, k, vc, g, beta, S0)
        else:
            o, S = self.gdn_sequential(q, k, vc, g, beta, S0)
        return dict(w=w, v_conv=vc, o=o, S=S, hist=hist_out)

    def jetblock_decode(self, x, W1, W2, q, k, v, g, beta, S0, hist, W: int = 4):
        """Decode steps with a leading step axis (x [n,B,D], ...). Each step runs
        generator -> conv with history -> single-token GDN update.
        Returns dict(o [n,B,H,dv], v_conv [n,B,H,dv], S, hist)."""
        n, B = x.shape[0], x.shape[1]
        H = q.shape[2]
        S = np.array(S0, dtype=np.float64, copy=True)
        h = np.array(hist, dtype=np.float64, copy=True)
        os_, vcs = [], []
        for s in range(n):
            w = self.kernel_gen(x[s][:, None, :], W1, W2, H, W)          # [B,1,H,W]
            vc, h = self.dyn_conv(np.asarray(v[s])[:, None], w, h)       # [B,1,H,dv]
            o, S = self.gdn_decode_step(q[s], k[s], vc[:, 0], g[s], beta[s], S)
            os_.append(o)
            vcs.append(vc[:, 0])
        return dict(o=np.stack(os_), v_conv=np.stack(vcs), S=S, hist=h)


_default = None


def get() -> Oracle:
    """The oracle built from this directory's source (compiled on first use)."""
    global _default
    with _lock:
        if _default is None:
            _default = Oracle()
    return _default
