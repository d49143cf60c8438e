"""JetBlock token mixer on B200: Python binding of the C ABI in include/jet.h.

Argument marshalling only: every step of the mixer runs in the CUDA kernels
of ``libjet.so`` (built in-tree by ``build.py``). torch supplies device memory
and the current stream. There is no CPU path: if the library is missing or
no CUDA device is present, the calls raise.

Function names match the C entry points:
  jet_kernel_gen, jet_dyn_conv_v, jet_gdn_prefill_workspace_size,
  jet_gdn_prefill_workspace_min, jet_gdn_prefill, jet_gdn_prefill_noalloc, jet_gdn_decode_step,
  jet_jetblock_decode_step, jet_conv_gdn_decode_step, jet_jetblock_prefill_workspace_size,
  jet_jetblock_prefill, jet_jetblock_decode_slots, jet_jetblock_prefill_varlen_workspace_size,
  jet_jetblock_prefill_varlen, jet_jetblock_prefill_range_workspace_size,
  jet_jetblock_prefill_range, jet_gdn_range_compose, jet_gdn_range_correct,
  jet_device_error, jet_status_string, jet_launch_count.
"""
from __future__ import annotations

import ctypes
import os

import torch

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libjet.so")

JET_F32, JET_BF16 = 0, 1
STATUS = {0: "JET_OK", 1: "JET_ERR_INVALID_ARG", 2: "JET_ERR_UNSUPPORTED", 3: "JET_ERR_MISALIGNED",
          4: "JET_ERR_CUDA", 5: "JET_ERR_TIMEOUT", 6: "JET_ERR_DEVICE", 7: "JET_ERR_WORKSPACE",
          8: "JET_ERR_TOO_LARGE", 9: "JET_ERR_LIBRARY"}
EXPORTS = ("jet_kernel_gen", "jet_dyn_conv_v", "jet_gdn_prefill_workspace_size", "jet_gdn_prefill_workspace_min",
           "jet_gdn_prefill",
           "jet_gdn_prefill_noalloc", "jet_gdn_decode_step", "jet_jetblock_decode_step", "jet_conv_gdn_decode_step",
           "jet_jetblock_prefill_workspace_size", "jet_jetblock_prefill", "jet_jetblock_decode_slots",
           "jet_jetblock_prefill_varlen_workspace_size", "jet_jetblock_prefill_varlen",
           "jet_jetblock_prefill_range_workspace_size", "jet_jetblock_prefill_range", "jet_gdn_range_compose",
           "jet_gdn_range_correct", "jet_jetblock_layer_workspace_size", "jet_jetblock_layer", "jet_device_error",
           "jet_status_string", "jet_launch_count")
NOALLOC_SCRATCH_BYTES = 16 << 20


class JetError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libjet.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"libjet.so not built at {path}: run linear_attention_lm_gen_b200/build.py")
    _lib = declare(ctypes.CDLL(path))
    return _lib


def declare(L: ctypes.CDLL) -> ctypes.CDLL:
    """Set the argument and result types of the C entry points on a loaded library."""
    P, I, Z, U = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_uint64
    L.jet_kernel_gen.argtypes = [P, P, P, P, I, I, I, I, I, I, I, P]
    L.jet_dyn_conv_v.argtypes = [P] * 8 + [I] * 8 + [P]
    L.jet_gdn_prefill_workspace_size.argtypes = [I] * 7
    L.jet_gdn_prefill_workspace_size.restype = Z
    L.jet_gdn_prefill_workspace_min.argtypes = [I] * 7
    L.jet_gdn_prefill_workspace_min.restype = Z
    L.jet_gdn_prefill.argtypes = [P] * 9 + [Z] + [I] * 7 + [P]
    L.jet_gdn_prefill_noalloc.argtypes = [P] * 8 + [I] * 7 + [P]
    L.jet_gdn_decode_step.argtypes = [P] * 7 + [I] * 5 + [P]
    L.jet_jetblock_decode_step.argtypes = [P] * 13 + [I] * 8 + [P]
    L.jet_conv_gdn_decode_step.argtypes = [P] * 10 + [I] * 5 + [P]
    L.jet_jetblock_prefill_workspace_size.argtypes = [I] * 7
    L.jet_jetblock_prefill_workspace_size.restype = Z
    L.jet_jetblock_prefill.argtypes = [P] * 14 + [Z] + [I] * 10 + [P]
    L.jet_jetblock_decode_slots.argtypes = [P] * 11 + [I] + [P] * 3 + [I] * 8 + [P]
    L.jet_jetblock_prefill_varlen_workspace_size.argtypes = [P, I, I, I, I, I, I]
    L.jet_jetblock_prefill_varlen_workspace_size.restype = Z
    L.jet_jetblock_prefill_varlen.argtypes = [P] * 14 + [Z] + [P] + [I] * 9 + [P]
    L.jet_jetblock_prefill_range_workspace_size.argtypes = [I] * 7
    L.jet_jetblock_prefill_range_workspace_size.restype = Z
    L.jet_jetblock_prefill_range.argtypes = [P] * 16 + [Z] + [I] * 10 + [P]
    L.jet_gdn_range_compose.argtypes = [P] * 4 + [I] * 5 + [P]
    L.jet_gdn_range_correct.argtypes = [P] * 3 + [I] * 6 + [P]
    L.jet_jetblock_layer_workspace_size.argtypes = [I] * 6
    L.jet_jetblock_layer_workspace_size.restype = Z
    L.jet_jetblock_layer.argtypes = [P] * 17 + [Z] + [I] * 9 + [P]
    L.jet_device_error.argtypes = [P]
    L.jet_status_string.argtypes = [I]
    L.jet_status_string.restype = ctypes.c_char_p
    L.jet_launch_count.argtypes = []
    L.jet_launch_count.restype = U
    for f in ("jet_kernel_gen", "jet_dyn_conv_v", "jet_gdn_prefill", "jet_gdn_prefill_noalloc",
              "jet_gdn_decode_step", "jet_jetblock_decode_step", "jet_conv_gdn_decode_step", "jet_jetblock_prefill",
              "jet_jetblock_decode_slots", "jet_jetblock_prefill_varlen", "jet_jetblock_prefill_range",
              "jet_gdn_range_compose",
              "jet_gdn_range_correct", "jet_jetblock_layer", "jet_device_error"):
        getattr(L, f).restype = I
    return L


# ---------------------------------------------------------------- marshalling
def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return JET_BF16
    if t.dtype == torch.float32:
        return JET_F32
    raise TypeError(f"unsupported dtype {t.dtype} (bf16 or float32)")


def _ptr(t, name, dtype=None, shape=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _check(fn, st):
    if st != 0:
        raise JetError(fn, st)


# ---------------------------------------------------------------- entry points
def jet_kernel_gen(x, W1, W2, H: int, conv_w=None, *, stream=None):
    """x [B,T,D], W1 [D,32], W2 [32,H*4] -> conv taps [B,T,H,4] float32."""
    L = load_library()
    B, T, D = x.shape
    dt = _dt(x)
    if conv_w is None:
        conv_w = torch.empty((B, T, H, 4), device=x.device, dtype=torch.float32)
    st = L.jet_kernel_gen(_ptr(x, "x"), _ptr(W1, "W1", x.dtype, (D, 32)), _ptr(W2, "W2", x.dtype, (32, H * 4)),
                          _ptr(conv_w, "conv_w", torch.float32, (B, T, H, 4)), B, T, D, H, 32, 4, dt, _stream(stream))
    _check("jet_kernel_gen", st)
    return conv_w


def jet_dyn_conv_v(x, W1, W2, v, hist_in=None, v_out=None, hist_out=None, conv_w_out=None, *, stream=None):
    """Generator + dynamic causal conv on V. v [B,T,H,dv] -> v' (same shape).
    Returns (v_out, hist_out); hist_out is None unless a buffer is given."""
    L = load_library()
    B, T, D = x.shape
    _, _, H, dv = v.shape
    dt = _dt(x)
    if v_out is None:
        v_out = torch.empty_like(v)
    st = L.jet_dyn_conv_v(_ptr(x, "x"), _ptr(W1, "W1", x.dtype, (D, 32)), _ptr(W2, "W2", x.dtype, (32, H * 4)),
                          _ptr(v, "v", x.dtype, (B, T, H, dv)),
                          _ptr(hist_in, "hist_in", x.dtype, (B, 3, H, dv)), _ptr(v_out, "v_out", x.dtype, (B, T, H, dv)),
                          _ptr(hist_out, "hist_out", x.dtype, (B, 3, H, dv)),
                          _ptr(conv_w_out, "conv_w_out", torch.float32, (B, T, H, 4)),
                          B, T, D, H, dv, 32, 4, dt, _stream(stream))
    _check("jet_dyn_conv_v", st)
    return v_out, hist_out


def jet_gdn_prefill_workspace_size(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Workspace bytes of the fastest prefill plan (chunk images + segment buffers)."""
    L = load_library()
    return int(L.jet_gdn_prefill_workspace_size(B, T, H, dk, dv, chunk,
                                                JET_BF16 if dtype == torch.bfloat16 else JET_F32))


def jet_gdn_prefill_workspace_min(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Smallest workspace jet_gdn_prefill accepts (segment buffers only)."""
    L = load_library()
    return int(L.jet_gdn_prefill_workspace_min(B, T, H, dk, dv, chunk,
                                               JET_BF16 if dtype == torch.bfloat16 else JET_F32))


def jet_gdn_prefill(q, k, v, g, beta, S0=None, o=None, S_out=None, workspace=None, *, stream=None):
    """Chunked Gated DeltaNet prefill. q,k [B,T,H,dk], v [B,T,H,dv], g,beta [B,T,H]
    float32, S0 [B,H,dv,dk] float32 or None. Returns (o, S_out)."""
    L = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, T, H, dv), device=q.device, dtype=q.dtype)
    if S_out is None:
        S_out = torch.empty((B, H, dv, dk), device=q.device, dtype=torch.float32)
    need = jet_gdn_prefill_workspace_size(B, T, H, dk, dv, 64, q.dtype)
    if workspace is None and need > 0:
        workspace = torch.empty(need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    st = L.jet_gdn_prefill(_ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, T, H, dv)),
                           _ptr(g, "g", torch.float32, (B, T, H)), _ptr(beta, "beta", torch.float32, (B, T, H)),
                           _ptr(S0, "S0", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, T, H, dv)),
                           _ptr(S_out, "S_out", torch.float32, (B, H, dv, dk)), _ptr(workspace, "workspace"),
                           ws_bytes, B, T, H, dk, dv, 64, dt, _stream(stream))
    _check("jet_gdn_prefill", st)
    return o, S_out


def jet_gdn_prefill_noalloc(q, k, v, g, beta, S0, o, S_out, *, stream=None):
    """jet_gdn_prefill without a workspace argument, for callers that cannot
    allocate: the library uses its own fixed scratch array (16 MiB per GPU).
    o and S_out must be given (nothing is allocated here either). Calls whose
    work overlaps on the GPU share that array and must be ordered by the caller."""
    L = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    st = L.jet_gdn_prefill_noalloc(_ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, T, H, dv)),
                                   _ptr(g, "g", torch.float32, (B, T, H)), _ptr(beta, "beta", torch.float32, (B, T, H)),
                                   _ptr(S0, "S0", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, T, H, dv)),
                                   _ptr(S_out, "S_out", torch.float32, (B, H, dv, dk)),
                                   B, T, H, dk, dv, 64, _dt(q), _stream(stream))
    _check("jet_gdn_prefill_noalloc", st)
    return o, S_out


def jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Workspace bytes of jet_jetblock_prefill (taps + the prefill's fastest plan)."""
    L = load_library()
    return int(L.jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, chunk,
                                                     JET_BF16 if dtype == torch.bfloat16 else JET_F32))


def jet_jetblock_prefill(x, W1, W2, q, k, v, g, beta, hist_in=None, hist_out=None, S0=None, o=None, S_out=None,
                         workspace=None, *, stream=None):
    """Generator + dynamic conv + chunked Gated DeltaNet over a prompt. x [B,T,D],
    q,k [B,T,H,dk], v [B,T,H,dv] raw, g,beta [B,T,H] float32, hist_in / hist_out
    [B,3,H,dv] or None, S0 [B,H,dv,dk] float32 or None. Returns (o, S_out)."""
    L = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    D = x.shape[-1]
    hidden, HW = W2.shape
    width = HW // H
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, T, H, dv), device=q.device, dtype=q.dtype)
    if S_out is None:
        S_out = torch.empty((B, H, dv, dk), device=q.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(max(1, jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, 64, q.dtype)),
                                device=q.device, dtype=torch.uint8)
    ws_bytes = workspace.numel() * workspace.element_size()
    st = L.jet_jetblock_prefill(
        _ptr(x, "x", q.dtype, (B, T, D)), _ptr(W1, "W1", q.dtype, (D, hidden)), _ptr(W2, "W2", q.dtype, (hidden, HW)),
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, T, H, dv)),
        _ptr(hist_in, "hist_in", q.dtype, (B, 3, H, dv)), _ptr(hist_out, "hist_out", q.dtype, (B, 3, H, dv)),
        _ptr(g, "g", torch.float32, (B, T, H)), _ptr(beta, "beta", torch.float32, (B, T, H)),
        _ptr(S0, "S0", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, T, H, dv)),
        _ptr(S_out, "S_out", torch.float32, (B, H, dv, dk)), _ptr(workspace, "workspace"), ws_bytes,
        B, T, D, H, dk, dv, hidden, width, 64, dt, _stream(stream))
    _check("jet_jetblock_prefill", st)
    return o, S_out


def _cu(cu_seqlens):
    """Sequence offsets as a host int32 array (a list, tuple or CPU tensor)."""
    import numpy as np
    if isinstance(cu_seqlens, torch.Tensor):
        if cu_seqlens.is_cuda:
            raise TypeError("cu_seqlens must be on the host: the launch plan is made from it")
        cu_seqlens = cu_seqlens.tolist()
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))


def jet_jetblock_prefill_varlen_workspace_size(cu_seqlens, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Workspace bytes of jet_jetblock_prefill_varlen for these sequence offsets."""
    L = load_library()
    cu = _cu(cu_seqlens)
    return int(L.jet_jetblock_prefill_varlen_workspace_size(cu.ctypes.data_as(ctypes.c_void_p), len(cu) - 1, H, dk,
                                                            dv, chunk, JET_BF16 if dtype == torch.bfloat16 else JET_F32))


def jet_jetblock_prefill_varlen(x, W1, W2, q, k, v, g, beta, cu_seqlens, hist_in=None, hist_out=None, S0=None, o=None,
                                S_out=None, workspace=None, *, stream=None):
    """The mixer over several prompts of different lengths in one call, packed
    along the token axis: x [total,D], q,k [total,H,dk], v [total,H,dv] raw,
    g,beta [total,H] float32; cu_seqlens (host) the nseq + 1 offsets;
    hist_in / hist_out [nseq,3,H,dv], S0 [nseq,H,dv,dk] or None. Returns
    (o [total,H,dv], S_out [nseq,H,dv,dk])."""
    L = load_library()
    cu = _cu(cu_seqlens)
    nseq = len(cu) - 1
    total, H, dk = q.shape
    dv = v.shape[-1]
    D = x.shape[-1]
    hidden, HW = W2.shape
    width = HW // H
    if o is None:
        o = torch.empty((total, H, dv), device=q.device, dtype=q.dtype)
    if S_out is None:
        S_out = torch.empty((nseq, H, dv, dk), device=q.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(max(16, jet_jetblock_prefill_varlen_workspace_size(cu, H, dk, dv, 64, q.dtype)),
                                device=q.device, dtype=torch.uint8)
    st = L.jet_jetblock_prefill_varlen(
        _ptr(x, "x", q.dtype, (total, D)), _ptr(W1, "W1", q.dtype, (D, hidden)), _ptr(W2, "W2", q.dtype, (hidden, HW)),
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (total, H, dv)),
        _ptr(hist_in, "hist_in", q.dtype, (nseq, 3, H, dv)), _ptr(hist_out, "hist_out", q.dtype, (nseq, 3, H, dv)),
        _ptr(g, "g", torch.float32, (total, H)), _ptr(beta, "beta", torch.float32, (total, H)),
        _ptr(S0, "S0", torch.float32, (nseq, H, dv, dk)), _ptr(o, "o", q.dtype, (total, H, dv)),
        _ptr(S_out, "S_out", torch.float32, (nseq, H, dv, dk)), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), cu.ctypes.data_as(ctypes.c_void_p), nseq, D, H, dk, dv, hidden,
        width, 64, _dt(q), _stream(stream))
    _check("jet_jetblock_prefill_varlen", st)
    return o, S_out


def jet_jetblock_prefill_range_workspace_size(B, T, H, dk, dv, chunk=64, dtype=torch.bfloat16) -> int:
    """Workspace bytes of jet_jetblock_prefill_range (taps + chunk images)."""
    L = load_library()
    return int(L.jet_jetblock_prefill_range_workspace_size(B, T, H, dk, dv, chunk,
                                                           JET_BF16 if dtype == torch.bfloat16 else JET_F32))


def jet_jetblock_prefill_range(x, W1, W2, q, k, v, g, beta, hist_in=None, hist_out=None, S0=None, first=False,
                               o=None, E_out=None, A_out=None, Qe_out=None, workspace=None, *, stream=None):
    """The mixer over one token range of a sequence split across GPUs.
    first=True: the range starts at S0 (or zero) for real and gets no
    transition; otherwise it runs from a zero start and also returns its
    transition A [B,H,dk,dk] and output-correction operand Qe. Returns
    (o, E, A, Qe); A and Qe are None for a first range."""
    L = load_library()
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    D = x.shape[-1]
    hidden, HW = W2.shape
    width = HW // H
    dev = q.device
    if o is None:
        o = torch.empty((B, T, H, dv), device=dev, dtype=q.dtype)
    if E_out is None:
        E_out = torch.empty((B, H, dv, dk), device=dev, dtype=torch.float32)
    if not first:
        if A_out is None:
            A_out = torch.empty((B, H, dk, dk), device=dev, dtype=torch.float32)
        if Qe_out is None:
            Qe_out = torch.empty((B, H, (T + 63) // 64, 64, dk), device=dev, dtype=q.dtype)
    if workspace is None:
        workspace = torch.empty(max(16, jet_jetblock_prefill_range_workspace_size(B, T, H, dk, dv, 64, q.dtype)),
                                device=dev, dtype=torch.uint8)
    st = L.jet_jetblock_prefill_range(
        _ptr(x, "x", q.dtype, (B, T, D)), _ptr(W1, "W1", q.dtype, (D, hidden)), _ptr(W2, "W2", q.dtype, (hidden, HW)),
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, T, H, dv)),
        _ptr(hist_in, "hist_in", q.dtype, (B, 3, H, dv)), _ptr(hist_out, "hist_out", q.dtype, (B, 3, H, dv)),
        _ptr(g, "g", torch.float32, (B, T, H)), _ptr(beta, "beta", torch.float32, (B, T, H)),
        _ptr(S0, "S0", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, T, H, dv)),
        _ptr(E_out, "E_out", torch.float32, (B, H, dv, dk)),
        _ptr(A_out, "A_out", torch.float32, (B, H, dk, dk)),
        _ptr(Qe_out, "Qe_out", q.dtype, (B, H, (T + 63) // 64, 64, dk)),
        _ptr(workspace, "workspace"), workspace.numel() * workspace.element_size(),
        B, T, D, H, dk, dv, hidden, width, 64, _dt(q), _stream(stream))
    _check("jet_jetblock_prefill_range", st)
    return o, E_out, A_out, Qe_out


def jet_gdn_range_compose(E, A, Sb=None, S_out=None, *, stream=None):
    """Start states of R ranges from their (E, A) pairs: E [R,B,H,dv,dk] and
    A [R,B,H,dk,dk] float32. Returns (Sb [R,B,H,dv,dk] bf16, entries 1.. are the
    ranges' start states; S_out [B,H,dv,dk] float32, the final state)."""
    L = load_library()
    R, B, H, dv, dk = E.shape
    if Sb is None:
        Sb = torch.empty((R, B, H, dv, dk), device=E.device, dtype=torch.bfloat16)
    if S_out is None:
        S_out = torch.empty((B, H, dv, dk), device=E.device, dtype=torch.float32)
    st = L.jet_gdn_range_compose(_ptr(E, "E", torch.float32), _ptr(A, "A", torch.float32, (R, B, H, dk, dk)),
                                 _ptr(Sb, "Sb", torch.bfloat16, (R, B, H, dv, dk)),
                                 _ptr(S_out, "S_out", torch.float32, (B, H, dv, dk)), R, B, H, dk, dv,
                                 _stream(stream))
    _check("jet_gdn_range_compose", st)
    return Sb, S_out


def jet_gdn_range_correct(Qe, Sb, o, *, stream=None):
    """o [B,T,H,dv] += the start-state term of a range: Qe from its range pass,
    Sb [B,H,dv,dk] bf16 its start state. Returns o."""
    L = load_library()
    B, T, H, dv = o.shape
    dk = Sb.shape[-1]
    st = L.jet_gdn_range_correct(_ptr(Qe, "Qe", o.dtype, (B, H, (T + 63) // 64, 64, dk)),
                                 _ptr(Sb, "Sb", torch.bfloat16, (B, H, dv, dk)), _ptr(o, "o"), B, T, H, dk, dv,
                                 _dt(o), _stream(stream))
    _check("jet_gdn_range_correct", st)
    return o


def jet_gdn_decode_step(q, k, v, g, beta, S, o=None, *, stream=None):
    """One decode step, S [B,H,dv,dk] float32 updated in place. q,k [B,H,dk],
    v [B,H,dv], g,beta [B,H]. Returns o [B,H,dv]."""
    L = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    st = L.jet_gdn_decode_step(_ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, H, dv)),
                               _ptr(g, "g", torch.float32, (B, H)), _ptr(beta, "beta", torch.float32, (B, H)),
                               _ptr(S, "S", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, H, dv)),
                               B, H, dk, dv, dt, _stream(stream))
    _check("jet_gdn_decode_step", st)
    return o


def jet_jetblock_decode_step(x, W1, W2, q, k, v, hist_in, hist_out, g, beta, S, o=None, taps=None, *,
                             stream=None):
    """Generator + conv + history shift + decode update for one new token per
    sequence. x [B,D], v [B,H,dv] raw, hist_in [B,3,H,dv] or None, hist_out
    [B,3,H,dv], S [B,H,dv,dk] float32 updated in place. Returns (o, taps)."""
    L = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    D = x.shape[-1]
    hidden, HW = W2.shape
    width = HW // H
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    if taps is None:
        taps = torch.empty((B, H, width), device=q.device, dtype=torch.float32)
    st = L.jet_jetblock_decode_step(
        _ptr(x, "x", q.dtype, (B, D)), _ptr(W1, "W1", q.dtype, (D, hidden)), _ptr(W2, "W2", q.dtype, (hidden, HW)),
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, H, dv)),
        _ptr(hist_in, "hist_in", q.dtype, (B, 3, H, dv)), _ptr(hist_out, "hist_out", q.dtype, (B, 3, H, dv)),
        _ptr(g, "g", torch.float32, (B, H)), _ptr(beta, "beta", torch.float32, (B, H)),
        _ptr(S, "S", torch.float32, (B, H, dv, dk)), _ptr(o, "o", q.dtype, (B, H, dv)),
        _ptr(taps, "taps", torch.float32, (B, H, width)),
        B, D, H, dk, dv, hidden, width, dt, _stream(stream))
    _check("jet_jetblock_decode_step", st)
    return o, taps


def jet_jetblock_decode_slots(x, W1, W2, q, k, v, g, beta, hist_pool, S_pool, slots, o=None, v_conv=None, taps=None,
                              *, stream=None):
    """One decode step for B sequences whose states and histories are pool
    entries: x [B,D], q,k [B,H,dk], v [B,H,dv] raw, g,beta [B,H] float32,
    hist_pool [N,3,H,dv] and S_pool [N,H,dv,dk] float32 updated in place at
    entries slots [B] (int32, distinct). Returns o [B,H,dv]."""
    L = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    D = x.shape[-1]
    hidden, HW = W2.shape
    width = HW // H
    N = S_pool.shape[0]
    if o is None:
        o = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    if v_conv is None:
        v_conv = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    st = L.jet_jetblock_decode_slots(
        _ptr(x, "x", q.dtype, (B, D)), _ptr(W1, "W1", q.dtype, (D, hidden)), _ptr(W2, "W2", q.dtype, (hidden, HW)),
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, H, dv)),
        _ptr(g, "g", torch.float32, (B, H)), _ptr(beta, "beta", torch.float32, (B, H)),
        _ptr(hist_pool, "hist_pool", q.dtype, (N, 3, H, dv)), _ptr(S_pool, "S_pool", torch.float32, (N, H, dv, dk)),
        _ptr(slots, "slots", torch.int32, (B,)), N, _ptr(o, "o", q.dtype, (B, H, dv)),
        _ptr(v_conv, "v_conv", q.dtype, (B, H, dv)), _ptr(taps, "taps", torch.float32, (B, H, width)),
        B, D, H, dk, dv, hidden, width, _dt(q), _stream(stream))
    _check("jet_jetblock_decode_slots", st)
    return o


def jet_conv_gdn_decode_step(q, k, v, hist_in, hist_out, taps, g, beta, S, o=None, *, stream=None):
    """Decode step with the conv of the new token fused in: v [B,H,dv] raw,
    taps [B,H,4] float32 from jet_kernel_gen, hist_in [B,3,H,dv] or None,
    hist_out [B,3,H,dv]; S updated in place. Returns o [B,H,dv]."""
    L = load_library()
    B, H, dk = q.shape
    dv = v.shape[-1]
    dt = _dt(q)
    if o is None:
        o = torch.empty((B, H, dv), device=q.device, dtype=q.dtype)
    st = L.jet_conv_gdn_decode_step(
        _ptr(q, "q"), _ptr(k, "k", q.dtype, q.shape), _ptr(v, "v", q.dtype, (B, H, dv)),
        _ptr(hist_in, "hist_in", q.dtype, (B, 3, H, dv)), _ptr(hist_out, "hist_out", q.dtype, (B, 3, H, dv)),
        _ptr(taps, "taps", torch.float32, (B, H, 4)), _ptr(g, "g", torch.float32, (B, H)),
        _ptr(beta, "beta", torch.float32, (B, H)), _ptr(S, "S", torch.float32, (B, H, dv, dk)),
        _ptr(o, "o", q.dtype, (B, H, dv)), B, H, dk, dv, dt, _stream(stream))
    _check("jet_conv_gdn_decode_step", st)
    return o


def jet_device_error(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error status."""
    return int(load_library().jet_device_error(_stream(stream)))


def jet_status_string(status: int) -> str:
    return load_library().jet_status_string(status).decode()


def jet_launch_count() -> int:
    return int(load_library().jet_launch_count())


def jet_jetblock_layer_workspace_size(B: int, T: int, D: int, H: int, dk: int, dv: int) -> int:
    """Workspace bytes of jet_jetblock_layer (0: not a supported shape)."""
    return int(load_library().jet_jetblock_layer_workspace_size(B, T, D, H, dk, dv))


def jet_jetblock_layer(x, Wq, Wk, Wv, Wg, Wb, Wz, Wo, gamma, W1, W2, hist_in=None, hist_out=None, S0=None, S_out=None,
                       y=None, workspace=None, *, stream=None):
    """The JetBlock layer: x [B,T,D] bf16 -> y [B,T,D] (projections, mixer,
    per-head RMSNorm with gamma [dv] and SiLU output gate, output projection).
    Wq, Wk [D,H*dk]; Wv, Wz [D,H*dv]; Wg, Wb [D,H]; Wo [H*dv,D]; W1, W2 the
    generator's. S0 / S_out [B,H,dv,dk] float32 (may be the same tensor: with
    T = 1 the state advances in place); hist_in / hist_out [B,3,H,dv].
    Returns (y, S_out)."""
    L = load_library()
    B, T, D = x.shape
    H = Wg.shape[1]
    dk = Wq.shape[1] // H
    dv = Wv.shape[1] // H
    bf = torch.bfloat16
    if y is None:
        y = torch.empty((B, T, D), device=x.device, dtype=bf)
    if S_out is None:
        S_out = torch.empty((B, H, dv, dk), device=x.device, dtype=torch.float32)
    if workspace is None:
        workspace = torch.empty(max(16, jet_jetblock_layer_workspace_size(B, T, D, H, dk, dv)), device=x.device,
                                dtype=torch.uint8)
    st = L.jet_jetblock_layer(
        _ptr(x, "x", bf), _ptr(Wq, "Wq", bf, (D, H * dk)), _ptr(Wk, "Wk", bf, (D, H * dk)),
        _ptr(Wv, "Wv", bf, (D, H * dv)), _ptr(Wg, "Wg", bf, (D, H)), _ptr(Wb, "Wb", bf, (D, H)),
        _ptr(Wz, "Wz", bf, (D, H * dv)), _ptr(Wo, "Wo", bf, (H * dv, D)), _ptr(gamma, "gamma", torch.float32, (dv,)),
        _ptr(W1, "W1", bf), _ptr(W2, "W2", bf), _ptr(hist_in, "hist_in", bf, (B, 3, H, dv)),
        _ptr(hist_out, "hist_out", bf, (B, 3, H, dv)), _ptr(S0, "S0", torch.float32, (B, H, dv, dk)),
        _ptr(S_out, "S_out", torch.float32, (B, H, dv, dk)), _ptr(y, "y", bf, (B, T, D)), _ptr(workspace, "workspace"),
        workspace.numel() * workspace.element_size(), B, T, D, H, dk, dv, W1.shape[1], W2.shape[1] // H, JET_BF16,
        _stream(stream))
    _check("jet_jetblock_layer", st)
    return y, S_out
