"""The C ABI without a GPU: the library loads, exports every entry point that
include/jet.h declares, and rejects bad arguments before any CUDA call.

Every call here that passes made-up pointer values also passes an argument
that the host-side checks reject first, so no kernel is ever launched.
"""
import ctypes
import os
import re

import pytest

import linear_attention_lm_gen_b200 as jet
from linear_attention_lm_gen_b200 import build as jbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jet.h")

OK, INVALID, UNSUPPORTED, MISALIGNED, WORKSPACE = 0, 1, 2, 3, 7
A = 1 << 20          # an aligned, never-dereferenced address
BF16, F32 = 1, 0


@pytest.fixture(scope="module")
def lib():
    jbuild.build()
    return jet.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(jet_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for f in ("jet_kernel_gen", "jet_dyn_conv_v", "jet_gdn_prefill", "jet_gdn_decode_step",
              "jet_gdn_prefill_workspace_size", "jet_device_error", "jet_status_string", "jet_launch_count"):
        assert f in names


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), f"libjet.so does not export {name}"
    assert set(declared_functions()) == set(jet.EXPORTS)


def test_status_strings(lib):
    for code, name in jet.STATUS.items():
        assert jet.jet_status_string(code) == name
    assert jet.jet_status_string(99) == "JET_ERR_UNKNOWN"


def test_launch_counter_is_readable(lib):
    assert jet.jet_launch_count() >= 0


def P(x):
    return ctypes.c_void_p(x)


def prefill(lib, q=A, k=A, v=A, g=A, b=A, S0=None, o=A, S=A, ws=None, wsb=0,
            B=1, T=64, H=2, dk=16, dv=32, chunk=64, dt=BF16):
    return lib.jet_gdn_prefill(P(q), P(k), P(v), P(g), P(b), P(S0), P(o), P(S), P(ws), wsb,
                               B, T, H, dk, dv, chunk, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), INVALID), (dict(o=None), INVALID), (dict(S=None), INVALID),
    (dict(B=0), INVALID), (dict(T=-1), INVALID), (dict(H=0), INVALID),
    (dict(dk=24), UNSUPPORTED), (dict(dk=144), UNSUPPORTED), (dict(dv=48), UNSUPPORTED),
    (dict(dv=288), UNSUPPORTED), (dict(chunk=32), UNSUPPORTED), (dict(dt=7), INVALID),
    (dict(q=A + 2), MISALIGNED), (dict(S0=A + 8), MISALIGNED), (dict(S=A + 4), MISALIGNED),
    (dict(g=A + 2), MISALIGNED),
    (dict(B=1 << 30, T=1 << 30, H=1 << 30), INVALID),
])
def test_prefill_rejects(lib, kw, expect):
    assert prefill(lib, **kw) == expect


def decode(lib, q=A, k=A, v=A, g=A, b=A, S=A, o=A, B=4, H=2, dk=16, dv=32, dt=BF16):
    return lib.jet_gdn_decode_step(P(q), P(k), P(v), P(g), P(b), P(S), P(o), B, H, dk, dv, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(S=None), INVALID), (dict(v=None), INVALID), (dict(B=0), INVALID),
    (dict(dk=8), UNSUPPORTED), (dict(dv=40), UNSUPPORTED), (dict(o=A + 1), MISALIGNED),
    (dict(S=A + 4), MISALIGNED), (dict(g=A + 2), MISALIGNED),
    (dict(dt=3), INVALID),
])
def test_decode_rejects(lib, kw, expect):
    assert decode(lib, **kw) == expect


def conv(lib, x=A, w1=A, w2=A, v=A, hin=None, vout=A + (1 << 24), hout=None, cw=None,
         B=1, T=8, D=64, H=2, dv=32, hidden=32, width=4, dt=BF16):
    return lib.jet_dyn_conv_v(P(x), P(w1), P(w2), P(v), P(hin), P(vout), P(hout), P(cw),
                              B, T, D, H, dv, hidden, width, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=None), INVALID), (dict(v=None), INVALID), (dict(vout=None), INVALID),
    (dict(hidden=16), UNSUPPORTED), (dict(width=3), UNSUPPORTED), (dict(D=60), UNSUPPORTED),
    (dict(dv=48), UNSUPPORTED), (dict(H=65), UNSUPPORTED),
    (dict(v=A + 2), MISALIGNED), (dict(hout=A + 8 + (1 << 25)), MISALIGNED),
    (dict(vout=A), INVALID),                                    # v_out overlaps v
    (dict(hin=A + (1 << 26), hout=A + (1 << 26) + 16), INVALID),  # histories overlap
    (dict(T=0), INVALID),
])
def test_dyn_conv_rejects(lib, kw, expect):
    assert conv(lib, **kw) == expect


def test_kernel_gen_rejects(lib):
    f = lib.jet_kernel_gen
    assert f(P(A), P(A), P(A), P(None), 1, 8, 64, 2, 32, 4, BF16, None) == INVALID
    assert f(P(A), P(A), P(A), P(A + 2), 1, 8, 64, 2, 32, 4, BF16, None) == MISALIGNED
    assert f(P(A), P(A), P(A), P(A), 1, 8, 64, 2, 8, 4, BF16, None) == UNSUPPORTED


def test_workspace_query_is_host_only(lib):
    n = jet.jet_gdn_prefill_workspace_size(1, 4096, 12, 96, 256)
    assert n >= 0
    if n > 0:
        assert prefill(lib, B=1, T=4096, H=12, dk=96, dv=256, ws=None, wsb=0) == WORKSPACE


def one_pass_bytes(B, T, H, dk, dv, P):
    """Segment buffers of the one-pass plan: end states E [B][P][H][dv][dk] and transitions
    [B][P][H][dk][dk+8] (float32), start states [B][P][H][dv][dk] and output corrections
    [B][H][chunks][64][dk] (bf16), each part rounded up to 1024 bytes (none when P = 1)."""
    if P == 1:
        return 0
    up = lambda x: -(-x // 1024) * 1024
    nct = -(-T // 64)
    return up(4 * B * P * H * dv * dk) + up(4 * B * P * H * dk * (dk + 8)) + up(2 * B * P * H * dv * dk) \
        + up(2 * B * H * nct * 64 * dk)


@pytest.mark.parametrize("B,T,H,dk,dv,img,P", [(1, 4096, 12, 96, 256, 48128, 4), (2, 1553, 2, 64, 128, 35840, 3),
                                               (1, 65536, 16, 128, 256, 52224, 3), (3, 100, 2, 96, 256, 48128, 1)])
def test_workspace_sizes(lib, B, T, H, dk, dv, img, P):
    # fastest plan = one image per (sequence, head, 64-token chunk) + the one-pass segment buffers,
    # P segments in one launch of B H (2 P - 1 + ...) CTAs within 148 SMs (value slices of every
    # segment + a transition slice for each segment after the first)
    lo = jet.jet_gdn_prefill_workspace_min(B, T, H, dk, dv)
    hi = jet.jet_gdn_prefill_workspace_size(B, T, H, dk, dv)
    assert hi == B * H * ((T + 63) // 64) * img + one_pass_bytes(B, T, H, dk, dv, P)
    ns = dv // 128
    assert B * H * (ns * P + P - 1) <= 148 and (P == 1 or B * H * (ns * (P + 1) + P) > 148 or
                                                 -(-T // 64) // (P + 1) < 8)
    assert lo % 256 == 0 and hi % 1024 == 0
    # a workspace below the minimum is refused before anything runs
    if lo > 0:
        assert prefill(lib, B=B, T=T, H=H, dk=dk, dv=dv, ws=A, wsb=lo - 16) == WORKSPACE


def test_workspace_is_zero_off_the_tensor_core_path():
    import torch
    # float32 inputs and key dims other than 64 / 96 / 128 run the FFMA kernel, which needs none
    for args, dt in (((1, 4096, 12, 96, 256), torch.float32), ((1, 4096, 2, 48, 64), torch.bfloat16)):
        assert jet.jet_gdn_prefill_workspace_min(*args, 64, dt) == 0
        assert jet.jet_gdn_prefill_workspace_size(*args, 64, dt) == 0


def test_python_binding_refuses_cpu_tensors():
    import torch
    x = torch.zeros(1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises((TypeError, RuntimeError, AssertionError)):
        jet.jet_kernel_gen(x, torch.zeros(64, 32, dtype=torch.bfloat16), torch.zeros(32, 8, dtype=torch.bfloat16),
                           H=2, conv_w=torch.zeros(1, 4, 2, 4))


def fused_decode(lib, x=A, w1=A, w2=A, q=A, k=A, v=A, hin=A + (1 << 16), hout=A + (1 << 18), g=A, b=A, S=A,
                 o=A + (1 << 24), taps=A, B=2, D=64, H=2, dk=16, dv=32, hidden=32, width=4, dt=BF16):
    return lib.jet_jetblock_decode_step(P(x), P(w1), P(w2), P(q), P(k), P(v), P(hin), P(hout), P(g), P(b), P(S),
                                        P(o), P(taps), B, D, H, dk, dv, hidden, width, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), INVALID), (dict(hout=None), INVALID), (dict(taps=None), INVALID), (dict(S=None), INVALID),
    (dict(hout=A + (1 << 16) + 64), INVALID),            # the new history may not overlap the old one
    (dict(dk=24), UNSUPPORTED), (dict(dv=48), UNSUPPORTED), (dict(hidden=16), UNSUPPORTED),
    (dict(S=A + 8), MISALIGNED), (dict(taps=A + 4), MISALIGNED), (dict(x=A + 2), MISALIGNED),
    (dict(o=A + 64), INVALID), (dict(o=A + (1 << 18)), INVALID),   # o holds v' first: it may not overlap v or hist_out
    (dict(o=A + (1 << 24) + 2), MISALIGNED),
])
def test_fused_decode_rejects(lib, kw, expect):
    assert fused_decode(lib, **kw) == expect


def jetblock_prefill(lib, x=A, w1=A, w2=A, q=A, k=A, v=A, hin=None, hout=None, g=A, b=A, S0=None,
                     o=A + (1 << 24), S_out=A, ws=A, ws_bytes=0, B=1, T=64, D=64, H=2, dk=96, dv=128, hidden=32,
                     width=4, chunk=64, dt=BF16):
    return lib.jet_jetblock_prefill(P(x), P(w1), P(w2), P(q), P(k), P(v), P(hin), P(hout), P(g), P(b), P(S0),
                                    P(o), P(S_out), P(ws), ws_bytes, B, T, D, H, dk, dv, hidden, width, chunk, dt,
                                    None)


@pytest.mark.parametrize("kw,expect", [
    (dict(), WORKSPACE),                                   # no workspace: refused before any launch
    (dict(ws=None), WORKSPACE), (dict(q=None), INVALID), (dict(S_out=None), INVALID),
    (dict(o=A + 64), INVALID),                             # o may not overlap v
    (dict(hout=A + 128), INVALID),                         # nor may the new history
    (dict(hin=A + (1 << 22), hout=A + (1 << 22) + 256), INVALID),
    (dict(chunk=32), UNSUPPORTED), (dict(width=3), UNSUPPORTED), (dict(dv=48), UNSUPPORTED),
    (dict(v=A + 8), MISALIGNED), (dict(g=A + 2), MISALIGNED), (dict(hout=A + (1 << 23) + 8), MISALIGNED),
])
def test_jetblock_prefill_rejects(lib, kw, expect):
    assert jetblock_prefill(lib, **kw) == expect


@pytest.mark.parametrize("B,T,H,dk,dv", [(1, 4096, 12, 96, 256), (2, 130, 3, 64, 128), (1, 65536, 16, 128, 256)])
def test_jetblock_prefill_workspace_is_taps_plus_the_fastest_plan(lib, B, T, H, dk, dv):
    taps = -(-B * T * H * 4 * 4 // 1024) * 1024
    n = jet.jet_jetblock_prefill_workspace_size(B, T, H, dk, dv)
    assert n == taps + jet.jet_gdn_prefill_workspace_size(B, T, H, dk, dv)
    # one byte short is refused before anything runs
    assert jetblock_prefill(lib, ws_bytes=n - 1, B=B, T=T, H=H, dk=dk, dv=dv, D=64,
                            o=A + (1 << 40), hin=None) == WORKSPACE


def test_jetblock_prefill_workspace_off_the_tensor_core_path():
    import torch
    # float32 (and shapes the tensor-core prefill does not take): taps + a v' buffer
    for (B, T, H, dk, dv, dt, es) in ((1, 64, 2, 16, 32, torch.float32, 4), (2, 100, 3, 48, 64, torch.bfloat16, 2)):
        up = lambda x: -(-x // 1024) * 1024
        assert jet.jet_jetblock_prefill_workspace_size(B, T, H, dk, dv, 64, dt) == up(B * T * H * 16) + up(B * T * H * dv * es)


def decode_slots(lib, x=A, w1=A, w2=A, q=A, k=A, v=A, g=A, b=A, hist=A, S=A, slots=A, n_slots=8, o=A,
                 vc=A + (1 << 22), taps=None, B=2, D=64, H=2, dk=16, dv=32, hidden=32, width=4, dt=BF16):
    return lib.jet_jetblock_decode_slots(P(x), P(w1), P(w2), P(q), P(k), P(v), P(g), P(b), P(hist), P(S), P(slots),
                                         n_slots, P(o), P(vc), P(taps), B, D, H, dk, dv, hidden, width, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(slots=None), INVALID), (dict(hist=None), INVALID), (dict(vc=None), INVALID),
    (dict(n_slots=0), INVALID), (dict(n_slots=1), INVALID),   # fewer pool entries than sequences
    (dict(vc=A + 32), INVALID),                                # the conv output may not overlap v
    (dict(dk=24), UNSUPPORTED), (dict(S=A + 8), MISALIGNED), (dict(slots=A + 2), MISALIGNED),
    (dict(hist=A + 8), MISALIGNED),
])
def test_decode_slots_rejects(lib, kw, expect):
    assert decode_slots(lib, **kw) == expect


def segments_from_workspace(B, T, H, dk, dv):
    """The number of sequence-parallel segments P the library plans, recovered from its minimum
    workspace: 4 * (B (P-1) H dv dk + B (P-1) H dk (dk + 8) + B P H dv dk) bytes (0 when P = 1)."""
    n = jet.jet_gdn_prefill_workspace_min(B, T, H, dk, dv)
    if n == 0:
        return 1
    per_seg = 4 * B * H * (2 * dv * dk + dk * (dk + 8))
    P = (n // 4 + B * H * (dv * dk + dk * (dk + 8))) * 4 // per_seg
    assert 4 * (B * (P - 1) * H * dv * dk + B * (P - 1) * H * dk * (dk + 8) + B * P * H * dv * dk) == n
    return P


@pytest.mark.parametrize("B,T,H,dk,dv,P", [
    (1, 4096, 12, 96, 256, 5),       # 2B prompt: 5 segments of 13 chunks, both phases within 148 SMs
    (1, 65536, 16, 128, 256, 4),     # 4B long prompt
    (1, 262144, 12, 96, 256, 5),
    (1, 64 * 14, 12, 96, 256, 1),    # segments keep at least 8 chunks: 14 chunks run in one pass
    (1, 64 * 15, 12, 96, 256, 2),    # ... and 15 split in two
    (8, 4096, 12, 96, 256, 1),       # a batch already fills the GPU
])
def test_segment_plan_of_the_stated_shapes(lib, B, T, H, dk, dv, P):
    assert segments_from_workspace(B, T, H, dk, dv) == P


@pytest.mark.parametrize("std,lang", [("c99", "c"), ("c++17", "c++")])
def test_header_is_plain_c(tmp_path, std, lang):
    # the boundary is a C ABI: the header compiles as strict C99 (and as C++) with no torch or CUDA types
    import shutil
    import subprocess
    cc = shutil.which("gcc" if lang == "c" else "g++")
    if cc is None:
        pytest.skip("no host compiler")
    src = tmp_path / "use_jet.c"
    src.write_text('#include "jet.h"\nint main(void) { return (int)jet_launch_count(); }\n')
    r = subprocess.run([cc, f"-std={std}", "-Wall", "-Wextra", "-Werror", "-pedantic", "-fsyntax-only", "-x", lang,
                        "-I", os.path.dirname(HEADER), str(src)], capture_output=True, text=True)
    assert r.returncode == 0, r.stderr


def test_noalloc_prefill_refuses_sizes_beyond_its_scratch(lib):
    # 16 heads, dk = 128, 65536 tokens: even the smallest plan's segment buffers (~18.0 MB)
    # exceed the 16 MiB array; the check is on the host and comes before any CUDA call
    TOO_LARGE = 8
    B, T, H, dk, dv = 1, 65536, 16, 128, 256
    assert jet.jet_gdn_prefill_workspace_min(B, T, H, dk, dv) > jet.NOALLOC_SCRATCH_BYTES
    st = lib.jet_gdn_prefill_noalloc(P(A), P(A), P(A), P(A), P(A), None, P(A), P(A), B, T, H, dk, dv, 64, BF16, None)
    assert st == TOO_LARGE
    assert jet.jet_status_string(st) == "JET_ERR_TOO_LARGE"
    # the 2B shapes fit at any length (segment buffers of at most 12.5 MB)
    assert jet.jet_gdn_prefill_workspace_min(1, 262144, 12, 96, 256) <= jet.NOALLOC_SCRATCH_BYTES
    # bad arguments are refused before the size check as well
    assert lib.jet_gdn_prefill_noalloc(None, P(A), P(A), P(A), P(A), None, P(A), P(A), B, T, H, dk, dv, 64, BF16,
                                       None) == INVALID


def test_the_library_has_no_test_hooks(lib):
    # the hook that makes a wait run out exists only in test builds
    assert not hasattr(lib, "jet_test_skip_p2a")


def prefill_range(lib, x=A, w1=A, w2=A, q=A, k=A, v=A, hin=None, hout=None, g=A, b=A, S0=None, o=A + (1 << 24),
                  E=A, Aout=A + (1 << 26), Qe=A + (1 << 27), ws=A, ws_bytes=1 << 30, B=1, T=256, D=64, H=2, dk=96,
                  dv=128, hidden=32, width=4, chunk=64, dt=BF16):
    return lib.jet_jetblock_prefill_range(P(x), P(w1), P(w2), P(q), P(k), P(v), P(hin), P(hout), P(g), P(b), P(S0),
                                          P(o), P(E), P(Aout), P(Qe), P(ws), ws_bytes, B, T, D, H, dk, dv, hidden,
                                          width, chunk, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(E=None), INVALID), (dict(Aout=None), INVALID),        # A and Qe come together
    (dict(Qe=None), INVALID), (dict(o=A + 64), INVALID),          # o may not overlap v
    (dict(dk=48), UNSUPPORTED), (dict(dt=F32), UNSUPPORTED),      # tensor-core shapes only
    (dict(dv=96), UNSUPPORTED), (dict(chunk=32), UNSUPPORTED),
    (dict(E=A + 8), MISALIGNED), (dict(Qe=A + (1 << 27) + 8), MISALIGNED),
    (dict(ws_bytes=1024), WORKSPACE), (dict(ws=None), WORKSPACE),
])
def test_prefill_range_rejects(lib, kw, expect):
    assert prefill_range(lib, **kw) == expect


def test_prefill_range_workspace_is_taps_plus_images(lib):
    B, T, H, dk, dv = 1, 4096, 12, 96, 256
    taps = -(-B * T * H * 16 // 1024) * 1024
    assert jet.jet_jetblock_prefill_range_workspace_size(B, T, H, dk, dv) == taps + B * H * (T // 64) * 48128
    assert jet.jet_jetblock_prefill_range_workspace_size(B, T, H, 48, dv) == 0    # not a tensor-core shape


@pytest.mark.parametrize("kw,expect", [
    (dict(R=1), INVALID), (dict(E=None), INVALID), (dict(dk=48), UNSUPPORTED), (dict(dv=200), UNSUPPORTED),
    (dict(Sb=A + 8), MISALIGNED), (dict(S=A), INVALID),             # the final state may not overlap E
])
def test_range_compose_rejects(lib, kw, expect):
    a = dict(E=A, Aa=A + (1 << 26), Sb=A + (1 << 27), S=A + (1 << 28), R=2, B=1, H=2, dk=96, dv=128)
    a.update(kw)
    assert lib.jet_gdn_range_compose(P(a["E"]), P(a["Aa"]), P(a["Sb"]), P(a["S"]), a["R"], a["B"], a["H"], a["dk"],
                                     a["dv"], None) == expect


@pytest.mark.parametrize("kw,expect", [
    (dict(Qe=None), INVALID), (dict(dk=48), UNSUPPORTED), (dict(dt=F32), UNSUPPORTED),
    (dict(o=A + 8), MISALIGNED), (dict(o=A), INVALID),               # o may not overlap Qe
])
def test_range_correct_rejects(lib, kw, expect):
    a = dict(Qe=A, Sb=A + (1 << 26), o=A + (1 << 27), B=1, T=256, H=2, dk=96, dv=128, dt=BF16)
    a.update(kw)
    assert lib.jet_gdn_range_correct(P(a["Qe"]), P(a["Sb"]), P(a["o"]), a["B"], a["T"], a["H"], a["dk"], a["dv"],
                                     a["dt"], None) == expect


def prefill_varlen(lib, x=A, w1=A, w2=A, q=A, k=A, v=A, hin=None, hout=None, g=A, b=A, S0=None, o=A + (1 << 24),
                   S=A + (1 << 26), ws=A, ws_bytes=1 << 30, cu=(0, 100, 300), nseq=None, D=64, H=2, dk=96, dv=128,
                   hidden=32, width=4, chunk=64, dt=BF16):
    arr = None if cu is None else (ctypes.c_int * len(cu))(*cu)
    n = (len(cu) - 1 if cu is not None else 2) if nseq is None else nseq
    return lib.jet_jetblock_prefill_varlen(P(x), P(w1), P(w2), P(q), P(k), P(v), P(hin), P(hout), P(g), P(b), P(S0),
                                           P(o), P(S), P(ws), ws_bytes, arr, n, D, H, dk, dv, hidden, width, chunk,
                                           dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(cu=None), INVALID), (dict(cu=(0, 100, 100)), INVALID),     # offsets: present, strictly increasing
    (dict(cu=(5, 100)), INVALID), (dict(cu=(0,), nseq=0), INVALID),  # from 0; at least one sequence
    (dict(cu=tuple(range(0, 2580, 10))), UNSUPPORTED),              # 257 sequences: more than one call takes
    (dict(dk=48), UNSUPPORTED), (dict(dt=F32), UNSUPPORTED),         # tensor-core shapes only
    (dict(dv=96), UNSUPPORTED), (dict(chunk=32), UNSUPPORTED),
    (dict(o=A + 64), INVALID), (dict(q=None), INVALID),              # o may not overlap v
    (dict(S=A + (1 << 26) + 8), MISALIGNED), (dict(hout=A + (1 << 27) + 4), MISALIGNED),
    (dict(ws_bytes=1024), WORKSPACE), (dict(ws=None), WORKSPACE),
])
def test_prefill_varlen_rejects(lib, kw, expect):
    assert prefill_varlen(lib, **kw) == expect


def test_prefill_varlen_workspace(lib):
    # lengths 1, 62, 237, 1253, 2543: one segment each fits one wave at H = 12, so the workspace
    # is the taps of every token plus one image per chunk (66 chunks), no one-pass buffers
    cu = [0, 1, 63, 300, 1553, 4096]
    H, dk, dv = 12, 96, 256
    assert jet.jet_jetblock_prefill_varlen_workspace_size(cu, H, dk, dv) == 4096 * H * 16 + 66 * H * 48128
    # two long prompts over two heads are split into segments: the one-pass buffers come on top
    two = jet.jet_jetblock_prefill_varlen_workspace_size([0, 4096, 8192], 2, dk, dv)
    assert two > -(-8192 * 2 * 16 // 1024) * 1024 + 128 * 2 * 48128
    assert jet.jet_jetblock_prefill_varlen_workspace_size(cu, H, 48, dv) == 0      # not a tensor-core shape
    assert jet.jet_jetblock_prefill_varlen_workspace_size([0, 10, 5], H, dk, dv) == 0
    assert jet.jet_jetblock_prefill_varlen_workspace_size(list(range(0, 2580, 10)), H, dk, dv) == 0


def layer(lib, x=A, wq=A, wk=A, wv=A, wg=A, wb=A, wz=A, wo=A, gamma=A, w1=A, w2=A, hin=None, hout=A + (1 << 24),
          S0=None, S=A + (1 << 26), y=A + (1 << 27), ws=A + (1 << 28), ws_bytes=1 << 40, B=1, T=64, D=64, H=2, dk=64,
          dv=128, hidden=32, width=4, dt=BF16):
    return lib.jet_jetblock_layer(P(x), P(wq), P(wk), P(wv), P(wg), P(wb), P(wz), P(wo), P(gamma), P(w1), P(w2),
                                  P(hin), P(hout), P(S0), P(S), P(y), P(ws), ws_bytes, B, T, D, H, dk, dv, hidden,
                                  width, dt, None)


@pytest.mark.parametrize("kw,expect", [
    (dict(x=None), INVALID), (dict(wz=None), INVALID), (dict(gamma=None), INVALID), (dict(y=None), INVALID),
    (dict(T=1, hout=None), INVALID),                                 # a decode step shifts the history
    (dict(dk=48), UNSUPPORTED), (dict(dv=96), UNSUPPORTED), (dict(dt=F32), UNSUPPORTED),
    (dict(D=72), UNSUPPORTED), (dict(hidden=16), UNSUPPORTED),
    (dict(gamma=A + 4), MISALIGNED), (dict(S=A + (1 << 26) + 8), MISALIGNED), (dict(wo=A + 1), MISALIGNED),
    (dict(ws_bytes=1024), WORKSPACE), (dict(ws=None), WORKSPACE),
])
def test_layer_rejects(lib, kw, expect):
    assert layer(lib, **kw) == expect


def test_layer_workspace_is_the_projections_plus_the_mixer(lib):
    B, T, D, H, dk, dv = 1, 4096, 1536, 12, 96, 256
    up = lambda b: -(-b // 1024) * 1024
    N = B * T
    own = 2 * up(N * H * dk * 2) + 3 * up(N * H * dv * 2) + 2 * up(N * H * 4)
    assert jet.jet_jetblock_layer_workspace_size(B, T, D, H, dk, dv) == \
        own + jet.jet_jetblock_prefill_workspace_size(B, T, H, dk, dv)
    # one new token per sequence: the decode kernels (taps only) instead of the prefill's workspace
    assert jet.jet_jetblock_layer_workspace_size(256, 1, D, H, dk, dv) == \
        2 * up(256 * H * dk * 2) + 3 * up(256 * H * dv * 2) + 2 * up(256 * H * 4) + up(256 * H * 16)
    assert jet.jet_jetblock_layer_workspace_size(B, T, D, H, 48, dv) == 0
    assert jet.jet_jetblock_layer_workspace_size(B, T, 72, H, dk, dv) == 0
