"""jet_gdn_prefill_noalloc: the prefill for callers that cannot allocate
device memory (graph capture, allocation-free serving loops, embedders with
a fixed memory budget). It takes its scratch from a fixed array inside the
library instead of a caller workspace.

Checks, through the C ABI: two calls in a row on different inputs give the
same outputs and final states as jet_gdn_prefill with a caller-allocated
workspace (within the bf16 parity tolerance used everywhere else), and a
size whose scratch would not fit the array is refused with
JET_ERR_TOO_LARGE before anything is launched. Collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, gpu_inputs, host64

pytestmark = pytest.mark.gpu

TOO_LARGE = 8


@pytest.fixture(scope="module")
def jet():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from linear_attention_lm_gen_b200 import build
    build.build()
    import linear_attention_lm_gen_b200 as m
    m.load_library()
    return m


def run_pair(jet, seed):
    # long enough for the sequence-parallel path, which is the one that needs scratch
    s = synth.JetShape("noalloc", B=1, T=1553, H=2, dk=96, dv=256, D=64)
    need = jet.jet_gdn_prefill_workspace_size(1, s.T, s.H, s.dk, s.dv)
    assert 0 < need <= jet.NOALLOC_SCRATCH_BYTES
    d = gpu_inputs(synth.prefill_inputs(s, seed=seed, gate_scale=0.01, s0_std=0.2))
    ws = torch.empty(need, device="cuda", dtype=torch.uint8)
    o_ref, S_ref = jet.jet_gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], workspace=ws)
    o = torch.full_like(o_ref, float("nan"))
    S_out = torch.full_like(S_ref, float("nan"))
    jet.jet_gdn_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, S_out)
    torch.cuda.synchronize()
    return o, S_out, o_ref, S_ref


def test_noalloc_prefill_matches_workspace_prefill_on_two_calls(jet):
    for seed in (31, 32):      # the second call sees the first call's leftovers in the scratch
        o, S_out, o_ref, S_ref = run_pair(jet, seed)
        assert_close(host64(o), host64(o_ref), "bf16", f"o (seed {seed})")
        assert_close(host64(S_out), host64(S_ref), "bf16", f"S (seed {seed})")
    assert jet.jet_device_error() == 0


def test_noalloc_prefill_refuses_sizes_beyond_its_scratch(jet):
    # 16 heads, dk = 128, 65536 tokens: the segment buffers need ~18.0 MB > 16 MiB
    B, T, H, dk, dv = 1, 65536, 16, 128, 256
    assert jet.jet_gdn_prefill_workspace_size(B, T, H, dk, dv) > jet.NOALLOC_SCRATCH_BYTES
    A = ctypes.c_void_p(1 << 20)        # aligned placeholders: the size check comes first
    L = jet.load_library()
    st = L.jet_gdn_prefill_noalloc(A, A, A, A, A, None, A, A, B, T, H, dk, dv, 64, 1, None)
    assert st == TOO_LARGE
    assert jet.jet_status_string(st) == "JET_ERR_TOO_LARGE"
