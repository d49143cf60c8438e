"""jet_gdn_prefill_noalloc: the prefill for callers that cannot allocate
device memory (work recorded into a CUDA graph, allocation-free serving
loops, embedders with a fixed memory budget). It takes its scratch from a
fixed array inside the library instead of a caller workspace.

Checks, through the C ABI, each on two calls in a row with different inputs
(the second call finds the first call's leftovers in the shared array):
  - a size whose fastest plan fits the array (chunk images + segment
    buffers): the outputs and final state equal jet_gdn_prefill's with a
    caller workspace bit for bit (the same plan runs), and match the float64
    oracle within the bf16 parity tolerance;
  - a size whose fastest plan does not fit but whose smallest one does (the
    2B prompt shape, 4096 tokens: about 49 MB against 12.5 MB): the entry
    point runs the fused low-memory plan inside the array; it equals
    jet_gdn_prefill given exactly the minimum workspace bit for bit, and
    matches the oracle.
The refusal of sizes beyond the array is a host-side check and is tested
without a GPU in test_abi_cpu.py. Collected last on purpose.
"""
import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, gpu_inputs, host64, to_oracle
from oracle import get as get_oracle

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def jet():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from linear_attention_lm_gen_b200 import build
    build.build()
    import linear_attention_lm_gen_b200 as m
    m.load_library()
    return m


def run_pair(jet, s, seed, ws_bytes):
    """The workspace entry point with `ws_bytes` of caller workspace, then the
    allocation-free one on the same inputs (outputs poisoned first)."""
    inp = synth.prefill_inputs(s, seed=seed, gate_scale=0.01, s0_std=0.2)
    d = gpu_inputs(inp)
    ws = torch.empty(ws_bytes, device="cuda", dtype=torch.uint8)
    o_ref, S_ref = jet.jet_gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], workspace=ws)
    o = torch.full_like(o_ref, float("nan"))
    S_out = torch.full_like(S_ref, float("nan"))
    jet.jet_gdn_prefill_noalloc(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, S_out)
    torch.cuda.synchronize()
    return inp, o, S_out, o_ref, S_ref


@pytest.mark.parametrize("B,T,H,plan", [(1, 1553, 2, "fastest"), (1, 4096, 12, "minimum")])
def test_noalloc_prefill_matches_the_workspace_prefill_and_the_oracle_on_two_calls(jet, B, T, H, plan):
    s = synth.JetShape("noalloc", B=B, T=T, H=H, dk=96, dv=256, D=64)
    need = jet.jet_gdn_prefill_workspace_size(B, T, H, s.dk, s.dv)
    need_min = jet.jet_gdn_prefill_workspace_min(B, T, H, s.dk, s.dv)
    assert 0 < need_min <= jet.NOALLOC_SCRATCH_BYTES
    if plan == "fastest":
        assert need <= jet.NOALLOC_SCRATCH_BYTES
        ws_bytes = need
    else:                                   # only the fused plan's segment buffers fit
        assert need > jet.NOALLOC_SCRATCH_BYTES
        ws_bytes = need_min
    orc = get_oracle()
    for seed in (31, 32):
        inp, o, S_out, o_ref, S_ref = run_pair(jet, s, seed, ws_bytes)
        assert torch.equal(o, o_ref), f"o differs from jet_gdn_prefill (seed {seed})"
        assert torch.equal(S_out, S_ref), f"S differs from jet_gdn_prefill (seed {seed})"
        ref = to_oracle(inp)
        ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], inp["S0"].astype(np.float64))
        assert_close(host64(o), ro, "bf16", f"o vs oracle (seed {seed})")
        assert_close(host64(S_out), rS, "bf16", f"S vs oracle (seed {seed})")
    assert jet.jet_device_error() == 0
