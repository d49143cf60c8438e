"""GPU: the sequence-parallel prefill's library calls, with the ranges of one
prompt run one after another on a single device (the exchange itself is
tested on CPU gloo ranks in test_seqpar_cpu.py): every range through
jet_jetblock_prefill_range (the first from the real start state, the others
from zero with their transition and output-correction operand), the pairs
composed by jet_gdn_range_compose, the later ranges corrected by
jet_gdn_range_correct. Outputs, final state and history must match the
float64 oracle over the whole prompt within the bf16 tolerance."""
import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, dev, gpu_inputs, host64, to_oracle
from oracle import get as get_oracle

pytestmark = pytest.mark.gpu

jet = None


@pytest.fixture(scope="module", autouse=True)
def _lib():
    global jet
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    from linear_attention_lm_gen_b200 import build
    build.build()
    import linear_attention_lm_gen_b200 as m
    m.load_library()
    jet = m
    yield
    assert m.jet_device_error() == 0


@pytest.mark.parametrize("bounds,H,dk,dv,D", [([0, 700, 1553], 2, 96, 256, 64),
                                              ([0, 130, 333, 520], 3, 128, 128, 128),
                                              ([0, 64, 129], 2, 64, 256, 64),
                                              ([0, 1100, 2300, 3000, 4096], 12, 96, 256, 1536)])
def test_ranges_compose_to_the_whole_prompt(bounds, H, dk, dv, D):
    B = 2 if bounds[-1] < 2000 else 1
    s = synth.JetShape("sp", B=B, T=bounds[-1], H=H, dk=dk, dv=dv, D=D)
    inp = synth.prefill_inputs(s, seed=81, s0_std=0.2, gate_scale=0.05)
    hist_np = synth.jetblock._draw(np.random.default_rng(4), (B, 3, H, dv), "bf16")
    d = gpu_inputs(inp)
    hist = dev(hist_np, "bf16")
    R = len(bounds) - 1
    outs, Es, As, Qes = [], [], [], []
    for r in range(R):
        a, b = bounds[r], bounds[r + 1]
        sl = lambda key: d[key][:, a:b].contiguous()
        halo = hist if r == 0 else d["v"][:, a - 3:a].contiguous()
        o, E, A, Qe = jet.jet_jetblock_prefill_range(sl("x"), d["W1"], d["W2"], sl("q"), sl("k"), sl("v"), sl("g"),
                                                     sl("beta"), halo, None, d["S0"] if r == 0 else None, r == 0)
        outs.append(o)
        Es.append(E)
        As.append(A if A is not None else torch.zeros((B, H, dk, dk), device="cuda"))
        Qes.append(Qe)
    Sb, S_final = jet.jet_gdn_range_compose(torch.stack(Es), torch.stack(As))
    for r in range(1, R):
        jet.jet_gdn_range_correct(Qes[r], Sb[r], outs[r])
    assert jet.jet_device_error() == 0
    ref = to_oracle(inp)
    r_ = get_oracle().jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"],
                                       ref["beta"], inp["S0"].astype(np.float64), synth.to_f64(hist_np, "bf16"))
    assert_close(host64(torch.cat(outs, 1)), r_["o"], "bf16", "o")
    assert_close(host64(S_final), r_["S"], "bf16", "S")


def test_a_single_first_range_equals_the_one_call_prefill():
    # 500 tokens (8 chunks, fewer than two segments' minimum): one segment in both, so the
    # same kernels run on the same data: bit for bit
    s = synth.JetShape("sp", B=2, T=500, H=3, dk=96, dv=256, D=64)
    assert jet.jet_gdn_prefill_workspace_min(2, 500, 3, 96, 256) == 0
    inp = synth.prefill_inputs(s, seed=82, s0_std=0.2)
    d = gpu_inputs(inp)
    h1 = torch.empty((2, 3, 3, 256), device="cuda", dtype=torch.bfloat16)
    h2 = torch.empty_like(h1)
    o1, S1 = jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"], None, h1,
                                      d["S0"])
    o2, E, A, Qe = jet.jet_jetblock_prefill_range(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"],
                                                  d["beta"], None, h2, d["S0"], True)
    assert A is None and Qe is None
    assert torch.equal(o1, o2) and torch.equal(S1, E) and torch.equal(h1, h2)
