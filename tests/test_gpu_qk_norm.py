"""GPU parity of the in-kernel L2 normalisation of q and k.

Every other parity case draws q and k already unit-norm, so there a kernel
that skipped the normalisation, or applied a folded 1/|k| factor once instead
of twice, would still pass. Here each q and k row is rescaled by 10**U(-1, 1)
and one key row and one query row are exactly zero (where eps = 1e-6 under
the square root decides the result), and every path that normalises is run
against the float64 oracle on the same stored values:
  - the tensor-core prefill, both plans (chunk images + chain, and the fused
    low-memory kernel), dk 64 / 96 / 128, with the normalisation folded into
    per-token scales of the tensor-core products;
  - the FFMA prefill, float32 and bf16;
  - the one-call mixer prefill (conv folded into the chunk images), with
    sequence-parallel segments;
  - the decode step, the decode step with the conv fused in, and the decode
    over a state cache.
Pass criteria as everywhere: bf16 rel-L2 <= 1e-2 and max-abs <= 5e-2,
float32 rel-L2 <= 1e-4, on outputs and final states.
"""
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


@pytest.fixture(scope="module")
def orc():
    return get_oracle()


def spread(inp, seed, lead):
    """q and k rows rescaled by 10**U(-1, 1); one zero key row and one zero
    query row at the given leading indices."""
    dt = inp["dtype"]
    kz, qz = lead
    out = dict(inp)
    out["k"] = synth.spread_qk_norms(inp["k"], dt, seed, zero_rows=[kz])
    out["q"] = synth.spread_qk_norms(inp["q"], dt, seed + 1, zero_rows=[qz])
    return out


def prefill_inputs(s, seed, **kw):
    inp = synth.prefill_inputs(s, seed=seed, **kw)
    T = s.T
    return spread(inp, seed, [(0, T // 3, 0), (s.B - 1, T // 2, s.H - 1)])


def shape(dtype, **kw):
    base = dict(name="qk", B=2, T=130, H=2, dk=16, dv=32, D=64, dtype=dtype)
    base.update(kw)
    return synth.JetShape(**base)


def check_norms(inp):
    n = np.linalg.norm(synth.to_f64(inp["k"], inp["dtype"]), axis=-1)
    assert n.min() == 0.0 and n.max() > 2.0 and np.sort(n.ravel())[1] < 0.5


@pytest.mark.parametrize("dtype,dk,dv", [("bf16", 64, 128), ("bf16", 96, 256), ("bf16", 128, 256),
                                         ("f32", 16, 32), ("bf16", 48, 64)])
@pytest.mark.parametrize("plan", ["split", "fused"])
def test_prefill_normalises_q_and_k(orc, dtype, dk, dv, plan):
    if plan == "fused" and (dtype == "f32" or dk == 48):
        pytest.skip("the FFMA prefill has one plan")
    s = shape(dtype, dk=dk, dv=dv)
    inp = prefill_inputs(s, seed=41, s0_std=0.2)
    check_norms(inp)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    o = torch.full_like(d["v"], float("nan"))
    S_out = torch.full((s.B, s.H, dv, dk), float("nan"), device="cuda")
    ws = None
    if plan == "fused":
        n = jet.jet_gdn_prefill_workspace_min(s.B, s.T, s.H, dk, dv, 64, d["q"].dtype)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    jet.jet_gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"], o, S_out, workspace=ws)
    ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], inp["S0"].astype(np.float64))
    assert_close(host64(o), ro, dtype, "o")
    assert_close(host64(S_out), rS, dtype, "S")
    # the zero query row gives exactly zero output, whatever the state
    b, t, h = s.B - 1, s.T // 2, s.H - 1
    assert torch.count_nonzero(o[b, t, h].float()) == 0


@pytest.mark.parametrize("B,T,H,dk,dv,D", [(1, 1553, 2, 96, 256, 64), (2, 333, 3, 128, 256, 128),
                                          (2, 130, 2, 64, 128, 64)])
def test_mixer_prefill_normalises_q_and_k(orc, B, T, H, dk, dv, D):
    s = shape("bf16", B=B, T=T, H=H, dk=dk, dv=dv, D=D)
    inp = prefill_inputs(s, seed=43, s0_std=0.2, gate_scale=0.05)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    hin_np = synth.jetblock._draw(np.random.default_rng(9), (B, 3, H, dv), "bf16")
    hout = torch.full((B, 3, H, dv), float("nan"), device="cuda", dtype=torch.bfloat16)
    o = torch.full_like(d["v"], float("nan"))
    S_out = torch.full((B, H, dv, dk), float("nan"), device="cuda")
    jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"],
                             dev(hin_np, "bf16"), hout, d["S0"], o, S_out)
    r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"],
                             inp["S0"].astype(np.float64), synth.to_f64(hin_np, "bf16"))
    assert_close(host64(o), r["o"], "bf16", "o")
    assert_close(host64(S_out), r["S"], "bf16", "S")
    np.testing.assert_array_equal(host64(hout), r["hist"])


def decode_inputs(s, steps, seed):
    inp = synth.decode_inputs(s, seed=seed, steps=steps)
    # step-major leading axes [n, B, H]
    return spread(inp, seed, [(0, 0, 0), (steps - 1, s.B - 1, s.H - 1)])


@pytest.mark.parametrize("dtype,H,dk,dv", [("bf16", 12, 96, 256), ("bf16", 2, 128, 256), ("f32", 2, 16, 32)])
@pytest.mark.parametrize("path", ["two_calls", "fused", "slots"])
def test_decode_normalises_q_and_k(orc, dtype, H, dk, dv, path):
    steps = 4
    s = synth.JetShape("qk", B=3, T=1, H=H, dk=dk, dv=dv, D=64, dtype=dtype)
    inp = decode_inputs(s, steps, seed=45)
    d = gpu_inputs(inp)
    S = d["S0"].clone()
    ha, hb = d["hist"].clone(), torch.empty_like(d["hist"])
    if path == "slots":           # pool of 5 entries, the batch on entries 4, 1, 2
        slots = [4, 1, 2]
        S_pool = torch.zeros((5, H, dv, dk), device="cuda")
        h_pool = torch.zeros((5, 3, H, dv), device="cuda", dtype=d["hist"].dtype)
        S_pool[slots] = S
        h_pool[slots] = ha
        idx = torch.tensor(slots, dtype=torch.int32, device="cuda")
    outs = []
    for t in range(steps):
        if path == "two_calls":
            vc, _ = jet.jet_dyn_conv_v(d["x"][t][:, None], d["W1"], d["W2"], d["v"][t][:, None], ha, None, hb)
            o = jet.jet_gdn_decode_step(d["q"][t], d["k"][t], vc[:, 0], d["g"][t], d["beta"][t], S)
            ha, hb = hb, ha
        elif path == "fused":     # generator, then conv + history shift + update in one pass over S
            o, _ = jet.jet_jetblock_decode_step(d["x"][t], d["W1"], d["W2"], d["q"][t], d["k"][t], d["v"][t], ha, hb,
                                                d["g"][t], d["beta"][t], S)
            ha, hb = hb, ha
        else:
            o = jet.jet_jetblock_decode_slots(d["x"][t], d["W1"], d["W2"], d["q"][t], d["k"][t], d["v"][t],
                                              d["g"][t], d["beta"][t], h_pool, S_pool, idx)
        outs.append(o)
    if path == "slots":
        S, ha = S_pool[slots], h_pool[slots]
    dt = dtype
    r = orc.jetblock_decode(synth.to_f64(inp["x"], dt), synth.to_f64(inp["W1"], dt), synth.to_f64(inp["W2"], dt),
                            synth.to_f64(inp["q"], dt), synth.to_f64(inp["k"], dt), synth.to_f64(inp["v"], dt),
                            inp["g"], inp["beta"], inp["S0"].astype(np.float64), synth.to_f64(inp["hist"], dt))
    assert_close(host64(torch.stack(outs)), r["o"], dt, "o")
    assert_close(host64(S), r["S"], dt, "S")
    np.testing.assert_array_equal(host64(ha), r["hist"])
    assert torch.count_nonzero(outs[-1][s.B - 1, s.H - 1].float()) == 0      # the zero query row
