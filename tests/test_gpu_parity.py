"""GPU parity: the CUDA library (through its C ABI) against the float64 oracle
on identical seeded inputs.

Pass criteria on outputs o and final states S (and conv history):
bf16 inputs -> relative L2 <= 1e-2 and max-abs <= 5e-2; float32 -> relative
L2 <= 1e-4. Stage checks of intermediate results use tighter bounds derived
from their arithmetic (stated beside each). Outputs are poisoned with NaN
before each call so unwritten elements fail the finiteness check.
"""
import numpy as np
import pytest
import torch

import synth
from jet_testlib import TOL, assert_close, dev, errors, gpu_inputs, host64, to_oracle
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


def nan_like(t):
    return torch.full_like(t, float("nan"))


def prefill(plan, q, k, v, g, beta, S0=None, o=None, S_out=None):
    """jet_gdn_prefill with the fastest plan ("split": chunk images, then the
    chain kernel) or, given only the minimum workspace, the fused plan."""
    ws = None
    if plan == "fused":
        B, T, H, dk = q.shape
        n = jet.jet_gdn_prefill_workspace_min(B, T, H, dk, v.shape[-1], 64, q.dtype)
        ws = torch.empty(max(n, 16), dtype=torch.uint8, device="cuda")
    return jet.jet_gdn_prefill(q, k, v, g, beta, S0, o, S_out, workspace=ws)


PLANS = ["split", "fused"]


def shape(dtype, **kw):
    base = dict(name="t", B=1, T=64, H=2, dk=16, dv=32, D=64, dtype=dtype)
    base.update(kw)
    return synth.JetShape(**base)


# ------------------------------------------------------------------ K3 decode
@pytest.mark.parametrize("dtype,H,dk,dv", [("f32", 2, 16, 32), ("bf16", 3, 96, 256), ("bf16", 2, 128, 256),
                                           ("bf16", 2, 48, 64), ("f32", 3, 128, 96)])
def test_decode_step_stage(orc, dtype, H, dk, dv):
    s = shape(dtype, B=5, T=0, H=H, dk=dk, dv=dv, D=64, steps=2)
    inp = synth.decode_inputs(s, seed=1)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    S = d["S0"].clone()
    Sref = inp["S0"].astype(np.float64)
    for step in range(2):
        o = nan_like(d["v"][step])
        jet.jet_gdn_decode_step(d["q"][step], d["k"][step], d["v"][step], d["g"][step], d["beta"][step], S, o)
        ro, Sref = orc.gdn_decode_step(ref["q"][step], ref["k"][step], ref["v"][step], ref["g"][step],
                                       ref["beta"][step], Sref)
        assert_close(host64(o), ro, dtype, f"o step {step}")
        # the state is float32 end to end: tight bound
        assert_close(host64(S), Sref, dtype, f"S step {step}", tol=dict(rel_l2=1e-5, max_abs=1e-5))


# ------------------------------------------------------------------ K1 generator + conv
@pytest.mark.parametrize("dtype,B,T,H,dv,D,hist", [
    ("f32", 1, 64, 2, 32, 64, False), ("f32", 2, 37, 2, 32, 64, True),
    ("bf16", 1, 100, 12, 256, 1536, False), ("bf16", 3, 37, 12, 256, 1536, True),
    ("bf16", 4, 1, 16, 256, 2048, True), ("bf16", 2, 2, 2, 64, 128, True), ("bf16", 1, 300, 2, 32, 64, False),
])
def test_generator_and_conv_stage(orc, dtype, B, T, H, dv, D, hist):
    s = shape(dtype, B=B, T=T, H=H, dv=dv, D=D)
    inp = synth.prefill_inputs(s, seed=2)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    hin_np = synth.jetblock._draw(np.random.default_rng(5), (B, 3, H, dv), dtype) if hist else None
    hin = dev(hin_np, dtype) if hist else None
    vout = nan_like(d["v"])
    hout = torch.full((B, 3, H, dv), float("nan"), device="cuda", dtype=d["v"].dtype)
    cw = torch.full((B, T, H, 4), float("nan"), device="cuda")
    jet.jet_dyn_conv_v(d["x"], d["W1"], d["W2"], d["v"], hin, vout, hout, cw)
    w = orc.kernel_gen(ref["x"], ref["W1"], ref["W2"], H)
    vc, hist_ref = orc.dyn_conv(ref["v"], w, synth.to_f64(hin_np, dtype) if hist else None)
    # taps: fp32 accumulation of bf16 / f32 products, no output rounding
    assert_close(host64(cw), w, dtype, "taps", tol=dict(rel_l2=1e-5, max_abs=1e-4))
    assert_close(host64(vout), vc, dtype, "v'")
    # the new history is a copy of raw V: bit-exact
    np.testing.assert_array_equal(host64(hout), hist_ref)
    # the generator-only entry point gives the same taps bit for bit
    cw2 = jet.jet_kernel_gen(d["x"], d["W1"], d["W2"], H)
    assert torch.equal(cw2, cw)


@pytest.mark.parametrize("B,T,H,D", [(1, 4096, 12, 1536), (2, 1553, 16, 2048), (1, 1024, 3, 80),
                                     (3, 5001, 12, 1536), (2, 16411, 12, 1536), (1, 33000, 3, 80)])
def test_generator_long_prompt(orc, B, T, H, D):
    # prompts of 1024+ tokens take the stand-alone generator (32 tokens per CTA, D in
    # 128-column slices: D = 80 is one partial slice, 2 x 1553 and 3 x 5001 tokens end
    # mid-CTA); from 32768 tokens on, 128 tokens per CTA in 64-column slices (D = 80: a
    # partial second slice; 2 x 16411 and 33000 tokens end mid-CTA)
    s = shape("bf16", B=B, T=T, H=H, dv=32, D=D)
    inp = synth.prefill_inputs(s, seed=4)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    cw = jet.jet_kernel_gen(d["x"], d["W1"], d["W2"], H, torch.full((B, T, H, 4), float("nan"), device="cuda"))
    w = orc.kernel_gen(ref["x"], ref["W1"], ref["W2"], H)
    assert_close(host64(cw), w, "bf16", "taps", tol=dict(rel_l2=1e-5, max_abs=1e-4))


def test_identity_taps_via_conv_stage(orc):
    # W2 = 0 gives zero taps: v' = 0 whatever V is (no hidden bias or tap offset)
    s = shape("bf16", T=70, H=2, dv=64, D=128)
    inp = synth.prefill_inputs(s, seed=3)
    d = gpu_inputs(inp)
    vout = nan_like(d["v"])
    jet.jet_dyn_conv_v(d["x"], d["W1"], torch.zeros_like(d["W2"]), d["v"], None, vout)
    assert torch.count_nonzero(vout.float()) == 0


# ------------------------------------------------------------------ K2 prefill
@pytest.mark.parametrize("dtype,H,dk,dv", [("f32", 2, 16, 32), ("bf16", 12, 96, 256), ("bf16", 2, 128, 256),
                                           ("bf16", 3, 32, 64), ("f32", 2, 64, 64), ("bf16", 2, 64, 128)])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 130, 333])
@pytest.mark.parametrize("s0", [False, True])
@pytest.mark.parametrize("plan", PLANS)
def test_prefill_gdn_stage(orc, dtype, H, dk, dv, T, s0, plan):
    s = shape(dtype, B=2, T=T, H=H, dk=dk, dv=dv, D=64)
    inp = synth.prefill_inputs(s, seed=T, s0_std=0.3 if s0 else None)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    o = nan_like(d["v"])
    S_out = torch.full((2, H, dv, dk), float("nan"), device="cuda")
    prefill(plan, d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("S0"), o, S_out)
    ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"],
                                inp["S0"].astype(np.float64) if s0 else None)
    assert_close(host64(o), ro, dtype, "o")
    assert_close(host64(S_out), rS, dtype, "S")


@pytest.mark.parametrize("dtype,dk", [("bf16", 96), ("f32", 16)])
@pytest.mark.parametrize("plan", PLANS)
def test_prefill_long_memory_gates(orc, dtype, dk, plan):
    # g = -0.01 softplus(N(0,1)): a ~ 0.99, so the state carries across many chunks
    s = shape(dtype, B=1, T=400, H=2, dk=dk, dv=64, D=64)
    inp = synth.prefill_inputs(s, seed=9, gate_scale=0.01, s0_std=0.1)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    o, S_out = prefill(plan, d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], inp["S0"].astype(np.float64))
    assert_close(host64(o), ro, dtype, "o")
    assert_close(host64(S_out), rS, dtype, "S")


@pytest.mark.parametrize("B,T,dk,s0,gate_scale", [(1, 1553, 96, True, 0.01), (2, 1600, 64, False, 0.01),
                                                  (1, 4096 + 64 * 9 + 5, 128, True, 1.0)])
@pytest.mark.parametrize("plan", PLANS)
def test_prefill_sequence_parallel_segments(orc, B, T, dk, s0, gate_scale, plan):
    # long enough for the segmented path (phase A, combine, phase C); long-memory
    # gates make the carried segment states matter
    import linear_attention_lm_gen_b200 as m
    assert m.jet_gdn_prefill_workspace_min(B, T, 2, dk, 256) > 0
    s = shape("bf16", B=B, T=T, H=2, dk=dk, dv=256, D=64)
    inp = synth.prefill_inputs(s, seed=21, gate_scale=gate_scale, s0_std=0.2 if s0 else None)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    o = nan_like(d["v"])
    S_out = torch.full((B, 2, 256, dk), float("nan"), device="cuda")
    prefill(plan, d["q"], d["k"], d["v"], d["g"], d["beta"], d.get("S0"), o, S_out)
    ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"],
                                inp["S0"].astype(np.float64) if s0 else None)
    assert_close(host64(o), ro, "bf16", "o")
    assert_close(host64(S_out), rS, "bf16", "S")


@pytest.mark.parametrize("plan", PLANS)
def test_prefill_segments_final_state_may_alias_initial_state(orc, plan):
    s = shape("bf16", B=1, T=2000, H=2, dk=96, dv=256, D=64)
    inp = synth.prefill_inputs(s, seed=22, gate_scale=0.01, s0_std=0.2)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    S = d["S0"].clone()
    o, _ = prefill(plan, d["q"], d["k"], d["v"], d["g"], d["beta"], S, None, S)
    ro, rS = orc.gdn_sequential(ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"], inp["S0"].astype(np.float64))
    assert_close(host64(o), ro, "bf16", "o")
    assert_close(host64(S), rS, "bf16", "S")


def test_prefill_state_alias_and_continuation(orc):
    # S_out may alias S0; prefill(T1) then prefill(T2) from its state = prefill(T1+T2)
    s = shape("bf16", B=2, T=200, H=2, dk=64, dv=64, D=64)
    inp = synth.prefill_inputs(s, seed=4, s0_std=0.2)
    d = gpu_inputs(inp)
    o_full, S_full = jet.jet_gdn_prefill(d["q"], d["k"], d["v"], d["g"], d["beta"], d["S0"])
    S = d["S0"].clone()
    parts = []
    for a, b in ((0, 77), (77, 200)):
        sl = lambda t: t[:, a:b].contiguous()
        o, _ = jet.jet_gdn_prefill(sl(d["q"]), sl(d["k"]), sl(d["v"]), sl(d["g"]), sl(d["beta"]), S, None, S)
        parts.append(o)
    e = errors(host64(torch.cat(parts, 1)), host64(o_full))
    assert e["rel_l2"] < 1e-2
    assert errors(host64(S), host64(S_full))["rel_l2"] < 1e-3


# ------------------------------------------------------------------ whole mixer, stated configs
def run_prefill(d, H, hist_out=False):
    vc, hout = jet.jet_dyn_conv_v(d["x"], d["W1"], d["W2"], d["v"], None, None,
                                  torch.empty((d["v"].shape[0], 3, H, d["v"].shape[-1]), device="cuda",
                                              dtype=d["v"].dtype) if hist_out else None)
    o, S = jet.jet_gdn_prefill(d["q"], d["k"], vc, d["g"], d["beta"])
    return vc, o, S, hout


@pytest.mark.parametrize("name", ["tiny_f32", "prefill_2b_t4096"])
@pytest.mark.parametrize("one_call", [False, True])
def test_config_prefill_full(orc, name, one_call):
    s = synth.CONFIGS[name]
    inp = synth.prefill_inputs(s, seed=0)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"])
    if one_call:     # jet_jetblock_prefill: generator, then the conv inside the prefill
        o, S = jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"])
    else:
        vc, o, S, _ = run_prefill(d, s.H)
        assert_close(host64(vc), r["v_conv"], s.dtype, f"{name} v'")
    assert_close(host64(o), r["o"], s.dtype, f"{name} o")
    assert_close(host64(S), r["S"], s.dtype, f"{name} S")


# ------------------------------------------------------------------ generator + conv inside the prefill
@pytest.mark.parametrize("dtype,B,T,H,dk,dv,D", [
    ("f32", 1, 64, 2, 16, 32, 64),            # float32: separate conv pass into the workspace + SIMT prefill
    ("bf16", 2, 130, 3, 64, 128, 64),
    ("bf16", 1, 333, 12, 96, 256, 1536),
    ("bf16", 2, 65, 2, 128, 256, 128),
    ("bf16", 3, 2, 2, 96, 128, 64),           # shorter than the conv window: the history carries through
    ("bf16", 2, 1553, 2, 96, 256, 64),        # sequence-parallel segments: conv halos at segment starts
    ("bf16", 2, 100, 3, 48, 64, 64),          # dk off the tensor-core path
])
@pytest.mark.parametrize("hist,s0", [(False, False), (True, True)])
def test_jetblock_prefill_matches_oracle(orc, dtype, B, T, H, dk, dv, D, hist, s0):
    s = shape(dtype, B=B, T=T, H=H, dk=dk, dv=dv, D=D)
    inp = synth.prefill_inputs(s, seed=T + 7, gate_scale=0.01 if T > 1000 else 1.0, s0_std=0.2 if s0 else None)
    d = gpu_inputs(inp)
    ref = to_oracle(inp)
    hin_np = synth.jetblock._draw(np.random.default_rng(6), (B, 3, H, dv), dtype) if hist else None
    hin = dev(hin_np, dtype) if hist else None
    hout = torch.full((B, 3, H, dv), float("nan"), device="cuda", dtype=d["v"].dtype)
    o = nan_like(d["v"])
    S_out = torch.full((B, H, dv, dk), float("nan"), device="cuda")
    jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"], hin, hout,
                             d.get("S0"), o, S_out)
    r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"],
                             inp["S0"].astype(np.float64) if s0 else None,
                             synth.to_f64(hin_np, dtype) if hist else None)
    assert_close(host64(o), r["o"], dtype, "o")
    assert_close(host64(S_out), r["S"], dtype, "S")
    np.testing.assert_array_equal(host64(hout), r["hist"])       # raw V: bit-exact


@pytest.mark.parametrize("B,T,H,dk,dv,D,hist,s0", [
    (1, 4096, 12, 96, 256, 1536, False, False),   # the 2B prompt shape
    (2, 1553, 2, 96, 256, 64, True, True),
    (2, 130, 3, 64, 128, 64, True, False),
    (1, 777, 2, 128, 256, 128, False, True),
])
def test_jetblock_prefill_agrees_with_the_two_calls(B, T, H, dk, dv, D, hist, s0):
    # the one-call prefill folds the conv into each chunk's UT transform instead of
    # rounding v' to bf16, so it agrees with the two-call path to bf16 accuracy
    # (both are checked against the oracle above); the history is a copy: bit-exact
    s = shape("bf16", B=B, T=T, H=H, dk=dk, dv=dv, D=D)
    inp = synth.prefill_inputs(s, seed=T, gate_scale=0.05, s0_std=0.2 if s0 else None)
    d = gpu_inputs(inp)
    hin = dev(synth.jetblock._draw(np.random.default_rng(8), (B, 3, H, dv), "bf16"), "bf16") if hist else None
    h1 = torch.full((B, 3, H, dv), float("nan"), device="cuda", dtype=torch.bfloat16)
    h2 = h1.clone()
    vc, _ = jet.jet_dyn_conv_v(d["x"], d["W1"], d["W2"], d["v"], hin, None, h1)
    o1, S1 = jet.jet_gdn_prefill(d["q"], d["k"], vc, d["g"], d["beta"], d.get("S0"))
    o2, S2 = jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"], hin, h2,
                                      d.get("S0"))
    assert torch.equal(h1, h2)
    assert_close(host64(o2), host64(o1), "bf16", "o")
    assert_close(host64(S2), host64(S1), "bf16", "S")


def sampled_prefill_reference(orc, inp, heads, rows, block=16384):
    """Oracle outputs of chosen (head, state-row) chains over every token: the
    generator for all tokens, then conv and recurrence restricted to those
    value channels (rows of S are independent chains)."""
    dt = inp["dtype"]
    B, T, H, _ = inp["q"].shape
    W1, W2 = synth.to_f64(inp["W1"], dt), synth.to_f64(inp["W2"], dt)
    w = np.empty((B, T, H, 4))
    for t0 in range(0, T, block):
        w[:, t0:t0 + block] = orc.kernel_gen(synth.to_f64(inp["x"][:, t0:t0 + block], dt), W1, W2, H)
    out = {}
    for h in heads:
        v = synth.to_f64(inp["v"][:, :, h:h + 1, rows], dt)
        vc, _ = orc.dyn_conv(v, w[:, :, h:h + 1])
        q = synth.to_f64(inp["q"][:, :, h:h + 1], dt)
        k = synth.to_f64(inp["k"][:, :, h:h + 1], dt)
        o, S = orc.gdn_sequential(q, k, vc, inp["g"][:, :, h:h + 1], inp["beta"][:, :, h:h + 1])
        out[h] = (o[:, :, 0], S[:, 0], vc[:, :, 0])
    return out


@pytest.mark.parametrize("name", ["prefill_4b_t65536", "prefill_2b_t262144"])
def test_config_long_prefill_sampled(orc, name):
    # configs 3 and 4a through both prefill paths: the two calls (conv pass, then the GDN
    # prefill) and the one call that the benchmark and the serving loop use (conv folded
    # into the chunk images); sampled (head, row) chains over every token against the oracle
    s = synth.CONFIGS[name]
    inp = synth.prefill_inputs(s, seed=0)
    d = gpu_inputs(inp)
    heads, rows = [0, s.H - 3], [0, 1, 100, 255]
    ref = sampled_prefill_reference(orc, inp, heads, rows)
    vc, o, S, _ = run_prefill(d, s.H)
    for h in heads:
        ro, rS, rvc = ref[h]
        assert_close(host64(o[:, :, h, rows]), ro, s.dtype, f"{name} two calls o head {h}")
        assert_close(host64(S[:, h, rows]), rS, s.dtype, f"{name} two calls S head {h}")
        assert_close(host64(vc[:, :, h, rows]), rvc, s.dtype, f"{name} v' head {h}")
    del vc, o, S
    hist = torch.full((s.B, 3, s.H, s.dv), float("nan"), device="cuda", dtype=d["v"].dtype)
    o, S = jet.jet_jetblock_prefill(d["x"], d["W1"], d["W2"], d["q"], d["k"], d["v"], d["g"], d["beta"], None, hist)
    for h in heads:
        ro, rS, _ = ref[h]
        assert_close(host64(o[:, :, h, rows]), ro, s.dtype, f"{name} one call o head {h}")
        assert_close(host64(S[:, h, rows]), rS, s.dtype, f"{name} one call S head {h}")
    assert torch.equal(hist, d["v"][:, -3:])                          # raw V of the last tokens: bit-exact
    if s.steps == 0:
        return
    # config 4b: s.steps decode steps at B = 1 (generator + conv + update fused,
    # jet_jetblock_decode_step) continuing from the one-call prefill's state and history
    del o
    dec = synth.decode_inputs(s.with_(B=1), seed=1, steps=s.steps)
    dd = gpu_inputs(dec)
    ha, hb = hist, torch.empty_like(hist)
    outs = []
    for t in range(s.steps):
        ot, _ = jet.jet_jetblock_decode_step(dd["x"][t], d["W1"], d["W2"], dd["q"][t], dd["k"][t], dd["v"][t], ha, hb,
                                             dd["g"][t], dd["beta"][t], S)
        outs.append(ot)
        ha, hb = hb, ha
    o_dec = torch.stack(outs)                                           # [n, 1, H, dv]
    dt = s.dtype
    f = lambda a: synth.to_f64(a, dt)
    for h in heads:
        _, rS, _ = ref[h]
        hist_h = f(inp["v"][:, -3:, h:h + 1, rows])                    # raw V of the last three prompt tokens
        r = orc.jetblock_decode(f(dec["x"]), f(inp["W1"]), f(inp["W2"][:, 4 * h:4 * h + 4]),
                                f(dec["q"][:, :, h:h + 1]), f(dec["k"][:, :, h:h + 1]),
                                f(dec["v"][:, :, h:h + 1, rows]), dec["g"][:, :, h:h + 1],
                                dec["beta"][:, :, h:h + 1], rS[:, None], hist_h)
        assert_close(host64(o_dec[:, :, h, rows]), r["o"][:, :, 0], dt, f"4b decode o head {h}")
        assert_close(host64(S[:, h, rows]), r["S"][:, 0], dt, f"4b decode S head {h}")


def run_decode(d, steps, B, H, dv, dtype_t, fused=False):
    """Per step: generator + conv with history ping-pong (T = 1), then the GDN
    decode step updating S in place (fused: the same as one
    jet_jetblock_decode_step call). Returns outputs [n,B,H,dv], S, history."""
    S = d["S0"].clone()
    ha, hb = d["hist"].clone(), torch.empty_like(d["hist"])
    outs = []
    for t in range(steps):
        if fused:
            o, _ = jet.jet_jetblock_decode_step(d["x"][t], d["W1"], d["W2"], d["q"][t], d["k"][t], d["v"][t], ha, hb,
                                                d["g"][t], d["beta"][t], S)
        else:
            vc, _ = jet.jet_dyn_conv_v(d["x"][t][:, None], d["W1"], d["W2"], d["v"][t][:, None], ha, None, hb)
            o = jet.jet_gdn_decode_step(d["q"][t], d["k"][t], vc[:, 0], d["g"][t], d["beta"][t], S)
        outs.append(o)
        ha, hb = hb, ha
    return torch.stack(outs), S, ha


@pytest.mark.parametrize("name,steps,seqs", [
    ("decode_2b_b256", 64, [0, 37, 128, 255]),
    ("decode_4b_b1", 16, [0]), ("decode_4b_b16", 16, [0, 15]), ("decode_4b_b64", 8, [0, 63]),
    ("decode_4b_b256", 8, [5, 200]), ("decode_4b_b1024", 4, [0, 511, 1023]),
])
@pytest.mark.parametrize("fused", [False, True])
def test_config_decode_sampled(orc, name, steps, seqs, fused):
    s = synth.CONFIGS[name]
    inp = synth.decode_inputs(s, seed=0, steps=steps)
    d = gpu_inputs(inp)
    o, S, hist = run_decode(d, steps, s.B, s.H, s.dv, d["v"].dtype, fused)
    sel = lambda a: np.ascontiguousarray(a[:, seqs])
    dt = s.dtype
    r = orc.jetblock_decode(synth.to_f64(sel(inp["x"]), dt), synth.to_f64(inp["W1"], dt), synth.to_f64(inp["W2"], dt),
                            synth.to_f64(sel(inp["q"]), dt), synth.to_f64(sel(inp["k"]), dt),
                            synth.to_f64(sel(inp["v"]), dt), sel(inp["g"]), sel(inp["beta"]),
                            inp["S0"][seqs].astype(np.float64), synth.to_f64(inp["hist"][seqs], dt))
    assert_close(host64(o[:, seqs]), r["o"], dt, f"{name} o")
    assert_close(host64(S[seqs]), r["S"], dt, f"{name} S")
    np.testing.assert_array_equal(host64(hist[seqs]), r["hist"])


def test_long_prefill_then_decode_continues(orc):
    # prefill T tokens, then decode n more from its state and history = prefill of T+n
    s = shape("bf16", B=2, T=150, H=12, dk=96, dv=256, D=1536)
    n = 6
    inp = synth.prefill_inputs(s, seed=11, T=s.T + n)
    d = gpu_inputs(inp)
    head = {k: v[:, :s.T].contiguous() for k, v in d.items() if k not in ("W1", "W2")}
    head.update(W1=d["W1"], W2=d["W2"])
    _, _, S, hist = run_prefill(head, s.H, hist_out=True)
    tail = {k: v[:, s.T:].transpose(0, 1).contiguous() for k, v in d.items() if k not in ("W1", "W2")}
    tail.update(W1=d["W1"], W2=d["W2"], S0=S, hist=hist)
    o, S_end, _ = run_decode(tail, n, s.B, s.H, s.dv, d["v"].dtype)
    ref = to_oracle(inp)
    r = orc.jetblock_prefill(ref["x"], ref["W1"], ref["W2"], ref["q"], ref["k"], ref["v"], ref["g"], ref["beta"])
    assert_close(host64(o.transpose(0, 1)), r["o"][:, s.T:], "bf16", "decoded o")
    assert_close(host64(S_end), r["S"], "bf16", "S after decode")


@pytest.mark.parametrize("dtype,H,dk,dv,hist", [("bf16", 12, 96, 256, True), ("bf16", 3, 128, 64, False),
                                                ("f32", 2, 16, 32, True)])
def test_fused_decode_step_equals_the_two_calls(orc, dtype, H, dk, dv, hist):
    # jet_jetblock_decode_step = jet_dyn_conv_v (T = 1) + jet_gdn_decode_step, step after step
    s = synth.JetShape("t", B=5, T=1, H=H, dk=dk, dv=dv, D=64, dtype=dtype)
    inp = synth.decode_inputs(s, seed=11, steps=6)
    d = gpu_inputs(inp)
    if not hist:
        d["hist"] = torch.zeros_like(d["hist"])
    o1, S1, h1 = run_decode(d, 6, s.B, s.H, s.dv, d["v"].dtype, fused=False)
    o2, S2, h2 = run_decode(d, 6, s.B, s.H, s.dv, d["v"].dtype, fused=True)
    # the fused call runs the same two kernels (the update reading v' from o): equal bit for bit
    assert torch.equal(h1, h2)
    assert torch.equal(o1, o2)
    assert torch.equal(S1, S2)
    # the taps it returns are the generator's
    taps = torch.empty((s.B, s.H, 4), device="cuda")
    jet.jet_jetblock_decode_step(d["x"][0], d["W1"], d["W2"], d["q"][0], d["k"][0], d["v"][0], d["hist"],
                                 torch.empty_like(d["hist"]), d["g"][0], d["beta"][0], d["S0"].clone(), None, taps)
    ref = jet.jet_kernel_gen(d["x"][0][:, None], d["W1"], d["W2"], H=s.H)
    assert torch.equal(taps, ref[:, 0])
