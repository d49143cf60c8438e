"""GPU: the variable-length prefill (one call over prompts of different
lengths packed along the token axis) against the float64 oracle run on each
prompt alone, and against one jet_jetblock_prefill per prompt; plus the
serving loop's rounds, which now pack every live prompt into one call."""
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


def packed_inputs(lens, H, dk, dv, D, seed, gate_scale=1.0):
    """One seeded draw per prompt (prompt i: seed + i), and the packed tensors."""
    per = []
    for i, T in enumerate(lens):
        s = synth.JetShape("vl", B=1, T=T, H=H, dk=dk, dv=dv, D=D)
        per.append(synth.prefill_inputs(s, seed=seed + i, gate_scale=gate_scale, s0_std=0.2))
    W1, W2 = per[0]["W1"], per[0]["W2"]                  # one layer: the first prompt's weights for all
    packed = {key: np.concatenate([p[key][0] for p in per]) for key in ("x", "q", "k", "v", "g", "beta")}
    S0 = np.stack([p["S0"][0] for p in per])
    return per, packed, W1, W2, S0


@pytest.mark.parametrize("lens,H,dk,dv,D", [([1, 63, 300, 1553, 4096], 12, 96, 256, 1536),
                                           ([2, 64, 65, 129, 700], 3, 128, 128, 128),
                                           ([5, 130, 3000], 2, 64, 256, 64)])
@pytest.mark.parametrize("hist", [False, True])
def test_varlen_prefill_matches_the_oracle_per_prompt(lens, H, dk, dv, D, hist):
    per, packed, W1, W2, S0 = packed_inputs(lens, H, dk, dv, D, seed=90, gate_scale=0.05)
    n = len(lens)
    hin_np = synth.jetblock._draw(np.random.default_rng(7), (n, 3, H, dv), "bf16") if hist else None
    d = {key: dev(val, "bf16") for key, val in packed.items() if key not in ("g", "beta")}
    d["g"], d["beta"] = dev(packed["g"], "f32"), dev(packed["beta"], "f32")
    w1, w2 = dev(W1, "bf16"), dev(W2, "bf16")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o = torch.full_like(d["v"], float("nan"))
    S_out = torch.full((n, H, dv, dk), float("nan"), device="cuda")
    hout = torch.full((n, 3, H, dv), float("nan"), device="cuda", dtype=torch.bfloat16)
    jet.jet_jetblock_prefill_varlen(d["x"], w1, w2, d["q"], d["k"], d["v"], d["g"], d["beta"], cu,
                                    dev(hin_np, "bf16") if hist else None, hout, dev(S0, "f32"), o, S_out)
    assert jet.jet_device_error() == 0
    orc = get_oracle()
    f = lambda a: synth.to_f64(a, "bf16")
    for i, T in enumerate(lens):
        p = per[i]
        r = orc.jetblock_prefill(f(p["x"]), f(W1), f(W2), f(p["q"]), f(p["k"]), f(p["v"]), p["g"], p["beta"],
                                 p["S0"].astype(np.float64), f(hin_np[i:i + 1]) if hist else None)
        assert_close(host64(o[cu[i]:cu[i + 1]]), r["o"][0], "bf16", f"o of prompt {i} ({T} tokens)")
        assert_close(host64(S_out[i]), r["S"][0], "bf16", f"S of prompt {i}")
        np.testing.assert_array_equal(host64(hout[i]), r["hist"][0])


def test_varlen_prefill_agrees_with_one_call_per_prompt():
    lens = [40, 300, 1000]
    per, packed, W1, W2, S0 = packed_inputs(lens, 2, 96, 256, 64, seed=95)
    d = {key: dev(val, "bf16") for key, val in packed.items() if key not in ("g", "beta")}
    d["g"], d["beta"] = dev(packed["g"], "f32"), dev(packed["beta"], "f32")
    w1, w2 = dev(W1, "bf16"), dev(W2, "bf16")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    o, S = jet.jet_jetblock_prefill_varlen(d["x"], w1, w2, d["q"], d["k"], d["v"], d["g"], d["beta"], cu,
                                           S0=dev(S0, "f32"))
    for i in range(len(lens)):
        sl = lambda key: d[key][cu[i]:cu[i + 1]].unsqueeze(0).contiguous()
        o1, S1 = jet.jet_jetblock_prefill(sl("x"), w1, w2, sl("q"), sl("k"), sl("v"), sl("g"), sl("beta"),
                                          S0=dev(S0[i:i + 1], "f32"))
        assert_close(host64(o[cu[i]:cu[i + 1]]), host64(o1[0]), "bf16", f"o of prompt {i}")
        assert_close(host64(S[i]), host64(S1[0]), "bf16", f"S of prompt {i}")


def test_varlen_prefill_normalises_q_and_k():
    # q and k rows of spread norms (10**U(-1, 1)), one key row and one query row exactly zero,
    # in different prompts: every prompt must still match the oracle, which normalises in float64
    lens = [70, 1, 200]
    per, packed, W1, W2, S0 = packed_inputs(lens, 2, 96, 128, 64, seed=97)
    packed["k"] = synth.spread_qk_norms(packed["k"], "bf16", 3, zero_rows=[(75, 1)])
    packed["q"] = synth.spread_qk_norms(packed["q"], "bf16", 4, zero_rows=[(10, 0)])
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    d = {key: dev(val, "bf16") for key, val in packed.items() if key not in ("g", "beta")}
    d["g"], d["beta"] = dev(packed["g"], "f32"), dev(packed["beta"], "f32")
    o, S = jet.jet_jetblock_prefill_varlen(d["x"], dev(W1, "bf16"), dev(W2, "bf16"), d["q"], d["k"], d["v"], d["g"],
                                           d["beta"], cu, S0=dev(S0, "f32"))
    assert jet.jet_device_error() == 0
    orc = get_oracle()
    f = lambda a: synth.to_f64(a, "bf16")
    for i in range(len(lens)):
        a, b = cu[i], cu[i + 1]
        r = orc.jetblock_prefill(f(packed["x"][a:b])[None], f(W1), f(W2), f(packed["q"][a:b])[None],
                                 f(packed["k"][a:b])[None], f(packed["v"][a:b])[None], packed["g"][a:b][None],
                                 packed["beta"][a:b][None], S0[i:i + 1].astype(np.float64))
        assert_close(host64(o[a:b]), r["o"][0], "bf16", f"o of prompt {i}")
        assert_close(host64(S[i]), r["S"][0], "bf16", f"S of prompt {i}")


def test_varlen_prefill_at_the_sequence_limit():
    # 256 prompts (the most one call takes) of 1 to 300 tokens, seeded: every prompt against one
    # jet_jetblock_prefill call of its own, and a sample of them against the oracle
    rng = np.random.default_rng(5)
    lens = rng.integers(1, 301, 256).tolist()
    per, packed, W1, W2, S0 = packed_inputs(lens, 2, 64, 128, 64, seed=300, gate_scale=0.1)
    d = {key: dev(val, "bf16") for key, val in packed.items() if key not in ("g", "beta")}
    d["g"], d["beta"] = dev(packed["g"], "f32"), dev(packed["beta"], "f32")
    w1, w2 = dev(W1, "bf16"), dev(W2, "bf16")
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    hout = torch.empty((256, 3, 2, 128), device="cuda", dtype=torch.bfloat16)
    o, S = jet.jet_jetblock_prefill_varlen(d["x"], w1, w2, d["q"], d["k"], d["v"], d["g"], d["beta"], cu,
                                           hist_out=hout, S0=dev(S0, "f32"))
    assert jet.jet_device_error() == 0
    for i in range(256):
        sl = lambda key: d[key][cu[i]:cu[i + 1]].unsqueeze(0).contiguous()
        h1 = torch.empty((1, 3, 2, 128), device="cuda", dtype=torch.bfloat16)
        o1, S1 = jet.jet_jetblock_prefill(sl("x"), w1, w2, sl("q"), sl("k"), sl("v"), sl("g"), sl("beta"),
                                          hist_out=h1, S0=dev(S0[i:i + 1], "f32"))
        assert_close(host64(o[cu[i]:cu[i + 1]]), host64(o1[0]), "bf16", f"o of prompt {i}")
        assert_close(host64(S[i]), host64(S1[0]), "bf16", f"S of prompt {i}")
        assert torch.equal(hout[i], h1[0])
    orc = get_oracle()
    f = lambda a: synth.to_f64(a, "bf16")
    for i in (0, 7, 100, 255):
        p = per[i]
        r = orc.jetblock_prefill(f(p["x"]), f(W1), f(W2), f(p["q"]), f(p["k"]), f(p["v"]), p["g"], p["beta"],
                                 p["S0"].astype(np.float64))
        assert_close(host64(o[cu[i]:cu[i + 1]]), r["o"][0], "bf16", f"o of prompt {i} vs the oracle")
        assert_close(host64(S[i]), r["S"][0], "bf16", f"S of prompt {i} vs the oracle")
