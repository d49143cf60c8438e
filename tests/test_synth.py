"""The seeded input recipe: deterministic, block-drawing equals one full draw,
bf16 rounding is round-to-nearest-even, distributions as stated."""
import numpy as np
import torch

import synth
from synth import jetblock as jb


def test_bf16_rounding_matches_torch_rne():
    rng = np.random.default_rng(0)
    a = np.concatenate([rng.standard_normal(100000) * 10.0 ** rng.integers(-6, 6, 100000),
                        [0.0, -0.0, 1.0, -1.0, 1.00390625, 1.01171875, 65504.0, 3.0e38]])
    bits = synth.bf16_bits_from_f64(a)
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(bits, ref)
    back = synth.bf16_bits_to_f64(bits)
    np.testing.assert_array_equal(back, torch.from_numpy(ref.view(np.int16)).view(torch.bfloat16).double().numpy())


def test_block_draws_equal_one_draw(monkeypatch):
    shape = jb.JetShape("t", B=2, T=37, H=3, dk=16, dv=32, D=48)
    full = synth.prefill_inputs(shape, seed=3)
    monkeypatch.setattr(jb, "_BLOCK_ELEMS", 100)      # force many small blocks
    blocked = synth.prefill_inputs(shape, seed=3)
    for key in ("x", "q", "k", "v", "beta", "g", "W1", "W2"):
        np.testing.assert_array_equal(full[key], blocked[key])


def test_prefill_recipe_properties():
    shape = synth.CONFIGS["tiny_f32"].with_(T=200)
    a = synth.prefill_inputs(shape, seed=0)
    b = synth.prefill_inputs(shape, seed=0)
    for key in ("x", "q", "k", "v", "beta", "g", "W1", "W2"):
        np.testing.assert_array_equal(a[key], b[key])
    assert a["x"].dtype == np.float32 and a["g"].dtype == np.float32
    np.testing.assert_allclose(np.linalg.norm(a["q"], axis=-1), 1.0, rtol=1e-6)
    np.testing.assert_allclose(np.linalg.norm(a["k"], axis=-1), 1.0, rtol=1e-6)
    assert np.all(a["g"] < 0) and np.all((a["beta"] > 0) & (a["beta"] < 1))
    # W1 ~ N(0, 1/D): sample variance near 1/64
    assert abs(np.var(a["W1"]) * 64 - 1) < 0.15
    assert a["W2"].shape == (32, shape.H * 4)


def test_bf16_recipe_and_decode_recipe():
    shape = synth.CONFIGS["decode_2b_b256"].with_(B=4, steps=3)
    d = synth.decode_inputs(shape, seed=0)
    assert d["x"].shape == (3, 4, 1536) and d["x"].dtype == np.uint16
    assert d["q"].shape == (3, 4, 12, 96) and d["v"].shape == (3, 4, 12, 256)
    assert d["S0"].shape == (4, 12, 256, 96) and d["S0"].dtype == np.float32
    assert d["hist"].shape == (4, 3, 12, 256) and d["hist"].dtype == np.uint16
    assert abs(d["S0"].std() - 0.02) < 0.001
    qn = np.linalg.norm(synth.to_f64(d["q"], "bf16"), axis=-1)
    np.testing.assert_allclose(qn, 1.0, atol=1e-2)


def test_config_table_matches_the_stated_shapes():
    c = synth.CONFIGS
    assert (c["prefill_2b_t4096"].T, c["prefill_2b_t4096"].H, c["prefill_2b_t4096"].dk) == (4096, 12, 96)
    assert (c["prefill_4b_t65536"].T, c["prefill_4b_t65536"].H, c["prefill_4b_t65536"].dk) == (65536, 16, 128)
    assert c["decode_2b_b256"].B == 256 and c["decode_2b_b256"].steps == 64
    assert c["prefill_2b_t262144"].T == 262144 and c["prefill_2b_t262144"].steps == 256
    for b in (1, 16, 64, 256, 1024):
        assert c[f"decode_4b_b{b}"].B == b and c[f"decode_4b_b{b}"].dk == 128
    for s in c.values():
        assert s.dv == 256 or s.name == "tiny_f32"
        assert s.R == 32 and s.W == 4


def test_spread_qk_norms_rescales_rows_and_zeroes_the_chosen_ones():
    shape = synth.CONFIGS["tiny_f32"].with_(T=50, dtype="bf16")
    a = synth.prefill_inputs(shape, seed=2)
    k = synth.spread_qk_norms(a["k"], "bf16", seed=2, zero_rows=[(0, 7, 1)])
    assert k.dtype == np.uint16 and k.shape == a["k"].shape
    n = np.linalg.norm(synth.to_f64(k, "bf16"), axis=-1)
    assert n[0, 7, 1] == 0.0
    rest = np.delete(n.ravel(), np.ravel_multi_index((0, 7, 1), n.shape))
    assert rest.min() > 0.09 and rest.max() < 11.0              # 10**U(-1, 1) times a unit row
    assert rest.min() < 0.2 and rest.max() > 5.0                # the range is actually spanned
    # its own stream: the same seed gives the same rows, and the main draw is untouched
    np.testing.assert_array_equal(k, synth.spread_qk_norms(a["k"], "bf16", seed=2, zero_rows=[(0, 7, 1)]))
    np.testing.assert_array_equal(a["k"], synth.prefill_inputs(shape, seed=2)["k"])
