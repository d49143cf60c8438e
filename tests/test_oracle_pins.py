"""Pins of the float64 oracle against things other than itself.

Each test checks the oracle against a closed form, a hand-worked example
(tests/golden/hand_worked.json), an identity named by the method (Jet-Nemotron
paper section 2.3 / 2.4), or an independent brute-force form (explicit
transition-matrix products, oracle/brute.py). Chosen so that a dropped term, a
wrong sign, a wrong index or a transposed operand in the oracle fails one.
"""
import json
import os

import numpy as np
import pytest

from oracle import brute, get as get_oracle

GOLD = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "hand_worked.json")))


@pytest.fixture(scope="module")
def orc():
    return get_oracle()


def rnd(seed):
    return np.random.default_rng(seed)


def unit(a):
    return a / np.linalg.norm(a, axis=-1, keepdims=True)


def gdn_inputs(rng, B=1, T=8, H=2, dk=4, dv=3, s0=True, long_memory=False):
    q = unit(rng.standard_normal((B, T, H, dk)))
    k = unit(rng.standard_normal((B, T, H, dk)))
    v = rng.standard_normal((B, T, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, H))))
    g = -np.logaddexp(0, rng.standard_normal((B, T, H))) * (0.01 if long_memory else 1.0)
    S0 = rng.standard_normal((B, H, dv, dk)) * 0.5 if s0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- generator
def test_generator_hand_worked(orc):
    c = GOLD["generator"]
    w = orc.kernel_gen(np.array([c["x"]]), np.array(c["W1"]), np.array(c["W2"]), H=1, W=2)
    np.testing.assert_allclose(w.reshape(-1), c["w"], rtol=1e-14, atol=1e-14)


def test_generator_zero_input_gives_zero_taps(orc):
    rng = rnd(1)
    W1, W2 = rng.standard_normal((64, 32)), rng.standard_normal((32, 8))
    w = orc.kernel_gen(np.zeros((5, 64)), W1, W2, H=2, W=4)
    assert np.all(w == 0.0)


def test_generator_silu_closed_form_and_selection(orc):
    # W1 routes x[d] into hidden unit r = perm[d]; W2 routes hidden unit r to
    # column c = sel[r]. Then w[c] = SiLU(x[d]) with SiLU(z) = z / (1 + e^-z).
    D, R, H, W = 5, 32, 2, 4
    z = np.array([0.0, 1.0, -2.5, 30.0, -30.0])
    W1 = np.zeros((D, R))
    perm = [7, 3, 30, 0, 12]
    for d, r in enumerate(perm):
        W1[d, r] = 1.0
    W2 = np.zeros((R, H * W))
    sel = {7: 5, 3: 0, 30: 7, 0: 2, 12: 3}
    for r, c in sel.items():
        W2[r, c] = 1.0
    w = orc.kernel_gen(z[None], W1, W2, H=H, W=W).reshape(-1)
    expect = np.zeros(H * W)
    for d, r in enumerate(perm):
        expect[sel[r]] = z[d] / (1 + np.exp(-z[d]))
    np.testing.assert_allclose(w, expect, rtol=1e-15, atol=1e-300)
    assert w[0] == 1.0 / (1 + np.exp(-1.0))            # SiLU(1) = sigmoid(1)
    assert abs(w[2] - 30.0) < 1e-11                     # SiLU(30) ~ 30
    assert -1e-11 < w[3] < 0.0                          # SiLU(-30) ~ -30 e^-30


def test_generator_linear_in_W2_and_nonlinear_in_x(orc):
    rng = rnd(2)
    x = rng.standard_normal((3, 16))
    W1 = rng.standard_normal((16, 32)) / 4
    A, Bm = rng.standard_normal((32, 8)), rng.standard_normal((32, 8))
    wa, wb = orc.kernel_gen(x, W1, A, 2), orc.kernel_gen(x, W1, Bm, 2)
    np.testing.assert_allclose(orc.kernel_gen(x, W1, A + Bm, 2), wa + wb, rtol=1e-12, atol=1e-12)
    # SiLU is not odd: w(-x) != -w(x)
    assert not np.allclose(orc.kernel_gen(-x, W1, A, 2), -wa)


# --------------------------------------------------------------------- conv
def test_conv_hand_worked(orc):
    c = GOLD["conv"]
    v = np.array(c["v"]).reshape(1, 3, 1, 1)
    w = np.array(c["w"]).reshape(1, 3, 1, 4)
    hist = np.array(c["hist"]).reshape(1, 3, 1, 1)
    out, hout = orc.dyn_conv(v, w, hist)
    np.testing.assert_array_equal(out.reshape(-1), c["out_with_hist"])
    np.testing.assert_array_equal(hout.reshape(-1), c["hist_out"])
    out0, _ = orc.dyn_conv(v, w, None)
    np.testing.assert_array_equal(out0.reshape(-1), c["out_no_hist"])


@pytest.mark.parametrize("tap", [0, 1, 2, 3])
def test_conv_unit_tap_is_shift(orc, tap):
    # taps e_0 = [1,0,0,0] is the identity on V; e_j shifts by j with zero fill
    rng = rnd(3)
    B, T, H, dv = 2, 9, 3, 5
    v = rng.standard_normal((B, T, H, dv))
    w = np.zeros((B, T, H, 4))
    w[..., tap] = 1.0
    out, _ = orc.dyn_conv(v, w, None)
    expect = np.zeros_like(v)
    expect[:, tap:] = v[:, : T - tap]
    np.testing.assert_array_equal(out, expect)


def test_conv_per_head_taps_and_linearity(orc):
    rng = rnd(4)
    B, T, H, dv = 1, 7, 2, 4
    v1, v2 = rng.standard_normal((2, B, T, H, dv))
    w = rng.standard_normal((B, T, H, 4))
    o1, _ = orc.dyn_conv(v1, w)
    o2, _ = orc.dyn_conv(v2, w)
    o12, _ = orc.dyn_conv(2 * v1 - 3 * v2, w)
    np.testing.assert_allclose(o12, 2 * o1 - 3 * o2, rtol=1e-12, atol=1e-12)
    # head 1's taps do not touch head 0
    w2 = w.copy()
    w2[:, :, 1] = 7.0
    o3, _ = orc.dyn_conv(v1, w2)
    np.testing.assert_array_equal(o3[:, :, 0], o1[:, :, 0])


@pytest.mark.parametrize("split", [1, 2, 3, 5])
def test_conv_history_continuation(orc, split):
    rng = rnd(5)
    B, T, H, dv = 2, 8, 2, 3
    v = rng.standard_normal((B, T, H, dv))
    w = rng.standard_normal((B, T, H, 4))
    hist0 = rng.standard_normal((B, 3, H, dv))
    full, hfull = orc.dyn_conv(v, w, hist0)
    a, ha = orc.dyn_conv(v[:, :split], w[:, :split], hist0)
    b, hb = orc.dyn_conv(v[:, split:], w[:, split:], ha)
    np.testing.assert_array_equal(np.concatenate([a, b], axis=1), full)
    np.testing.assert_array_equal(hb, hfull)
    np.testing.assert_array_equal(hfull, v[:, T - 3:])


# ---------------------------------------------------------------------- GDN
def test_gdn_hand_worked(orc):
    c = GOLD["gdn"]
    q = np.array(c["q"]).reshape(1, 2, 1, 2)
    k = np.array(c["k"]).reshape(1, 2, 1, 2)
    v = np.array(c["v"]).reshape(1, 2, 1, 1)
    g = np.array(c["g"]).reshape(1, 2, 1)
    beta = np.array(c["beta"]).reshape(1, 2, 1)
    for fn in (orc.gdn_sequential, orc.gdn_chunked):
        o, S = fn(q, k, v, g, beta)
        np.testing.assert_allclose(o.reshape(-1), c["o"], rtol=1e-5)
        np.testing.assert_allclose(S.reshape(1, 2), c["S"], rtol=1e-5)
    S = np.zeros((1, 1, 1, 2))
    outs = []
    for t in range(2):
        o, S = orc.gdn_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        outs.append(o.item())
    np.testing.assert_allclose(outs, c["o"], rtol=1e-5)


@pytest.mark.parametrize("seed,s0", [(0, False), (1, True), (2, True)])
def test_gdn_sequential_equals_transition_products(orc, seed, s0):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(seed), B=2, T=11, H=2, dk=5, dv=3, s0=s0)
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    ob, Sb = brute.gdn_transition_products(q, k, v, g, beta, S0)
    np.testing.assert_allclose(o, ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, Sb, rtol=1e-11, atol=1e-12)


def test_gdn_alpha1_beta0_leaves_state(orc):
    q, k, v, _, _, S0 = gdn_inputs(rnd(6), T=9)
    z = np.zeros(q.shape[:3])
    o, S = orc.gdn_sequential(q, k, v, z, z, S0)
    np.testing.assert_array_equal(S, S0)
    qh = q / np.sqrt(np.sum(q * q, -1, keepdims=True) + 1e-6)
    np.testing.assert_allclose(o, np.einsum("bhij,bthj->bthi", S0, qh), rtol=1e-13, atol=1e-14)


def test_gdn_orthonormal_keys_store_values_exactly(orc):
    rng = rnd(7)
    dk, dv, T = 6, 4, 6
    Q, _ = np.linalg.qr(rng.standard_normal((dk, dk)))
    keys = Q.T[:T]                                   # orthonormal rows
    k = keys.reshape(1, T, 1, dk)
    v = rng.standard_normal((1, T, 1, dv))
    one = np.ones((1, T, 1))
    for fn in (orc.gdn_sequential, orc.gdn_chunked):
        o, S = fn(k, k, v, 0 * one, one)
        khat = keys / np.sqrt(1 + 1e-6)
        # S k_j = v_j for every stored key (eps shifts norms by 1e-6)
        np.testing.assert_allclose(S[0, 0] @ khat.T, v[0, :, 0].T, rtol=3e-6, atol=3e-6)
        # querying with k_j right after storing it returns v_j
        np.testing.assert_allclose(o[0, :, 0], v[0, :, 0], rtol=3e-6, atol=3e-6)


def test_gdn_beta0_decays_state(orc):
    q, k, v, g, _, S0 = gdn_inputs(rnd(8), T=10)
    o, S = orc.gdn_sequential(q, k, v, g, np.zeros_like(g), S0)
    decay = np.exp(g.sum(axis=1))                    # [B,H]
    np.testing.assert_allclose(S, S0 * decay[..., None, None], rtol=1e-13, atol=1e-15)


def test_gdn_delta_rule_overwrites(orc):
    rng = rnd(9)
    dk, dv = 5, 3
    kk = unit(rng.standard_normal(dk))
    k = np.stack([kk, kk]).reshape(1, 2, 1, dk)
    v = rng.standard_normal((1, 2, 1, dv))
    one = np.ones((1, 2, 1))
    _, S = orc.gdn_sequential(k, k, v, 0 * one, one)
    np.testing.assert_allclose(S[0, 0] @ (kk / np.sqrt(1 + 1e-6)), v[0, 1, 0], rtol=1e-5, atol=1e-5)


def test_gdn_joint_linearity_in_state_and_values(orc):
    rng = rnd(10)
    q, k, va, g, beta, Sa = gdn_inputs(rng, T=12)
    vb, Sb = rng.standard_normal(va.shape), rng.standard_normal(Sa.shape)
    oa, SA = orc.gdn_sequential(q, k, va, g, beta, Sa)
    ob, SB = orc.gdn_sequential(q, k, vb, g, beta, Sb)
    oc, SC = orc.gdn_sequential(q, k, 2 * va - vb, g, beta, 2 * Sa - Sb)
    np.testing.assert_allclose(oc, 2 * oa - ob, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(SC, 2 * SA - SB, rtol=1e-11, atol=1e-12)


def test_gdn_value_channel_permutation(orc):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(11), T=7, dv=5)
    perm = np.array([3, 0, 4, 1, 2])
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    op, Sp = orc.gdn_sequential(q, k, v[..., perm], g, beta, S0[:, :, perm])
    np.testing.assert_array_equal(op, o[..., perm])
    np.testing.assert_array_equal(Sp, S[:, :, perm])


@pytest.mark.parametrize("T,C", [(1, 64), (63, 64), (64, 64), (65, 64), (130, 64), (37, 8)])
@pytest.mark.parametrize("long_memory", [False, True])
def test_gdn_chunked_equals_sequential(orc, T, C, long_memory):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(T), B=2, T=T, H=2, dk=16, dv=8, long_memory=long_memory)
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    oc, Sc = orc.gdn_chunked(q, k, v, g, beta, S0, C=C)
    np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(Sc, S, rtol=1e-10, atol=1e-12)


def test_gdn_chunked_survives_deep_gate_underflow(orc):
    # cumulative log gates far below -745 within one chunk: exp(G) underflows
    q, k, v, g, beta, S0 = gdn_inputs(rnd(12), T=64, dk=8, dv=4)
    g = g * 0 - 30.0
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    oc, Sc = orc.gdn_chunked(q, k, v, g, beta, S0)
    assert np.all(np.isfinite(oc)) and np.all(np.isfinite(Sc))
    np.testing.assert_allclose(oc, o, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(Sc, S, rtol=1e-10, atol=1e-12)


def test_gdn_decode_steps_equal_sequential(orc):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(13), B=3, T=6, H=2, dk=8, dv=4)
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    St = S0.copy()
    for t in range(6):
        ot, St = orc.gdn_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], St)
        np.testing.assert_allclose(ot, o[:, t], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(St, S, rtol=1e-12, atol=1e-13)


def test_gdn_contraction_bound(orc):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(14), T=20, dk=6, dv=4)
    S = S0.copy()
    for t in range(20):
        prev = np.linalg.norm(S[0, 0], 2)
        _, S = orc.gdn_decode_step(q[:, t], k[:, t], v[:, t], g[:, t], beta[:, t], S)
        bound = np.exp(g[0, t, 0]) * prev + beta[0, t, 0] * np.linalg.norm(v[0, t, 0])
        assert np.linalg.norm(S[0, 0], 2) <= bound * (1 + 1e-12)


def test_gdn_l2_normalises_q_and_k(orc):
    q, k, v, g, beta, S0 = gdn_inputs(rnd(15), T=9)
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    o2, S2 = orc.gdn_sequential(3.0 * q, 0.5 * k, v, g, beta, S0)  # eps 1e-6 moves norms by ~4e-6
    np.testing.assert_allclose(o2, o, rtol=1e-4, atol=2e-5)
    np.testing.assert_allclose(S2, S, rtol=1e-4, atol=2e-5)
    # without the normalisation a 3x query would triple the output
    assert np.abs(o2).max() < 2 * np.abs(o).max()


# ----------------------------------------------------------- whole mixer
def test_mixer_prefill_then_decode_continues(orc):
    rng = rnd(16)
    B, T, n, H, dk, dv, D = 2, 10, 4, 2, 8, 6, 12
    x = rng.standard_normal((B, T + n, D))
    q, k = unit(rng.standard_normal((2, B, T + n, H, dk)))
    v = rng.standard_normal((B, T + n, H, dv))
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T + n, H))))
    g = -np.logaddexp(0, rng.standard_normal((B, T + n, H)))
    W1, W2 = rng.standard_normal((D, 32)) / 4, rng.standard_normal((32, H * 4)) / 6
    full = orc.jetblock_prefill(x, W1, W2, q, k, v, g, beta)
    pre = orc.jetblock_prefill(x[:, :T], W1, W2, q[:, :T], k[:, :T], v[:, :T], g[:, :T], beta[:, :T])
    sw = lambda a: np.swapaxes(a[:, T:], 0, 1)       # [B,n,...] -> [n,B,...]
    dec = orc.jetblock_decode(sw(x), W1, W2, sw(q), sw(k), sw(v), sw(g), sw(beta), pre["S"], pre["hist"])
    np.testing.assert_allclose(np.swapaxes(dec["o"], 0, 1), full["o"][:, T:], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(dec["S"], full["S"], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(dec["hist"], full["hist"])
    # the conv output of the prefill part is the conv of the first T tokens
    np.testing.assert_allclose(pre["v_conv"], full["v_conv"][:, :T], rtol=1e-14)


def test_mixer_identity_taps_reduce_to_plain_gdn(orc):
    # Generator whose taps are exactly [1,0,0,0] (W1 = 0 gives h = 0, so use a
    # bias-free route: x = 0, then taps are 0). Instead force taps through the
    # conv stage directly: conv with e_0 leaves V, so the mixer equals GDN(V).
    q, k, v, g, beta, S0 = gdn_inputs(rnd(17), T=9)
    w = np.zeros(v.shape[:3] + (4,))
    w[..., 0] = 1.0
    vc, _ = orc.dyn_conv(v, w)
    o1, S1 = orc.gdn_sequential(q, k, vc, g, beta, S0)
    o2, S2 = orc.gdn_sequential(q, k, v, g, beta, S0)
    np.testing.assert_array_equal(o1, o2)
    np.testing.assert_array_equal(S1, S2)


def test_gdn_l2_norm_eps_on_zero_and_tiny_vectors(orc):
    # eps sits under the square root: a zero key leaves only the decay (S_t = a_t S_{t-1}),
    # a zero query gives o_t = 0, and a key of norm 1e-3 is scaled by 1/sqrt(1e-6 + 1e-6)
    q, k, v, g, beta, S0 = gdn_inputs(rnd(18), T=3)
    k[0, 1, 0] = 0.0
    q[0, 2, 1] = 0.0
    o, S = orc.gdn_sequential(q, k, v, g, beta, S0)
    o1, S1 = orc.gdn_sequential(q[:, :1], k[:, :1], v[:, :1], g[:, :1], beta[:, :1], S0)
    o2, S2 = orc.gdn_sequential(q[:, :2], k[:, :2], v[:, :2], g[:, :2], beta[:, :2], S0)
    np.testing.assert_allclose(S2[0, 0], np.exp(g[0, 1, 0]) * S1[0, 0], rtol=1e-14, atol=0)
    np.testing.assert_array_equal(o[0, 2, 1], 0.0)
    # one token from S0 with a tiny key: u = S0 k / sqrt(|k|^2 + eps), written out by hand
    kt = k[:, :1].copy()
    kt[0, 0, 0] *= 1e-3 / np.linalg.norm(kt[0, 0, 0])
    qt = q[:, :1]
    _, St = orc.gdn_sequential(qt, kt, v[:, :1], g[:, :1], beta[:, :1], S0)
    kh = kt[0, 0, 0] / np.sqrt(1e-6 + 1e-6)
    a, b = np.exp(g[0, 0, 0]), beta[0, 0, 0]
    Sx = S0[0, 0]
    want = a * (Sx - b * np.outer(Sx @ kh, kh)) + b * np.outer(v[0, 0, 0], kh)
    np.testing.assert_allclose(St[0, 0], want, rtol=1e-12, atol=1e-14)
