"""Pins of the float64 oracle of the JetBlock layer around the mixer
(oracle/layer.py). The pages give no form for the projections, the gates or
the output (Jet-Nemotron paper, section 2.4), so the layer is our reading;
these pins fix its arithmetic against closed forms, hand-worked values and
invariances, and a set of planted mistakes must each fail one of them."""
import numpy as np
import pytest

from oracle import get as get_oracle
from oracle import layer as L


def hand_output_case():
    """Two heads of four channels; every value is worked out by hand:
    head 0: o = (3, 4, 0, 0), mean o^2 = 6.25, rms = 2.5; gamma = (1, 0.5, 2, 1)
            r = (1.2, 0.8, 0, 0); z = (40, 40, -40, 0): SiLU = (40, 40, ~0, 0)
            u = (48, 32, 0, 0), sum 80
    head 1: o = (1, -1, 1, -1), rms = 1; r = (1, -0.5, 2, -1)
            z = (0, -40, 40, 40): SiLU = (0, ~0, 40, 40); u = (0, ~0, 80, -40), sum 40
    Wo sums head 0 into y_0 and head 1 into y_1: y = (80, 40), up to the eps
    under the square root (a relative shift below 1e-6)."""
    o = np.array([[3.0, 4.0, 0.0, 0.0], [1.0, -1.0, 1.0, -1.0]])
    z = np.array([[40.0, 40.0, -40.0, 0.0], [0.0, -40.0, 40.0, 40.0]])
    gamma = np.array([1.0, 0.5, 2.0, 1.0])
    Wo = np.zeros((8, 2))
    Wo[0:4, 0] = 1.0
    Wo[4:8, 1] = 1.0
    return o, z, gamma, Wo


def test_output_stage_hand_worked():
    o, z, gamma, Wo = hand_output_case()
    np.testing.assert_allclose(L.output(o, z, gamma, Wo), [80.0, 40.0], atol=1e-4)


def test_output_stage_of_a_zero_head_is_zero_not_nan():
    # the eps sits under the square root: an all-zero head gives r = 0
    o, z, gamma, Wo = hand_output_case()
    o[1] = 0.0
    np.testing.assert_allclose(L.output(o, z, gamma, Wo), [80.0, 0.0], atol=1e-4)


def test_closed_forms_of_the_gates_and_projections():
    rng = np.random.default_rng(0)
    H, dk, dv, D = 2, 3, 4, 2 * 3 + 2 * 4
    x = rng.standard_normal((5, D))
    sel = lambda a, n: np.eye(D)[:, a:a + n]                     # picks x[..., a:a+n]
    Wg = np.zeros((D, H))
    Wb = np.zeros((D, H))
    Wb[0, 1] = 1.0                                               # b of head 1 = sigmoid(x_0)
    Wg[1, 0] = 1.0                                               # g of head 0 = -softplus(x_1)
    q, k, v, z, g, b = L.projections(x, sel(0, H * dk), sel(H * dk, H * dk), sel(0, H * dv), Wg, Wb,
                                     sel(2, H * dv), H)
    np.testing.assert_array_equal(q, x[:, :6].reshape(5, H, dk))
    np.testing.assert_array_equal(k, x[:, 6:12].reshape(5, H, dk))
    np.testing.assert_array_equal(v, x[:, :8].reshape(5, H, dv))
    np.testing.assert_array_equal(z, x[:, 2:10].reshape(5, H, dv))
    np.testing.assert_allclose(g[:, 1], -np.log(2.0), rtol=1e-15)               # zero logits
    np.testing.assert_allclose(b[:, 0], 0.5, rtol=1e-15)
    np.testing.assert_allclose(g[:, 0], -np.log1p(np.exp(x[:, 1])), rtol=1e-13)
    np.testing.assert_allclose(b[:, 1], 1.0 / (1.0 + np.exp(-x[:, 0])), rtol=1e-13)
    assert np.all(g <= 0) and np.all((b > 0) & (b < 1))


def layer_inputs(seed, B=1, T=70, D=24, H=2, dk=8, dv=8):
    rng = np.random.default_rng(seed)
    w = lambda *s: rng.standard_normal(s) / np.sqrt(s[0])
    return dict(x=rng.standard_normal((B, T, D)), Wq=w(D, H * dk), Wk=w(D, H * dk), Wv=w(D, H * dv), Wg=w(D, H),
                Wb=w(D, H), Wz=w(D, H * dv), Wo=w(H * dv, D), gamma=1.0 + 0.1 * rng.standard_normal(dv),
                W1=w(D, 32), W2=w(32, H * 4))


def run(orc, d, **kw):
    a = dict(d, **kw)
    return L.layer_prefill(orc, a["x"], a["Wq"], a["Wk"], a["Wv"], a["Wg"], a["Wb"], a["Wz"], a["Wo"], a["gamma"],
                           a["W1"], a["W2"])


def test_zero_gate_weights_give_a_zero_output():
    d = layer_inputs(1)
    y = run(get_oracle(), d, Wz=np.zeros_like(d["Wz"]))["y"]
    assert np.all(y == 0.0)


def test_output_does_not_depend_on_the_scale_of_v():
    # from a zero state the mixer's outputs are linear in v; the per-head norm removes the scale
    orc = get_oracle()
    d = layer_inputs(2)
    # (values large enough that the eps under the square root is negligible: mean o^2 >= 3)
    y1 = run(orc, d, Wv=1e3 * d["Wv"])["y"]
    y2 = run(orc, d, Wv=7e3 * d["Wv"])["y"]
    np.testing.assert_allclose(y2, y1, rtol=1e-5, atol=1e-9)


def test_decode_steps_continue_the_prefill():
    # the layer over T tokens equals the layer over T - 3 tokens followed by 3 decode steps
    orc = get_oracle()
    d = layer_inputs(3)
    full = run(orc, d)
    a = dict(d, x=d["x"][:, :-3])
    head = L.layer_prefill(orc, a["x"], d["Wq"], d["Wk"], d["Wv"], d["Wg"], d["Wb"], d["Wz"], d["Wo"], d["gamma"],
                           d["W1"], d["W2"])
    xs = np.transpose(d["x"][:, -3:], (1, 0, 2))                         # [n, B, D]
    tail = L.layer_decode(orc, xs, d["Wq"], d["Wk"], d["Wv"], d["Wg"], d["Wb"], d["Wz"], d["Wo"], d["gamma"],
                          d["W1"], d["W2"], head["S"], head["hist"])
    np.testing.assert_allclose(np.transpose(tail["y"], (1, 0, 2)), full["y"][:, -3:], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(tail["S"], full["S"], rtol=1e-9, atol=1e-11)


# ---- planted mistakes: each must fail at least one pin above
def _mut_norm_over_heads(o, z, gamma, Wo, eps=L.RMS_EPS, interface=None):
    r = o / np.sqrt(np.mean(o * o, axis=-2, keepdims=True) + eps) * gamma
    return (r * L.silu(z)).reshape(o.shape[:-2] + (-1,)) @ Wo


def _mut_gamma_before_norm(o, z, gamma, Wo, eps=L.RMS_EPS, interface=None):
    og = o * gamma
    r = og / np.sqrt(np.mean(og * og, axis=-1, keepdims=True) + eps)
    return (r * L.silu(z)).reshape(o.shape[:-2] + (-1,)) @ Wo


def _mut_no_silu(o, z, gamma, Wo, eps=L.RMS_EPS, interface=None):
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * gamma
    return (r * z).reshape(o.shape[:-2] + (-1,)) @ Wo


def _mut_no_norm(o, z, gamma, Wo, eps=L.RMS_EPS, interface=None):
    return (o * gamma * L.silu(z)).reshape(o.shape[:-2] + (-1,)) @ Wo


def _mut_eps_outside(o, z, gamma, Wo, eps=L.RMS_EPS, interface=None):
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True)) * gamma
    return (r * L.silu(z)).reshape(o.shape[:-2] + (-1,)) @ Wo


@pytest.mark.parametrize("mutant", [_mut_norm_over_heads, _mut_gamma_before_norm, _mut_no_silu, _mut_no_norm,
                                    _mut_eps_outside])
def test_a_planted_output_mistake_fails_a_pin(monkeypatch, mutant):
    monkeypatch.setattr(L, "output", mutant)
    failed = False
    for pin in (test_output_stage_hand_worked, test_output_stage_of_a_zero_head_is_zero_not_nan,
                test_output_does_not_depend_on_the_scale_of_v):
        try:
            with np.errstate(all="ignore"):
                pin()
        except AssertionError:
            failed = True
    assert failed


@pytest.mark.parametrize("which", ["g_sign", "b_as_softplus", "swap_qk"])
def test_a_planted_projection_mistake_fails_a_pin(monkeypatch, which):
    good = L.projections

    def bad(x, Wq, Wk, Wv, Wg, Wb, Wz, H, interface=None):
        q, k, v, z, g, b = good(x, Wq, Wk, Wv, Wg, Wb, Wz, H, interface)
        if which == "g_sign":
            g = -g
        elif which == "b_as_softplus":
            b = L.softplus(x @ Wb)
        else:
            q, k = k, q
        return q, k, v, z, g, b
    monkeypatch.setattr(L, "projections", bad)
    with pytest.raises(AssertionError):
        test_closed_forms_of_the_gates_and_projections()


def test_bf16_rounding_of_the_interfaces():
    # round to nearest even at bf16 (8 significand bits): exact values stay, halfway cases go to even
    # spacing 512 at 2^16: 65536 + 256 is halfway to an odd neighbour (stays), + 768 halfway to an even one
    np.testing.assert_array_equal(L.bf16(np.array([1.0, -2.5, 0.0, 65536 + 256, 65536 + 768])),
                                  [1.0, -2.5, 0.0, 65536, 65536 + 1024])
    np.testing.assert_array_equal(L.bf16(np.array([1 + 2 ** -8, 1 + 3 * 2 ** -8, 1 + 2 ** -7])),
                                  [1.0, 1 + 2 ** -6, 1 + 2 ** -7])
    np.testing.assert_array_equal(L.bf16(np.array([1 + 2 ** -8 + 2 ** -20])), [1 + 2 ** -7])
