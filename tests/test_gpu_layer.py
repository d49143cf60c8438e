"""GPU: the JetBlock layer around the mixer (jet_jetblock_layer) against the
float64 oracle of the same layer (oracle/layer.py): projections on cuBLAS,
gates, the mixer, per-head RMSNorm with the SiLU output gate, output
projection. Prefill with and without an initial state and history, and
decode steps (T = 1) advancing the state in place."""
import numpy as np
import pytest
import torch

import synth
from jet_testlib import assert_close, dev, host64
from oracle import get as get_oracle
from oracle import layer as olayer

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


def assert_layer_close(y, r, what="y"):
    """y against the oracle's layer with its stage interfaces rounded as the layer stores them (q, k, v, z,
    o and the gated output in bf16, the gate logits in float32): the bf16 bound of the mixer (rel-L2
    <= 1e-2, max-abs <= 5e-2) over every token. Against the unrounded oracle the bound would not hold
    for the few tokens whose mixer output is near zero, where the per-head RMSNorm magnifies the bf16
    rounding of q, k and v."""
    assert_close(y, r["y"], "bf16", what)


def assert_hist(h, ref):
    """The new history is raw v = x Wv rounded to bf16. The GPU rounds its float32-accumulated GEMM result,
    the oracle its float64 product: where the two sums fall on either side of a rounding boundary the
    stored values differ by one bf16 step (2^-7 relative at most), and where the sum cancels to a value
    far below its terms, by the float32 accumulation error of D terms of size about 1 / sqrt(D)
    (D 2^-24 / sqrt(D) < 1e-5 absolute for D <= 2048, against values of size 1); everywhere else they
    are equal."""
    np.testing.assert_allclose(h, ref, rtol=2.0 ** -7, atol=1e-5)
    assert np.mean(h != ref) < 1e-2


def layer_weights(seed, D, H, dk, dv):
    """bf16 weights ~ N(0, 1/fan_in), gamma = 1 + 0.1 N(0, 1) float32, and the generator's."""
    rng = np.random.default_rng(seed)
    bf = lambda *shape: synth.jetblock._draw(rng, shape, "bf16", scale=1.0 / np.sqrt(shape[0]))
    w = dict(Wq=bf(D, H * dk), Wk=bf(D, H * dk), Wv=bf(D, H * dv), Wg=bf(D, H), Wb=bf(D, H), Wz=bf(D, H * dv),
             Wo=bf(H * dv, D), W1=bf(D, 32), W2=bf(32, H * 4))
    w["gamma"] = (1.0 + 0.1 * rng.standard_normal(dv)).astype(np.float32)
    return w


ORDER = ("Wq", "Wk", "Wv", "Wg", "Wb", "Wz", "Wo", "gamma", "W1", "W2")


def f64(w):
    return {k: (synth.to_f64(v, "bf16") if v.dtype == np.uint16 else v.astype(np.float64)) for k, v in w.items()}


def gpu(w):
    return {k: dev(v, "bf16" if v.dtype == np.uint16 else "f32") for k, v in w.items()}


@pytest.mark.parametrize("B,T,D,H,dk,dv", [(2, 150, 64, 2, 64, 128), (1, 300, 1536, 12, 96, 256),
                                          (1, 200, 256, 2, 128, 256)])
@pytest.mark.parametrize("state", [False, True])
def test_layer_prefill_matches_the_oracle(B, T, D, H, dk, dv, state):
    w = layer_weights(B * 1000 + T, D, H, dk, dv)
    rng = np.random.default_rng(T)
    x = synth.jetblock._draw(rng, (B, T, D), "bf16")
    S0 = synth.jetblock._draw(rng, (B, H, dv, dk), "f32", scale=0.2) if state else None
    hist = synth.jetblock._draw(rng, (B, 3, H, dv), "bf16") if state else None
    g = gpu(w)
    hout = torch.full((B, 3, H, dv), float("nan"), device="cuda", dtype=torch.bfloat16)
    y, S = jet.jet_jetblock_layer(dev(x, "bf16"), *[g[k] for k in ORDER],
                                  hist_in=dev(hist, "bf16") if state else None, hist_out=hout,
                                  S0=dev(S0, "f32") if state else None)
    assert jet.jet_device_error() == 0
    f = f64(w)
    r = olayer.layer_prefill(get_oracle(), synth.to_f64(x, "bf16"), *[f[k] for k in ORDER],
                             S0=S0.astype(np.float64) if state else None,
                             hist=synth.to_f64(hist, "bf16") if state else None, interface="bf16")
    assert_layer_close(host64(y), r)
    assert_close(host64(S), r["S"], "bf16", "S")
    assert_hist(host64(hout), r["hist"])


@pytest.mark.parametrize("B,D,H,dk,dv", [(4, 128, 2, 128, 256), (3, 1536, 12, 96, 256)])
def test_layer_decode_steps_match_the_oracle(B, D, H, dk, dv):
    n = 3
    w = layer_weights(7 + B, D, H, dk, dv)
    rng = np.random.default_rng(B)
    x = synth.jetblock._draw(rng, (n, B, D), "bf16")
    S0 = synth.jetblock._draw(rng, (B, H, dv, dk), "f32", scale=0.02)
    hist = synth.jetblock._draw(rng, (B, 3, H, dv), "bf16")
    g = gpu(w)
    S = dev(S0, "f32")
    hs = [dev(hist, "bf16"), torch.empty((B, 3, H, dv), device="cuda", dtype=torch.bfloat16)]
    ys = []
    for t in range(n):
        y, _ = jet.jet_jetblock_layer(dev(x[t], "bf16")[:, None], *[g[k] for k in ORDER], hist_in=hs[t % 2],
                                      hist_out=hs[(t + 1) % 2], S0=S, S_out=S)     # the state advances in place
        ys.append(host64(y[:, 0]))
    assert jet.jet_device_error() == 0
    f = f64(w)
    r = olayer.layer_decode(get_oracle(), synth.to_f64(x, "bf16"), *[f[k] for k in ORDER], S0.astype(np.float64),
                            synth.to_f64(hist, "bf16"), interface="bf16")
    assert_layer_close(np.stack(ys), r)
    assert_close(host64(S), r["S"], "bf16", "S")
    assert_hist(host64(hs[n % 2]), r["hist"])
