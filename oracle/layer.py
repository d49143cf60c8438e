"""Float64 oracle of the JetBlock layer around the mixer.

TEST INFRASTRUCTURE ONLY (like the rest of this package): the CUDA library
never imports or calls it.

The Jet-Nemotron paper (section 2.4, new attention block design) says only
that the block takes its queries, keys, values and the generator's input
from the shared block input x, and that the dynamic conv acts on V alone
(no static conv on Q or K); it gives no form for the projections, the gates
or the output. This module fixes the plainest reading, the Gated DeltaNet
layer without its short convolutions:

  q = x Wq, k = x Wk        [D -> H dk]   (L2-normalised inside the mixer)
  v = x Wv                   [D -> H dv]   (raw: the mixer applies the dynamic conv)
  g = -softplus(x Wg)        [D -> H]      (log decay, g <= 0)
  b = sigmoid(x Wb)          [D -> H]      (write strength, 0 < b < 1)
  o = mixer(x; q, k, v, g, b)              (generator + dynamic conv + gated delta rule)
  r = o / sqrt(mean_dv(o^2) + eps) * gamma (per token and head; gamma [dv])
  y = (r * SiLU(x Wz)) Wo    [H dv -> D]   (Wz [D -> H dv])

Each matrix product is numpy's float64 matmul (a library primitive); no
intermediate is rounded. The mixer is the compiled oracle's.
"""
from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6


def silu(z):
    return z / (1.0 + np.exp(-z))


def softplus(z):
    return np.logaddexp(0.0, z)


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H: int):
    """x [..., D] -> q, k [..., H, dk], v, z [..., H, dv], g, b [..., H]."""
    lead = x.shape[:-1]
    dk = Wq.shape[1] // H
    dv = Wv.shape[1] // H
    q = (x @ Wq).reshape(lead + (H, dk))
    k = (x @ Wk).reshape(lead + (H, dk))
    v = (x @ Wv).reshape(lead + (H, dv))
    z = (x @ Wz).reshape(lead + (H, dv))
    g = -softplus(x @ Wg)
    b = sigmoid(x @ Wb)
    return q, k, v, z, g, b


def output(o, z, gamma, Wo, eps: float = RMS_EPS):
    """o, z [..., H, dv], gamma [dv], Wo [H dv, D] -> y [..., D]."""
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * gamma
    u = r * silu(z)
    return u.reshape(o.shape[:-2] + (-1,)) @ Wo


def layer_prefill(orc, x, Wq, Wk, Wv, Wg, Wb, Wz, Wo, gamma, W1, W2, S0=None, hist=None):
    """The layer over a prompt: x [B,T,D]. Returns dict(y [B,T,D], o, S, hist)."""
    H = Wg.shape[1]
    q, k, v, z, g, b = projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H)
    r = orc.jetblock_prefill(x, W1, W2, q, k, v, g, b, S0, hist)
    return dict(y=output(r["o"], z, gamma, Wo), o=r["o"], S=r["S"], hist=r["hist"])


def layer_decode(orc, x, Wq, Wk, Wv, Wg, Wb, Wz, Wo, gamma, W1, W2, S0, hist):
    """n decode steps: x [n,B,D]; S0 [B,H,dv,dk], hist [B,3,H,dv]. Returns
    dict(y [n,B,D], o [n,B,H,dv], S, hist)."""
    H = Wg.shape[1]
    q, k, v, z, g, b = projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H)
    r = orc.jetblock_decode(x, W1, W2, q, k, v, g, b, S0, hist)
    return dict(y=output(r["o"], z, gamma, Wo), o=r["o"], S=r["S"], hist=r["hist"])
