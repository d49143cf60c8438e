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

Each matrix product is numpy's float64 matmul (a library primitive). With
interface="bf16" the values that cross a stage boundary are rounded to the
dtype they have there when the layer runs on bf16 tensors: q, k, v and z to
bf16 (the mixer's and the gate's inputs), the logits of g and b to float32,
the mixer output o to bf16, and the gated output to bf16 (the output
projection's input); every stage in between is float64. Without it no
intermediate is rounded. The mixer is the compiled oracle's.
"""
from __future__ import annotations

import numpy as np

RMS_EPS = 1e-6


def bf16(a):
    """Round float64 values to bfloat16 (via float32, round to nearest even) and back."""
    f = np.asarray(a, dtype=np.float64).astype(np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def f32(a):
    return np.asarray(a, dtype=np.float64).astype(np.float32).astype(np.float64)


def silu(z):
    return z / (1.0 + np.exp(-z))


def softplus(z):
    return np.logaddexp(0.0, z)


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-z))


def projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H: int, interface=None):
    """x [..., D] -> q, k [..., H, dk], v, z [..., H, dv], g, b [..., H]."""
    lead = x.shape[:-1]
    dk = Wq.shape[1] // H
    dv = Wv.shape[1] // H
    rt = bf16 if interface == "bf16" else (lambda a: a)
    rl = f32 if interface == "bf16" else (lambda a: a)
    q = rt(x @ Wq).reshape(lead + (H, dk))
    k = rt(x @ Wk).reshape(lead + (H, dk))
    v = rt(x @ Wv).reshape(lead + (H, dv))
    z = rt(x @ Wz).reshape(lead + (H, dv))
    g = -softplus(rl(x @ Wg))
    b = sigmoid(rl(x @ Wb))
    return q, k, v, z, g, b


def output(o, z, gamma, Wo, eps: float = RMS_EPS, interface=None):
    """o, z [..., H, dv], gamma [dv], Wo [H dv, D] -> y [..., D]."""
    rt = bf16 if interface == "bf16" else (lambda a: a)
    o = rt(o)
    r = o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * gamma
    u = rt(r * silu(z))
    return u.reshape(o.shape[:-2] + (-1,)) @ Wo


def layer_prefill(orc, x, Wq, Wk, Wv, Wg, Wb, Wz, Wo, gamma, W1, W2, S0=None, hist=None, interface=None):
    """The layer over a prompt: x [B,T,D]. Returns dict(y [B,T,D], o, S, hist)."""
    H = Wg.shape[1]
    q, k, v, z, g, b = projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H, interface)
    r = orc.jetblock_prefill(x, W1, W2, q, k, v, g, b, S0, hist)
    return dict(y=output(r["o"], z, gamma, Wo, interface=interface), o=r["o"], S=r["S"], hist=r["hist"])


def layer_decode(orc, x, Wq, Wk, Wv, Wg, Wb, Wz, Wo, gamma, W1, W2, S0, hist, interface=None):
    """n decode steps: x [n,B,D]; S0 [B,H,dv,dk], hist [B,3,H,dv]. Returns
    dict(y [n,B,D], o [n,B,H,dv], S, hist)."""
    H = Wg.shape[1]
    q, k, v, z, g, b = projections(x, Wq, Wk, Wv, Wg, Wb, Wz, H, interface)
    r = orc.jetblock_decode(x, W1, W2, q, k, v, g, b, S0, hist)
    return dict(y=output(r["o"], z, gamma, Wo, interface=interface), o=r["o"], S=r["S"], hist=r["hist"])
