"""Brute-force forms of the Gated DeltaNet recurrence for tiny inputs (numpy).

TEST INFRASTRUCTURE ONLY. Written independently of ``jet_oracle.c`` so the two
can pin each other: here the state is built from explicit products of dense
dk x dk transition matrices (Jet-Nemotron paper section 2.3, gated delta
rule), never from the token update itself:

  S_t = S_{t-1} A_t + b_t v_t k_t^T,   A_t = a_t (I - b_t k_t k_t^T)
  =>  S_t = S_0 A_1 ... A_t + sum_{s<=t} b_s v_s k_s^T A_{s+1} ... A_t,
  o_t = S_t q_t.

Only for T <= 16 and dk <= 8 or so: the cost is O(T^2) matrix products.
"""
from __future__ import annotations

import numpy as np


def _unit(x, eps=1e-6):
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def _prod(mats, n):
    P = np.eye(n)
    for M in mats:
        P = P @ M
    return P


def gdn_transition_products(q, k, v, g, beta, S0=None, eps=1e-6):
    """q,k [B,T,H,dk], v [B,T,H,dv], g,beta [B,T,H] (float64).
    Returns (o [B,T,H,dv], S_T [B,H,dv,dk]) from the explicit product formula."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    qh, kh = _unit(q, eps), _unit(k, eps)
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dv, dk))
    for b in range(B):
        for h in range(H):
            S0bh = np.zeros((dv, dk)) if S0 is None else S0[b, h]
            A = [np.exp(g[b, t, h]) * (np.eye(dk) - beta[b, t, h] * np.outer(kh[b, t, h], kh[b, t, h]))
                 for t in range(T)]
            for t in range(T):
                S = S0bh @ _prod(A[: t + 1], dk)
                for s in range(t + 1):
                    S = S + beta[b, s, h] * np.outer(v[b, s, h], kh[b, s, h]) @ _prod(A[s + 1: t + 1], dk)
                o[b, t, h] = S @ qh[b, t, h]
                if t == T - 1:
                    S_T[b, h] = S
            if T == 0:
                S_T[b, h] = S0bh
    return o, S_T
