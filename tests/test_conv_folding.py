"""The algebra behind folding the dynamic conv into the chunked prefill
(Jet-Nemotron paper, section 2.4 conv on V; section 2.3 gated delta rule in
chunked UT form), checked in float64 with numpy.

For a chunk of C tokens, U = T1 V' with V' the conv of V:
  v'_i = sum_{j=0..3} w_i[j] v_{i-j}   (v_{-3..-1}: the previous chunk's tail)
The preparation kernel writes M and MH instead of T1 so that
  U = M V + MH V_prev,
  M[r][s]  = sum_{j=0..3} w_{s+j}[j] T1[r][s+j]   (s = 0..C-1, T1[r][i] = 0 past C)
  MH[r][s] = sum_{j=-s..3} w_{s+j}[j] T1[r][s+j]   (s = -3..-1)
"""
import numpy as np
import pytest


def conv(v, v_prev, w):
    # v [C, n], v_prev [3, n] (tokens -3..-1), w [C, 4] -> v' [C, n]
    ext = np.concatenate([v_prev, v])
    return np.stack([sum(w[i, j] * ext[3 + i - j] for j in range(4)) for i in range(v.shape[0])])


def fold(T1, w):
    C = T1.shape[0]
    M = np.zeros_like(T1)
    MH = np.zeros((C, 3))                  # columns s = -3, -2, -1
    for r in range(C):
        for s in range(C):
            M[r, s] = sum(w[s + j, j] * T1[r, s + j] for j in range(4) if s + j < C)
        for s in (-3, -2, -1):
            MH[r, s + 3] = sum(w[s + j, j] * T1[r, s + j] for j in range(-s, 4))
    return M, MH


@pytest.mark.parametrize("C,L", [(64, 64), (64, 37), (16, 2)])
def test_folded_conv_equals_conv_then_ut(C, L):
    rng = np.random.default_rng(C + L)
    n = 5
    T1 = np.tril(rng.standard_normal((C, C)))
    T1[:, L:] = 0.0                        # tokens past the chunk end carry no weight (beta = 0)
    w = rng.standard_normal((C, 4))
    w[L:] = 0.0                            # taps past the end are zero in the kernel
    v = rng.standard_normal((C, n))
    v[L:] = rng.standard_normal((C - L, n)) * 1e3   # whatever the tile holds past the end
    v_prev = rng.standard_normal((3, n))
    M, MH = fold(T1, w)
    np.testing.assert_allclose(M @ v + MH @ v_prev, T1 @ conv(v, v_prev, w), rtol=1e-12, atol=1e-9)
    assert np.allclose(M, np.tril(M))      # still lower triangular: M[r][s] = 0 for s > r
    assert not M[:, L:].any()              # values past the chunk end meet zero weights


def test_folding_with_identity_taps_is_t1():
    rng = np.random.default_rng(1)
    T1 = np.tril(rng.standard_normal((64, 64)))
    w = np.zeros((64, 4))
    w[:, 0] = 1.0
    M, MH = fold(T1, w)
    np.testing.assert_array_equal(M, T1)
    assert not MH.any()
