"""Pins of the absorbed MLA decode oracle (CPU only): KDA ledger, derivation DER2 -- q absorbs W_UK and
meets the latent c directly, K and V are never decompressed.

The absorbed form is pinned by the decompressed one (K = c W_UK^T, V = c W_UV^T per head and the
textbook softmax attention), and by special cases: one cached position, a zero query, permutation
of the positions, ragged lengths.  A planted slip -- W_UK transposed, the softmax over heads instead
of positions, W_UV applied before the weighted sum with the wrong axis, the scale dropped -- fails
one of them.
"""
import numpy as np
import pytest

from oracle import mla


def _problem(B=3, T=11, H=4, d_q=8, d_v=6, r=5, seed=0):
    g = np.random.default_rng(777 + seed)
    q = g.standard_normal((B, H, d_q))
    W_UK = g.standard_normal((H, d_q, r)) / np.sqrt(d_q)
    W_UV = g.standard_normal((H, d_v, r)) / np.sqrt(r)
    c = g.standard_normal((B, T, r))
    return q, W_UK, W_UV, c


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_absorbed_equals_decompressed(seed):
    q, W_UK, W_UV, c = _problem(seed=seed)
    a = mla.absorbed(q, W_UK, W_UV, c)
    d = mla.decompressed(q, W_UK, W_UV, c)
    assert np.allclose(a, d, rtol=1e-12, atol=1e-13)


def test_scale_enters_the_scores():
    q, W_UK, W_UV, c = _problem(seed=3)
    a1 = mla.absorbed(q, W_UK, W_UV, c)
    a2 = mla.absorbed(q, W_UK, W_UV, c, scale=1.0 / np.sqrt(q.shape[-1]))
    assert np.array_equal(a1, a2)                                 # the default
    a3 = mla.absorbed(q, W_UK, W_UV, c, scale=2.0)
    assert np.allclose(a3, mla.decompressed(q, W_UK, W_UV, c, scale=2.0), rtol=1e-12, atol=1e-13)
    assert not np.allclose(a1, a3, rtol=1e-3)


def test_single_position_gives_its_value():
    q, W_UK, W_UV, c = _problem(T=1, seed=4)
    o = mla.absorbed(q, W_UK, W_UV, c)
    expect = np.einsum("hvr,br->bhv", W_UV, c[:, 0])
    assert np.allclose(o, expect, rtol=1e-13, atol=1e-14)


def test_zero_query_averages_the_values():
    q, W_UK, W_UV, c = _problem(seed=5)
    o = mla.absorbed(np.zeros_like(q), W_UK, W_UV, c)
    expect = np.einsum("hvr,br->bhv", W_UV, c.mean(axis=1))
    assert np.allclose(o, expect, rtol=1e-13, atol=1e-14)


def test_positions_are_a_set():
    q, W_UK, W_UV, c = _problem(seed=6)
    perm = np.random.default_rng(1).permutation(c.shape[1])
    assert np.allclose(mla.absorbed(q, W_UK, W_UV, c), mla.absorbed(q, W_UK, W_UV, c[:, perm]), rtol=1e-12,
                       atol=1e-13)


def test_ragged_lengths_ignore_the_tail():
    q, W_UK, W_UV, c = _problem(B=3, T=9, seed=7)
    lengths = [9, 4, 1]
    o = mla.absorbed(q, W_UK, W_UV, c, lengths=lengths)
    for b, L in enumerate(lengths):
        ob = mla.absorbed(q[b:b + 1], W_UK, W_UV, c[b:b + 1, :L])
        assert np.allclose(o[b], ob[0], rtol=1e-13, atol=1e-14)
    c2 = c.copy()
    c2[1, 4:] = 1e3   # garbage past the length changes nothing
    assert np.array_equal(mla.absorbed(q, W_UK, W_UV, c2, lengths=lengths), o)


def test_hand_computed_two_positions():
    # one head, d_q = r = d_v = 1, W = 1: scores q c_t, o = sum_t softmax_t c_t
    q = np.array([[[2.0]]])
    c = np.array([[[0.0], [1.0]]])
    W = np.ones((1, 1, 1))
    o = mla.absorbed(q, W, W, c, scale=1.0)[0, 0, 0]
    e = np.exp(2.0)
    assert abs(o - e / (1.0 + e)) < 1e-15
