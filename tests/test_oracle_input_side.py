"""Pins of the oracle's optional input-side pre-step (CPU only): L2-normalising q and k over the K
channels (the DeltaNet-family digest assumes L2-normalised keys) and taking beta as a logit through
the logistic sigmoid (KDA notes, "KDA 递归核心": beta is the write strength).

Chosen so that a plausible slip -- normalising over the token or head axis instead of K, a missing
square root, the sigmoid's sign flipped, the floor applied to the squared norm -- fails one of them.
"""
import numpy as np
import scipy.special

import oracle


def _rng(seed):
    return np.random.default_rng(31337 + seed)


def _raw(B=2, T=7, H=2, HV=4, K=8, V=5, seed=0):
    r = _rng(seed)
    q = 3.0 * r.standard_normal((B, T, H, K))
    k = 0.5 * r.standard_normal((B, T, H, K))
    v = r.standard_normal((B, T, HV, V))
    g = -0.2 * r.random((B, T, HV, K))
    bl = 2.0 * r.standard_normal((B, T, HV))
    S0 = 0.1 * r.standard_normal((B, HV, K, V))
    return q, k, v, g, bl, S0


def test_normalised_vectors_have_unit_norm_over_K():
    q, k, _, _, bl, _ = _raw()
    qn, kn, b = oracle.input_side(q, k, bl, l2norm_qk=True)
    assert np.allclose(np.linalg.norm(qn, axis=-1), 1.0, atol=1e-14)
    assert np.allclose(np.linalg.norm(kn, axis=-1), 1.0, atol=1e-14)
    # direction kept: a positive multiple of the input, per (token, head)
    ratio = qn / q
    assert np.allclose(ratio, ratio[..., :1], rtol=1e-12) and np.all(ratio > 0)
    assert np.array_equal(b, bl)  # beta untouched without beta_logits


def test_hand_computed_vector():
    q = np.array([[[[3.0, 4.0]]]])
    qn, kn, _ = oracle.input_side(q, q, np.zeros((1, 1, 1)), l2norm_qk=True)
    assert np.allclose(qn[0, 0, 0], [0.6, 0.8], atol=1e-15)


def test_zero_and_tiny_vectors_use_the_floor():
    q = np.zeros((1, 1, 1, 4))
    tiny = np.full((1, 1, 1, 4), 1e-9)  # norm 2e-9 < 1e-6: divided by the floor, not by its norm
    qn, kn, _ = oracle.input_side(q, tiny, np.zeros((1, 1, 1)), l2norm_qk=True)
    assert np.all(qn == 0.0)
    assert np.allclose(kn, tiny / oracle.NORM_FLOOR, rtol=1e-15)


def test_sigmoid_values():
    x = np.linspace(-30, 30, 121).reshape(1, 121, 1)
    _, _, b = oracle.input_side(np.ones((1, 121, 1, 2)), np.ones((1, 121, 1, 2)), x, beta_logits=True)
    assert np.allclose(b, scipy.special.expit(x), rtol=1e-14, atol=0)
    assert b[0, 60, 0] == 0.5                       # sigma(0) = 1/2
    assert np.allclose(b + b[:, ::-1], 1.0, atol=1e-15)  # sigma(x) + sigma(-x) = 1
    assert np.all(np.diff(b[0, :, 0]) > 0)


def test_both_off_is_identity():
    q, k, _, _, bl, _ = _raw(seed=1)
    qn, kn, b = oracle.input_side(q, k, bl)
    assert np.array_equal(qn, q) and np.array_equal(kn, k) and np.array_equal(b, bl)


def test_forward_with_input_side_is_scale_invariant_in_q_and_k():
    """With normalisation in the op, rescaling the raw q and k by positive factors changes nothing."""
    q, k, v, g, bl, S0 = _raw(seed=2)
    r = _rng(3)
    cq = np.exp(r.standard_normal(q.shape[:-1] + (1,)))
    ck = np.exp(r.standard_normal(k.shape[:-1] + (1,)))
    o1, S1 = oracle.forward(q, k, v, g, bl, None, None, S0, l2norm_qk=True, beta_logits=True)
    o2, S2 = oracle.forward(q * cq, k * ck, v, g, bl, None, None, S0, l2norm_qk=True, beta_logits=True)
    assert np.allclose(o1, o2, rtol=1e-12, atol=1e-14) and np.allclose(S1, S2, rtol=1e-12, atol=1e-14)


def test_forward_with_input_side_equals_forward_on_prepared_inputs():
    q, k, v, g, bl, S0 = _raw(seed=4)
    qn = q / np.linalg.norm(q, axis=-1, keepdims=True)
    kn = k / np.linalg.norm(k, axis=-1, keepdims=True)
    b = scipy.special.expit(bl)
    o1, S1 = oracle.forward(q, k, v, g, bl, None, None, S0, l2norm_qk=True, beta_logits=True)
    o2, S2 = oracle.forward(qn, kn, v, g, b, None, None, S0)
    assert np.allclose(o1, o2, rtol=1e-13, atol=1e-15) and np.allclose(S1, S2, rtol=1e-13, atol=1e-15)
    # and it is not the forward pass on the raw inputs
    o3, _ = oracle.forward(q, k, v, g, bl, None, None, S0)
    assert not np.allclose(o1, o3, rtol=1e-3)


def test_reconstruction_invariant_holds_after_normalisation():
    """KDA notes, step 3 with a unit key and beta = 1 (logit 40 rounds to 1 in float64): k_t . S_t = v_t
    for the last token, whatever the raw key's norm."""
    q, k, v, g, bl, S0 = _raw(seed=5, B=1, H=1, HV=1)
    bl = np.full_like(bl, 40.0)
    qn, kn, b = oracle.input_side(q, k, bl, l2norm_qk=True, beta_logits=True)
    assert np.all(b == 1.0)
    _, S = oracle.forward(q, k, v, g, bl, None, None, S0, l2norm_qk=True, beta_logits=True)
    assert np.allclose(kn[0, -1, 0] @ S[0, 0], v[0, -1, 0], atol=1e-12)
