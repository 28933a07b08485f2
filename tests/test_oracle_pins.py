"""Pins of the float64 oracle against what the pages and the mathematics fix (CPU only).

Each test names the property and where it comes from.  Together they are chosen
so that a plausible slip in the oracle -- rate inside/outside the wrong
function, a transposed decay, the prediction taken before the decay, a wrong
sign in the residual, beta in the wrong place, a missing read-out scale, a
tiled instead of repeat_interleave'd head map, an exclusive instead of
inclusive prefix sum -- fails at least one of them.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.special

import oracle

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
rng_seed = 20240607


def _rng(extra=0):
    return np.random.default_rng(rng_seed + extra)


def _unit(x, axis=-1):
    return x / np.linalg.norm(x, axis=axis, keepdims=True)


def _rand_problem(B=1, T=12, H=1, HV=1, K=8, V=6, seed=0, g_scale=0.3, with_S0=True):
    r = _rng(seed)
    q = _unit(r.standard_normal((B, T, H, K)))
    k = _unit(r.standard_normal((B, T, H, K)))
    v = r.standard_normal((B, T, HV, V))
    g = -g_scale * r.random((B, T, HV, K))
    beta = r.random((B, T, HV))
    S0 = 0.3 * r.standard_normal((B, HV, K, V)) if with_S0 else None
    return q, k, v, g, beta, S0


# ---------------------------------------------------------------- gate ------------------------

def test_gate_worked_example_matches_page():
    """KDA notes, "Gate 激活", §初始化与默认值: g ~ -0.09, exp(g) ~ 0.91 (91 %), floor exp(-5) ~ 0.0067."""
    with open(os.path.join(GOLDEN, "gate_worked_example.json")) as f:
        gold = json.load(f)
    x = gold["inputs"]
    g = oracle.gate(np.array([[[x["g_raw"]]]]), np.array([x["A_log"]]), np.array([[x["dt_bias"]]]),
                    mode=oracle.GATE_SAFE, lower_bound=x["lower_bound"])[0, 0, 0]
    p = gold["printed"]
    assert round(g, p["g"]["decimals"]) == p["g"]["value"]
    assert round(math.exp(g), p["exp_g"]["decimals"]) == p["exp_g"]["value"]
    assert round(100 * math.exp(g)) == p["retention_percent"]["value"]
    # the floor: safe gate saturates at L, exp(L) as printed
    g_sat = oracle.gate(np.array([[[1e4]]]), np.array([0.0]), None, mode=oracle.GATE_SAFE,
                        lower_bound=x["lower_bound"])[0, 0, 0]
    assert g_sat == x["lower_bound"]
    assert round(math.exp(g_sat), p["exp_lower_bound"]["decimals"]) == p["exp_lower_bound"]["value"]


def test_safe_gate_rate_inside_sigmoid():
    """Table "两种 Gate": safe g = L*sigmoid(rate*input).  sigmoid(0) = 1/2 for every rate, so at
    input 0 the gate is L/2 whatever A_log is; with rate outside the sigmoid it would scale."""
    HV, K = 3, 4
    A_log = np.array([-1.0, 0.0, 1.5])
    dt_bias = _rng(1).standard_normal((HV, K))
    g_raw = -dt_bias[None, None]                        # input = 0 everywhere
    g = oracle.gate(g_raw, A_log, dt_bias, mode=oracle.GATE_SAFE, lower_bound=-3.0)
    np.testing.assert_allclose(g, -1.5, rtol=0, atol=1e-15)


def test_standard_gate_rate_outside_softplus():
    """Table "两种 Gate": standard g = -rate*softplus(input); softplus(0) = ln 2, so g = -exp(A_log)*ln 2."""
    A_log = np.array([-1.0, 0.0, 1.5])
    g = oracle.gate(np.zeros((1, 1, 3, 2)), A_log, None, mode=oracle.GATE_STANDARD)
    np.testing.assert_allclose(g[0, 0, :, 0], -np.exp(A_log) * math.log(2.0), rtol=1e-15)


def test_gate_ranges_limits_and_symmetries():
    """Ranges [L, 0] (safe) and (-inf, 0] (standard); limits; sigmoid(-x) = 1 - sigmoid(x) and
    softplus(x) - softplus(-x) = x give g(x) + g(-x) = L and g(x) - g(-x) = -rate*x."""
    r = _rng(2)
    HV, K = 4, 16
    A_log = r.uniform(-1, 1, HV)
    x = 6 * r.standard_normal((2, 5, HV, K))
    L = -5.0
    gs = oracle.gate(x, A_log, None, mode=oracle.GATE_SAFE, lower_bound=L)
    gs_neg = oracle.gate(-x, A_log, None, mode=oracle.GATE_SAFE, lower_bound=L)
    assert np.all(gs <= 0) and np.all(gs >= L)
    np.testing.assert_allclose(gs + gs_neg, L, atol=1e-13)
    gt = oracle.gate(x, A_log, None, mode=oracle.GATE_STANDARD)
    gt_neg = oracle.gate(-x, A_log, None, mode=oracle.GATE_STANDARD)
    assert np.all(gt <= 0)
    rate = np.exp(A_log)[None, None, :, None]
    np.testing.assert_allclose(gt - gt_neg, -rate * x, atol=1e-12)
    # limits
    big = np.full((1, 1, 1, 1), 800.0)
    assert oracle.gate(big, np.zeros(1), None, mode=oracle.GATE_SAFE, lower_bound=L)[0, 0, 0, 0] == L
    assert oracle.gate(-big, np.zeros(1), None, mode=oracle.GATE_SAFE, lower_bound=L)[0, 0, 0, 0] == 0.0
    np.testing.assert_allclose(oracle.gate(big, np.zeros(1), None, mode=oracle.GATE_STANDARD)[0, 0, 0, 0], -800.0)
    assert oracle.gate(-big, np.zeros(1), None, mode=oracle.GATE_STANDARD)[0, 0, 0, 0] == 0.0


def test_gate_against_library_routines():
    """The gate is sigmoid / softplus of an affine input: compare with scipy's expit and numpy's logaddexp."""
    r = _rng(3)
    HV, K = 3, 8
    A_log = r.uniform(-1, 0.5, HV)
    dt_bias = -4 + 0.1 * r.standard_normal((HV, K))
    g_raw = r.standard_normal((2, 7, HV, K))
    inp = g_raw + dt_bias[None, None]
    rate = np.exp(A_log)[None, None, :, None]
    np.testing.assert_allclose(oracle.gate(g_raw, A_log, dt_bias, mode=oracle.GATE_SAFE, lower_bound=-5.0),
                               -5.0 * scipy.special.expit(rate * inp), rtol=1e-14)
    np.testing.assert_allclose(oracle.gate(g_raw, A_log, dt_bias, mode=oracle.GATE_STANDARD),
                               -rate * np.logaddexp(0.0, inp), rtol=1e-14)


def test_gate_dt_bias_broadcast_is_per_head_and_channel():
    """dt_bias is [HV, K] (KDA ledger symbol table): distinct per (head, channel) entries must land in place."""
    HV, K = 3, 5
    dt_bias = np.arange(HV * K, dtype=np.float64).reshape(HV, K) / 7.0 - 1.0
    g = oracle.gate(np.zeros((1, 2, HV, K)), np.zeros(HV), dt_bias, mode=oracle.GATE_STANDARD)
    np.testing.assert_allclose(g[0, 1], -np.logaddexp(0.0, dt_bias), rtol=1e-14)


def test_safe_gate_requires_lower_bound():
    with pytest.raises(ValueError):
        oracle.gate(np.zeros((1, 1, 1, 1)), np.zeros(1), None, mode=oracle.GATE_SAFE, lower_bound=None)


# ----------------------------------------------------------- recurrence ----------------------

@pytest.mark.parametrize("seed", [0, 1, 2])
def test_immediate_reconstruction(seed):
    """DeltaNet-family digest ("DeltaNet: ..."): with a unit key and beta = 1 the state returns v_t exactly
    when read with the same key.  Reading with q_t = k_t gives o_t = scale * k_t . S_t = v_t / sqrt(K),
    whatever the decay and the history."""
    q, k, v, g, beta, S0 = _rand_problem(T=20, K=8, V=5, seed=10 + seed)
    beta[:] = 1.0
    o, _ = oracle.recurrent(k, k, v, g, beta, S0)
    np.testing.assert_allclose(o, v / math.sqrt(8), atol=1e-13)


def test_partial_reconstruction_general_beta():
    """Same section: re-reading with the same unit key gives (1 - beta) k.S_dec + beta v."""
    q, k, v, g, beta, S0 = _rand_problem(T=9, K=6, V=4, seed=21)
    t = 8
    _, S_prev = oracle.recurrent(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t], S0)
    o, _ = oracle.recurrent(k[:, :t + 1], k[:, :t + 1], v[:, :t + 1], g[:, :t + 1], beta[:, :t + 1], S0)
    kt, bt = k[0, t, 0], beta[0, t, 0]
    S_dec = np.exp(g[0, t, 0])[:, None] * S_prev[0, 0]
    expect = (1 - bt) * (kt @ S_dec) + bt * v[0, t, 0]
    np.testing.assert_allclose(o[0, t, 0] * math.sqrt(6), expect, atol=1e-13)


def test_null_step_leaves_state_unchanged():
    """beta = 0 and g = 0: nothing decays and nothing is written, so S_t = S_{t-1} and o_t = scale q_t.S0."""
    q, k, v, g, beta, S0 = _rand_problem(T=7, K=8, V=6, seed=30)
    g[:] = 0.0
    beta[:] = 0.0
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o[0, :, 0], np.einsum("tk,kv->tv", q[0, :, 0], S0[0, 0]) / math.sqrt(8), atol=1e-14)


def test_decay_only_acts_on_key_channels():
    """KDA notes warning box: exp(g_t) is broadcast over V -- the decay is per KEY channel (row of S).
    With beta = 0: S_T = diag(exp(sum_t g_t)) S0 and o_t = scale (q_t * exp(Gam_t)) . S0."""
    q, k, v, g, beta, S0 = _rand_problem(T=10, K=7, V=5, seed=40, g_scale=0.8)
    beta[:] = 0.0
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    Gam = np.cumsum(g[0, :, 0], axis=0)
    np.testing.assert_allclose(S[0, 0], np.exp(Gam[-1])[:, None] * S0[0, 0], rtol=1e-13)
    np.testing.assert_allclose(o[0, :, 0], np.einsum("tk,kv->tv", q[0, :, 0] * np.exp(Gam), S0[0, 0]) / math.sqrt(7),
                               atol=1e-14)


def test_locality_orthogonal_query_unchanged():
    """DeltaNet-family digest: the update is local in key space -- with no decay, a query orthogonal to k_t
    reads the same before and after step t."""
    q, k, v, g, beta, S0 = _rand_problem(T=6, K=8, V=5, seed=50)
    g[:] = 0.0
    t = 5
    kt = k[0, t, 0]
    qo = _unit(q[0, t, 0] - (q[0, t, 0] @ kt) * kt)
    q2 = q.copy()
    q2[0, t, 0] = qo
    _, S_prev = oracle.recurrent(q[:, :t], k[:, :t], v[:, :t], g[:, :t], beta[:, :t], S0)
    o, _ = oracle.recurrent(q2, k, v, g, beta, S0)
    np.testing.assert_allclose(o[0, t, 0], (qo @ S_prev[0, 0]) / math.sqrt(8), atol=1e-14)


def test_linear_attention_special_case():
    """DeltaNet-family digest: with orthonormal keys, no decay, beta = 1 and S0 = 0 nothing is ever
    predicted (k_t.S = 0), so the delta rule writes v_t k_t^T exactly like causal linear attention:
    o_t = scale * sum_{j<=t} (q_t . k_j) v_j."""
    T, K, V = 8, 8, 5
    r = _rng(60)
    Qm, _ = np.linalg.qr(r.standard_normal((K, K)))
    k = Qm[:, :T].T.reshape(1, T, 1, K)
    q = _unit(r.standard_normal((1, T, 1, K)))
    v = r.standard_normal((1, T, 1, V))
    o, _ = oracle.recurrent(q, k, v, np.zeros((1, T, 1, K)), np.ones((1, T, 1)), None)
    scores = np.tril(q[0, :, 0] @ k[0, :, 0].T)
    np.testing.assert_allclose(o[0, :, 0], scores @ v[0, :, 0] / math.sqrt(K), atol=1e-13)


def test_gva_is_repeat_interleave_not_tile():
    """KDA notes input table: q, k are repeat_interleave'd from H to HV heads (head hv reads hv // G)."""
    B, T, H, HV, K, V = 1, 9, 2, 6, 4, 3
    r = _rng(70)
    q = _unit(r.standard_normal((B, T, H, K)))
    k = _unit(r.standard_normal((B, T, H, K)))
    v = r.standard_normal((B, T, HV, V))
    g = -0.2 * r.random((B, T, HV, K))
    beta = r.random((B, T, HV))
    o, S = oracle.recurrent(q, k, v, g, beta)
    o_rep, S_rep = oracle.recurrent(np.repeat(q, 3, axis=2), np.repeat(k, 3, axis=2), v, g, beta)
    np.testing.assert_array_equal(o, o_rep)
    np.testing.assert_array_equal(S, S_rep)
    o_tile, _ = oracle.recurrent(np.tile(q, (1, 1, 3, 1)), np.tile(k, (1, 1, 3, 1)), v, g, beta)
    assert np.abs(o_tile - o).max() > 1e-3


def test_linear_in_values_and_initial_state():
    """For fixed (q, k, g, beta) the map (v, S0) -> (o, S_T) is linear."""
    q, k, v1, g, beta, S01 = _rand_problem(B=2, T=11, HV=2, H=1, K=5, V=4, seed=80)
    r = _rng(81)
    v2 = r.standard_normal(v1.shape)
    S02 = r.standard_normal(S01.shape)
    a, b = 0.7, -1.9
    o1, S1 = oracle.recurrent(q, k, v1, g, beta, S01)
    o2, S2 = oracle.recurrent(q, k, v2, g, beta, S02)
    o, S = oracle.recurrent(q, k, a * v1 + b * v2, g, beta, a * S01 + b * S02)
    np.testing.assert_allclose(o, a * o1 + b * o2, atol=1e-12)
    np.testing.assert_allclose(S, a * S1 + b * S2, atol=1e-12)


def test_value_columns_are_independent():
    """DeltaNet-family digest ("Chunkwise KDA"): the causal solve runs per value channel, so column j of
    (o, S_T) depends only on column j of (v, S0)."""
    q, k, v, g, beta, S0 = _rand_problem(T=13, K=6, V=5, seed=90)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    o_c, S_c = oracle.recurrent(q, k, v[..., 2:3], g, beta, S0[..., 2:3])
    np.testing.assert_allclose(o_c[..., 0], o[..., 2], atol=1e-14)
    np.testing.assert_allclose(S_c[..., 0], S[..., 2], atol=1e-14)


def test_scale_defaults_to_inverse_sqrt_k_and_is_applied_at_read():
    """KDA notes step 4 / ledger DER1: o_t = (1/sqrt(K)) q_t . S_t.  One token from S0 = 0 with beta = 1:
    S_1 = k v^T, so o = scale (q.k) v."""
    K, V = 9, 3
    r = _rng(100)
    q = _unit(r.standard_normal((1, 1, 1, K)))
    k = _unit(r.standard_normal((1, 1, 1, K)))
    v = r.standard_normal((1, 1, 1, V))
    o, _ = oracle.recurrent(q, k, v, np.zeros((1, 1, 1, K)), np.ones((1, 1, 1)))
    np.testing.assert_allclose(o[0, 0, 0], (q[0, 0, 0] @ k[0, 0, 0]) * v[0, 0, 0] / 3.0, atol=1e-15)
    o2, _ = oracle.recurrent(q, k, v, np.zeros((1, 1, 1, K)), np.ones((1, 1, 1)), scale=0.5)
    np.testing.assert_allclose(o2, o * 1.5, atol=1e-15)


def test_two_token_brute_force_scalar():
    """K = V = 1 by hand: the recurrence is the scalar delta rule s_t = a s + b k (v - k a s)."""
    q = np.array([0.5, -1.0]).reshape(1, 2, 1, 1)
    k = np.array([1.0, 0.5]).reshape(1, 2, 1, 1)
    v = np.array([2.0, -3.0]).reshape(1, 2, 1, 1)
    g = np.log(np.array([0.5, 0.25])).reshape(1, 2, 1, 1)
    beta = np.array([0.5, 1.0]).reshape(1, 2, 1)
    S0 = np.array([4.0]).reshape(1, 1, 1, 1)
    # token 0: S_dec = 2, p = 2, r = 0, S = 2, o = 0.5*2 = 1
    # token 1: S_dec = 0.5, p = 0.25, r = -3.25, S = 0.5 + 0.5*(-3.25) = -1.125, o = -1*-1.125 = 1.125
    o, S = oracle.recurrent(q, k, v, g, beta, S0, scale=1.0)
    np.testing.assert_allclose(o.ravel(), [1.0, 1.125], atol=1e-15)
    np.testing.assert_allclose(S.ravel(), [-1.125], atol=1e-15)


# ------------------------------------------------------ independent forms ----------------------

@pytest.mark.parametrize("C", [1, 4, 7, 16, 70])
def test_chunkwise_equals_recurrence(C):
    """DeltaNet-family digest, "Chunkwise KDA" and the KDA ledger claim C3: the chunked schedule gives
    exactly the recurrent result, for any chunk length (including a ragged last chunk and C > T)."""
    q, k, v, g, beta, S0 = _rand_problem(B=2, T=37, H=2, HV=4, K=8, V=6, seed=110, g_scale=0.6)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    oc, Sc = oracle.chunkwise(q, k, v, g, beta, S0, chunk=C)
    scale_o, scale_S = np.abs(o).max(), np.abs(S).max()
    assert np.abs(oc - o).max() <= 1e-12 * scale_o
    assert np.abs(Sc - S).max() <= 1e-12 * scale_S


def test_chunkwise_equals_recurrence_tiny_workload():
    """Same claim on the tiny fp32 workload's shapes (B1 T64 H=HV=2 K=V=16, chunk 16) with strong decay."""
    q, k, v, g, beta, S0 = _rand_problem(B=1, T=64, H=2, HV=2, K=16, V=16, seed=120, g_scale=5.0, with_S0=False)
    o, S = oracle.recurrent(q, k, v, g, beta, None)
    oc, Sc = oracle.chunkwise(q, k, v, g, beta, None, chunk=16)
    assert np.abs(oc - o).max() <= 1e-12 * np.abs(o).max()
    assert np.abs(Sc - S).max() <= 1e-12 * np.abs(S).max()


def test_dplr_transition_form_equals_recurrence():
    """DeltaNet-family digest, "diagonal-low-rank transition": S_t = S_{t-1} A_t + beta v k^T with
    A_t = D_t (I - beta k k^T), evaluated with dense matrices, reproduces the recurrence."""
    q, k, v, g, beta, S0 = _rand_problem(B=1, T=15, H=1, HV=2, K=6, V=4, seed=130, g_scale=0.5)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    od, Sd = oracle.dplr(q, k, v, g, beta, S0)
    np.testing.assert_allclose(od, o, atol=1e-13)
    np.testing.assert_allclose(Sd, S, atol=1e-13)


def test_forward_applies_gate_then_recurrence():
    q, k, v, graw, beta, S0 = _rand_problem(T=5, K=4, V=3, seed=140)
    A_log = np.array([0.3])
    dt_bias = -4 + 0.1 * _rng(141).standard_normal((1, 4))
    o, S = oracle.forward(q, k, v, graw, beta, A_log, dt_bias, S0, gate_mode=oracle.GATE_SAFE, lower_bound=-5.0)
    g = oracle.gate(graw, A_log, dt_bias, mode=oracle.GATE_SAFE, lower_bound=-5.0)
    o2, S2 = oracle.recurrent(q, k, v, g, beta, S0)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(S, S2)


def test_split_and_resume_equals_single_pass():
    """Stateful serving (DeltaNet-family digest, fused recurrent section): S_T of one call is S0 of the next."""
    q, k, v, g, beta, S0 = _rand_problem(B=1, T=20, K=5, V=4, seed=150)
    o, S = oracle.recurrent(q, k, v, g, beta, S0)
    o1, S1 = oracle.recurrent(q[:, :8], k[:, :8], v[:, :8], g[:, :8], beta[:, :8], S0)
    o2, S2 = oracle.recurrent(q[:, 8:], k[:, 8:], v[:, 8:], g[:, 8:], beta[:, 8:], S1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=1), o, atol=1e-15)
    np.testing.assert_allclose(S2, S, atol=1e-15)
