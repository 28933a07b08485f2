"""Pins for the float64 reverse mode of the oracle (``oracle.backward``).

The reverse mode is derived, not printed on the pages, so it is pinned to something other than
itself: central finite differences of the forward oracle (which has its own pins), and two
structural facts of the recurrence -- outputs and final state are linear in (v, S0), so their
gradient with respect to v does not depend on v; and with beta = 0 nothing is written, so v has
no effect at all.  The chunkwise reverse mode, written separately from the chunk equations, must
agree with the token-by-token one for every chunk length, ragged tails included.
"""
import numpy as np
import pytest

import oracle
from oracle import backward as obw

GATES = [(oracle.GATE_NONE, None), (oracle.GATE_SAFE, -5.0), (oracle.GATE_STANDARD, None)]


def _case(seed, B=2, T=6, H=1, HV=2, K=3, V=2, gate_mode=oracle.GATE_SAFE):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, HV, V))
    if gate_mode == oracle.GATE_NONE:
        g = -rng.uniform(0.05, 1.0, (B, T, HV, K))          # log decay given directly
    else:
        g = rng.standard_normal((B, T, HV, K))              # g_raw
    beta = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, HV))))
    A_log = rng.uniform(-0.5, 0.5, HV)
    dt_bias = -1.0 + 0.3 * rng.standard_normal((HV, K))
    S0 = 0.3 * rng.standard_normal((B, HV, K, V))
    dO = rng.standard_normal((B, T, HV, V))
    dS_T = rng.standard_normal((B, HV, K, V))
    return dict(q=q, k=k, v=v, g=g, beta=beta, A_log=A_log, dt_bias=dt_bias, S0=S0), dO, dS_T


def _loss(x, dO, dS_T, gate_mode, lb):
    o, S = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                          gate_mode=gate_mode, lower_bound=lb)
    return float(np.sum(dO * o) + np.sum(dS_T * S))


# gradient key in the backward result for each input
GRAD_OF = {"q": "dq", "k": "dk", "v": "dv", "beta": "dbeta", "S0": "dS0"}


@pytest.mark.parametrize("gate_mode,lb", GATES)
def test_gradients_match_central_differences(gate_mode, lb):
    x, dO, dS_T = _case(11 + gate_mode, gate_mode=gate_mode)
    grads = obw.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"], dO, dS_T,
                         gate_mode=gate_mode, lower_bound=lb)
    keys = dict(GRAD_OF)
    if gate_mode == oracle.GATE_NONE:
        keys["g"] = "dg"
    else:
        keys.update(g="dg_raw", A_log="dA_log", dt_bias="ddt_bias")
    rng = np.random.default_rng(5)
    eps = 1e-6
    for name, gname in keys.items():
        a = x[name]
        an = grads[gname]
        assert an.shape == a.shape, (name, an.shape, a.shape)
        idx = [tuple(int(rng.integers(0, n)) for n in a.shape) for _ in range(12)]
        for ix in idx:
            xp = {kk: vv.copy() for kk, vv in x.items()}
            xm = {kk: vv.copy() for kk, vv in x.items()}
            xp[name][ix] += eps
            xm[name][ix] -= eps
            fd = (_loss(xp, dO, dS_T, gate_mode, lb) - _loss(xm, dO, dS_T, gate_mode, lb)) / (2 * eps)
            assert abs(fd - an[ix]) <= 1e-6 * max(1.0, abs(fd)), (name, ix, fd, an[ix])


def test_gva_gradients_add_over_the_group():
    # one q/k head read by two value heads: its gradient is the sum of the two heads' gradients
    x, dO, dS_T = _case(3, H=1, HV=2, gate_mode=oracle.GATE_NONE)
    full = obw.recurrent_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], dO, dS_T)
    parts = []
    for hv in range(2):
        sl = slice(hv, hv + 1)
        parts.append(obw.recurrent_backward(x["q"], x["k"], x["v"][:, :, sl], x["g"][:, :, sl], x["beta"][:, :, sl],
                                            x["S0"][:, sl], dO[:, :, sl], dS_T[:, sl]))
    np.testing.assert_allclose(full["dq"], parts[0]["dq"] + parts[1]["dq"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(full["dk"], parts[0]["dk"] + parts[1]["dk"], rtol=1e-12, atol=1e-12)


def test_value_gradient_does_not_depend_on_values():
    x, dO, dS_T = _case(7, gate_mode=oracle.GATE_NONE)
    g1 = obw.recurrent_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], dO, dS_T)
    v2 = np.random.default_rng(8).standard_normal(x["v"].shape) * 3.0
    S02 = np.random.default_rng(9).standard_normal(x["S0"].shape)
    g2 = obw.recurrent_backward(x["q"], x["k"], v2, x["g"], x["beta"], S02, dO, dS_T)
    np.testing.assert_allclose(g1["dv"], g2["dv"], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g1["dS0"], g2["dS0"], rtol=1e-12, atol=1e-12)


def test_nothing_written_means_no_value_gradient():
    x, dO, dS_T = _case(13, gate_mode=oracle.GATE_NONE)
    x["beta"] = np.zeros_like(x["beta"])
    gr = obw.recurrent_backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["S0"], dO, dS_T)
    assert np.all(gr["dv"] == 0.0)


@pytest.mark.parametrize("chunk", [1, 4, 7, 16, 70])
@pytest.mark.parametrize("H,HV", [(1, 2), (2, 2)])
def test_chunkwise_reverse_mode_equals_recurrent(chunk, H, HV):
    # the chunked form a backward kernel would follow, against the token-by-token reverse mode:
    # ragged last chunk (T = 19), a chunk longer than the sequence, GVA
    rng = np.random.default_rng(100 + chunk + HV)
    B, T, K, V = 2, 19, 4, 3
    q = rng.standard_normal((B, T, H, K))
    k = rng.standard_normal((B, T, H, K))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, HV, V))
    g = -rng.uniform(0.02, 1.5, (B, T, HV, K))
    beta = rng.uniform(0.05, 0.95, (B, T, HV))
    S0 = rng.standard_normal((B, HV, K, V))
    dO = rng.standard_normal((B, T, HV, V))
    dS_T = rng.standard_normal((B, HV, K, V))
    ref = obw.recurrent_backward(q, k, v, g, beta, S0, dO, dS_T)
    got = obw.chunkwise_backward(q, k, v, g, beta, S0, dO, dS_T, chunk=chunk)
    for key in ref:
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-10, atol=1e-12 * np.abs(ref[key]).max(),
                                   err_msg=key)


def test_chunkwise_reverse_mode_without_state_terms():
    # no initial state and no final-state gradient: only the outputs drive the gradients
    rng = np.random.default_rng(4)
    B, T, H, HV, K, V = 1, 10, 1, 1, 3, 2
    q, k = rng.standard_normal((B, T, H, K)), rng.standard_normal((B, T, H, K))
    v, g = rng.standard_normal((B, T, HV, V)), -rng.uniform(0.1, 0.8, (B, T, HV, K))
    beta, dO = rng.uniform(0.1, 0.9, (B, T, HV)), rng.standard_normal((B, T, HV, V))
    ref = obw.recurrent_backward(q, k, v, g, beta, None, dO, None)
    got = obw.chunkwise_backward(q, k, v, g, beta, None, dO, None, chunk=4)
    for key in ref:
        np.testing.assert_allclose(got[key], ref[key], rtol=1e-10, atol=1e-13, err_msg=key)
