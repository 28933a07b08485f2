"""GPU parity: the CUDA path through the C ABI against the float64 oracle on the same seeded bits.

Bar (stated for this forward pass): max|x - x_ref| / max|x_ref| <= 1e-4 for float32 inputs and
<= 5e-3 for bfloat16 inputs, for the outputs o and for the final state.
Full-size workloads run the GPU exactly as the benchmark launches it and compare sampled
(b, hv) pairs -- every token and every state element of those pairs -- with the oracle.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_NONE, GATE_SAFE, GATE_STANDARD, WORKLOADS, Workload, make_inputs
from parity_util import TOL, oracle_pairs, rel_err, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def _run_chunk(xd, w, **kw):
    kw.setdefault("check_status", "workspace" not in kw)
    return kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                         chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, **kw)


def _check_full(w, x, o, S, tol=None):
    tol = tol or TOL[w.dtype]
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                                  gate_mode=w.gate_mode, lower_bound=w.lower_bound)
    eo, eS = rel_err(o, o_ref), rel_err(S, S_ref)
    assert eo <= tol, f"o rel err {eo:.3e} > {tol}"
    assert eS <= tol, f"S_T rel err {eS:.3e} > {tol}"
    return eo, eS


def _check_pairs(w, x, o, S, pairs, tol=None):
    tol = tol or TOL[w.dtype]
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    o_ref = np.stack([r[0] for r in refs])
    S_ref = np.stack([r[1] for r in refs])
    eo, eS = rel_err(o_gpu, o_ref), rel_err(S_gpu, S_ref)
    assert eo <= tol, f"o rel err {eo:.3e} > {tol} on pairs {pairs}"
    assert eS <= tol, f"S_T rel err {eS:.3e} > {tol} on pairs {pairs}"
    return eo, eS


# ------------------------------------------------------------------ workloads, as benchmarked ---

def test_workload1_tiny_fp32_full():
    w = WORKLOADS[1]
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


def test_workload2_gva_prefill_full():
    w = WORKLOADS[2]
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


def test_workload3_training_prefill_sampled():
    w = WORKLOADS[3]
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_pairs(w, x, o, S, sample_pairs(w.B, w.HV, 6))


def test_workload4_long_prefill_sampled():
    w = WORKLOADS[4]
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_pairs(w, x, o, S, sample_pairs(w.B, w.HV, 3))


def _decode_run(w, x, steps):
    """`steps` consecutive kda_recurrent_step calls on the workload's [B, steps, ...] token stream."""
    xd = to_dev(x)
    S = xd["S0"].clone() if xd["S0"] is not None else torch.zeros(w.B, w.HV, w.K, w.V, device="cuda")
    outs = []
    for t in range(steps):
        outs.append(kda.recurrent_step(xd["q"][:, t].contiguous(), xd["k"][:, t].contiguous(),
                                       xd["v"][:, t].contiguous(), xd["g"][:, t].contiguous(),
                                       xd["beta"][:, t].contiguous(), S, xd["A_log"], xd["dt_bias"],
                                       gate_mode=w.gate_mode, lower_bound=w.lower_bound))
    torch.cuda.synchronize()
    return torch.stack(outs, dim=1), S


def test_workload5_decode_sampled():
    w = WORKLOADS[5]
    x = make_inputs(w)
    o, S = _decode_run(w, x, w.decode_steps)
    _check_pairs(w, x, o, S, sample_pairs(w.B, w.HV, 8))


# -------------------------------------------------------------------------- shapes and edges ---

def _small(B=2, T=100, H=2, HV=4, K=128, V=128, chunk=64, dtype=torch.bfloat16, gate=GATE_SAFE, S0=0.02,
           A_log=(-0.5, 0.5), lb=-5.0):
    return Workload(99, "edge", B, T, H, HV, K, V, chunk, dtype, gate, lb, A_log, -4.0, 0.1, S0)


@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 100, 191])
def test_ragged_lengths(T):
    w = _small(T=T)
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


@pytest.mark.parametrize("K,V", [(16, 16), (32, 64), (64, 32), (64, 128), (128, 64), (128, 16)])
@pytest.mark.parametrize("chunk", [16, 64])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shapes_chunks_dtypes(K, V, chunk, dtype):
    w = _small(T=75, K=K, V=V, chunk=chunk, dtype=dtype)
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


@pytest.mark.parametrize("H,HV", [(4, 4), (2, 4), (1, 4), (3, 12)])
@pytest.mark.parametrize("gate", [GATE_SAFE, GATE_STANDARD])
def test_gva_and_gates(H, HV, gate):
    w = _small(H=H, HV=HV, gate=gate, T=130, A_log=(-1.0, 0.5))
    x = make_inputs(w)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


def test_gate_none_with_precomputed_decay():
    w = _small(T=90)
    x = make_inputs(w)
    g = oracle.gate(x["g"], x["A_log"], x["dt_bias"], mode=GATE_SAFE, lower_bound=-5.0)
    xg = dict(x, g=torch.from_numpy(g).to(torch.float32))
    w32 = _small(T=90, dtype=torch.float32, gate=GATE_NONE)
    xg = {k_: (v_.float() if isinstance(v_, torch.Tensor) and v_.dtype == torch.bfloat16 else v_) for k_, v_ in xg.items()}
    o, S = _run_chunk(to_dev(xg), w32)
    torch.cuda.synchronize()
    _check_full(w32, xg, o, S)


def test_dt_bias_none_and_S0_none_equals_zeros():
    w = _small(T=80, S0=None)
    x = make_inputs(w)
    x["dt_bias"] = None
    xd = to_dev(x)
    o1, S1 = _run_chunk(xd, w)
    xd0 = dict(xd, S0=torch.zeros(w.B, w.HV, w.K, w.V, device="cuda"))
    o2, S2 = _run_chunk(xd0, w)
    torch.cuda.synchronize()
    assert torch.equal(o1, o2) and torch.equal(S1, S2)
    _check_full(w, x, o1, S1)


def test_split_and_resume_equals_single_call():
    """S_T of one call is S0 of the next (stateful serving)."""
    w = _small(T=256)
    x = make_inputs(w)
    xd = to_dev(x)
    o, S = _run_chunk(xd, w)
    T1 = 128
    first = {k_: (v_[:, :T1].contiguous() if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in xd.items()}
    second = {k_: (v_[:, T1:].contiguous() if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in xd.items()}
    o1, S1 = _run_chunk(first, w)
    second["S0"] = S1
    o2, S2 = _run_chunk(second, w)
    torch.cuda.synchronize()
    _check_full(w, x, torch.cat([o1, o2], dim=1), S2)
    _check_full(w, x, o, S)


def test_in_place_state_update():
    w = _small(T=70)
    x = make_inputs(w)
    xd = to_dev(x)
    S_buf = xd["S0"].clone()
    o, S = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], S_buf,
                         chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound, S_T=S_buf)
    torch.cuda.synchronize()
    _check_full(w, x, o, S_buf)


def test_prefill_then_decode_handoff():
    """Prefill T tokens, then 16 decode steps from S_T, equals the recurrence over T + 16 tokens."""
    w = _small(B=2, T=144, H=2, HV=4)
    x = make_inputs(w)
    xd = to_dev(x)
    T1 = 128
    pre = {k_: (v_[:, :T1].contiguous() if k_ in ("q", "k", "v", "g", "beta") else v_) for k_, v_ in xd.items()}
    o1, S = _run_chunk(pre, w)
    outs = []
    for t in range(T1, w.T):
        outs.append(kda.recurrent_step(xd["q"][:, t].contiguous(), xd["k"][:, t].contiguous(),
                                       xd["v"][:, t].contiguous(), xd["g"][:, t].contiguous(),
                                       xd["beta"][:, t].contiguous(), S, xd["A_log"], xd["dt_bias"],
                                       gate_mode=w.gate_mode, lower_bound=w.lower_bound))
    torch.cuda.synchronize()
    o = torch.cat([o1, torch.stack(outs, dim=1)], dim=1)
    _check_full(w, x, o, S)


@pytest.mark.parametrize("K,V", [(16, 16), (64, 128), (128, 128), (128, 32)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("gate", [GATE_SAFE, GATE_STANDARD])
def test_decode_small(K, V, dtype, gate):
    w = Workload(98, "decode-edge", 3, 9, 2, 4, K, V, 64, dtype, gate, -5.0, (-1.0, 0.5), -4.0, 0.1, 0.02,
                 decode_steps=9)
    x = make_inputs(w)
    o, S = _decode_run(w, x, w.T)
    _check_full(w, x, o, S)


# -------------------------------------------------------------------------------- stress -------

def test_stress_strong_decay_every_token():
    """g_raw large and positive: the safe gate sits at its floor L on every token and channel
    (in-chunk log-decay spans reach 64 * 5 = 320)."""
    w = _small(T=200, lb=-5.0)
    x = make_inputs(w)
    x["g"] = (x["g"].float().abs() * 20 + 30).to(w.dtype)
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


def test_stress_standard_gate_extreme_values():
    w = _small(T=150, gate=GATE_STANDARD, A_log=(1.0, 2.0))
    x = make_inputs(w)
    x["g"] = (x["g"].float() * 8).to(w.dtype)   # per-token decays down to about -exp(2)*30
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)


def test_stress_beta_one_unit_keys_reconstruction():
    """beta = 1 with q = k (unit): every output is v / sqrt(K) exactly in exact arithmetic."""
    w = _small(T=130, dtype=torch.float32)
    x = make_inputs(w)
    x["beta"] = torch.ones_like(x["beta"])
    x["q"] = x["k"].clone()
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    _check_full(w, x, o, S)
    G = w.HV // w.H
    expect = x["v"] / math.sqrt(w.K)
    assert rel_err(o.cpu(), expect.double().numpy()) <= 1e-4


def test_no_decay_no_write_keeps_state():
    w = _small(T=64, gate=GATE_NONE, dtype=torch.float32)
    x = make_inputs(w)
    x["g"] = torch.zeros_like(x["g"])
    x["beta"] = torch.zeros_like(x["beta"])
    o, S = _run_chunk(to_dev(x), w)
    torch.cuda.synchronize()
    assert rel_err(S.cpu(), x["S0"].double().numpy()) <= 1e-6


# ---------------------------------------------------------------------- gate kernel, status ----

@pytest.mark.parametrize("mode", [GATE_SAFE, GATE_STANDARD])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_gate_kernel(mode, dtype):
    w = _small(T=33, dtype=dtype)
    x = make_inputs(w)
    g = kda.gate(x["g"].cuda(), x["A_log"].cuda(), x["dt_bias"].cuda(), mode=mode, lower_bound=-5.0)
    torch.cuda.synchronize()
    ref = oracle.gate(x["g"], x["A_log"], x["dt_bias"], mode=mode, lower_bound=-5.0)
    assert np.abs(g.cpu().double().numpy() - ref).max() <= 2e-6 * max(1.0, np.abs(ref).max())


def test_read_status_ok_after_call():
    w = _small(T=64)
    x = to_dev(make_inputs(w))
    ws = torch.zeros(kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk), dtype=torch.uint8, device="cuda")
    _run_chunk(x, w, workspace=ws)
    kda.read_status(ws)


def test_non_contiguous_output_rejected():
    w = _small(T=64)
    x = to_dev(make_inputs(w))
    big = torch.empty(w.B, 2 * w.T, w.HV, w.V, dtype=w.dtype, device="cuda")
    with pytest.raises(kda.KdaError):
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"], chunk=64,
                      gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=big[:, ::2])


def test_invalid_call_launches_nothing():
    w = _small(T=64)
    x = to_dev(make_inputs(w))
    o = torch.full((w.B, w.T, w.HV, w.V), 7.0, dtype=w.dtype, device="cuda")
    with pytest.raises(kda.KdaError) as e:
        kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"], chunk=32,
                      gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=o)
    assert e.value.status == kda.ERR_UNSUPPORTED
    torch.cuda.synchronize()
    assert torch.all(o == 7.0)
