"""GPU parity of both tensor-core prefill schedules (bf16 inputs, K = V = 128, chunk 64).

``kda_chunk_fwd`` runs the two-pass schedule (chunk-parallel local work, then the state recurrence)
when it is given ``kda_chunk_fwd_workspace_size`` bytes of workspace, and the single-pass schedule
(one CTA per (sequence, value head)) when it is given only the 256-byte status block.  Each case
here runs both and checks each against the float64 oracle on the same seeded inputs, with the bar
of the other parity tests: max|x - x_ref| / max|x_ref| <= 5e-3 for o and the final state.
The (B, HV) sizes reach every value-block width of the state pass (16, 32 and 64 columns); above
96 pairs only the single pass is offered.
"""
import numpy as np
import pytest
import torch

import oracle
from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_NONE, GATE_SAFE, GATE_STANDARD, WORKLOADS, Workload, make_inputs
from parity_util import TOL, oracle_pairs, rel_err, sample_pairs, to_dev

pytestmark = pytest.mark.gpu

SCHEDULES = ("two_pass", "single_pass")


def _workspace(w, schedule):
    if schedule == "single_pass":
        return torch.empty(256, dtype=torch.uint8, device="cuda")
    need = kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
    if w.B * w.HV > 96:  # the two-pass schedule is not offered for this many pairs
        assert need == 256
        pytest.skip("more (sequence, head) pairs than the two-pass schedule takes")
    assert need > 256
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    assert kda.schedule(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk, w.dtype, need) in (kda.SCHEDULE_TC_TWO_PASS,
                                                                                kda.SCHEDULE_TC_TWO_PASS_SCAN)
    return ws


def _run(w, xd, schedule, **kw):
    ws = _workspace(w, schedule)
    o, S = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                         chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws, **kw)
    kda.read_status(ws)
    return o, S


def _ref(w, x):
    return oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                          gate_mode=w.gate_mode, lower_bound=w.lower_bound)


def _wl(B=1, T=200, H=2, HV=4, gate=GATE_SAFE, S0=0.02, A_log=(-0.5, 0.5), lb=-5.0, dt_mean=-4.0, dt_std=0.1):
    return Workload(98, "schedule case", B, T, H, HV, 128, 128, 64, torch.bfloat16, gate, lb, A_log, dt_mean, dt_std,
                    S0)


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("T", [1, 2, 63, 64, 65, 127, 200, 1000])
def test_ragged_lengths_both_schedules(schedule, T):
    w = _wl(T=T)
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), schedule)
    o_ref, S_ref = _ref(w, x)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


# (B, HV) reaching value blocks of 16 (<= 18 pairs) and 32 columns (more pairs), and the single-pass schedule's counts
@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("B,H,HV", [(1, 1, 1), (2, 4, 8), (3, 5, 10), (1, 8, 32), (5, 8, 8), (2, 16, 48), (4, 8, 24)])
def test_pair_counts_both_schedules(schedule, B, H, HV):
    w = _wl(B=B, T=130, H=H, HV=HV)
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), schedule)
    pairs = sample_pairs(B, HV, 4)
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    assert rel_err(o_gpu, np.stack([r[0] for r in refs])) <= TOL[w.dtype]
    assert rel_err(S_gpu, np.stack([r[1] for r in refs])) <= TOL[w.dtype]


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("gate", [GATE_SAFE, GATE_STANDARD])
def test_gates_and_no_initial_state(schedule, gate):
    w = _wl(T=150, gate=gate, S0=None, lb=-5.0 if gate == GATE_SAFE else 0.0, A_log=(-1.0, 0.5))
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), schedule)
    o_ref, S_ref = _ref(w, x)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_precomputed_decay(schedule):
    w = _wl(T=150)
    x = make_inputs(w)
    g_log = oracle.gate(x["g"], x["A_log"], x["dt_bias"], mode=GATE_SAFE, lower_bound=w.lower_bound)
    x2 = dict(x, g=torch.from_numpy(g_log).to(torch.bfloat16))
    w2 = Workload(97, "decay given", w.B, w.T, w.H, w.HV, 128, 128, 64, torch.bfloat16, GATE_NONE, 0.0, None, 0.0,
                  0.0, 0.02)
    o, S = _run(w2, to_dev(x2), schedule)
    o_ref, S_ref = oracle.forward(x2["q"], x2["k"], x2["v"], x2["g"], x2["beta"], None, None, x2["S0"],
                                  gate_mode=GATE_NONE)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("schedule", SCHEDULES)
def test_strong_decay_takes_exact_path(schedule):
    # dt_bias far positive: every gate value near the lower bound (-5 per token), so the in-chunk
    # log-decay span exceeds the factorised path's limit and chunks take the exact path
    w = _wl(T=190, dt_mean=6.0, dt_std=0.0)
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), schedule)
    o_ref, S_ref = _ref(w, x)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("schedule", SCHEDULES)
@pytest.mark.parametrize("c_last", [-1.75, -2.5])
def test_short_last_chunk_decay_spans(schedule, c_last):
    # a 20-token last chunk with a constant log-decay per token: its span Gam_0 - Gam_end is
    # 19 |c_last| = 33.25 (factorised path, reference point = its last row) or 47.5 (exact path);
    # the full first chunk decays gently (-0.5 per token)
    w = _wl(T=84)
    x = make_inputs(w)
    g_log = torch.full((w.B, w.T, w.HV, 128), -0.5, dtype=torch.float32)
    g_log[:, 64:] = c_last
    x2 = dict(x, g=g_log.to(torch.bfloat16))
    w2 = Workload(96, "short chunk", w.B, w.T, w.H, w.HV, 128, 128, 64, torch.bfloat16, GATE_NONE, 0.0, None, 0.0, 0.0,
                  0.02)
    o, S = _run(w2, to_dev(x2), schedule)
    o_ref, S_ref = oracle.forward(x2["q"], x2["k"], x2["v"], x2["g"], x2["beta"], None, None, x2["S0"],
                                  gate_mode=GATE_NONE)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


def test_schedules_agree_on_the_same_call():
    # both schedules on one set of device inputs, each against the oracle
    w = _wl(B=2, T=333, H=2, HV=6)
    x = make_inputs(w)
    xd = to_dev(x)
    o_ref, S_ref = _ref(w, x)
    for schedule in SCHEDULES:
        o, S = _run(w, xd, schedule)
        assert rel_err(o, o_ref) <= TOL[w.dtype]
        assert rel_err(S, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("wid", [2, 4])
def test_benchmark_workloads_single_pass_sampled(wid):
    # the benchmark runs these with the two-pass schedule (test_parity_gpu); here the other one
    w = WORKLOADS[wid]
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), "single_pass")
    pairs = sample_pairs(w.B, w.HV, 3)
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    assert rel_err(o_gpu, np.stack([r[0] for r in refs])) <= TOL[w.dtype]
    assert rel_err(S_gpu, np.stack([r[1] for r in refs])) <= TOL[w.dtype]


def test_in_place_state_two_pass():
    w = _wl(T=140)
    x = make_inputs(w)
    xd = to_dev(x)
    S = xd["S0"].clone()
    ws = _workspace(w, "two_pass")
    o, S_out = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], S,
                             chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound, S_T=S, workspace=ws)
    kda.read_status(ws)
    assert S_out.data_ptr() == S.data_ptr()
    o_ref, S_ref = _ref(w, x)
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


# Shapes at the edges of the two-pass schedule's choices: many chunk records per pair (value blocks
# of 32 columns), many pairs (blocks of 64), and a ragged last chunk across several sequences.
@pytest.mark.parametrize("B,H,HV,T", [(1, 2, 4, 16384),
                                      (1, 37, 37, 448),
                                      (1, 38, 38, 64),
                                      (3, 2, 6, 700)])
def test_two_pass_edge_shapes(B, H, HV, T):
    w = _wl(B=B, T=T, H=H, HV=HV)
    x = make_inputs(w)
    o, S = _run(w, to_dev(x), "two_pass")
    pairs = sample_pairs(B, HV, 3)
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    assert rel_err(o_gpu, np.stack([r[0] for r in refs])) <= TOL[w.dtype]
    assert rel_err(S_gpu, np.stack([r[1] for r in refs])) <= TOL[w.dtype]


def test_two_pass_repeated_calls_reuse_workspace():
    # records left in the workspace by one call must not leak into the next call's results
    w = _wl(B=2, T=300, H=2, HV=4)
    ws = _workspace(w, "two_pass")
    outs = []
    for seed in (11, 12, 11):
        xd = to_dev(make_inputs(w, seed=seed))
        o, S = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                             chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws)
        kda.read_status(ws)
        outs.append((o.clone(), S.clone()))
    assert torch.equal(outs[0][0], outs[2][0]) and torch.equal(outs[0][1], outs[2][1])
    assert not torch.equal(outs[0][0], outs[1][0])
