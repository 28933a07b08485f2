"""GPU parity of the two-pass schedule with its state pass split along the sequence
(KDA_SCHEDULE_TC_TWO_PASS_SCAN) against the float64 oracle.

For long sequences with few (sequence, head) pairs the chunk-to-chunk state recurrence is split into
segments: every segment's affine chunk map S -> M S + b is carried through its chunks in parallel, the
segments are chained in order, and each segment's chunks are rerun from its true entering state with
the outputs.  The cases have segment counts and ragged tails the planner produces (a last segment
shorter than the others, a last chunk shorter than 64 tokens), initial states, both gates, the exact
(strong-decay) path and an in-place state update.  Bar: max|x - x_ref| / max|x_ref| <= 5e-3 (bf16
inputs) for o and the final state, every token and state element of the sampled pairs.
"""
import numpy as np
import pytest
import torch

from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_SAFE, GATE_STANDARD, Workload, make_inputs
from parity_util import TOL, oracle_pairs, rel_err, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def _wl(B, T, H, HV, gate=GATE_SAFE, S0=0.02, dt_mean=-4.0, A_log=(-0.5, 0.5)):
    lb = -5.0 if gate == GATE_SAFE else 0.0
    return Workload(93, "scan case", B, T, H, HV, 128, 128, 64, torch.bfloat16, gate, lb, A_log, dt_mean, 0.1, S0)


def _run(w, xd, S_T=None):
    need = kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
    assert kda.schedule(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk, w.dtype, need) == kda.SCHEDULE_TC_TWO_PASS_SCAN
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o, S = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                         chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws, S_T=S_T)
    kda.read_status(ws)
    return o, S


def _check(w, x, o, S, n=3):
    pairs = sample_pairs(w.B, w.HV, n)
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    eo = rel_err(o_gpu, np.stack([r[0] for r in refs]))
    eS = rel_err(S_gpu, np.stack([r[1] for r in refs]))
    assert eo <= TOL[w.dtype], f"o rel err {eo:.3e}"
    assert eS <= TOL[w.dtype], f"S rel err {eS:.3e}"


@pytest.mark.parametrize("B,H,HV,T,gate", [(1, 2, 4, 5000, GATE_SAFE),           # 79 chunks, ragged last chunk
                                           (2, 2, 2, 9000, GATE_STANDARD),       # a short last segment
                                           (1, 4, 8, 8192 - 5, GATE_SAFE),       # GVA
                                           (1, 1, 1, 64 * 300 + 63, GATE_STANDARD)])  # one pair, many segments
def test_scan_ragged_and_segmented(B, H, HV, T, gate):
    w = _wl(B, T, H, HV, gate=gate, A_log=(-1.0, 0.5))
    x = make_inputs(w)
    o, S = _run(w, to_dev(x))
    torch.cuda.synchronize()
    _check(w, x, o, S, n=3)


def test_scan_without_initial_state_and_bias():
    w = _wl(1, 6000, 1, 1, S0=None)
    x = make_inputs(w)
    x["dt_bias"] = None
    o, S = _run(w, to_dev(x))
    torch.cuda.synchronize()
    _check(w, x, o, S, n=4)


def test_scan_strong_decay_exact_path():
    w = _wl(1, 6000, 2, 4, dt_mean=6.0)
    x = make_inputs(w)
    o, S = _run(w, to_dev(x))
    torch.cuda.synchronize()
    _check(w, x, o, S, n=4)


def test_scan_in_place_state():
    w = _wl(1, 5000, 2, 2)
    x = make_inputs(w)
    xd = to_dev(x)
    S_buf = xd["S0"].clone()
    xd["S0"] = S_buf
    o, S = _run(w, xd, S_T=S_buf)
    torch.cuda.synchronize()
    assert S.data_ptr() == S_buf.data_ptr()
    _check(w, x, o, S_buf, n=4)


def test_scan_repeats_bit_exactly_and_matches_single_pass_on_sampled_pairs():
    w = _wl(2, 8187, 2, 4)
    x = make_inputs(w)
    xd = to_dev(x)
    o1, S1 = _run(w, xd)
    o1b, S1b = _run(w, xd)
    assert torch.equal(o1, o1b) and torch.equal(S1, S1b)  # records and carries left by a call change nothing
    ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o2, S2 = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                           chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws)
    kda.read_status(ws)
    torch.cuda.synchronize()
    _check(w, x, o1, S1, n=3)
    _check(w, x, o2, S2, n=3)
