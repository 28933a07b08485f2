"""GPU parity of the two-pass schedule on inputs far from unit magnitude, against the float64 oracle.

The two-pass records hold G = Kend^T Wtil, Q' = Qtil - A Wtil and KU = Kend^T U as fp16 tiles scaled by
one power of two each, and the state pass feeds the tensor core fp16(S 2^-sig) with sig from a bound
carried through the chain.  These cases move the magnitudes that set those exponents away from 1: the
values (U, KU, A U, the state and the outputs scale with v), the queries (Q', the outputs), the keys (G,
KU; small, so that the delta rule stays contractive) and the entering state, on both the unsplit and the
split state pass.  Bar: max|x - x_ref| / max|x_ref| <= 5e-3 (bf16 inputs) for o and the final state.
"""
import numpy as np
import pytest
import torch

import oracle
from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_SAFE, GATE_STANDARD, Workload, make_inputs
from parity_util import TOL, oracle_pairs, rel_err, sample_pairs, to_dev

pytestmark = pytest.mark.gpu


def _wl(B, T, H, HV, gate=GATE_SAFE, S0=0.02):
    lb = -5.0 if gate == GATE_SAFE else 0.0
    return Workload(94, "scale case", B, T, H, HV, 128, 128, 64, torch.bfloat16, gate, lb, (-1.0, 0.5), -4.0, 0.1, S0)


def _scaled(x, v=1.0, q=1.0, k=1.0, S0=1.0):
    y = dict(x)
    for name, f in (("v", v), ("q", q), ("k", k)):
        y[name] = (x[name].float() * f).to(torch.bfloat16)
    if x["S0"] is not None:
        y["S0"] = x["S0"] * S0 * v  # the state carries the values' scale
    return y


def _run(w, xd, expect):
    need = kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
    assert kda.schedule(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk, w.dtype, need) == expect
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    o, S = kda.chunk_fwd(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], xd["A_log"], xd["dt_bias"], xd["S0"],
                         chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound, workspace=ws)
    kda.read_status(ws)
    return o, S


SCALES = [dict(v=1e3), dict(v=1e-3), dict(q=30.0), dict(k=0.05), dict(S0=300.0), dict(v=1e-2, q=8.0, k=0.3)]


@pytest.mark.parametrize("sc", SCALES, ids=lambda d: ",".join(f"{k}{v:g}" for k, v in d.items()))
@pytest.mark.parametrize("gate", [GATE_SAFE, GATE_STANDARD])
def test_two_pass_scaled_inputs(sc, gate):
    w = _wl(2, 300, 2, 4, gate=gate)
    x = _scaled(make_inputs(w), **sc)
    o, S = _run(w, to_dev(x), kda.SCHEDULE_TC_TWO_PASS)
    o_ref, S_ref = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                                  gate_mode=w.gate_mode, lower_bound=w.lower_bound)
    assert np.all(np.isfinite(o.float().cpu().numpy())) and np.all(np.isfinite(S.float().cpu().numpy()))
    assert rel_err(o, o_ref) <= TOL[w.dtype]
    assert rel_err(S, S_ref) <= TOL[w.dtype]


@pytest.mark.parametrize("sc", [dict(v=1e3), dict(v=1e-3, S0=100.0)], ids=["v1e3", "v1e-3,S0100"])
def test_split_state_pass_scaled_inputs(sc):
    w = _wl(1, 5000, 2, 4)
    x = _scaled(make_inputs(w), **sc)
    o, S = _run(w, to_dev(x), kda.SCHEDULE_TC_TWO_PASS_SCAN)
    pairs = sample_pairs(w.B, w.HV, 2)
    refs = oracle_pairs(x, w, pairs)
    o_gpu = torch.stack([o[b, :, hv] for b, hv in pairs]).cpu()
    S_gpu = torch.stack([S[b, hv] for b, hv in pairs]).cpu()
    assert rel_err(o_gpu, np.stack([r[0] for r in refs])) <= TOL[w.dtype]
    assert rel_err(S_gpu, np.stack([r[1] for r in refs])) <= TOL[w.dtype]
