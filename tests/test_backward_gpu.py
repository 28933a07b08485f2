"""GPU parity of the reverse mode (kda_backward) against the float64 reverse-mode oracle
(oracle.backward, pinned by central finite differences of the forward oracle).

The loss is sum(dO * o) + sum(dS_T * S_T) with seeded dO and dS_T; the kernel's gradients for q, k, v,
g (g_raw and the gate parameters when the op applies the gate), beta and S0 are compared tensor by
tensor, max|x - x_ref| / max|x_ref|, at the forward pass's bars (1e-4 float32 inputs, 5e-3 bfloat16
inputs).  The kernel computes in float32 from the exact input bits, so the measured errors sit far below
the bars; the cases cover workloads 1 and 2 at full size, every K / V, both gates and none, GVA, ragged
lengths, and absent initial state / final-state gradient.
"""
import numpy as np
import pytest
import torch

from oracle import backward as obwd
from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_NONE, GATE_SAFE, GATE_STANDARD, WORKLOADS, Workload, make_inputs
from parity_util import TOL, rel_err, to_dev

pytestmark = pytest.mark.gpu


def _grads(w, x, with_dST=True, seed=5):
    gen = torch.Generator().manual_seed(seed)
    dO = torch.randn(w.B, w.T, w.HV, w.V, generator=gen).to(w.dtype)
    dS_T = torch.randn(w.B, w.HV, w.K, w.V, generator=gen) if with_dST else None
    xd = to_dev(x)
    got = kda.backward(xd["q"], xd["k"], xd["v"], xd["g"], xd["beta"], dO.cuda(), xd["A_log"], xd["dt_bias"],
                       xd["S0"], None if dS_T is None else dS_T.cuda(), gate_mode=w.gate_mode,
                       lower_bound=w.lower_bound)
    torch.cuda.synchronize()
    ref = obwd.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"], dO, dS_T,
                        gate_mode=w.gate_mode, lower_bound=w.lower_bound)
    tol = TOL[w.dtype]
    pairs = [("dq", "dq"), ("dk", "dk"), ("dv", "dv"), ("dbeta", "dbeta"), ("dS0", "dS0")]
    if w.gate_mode == GATE_NONE:
        pairs.append(("dg", "dg"))
    else:
        pairs += [("dg", "dg_raw"), ("dA_log", "dA_log")]
        if x["dt_bias"] is not None:
            pairs.append(("ddt_bias", "ddt_bias"))
    errs = {}
    for mine, theirs in pairs:
        errs[mine] = rel_err(got[mine], ref[theirs])
        assert errs[mine] <= tol, f"{mine}: rel err {errs[mine]:.3e} > {tol}"
    return errs


@pytest.mark.parametrize("wid", [1, 2])
def test_workloads_full(wid):
    w = WORKLOADS[wid]
    _grads(w, make_inputs(w))


def _small(B=2, T=37, H=2, HV=4, K=32, V=16, dtype=torch.float32, gate=GATE_SAFE, S0=0.02):
    lb = -5.0 if gate == GATE_SAFE else 0.0
    return Workload(92, "backward case", B, T, H, HV, K, V, 64, dtype, gate, lb, (-1.0, 0.5), -4.0, 0.1, S0)


@pytest.mark.parametrize("K,V", [(16, 16), (32, 64), (64, 32), (128, 128), (128, 16), (16, 128)])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_shapes_and_dtypes(K, V, dtype):
    w = _small(K=K, V=V, dtype=dtype, T=29)
    _grads(w, make_inputs(w))


@pytest.mark.parametrize("gate", [GATE_NONE, GATE_SAFE, GATE_STANDARD])
@pytest.mark.parametrize("H,HV", [(4, 4), (1, 4), (2, 6)])
def test_gates_and_gva(gate, H, HV):
    w = _small(H=H, HV=HV, gate=gate, T=21, K=64, V=32)
    x = make_inputs(w)
    if gate == GATE_NONE:  # a log decay given directly
        x["g"] = (-0.3 * torch.rand(x["g"].shape, generator=torch.Generator().manual_seed(3))).to(w.dtype)
    _grads(w, x)


@pytest.mark.parametrize("T", [1, 7, 8, 9, 64, 100])
def test_ragged_lengths_no_initial_state(T):
    w = _small(T=T, S0=None, K=32, V=32)
    x = make_inputs(w)
    x["dt_bias"] = None
    _grads(w, x, with_dST=False)
