"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory.

Such callers only hold buffers someone else allocated (an outer runtime with a fixed memory
budget and no allocator to hand out, or a serving loop where allocating on the call path is
not allowed), so they cannot pass the workspace kda_chunk_fwd needs.  The no-allocation entry
point takes its workspace from a fixed array inside the library.  Here it is called through the
C ABI twice in a row and each result is checked against kda_chunk_fwd's on the same inputs.
The built-in array is too small for the two-pass schedule's per-chunk records, so the no-allocation
call runs the single-pass schedule; the reference call is given a 256-byte workspace, which selects
the same schedule, so the two must agree bit for bit (and so within the tolerance the other GPU tests
use).  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_SAFE, GATE_STANDARD, Workload, make_inputs

pytestmark = pytest.mark.gpu

TOL = {torch.float32: 1e-4, torch.bfloat16: 5e-3}


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.all(np.isfinite(x))
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


@pytest.mark.parametrize("dtype,K,V,gate", [(torch.bfloat16, 128, 128, GATE_SAFE),
                                            (torch.bfloat16, 128, 128, GATE_STANDARD),
                                            (torch.float32, 64, 32, GATE_SAFE)])
def test_noalloc_matches_chunk_fwd_two_calls(dtype, K, V, gate):
    w = Workload(97, "noalloc", 2, 150, 2, 4, K, V, 64, dtype, gate, -5.0, (-1.0, 0.5), -4.0, 0.1, 0.02)
    x = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in make_inputs(w).items()}
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"])
    kw = dict(chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound)
    small_ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o_ref, S_ref = kda.chunk_fwd(*args, **kw, workspace=small_ws)
    kda.read_status(small_ws)
    for _ in range(2):
        o, S = kda.chunk_fwd_noalloc(*args, **kw)
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(S, S_ref)
        assert _rel(o, o_ref) <= TOL[dtype]
        assert _rel(S, S_ref) <= TOL[dtype]
