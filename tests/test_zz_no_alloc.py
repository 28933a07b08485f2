"""kda_chunk_fwd_noalloc: the prefill for callers that cannot allocate device memory.

Such callers only hold buffers someone else allocated (an outer runtime with a fixed memory
budget and no allocator to hand out, or a serving loop where allocating on the call path is
not allowed), so they cannot pass the workspace kda_chunk_fwd needs.  The no-allocation entry
point takes its workspace from a fixed array inside the library.  Here it is called through the
C ABI twice in a row, into output buffers allocated beforehand, and each result is checked against
kda_chunk_fwd's on the same inputs; across those calls neither the device's free memory nor torch's
allocation count may change.  The built-in array is too small for the two-pass schedule's per-chunk
records, so the no-allocation call runs the single-pass schedule (or the CUDA-core kernel for the
other shapes); the reference call is given a 256-byte workspace, which selects the same schedule, so
the two must agree bit for bit (and so within the tolerance the other GPU tests use).
This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_SAFE, GATE_STANDARD, Workload, make_inputs
from parity_util import TOL

pytestmark = pytest.mark.gpu


def _rel(x, ref):
    x = x.double().cpu().numpy()
    ref = ref.double().cpu().numpy()
    assert np.all(np.isfinite(x))
    return float(np.abs(x - ref).max() / max(np.abs(ref).max(), 1e-30))


def _allocs():
    return torch.cuda.memory_stats().get("allocation.all.allocated", 0)


@pytest.mark.parametrize("dtype,K,V,chunk,T,gate", [(torch.bfloat16, 128, 128, 64, 150, GATE_SAFE),
                                                    (torch.bfloat16, 128, 128, 64, 150, GATE_STANDARD),
                                                    (torch.bfloat16, 128, 128, 64, 40, GATE_SAFE),
                                                    (torch.bfloat16, 128, 128, 16, 70, GATE_SAFE),
                                                    (torch.float32, 64, 32, 64, 150, GATE_SAFE)])
def test_noalloc_matches_chunk_fwd_two_calls(dtype, K, V, chunk, T, gate):
    w = Workload(97, "noalloc", 2, T, 2, 4, K, V, chunk, dtype, gate, -5.0, (-1.0, 0.5), -4.0, 0.1, 0.02)
    x = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in make_inputs(w).items()}
    args = (x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"])
    kw = dict(chunk=w.chunk, gate_mode=w.gate_mode, lower_bound=w.lower_bound)
    small_ws = torch.empty(256, dtype=torch.uint8, device="cuda")
    o_ref, S_ref = kda.chunk_fwd(*args, **kw, workspace=small_ws)
    kda.read_status(small_ws)
    o = torch.empty_like(o_ref)
    S = torch.empty_like(S_ref)
    kept = [(torch.empty_like(o_ref), torch.empty_like(S_ref)) for _ in range(2)]  # results of the two calls
    kda.chunk_fwd_noalloc(*args, **kw, o=o, S_T=S)  # the first call on a device may load device code
    kda.noalloc_read_status()
    torch.cuda.synchronize()
    # nothing in this region allocates: outputs, copies and the status read-back use existing memory
    free0, allocs0 = torch.cuda.mem_get_info()[0], _allocs()
    for i in range(2):
        o.fill_(0)
        S.fill_(0)
        kda.chunk_fwd_noalloc(*args, **kw, o=o, S_T=S)
        kda.noalloc_read_status()
        kept[i][0].copy_(o)
        kept[i][1].copy_(S)
    torch.cuda.synchronize()
    free1, allocs1 = torch.cuda.mem_get_info()[0], _allocs()
    assert free1 == free0 and allocs1 == allocs0
    for oi, Si in kept:
        assert torch.equal(oi, o_ref) and torch.equal(Si, S_ref)
        assert _rel(oi, o_ref) <= TOL[dtype]
        assert _rel(Si, S_ref) <= TOL[dtype]


@pytest.mark.parametrize("over,status", [(dict(chunk=32), kda.ERR_UNSUPPORTED), (dict(H=3), kda.ERR_INVALID_ARG),
                                         (dict(K=48), kda.ERR_UNSUPPORTED)])
def test_noalloc_rejects_bad_sizes_and_launches_nothing(over, status):
    w = Workload(97, "noalloc", 1, 64, 2, 4, 128, 128, 64, torch.bfloat16, GATE_SAFE, -5.0, (-1.0, 0.5), -4.0, 0.1,
                 None)
    x = {n: (t.cuda() if isinstance(t, torch.Tensor) else t) for n, t in make_inputs(w).items()}
    o = torch.full((w.B, w.T, w.HV, w.V), 7.0, dtype=w.dtype, device="cuda")
    S_T = torch.full((w.B, w.HV, w.K, w.V), 7.0, dtype=torch.float32, device="cuda")
    a = dict(B=w.B, T=w.T, H=w.H, HV=w.HV, K=w.K, V=w.V, chunk=w.chunk)
    a.update(over)
    ptr = lambda t: None if t is None else t.data_ptr()  # noqa: E731
    st = kda.lib.kda_chunk_fwd_noalloc(ptr(x["q"]), ptr(x["k"]), ptr(x["v"]), ptr(x["g"]), ptr(x["beta"]),
                                       ptr(x["A_log"]), ptr(x["dt_bias"]), None, a["B"], a["T"], a["H"], a["HV"],
                                       a["K"], a["V"], a["chunk"], GATE_SAFE, -5.0, -1.0, kda.BF16, ptr(o), ptr(S_T),
                                       torch.cuda.current_stream().cuda_stream)
    assert st == status and kda.last_error() != ""
    torch.cuda.synchronize()
    assert torch.all(o == 7.0) and torch.all(S_T == 7.0)
