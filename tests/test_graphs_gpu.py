"""CUDA-graph capture of the library's entry points (how a serving loop replays them).

Each entry point only enqueues work on the caller's stream (kernel launches, one small memset of
the status word) and allocates nothing, so it can be captured into a CUDA graph once and replayed
with new inputs copied into the captured buffers.  Replays must reproduce direct calls bit for bit.
"""
import pytest
import torch

from kimi_delta_attention_33_b200 import kda
from kimi_delta_attention_33_b200.inputs import GATE_SAFE, Workload, make_inputs
from parity_util import to_dev

pytestmark = pytest.mark.gpu


def _prefill_case(B, HV, T):
    return Workload(96, "graph", B, T, 2, HV, 128, 128, 64, torch.bfloat16, GATE_SAFE, -5.0, (-0.5, 0.5), -4.0, 0.1,
                    0.02)


@pytest.mark.parametrize("B,HV,T,small_ws", [(2, 4, 200, False), (2, 4, 200, True), (1, 8, 130, False)])
def test_prefill_graph_replay_matches_direct_calls(B, HV, T, small_ws):
    w = _prefill_case(B, HV, T)
    xa, xb = to_dev(make_inputs(w, seed=21)), to_dev(make_inputs(w, seed=22))
    need = 256 if small_ws else kda.workspace_size(w.B, w.T, w.H, w.HV, w.K, w.V, w.chunk)
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    names = ("q", "k", "v", "g", "beta", "S0", "A_log", "dt_bias")  # every input lives in a captured buffer
    buf = {n: xa[n].clone() for n in names}
    o = torch.empty(w.B, w.T, w.HV, w.V, dtype=w.dtype, device="cuda")
    S_T = torch.empty(w.B, w.HV, w.K, w.V, dtype=torch.float32, device="cuda")

    def call():
        kda.chunk_fwd(buf["q"], buf["k"], buf["v"], buf["g"], buf["beta"], buf["A_log"], buf["dt_bias"], buf["S0"],
                      chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=o, S_T=S_T, workspace=ws)

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        call()  # warm-up outside the capture (first-call set-up)
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for x in (xb, xa):
        for n in names:
            buf[n].copy_(x[n])
        graph.replay()
        torch.cuda.synchronize()
        kda.read_status(ws)
        o_ref, S_ref = kda.chunk_fwd(x["q"], x["k"], x["v"], x["g"], x["beta"], x["A_log"], x["dt_bias"], x["S0"],
                                     chunk=64, gate_mode=w.gate_mode, lower_bound=w.lower_bound,
                                     workspace=torch.empty(need, dtype=torch.uint8, device="cuda"))
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(S_T, S_ref)


def test_decode_graph_of_several_steps():
    B, H, HV, K, V, steps = 8, 4, 8, 128, 128, 6
    w = Workload(95, "graph decode", B, steps, H, HV, K, V, 64, torch.bfloat16, GATE_SAFE, -5.0, None, -4.0, 0.0, 0.02)
    x = to_dev(make_inputs(w, seed=31))
    per = {n: x[n].transpose(0, 1).contiguous() for n in ("q", "k", "v", "g", "beta")}  # [steps, B, ...]
    S = x["S0"].clone()
    outs = torch.empty(steps, B, HV, V, dtype=w.dtype, device="cuda")

    def run_steps(state):
        for t in range(steps):
            kda.recurrent_step(per["q"][t], per["k"][t], per["v"][t], per["g"][t], per["beta"][t], state, x["A_log"],
                               x["dt_bias"], gate_mode=w.gate_mode, lower_bound=w.lower_bound, o=outs[t])

    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        run_steps(x["S0"].clone())
    torch.cuda.current_stream().wait_stream(s)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run_steps(S)
    S.copy_(x["S0"])
    graph.replay()
    torch.cuda.synchronize()
    got_o, got_S = outs.clone(), S.clone()
    S_ref = x["S0"].clone()
    ref = []
    for t in range(steps):
        ref.append(kda.recurrent_step(per["q"][t], per["k"][t], per["v"][t], per["g"][t], per["beta"][t], S_ref,
                                      x["A_log"], x["dt_bias"], gate_mode=w.gate_mode, lower_bound=w.lower_bound))
    torch.cuda.synchronize()
    assert torch.equal(got_o, torch.stack(ref)) and torch.equal(got_S, S_ref)
