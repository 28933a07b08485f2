"""Host-side checks of the C ABI (no GPU needed): the library loads, exports every symbol
``include/kda.h`` declares, and rejects bad arguments with the documented status before
launching anything."""
import ctypes
import os
import re

import pytest

from kimi_delta_attention_33_b200 import kda

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "kda.h")
FAKE = 0x10000  # a 16-byte-aligned non-null address; validation fails before anything touches it


def _declared():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"\b(kda_[a-z_0-9]+)\s*\(", text)


def test_header_declarations_are_all_exported():
    names = _declared()
    assert names, "no declarations parsed"
    assert tuple(names) == kda.EXPORTS
    for n in names:
        assert hasattr(kda.lib, n), f"{n} not exported by libkda.so"


def test_version_and_empty_error():
    assert "sm_100a" in kda.version()
    assert isinstance(kda.last_error(), str)


def _chunk(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, A_log=FAKE, dt_bias=FAKE, S0=None, B=1, T=64, H=2, HV=2,
             K=128, V=128, chunk=64, gate=kda.GATE_SAFE, lb=-5.0, scale=-1.0, dtype=kda.BF16, o=FAKE * 2,
             S_T=None, ws=FAKE * 3, ws_bytes=1 << 20, stream=None)
    a.update(over)
    return kda.lib.kda_chunk_fwd(a["q"], a["k"], a["v"], a["g"], a["beta"], a["A_log"], a["dt_bias"], a["S0"], a["B"],
                                 a["T"], a["H"], a["HV"], a["K"], a["V"], a["chunk"], a["gate"], a["lb"], a["scale"],
                                 a["dtype"], a["o"], a["S_T"], a["ws"], a["ws_bytes"], a["stream"])


def _step(**over):
    a = dict(q=FAKE, k=FAKE, v=FAKE, g=FAKE, beta=FAKE, A_log=FAKE, dt_bias=None, B=4, H=2, HV=4, K=128, V=128,
             gate=kda.GATE_SAFE, lb=-5.0, scale=-1.0, dtype=kda.BF16, S=FAKE * 4, o=FAKE * 2, stream=None)
    a.update(over)
    return kda.lib.kda_recurrent_step(a["q"], a["k"], a["v"], a["g"], a["beta"], a["A_log"], a["dt_bias"], a["B"],
                                      a["H"], a["HV"], a["K"], a["V"], a["gate"], a["lb"], a["scale"], a["dtype"],
                                      a["S"], a["o"], a["stream"])


@pytest.mark.parametrize("over,status", [
    (dict(q=None), kda.ERR_INVALID_ARG),
    (dict(o=None), kda.ERR_INVALID_ARG),
    (dict(HV=3), kda.ERR_INVALID_ARG),
    (dict(B=0), kda.ERR_INVALID_ARG),
    (dict(T=0), kda.ERR_INVALID_ARG),
    (dict(K=48), kda.ERR_UNSUPPORTED),
    (dict(V=256), kda.ERR_UNSUPPORTED),
    (dict(chunk=32), kda.ERR_UNSUPPORTED),
    (dict(lb=float("nan")), kda.ERR_INVALID_ARG),
    (dict(lb=0.5), kda.ERR_INVALID_ARG),
    (dict(A_log=None), kda.ERR_INVALID_ARG),
    (dict(gate=7), kda.ERR_INVALID_ARG),
    (dict(dtype=5), kda.ERR_INVALID_ARG),
    (dict(v=FAKE + 4), kda.ERR_INVALID_ARG),
    (dict(ws=None), kda.ERR_INVALID_ARG),
    (dict(ws_bytes=16), kda.ERR_INVALID_ARG),
    (dict(o=FAKE), kda.ERR_INVALID_ARG),
])
def test_chunk_fwd_rejects_bad_arguments(over, status):
    assert _chunk(**over) == status
    assert kda.last_error() != ""


@pytest.mark.parametrize("over,status", [
    (dict(S=None), kda.ERR_INVALID_ARG),
    (dict(beta=None), kda.ERR_INVALID_ARG),
    (dict(HV=6, H=4), kda.ERR_INVALID_ARG),
    (dict(K=100), kda.ERR_UNSUPPORTED),
    (dict(gate=kda.GATE_SAFE, lb=float("inf")), kda.ERR_INVALID_ARG),
    (dict(o=FAKE * 4), kda.ERR_INVALID_ARG),
    (dict(S=FAKE * 4 + 8), kda.ERR_INVALID_ARG),
])
def test_recurrent_step_rejects_bad_arguments(over, status):
    assert _step(**over) == status
    assert kda.last_error() != ""


def test_gate_rejects_bad_arguments():
    L = kda.lib
    assert L.kda_gate(None, kda.BF16, FAKE, None, 1, 1, 1, 16, kda.GATE_SAFE, -5.0, FAKE, None) == kda.ERR_INVALID_ARG
    assert L.kda_gate(FAKE, kda.BF16, FAKE, None, 1, 1, 1, 16, kda.GATE_NONE, -5.0, FAKE, None) == kda.ERR_INVALID_ARG
    assert L.kda_gate(FAKE, kda.BF16, FAKE, None, 1, 1, 1, 16, kda.GATE_SAFE, float("nan"), FAKE,
                      None) == kda.ERR_INVALID_ARG
    assert L.kda_gate(FAKE, kda.BF16, FAKE, None, 0, 1, 1, 16, kda.GATE_STANDARD, 0.0, FAKE,
                      None) == kda.ERR_INVALID_ARG


def test_workspace_size():
    assert kda.workspace_size(2, 1024, 4, 8, 128, 128, 64) >= 256
    assert kda.workspace_size(1, 64, 2, 2, 16, 16, 16) >= 256
    assert kda.workspace_size(1, 64, 2, 3, 16, 16, 16) == 0
    assert kda.workspace_size(1, 64, 2, 2, 16, 16, 32) == 0
    assert kda.workspace_size(1, 64, 2, 2, 24, 16, 16) == 0


def test_read_status_rejects_null():
    assert kda.lib.kda_read_status(None, None) == kda.ERR_INVALID_ARG


def test_workspace_size_two_pass_records():
    # K = V = 128, chunk 64: the status block plus one 115712-byte record per chunk per (b, hv)
    B, T, HV = 2, 1000, 8
    nc = (T + 63) // 64
    assert kda.workspace_size(B, T, 4, HV, 128, 128, 64) == 256 + B * HV * nc * 115712
    assert kda.workspace_size(B, T, 4, HV, 128, 64, 64) == 256
    assert kda.workspace_size(B, T, 4, HV, 128, 128, 16) == 256
    assert kda.workspace_size(12, T, 8, 8, 128, 128, 64) == 256 + 12 * 8 * nc * 115712  # 96 pairs
    assert kda.workspace_size(13, T, 8, 8, 128, 128, 64) == 256                          # 104 pairs


def test_schedule_choice():
    L = kda.lib
    full = kda.workspace_size(2, 1000, 4, 8, 128, 128, 64)
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, kda.BF16, full) == kda.SCHEDULE_TC_TWO_PASS
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, kda.BF16, full - 1) == kda.SCHEDULE_TC_SINGLE_PASS
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, kda.BF16, 256) == kda.SCHEDULE_TC_SINGLE_PASS
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, kda.F32, full) == kda.SCHEDULE_CUDA_CORE
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 64, 128, 64, kda.BF16, full) == kda.SCHEDULE_CUDA_CORE
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 16, kda.BF16, full) == kda.SCHEDULE_CUDA_CORE
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, kda.BF16, 255) == -1
    assert L.kda_chunk_fwd_schedule(2, 1000, 3, 8, 128, 128, 64, kda.BF16, full) == -1
    assert L.kda_chunk_fwd_schedule(2, 1000, 4, 8, 128, 128, 64, 9, full) == -1
    assert kda.schedule(2, 1000, 4, 8, 128, 128, 64) == kda.SCHEDULE_TC_TWO_PASS
    assert L.kda_chunk_fwd_schedule(8, 1000, 16, 16, 128, 128, 64, kda.BF16, 1 << 40) == kda.SCHEDULE_TC_SINGLE_PASS
    assert kda.uses_tensor_cores(128, 128, 64) and not kda.uses_tensor_cores(64, 64, 64)


def test_split_state_pass_plan():
    # The state pass splits along the sequence only where the unsplit chains leave the SMs idle: a few (sequence, head)
    # pairs with long sequences.  The benchmark workloads 2 (16 pairs x 16 chunks) and 4 (32 pairs x 1024 chunks) keep
    # one chain per value block; 4 pairs x 79 chunks and 1 pair x 94 chunks split (the GPU scan tests' shapes).
    L = kda.lib
    def plan(B, T, H, HV):
        return L.kda_chunk_fwd_schedule(B, T, H, HV, 128, 128, 64, kda.BF16, kda.workspace_size(B, T, H, HV, 128, 128, 64))
    assert plan(2, 1024, 4, 8) == kda.SCHEDULE_TC_TWO_PASS
    assert plan(1, 65536, 8, 32) == kda.SCHEDULE_TC_TWO_PASS
    assert plan(1, 5000, 2, 4) == kda.SCHEDULE_TC_TWO_PASS_SCAN
    assert plan(1, 6000, 1, 1) == kda.SCHEDULE_TC_TWO_PASS_SCAN
    assert kda.schedule_launches(1, 5000, 2, 4, 128, 128, 64) == 4   # prep, carry, segment chain, outputs
    assert kda.schedule_launches(1, 65536, 8, 32, 128, 128, 64) == 2  # prep, state


def test_two_pass_limits():
    L = kda.lib
    # token stride (HV x 256 bytes) x T must stay below 2^40 bytes for the prep pass's tensor maps
    T = 1 << 27  # 32 heads x 256 B x 2^27 = 2^40
    assert kda.workspace_size(1, T, 8, 32, 128, 128, 64) == 256
    assert L.kda_chunk_fwd_schedule(1, T, 8, 32, 128, 128, 64, kda.BF16, 1 << 62) == kda.SCHEDULE_TC_SINGLE_PASS
    assert kda.workspace_size(1, T - 64, 8, 32, 128, 128, 64) > 256
    # fewer than 2^30 chunks in all: 64 pairs x 2^24 chunks of 64 tokens is 2^30
    T2 = 1 << 30
    assert kda.workspace_size(64, T2, 1, 1, 128, 128, 64) == 256
    assert kda.workspace_size(64, T2 - 64, 1, 1, 128, 128, 64) > 256


def test_input_option_entry_points_validate_before_launch():
    L = kda.lib
    # unknown flag bits
    assert L.kda_chunk_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, 2, 128, 128, 64,
                              kda.GATE_SAFE, -5.0, -1.0, kda.BF16, 8, FAKE * 2, None, FAKE * 3, 1 << 20,
                              None) == kda.ERR_INVALID_ARG
    assert L.kda_recurrent_step_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 2, 4, 128, 128, kda.GATE_SAFE, -5.0,
                                   -1.0, kda.BF16, 4, FAKE * 4, FAKE * 2, None) == kda.ERR_INVALID_ARG
    # the documented flags pass validation and fail on the next bad argument as kda_chunk_fwd does
    flags = kda.INPUT_L2NORM_QK | kda.INPUT_BETA_LOGITS
    assert L.kda_chunk_fwd_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, None, 1, 64, 2, 2, 128, 128, 32,
                              kda.GATE_SAFE, -5.0, -1.0, kda.BF16, flags, FAKE * 2, None, FAKE * 3, 1 << 20,
                              None) == kda.ERR_UNSUPPORTED
    assert L.kda_recurrent_step_ex(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 4, 2, 4, 128, 128, kda.GATE_SAFE, -5.0,
                                   -1.0, kda.BF16, flags, None, FAKE * 2, None) == kda.ERR_INVALID_ARG


def test_backward_validates_before_launch():
    L = kda.lib
    # the states saved every 8 tokens, the fp32 decays of every (token, value head, key channel) and the fp32
    # residuals of every (token, value head, value column)
    assert kda.backward_workspace_size(2, 100, 2, 4, 128, 64) == (2 * 4 * 13 * 128 * 64 + 2 * 100 * 4 * (128 + 64)) * 4
    assert kda.backward_workspace_size(2, 100, 3, 4, 128, 64) == 0

    def call(**over):
        a = dict(q=FAKE, dq=FAKE * 5, K=128, ws_bytes=1 << 30, gate=kda.GATE_SAFE, lb=-5.0, HV=4, H=2)
        a.update(over)
        return L.kda_backward(a["q"], FAKE, FAKE, FAKE, FAKE, FAKE, None, None, FAKE * 2, None, 2, 100, a["H"],
                              a["HV"], a["K"], 64, a["gate"], a["lb"], -1.0, kda.BF16, a["dq"], FAKE * 6, FAKE * 7,
                              FAKE * 8, FAKE * 9, None, None, None, FAKE * 3, a["ws_bytes"], None)
    assert call(q=None) == kda.ERR_INVALID_ARG
    assert call(dq=None) == kda.ERR_INVALID_ARG
    assert call(K=48) == kda.ERR_UNSUPPORTED
    assert call(HV=3) == kda.ERR_INVALID_ARG
    assert call(lb=float("nan")) == kda.ERR_INVALID_ARG
    assert call(ws_bytes=1024) == kda.ERR_INVALID_ARG
    assert call(dq=FAKE) == kda.ERR_INVALID_ARG  # an output aliasing an input
    assert kda.last_error() != ""


def test_mla_decode_validates_before_launch():
    L = kda.lib
    assert kda.mla_decode_workspace_size(64, 4096, 96, 128, 128, 512) > 0
    assert kda.mla_decode_workspace_size(64, 4096, 96, 96, 128, 512) == 0
    assert kda.mla_decode_workspace_size(64, 4096, 96, 128, 128, 1024) == 0

    def call(**over):
        a = dict(q=FAKE, o=FAKE * 5, dq=128, r=512, dtype=kda.BF16, ws=1 << 30, H=96)
        a.update(over)
        return L.kda_mla_decode(a["q"], FAKE * 2, FAKE * 3, FAKE * 4, None, 4, 64, a["H"], a["dq"], 128, a["r"], -1.0,
                                a["dtype"], a["o"], FAKE * 6, a["ws"], None)
    assert call(q=None) == kda.ERR_INVALID_ARG
    assert call(dq=96) == kda.ERR_UNSUPPORTED
    assert call(r=64) == kda.ERR_UNSUPPORTED
    assert call(dtype=kda.F32) == kda.ERR_UNSUPPORTED
    assert call(ws=16) == kda.ERR_INVALID_ARG
    assert call(o=FAKE) == kda.ERR_INVALID_ARG
    assert call(H=0) == kda.ERR_INVALID_ARG
