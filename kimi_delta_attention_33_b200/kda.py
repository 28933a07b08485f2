"""Python binding of ``libkda.so`` (the C ABI in ``include/kda.h``).

Argument marshalling only: every step of the forward pass runs in the library's
CUDA kernels.  PyTorch provides device memory and the current stream.  There is
no fallback of any kind -- importing this module raises if the shared library is
missing, and each call raises ``KdaError`` with the library's own message when
the C ABI returns an error status.

Functions mirror the C entry points:

* ``gate(g_raw, A_log, dt_bias, mode, lower_bound)``  -> float32 log decay
* ``chunk_fwd(q, k, v, g, beta, ...)``                 -> (o, S_T)
* ``recurrent_step(q, k, v, g, beta, S, ...)``         -> o  (S updated in place)
* ``read_status(workspace)``                           -> synchronise and check the device status word
* ``schedule(B, T, H, HV, K, V, chunk, dtype, ws)``     -> which kernels ``chunk_fwd`` runs
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkda.so")

GATE_NONE, GATE_SAFE, GATE_STANDARD = 0, 1, 2
F32, BF16 = 0, 1
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_TIMEOUT = 0, 1, 2, 3, 4
STATUS_NAMES = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_CUDA",
                4: "KDA_ERR_TIMEOUT"}

# Every symbol include/kda.h declares, in declaration order.
EXPORTS = ("kda_last_error", "kda_version", "kda_gate", "kda_chunk_fwd_workspace_size", "kda_chunk_fwd",
           "kda_chunk_fwd_ex", "kda_chunk_fwd_schedule", "kda_read_status", "kda_chunk_fwd_noalloc",
           "kda_chunk_fwd_noalloc_read_status", "kda_recurrent_step", "kda_recurrent_step_ex",
           "kda_backward_workspace_size", "kda_backward", "kda_mla_decode_workspace_size", "kda_mla_decode")
INPUT_RAW, INPUT_L2NORM_QK, INPUT_BETA_LOGITS = 0, 1, 2
SCHEDULE_CUDA_CORE, SCHEDULE_TC_SINGLE_PASS, SCHEDULE_TC_TWO_PASS, SCHEDULE_TC_TWO_PASS_SCAN = 0, 1, 2, 3
SCHEDULE_NAMES = {0: "cuda_core", 1: "tc_single_pass", 2: "tc_two_pass", 3: "tc_two_pass_scan"}
# kernels one kda_chunk_fwd call launches, per schedule
SCHEDULE_LAUNCHES = {0: 1, 1: 1, 2: 2, 3: 4}


class KdaError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {message}")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(f"{LIB_PATH} is missing: build it with `python -m kimi_delta_attention_33_b200.build` "
                      "(this package has no fallback path)")

lib = ctypes.CDLL(LIB_PATH)
_vp, _fp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.kda_last_error.restype = ctypes.c_char_p
lib.kda_last_error.argtypes = []
lib.kda_version.restype = ctypes.c_char_p
lib.kda_version.argtypes = []
lib.kda_gate.restype = _i
lib.kda_gate.argtypes = [_vp, _i, _fp, _fp, _i, _i, _i, _i, _i, _f, _fp, _vp]
lib.kda_chunk_fwd_workspace_size.restype = _sz
lib.kda_chunk_fwd_workspace_size.argtypes = [_i] * 7
lib.kda_chunk_fwd.restype = _i
lib.kda_chunk_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp, _fp] + [_i] * 7 + [_i, _f, _f, _i, _vp, _fp, _vp,
                                                                                  _sz, _vp]
lib.kda_chunk_fwd_ex.restype = _i
lib.kda_chunk_fwd_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp, _fp] + [_i] * 7 + [_i, _f, _f, _i, ctypes.c_uint,
                                                                                     _vp, _fp, _vp, _sz, _vp]
lib.kda_chunk_fwd_schedule.restype = _i
lib.kda_chunk_fwd_schedule.argtypes = [_i] * 7 + [_i, _sz]
lib.kda_read_status.restype = _i
lib.kda_read_status.argtypes = [_vp, _vp]
lib.kda_chunk_fwd_noalloc.restype = _i
lib.kda_chunk_fwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp, _fp] + [_i] * 7 + [_i, _f, _f, _i, _vp, _fp,
                                                                                          _vp]
lib.kda_chunk_fwd_noalloc_read_status.restype = _i
lib.kda_chunk_fwd_noalloc_read_status.argtypes = [_vp]
lib.kda_recurrent_step.restype = _i
lib.kda_recurrent_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp] + [_i] * 5 + [_i, _f, _f, _i, _fp, _vp, _vp]
lib.kda_recurrent_step_ex.restype = _i
lib.kda_recurrent_step_ex.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp] + [_i] * 5 + [_i, _f, _f, _i, ctypes.c_uint,
                                                                                     _fp, _vp, _vp]


lib.kda_backward_workspace_size.restype = _sz
lib.kda_backward_workspace_size.argtypes = [_i] * 6
lib.kda_backward.restype = _i
lib.kda_backward.argtypes = [_vp, _vp, _vp, _vp, _vp, _fp, _fp, _fp, _vp, _fp] + [_i] * 6 + [_i, _f, _f, _i] + \
    [_fp] * 8 + [_vp, _sz, _vp]


lib.kda_mla_decode_workspace_size.restype = _sz
lib.kda_mla_decode_workspace_size.argtypes = [_i] * 6
lib.kda_mla_decode.restype = _i
lib.kda_mla_decode.argtypes = [_vp, _vp, _vp, _vp, _vp] + [_i] * 6 + [_f, _i, _vp, _vp, _sz, _vp]


def version() -> str:
    return lib.kda_version().decode()


def last_error() -> str:
    return lib.kda_last_error().decode()


def _check(status: int):
    if status != OK:
        raise KdaError(status, last_error())


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise KdaError(ERR_UNSUPPORTED, f"per-token tensors must be bfloat16 or float32, got {t.dtype}")


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _require_cuda(*ts):
    for t in ts:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise KdaError(ERR_INVALID_ARG, "tensors must be contiguous CUDA tensors")


def _require_out(t, shape, dtype):
    if not t.is_cuda or not t.is_contiguous() or tuple(t.shape) != tuple(shape) or t.dtype != dtype:
        raise KdaError(ERR_INVALID_ARG, f"output tensor must be a contiguous CUDA tensor of shape {tuple(shape)} "
                                        f"and dtype {dtype} (got {tuple(t.shape)}, {t.dtype}, "
                                        f"contiguous={t.is_contiguous()})")


def gate(g_raw: torch.Tensor, A_log: torch.Tensor, dt_bias: torch.Tensor | None = None, *, mode: int = GATE_SAFE,
         lower_bound: float | None = None, out: torch.Tensor | None = None) -> torch.Tensor:
    """Gate activation.  g_raw [B, T, HV, K] -> float32 log decay of the same shape."""
    _require_cuda(g_raw, A_log, dt_bias)
    B, T, HV, K = g_raw.shape
    if out is None:
        out = torch.empty(g_raw.shape, dtype=torch.float32, device=g_raw.device)
    _require_out(out, g_raw.shape, torch.float32)
    lb = float("nan") if lower_bound is None else float(lower_bound)
    _check(lib.kda_gate(_ptr(g_raw), _dtype_code(g_raw), _ptr(A_log), _ptr(dt_bias), B, T, HV, K, int(mode), lb,
                        _ptr(out), _stream(g_raw.device)))
    return out


def workspace_size(B, T, H, HV, K, V, chunk) -> int:
    return int(lib.kda_chunk_fwd_workspace_size(B, T, H, HV, K, V, chunk))


def _input_flags(l2norm_qk: bool, beta_logits: bool) -> int:
    return (INPUT_L2NORM_QK if l2norm_qk else 0) | (INPUT_BETA_LOGITS if beta_logits else 0)


def chunk_fwd(q, k, v, g, beta, A_log=None, dt_bias=None, S0=None, *, chunk: int = 64,
              gate_mode: int = GATE_NONE, lower_bound: float | None = None, scale: float | None = None,
              output_final_state: bool = True, S_T: torch.Tensor | None = None, o: torch.Tensor | None = None,
              workspace: torch.Tensor | None = None, check_status: bool = False, l2norm_qk: bool = False,
              beta_logits: bool = False):
    """Chunked prefill.  q, k [B,T,H,K]; v [B,T,HV,V]; g [B,T,HV,K] (g_raw if gate_mode != NONE);
    beta [B,T,HV]; S0 [B,HV,K,V] fp32 or None.  Returns ``(o, S_T)`` (``S_T`` None unless requested).
    ``l2norm_qk`` / ``beta_logits`` select the in-kernel input steps (``kda_chunk_fwd_ex``)."""
    _require_cuda(q, k, v, g, beta, A_log, dt_bias, S0)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty((B, T, HV, V), dtype=q.dtype, device=q.device)
    if S_T is None and output_final_state:
        S_T = torch.empty((B, HV, K, V), dtype=torch.float32, device=q.device)
    _require_out(o, (B, T, HV, V), q.dtype)
    if S_T is not None:
        _require_out(S_T, (B, HV, K, V), torch.float32)
    need = workspace_size(B, T, H, HV, K, V, chunk)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    lb = float("nan") if lower_bound is None else float(lower_bound)
    sc = -1.0 if scale is None else float(scale)
    flags = _input_flags(l2norm_qk, beta_logits)
    if flags == 0:
        _check(lib.kda_chunk_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                                 _ptr(S0), B, T, H, HV, K, V, int(chunk), int(gate_mode), lb, sc, _dtype_code(q),
                                 _ptr(o), _ptr(S_T), _ptr(workspace), workspace.numel(), _stream(q.device)))
    else:
        _check(lib.kda_chunk_fwd_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                                    _ptr(S0), B, T, H, HV, K, V, int(chunk), int(gate_mode), lb, sc, _dtype_code(q),
                                    flags, _ptr(o), _ptr(S_T), _ptr(workspace), workspace.numel(),
                                    _stream(q.device)))
    if check_status:
        read_status(workspace)
    return o, S_T


def chunk_fwd_noalloc(q, k, v, g, beta, A_log=None, dt_bias=None, S0=None, *, chunk: int = 64,
                      gate_mode: int = GATE_NONE, lower_bound: float | None = None, scale: float | None = None,
                      S_T: torch.Tensor | None = None, o: torch.Tensor | None = None):
    """``chunk_fwd`` through ``kda_chunk_fwd_noalloc``: the library supplies the workspace from its own
    fixed device array, for callers that cannot allocate one.  Outputs are still passed in (or made
    here by torch when omitted)."""
    _require_cuda(q, k, v, g, beta, A_log, dt_bias, S0)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    if o is None:
        o = torch.empty((B, T, HV, V), dtype=q.dtype, device=q.device)
    if S_T is None:
        S_T = torch.empty((B, HV, K, V), dtype=torch.float32, device=q.device)
    _require_out(o, (B, T, HV, V), q.dtype)
    _require_out(S_T, (B, HV, K, V), torch.float32)
    lb = float("nan") if lower_bound is None else float(lower_bound)
    sc = -1.0 if scale is None else float(scale)
    _check(lib.kda_chunk_fwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                                     _ptr(S0), B, T, H, HV, K, V, int(chunk), int(gate_mode), lb, sc, _dtype_code(q),
                                     _ptr(o), _ptr(S_T), _stream(q.device)))
    return o, S_T


def noalloc_read_status(device=None):
    """Synchronise the current stream and raise ``KdaError`` if the last ``chunk_fwd_noalloc`` call on
    this device had a bounded wait give up."""
    _check(lib.kda_chunk_fwd_noalloc_read_status(_stream(device)))


def read_status(workspace: torch.Tensor):
    """Synchronise the current stream and raise ``KdaError`` if a chunk call's bounded wait gave up."""
    _check(lib.kda_read_status(_ptr(workspace), _stream(workspace.device)))


def recurrent_step(q, k, v, g, beta, S, A_log=None, dt_bias=None, *, gate_mode: int = GATE_NONE,
                   lower_bound: float | None = None, scale: float | None = None, o: torch.Tensor | None = None,
                   l2norm_qk: bool = False, beta_logits: bool = False):
    """One fused decode step.  q, k [B,H,K] (or [B,1,H,K]); v [B,HV,V]; g [B,HV,K]; beta [B,HV];
    S [B,HV,K,V] fp32 updated in place.  Returns o [B,HV,V] (shaped like v)."""
    _require_cuda(q, k, v, g, beta, S, A_log, dt_bias)
    B, H, K = q.shape[0], q.shape[-2], q.shape[-1]
    HV, V = v.shape[-2], v.shape[-1]
    if o is None:
        o = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    _require_out(o, v.shape, q.dtype)
    _require_out(S, (B, HV, K, V), torch.float32)
    lb = float("nan") if lower_bound is None else float(lower_bound)
    sc = -1.0 if scale is None else float(scale)
    flags = _input_flags(l2norm_qk, beta_logits)
    if flags == 0:
        _check(lib.kda_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias),
                                      B, H, HV, K, V, int(gate_mode), lb, sc, _dtype_code(q), _ptr(S), _ptr(o),
                                      _stream(q.device)))
    else:
        _check(lib.kda_recurrent_step_ex(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log),
                                         _ptr(dt_bias), B, H, HV, K, V, int(gate_mode), lb, sc, _dtype_code(q),
                                         flags, _ptr(S), _ptr(o), _stream(q.device)))
    return o


def backward_workspace_size(B, T, H, HV, K, V) -> int:
    return int(lib.kda_backward_workspace_size(B, T, H, HV, K, V))


def backward(q, k, v, g, beta, dO, A_log=None, dt_bias=None, S0=None, dS_T=None, *, gate_mode: int = GATE_NONE,
             lower_bound: float | None = None, scale: float | None = None, need_dS0: bool = True,
             workspace: torch.Tensor | None = None, out: dict | None = None) -> dict:
    """Reverse mode of ``chunk_fwd`` (``kda_backward``): gradients of a loss given ``dO`` (and ``dS_T``).
    Returns a dict of float32 tensors ``dq, dk, dv, dg, dbeta`` (+ ``dS0``; + ``dA_log, ddt_bias`` when a
    gate ran); ``dg`` is the gradient with respect to the ``g`` argument (g_raw when a gate ran)."""
    _require_cuda(q, k, v, g, beta, dO, A_log, dt_bias, S0, dS_T)
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    dev = q.device
    f32 = dict(dtype=torch.float32, device=dev)
    o = out if out is not None else {}
    o.setdefault("dq", torch.empty(B, T, H, K, **f32))
    o.setdefault("dk", torch.empty(B, T, H, K, **f32))
    o.setdefault("dv", torch.empty(B, T, HV, V, **f32))
    o.setdefault("dg", torch.empty(B, T, HV, K, **f32))
    o.setdefault("dbeta", torch.empty(B, T, HV, **f32))
    if need_dS0:
        o.setdefault("dS0", torch.empty(B, HV, K, V, **f32))
    if gate_mode != GATE_NONE:
        o.setdefault("dA_log", torch.empty(HV, **f32))
        if dt_bias is not None:
            o.setdefault("ddt_bias", torch.empty(HV, K, **f32))
    need = backward_workspace_size(B, T, H, HV, K, V)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    lb = float("nan") if lower_bound is None else float(lower_bound)
    sc = -1.0 if scale is None else float(scale)
    _check(lib.kda_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(A_log), _ptr(dt_bias), _ptr(S0),
                            _ptr(dO), _ptr(dS_T), B, T, H, HV, K, V, int(gate_mode), lb, sc, _dtype_code(q),
                            _ptr(o["dq"]), _ptr(o["dk"]), _ptr(o["dv"]), _ptr(o["dg"]), _ptr(o["dbeta"]),
                            _ptr(o.get("dS0")), _ptr(o.get("dA_log")), _ptr(o.get("ddt_bias")), _ptr(workspace),
                            workspace.numel(), _stream(dev)))
    return o


def mla_decode_workspace_size(B, T, H, d_q, d_v, r) -> int:
    return int(lib.kda_mla_decode_workspace_size(B, T, H, d_q, d_v, r))


def mla_decode(q, W_UK, W_UV, c, lengths=None, *, scale: float | None = None, o: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None) -> torch.Tensor:
    """Absorbed MLA decode (``kda_mla_decode``).  q [B,H,d_q], W_UK [H,d_q,r], W_UV [H,d_v,r], c [B,T,r] (bf16);
    lengths [B] int32 or None.  Returns o [B,H,d_v] bf16."""
    _require_cuda(q, W_UK, W_UV, c, lengths)
    B, H, d_q = q.shape
    T, r = c.shape[1], c.shape[2]
    d_v = W_UV.shape[1]
    if o is None:
        o = torch.empty(B, H, d_v, dtype=q.dtype, device=q.device)
    _require_out(o, (B, H, d_v), q.dtype)
    if lengths is not None and lengths.dtype != torch.int32:
        raise KdaError(ERR_INVALID_ARG, "lengths must be int32")
    need = mla_decode_workspace_size(B, T, H, d_q, d_v, r)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=q.device)
    sc = -1.0 if scale is None else float(scale)
    _check(lib.kda_mla_decode(_ptr(q), _ptr(W_UK), _ptr(W_UV), _ptr(c), _ptr(lengths), B, T, H, d_q, d_v, r, sc,
                              _dtype_code(q), _ptr(o), _ptr(workspace), workspace.numel(), _stream(q.device)))
    return o


def schedule(B, T, H, HV, K, V, chunk, dtype: torch.dtype = torch.bfloat16, workspace_bytes: int | None = None) -> int:
    """The schedule kda_chunk_fwd runs for these sizes (SCHEDULE_* value); ``workspace_bytes`` defaults
    to ``workspace_size(...)``, the size ``chunk_fwd`` allocates when given no workspace."""
    if workspace_bytes is None:
        workspace_bytes = max(workspace_size(B, T, H, HV, K, V, chunk), 256)
    code = F32 if dtype == torch.float32 else BF16
    s = int(lib.kda_chunk_fwd_schedule(B, T, H, HV, K, V, chunk, code, workspace_bytes))
    if s < 0:
        raise KdaError(ERR_INVALID_ARG, "kda_chunk_fwd rejects these sizes")
    return s


def schedule_launches(B, T, H, HV, K, V, chunk, dtype: torch.dtype = torch.bfloat16,
                      workspace_bytes: int | None = None) -> int:
    """Number of kernels one ``chunk_fwd`` call launches for these sizes and workspace."""
    return SCHEDULE_LAUNCHES[schedule(B, T, H, HV, K, V, chunk, dtype, workspace_bytes)]


def uses_tensor_cores(K: int, V: int, chunk: int, dtype: torch.dtype = torch.bfloat16) -> bool:
    """Whether kda_chunk_fwd runs these sizes on a tensor-core schedule (else the CUDA-core kernel)."""
    return schedule(1, 1, 1, 1, K, V, chunk, dtype, 256) != SCHEDULE_CUDA_CORE


def default_scale(K: int) -> float:
    return 1.0 / math.sqrt(K)
