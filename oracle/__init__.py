"""Float64 CPU oracle for the Kimi Delta Attention (KDA) forward pass.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this package.  The
CUDA library never reaches it, and it never reaches the CUDA library: the two
share nothing but the seeded input generator, which holds none of the method's
arithmetic.

What it computes (page title, then section):

* ``gate``        -- KDA notes, "Gate 激活", table "两种 Gate" and its itemised
  definitions (input = g_raw + dt_bias, rate = exp(A_log)).
* ``recurrent``   -- KDA notes, "KDA 递归核心", §逐步公式 steps 1-4; KDA ledger
  DER1; DeltaNet-family digest, "Kimi Delta Attention: channel-wise decay".
* ``forward``     -- gate (when asked) followed by ``recurrent``: the result the
  chunked prefill and the decode step must both reproduce.
* ``chunkwise``   -- DeltaNet-family digest, "Chunkwise KDA": an independent
  second algorithm, used only to pin ``recurrent``.
* ``dplr``        -- DeltaNet-family digest, "diagonal-low-rank transition": the
  same recurrence through explicit dense K x K transition matrices, a third
  independent form used only to pin ``recurrent``.
* ``input_side``  -- the op's optional input-side steps as a separate float64
  pre-step: q, k divided by their L2 norm over the K channels per token and
  head (the DeltaNet-family digest assumes L2-normalised keys), and beta taken
  as a logit through the logistic sigmoid (KDA notes, "KDA 递归核心": beta is the
  write strength, a value in (0, 1)).  ``forward`` applies it when asked.
* ``backward`` (module ``oracle.backward``) -- the reverse mode of ``forward``,
  derived step by step from the recurrence and the gates, pinned by central
  finite differences of ``forward``: the reference for a backward pass; and
  ``chunkwise_backward``, the reverse mode of the chunkwise equations, pinned
  against it.

Every pinned property is listed in the tests; nothing here is "parity
unpinned".  The compiled part lives in ``kda_oracle.c`` (plain C, float64,
OpenMP over independent (b, hv) pairs) and is built by ``build()``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "libkda_oracle.so")
# The mutation tests point this at a deliberately broken build of a copy of kda_oracle.c.
_LIB_OVERRIDE = os.environ.get("KDA_ORACLE_LIB")
_lock = threading.Lock()
_lib = None

GATE_NONE = 0
GATE_SAFE = 1
GATE_STANDARD = 2


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``libkda_oracle.so`` (gcc, -O2, OpenMP, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-fno-fast-math", "-fPIC", "-shared", "-std=c99",
           "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            dp = ctypes.POINTER(ctypes.c_double)
            lib.kda_oracle_gate.argtypes = [dp, dp, dp, ctypes.c_long, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_int, ctypes.c_double, dp]
            lib.kda_oracle_gate.restype = ctypes.c_int
            sig = [dp, dp, dp, dp, dp, dp] + [ctypes.c_int] * 6
            lib.kda_oracle_recurrent.argtypes = sig + [ctypes.c_double, dp, dp]
            lib.kda_oracle_recurrent.restype = None
            lib.kda_oracle_chunkwise.argtypes = sig + [ctypes.c_int, ctypes.c_double, dp, dp]
            lib.kda_oracle_chunkwise.restype = None
            lib.kda_oracle_num_threads.argtypes = []
            lib.kda_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def num_threads() -> int:
    """OpenMP threads the oracle's parallel loops use (capped in practice by B*HV)."""
    return int(_load().kda_oracle_num_threads())


def _f64(x):
    """Exact upcast of a numpy array or a CPU torch tensor (bf16 / fp32 / fp64) to float64."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast through torch, bit-exact
        import torch
        x = x.detach().to("cpu", torch.float64).contiguous().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def gate(g_raw, A_log, dt_bias=None, *, mode=GATE_SAFE, lower_bound=None):
    """Gate activation, float64.  g_raw [..., HV, K]; A_log [HV]; dt_bias [HV, K] or None.

    SAFE: ``lower_bound * sigmoid(exp(A_log) * (g_raw + dt_bias))``;
    STANDARD: ``-exp(A_log) * softplus(g_raw + dt_bias)``.
    """
    g_raw = _f64(g_raw)
    A_log = _f64(A_log)
    dt_bias = _f64(dt_bias)
    HV, K = g_raw.shape[-2:]
    if mode == GATE_SAFE and (lower_bound is None or not np.isfinite(lower_bound)):
        raise ValueError("safe gate needs a finite lower_bound")
    out = np.empty_like(g_raw)
    rows = g_raw.size // (HV * K)
    rc = _load().kda_oracle_gate(_ptr(g_raw), _ptr(A_log), _ptr(dt_bias), rows, HV, K, int(mode),
                                 float(lower_bound if lower_bound is not None else 0.0), _ptr(out))
    if rc != 0:
        raise ValueError(f"bad gate mode {mode}")
    return out


def _shapes(q, v):
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    if HV % H:
        raise ValueError("HV must be a multiple of H")
    return B, T, H, HV, K, V


def recurrent(q, k, v, g, beta, S0=None, *, scale=None):
    """Naive per-token KDA recurrence in float64; ``g`` is the log-space decay.

    Returns ``(o [B,T,HV,V], S_T [B,HV,K,V])`` as float64 numpy arrays.
    """
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, HV, K, V = _shapes(q, v)
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    o = np.empty((B, T, HV, V))
    S = np.empty((B, HV, K, V))
    _load().kda_oracle_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                 B, T, H, HV, K, V, float(scale), _ptr(o), _ptr(S))
    return o, S


def chunkwise(q, k, v, g, beta, S0=None, *, chunk=64, scale=None):
    """The pages' chunkwise equations in float64 (independent of ``recurrent``)."""
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, HV, K, V = _shapes(q, v)
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    o = np.empty((B, T, HV, V))
    S = np.empty((B, HV, K, V))
    _load().kda_oracle_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(S0),
                                 B, T, H, HV, K, V, int(chunk), float(scale), _ptr(o), _ptr(S))
    return o, S


def dplr(q, k, v, g, beta, S0=None, *, scale=None):
    """The recurrence as a diagonal-plus-low-rank transition, with dense matrices.

    DeltaNet-family digest, "diagonal-low-rank transition": in the value-major
    layout the update reads S_t = S_{t-1} A_t + beta_t v_t k_t^T with
    A_t = D_t (I - beta_t k_t k_t^T).  In this library's key-major layout that is
    S_t = A_t^T S_{t-1} + beta_t k_t v_t^T, i.e. (I - beta_t k_t k_t^T) D_t S_{t-1} + ...
    Built with explicit K x K numpy matrices; tiny inputs only.
    """
    q, k, v, g, beta, S0 = (_f64(x) for x in (q, k, v, g, beta, S0))
    B, T, H, HV, K, V = _shapes(q, v)
    G = HV // H
    if scale is None:
        scale = 1.0 / np.sqrt(K)
    o = np.empty((B, T, HV, V))
    S_out = np.empty((B, HV, K, V))
    eye = np.eye(K)
    for b in range(B):
        for hv in range(HV):
            h = hv // G
            S = np.zeros((K, V)) if S0 is None else S0[b, hv].copy()
            for t in range(T):
                kt = k[b, t, h][:, None]
                D = np.diag(np.exp(g[b, t, hv]))
                A = D @ (eye - beta[b, t, hv] * (kt @ kt.T))   # value-major transition
                S = A.T @ S + beta[b, t, hv] * (kt @ v[b, t, hv][None, :])
                o[b, t, hv] = scale * (q[b, t, h][None, :] @ S)[0]
            S_out[b, hv] = S
    return o, S_out


NORM_FLOOR = 1e-6  # a vector with a smaller norm is divided by this instead (a zero vector stays zero)


def input_side(q, k, beta, *, l2norm_qk=False, beta_logits=False):
    """The optional input-side steps, float64: returns ``(q, k, beta)``.

    ``l2norm_qk``: every q and k vector (last axis, the K channels of one token and head) is divided by
    ``max(||x||_2, NORM_FLOOR)``.  ``beta_logits``: beta is mapped through ``1 / (1 + exp(-beta))``.
    With both off the inputs come back unchanged (upcast to float64)."""
    q, k, beta = _f64(q), _f64(k), _f64(beta)
    if l2norm_qk:
        q = q / np.maximum(np.sqrt(np.sum(q * q, axis=-1, keepdims=True)), NORM_FLOOR)
        k = k / np.maximum(np.sqrt(np.sum(k * k, axis=-1, keepdims=True)), NORM_FLOOR)
    if beta_logits:
        beta = 1.0 / (1.0 + np.exp(-beta))
    return q, k, beta


def forward(q, k, v, g, beta, A_log=None, dt_bias=None, S0=None, *, gate_mode=GATE_NONE,
            lower_bound=None, scale=None, l2norm_qk=False, beta_logits=False):
    """The input-side steps (when asked), the gate (if ``gate_mode`` is SAFE or STANDARD, ``g`` holds
    g_raw), then the recurrence."""
    if l2norm_qk or beta_logits:
        q, k, beta = input_side(q, k, beta, l2norm_qk=l2norm_qk, beta_logits=beta_logits)
    if gate_mode != GATE_NONE:
        g = gate(g, A_log, dt_bias, mode=gate_mode, lower_bound=lower_bound)
    return recurrent(q, k, v, g, beta, S0, scale=scale)
