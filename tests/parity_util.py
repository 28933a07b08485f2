"""Shared helpers for the GPU parity tests: run the CUDA path, run the oracle on the same bits, compare."""
from __future__ import annotations

import os

import numpy as np
import torch

import oracle
from kimi_delta_attention_33_b200.inputs import make_inputs

# Tolerances stated for the forward pass: max|x - x_ref| / max|x_ref| per output tensor.
TOL = {torch.float32: 1e-4, torch.bfloat16: 5e-3}


# Every relative error measured in this session, as (test id, error), in call order; the terminal
# summary (conftest.py) prints them so the headroom under the bar is visible in every run.
ERRORS: list = []


def rel_err(x, ref) -> float:
    x = np.asarray(x.detach().cpu().double() if hasattr(x, "detach") else x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert np.all(np.isfinite(x)), "non-finite values in GPU output"
    denom = np.abs(ref).max()
    err = float(np.abs(x - ref).max() / (denom if denom > 0 else 1.0))
    test = os.environ.get("PYTEST_CURRENT_TEST", "?").split(" ")[0]
    ERRORS.append((test, err))
    return err


def to_dev(x: dict, device="cuda") -> dict:
    return {k: (v.to(device) if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def oracle_pairs(x: dict, w, pairs, *, S0_override=None, gate_mode=None, lower_bound=None):
    """Oracle (o, S_T) for a list of (b, hv) pairs, each on its own sliced inputs at full T."""
    G = w.HV // w.H
    gm = w.gate_mode if gate_mode is None else gate_mode
    lb = w.lower_bound if lower_bound is None else lower_bound
    out = []
    S0 = x["S0"] if S0_override is None else S0_override
    for b, hv in pairs:
        h = hv // G
        s0 = None if S0 is None else S0[b:b + 1, hv:hv + 1]
        dtb = None if x.get("dt_bias") is None else x["dt_bias"][hv:hv + 1]
        o, S = oracle.forward(x["q"][b:b + 1, :, h:h + 1], x["k"][b:b + 1, :, h:h + 1], x["v"][b:b + 1, :, hv:hv + 1],
                              x["g"][b:b + 1, :, hv:hv + 1], x["beta"][b:b + 1, :, hv:hv + 1],
                              x["A_log"][hv:hv + 1], dtb, s0, gate_mode=gm, lower_bound=lb)
        out.append((o[0, :, 0], S[0, 0]))
    return out


def sample_pairs(B, HV, n, seed=7):
    rng = np.random.default_rng(seed)
    allp = [(b, hv) for b in range(B) for hv in range(HV)]
    if len(allp) <= n:
        return allp
    idx = rng.choice(len(allp), size=n, replace=False)
    chosen = [allp[i] for i in sorted(idx)]
    # always include the first and last pair (edges of the grid)
    for p in (allp[0], allp[-1]):
        if p not in chosen:
            chosen[0 if p == allp[0] else -1] = p
    return chosen


def workload_inputs(w, seed=None):
    return make_inputs(w, seed=seed)
