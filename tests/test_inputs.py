"""The seeded input generator: deterministic, right shapes, dtypes and distributions (CPU)."""
import torch

from kimi_delta_attention_33_b200.inputs import GATE_SAFE, GATE_STANDARD, WORKLOADS, make_inputs


def test_deterministic_and_shaped():
    w = WORKLOADS[1]
    a, b = make_inputs(w), make_inputs(w)
    for key in ("q", "k", "v", "g", "beta", "A_log", "dt_bias"):
        assert torch.equal(a[key], b[key])
    assert a["S0"] is None
    assert a["q"].shape == (1, 64, 2, 16) and a["v"].shape == (1, 64, 2, 16)
    assert a["g"].shape == (1, 64, 2, 16) and a["beta"].shape == (1, 64, 2)
    assert a["q"].dtype == torch.float32
    assert torch.all(a["A_log"] == 0) and torch.all(a["dt_bias"] == -4.0)


def test_distributions_small_versions():
    for wid in (2, 3, 4, 5):
        w = WORKLOADS[wid].scaled(B=1, T=32)
        x = make_inputs(w)
        assert x["q"].dtype == torch.bfloat16
        n = x["q"].float().norm(dim=-1)
        assert torch.allclose(n, torch.ones_like(n), atol=1e-2)
        assert torch.all(x["beta"] > 0) and torch.all(x["beta"] < 1)
        assert x["v"].shape[2] == w.HV and x["q"].shape[2] == w.H
        if w.S0_std is not None:
            assert x["S0"].shape == (1, w.HV, w.K, w.V) and x["S0"].dtype == torch.float32
    assert WORKLOADS[4].gate_mode == GATE_STANDARD and WORKLOADS[2].gate_mode == GATE_SAFE
    lo, hi = WORKLOADS[4].A_log_range
    a = make_inputs(WORKLOADS[4].scaled(T=8))["A_log"]
    assert torch.all(a >= lo) and torch.all(a <= hi)


def test_seed_changes_draws():
    w = WORKLOADS[2].scaled(T=16)
    assert not torch.equal(make_inputs(w, seed=1)["v"], make_inputs(w, seed=2)["v"])
