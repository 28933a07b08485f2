import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a); parity tests against the oracle")


def pytest_collection_modifyitems(config, items):
    try:
        import torch
        has_cuda = torch.cuda.is_available()
    except Exception:  # pragma: no cover
        has_cuda = False
    if has_cuda:
        return
    skip = pytest.mark.skip(reason="no CUDA device")
    for item in items:
        if "gpu" in item.keywords:
            item.add_marker(skip)


def pytest_terminal_summary(terminalreporter, exitstatus, config):
    """Print the relative errors the parity tests measured (max|x - x_ref| / max|x_ref|, o and the
    final state in the order each test checks them): the workload tests one per line, then the largest
    errors of all other tests, then the largest overall.  The bars are 1e-4 (float32 inputs) and 5e-3
    (bfloat16 inputs)."""
    mod = sys.modules.get("parity_util")
    rows = getattr(mod, "ERRORS", None) if mod is not None else None
    if not rows:
        return
    per = {}
    for test, err in rows:
        per.setdefault(test, []).append(err)
    tr = terminalreporter
    tr.write_sep("-", "parity: relative errors against the oracle (bars: 1e-4 fp32, 5e-3 bf16)")
    work = [t for t in per if "workload" in t]
    for t in work:
        tr.write_line(f"{t.split('::')[-1]}: " + ", ".join(f"{e:.3e}" for e in per[t]))
    rest = sorted(((max(v), t) for t, v in per.items() if t not in work), reverse=True)[:8]
    for e, t in rest:
        tr.write_line(f"{t.split('::')[-1]}: max {e:.3e}")
    worst = max(rows, key=lambda r: r[1])
    tr.write_line(f"largest relative error of {len(rows)} checks: {worst[1]:.3e} ({worst[0].split('::')[-1]})")
