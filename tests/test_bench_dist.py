"""bench.py's multi-process path on CPU: two ranks under torch.distributed.run over gloo.

The forward pass shards independent (sequence, head) work across ranks with no data-path
collective; the only communication is the barrier and the MAX of the per-rank device times, and
the whole-job value is every rank's units over the slowest rank's time (weak scaling).  These
tests check that plumbing with two real processes, and that the reference arm prints its one line
from rank 0 only."""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _torchrun(args, env=None, timeout=180):
    cmd = [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", "--nproc-per-node=2",
           "--master-addr=127.0.0.1", f"--master-port={_free_port()}"] + args
    e = dict(os.environ, **(env or {}))
    e.pop("CUDA_VISIBLE_DEVICES", None)
    return subprocess.run(cmd, cwd=ROOT, env=e, capture_output=True, text=True, timeout=timeout)


def test_two_ranks_barrier_max_and_weak_scaling(tmp_path):
    r = _torchrun([os.path.join(ROOT, "tests", "dist_worker.py")], env={"KDA_DIST_OUT": str(tmp_path)})
    assert r.returncode == 0, r.stdout + r.stderr
    res = [json.load(open(tmp_path / f"rank{k}.json")) for k in range(2)]
    for k, d in enumerate(res):
        assert d["rank"] == k and d["ws"] == 2 and d["local"] == k
        assert d["max"] == 20.0                       # MAX over ranks reaches every rank
        assert d["ms_per_step"] == pytest.approx(50.0)  # slowest rank: 200 ms over 4 steps
        assert d["value"] == pytest.approx(2 * 1000 * 4 / 0.2)
    assert res[0]["seed"] == 1002 and res[1]["seed"] != res[0]["seed"]  # rank 0 = the workload's own inputs


def test_reference_arm_prints_from_rank0_only():
    r = _torchrun(["bench.py", "--impl", "reference", "--workload", "1", "--steps", "1", "--warmup", "0"])
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["n_gpus"] == 2 and d["unit"] == "tokens/s" and d["value"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle"


def test_gpus_flag_launches_that_many_ranks():
    """`bench.py --gpus 2`, started as a plain process, relaunches itself as two ranks under
    torch.distributed.run; --dry-plumbing keeps it on CPU (gloo), touching no device."""
    e = dict(os.environ)
    e.pop("CUDA_VISIBLE_DEVICES", None)
    for k in ("WORLD_SIZE", "RANK", "LOCAL_RANK", "MASTER_ADDR", "MASTER_PORT"):
        e.pop(k, None)
    r = subprocess.run([sys.executable, "bench.py", "--gpus", "2", "--dry-plumbing", "--steps", "3"], cwd=ROOT,
                       env=e, capture_output=True, text=True, timeout=180)
    assert r.returncode == 0, r.stdout + r.stderr
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1, r.stdout
    d = json.loads(lines[0])
    assert d["n_gpus"] == 2 and d["steps"] == 3 and d["scaling"] == "weak"
    # slowest rank: 20 ms per step; both ranks' 1000 units per step
    assert d["ms_per_step"] == pytest.approx(20.0) and d["value"] == pytest.approx(2 * 1000 / 0.02)
