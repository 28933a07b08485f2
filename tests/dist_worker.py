"""Worker for the world-size-2 test of bench.py's multi-process plumbing (launched by
torch.distributed.run from test_bench_dist.py; gloo on CPU, 127.0.0.1).  Each rank reports, as
one JSON line, what bench.py's helpers returned for a rank-dependent input."""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
from kimi_delta_attention_33_b200.inputs import WORKLOADS  # noqa: E402


def main():
    ws, rank, local = bench.dist_setup(backend="gloo")
    bench.barrier(ws)
    mx = bench.max_over_ranks(10.0 * (rank + 1), ws)
    value, ms_per_step = bench.aggregate(1000, 4, 100.0 * (rank + 1), ws)
    seed = bench.rank_seed(WORKLOADS[2], rank)
    out = os.environ["KDA_DIST_OUT"]
    with open(os.path.join(out, f"rank{rank}.json"), "w") as f:
        json.dump({"rank": rank, "ws": ws, "local": local, "max": mx, "value": value, "ms_per_step": ms_per_step,
                   "seed": seed}, f)
    bench.barrier(ws)
    dist.destroy_process_group()


if __name__ == "__main__":
    main()
