"""One rank of the two-rank gloo test of bench.py's multi-rank plumbing (CPU only):
rendezvous, barrier, whole-job aggregation (units summed, time maxed over ranks),
per-rank input streams, and the reference arm's rank-0-only rule.
Usage: RANK=r WORLD_SIZE=2 MASTER_ADDR=127.0.0.1 MASTER_PORT=p python _multirank_worker.py out.json"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import bench  # noqa: E402
import moe_inputs as mi  # noqa: E402


def main():
    out = sys.argv[1]
    ws_n, rank, _ = bench.dist_setup("gloo")
    try:
        bench.barrier(ws_n)
        units, max_ms = bench.aggregate((rank + 1) * 1.0e9, 10.0 * (rank + 1), ws_n)
        w = mi.WORKLOADS["tiny"]
        x = mi.make_x(w.T, w.H, mi.sub_seed(bench.rank_seed(w, rank), 0, 1))
        again = mi.make_x(w.T, w.H, mi.sub_seed(bench.rank_seed(w, rank), 0, 1))
        xs = [torch.empty_like(x) for _ in range(ws_n)]
        dist.all_gather(xs, x)
        ref = bench.run_reference(None, ws_n, rank) if rank != 0 else "not run"
        bench.barrier(ws_n)
        json.dump({"rank": rank, "world": ws_n, "units": units, "max_ms": max_ms,
                   "x_repeatable": bool(torch.equal(x, again)),
                   "x_distinct": not torch.equal(xs[0], xs[1]),
                   "ref": ref}, open(out, "w"))
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
