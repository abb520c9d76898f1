"""One rank of the expert-parallel gloo test (CPU only): this rank's partial
output of the layer -- computed from the oracle's per-slot expert outputs for
the experts it owns (the GPU kernels' part, which the GPU tests check) -- and
the all-reduce that combines the ranks' partials.
Usage: RANK=r WORLD_SIZE=n MASTER_ADDR=127.0.0.1 MASTER_PORT=p python _ep_worker.py out.json"""
import json
import os
import sys
from datetime import timedelta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402
import torch.distributed as dist  # noqa: E402

import moe_inputs as mi  # noqa: E402
import oracle as orc  # noqa: E402
from int4_routed_expert_softmax_b200 import ep  # noqa: E402


def main():
    out_path = sys.argv[1]
    dist.init_process_group("gloo", timeout=timedelta(seconds=60))
    rank, world = dist.get_rank(), dist.get_world_size()
    try:
        w = mi.Workload("ep", H=256, I=128, E=16, k=4, T=6, seed=41)
        x, Wr, blobs = mi.make_layer(w, 0, "cpu")
        ref, tr = orc.moe_layer(x.numpy(), Wr.numpy(), blobs.numpy(), w.H, w.I, w.E, w.k, trace=True)
        lo, hi = ep.expert_range(w.E, world, rank)
        part = np.zeros((w.T, w.H), np.float32)
        for t in range(w.T):
            acc = tr["y"][t, w.k].copy() if ep.owns_shared(rank) else np.zeros(w.H, np.float32)
            for s in range(w.k):
                if lo <= int(tr["idx"][t, s]) < hi:
                    acc = (acc + np.float32(tr["w"][t, s]) * tr["y"][t, s]).astype(np.float32)
            part[t] = acc
        out = torch.from_numpy(part)
        ep.reduce_partials(out)
        got = out.numpy().astype(np.float64)
        rel = float(np.linalg.norm(got - ref) / np.linalg.norm(ref))
        mx = float(np.abs(got - ref).max() / np.sqrt(np.mean(ref.astype(np.float64) ** 2)))
        gathered = [torch.empty_like(out) for _ in range(world)]
        dist.all_gather(gathered, out)
        same = all(torch.equal(g, gathered[0]) for g in gathered)
        owned = [int(e) for e in tr["idx"].reshape(-1) if lo <= int(e) < hi]
        json.dump({"rank": rank, "world": world, "lo": lo, "hi": hi, "rel": rel, "max": mx, "same": same,
                   "owned_pairs": len(owned)}, open(out_path, "w"))
    finally:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
