"""Expert parallelism on CPU ranks: the expert partition and the exchange step
(all-reduce of the ranks' partial outputs) over gloo, with the partials taken
from the oracle's per-slot expert outputs -- the part the GPU kernels compute,
which tests/test_gpu_ep.py checks on a GPU."""
import json
import os
import socket
import subprocess
import sys

import pytest

from int4_routed_expert_softmax_b200 import ep

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("E,world", [(256, 1), (256, 2), (256, 3), (256, 8), (16, 4), (5, 4), (1, 1), (3, 4)])
def test_expert_range_partitions(E, world):
    ranges = [ep.expert_range(E, world, r) for r in range(world)]
    assert ranges[0][0] == 0 and ranges[-1][1] == E
    for (lo, hi), (lo2, _) in zip(ranges, ranges[1:]):
        assert hi == lo2                                  # contiguous, disjoint
    sizes = [hi - lo for lo, hi in ranges]
    assert max(sizes) - min(sizes) <= 1 and sum(sizes) == E
    assert [ep.owns_shared(r) for r in range(world)] == [True] + [False] * (world - 1)


def test_expert_range_rejects_bad_arguments():
    for args in [(0, 1, 0), (16, 0, 0), (16, 2, 2), (16, 2, -1)]:
        with pytest.raises(ValueError):
            ep.expert_range(*args)


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


@pytest.mark.parametrize("world", [2, 3])
def test_partials_all_reduce_to_the_layer(tmp_path, world):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE=str(world), CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "_ep_worker.py"),
                                       str(tmp_path / f"rank{r}.json")], env=env))
    try:
        codes = [p.wait(timeout=180) for p in procs]
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    assert codes == [0] * world
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(world)]
    assert sum(d["owned_pairs"] for d in res) == 6 * 4          # every (token, slot) pair owned once
    for d in res:
        assert d["same"]                                          # every rank holds the same output
        assert d["rel"] <= 1e-6 and d["max"] <= 1e-5, d           # sums reordered: a few ulps
