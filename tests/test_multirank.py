"""bench.py's multi-rank path on two gloo ranks (CPU): the same steps that run one
rank per GPU over NCCL, without a GPU."""
import json
import os
import socket
import subprocess
import sys

HERE = os.path.dirname(os.path.abspath(__file__))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_ranks_aggregate_and_replicas(tmp_path):
    port = _free_port()
    procs = []
    for r in range(2):
        env = dict(os.environ, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(r),
                   LOCAL_RANK=str(r), WORLD_SIZE="2", CUDA_VISIBLE_DEVICES="")
        procs.append(subprocess.Popen([sys.executable, os.path.join(HERE, "_multirank_worker.py"),
                                       str(tmp_path / f"rank{r}.json")], env=env))
    try:
        codes = [p.wait(timeout=180) for p in procs]
    finally:
        for p in procs:
            if p.poll() is None:
                p.kill()
    assert codes == [0, 0]
    res = [json.load(open(tmp_path / f"rank{r}.json")) for r in range(2)]
    for r, d in enumerate(res):
        assert d["rank"] == r and d["world"] == 2
        assert d["units"] == 3.0e9          # units of both ranks
        assert d["max_ms"] == 20.0          # the slower rank's time
        assert d["x_repeatable"] and d["x_distinct"]
    assert res[1]["ref"] is None            # the reference arm works on rank 0 only
