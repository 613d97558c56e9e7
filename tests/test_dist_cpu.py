"""Multi-process plumbing of bench.py on CPU (gloo, world size 2).

The certified path shards by independent rows with no exchange step, so the
only cross-rank operations are the barriers around the timed region and the
maximum of the per-rank times.  These run here as two gloo processes.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import json, os, sys, time
sys.path.insert(0, %(root)r)
import torch
import bench
rank, world, local = bench.dist_env()
dist = bench.init_dist(world, "gloo")
dev = torch.device("cpu")
bench.barrier(dist, dev)
secs = 0.05 * (rank + 1)          # rank 1 is the slow one
time.sleep(secs)
bench.barrier(dist, dev)
slowest = bench.max_over_ranks(secs, dist, dev)
value = bench.aggregate(32, 10, world, slowest)
print(json.dumps({"rank": rank, "world": world, "slowest": slowest, "value": value}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def test_two_rank_max_and_aggregate(tmp_path):
    script = tmp_path / "worker.py"
    script.write_text(WORKER % {"root": ROOT})
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=120)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    for o in outs:
        assert o["world"] == 2
        assert o["slowest"] == pytest.approx(0.10)
        # 2 ranks x 10 steps x 32 query heads over the slowest rank's time
        assert o["value"] == pytest.approx(640 / 0.10)


def test_single_process_defaults(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    assert bench.dist_env() == (0, 1, 0)
    assert bench.init_dist(1, "gloo") is None
    assert bench.max_over_ranks(1.5, None, None) == 1.5
    assert bench.aggregate(32, 100, 1, 2.0) == 1600.0


def test_bench_rejects_short_warmup():
    sys.path.insert(0, ROOT)
    import bench
    with pytest.raises(SystemExit):
        bench.main(["--warmup", "2"])
