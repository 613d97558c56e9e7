"""Sequence-sharded certified Top-k (certified_top_sparse_b200/seqshard.py) on
CPU: two gloo ranks hold the two halves of every row's keys (an odd split),
run the exchange, and must reproduce the fp64 oracle's k, index set, TV,
output, error and KL; one process holding all keys must give the same k and
index set (the decision is an integer sum, independent of the rank count).
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from certified_top_sparse_b200 import seqshard  # noqa: E402
import oracle  # noqa: E402

N, D, ROWS, EPS = 6001, 64, 4, 0.01


def problem():
    rng = np.random.default_rng(4242)
    q = rng.standard_normal((1, ROWS, 1, D)).astype(np.float32)
    q *= np.array([0.5, 1.0, 2.0, 3.0], np.float32)[None, :, None, None]
    K = rng.standard_normal((1, ROWS, N, D)).astype(np.float32)
    V = rng.standard_normal((1, ROWS, N, D)).astype(np.float32)
    return q, K, V


def shard_inputs(q, K, V, lo, hi):
    """This rank's logits (fp64, divided by sqrt(64) = 8 exactly) and value rows."""
    qq = torch.from_numpy(q[0, :, 0, :]).double()
    Kk = torch.from_numpy(K[0, :, lo:hi, :]).double()
    s = torch.einsum("rd,rkd->rk", qq, Kk) / 8.0
    return s, torch.from_numpy(V[0, :, lo:hi, :]).double()


def tied_problem():
    """Logits on a coarse grid (many exact ties, also across the shard
    boundary): the cut falls inside a run of equal logits, so the lower index
    must win across ranks."""
    rng = np.random.default_rng(777)
    q = np.zeros((1, ROWS, 1, D), np.float32)
    q[..., 0] = 1.0
    K = np.zeros((1, ROWS, N, D), np.float32)
    K[..., 0] = (rng.integers(0, 6, size=(1, ROWS, N)) * 2.0).astype(np.float32)  # logits 0, .25, ... 1.25
    V = rng.standard_normal((1, ROWS, N, D)).astype(np.float32)
    return q, K, V


WORKER = r"""
import json, os, sys
sys.path.insert(0, %(root)r)
sys.path.insert(0, os.path.join(%(root)r, "tests"))
import torch
import torch.distributed as dist
from test_seqshard_cpu import problem, tied_problem, shard_inputs, N, EPS
from certified_top_sparse_b200 import seqshard
import datetime
dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
rank, world = dist.get_rank(), dist.get_world_size()
q, K, V = tied_problem() if os.environ.get("CTA_TIED") else problem()
bounds = [0, 2999, N]          # an odd split
s, v = shard_inputs(q, K, V, bounds[rank], bounds[rank + 1])
r = seqshard.certify_sharded(s, v, bounds[rank], EPS)
print(json.dumps({"rank": rank, "k": r["k"].tolist(), "idx": [x.tolist() for x in r["idx"]],
                  "tv": r["tv"].tolist(), "kl": r["kl"].tolist(), "err": r["err"].tolist(),
                  "out": r["out"].tolist()}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    sock = socket.socket()
    sock.bind(("127.0.0.1", 0))
    port = sock.getsockname()[1]
    sock.close()
    return port


def _check(res, ora):
    assert list(res["k"]) == [int(x) for x in ora["k"]]
    for r in range(ROWS):
        assert np.array_equal(np.asarray(res["idx"][r]), ora["idx"][r])
    assert np.allclose(res["tv"], ora["tv"], rtol=0, atol=1e-12)
    assert np.allclose(res["err"], ora["err"], rtol=1e-9, atol=1e-13)
    assert np.allclose(res["kl"], ora["kl"], rtol=1e-9, atol=1e-12)
    out = np.asarray(res["out"])
    scale = np.abs(ora["out"]).max(axis=1, keepdims=True)
    assert np.all(np.abs(out - ora["out"]) <= 1e-10 * scale)


def _oracle(make=problem):
    q, K, V = make()
    return oracle.certified_topk_attn(q, K, V, EPS, n_heads=ROWS, n_kv_heads=ROWS, dtype=oracle.F32)


def test_one_process_matches_oracle():
    q, K, V = problem()
    s, v = shard_inputs(q, K, V, 0, N)
    r = seqshard.certify_sharded(s, v, 0, EPS)
    _check({"k": r["k"].tolist(), "idx": r["idx"], "tv": r["tv"].numpy(), "kl": r["kl"].numpy(),
            "err": r["err"].numpy(), "out": r["out"].numpy()}, _oracle())


@pytest.mark.parametrize("tied", [False, True])
def test_two_gloo_ranks_match_oracle(tmp_path, tied):
    script = tmp_path / "worker.py"
    script.write_text(WORKER % {"root": ROOT})
    port = _free_port()
    procs = []
    for rank in range(2):
        env = dict(os.environ, RANK=str(rank), WORLD_SIZE="2", LOCAL_RANK=str(rank),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
        if tied:
            env["CTA_TIED"] = "1"
        procs.append(subprocess.Popen([sys.executable, str(script)], env=env,
                                      stdout=subprocess.PIPE, stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        o, e = p.communicate(timeout=180)
        assert p.returncode == 0, e
        outs.append(json.loads(o.strip().splitlines()[-1]))
    ora = _oracle(tied_problem if tied else problem)
    for res in outs:  # every rank holds the whole result
        _check(res, ora)
    assert outs[0]["idx"] == outs[1]["idx"] and outs[0]["out"] == outs[1]["out"]


def test_bracket_contains_the_cut_on_a_two_level_row():
    # 10 keys at logit 0 and 1000 keys 12 halvings lower: the bracket must
    # keep the top level for certain only if the cut lies below it
    s = torch.cat([torch.zeros(10), torch.full((1000,), -12 * np.log(2.0))]).double()[None, :]
    V = torch.randn(1, 1010, 4, dtype=torch.float64)
    r = seqshard.certify_sharded(s, V, 0, 0.05)
    Z = 10 + 1000 * 2.0 ** -12
    # minimal k: the tail of 1000 - j low keys has mass (1000 - j) 2^-12 <= 0.05 Z
    need = int(np.ceil(1000 - 0.05 * Z * 2 ** 12))
    assert int(r["k"][0]) == 10 + max(0, need)
    assert r["tv"][0] <= 0.05


@pytest.mark.parametrize("seed,sigma,eps", [(1, 1.0, 0.01), (2, 3.0, 0.001), (3, 0.3, 0.1),
                                            (4, 6.0, 1e-4), (5, 1.5, 0.5)])
def test_bracket_brackets_the_oracles_cut(seed, sigma, eps):
    # From the level counts alone, every key below bin g_hi must be one the
    # oracle keeps and every key from bin g_lo on one it drops.
    rng = np.random.default_rng(seed)
    n = 20000
    s = rng.standard_normal(n) * sigma
    s[rng.integers(0, n, 5)] += 4 * sigma  # a few large logits
    s = s.astype(np.float32)               # the oracle's inputs: q = 1, d = 1, K = s
    ora = oracle.certified_topk_attn(np.ones((1, 1, 1, 1), np.float32), s.reshape(1, 1, n, 1),
                                     np.zeros((1, 1, n, 1), np.float32), eps,
                                     n_heads=1, n_kv_heads=1, dtype=oracle.F32)
    kept = np.zeros(n, bool)
    kept[ora["idx"][0]] = True
    assert kept.sum() == ora["k"][0]
    s64 = s.astype(np.float64)
    a = (s64.max() - s64) / np.log(2.0)
    g = np.floor(a * seqshard.LEVELS).astype(np.int64)
    G = seqshard.LEVELS * seqshard.FRAME_OCTAVES
    counts = np.bincount(g[g < G], minlength=G)[None, :]
    deep = np.array([(g >= G).sum()])
    g_lo, g_hi = seqshard.bracket(torch.from_numpy(counts), torch.from_numpy(deep), eps)
    g_lo, g_hi = g_lo[0], g_hi[0]
    assert g_hi < g_lo
    assert kept[g < g_hi].all()
    assert not kept[g >= g_lo].any()
