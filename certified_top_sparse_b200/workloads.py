"""Seeded synthetic inputs for the five certified Top-k workloads.

This module only draws random inputs; it holds none of the method's
arithmetic.  Both the CUDA path and the fp64 oracle read the bytes it makes,
so the two sides always see identical inputs (bf16 values are rounded once,
here, with round-to-nearest-even).

Workloads (sizes as defaults; tests shrink them):

* ``tiny``   - Gaussian-score rows: B=1, 8 heads (MHA), d=64, n=1024, one query
  per head, fp32; K, V rows i.i.d. N(0, I); q = sigma sqrt(d) u/||u||, sigma
  cycling 1, 2, 3 over heads, so the logits are N(0, sigma^2); eps = 0.01.
* ``bert``   - BERT-base-shaped all-query self-attention: B=8, 12 heads, n=m=512,
  d=64, bf16 Q, K, V ~ N(0, 1).  Heads 0-5 as drawn ("diffuse").  Heads 6-11
  ("sharp"): each query picks 1-4 planted keys and its q is shifted by the
  minimum-norm vector that raises exactly those keys' logits by +8.
* ``sweep``  - one head, m = 256 queries, fp32, d=64, K, V rows N(0, I),
  ||q|| = sigma sqrt(d), for n in {4096, 16384, 65536, 262144} x sigma in
  {0.5, 1, 2, 3}; each cell is certified at eps in {0.1, 0.01, 0.001}.
* ``decode32k`` - GQA decode: B=4, 32 query heads, 8 KV heads, d=128,
  n=32768, bf16, K, V ~ N(0, I), q ~ N(0, I), eps = 0.01, with a sink key
  (+6 logit), a recent window of 256 keys (+2) and 16 needle keys (+5) per
  (batch, KV head).
* ``decode128k`` - the same structure at B=1, n=131072, with a fixed cache and
  64 decode steps of fresh queries; eps in {0.1, 0.01}.

The attention structure of the decode workloads is written through two
reserved channels: q[0] = q[1] = sqrt(d) for every query, and channel 0/1 of
each key carries the logit offset (k[0] = 6 for the sink, 2 for the window,
k[1] = 5 for needles, 0 elsewhere), so every query head sees the stated
offsets on top of an N(0, ~1) background.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

SEED_BASE = 1000
WORKLOADS = ("tiny", "bert", "sweep", "decode32k", "decode128k")


@dataclass
class Problem:
    """One call's worth of inputs, as CPU tensors (bf16 or fp32)."""

    name: str
    q: torch.Tensor          # [batch, n_heads, m, d]
    K: torch.Tensor          # [batch, n_kv_heads, n, d]
    V: torch.Tensor          # [batch, n_kv_heads, n, d]
    eps: float
    batch: int
    n_heads: int
    n_kv_heads: int
    m: int
    n: int
    d: int
    meta: dict = field(default_factory=dict)

    @property
    def dtype(self) -> torch.dtype:
        return self.q.dtype

    @property
    def rows(self) -> int:
        return self.batch * self.n_heads * self.m


def _round(x: np.ndarray, dtype: torch.dtype) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(dtype) if dtype != torch.float32 else t.clone()


def raw_words(t: torch.Tensor) -> np.ndarray:
    """The bytes of a CPU tensor as numpy: float32 as is, bf16 as uint16 words."""
    t = t.contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    assert t.dtype == torch.float32
    return t.numpy()


def _sphere_queries(rng, rows: int, d: int, sigma) -> np.ndarray:
    u = rng.standard_normal((rows, d))
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    return (np.asarray(sigma, dtype=np.float64).reshape(-1, 1) * math.sqrt(d)) * u


def tiny(n: int = 1024, d: int = 64, n_heads: int = 8, eps: float = 0.01,
         sigmas=(1.0, 2.0, 3.0), seed: int = SEED_BASE + 0) -> Problem:
    rng = np.random.default_rng(seed)
    sig = np.array([sigmas[h % len(sigmas)] for h in range(n_heads)])
    q = _sphere_queries(rng, n_heads, d, sig).reshape(1, n_heads, 1, d)
    K = rng.standard_normal((1, n_heads, n, d))
    V = rng.standard_normal((1, n_heads, n, d))
    return Problem("tiny", _round(q, torch.float32), _round(K, torch.float32),
                   _round(V, torch.float32), eps, 1, n_heads, n_heads, 1, n, d,
                   {"sigma_by_head": sig.tolist()})


def bert(batch: int = 8, n_heads: int = 12, n: int = 512, d: int = 64, eps: float = 0.01,
         sharp_from: int | None = None, plant_logit: float = 8.0,
         seed: int = SEED_BASE + 1) -> Problem:
    """All-query self-attention (m = n).  Heads >= sharp_from get planted keys."""
    rng = np.random.default_rng(seed)
    if sharp_from is None:
        sharp_from = n_heads // 2
    Q = rng.standard_normal((batch, n_heads, n, d))
    Kf = rng.standard_normal((batch, n_heads, n, d))
    Vf = rng.standard_normal((batch, n_heads, n, d))
    K = _round(Kf, torch.bfloat16)
    Kd = K.double().numpy()
    planted = {}
    for b in range(batch):
        for h in range(sharp_from, n_heads):
            for j in range(n):
                mq = int(rng.integers(1, 5))
                S = rng.choice(n, size=mq, replace=False)
                KS = Kd[b, h, S, :]                       # [mq, d]
                target = np.full(mq, plant_logit * math.sqrt(d))
                shift = KS.T @ np.linalg.solve(KS @ KS.T, target)
                Q[b, h, j, :] += shift
                planted[(b, h, j)] = np.sort(S)
    return Problem("bert", _round(Q, torch.bfloat16), K, _round(Vf, torch.bfloat16), eps,
                   batch, n_heads, n_heads, n, n, d,
                   {"sharp_from": sharp_from, "planted": planted})


SWEEP_N = (4096, 16384, 65536, 262144)
SWEEP_SIGMA = (0.5, 1.0, 2.0, 3.0)
SWEEP_EPS = (0.1, 0.01, 0.001)


def sweep_cell(n: int, sigma: float, m: int = 256, d: int = 64, eps: float = 0.01,
               seed: int | None = None) -> Problem:
    """One (n, sigma) cell: one head, m queries sharing K; eps is per call."""
    if seed is None:
        seed = SEED_BASE + 2 + 1000 * (SWEEP_N.index(n) if n in SWEEP_N else n) \
            + 10 * (SWEEP_SIGMA.index(sigma) if sigma in SWEEP_SIGMA else 0)
    rng = np.random.default_rng(seed)
    q = _sphere_queries(rng, m, d, np.full(m, sigma)).reshape(1, 1, m, d)
    K = rng.standard_normal((1, 1, n, d))
    V = rng.standard_normal((1, 1, n, d))
    return Problem("sweep", _round(q, torch.float32), _round(K, torch.float32),
                   _round(V, torch.float32), eps, 1, 1, 1, m, n, d, {"sigma": sigma})


def _decode_cache(rng, batch, n_kv_heads, n, d, n_needles=16, window=256,
                  sink=6.0, recent=2.0, needle=5.0):
    K = rng.standard_normal((batch, n_kv_heads, n, d), dtype=np.float32)
    V = rng.standard_normal((batch, n_kv_heads, n, d), dtype=np.float32)
    K[:, :, :, 0:2] = 0.0
    K[:, :, 0, 0] = sink
    w0 = max(1, n - window)
    K[:, :, w0:, 0] = recent
    needles = np.zeros((batch, n_kv_heads, n_needles), np.int64)
    hi = max(2, n - window - 1)
    for b in range(batch):
        for g in range(n_kv_heads):
            cnt = min(n_needles, hi - 1)
            sel = np.sort(rng.choice(np.arange(1, hi), size=cnt, replace=False))
            needles[b, g, :cnt] = sel
            K[b, g, sel, 1] = needle
    return K, V, needles


def decode_queries(rng, batch, n_heads, d) -> np.ndarray:
    q = rng.standard_normal((batch, n_heads, 1, d), dtype=np.float32)
    q[..., 0:2] = math.sqrt(d)
    return q


def decode32k(batch: int = 4, n_heads: int = 32, n_kv_heads: int = 8, n: int = 32768,
              d: int = 128, eps: float = 0.01, seed: int = SEED_BASE + 3) -> Problem:
    rng = np.random.default_rng(seed)
    K, V, needles = _decode_cache(rng, batch, n_kv_heads, n, d)
    q = decode_queries(rng, batch, n_heads, d)
    return Problem("decode32k", _round(q, torch.bfloat16), _round(K, torch.bfloat16),
                   _round(V, torch.bfloat16), eps, batch, n_heads, n_kv_heads, 1, n, d,
                   {"needles": needles})


DECODE128K_STEPS = 64


def decode128k(batch: int = 1, n_heads: int = 32, n_kv_heads: int = 8, n: int = 131072,
               d: int = 128, eps: float = 0.01, steps: int = DECODE128K_STEPS,
               seed: int = SEED_BASE + 4) -> Problem:
    """Fixed cache plus ``steps`` fresh query sets; ``q`` is step 0, the rest
    are in ``meta['q_steps']`` ([steps, batch, n_heads, 1, d])."""
    rng = np.random.default_rng(seed)
    K, V, needles = _decode_cache(rng, batch, n_kv_heads, n, d)
    qs = []
    for t in range(steps):
        qs.append(decode_queries(np.random.default_rng(SEED_BASE + 5 * 1000 + t), batch,
                                 n_heads, d))
    q_steps = _round(np.stack(qs), torch.bfloat16)
    return Problem("decode128k", q_steps[0].clone(), _round(K, torch.bfloat16),
                   _round(V, torch.bfloat16), eps, batch, n_heads, n_kv_heads, 1, n, d,
                   {"needles": needles, "q_steps": q_steps})


def make(name: str, **kw) -> Problem:
    """Build a workload by name with optional size overrides."""
    if name == "tiny":
        return tiny(**kw)
    if name == "bert":
        return bert(**kw)
    if name == "sweep":
        return sweep_cell(**kw)
    if name == "decode32k":
        return decode32k(**kw)
    if name == "decode128k":
        return decode128k(**kw)
    raise KeyError(name)
