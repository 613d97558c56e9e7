"""GPU <-> oracle parity helpers (shared by the GPU test files, bench and smoke).

Tolerances (the stated targets of the build, in writing):
  * k_eps and the kept index set: bit-exact, except rows in an exemption class
      M: the oracle's TV(k) or TV(k-1) lies within `window` (1e-6) of eps, so
         an fp32 logit may legitimately move the cut by one key;
      T: the oracle's gap u_(k) - u_(k+1) is within the fp32 dot-product
         rounding bound gamma_d (sum|q k_(k)| + sum|q k_(k+1)|), so fp32 logits
         may legitimately swap the two boundary keys.
    Exempt rows that differ must still be valid: GPU TV <= eps, and the GPU
    set differs from the oracle's by a few boundary keys.  Counts of class M
    at 1e-6 / 1e-7 / 1e-8 / 1e-9 and of class T are reported.
  * out: per row ||out_gpu - out_ref||_inf <= tol * ||out_ref||_inf with
    tol = 1e-5 (fp32 inputs) or 3e-3 (bf16 inputs and output).
  * TV and KL: within 1e-6 absolute.
  * err: |err_gpu - err_ref| <= 1e-4 err_ref + 1e-7.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from certified_top_sparse_b200 import workloads as W

WINDOWS = (1e-6, 1e-7, 1e-8, 1e-9)


def out_tol(prob: W.Problem) -> float:
    return 1e-5 if prob.q.dtype == torch.float32 else 3e-3


def oracle_dtype(prob: W.Problem) -> int:
    return oracle.F32 if prob.q.dtype == torch.float32 else oracle.BF16


def run_oracle(prob: W.Problem, eps: float, **kw):
    return oracle.certified_topk_attn(
        W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V), eps,
        n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads, dtype=oracle_dtype(prob),
        batch=prob.batch, m=prob.m, **kw)


def sub_problem(prob: W.Problem, b: int, kvh: int, q=None) -> W.Problem:
    """The rows of one (batch, KV head) group as a problem of its own."""
    g = prob.n_heads // prob.n_kv_heads
    qq = prob.q if q is None else q
    return W.Problem(prob.name, qq[b:b + 1, kvh * g:(kvh + 1) * g].contiguous(),
                     prob.K[b:b + 1, kvh:kvh + 1].contiguous(),
                     prob.V[b:b + 1, kvh:kvh + 1].contiguous(), prob.eps, 1, g, 1, prob.m,
                     prob.n, prob.d)


def group_rows(prob: W.Problem, b: int, kvh: int) -> np.ndarray:
    g = prob.n_heads // prob.n_kv_heads
    first = (b * prob.n_heads + kvh * g) * prob.m
    return np.arange(first, first + g * prob.m)


def to_host(res: dict) -> dict:
    h = {}
    for k, v in res.items():
        if v is None:
            h[k] = None
        elif k == "out":
            h[k] = v.float().reshape(-1, v.shape[-1]).cpu().numpy().astype(np.float64)
        elif k == "idx":
            h[k] = v.reshape(-1, v.shape[-1]).cpu().numpy()
        else:
            h[k] = v.reshape(-1).cpu().numpy()
    return h


def compare(prob: W.Problem, eps: float, gpu: dict, ora: dict, rows=None, window: float = 1e-6):
    """Compare host copies of GPU results (rows `rows` of the GPU arrays, or
    all) with an oracle run over the same rows.  Returns a report dict;
    raises AssertionError on any violation."""
    if rows is None:
        rows = np.arange(len(ora["k"]))
    kg = gpu["k"][rows].astype(np.int64)
    ko = ora["k"].astype(np.int64)
    nrow = len(rows)
    tol = out_tol(prob)
    classM = {w: (np.abs(ora["tv"] - eps) <= w) | (np.abs(ora["tv_km1"] - eps) <= w)
              for w in WINDOWS}
    classT = np.nan_to_num(ora["gap_u"], nan=np.inf) <= np.nan_to_num(ora["tie_bound"], nan=-1.0)
    exempt = classM[window] | classT
    exact = np.zeros(nrow, bool)
    bad = []
    for j, r in enumerate(rows):
        ig = gpu["idx"][r, : kg[j]]
        io = ora["idx"][j]
        exact[j] = kg[j] == ko[j] and np.array_equal(ig, io)
        if exact[j]:
            continue
        if not exempt[j]:
            bad.append((int(r), "mismatch outside exemption", int(kg[j]), int(ko[j])))
            continue
        # exempt and different: must still be a valid certified truncation
        sym = len(np.setxor1d(ig, io))
        if not (gpu["tv"][r] <= eps and sym <= 8 and np.all(np.diff(ig) > 0)):
            bad.append((int(r), "invalid exempt row", int(kg[j]), int(ko[j]), sym))
    assert not bad, f"{len(bad)} bad rows, first: {bad[:5]}"
    ex = np.where(exact)[0]
    # TV and KL within 1e-6 on rows with the same kept set
    dtv = np.abs(gpu["tv"][rows][ex] - ora["tv"][ex])
    assert np.all(dtv <= 1e-6), f"TV off by {dtv.max()}"
    if gpu.get("kl") is not None:
        dkl = np.abs(gpu["kl"][rows][ex] - ora["kl"][ex])
        assert np.all(dkl <= 1e-6), f"KL off by {dkl.max()}"
    # outputs
    og = gpu["out"][rows][ex]
    oo = ora["out"][ex]
    scale = np.abs(oo).max(axis=1)
    rel = np.abs(og - oo).max(axis=1) / np.maximum(scale, 1e-30)
    assert np.all(rel <= tol), f"out rel err {rel.max()} > {tol}"
    # exact head-tail error
    if gpu.get("err") is not None:
        eg = gpu["err"][rows][ex].astype(np.float64)
        eo = ora["err"][ex]
        derr = np.abs(eg - eo)
        assert np.all(derr <= 1e-4 * eo + 1e-7), f"err off: max {derr.max()} (rel {np.max(derr / np.maximum(eo, 1e-30))})"
    return {
        "rows": nrow, "exact": int(exact.sum()), "differing_exempt": int((~exact).sum()),
        "classM": {f"{w:g}": int(classM[w].sum()) for w in WINDOWS}, "classT": int(classT.sum()),
        "max_out_rel": float(rel.max()) if len(rel) else 0.0,
        "max_tv_abs": float(dtv.max()) if len(dtv) else 0.0,
    }
