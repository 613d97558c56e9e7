"""GPU <-> oracle parity helpers (shared by the GPU test files, bench and smoke).

Tolerances (the stated targets of the build, in writing):
  * k_eps and the kept index set: bit-exact, except rows in an exemption class
      M: the oracle's TV(k) or TV(k-1) lies within `window` (1e-6) of eps, so
         an fp32 logit may legitimately move the cut by one key;
      T: the oracle's gap u_(k) - u_(k+1) is within the fp32 dot-product
         rounding bound gamma_d (sum|q k_(k)| + sum|q k_(k+1)|), so fp32 logits
         may legitimately swap the two boundary keys.
    An exempt row whose set differs must still be a valid minimal
    certificate under the oracle's own fp64 masses, judged on the GPU's set
    (oracle.eval_kept_set): TV_oracle(GPU set) <= eps + window, and dropping
    the set's lowest-ranked key gives TV_oracle > eps - window; the set is
    ascending, distinct, and differs from the oracle's by at most 8 keys; and
    the GPU's TV, KL, err and output on that row match the oracle's values for
    the GPU's set with the tolerances below.  With ``strict_window`` every
    row outside class M at that window and outside class T must be exact.
    Counts of class M at 1e-6 / 1e-7 / 1e-8 / 1e-9 and of class T are
    reported.
  * out, fp32: per row ||out_gpu - out_ref||_inf <= 1e-5 ||out_ref||_inf.
  * out, bf16: compared in the output precision.  Rounding to bf16 (8
    significant bits) alone moves a value by up to 2^-8 = 3.9e-3 relative,
    more than a 3e-3 budget, so the GPU's bf16 output must equal the oracle's
    fp64 output rounded to bf16, except where that value lies within
    1e-5 * ||out_ref||_inf of a bf16 rounding midpoint (there the other
    neighbour is allowed).  This checks the pre-rounding value to 1e-5 of the
    row scale - tighter than 3e-3 - and the per-row relative error is also
    reported.
  * TV and KL: within 1e-6 absolute.
  * err: |err_gpu - err_ref| <= 1e-4 err_ref + 1e-7.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from certified_top_sparse_b200 import workloads as W

WINDOWS = (1e-6, 1e-7, 1e-8, 1e-9)


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp64 -> nearest bf16 (round to nearest even), returned as fp64."""
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float64)).to(torch.bfloat16) \
        .double().numpy()


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


def check_out(og: np.ndarray, oo: np.ndarray, dtype: torch.dtype):
    """Output check of the module docstring; og, oo are [rows, d] fp64.
    Returns the per-row relative errors and the count of bf16 outputs that
    took the other rounding neighbour."""
    scale = np.abs(oo).max(axis=1)
    rel = np.abs(og - oo).max(axis=1) / np.maximum(scale, 1e-30)
    if dtype == torch.float32:
        assert np.all(rel <= 1e-5), f"out rel err {rel.max()} > 1e-5"
        return rel, 0
    # arithmetic allowance before the final rounding: 1e-5 of the row scale
    delta = 1e-5 * scale[:, None]
    rounded = bf16_round(oo)
    border = bf16_round(oo + delta) != bf16_round(oo - delta)
    same = og == rounded
    assert np.all(same | border), \
        f"{int((~same & ~border).sum())} bf16 outputs differ from the rounded reference"
    assert np.all(np.abs(og - oo) <= 2.0 ** -8 * np.abs(oo) + 1.01 * delta), \
        "bf16 output off by more than rounding + 1e-5 of the row scale"
    return rel, int((~same).sum())


def _eval_sets(prob: W.Problem, sets):
    return oracle.eval_kept_set(W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V),
                                sets, n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads,
                                dtype=oracle_dtype(prob), batch=prob.batch, m=prob.m)


def compare(prob: W.Problem, eps: float, gpu: dict, ora: dict, rows=None, window: float = 1e-6,
            strict_window: float | None = None):
    """Compare host copies of GPU results (rows `rows` of the GPU arrays, or
    all) with an oracle run over the same rows.  Returns a report dict;
    raises AssertionError on any violation."""
    if rows is None:
        rows = np.arange(len(ora["k"]))
    kg = gpu["k"][rows].astype(np.int64)
    ko = ora["k"].astype(np.int64)
    nrow = len(rows)
    classM = {w: (np.abs(ora["tv"] - eps) <= w) | (np.abs(ora["tv_km1"] - eps) <= w)
              for w in WINDOWS}
    classT = np.nan_to_num(ora["gap_u"], nan=np.inf) <= np.nan_to_num(ora["tie_bound"], nan=-1.0)
    exempt = classM[window] | classT
    exact = np.zeros(nrow, bool)
    bad = []
    gsets = []
    for j, r in enumerate(rows):
        ig = gpu["idx"][r, : kg[j]]
        io = ora["idx"][j]
        gsets.append(ig)
        exact[j] = kg[j] == ko[j] and np.array_equal(ig, io)
        if exact[j]:
            continue
        if not exempt[j]:
            bad.append((int(r), "mismatch outside exemption", int(kg[j]), int(ko[j])))
            continue
        sym = len(np.setxor1d(ig, io))
        if not (kg[j] >= 1 and np.all(np.diff(ig) > 0) and ig[0] >= 0 and ig[-1] < prob.n
                and sym <= 8):
            bad.append((int(r), "malformed exempt row", int(kg[j]), int(ko[j]), sym))
    assert not bad, f"{len(bad)} bad rows, first: {bad[:5]}"
    if strict_window is not None:
        must = ~(classM[strict_window] | classT)
        assert np.all(exact[must]), \
            f"{int((~exact & must).sum())} rows outside class M({strict_window:g}) and T differ"
    diff = np.where(~exact)[0]
    ev = None
    if len(diff):
        # the GPU's set judged with the oracle's fp64 masses
        ev = _eval_sets(prob, [gsets[j] if not exact[j] else ora["idx"][j] for j in range(nrow)])
        tvg = ev["tv"][diff]
        assert np.all(tvg <= eps + window), f"GPU set not certified: TV_oracle {tvg.max()}"
        tvm = ev["tv_drop_lowest"][diff]
        assert np.all(tvm > eps - window), f"GPU set not minimal: TV_oracle(k-1) {tvm.min()}"
    # expected values per row: the oracle's top-k values, or on differing
    # exempt rows the oracle's values for the GPU's set
    exp_tv, exp_kl, exp_err = ora["tv"].copy(), ora["kl"].copy(), ora["err"].copy()
    exp_out = ora["out"].copy()
    if ev is not None:
        exp_tv[diff], exp_kl[diff], exp_err[diff] = ev["tv"][diff], ev["kl"][diff], ev["err"][diff]
        exp_out[diff] = ev["out"][diff]
    # TV and KL within 1e-6
    dtv = np.abs(gpu["tv"][rows] - exp_tv)
    assert np.all(dtv <= 1e-6), f"TV off by {dtv.max()}"
    if gpu.get("kl") is not None:
        dkl = np.abs(gpu["kl"][rows] - exp_kl)
        assert np.all(dkl <= 1e-6), f"KL off by {dkl.max()}"
    # outputs
    rel, n_ulp = check_out(gpu["out"][rows], exp_out, prob.q.dtype)
    # exact head-tail error
    if gpu.get("err") is not None:
        eg = gpu["err"][rows].astype(np.float64)
        derr = np.abs(eg - exp_err)
        assert np.all(derr <= 1e-4 * exp_err + 1e-7), \
            f"err off: max {derr.max()} (rel {np.max(derr / np.maximum(exp_err, 1e-30))})"
    # single-gap certificate: the same gap up to the fp32 rounding of the two
    # boundary logits (tie_bound covers both), and never below TV
    ex = np.where(exact)[0]
    if gpu.get("gap") is not None:
        gg = gpu["gap"][rows].astype(np.float64)
        assert np.all(gg >= gpu["tv"][rows].astype(np.float64) * (1 - 1e-6) - 1e-7), \
            "single-gap bound below TV"
        go = ora["gap_bound"][ex]
        tb = np.nan_to_num(ora["tie_bound"][ex], nan=0.0)
        tol = go * np.expm1(2.0 * tb / math.sqrt(prob.d)) + 1e-6 * go + 1e-9
        dg = np.abs(gg[ex] - go)
        assert np.all(dg <= tol), f"gap bound off: max {dg.max()} (tol {tol[np.argmax(dg)]})"
    return {
        "rows": nrow, "exact": int(exact.sum()), "differing_exempt": int((~exact).sum()),
        "classM": {f"{w:g}": int(classM[w].sum()) for w in WINDOWS}, "classT": int(classT.sum()),
        "max_out_rel": float(rel.max()) if len(rel) else 0.0, "bf16_ulp_diffs": n_ulp,
        "max_tv_abs": float(dtv.max()) if len(dtv) else 0.0,
    }
