"""Sequence-sharded certified Top-k: the exchange between ranks that hold
disjoint key ranges of the same rows.

When one row's keys do not fit one GPU (or one GPU's bandwidth), rank r holds
keys [n_r, n_{r+1}) of every row and computes, on its own keys, what the
single-GPU path computes per key range: logits, a level histogram, exact
fixed-point masses on either side of a bracket, the window keys as candidates
and value sums.  The certificate needs whole-row quantities, so the ranks
exchange, in this order (every rank takes the same collectives in the same
order):

  1. all-reduce (max) of the row maxima                  -> the common frame;
  2. all-reduce (sum) of integer level counts            -> the bracket of the
     cut, computed identically on every rank from the summed counts;
  3. all-reduce (sum) of the exact masses of the keys above, inside and below
     the bracket (128-bit integers as 31-bit limbs)      -> Z, exactly;
  4. all-gather of the window keys (logit, global index, exact mass)
                                                          -> the exact cut, found
     identically on every rank by walking the window in ranking order;
  5. all-reduce (sum) of the value sums of the kept and the dropped keys and
     of their weights (fp64)                              -> out, err, KL;
  6. all-gather of the kept indices (ranks hold ascending key ranges, so the
     concatenation in rank order is ascending).

The method is the certified Top-k truncation of "A Mathematical Theory of
Top-k Sparse Attention via Total Variation Distance" (arXiv 2512.07647,
abstract): the minimal k_eps with discarded tail mass TV <= eps, the output
mu_head and the error tau ||mu_tail - mu_head||.  Everything that decides k
is an integer sum (order-free, so the result does not depend on the number
of ranks); the output sums are fp64.

This module is the exchange protocol, written with torch.distributed
collectives (NCCL between GPUs, gloo on CPU); each rank's per-key work is
passed in as tensors (in a GPU deployment the library's logits and value
kernels produce them on the rank's key range).  It is tested with two gloo
ranks on CPU and has not been measured on hardware.
"""
from __future__ import annotations

import math

import torch

LEVELS = 64          # levels per halving of the weight (the bracket's resolution)
FRAME_OCTAVES = 48   # levels counted individually below the row maximum; deeper keys share one bin
MASS_BITS = 62       # exact masses: w in units of 2^-62
LIMB = 31            # limb width of the exact sums (sums of < 2^32 keys fit int64)


def _all_reduce(t: torch.Tensor, op, group):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=op, group=group)
    return t


def _all_gather_padded(t: torch.Tensor, group) -> list[torch.Tensor]:
    """All-gather of a [count, ...] tensor whose count differs per rank."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()):
        return [t]
    world = dist.get_world_size(group)
    cnt = torch.tensor([t.shape[0]], dtype=torch.int64, device=t.device)
    cnts = [torch.zeros_like(cnt) for _ in range(world)]
    dist.all_gather(cnts, cnt, group=group)
    mx = int(max(c.item() for c in cnts))
    pad = torch.zeros((mx, *t.shape[1:]), dtype=t.dtype, device=t.device)
    pad[: t.shape[0]] = t
    outs = [torch.zeros_like(pad) for _ in range(world)]
    dist.all_gather(outs, pad, group=group)
    return [o[: int(c.item())] for o, c in zip(outs, cnts)]


def _limbs(m: torch.Tensor) -> torch.Tensor:
    """[rows, keys] int64 masses (< 2^62) -> [rows, 2] per-row sums of the low
    and high 31-bit limbs (exact for fewer than 2^32 keys)."""
    lo = (m & ((1 << LIMB) - 1)).sum(dim=1)
    hi = (m >> LIMB).sum(dim=1)
    return torch.stack([lo, hi], dim=1)


def _from_limbs(l) -> int:
    return int(l[0]) + (int(l[1]) << LIMB)


def _certified(Z: int, C: int, eps: float) -> bool:
    """(Z - C) / Z <= eps, in fp64 on the exact integers."""
    return float(Z - C) / float(Z) <= eps


def bracket(counts: torch.Tensor, deep: torch.Tensor, eps: float) -> tuple[list, list]:
    """Per row, the bins [g_hi, g_lo) that hold the cut, from summed level
    counts.  Bin g holds keys with LEVELS * a in [g, g + 1), a = log2(w_max / w),
    so a key's weight lies in [2^-(g+1)/LEVELS, 2^-g/LEVELS]; `deep` counts the
    keys below the frame (w <= 2^-FRAME_OCTAVES).  Keys in bins below g_hi are
    kept for certain, keys in bins from g_lo on are dropped for certain."""
    rows, G = counts.shape
    g = torch.arange(G, dtype=torch.float64)
    hi_w = torch.exp2(-g / LEVELS)
    lo_w = torch.exp2(-(g + 1) / LEVELS)
    slack = 1e-12  # covers the fp64 rounding of the bounds' sums
    g_lo_out, g_hi_out = [], []
    for r in range(rows):
        c = counts[r].to(torch.float64)
        up = c * hi_w * (1 + slack)
        dn = c * lo_w * (1 - slack)
        deep_up = float(deep[r]) * 2.0 ** -FRAME_OCTAVES * (1 + slack)
        # mass of the keys in bins >= g (suffix sums), upper and lower bounds
        Dup = torch.flip(torch.cumsum(torch.flip(up, [0]), 0), [0]) + deep_up
        Ddn = torch.flip(torch.cumsum(torch.flip(dn, [0]), 0), [0])
        ZU, ZL = float(Dup[0]), float(Ddn[0])
        tail = torch.nonzero(Dup <= eps * ZL).flatten()
        g_lo = int(tail[0]) if len(tail) else (G if deep_up <= eps * ZL else G + 1)
        head = torch.nonzero(Ddn > eps * ZU).flatten()
        g_hi = int(head[-1]) if len(head) else 0
        if g_lo <= g_hi:  # inconsistent bounds cannot happen; keep every key in the window
            g_lo, g_hi = G + 1, 0
        g_lo_out.append(g_lo)
        g_hi_out.append(g_hi)
    return g_lo_out, g_hi_out


def certify_sharded(s: torch.Tensor, V: torch.Tensor, key0: int, eps: float, group=None) -> dict:
    """One rank's part of sequence-sharded certified Top-k.

    s: [rows, n_local] fp64 logits (q.k / sqrt(d)) of this rank's keys, whose
    global indices are key0 ... key0 + n_local - 1; V: [rows, n_local, d] the
    value rows each row reads (fp64 or fp32).  Returns, identical on every
    rank: k [rows], idx (list of ascending int64 tensors), tv, kl, err [rows]
    and out [rows, d] (fp64).
    """
    import torch.distributed as dist
    rows, nl = s.shape
    dev = s.device  # every exchanged tensor lives here (a GPU for NCCL, the CPU for gloo)
    s = s.to(torch.float64)
    V = V.to(device=dev, dtype=torch.float64)
    # 1. the row maxima
    M = s.max(dim=1).values if nl else torch.full((rows,), -math.inf, dtype=torch.float64, device=dev)
    _all_reduce(M, dist.ReduceOp.MAX, group)
    a = (M[:, None] - s) * (1.0 / math.log(2.0))           # log2(w_max / w) >= 0
    w = torch.exp2(-a)
    # 2. level counts in the common frame
    G = LEVELS * FRAME_OCTAVES
    gi = torch.floor(a * LEVELS).to(torch.int64)
    counts = torch.zeros((rows, G), dtype=torch.int64, device=dev)
    inframe = gi < G
    counts.scatter_add_(1, torch.where(inframe, gi, 0), inframe.to(torch.int64))
    deep = (~inframe).sum(dim=1)
    _all_reduce(counts, dist.ReduceOp.SUM, group)
    _all_reduce(deep, dist.ReduceOp.SUM, group)
    g_lo, g_hi = bracket(counts.cpu(), deep.cpu(), eps)
    glo = torch.tensor(g_lo, dtype=torch.int64, device=dev)[:, None]
    ghi = torch.tensor(g_hi, dtype=torch.int64, device=dev)[:, None]
    head = gi < ghi
    tail = gi >= glo
    win = ~head & ~tail
    # 3. exact masses above, inside and below the bracket
    m = torch.round(torch.ldexp(w, torch.tensor(MASS_BITS, device=dev))).to(torch.int64)
    sums = torch.stack([_limbs(torch.where(head, m, 0)), _limbs(torch.where(win, m, 0)),
                        _limbs(torch.where(tail, m, 0))], dim=1)  # [rows, 3, 2]
    _all_reduce(sums, dist.ReduceOp.SUM, group)
    sums_h = sums.cpu()
    # 4. the window keys, gathered; the exact cut
    gidx = torch.arange(key0, key0 + nl, dtype=torch.int64, device=dev)
    cuts = []
    for r in range(rows):
        sel = torch.nonzero(win[r]).flatten()
        mine = torch.stack([s[r, sel], gidx[sel].to(torch.float64)], 1) \
            if len(sel) else torch.zeros((0, 2), dtype=torch.float64, device=dev)
        # masses travel as exact integers, in two 31-bit halves
        mine_m = torch.stack([m[r, sel] >> LIMB, m[r, sel] & ((1 << LIMB) - 1)], 1) \
            if len(sel) else torch.zeros((0, 2), dtype=torch.int64, device=dev)
        allc = torch.cat(_all_gather_padded(mine, group), 0).cpu()
        allm = torch.cat(_all_gather_padded(mine_m, group), 0).cpu()
        Zr = sum(_from_limbs(sums_h[r, j]) for j in range(3))
        C = _from_limbs(sums_h[r, 0])
        # ranking: logit descending, then index ascending
        order = sorted(range(allc.shape[0]), key=lambda i: (-float(allc[i, 0]), int(allc[i, 1])))
        cut = None
        for i in order:
            C += (int(allm[i, 0]) << LIMB) + int(allm[i, 1])
            if _certified(Zr, C, eps):
                cut = (float(allc[i, 0]), int(allc[i, 1]), C)
                break
        if cut is None:
            raise RuntimeError("the bracket did not contain the cut")
        cuts.append(cut)
    # 5. kept and dropped value sums and weights
    kept = head.clone()
    for r in range(rows):
        xs, ix, _ = cuts[r]
        kept[r] |= win[r] & ((s[r] > xs) | ((s[r] == xs) & (gidx <= ix)))
    kf = kept.to(torch.float64)
    part = torch.stack([torch.einsum("rk,rkd->rd", w * kf, V), torch.einsum("rk,rkd->rd", w * (1 - kf), V)], 1)
    wsum = torch.stack([(w * kf).sum(1), (w * (1 - kf)).sum(1)], 1)
    nk = kept.sum(1)
    _all_reduce(part, dist.ReduceOp.SUM, group)
    _all_reduce(wsum, dist.ReduceOp.SUM, group)
    _all_reduce(nk, dist.ReduceOp.SUM, group)
    # 6. the kept indices, ascending over the ranks
    idx = [torch.cat(_all_gather_padded(gidx[kept[r]], group), 0).cpu() for r in range(rows)]
    part, wsum, nk = part.cpu(), wsum.cpu(), nk.cpu()
    out = torch.zeros((rows, V.shape[-1]), dtype=torch.float64)
    tv = torch.zeros(rows, dtype=torch.float64)
    kl = torch.zeros(rows, dtype=torch.float64)
    err = torch.zeros(rows, dtype=torch.float64)
    for r in range(rows):
        Zr = sum(_from_limbs(sums_h[r, j]) for j in range(3))
        C = cuts[r][2]
        tv[r] = float(Z_minus := Zr - C) / float(Zr)
        hm = math.ldexp(float(C), -MASS_BITS)
        out[r] = part[r, 0] / hm
        kl[r] = math.log1p(float(wsum[r, 1] / wsum[r, 0]))
        if Z_minus > 0:
            mu_t = part[r, 1] / math.ldexp(float(Z_minus), -MASS_BITS)
            err[r] = tv[r] * torch.linalg.vector_norm(mu_t - out[r])
    return {"k": nk, "idx": idx, "tv": tv, "kl": kl, "err": err, "out": out}
