"""GPU <-> fp64 oracle parity of cta_certified_topk_attn, called through the C ABI.

Small cases span several chunks with a ragged tail and run the oracle on
every row; the five full-size workloads run the GPU in the launch
configuration the benchmark times and compare sampled rows (whole
(batch, KV-head) groups, which the oracle computes as problems of their own).
Tolerances and exemption classes are stated in tests/parity.py.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from certified_top_sparse_b200 import workloads as W
import certified_top_sparse_b200 as cta
from parity import check_out, compare, group_rows, run_oracle, sub_problem, to_host

pytestmark = pytest.mark.gpu

REPORT = os.environ.get("CTA_PARITY_REPORT")


def _report(name, rep):
    if REPORT:
        with open(REPORT, "a") as f:
            f.write(json.dumps({"case": name, **rep}) + "\n")


def gpu_run(prob: W.Problem, eps: float, q=None, **kw):
    dev = torch.device("cuda")
    qq = (prob.q if q is None else q).to(dev)
    K, V = prob.K.to(dev), prob.V.to(dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    kw.setdefault("want_gap", True)
    res = cta.cta_certified_topk_attn(qq, K, V, eps, status_dev=status, **kw)
    torch.cuda.synchronize()
    h = to_host(res)
    h["status"] = int(status.item())
    return h


def check(prob, eps, name, **kw):
    g = gpu_run(prob, eps, **kw)
    assert g["status"] == 0, f"device status {g['status']:#x}"
    o = run_oracle(prob, eps)
    rep = compare(prob, eps, g, o)
    _report(name, rep)
    return g, o, rep


# ---------------------------------------------------------------------------
# small cases, every row checked


@pytest.mark.parametrize("n", [1, 2, 3, 17, 255, 256, 257, 1000, 3001, 9999])
def test_ragged_n_fp32_d64(n):
    prob = W.tiny(n=n, d=64, n_heads=4)
    check(prob, 0.01, f"tiny n={n}")


def test_tiny_full_config():
    prob = W.tiny()
    g, o, rep = check(prob, prob.eps, "tiny (full config)")
    assert rep["exact"] == prob.rows


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.float32, 128),
                                     (torch.bfloat16, 64), (torch.bfloat16, 128)])
@pytest.mark.parametrize("eps", [0.3, 0.01, 1e-4])
def test_dtype_and_head_dim(dtype, d, eps):
    prob = W.decode32k(batch=2, n_heads=8, n_kv_heads=2, n=5000 + d, d=d)
    if dtype == torch.float32:
        prob.q, prob.K, prob.V = prob.q.float(), prob.K.float(), prob.V.float()
    check(prob, eps, f"decode {dtype} d={d} eps={eps}")


@pytest.mark.parametrize("n_heads,n_kv,m", [(8, 8, 1), (16, 2, 1), (6, 2, 3), (4, 1, 5), (2, 2, 33)])
def test_gqa_groups_and_query_rows(n_heads, n_kv, m):
    rng = np.random.default_rng(n_heads * 100 + m)
    d, n = 64, 2500
    q = torch.from_numpy(rng.standard_normal((2, n_heads, m, d)).astype(np.float32) * 1.5)
    K = torch.from_numpy(rng.standard_normal((2, n_kv, n, d)).astype(np.float32))
    V = torch.from_numpy(rng.standard_normal((2, n_kv, n, d)).astype(np.float32))
    prob = W.Problem("gqa", q, K, V, 0.05, 2, n_heads, n_kv, m, n, d)
    check(prob, 0.05, f"gqa h={n_heads} kv={n_kv} m={m}")


# bf16 values with d = 128 take the tensor-core output pass: row tiles of 1, 2
# and 4 rows, partial last tiles, several tiles per KV group, m > 1, ragged
# key tails and (batch 8) several work items per CTA.
@pytest.mark.parametrize("n_heads,n_kv,m,n", [(8, 8, 1, 2500), (8, 4, 1, 2500), (3, 1, 1, 2500),
                                              (16, 2, 1, 2500), (6, 2, 3, 1111), (2, 2, 33, 700),
                                              (4, 1, 1, 128), (4, 1, 1, 129), (4, 2, 1, 9999)])
def test_gqa_groups_bf16_d128_tensor_core_values(n_heads, n_kv, m, n):
    rng = np.random.default_rng(n_heads * 1000 + m * 10 + n)
    d = 128
    q = rng.standard_normal((2, n_heads, m, d)).astype(np.float32) * 1.5
    K = rng.standard_normal((2, n_kv, n, d)).astype(np.float32)
    V = rng.standard_normal((2, n_kv, n, d)).astype(np.float32)
    bf = lambda a: torch.from_numpy(a).to(torch.bfloat16)
    prob = W.Problem("gqa-bf16", bf(q), bf(K), bf(V), 0.05, 2, n_heads, n_kv, m, n, d)
    check(prob, 0.05, f"gqa bf16 d=128 h={n_heads} kv={n_kv} m={m} n={n}")


@pytest.mark.parametrize("n", [1, 17, 100, 127])
def test_bf16_d128_shorter_than_one_stage(n):
    # fewer keys than one 128-key tensor-core stage: the CUDA-core kernels take over
    rng = np.random.default_rng(7000 + n)
    d = 128
    bf = lambda a: torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16)
    q = bf(rng.standard_normal((1, 8, 1, d)) * 1.5)
    K, V = bf(rng.standard_normal((1, 2, n, d))), bf(rng.standard_normal((1, 2, n, d)))
    prob = W.Problem("short-bf16", q, K, V, 0.05, 1, 8, 2, 1, n, d)
    check(prob, 0.05, f"bf16 d=128 n={n}")


@pytest.mark.parametrize("want_err", [True, False])
def test_tensor_core_values_many_items_per_cta(want_err):
    # 64 (batch, KV head) units of 20000 keys: about four work items per CTA
    prob = W.decode32k(batch=8, n_heads=32, n_kv_heads=8, n=20000, d=128)
    g = gpu_run(prob, 0.01, want_err=want_err, want_kl=want_err)
    assert g["status"] == 0
    for b, kvh in ((0, 0), (3, 5), (7, 7)):
        sub = sub_problem(prob, b, kvh)
        rows = group_rows(prob, b, kvh)
        o = run_oracle(sub, 0.01)
        gg = {k: v for k, v in g.items()}
        if not want_err:
            gg["err"] = None
            gg["kl"] = None
        compare(sub, 0.01, gg, o, rows=rows)


@pytest.mark.parametrize("want_err", [True, False])
def test_back_to_back_calls_share_one_workspace(want_err):
    # Calls issued back to back on one stream with one workspace and no host
    # synchronisation between them: the next call's logits pass overlaps this
    # call's finalisation and the value pass starts during selection.  Every
    # call must still match the oracle.
    prob = W.decode128k(batch=1, n=40000, steps=4)
    dev = torch.device("cuda")
    K, V = prob.K.to(dev), prob.V.to(dev)
    qs = prob.meta["q_steps"].to(dev)
    ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                            batch=prob.batch), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    results = []
    for t in range(4):
        results.append(cta.cta_certified_topk_attn(qs[t], K, V, 0.01, workspace=ws,
                                                   status_dev=status, want_err=want_err,
                                                   want_kl=want_err, want_gap=True))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for t in range(4):
        g = to_host(results[t])
        for kvh in (0, 5):
            sub = sub_problem(prob, 0, kvh, q=prob.meta["q_steps"][t])
            o = run_oracle(sub, 0.01)
            compare(sub, 0.01, g, o, rows=group_rows(prob, 0, kvh))


@pytest.mark.parametrize("last_write", ["K", "V", "q"])
def test_inputs_written_by_the_preceding_kernel(last_write):
    # The caller appends the new key and value rows and writes the query with
    # its own kernels on the same stream, immediately before each call, with
    # no host synchronisation.  The new key is made to dominate the query's
    # logits, so a pass that read K, V or q before those kernels finished
    # would select or weight the wrong rows.  `last_write` is the tensor the
    # kernel just before the call writes.
    prob = W.decode128k(batch=1, n=40000, steps=4)
    dev = torch.device("cuda")
    g = prob.n_heads // prob.n_kv_heads
    K, V = prob.K.to(dev), prob.V.to(dev)
    q_dev = torch.zeros_like(prob.q, device=dev)
    ws = torch.empty(cta.cta_workspace_size(prob.n, prob.d, prob.n_heads, prob.n_kv_heads,
                                            batch=prob.batch), dtype=torch.uint8, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    rng = np.random.default_rng(77)
    steps = []
    for t in range(4):
        q_t = prob.meta["q_steps"][t]                          # [1, heads, 1, d]
        # a key along the summed queries of each KV group, scaled up
        qsum = q_t.float().reshape(prob.n_kv_heads, g, prob.d).sum(1)
        k_new = (qsum / qsum.norm(dim=1, keepdim=True) * (3.0 + t)).to(torch.bfloat16)
        v_new = torch.from_numpy(rng.standard_normal((prob.n_kv_heads, prob.d)).astype(np.float32) * 4.0
                                 ).to(torch.bfloat16)
        steps.append((q_t, k_new, v_new))
    writes_dev = [(a.to(dev), b.to(dev), c.to(dev)) for a, b, c in steps]
    torch.cuda.synchronize()
    big = torch.zeros(64 << 20, dtype=torch.float32, device=dev)  # delays the stream a little
    results = []
    for t, (q_t, k_new, v_new) in enumerate(writes_dev):
        big.add_(1.0)
        writes = {"q": lambda: q_dev.copy_(q_t),
                  "K": lambda: K[0, :, -1, :].copy_(k_new),
                  "V": lambda: V[0, :, -1, :].copy_(v_new)}
        for name in [x for x in ("q", "K", "V") if x != last_write] + [last_write]:
            writes[name]()
        results.append(cta.cta_certified_topk_attn(q_dev, K, V, 0.01, workspace=ws,
                                                   status_dev=status, want_err=True,
                                                   want_kl=True, want_gap=True))
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    K_h, V_h = prob.K.clone(), prob.V.clone()
    for t, (q_t, k_new, v_new) in enumerate(steps):
        K_h[0, :, -1, :] = k_new
        V_h[0, :, -1, :] = v_new
        mod = W.Problem(prob.name, q_t.clone(), K_h.clone(), V_h.clone(), prob.eps, prob.batch,
                        prob.n_heads, prob.n_kv_heads, prob.m, prob.n, prob.d)
        gres = to_host(results[t])
        for kvh in (0, 3, 7):
            sub = sub_problem(mod, 0, kvh)
            o = run_oracle(sub, 0.01)
            rows = group_rows(prob, 0, kvh)
            # the new key is among the kept keys of every row of the group
            assert all(prob.n - 1 in o["idx"][j] for j in range(len(rows)))
            compare(sub, 0.01, gres, o, rows=rows)


def test_bert_small_all_query():
    prob = W.bert(batch=1, n_heads=4, n=512, d=64, sharp_from=2)
    g, o, rep = check(prob, prob.eps, "bert small")


def _all_query(n, d, heads, dtype, seed, scale=1.0, levels=None):
    """Self-attention shaped problem (m = n, one KV head per query head)."""
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((1, heads, n, d)) * scale
    K = rng.standard_normal((1, heads, n, d))
    V = rng.standard_normal((1, heads, n, d))
    if levels is not None:  # keys drawn from a few distinct rows: many exactly tied logits
        K = K[:, :, rng.integers(0, levels, n), :]
    t = lambda a: torch.from_numpy(a.astype(np.float32)).to(dtype)
    return W.Problem("allq", t(q), t(K), t(V), 0.01, 1, heads, heads, n, n, d)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("want_err", [True, False])
def test_all_query_tensor_core_path(d, want_err):
    """bf16, 128-row tiles, n a multiple of 256: tcgen05 logits and value sums."""
    prob = _all_query(512, d, 2, torch.bfloat16, seed=d + int(want_err))
    check(prob, prob.eps, f"all-query tcgen05 d={d} err={want_err}", want_err=want_err,
          want_kl=want_err)


@pytest.mark.parametrize("n,dtype", [(384, torch.bfloat16), (512, torch.float32),
                                     (1024, torch.bfloat16), (96, torch.float32)])
def test_all_query_cuda_core_paths(n, dtype):
    """Short rows outside the tensor-core shapes: CUDA-core logits, warp-per-row selection."""
    prob = _all_query(n, 64, 2, dtype, seed=n)
    check(prob, prob.eps, f"all-query n={n} {dtype}")


@pytest.mark.parametrize("levels", [1, 3])
def test_short_rows_exact_ties(levels):
    """Keys from 1 or 3 distinct rows: whole bins of tied logits, resolved by the
    lower index (all-equal logits keep exactly ceil((1 - eps) n) keys)."""
    prob = _all_query(512, 64, 1, torch.bfloat16, seed=7, levels=levels)
    g, o, rep = check(prob, prob.eps, f"short rows ties levels={levels}")
    assert rep["exact"] == prob.rows
    if levels == 1:
        assert np.all(g["k"].reshape(-1) == 507)


def test_sweep_cell_small():
    prob = W.sweep_cell(n=4096, sigma=2.0, m=64)
    for eps in W.SWEEP_EPS:
        check(prob, eps, f"sweep n=4096 eps={eps}")


# ---------------------------------------------------------------------------
# degenerate inputs: ties, radix narrowing, extremes


def test_uniform_logits_all_ties_radix_path():
    """q = 0: every logit ties, the boundary bin holds all n keys (> shared
    capacity) and the radix narrowing over the key index decides the cut:
    k = least k with (n-k)/n <= eps, kept keys 0..k-1."""
    n, d = 100003, 64
    rng = np.random.default_rng(5)
    q = torch.zeros(1, 2, 1, d)
    K = torch.from_numpy(rng.standard_normal((1, 2, n, d)).astype(np.float32))
    V = torch.from_numpy(rng.standard_normal((1, 2, n, d)).astype(np.float32))
    prob = W.Problem("uniform", q, K, V, 0.3, 1, 2, 2, 1, n, d)
    g, o, rep = check(prob, 0.3, "uniform ties n=100003")
    assert np.all(g["k"] == o["k"])
    assert g["idx"][0, : g["k"][0]].tolist() == list(range(g["k"][0]))


def test_near_uniform_logits_radix_on_logit_bits():
    """Logits spread over ~1e-4: all keys share the first value bin, so the
    cut is found by radix digits of the logit bits."""
    n, d = 60000, 64
    prob = W.tiny(n=n, d=d, n_heads=2, sigmas=(1e-4, 3e-4))
    check(prob, 0.2, "near-uniform n=60000")


def test_one_dominant_key():
    n, d = 20000, 64
    q = torch.zeros(1, 1, 1, d)
    q[..., 0] = 8.0
    K = torch.zeros(1, 1, n, d)
    K[0, 0, 777, 0] = 40.0
    V = torch.randn(1, 1, n, d, generator=torch.Generator().manual_seed(3))
    prob = W.Problem("spike", q, K, V, 1e-3, 1, 1, 1, 1, n, d)
    g, o, rep = check(prob, 1e-3, "one dominant key")
    assert g["k"][0] == 1 and g["idx"][0, 0] == 777


def _sink_over_subquantum_background(n, d, dtype, gap_octaves):
    """One key 'gap_octaves' halvings of the weight above n - 1 tied background
    keys: each background weight is 2^-gap_octaves of the top one.  With
    gap_octaves just above 63 - ceil(log2 n), a fixed-point scale chosen from n
    alone (2^(62 - ceil(log2 n))) rounds every background weight to zero and
    would certify k = 1, TV = 0, although the true tail mass is
    (n - 1) 2^-gap_octaves / (1 + ...)."""
    s = gap_octaves * math.log(2.0) * math.sqrt(d)  # logit gap in dot-product units
    q = torch.zeros(1, 1, 1, d)
    q[..., 0] = 1.0
    K = torch.zeros(1, 1, n, d)
    K[0, 0, 0, 0] = s
    V = torch.randn(1, 1, n, d, generator=torch.Generator().manual_seed(11))
    if dtype == torch.bfloat16:
        q, K, V = q.to(dtype), K.to(dtype), V.to(dtype)
    return W.Problem("sink-subquantum", q, K, V, 1e-6, 1, 1, 1, 1, n, d)


@pytest.mark.parametrize("dtype,d", [(torch.float32, 64), (torch.bfloat16, 128)])
def test_mass_rounding_cannot_hide_a_large_tail(dtype, d):
    """n = 2^23: the background holds ~6e-6 of the mass in keys each below
    half of a unit of the old n-based fixed-point scale; the certificate must
    still see it (k > 1, TV = the oracle's)."""
    n = 1 << 23
    prob = _sink_over_subquantum_background(n, d, dtype, gap_octaves=40.3)
    g, o, rep = check(prob, 1e-6, f"sink over sub-quantum background {dtype} d={d}")
    assert o["tv_km1"][0] > 1e-6 and o["k"][0] > 1 and g["k"][0] > 1
    # The ~1.35M tied background keys each carry ~7e-13 of the mass; fp32
    # weights (an exponent of ~40.3 has a unit in the last place of ~4e-6)
    # move the cut among them by a few keys, which compare() has judged with
    # the oracle's own masses.  What must not happen is the collapse to k = 1.
    dropped = prob.n - int(o["k"][0])
    assert abs(int(g["k"][0]) - int(o["k"][0])) <= 1e-5 * dropped + 1
    assert abs(float(g["tv"][0]) - float(o["tv"][0])) <= 1e-7


@pytest.mark.parametrize("eps", [0.999, 0.5, 1e-7])
def test_extreme_eps(eps):
    prob = W.tiny(n=4096, d=64, n_heads=3)
    check(prob, eps, f"extreme eps={eps}")


def test_no_err_path_matches_err_path_bitwise():
    prob = W.decode32k(batch=1, n_heads=8, n_kv_heads=2, n=7000, d=128)
    a = gpu_run(prob, 0.1)
    b = gpu_run(prob, 0.1, want_err=False, want_kl=False)
    for key in ("k", "tv"):
        assert np.array_equal(a[key], b[key])
    for r in range(prob.rows):
        assert np.array_equal(a["idx"][r, : a["k"][r]], b["idx"][r, : b["k"][r]])
    assert np.array_equal(a["out"], b["out"])


def test_deterministic_repeat():
    prob = W.decode32k(batch=1, n_heads=8, n_kv_heads=2, n=20000, d=128)
    a = gpu_run(prob, 0.01)
    b = gpu_run(prob, 0.01)
    for key in ("k", "tv", "err", "kl", "out"):
        assert np.array_equal(a[key], b[key]), key


def test_nonfinite_input_sets_status():
    prob = W.tiny(n=3000, d=64, n_heads=2)
    prob.K[0, 1, 1234, 5] = float("nan")
    g = gpu_run(prob, 0.01)
    assert g["status"] & cta.CTA_DEV_NONFINITE
    # the row that does not read the bad key is unaffected
    o = run_oracle(W.Problem("row0", prob.q[:, :1].contiguous(), prob.K[:, :1].contiguous(),
                             prob.V[:, :1].contiguous(), 0.01, 1, 1, 1, 1, prob.n, prob.d), 0.01)
    assert g["k"][0] == o["k"][0]


def test_dense_reference_matches_oracle():
    import oracle
    for prob in (W.tiny(n=3333, d=64, n_heads=4),
                 W.decode32k(batch=1, n_heads=8, n_kv_heads=2, n=4444, d=128)):
        dev = torch.device("cuda")
        out = cta.cta_dense_attn(prob.q.to(dev), prob.K.to(dev), prob.V.to(dev))
        torch.cuda.synchronize()
        og = out.float().reshape(prob.rows, -1).cpu().numpy().astype(np.float64)
        oo = oracle.dense_attn(W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V),
                               n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads,
                               dtype=oracle.F32 if prob.q.dtype == torch.float32 else oracle.BF16)
        check_out(og, oo, prob.q.dtype)


def test_err_equals_distance_to_dense_fp32():
    """GPU-internal identity: err = ||Attn - Attn_k|| with Attn from cta_dense_attn."""
    prob = W.tiny(n=8192, d=64, n_heads=6)
    dev = torch.device("cuda")
    q, K, V = prob.q.to(dev), prob.K.to(dev), prob.V.to(dev)
    res = cta.cta_certified_topk_attn(q, K, V, 0.01)
    dense = cta.cta_dense_attn(q, K, V)
    torch.cuda.synchronize()
    direct = (dense - res["out"]).double().reshape(prob.rows, -1).norm(dim=1).cpu().numpy()
    err = res["err"].double().reshape(-1).cpu().numpy()
    assert np.allclose(err, direct, rtol=1e-3, atol=1e-6)
    # TV = 1 - exp(-KL) between the two independent reductions
    tv = res["tv"].double().reshape(-1).cpu().numpy()
    kl = res["kl"].double().reshape(-1).cpu().numpy()
    assert np.all(np.abs(tv + np.expm1(-kl)) <= 1e-6)


# ---------------------------------------------------------------------------
# full-size workloads: GPU at full size, oracle on sampled groups


def _sampled(prob, eps, groups, name, q=None, strict_window=1e-7):
    """Full-size GPU run, oracle on sampled groups.  Every sampled row outside
    class M at `strict_window` (and outside class T) must be exact."""
    g = gpu_run(prob, eps, q=q)
    assert g["status"] == 0
    reps = []
    for (b, kvh) in groups:
        sub = sub_problem(prob, b, kvh, q=q)
        o = run_oracle(sub, eps)
        reps.append(compare(sub, eps, g, o, rows=group_rows(prob, b, kvh),
                            strict_window=strict_window))
    rep = {"rows": sum(r["rows"] for r in reps), "exact": sum(r["exact"] for r in reps),
           "differing_exempt": sum(r["differing_exempt"] for r in reps),
           "classM": {w: sum(r["classM"][w] for r in reps) for w in reps[0]["classM"]},
           "classT": sum(r["classT"] for r in reps),
           "max_out_rel": max(r["max_out_rel"] for r in reps)}
    _report(name, rep)
    return g


def test_full_decode32k_sampled():
    prob = W.decode32k()
    _sampled(prob, prob.eps, [(0, 0), (1, 5), (3, 7)], "decode32k full (3 sampled groups)")


@pytest.mark.parametrize("eps", [0.01, 0.1])
def test_full_decode128k_sampled(eps):
    prob = W.decode128k(steps=3)
    for t in range(3):
        _sampled(prob, eps, [(0, t), (0, 7 - t)], f"decode128k eps={eps} step={t}",
                 q=prob.meta["q_steps"][t])


def test_full_bert_sampled():
    prob = W.bert()
    g = gpu_run(prob, prob.eps)
    assert g["status"] == 0
    for (b, h) in [(0, 0), (3, 5), (5, 6), (7, 11)]:
        sub = W.Problem("bert", prob.q[b:b + 1, h:h + 1].contiguous(),
                        prob.K[b:b + 1, h:h + 1].contiguous(), prob.V[b:b + 1, h:h + 1].contiguous(),
                        prob.eps, 1, 1, 1, prob.m, prob.n, prob.d)
        o = run_oracle(sub, prob.eps)
        rep = compare(sub, prob.eps, g, o, rows=group_rows(prob, b, h))
        _report(f"bert full (b={b}, h={h})", rep)


def test_full_sweep_gaussian_rule_and_sampled_parity():
    from scipy import special
    for n in W.SWEEP_N:
        for sigma in W.SWEEP_SIGMA:
            prob = W.sweep_cell(n=n, sigma=sigma)
            for eps in W.SWEEP_EPS:
                g = gpu_run(prob, eps)
                assert g["status"] == 0
                frac = g["k"].mean() / n
                pred = float(special.ndtr(-(sigma + special.ndtri(eps))))
                if n >= 65536:
                    assert abs(frac - pred) <= 0.01, (n, sigma, eps, frac, pred)
                rows = np.arange(0, prob.m, 37)
                sub = W.Problem("sweep", prob.q[:, :, rows].contiguous(), prob.K, prob.V, eps, 1,
                                1, 1, len(rows), n, prob.d)
                o = run_oracle(sub, eps)
                rep = compare(sub, eps, g, o, rows=rows)
                rep["k_over_n"] = frac
                rep["rule"] = pred
                _report(f"sweep n={n} sigma={sigma} eps={eps}", rep)
