"""Pins for the fp64 oracle: what the pages and the mathematics fix.

Each test checks the oracle against something other than itself:
  * a hand-derived worked example (tests/golden/worked_example.json);
  * the identity TV = discarded tail mass = 1 - exp(-KL(P-hat || P)) and the
    definition TV = 1/2 sum |P - P-hat|, computed independently;
  * the exact head-tail factorisation of the output error against a plain
    dense softmax attention, and the diameter bound;
  * the Var_P(V) refinement (derived by the law of total variance);
  * brute force over all subsets on tiny n;
  * closed-form special cases (uniform logits, one dominant key);
  * the single-gap bound (derived from the ordered logits).
Source of every definition: abstract of "A Mathematical Theory of Top-k Sparse
Attention via Total Variation Distance" (arXiv 2512.07647v1, fugumt.com page).
"""
import itertools
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest

import oracle
from certified_top_sparse_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "worked_example.json")


def _ev(expr: str) -> float:
    return float(eval(expr.replace("^", "**"), {"__builtins__": {}},
                      {"ln": math.log, "sqrt": math.sqrt}))


def _run(prob: W.Problem, eps=None, **kw):
    dt = oracle.BF16 if prob.q.dtype != np.float32 and str(prob.q.dtype) == "torch.bfloat16" \
        else oracle.F32
    return oracle.certified_topk_attn(
        W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V),
        prob.eps if eps is None else eps, n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads,
        dtype=dt, batch=prob.batch, m=prob.m, **kw)


# ---------------------------------------------------------------------------
# worked example


@pytest.mark.parametrize("case", json.load(open(GOLDEN))["cases"], ids=lambda c: c["name"])
def test_worked_example(case):
    d = case["d"]
    q = np.array(case["q"], np.float32).reshape(1, 1, 1, d)
    K = np.array(case["K"], np.float32).reshape(1, 1, -1, d)
    V = np.array(case["V"], np.float32).reshape(1, 1, -1, d)
    r = oracle.certified_topk_attn(q, K, V, case["eps"], n_heads=1, n_kv_heads=1, want_diam=True)
    e = case["expect"]
    # fp32 rounding of ln 4 and ln 2 perturbs the masses by ~4e-9 relative.
    tol = 1e-7
    assert int(r["k"][0]) == e["k"]
    assert r["idx"][0].tolist() == e["idx"]
    for key in ("tv", "tv_km1", "head_mass", "kl", "err", "diam", "var_p"):
        if key in e:
            assert r[key][0] == pytest.approx(_ev(e[key]), abs=tol), key
    np.testing.assert_allclose(r["out"][0], [_ev(x) for x in e["out"]], atol=tol)
    if "attn" in e:
        np.testing.assert_allclose(r["attn"][0], [_ev(x) for x in e["attn"]], atol=tol)


# ---------------------------------------------------------------------------
# identities and bounds on seeded random rows


def _small_problems():
    yield W.tiny(n=700, d=64, n_heads=6)
    yield W.decode32k(batch=1, n_heads=8, n_kv_heads=2, n=3000, d=128)
    yield W.bert(batch=1, n_heads=2, n=96, d=64, sharp_from=1)
    yield W.sweep_cell(n=2048, sigma=2.0, m=8, eps=0.1)


@pytest.mark.parametrize("prob", list(_small_problems()), ids=lambda p: p.name)
def test_tv_identities_and_factorisation(prob):
    r = _run(prob, want_diam=prob.n <= 1024)
    # TV three ways: tail mass, definition, 1 - exp(-KL) (paper abstract identity).
    np.testing.assert_allclose(r["tv_def"], r["tv"], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["one_minus_exp_neg_kl"], r["tv"], rtol=0, atol=1e-12)
    # KL(P-hat || P) = -log H exactly for a truncation.
    np.testing.assert_allclose(r["kl"], -np.log(r["head_mass"]), rtol=1e-10, atol=1e-13)
    # Head-tail factorisation against a plain dense attention pass.
    np.testing.assert_allclose(r["err"], r["err_direct"], rtol=1e-10, atol=1e-14)
    dense = oracle.dense_attn(W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V),
                              n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads,
                              dtype=oracle.BF16 if "bfloat16" in str(prob.q.dtype) else oracle.F32,
                              batch=prob.batch, m=prob.m)
    np.testing.assert_allclose(r["attn"], dense, rtol=0, atol=1e-12)
    direct = np.linalg.norm(dense - r["out"], axis=1)
    np.testing.assert_allclose(r["err"], direct, rtol=1e-9, atol=1e-13)
    # Certificate and minimality: TV(k) <= eps < TV(k-1).
    assert np.all(r["tv"] <= prob.eps)
    assert np.all(r["tv_km1"] > prob.eps)
    # Diameter bound and the Var_P(V) refinement.
    if prob.n <= 1024:
        assert np.all(r["err"] <= r["tv"] * r["diam"] * (1 + 1e-12))
    tau = r["tv"]
    assert np.all(r["err"] ** 2 <= tau / (1 - tau) * r["var_p"] * (1 + 1e-9) + 1e-300)
    # Single-gap bound from the ordered logits.
    assert np.all(r["tv"] <= r["gap_bound"] * (1 + 1e-12))
    # idx: ascending, unique, in range; out is a convex combination of the head rows.
    for row, ids in enumerate(r["idx"]):
        assert len(ids) == r["k"][row]
        assert np.all(np.diff(ids) > 0) and ids[0] >= 0 and ids[-1] < prob.n


def test_rows_match_independent_softmax():
    """P, ranking and k recomputed with numpy from the same bytes."""
    prob = W.decode32k(batch=1, n_heads=4, n_kv_heads=2, n=777, d=128)
    r = _run(prob)
    q = prob.q.float().numpy().astype(np.float64)
    K = prob.K.float().numpy().astype(np.float64)
    V = prob.V.float().numpy().astype(np.float64)
    g = prob.n_heads // prob.n_kv_heads
    for h in range(prob.n_heads):
        u = K[0, h // g] @ q[0, h, 0]
        s = u / math.sqrt(prob.d)
        order = np.lexsort((np.arange(prob.n), -u))
        P = np.exp(s - s.max())
        P /= P.sum()
        tail = np.concatenate([np.cumsum(P[order][::-1])[::-1][1:], [0.0]])  # tail after top-(r+1)
        k = int(np.argmax(tail <= prob.eps)) + 1
        assert k == r["k"][h]
        assert sorted(order[:k].tolist()) == r["idx"][h].tolist()
        head = order[:k]
        mu = (P[head, None] * V[0, h // g, head]).sum(0) / P[head].sum()
        np.testing.assert_allclose(r["out"][h], mu, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------
# brute force on tiny n


def _rows_with_logits(logits, d=8, seed=0):
    """A problem whose query/key bytes realise the given logit rows exactly in
    fp64 (keys carry the logit in channel 0 and q = (sqrt(d), 0, ...))."""
    logits = np.asarray(logits, np.float32)
    rows, n = logits.shape
    rng = np.random.default_rng(seed)
    q = np.zeros((1, rows, 1, d), np.float32)
    q[..., 0] = math.sqrt(d)  # sqrt(8) is not exact in fp32; the oracle uses the fp32 value
    K = np.zeros((1, rows, n, d), np.float32)
    K[0, :, :, 0] = logits
    V = rng.standard_normal((1, rows, n, d)).astype(np.float32)
    return q, K, V


@pytest.mark.parametrize("seed", range(6))
def test_bruteforce_minimal_k_and_optimal_set(seed):
    rng = np.random.default_rng(100 + seed)
    rows, n = 4, 10
    logits = rng.normal(0, 1.5, (rows, n)).round(1)      # rounding to 0.1 creates ties
    q, K, V = _rows_with_logits(logits, seed=seed)
    for eps in (0.05, 0.2, 0.45):
        r = oracle.certified_topk_attn(q, K, V, eps, n_heads=rows, n_kv_heads=rows)
        for row in range(rows):
            u = K[0, row, :, 0].astype(np.float64) * float(q[0, row, 0, 0])
            s = u / math.sqrt(8)
            P = np.exp(s - s.max())
            P /= P.sum()
            best = {}
            for size in range(1, n + 1):
                best[size] = max(sum(P[list(c)]) for c in itertools.combinations(range(n), size))
            feasible = [size for size in range(1, n + 1) if 1 - best[size] <= eps]
            margins = [abs(1 - best[size] - eps) for size in range(1, n + 1)]
            if min(margins) < 1e-12:
                continue  # a boundary within rounding: skip, brute force in fp64 cannot decide
            k = min(feasible)
            assert r["k"][row] == k
            ids = r["idx"][row]
            assert sum(P[ids]) == pytest.approx(best[k], rel=1e-12)
            # among equal-mass optimal sets, the lower-index tie-break is used
            order = sorted(range(n), key=lambda i: (-u[i], i))
            assert sorted(order[:k]) == ids.tolist()


# ---------------------------------------------------------------------------
# closed-form special cases


@pytest.mark.parametrize("n", [1, 2, 7, 100, 1000, 4097])
@pytest.mark.parametrize("eps", [0.5, 0.3, 0.1, 0.01, 1e-3, 0.999])
def test_uniform_logits_exact(n, eps):
    """q = 0: P_i = 1/n, so k_eps is the least k with (n-k)/n <= eps, in exact
    rationals on the fp64 value of eps (the discarded mass (n-k)/n is computed
    by the oracle as an exact integer count divided by n)."""
    q = np.zeros((1, 1, 1, 16), np.float32)
    rng = np.random.default_rng(n)
    K = rng.standard_normal((1, 1, n, 16)).astype(np.float32)
    V = rng.standard_normal((1, 1, n, 16)).astype(np.float32)
    r = oracle.certified_topk_attn(q, K, V, eps, n_heads=1, n_kv_heads=1)
    e = Fraction(eps)
    k = next(k for k in range(1, n + 1) if Fraction(n - k, n) <= e)
    if k > 1 and abs(Fraction(n - k + 1, n) - e) < Fraction(1, 2**50):
        # (n-k+1)/n lies within fp64 rounding of eps: the fp64 test may keep k-1.
        assert r["k"][0] in (k - 1, k)
        k = int(r["k"][0])
    assert r["k"][0] == k
    assert r["idx"][0].tolist() == list(range(k))         # ties: lowest indices first
    assert r["tv"][0] == pytest.approx((n - k) / n, abs=1e-15)
    np.testing.assert_allclose(r["out"][0], V[0, 0, :k].astype(np.float64).mean(0), atol=1e-12)


@pytest.mark.parametrize("n", [2, 64, 5000])
def test_one_dominant_key(n):
    """One key 40 logits above the rest: k = 1 for every eps above the tail
    mass (n-1)e^-40/(1 + (n-1)e^-40); TV equals that closed form."""
    d = 4
    q = np.array([[[[2.0, 0, 0, 0]]]], np.float32)
    K = np.zeros((1, 1, n, d), np.float32)
    j = n // 3
    K[0, 0, j, 0] = 40.0
    V = np.arange(n * d, dtype=np.float32).reshape(1, 1, n, d) / (n * d)
    tail = (n - 1) * math.exp(-40.0) / (1 + (n - 1) * math.exp(-40.0))
    r = oracle.certified_topk_attn(q, K, V, 1e-6, n_heads=1, n_kv_heads=1)
    assert r["k"][0] == 1 and r["idx"][0].tolist() == [j]
    assert r["tv"][0] == pytest.approx(tail, rel=1e-12)
    np.testing.assert_allclose(r["out"][0], V[0, 0, j].astype(np.float64), atol=0)
    # eps = half the tail: the n-1 equal keys must shrink to at most (n-1)/2,
    # so k = ceil((n+1)/2) (n even here, no exact boundary), lowest indices first.
    r2 = oracle.certified_topk_attn(q, K, V, tail * 0.5, n_heads=1, n_kv_heads=1)
    k2 = (n + 2) // 2
    assert r2["k"][0] == k2
    others = [i for i in range(n) if i != j][: k2 - 1]
    assert r2["idx"][0].tolist() == sorted(others + [j])


def test_two_keys_closed_form():
    """n = 2 with logit gap D: P = (1/(1+e^-D), e^-D/(1+e^-D))."""
    d = 4
    for D in (0.0, 0.5, 3.0, 10.0):
        q = np.array([[[[2.0, 0, 0, 0]]]], np.float32)
        K = np.zeros((1, 1, 2, d), np.float32)
        K[0, 0, 1, 0] = D  # key 1 is the larger one
        V = np.zeros((1, 1, 2, d), np.float32)
        V[0, 0, 0, 1] = 1.0
        V[0, 0, 1, 0] = 1.0
        p_small = math.exp(-float(np.float32(D))) / (1 + math.exp(-float(np.float32(D))))
        for eps in (0.6 * p_small, 1.5 * p_small):
            if eps >= 1:
                continue
            r = oracle.certified_topk_attn(q, K, V, eps, n_heads=1, n_kv_heads=1)
            if eps >= p_small:
                assert r["k"][0] == 1 and r["idx"][0].tolist() == ([1] if D > 0 else [0])
                assert r["tv"][0] == pytest.approx(p_small, rel=1e-13)
                assert r["err"][0] == pytest.approx(p_small * math.sqrt(2), rel=1e-12)
                # one kept and one dropped key: the single-gap bound is exact
                assert r["gap_bound"][0] == pytest.approx(p_small, rel=1e-12)
            else:
                assert r["k"][0] == 2 and r["tv"][0] == 0.0 and r["err"][0] == 0.0


def test_single_gap_bound_exact_for_two_logit_levels():
    """k keys at logit a and n - k at logit b < a: TV(k) = (n-k) e^b / (k e^a + (n-k) e^b)
    = 1 / (1 + k/(n-k) e^(a-b)), which is the single-gap bound itself."""
    d = 16
    for n, k, gap in ((10, 3, 1.5), (50, 7, 3.0), (9, 1, 0.25)):
        q = np.zeros((1, 1, 1, d), np.float32)
        q[0, 0, 0, 0] = 4.0
        K = np.zeros((1, 1, n, d), np.float32)
        hi = np.random.default_rng(n).choice(n, size=k, replace=False)
        K[0, 0, hi, 0] = gap  # scaled logit gap: 4 * gap / sqrt(16) = gap
        V = np.random.default_rng(k).standard_normal((1, 1, n, d)).astype(np.float32)
        tv_k = 1.0 / (1.0 + k / (n - k) * math.exp(gap))
        tv_km1 = ((n - k) + math.exp(gap)) / (k * math.exp(gap) + (n - k))  # k - 1 of the top kept
        eps = tv_k + 0.25 * (tv_km1 - tv_k)
        r = oracle.certified_topk_attn(q, K, V, eps, n_heads=1, n_kv_heads=1)
        assert r["k"][0] == k and r["idx"][0].tolist() == sorted(hi.tolist())
        assert r["tv"][0] == pytest.approx(tv_k, rel=1e-12)
        assert r["gap_bound"][0] == pytest.approx(tv_k, rel=1e-12)


def test_gqa_head_mapping():
    """Query head h reads KV head h // (n_heads / n_kv_heads): permuting KV heads
    permutes the results of the matching query-head blocks."""
    prob = W.decode32k(batch=2, n_heads=8, n_kv_heads=4, n=300, d=128)
    r = _run(prob)
    perm = [2, 0, 3, 1]
    K2 = prob.K[:, perm].contiguous()
    V2 = prob.V[:, perm].contiguous()
    qperm = []
    for new_kv in range(4):
        old_kv = perm[new_kv]
        qperm += [old_kv * 2, old_kv * 2 + 1]
    q2 = prob.q[:, qperm].contiguous()
    r2 = oracle.certified_topk_attn(W.raw_words(q2), W.raw_words(K2), W.raw_words(V2), prob.eps,
                                    n_heads=8, n_kv_heads=4, dtype=oracle.BF16, batch=2)
    k1 = r["k"].reshape(2, 8)
    k2 = r2["k"].reshape(2, 8)
    np.testing.assert_array_equal(k2, k1[:, qperm])


# ---------------------------------------------------------------------------
# the truncation to a given kept set, and the fp32 tie allowance

KEPT = os.path.join(os.path.dirname(__file__), "golden", "kept_set_and_tie_bound.json")


def _ev2(expr: str) -> float:
    return float(eval(expr.replace("^", "**"), {"__builtins__": {}},
                      {"ln": math.log, "sqrt": math.sqrt, "exp": math.exp}))


def test_eval_kept_set_hand_derived():
    """Arbitrary (non-top-k) kept sets of the four-key example, hand-derived."""
    c = json.load(open(KEPT))["kept_set_cases"]
    d = c["d"]
    q = np.array(c["q"], np.float32).reshape(1, 1, 1, d)
    K = np.array(c["K"], np.float32).reshape(1, 1, -1, d)
    V = np.array(c["V"], np.float32).reshape(1, 1, -1, d)
    for s in c["sets"]:
        r = oracle.eval_kept_set(q, K, V, [s["set"]], n_heads=1, n_kv_heads=1)
        for key in ("tv", "kl", "err", "tv_drop_lowest"):
            assert r[key][0] == pytest.approx(_ev2(s[key]), abs=1e-7), (s["set"], key)
        np.testing.assert_allclose(r["out"][0], [_ev2(x) for x in s["out"]], atol=1e-7)


@pytest.mark.parametrize("prob", list(_small_problems()), ids=lambda p: p.name)
def test_eval_kept_set_on_the_top_k_set(prob):
    """On the certified set itself the set evaluation reproduces the main
    routine's TV, KL, err and output, and dropping the lowest kept key gives
    TV(k - 1); on a perturbed set (the last kept key swapped for the first
    dropped one) TV grows by exactly their mass difference."""
    o = _run(prob)
    dt = oracle.BF16 if str(prob.q.dtype) == "torch.bfloat16" else oracle.F32
    raw = dict(n_heads=prob.n_heads, n_kv_heads=prob.n_kv_heads, dtype=dt, batch=prob.batch,
               m=prob.m)
    e = oracle.eval_kept_set(W.raw_words(prob.q), W.raw_words(prob.K), W.raw_words(prob.V),
                             o["idx"], **raw)
    np.testing.assert_allclose(e["tv"], o["tv"], rtol=1e-10, atol=1e-14)
    np.testing.assert_allclose(e["kl"], o["kl"], rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(e["err"], o["err"], rtol=1e-9, atol=1e-14)
    np.testing.assert_allclose(e["out"], o["out"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(e["tv_drop_lowest"], o["tv_km1"], rtol=1e-10, atol=1e-14)


def test_eval_kept_set_brute_force_masses():
    """TV of random subsets of a tiny row equals the dropped mass of an
    independent numpy softmax (fp64 from the same fp32 inputs)."""
    rng = np.random.default_rng(5)
    n, d = 11, 8
    q = rng.standard_normal((1, 1, 1, d)).astype(np.float32) * 2
    K = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    V = rng.standard_normal((1, 1, n, d)).astype(np.float32)
    u = K[0, 0].astype(np.float64) @ q[0, 0, 0].astype(np.float64)
    P = np.exp((u - u.max()) / math.sqrt(d))
    P /= P.sum()
    order = sorted(range(n), key=lambda i: (-u[i], i))
    for trial in range(40):
        size = int(rng.integers(1, n + 1))
        s = rng.choice(n, size, replace=False)
        r = oracle.eval_kept_set(q, K, V, [s], n_heads=1, n_kv_heads=1)
        keep = np.zeros(n, bool)
        keep[s] = True
        assert r["tv"][0] == pytest.approx(P[~keep].sum(), abs=1e-13)
        low = max(s, key=lambda i: order.index(i))
        assert r["tv_drop_lowest"][0] == pytest.approx(P[~keep].sum() + P[low], abs=1e-13)
        mu = (P[keep, None] * V[0, 0][keep].astype(np.float64)).sum(0) / P[keep].sum()
        np.testing.assert_allclose(r["out"][0], mu, rtol=1e-12, atol=1e-13)


def test_tie_bound_hand_derived():
    """The fp32 rounding allowance of the boundary keys (class T of the parity
    tests): gamma_d with 2^-24 and absolute products of both boundary keys."""
    c = json.load(open(KEPT))["tie_bound_case"]
    d = c["d"]
    q = np.array(c["q"], np.float32).reshape(1, 1, 1, d)
    K = np.array(c["K"], np.float32).reshape(1, 1, -1, d)
    V = np.zeros_like(K)
    r = oracle.certified_topk_attn(q, K, V, c["eps"], n_heads=1, n_kv_heads=1)
    e = c["expect"]
    assert int(r["k"][0]) == e["k"] and r["idx"][0].tolist() == e["idx"]
    assert r["gap_u"][0] == _ev2(e["gap_u"])
    assert r["tie_bound"][0] == pytest.approx(_ev2(e["tie_bound"]), rel=1e-15)
    assert r["tv"][0] == pytest.approx(_ev2(e["tv"]), rel=1e-12)
    assert r["gap_bound"][0] == pytest.approx(_ev2(e["gap_bound"]), rel=1e-12)
