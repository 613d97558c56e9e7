"""Pin: the Gaussian-score design rule k_eps / n ~ Phi_c(sigma + Phi^{-1}(eps)).

The abstract of "A Mathematical Theory of Top-k Sparse Attention via Total
Variation Distance" (arXiv 2512.07647v1, fugumt.com page) states that under
i.i.d. Gaussian scores s_i ~ N(mu, sigma^2) the minimal k_eps with
TV <= eps satisfies k_eps / n ~ Phi_c(sigma + Phi^{-1}(eps)) asymptotically.

The rule is asymptotic, so the check is on the row mean of k_eps / n at large
n.  Independently of the page, the rule follows from the Gaussian identity
E[e^s 1{s < t}] = e^{mu + sigma^2/2} Phi((t - mu)/sigma - sigma): the tail
mass below the cut t equals eps when (t - mu)/sigma = sigma + Phi^{-1}(eps),
and the fraction of keys above the cut is then Phi_c(sigma + Phi^{-1}(eps)).
The second test checks that identity by quadrature, so a wrong rule in the
first test could not pass by accident.
"""
import numpy as np
import pytest
from scipy import integrate, special

import oracle
from certified_top_sparse_b200 import workloads as W


def predicted_fraction(sigma: float, eps: float) -> float:
    return float(special.ndtr(-(sigma + special.ndtri(eps))))


@pytest.mark.parametrize("sigma", W.SWEEP_SIGMA)
def test_gaussian_rule_n65536(sigma):
    n, m = 65536, 64
    prob = W.sweep_cell(n=n, sigma=sigma, m=m)
    for eps in W.SWEEP_EPS:
        r = oracle.certified_topk_attn(W.raw_words(prob.q), W.raw_words(prob.K),
                                       W.raw_words(prob.V), eps, n_heads=1, n_kv_heads=1, m=m,
                                       select_only=True)
        frac = r["k"].mean() / n
        pred = predicted_fraction(sigma, eps)
        assert abs(frac - pred) <= 0.01, (sigma, eps, frac, pred)
        # every row still carries its certificate and is minimal
        assert np.all(r["tv"] <= eps) and np.all(r["tv_km1"] > eps)


@pytest.mark.slow
@pytest.mark.parametrize("sigma", (1.0, 2.0))
def test_gaussian_rule_n262144(sigma):
    n, m = 262144, 16
    prob = W.sweep_cell(n=n, sigma=sigma, m=m)
    for eps in W.SWEEP_EPS:
        r = oracle.certified_topk_attn(W.raw_words(prob.q), W.raw_words(prob.K),
                                       W.raw_words(prob.V), eps, n_heads=1, n_kv_heads=1, m=m,
                                       select_only=True)
        frac = r["k"].mean() / n
        assert abs(frac - predicted_fraction(sigma, eps)) <= 0.005, (sigma, eps, frac)


@pytest.mark.parametrize("sigma", (0.5, 1.0, 2.0, 3.0))
@pytest.mark.parametrize("eps", (0.1, 0.01, 0.001))
def test_gaussian_tail_identity_by_quadrature(sigma, eps):
    """The fraction Phi_c(sigma + Phi^{-1}(eps)) of N(0, sigma^2) scores lies
    above the cut t = sigma (sigma + Phi^{-1}(eps)), and the softmax mass below
    that cut is eps (integrals done numerically)."""
    t = sigma * (sigma + special.ndtri(eps))
    pdf = lambda s: np.exp(-0.5 * (s / sigma) ** 2) / (sigma * np.sqrt(2 * np.pi))
    below, _ = integrate.quad(lambda s: np.exp(s) * pdf(s), -np.inf, t, epsabs=1e-13)
    total = np.exp(sigma**2 / 2)
    assert below / total == pytest.approx(eps, rel=1e-7)
    frac_above, _ = integrate.quad(pdf, t, np.inf, epsabs=1e-13)
    assert frac_above == pytest.approx(predicted_fraction(sigma, eps), abs=1e-9)
