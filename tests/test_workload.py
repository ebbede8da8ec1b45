"""The seeded synthetic inputs and the histogram statistics (host logic, no GPU).

The routing skew is drawn as p ~ Dirichlet(alpha * 1_E) in log space; its
marginal moments have a closed form (mean 1/E, variance (1/E)(1 - 1/E) /
(E alpha + 1)), which the sampler must reproduce over many draws.
"""

import math

import numpy as np
import pytest
import torch

from grouped_gemm_02_b200 import stats
from grouped_gemm_02_b200 import workload as wl


@pytest.mark.parametrize("E,alpha", [(8, 0.5), (16, 2.0), (4, 0.05)])
def test_dirichlet_marginal_moments(E, alpha):
    draws = np.stack([np.exp(wl.dirichlet_log_p(E, alpha, seed)) for seed in range(3000)])
    assert np.allclose(draws.sum(axis=1), 1.0, atol=1e-12)
    assert np.all(np.isfinite(np.log(draws)))
    mean_ref = 1.0 / E
    var_ref = (1.0 / E) * (1.0 - 1.0 / E) / (E * alpha + 1.0)
    # 3000 draws: the sample mean is within a few standard errors, the variance within ~10%
    assert abs(draws.mean() - mean_ref) < 1e-3
    assert abs(draws.var(axis=0).mean() / var_ref - 1.0) < 0.12


def test_dirichlet_skew_grows_as_alpha_shrinks():
    def eff(alpha):
        vals = []
        for seed in range(50):
            p = np.exp(wl.dirichlet_log_p(64, alpha, seed))
            vals.append(math.exp(-(p * np.log(p)).sum()))
        return float(np.mean(vals))
    e = [eff(a) for a in (0.02, 0.1, 1.0, 10.0)]
    assert e[0] < e[1] < e[2] < e[3] < 64.0
    assert e[0] < 4.0 and e[3] > 50.0


def test_dirichlet_and_inputs_are_seeded():
    assert np.array_equal(wl.dirichlet_log_p(64, 0.1, 7), wl.dirichlet_log_p(64, 0.1, 7))
    assert not np.array_equal(wl.dirichlet_log_p(64, 0.1, 7), wl.dirichlet_log_p(64, 0.1, 8))
    s = wl.TINY
    a, b, c = wl.make_inputs(s, seed=3), wl.make_inputs(s, seed=3), wl.make_inputs(s, seed=4)
    for n in a:
        assert torch.equal(a[n], b[n]), n
    assert not torch.equal(a["W1"], c["W1"])
    assert a["x"].shape == (s.T, s.d) and a["W1"].shape == (s.E, s.f, s.d) and a["W2"].shape == (s.E, s.d, s.f)
    assert a["bias"].dtype == torch.float32
    assert np.allclose(np.exp(a["bias"].double().numpy()).sum(), 1.0, atol=1e-5)


def test_weight_scale_follows_fan_in():
    s = wl.DECODE64.with_(E=2)
    w = wl.make_weights(s, seed=1)
    assert abs(w["W1"].float().std().item() * math.sqrt(s.d) - 1.0) < 0.01
    assert abs(w["W2"].float().std().item() * math.sqrt(s.f) - 1.0) < 0.01
    assert abs(w["W1"].float().mean().item()) < 1e-3


@pytest.mark.parametrize("T,E,k,alpha", [(64, 8, 2, 1.0), (300, 64, 8, 0.1), (5, 384, 8, 0.02), (10, 8, 8, 1.0)])
def test_random_routing_picks_k_distinct_experts(T, E, k, alpha):
    idx = wl.random_routing(T, E, k, alpha, seed=T).numpy()
    assert idx.shape == (T, k) and idx.dtype == np.int32
    assert idx.min() >= 0 and idx.max() < E
    assert all(len(set(row)) == k for row in idx)
    assert np.array_equal(idx, wl.random_routing(T, E, k, alpha, seed=T).numpy())


def test_histogram_stats_by_hand():
    r = stats.histogram_stats([2, 2, 0, 0])
    assert r == {"max_count": 2.0, "mean_count": 1.0, "empty_experts": 2, "active_experts": 2,
                 "effective_experts": pytest.approx(2.0)}
    assert stats.histogram_stats([5] * 7)["effective_experts"] == pytest.approx(7.0)
    assert stats.histogram_stats([0, 9, 0])["effective_experts"] == pytest.approx(1.0)
    assert stats.histogram_stats([0, 0])["effective_experts"] == 1.0
