"""Pins of the oracle's cross-layer routing divergence and held-out Hessian error, and of the input
generator's routing-sharpness knob and held-out split (CPU only).

The divergence is the total-variation distance of two layers' expert frequencies (the CLHA page,
sections 4-5, relates CLHA's gains to cross-layer routing divergence without defining it); it is
checked against its characterisation as the largest difference in probability that the two
frequency vectors give to any set of experts, which shares no arithmetic with the half-L1 sum.
"""
import itertools

import numpy as np
import pytest
import torch

from oracle import clha_oracle as O
from synth import workload


def test_worked_examples():
    # (3,1,0,0)/4 vs (1,1,1,1)/4: |0.75-0.25| + 0 + 0.25 + 0.25 = 1.0, halved: 0.5
    # (2,2)/4 vs (1,3)/4: 0.25 + 0.25 = 0.5, halved: 0.25
    # (3,1,0,0)/4 vs (2,2,0,0)/4: 0.25 + 0.25, halved: 0.25
    tv = O.routing_divergence([[3, 1, 0, 0], [1, 1, 1, 1], [2, 2, 0, 0]])
    assert tv[0, 1] == 0.5 and tv[0, 2] == 0.25 and tv[1, 2] == 0.5
    assert O.routing_divergence([[2, 2], [1, 3]])[0, 1] == 0.25


def test_largest_set_probability_difference():
    """TV(p, q) = max over expert sets A of |p(A) - q(A)|, by enumerating every set."""
    rng = np.random.default_rng(7)
    for E in (1, 2, 5, 9):
        c = rng.integers(0, 40, size=(3, E))
        c[:, 0] += 1
        tv = O.routing_divergence(c)
        p = c / c.sum(1, keepdims=True)
        for a, b in itertools.combinations(range(3), 2):
            best = 0.0
            for r in range(E + 1):
                for A in itertools.combinations(range(E), r):
                    idx = list(A)
                    best = max(best, abs(p[a, idx].sum() - p[b, idx].sum()))
            assert abs(tv[a, b] - best) < 1e-14


def test_metric_properties():
    rng = np.random.default_rng(11)
    c = rng.integers(0, 1000, size=(6, 17))
    c[:, 3] += 1
    tv = O.routing_divergence(c)
    assert np.all(np.diag(tv) == 0) and np.array_equal(tv, tv.T)
    assert np.all((tv >= 0) & (tv <= 1))
    for a, b, m in itertools.permutations(range(6), 3):
        assert tv[a, b] <= tv[a, m] + tv[m, b] + 1e-15
    # frequencies, not counts: scaling one layer's counts changes nothing
    c2 = c.copy()
    c2[2] *= 7
    assert np.array_equal(O.routing_divergence(c2), tv)
    # relabelling the experts of every layer alike changes nothing
    perm = rng.permutation(17)
    assert np.array_equal(O.routing_divergence(c[:, perm]), tv)
    # disjoint supports: 1
    assert O.routing_divergence([[5, 0, 3, 0], [0, 2, 0, 9]])[0, 1] == 1.0


def test_layer_without_tokens_is_rejected():
    with pytest.raises(ValueError):
        O.routing_divergence([[1, 2], [0, 0]])


def test_hessian_error_direct_forms():
    """Under the rt aggregate the error is (2 / sum n) sum over the pooled tokens of |(W_hat - W) x|^2;
    with alpha = (1, 0) it is the hook layer's own (2 / n_a) |(W_hat - W) X_a^T|^2 (the CLHA page
    §2.1 Proposition 1 written per token)."""
    rng = np.random.default_rng(3)
    d_out, d = 5, 12
    W = rng.standard_normal((d_out, d))
    W_hat = W + 0.1 * rng.standard_normal((d_out, d))
    Xa, Xb = rng.standard_normal((30, d)), 2.0 * rng.standard_normal((17, d))
    S, n = [O.gram(Xa), O.gram(Xb)], [30, 17]
    D = W_hat - W
    pooled = sum(float(np.dot(D @ x, D @ x)) for x in np.vstack([Xa, Xb]))
    assert abs(O.hessian_error(W, W_hat, S, n, "rt") - 2.0 / 47 * pooled) < 1e-10 * pooled
    hook = sum(float(np.dot(D @ x, D @ x)) for x in Xa)
    got = O.hessian_error(W, W_hat, S, n, "explicit", (1.0, 0.0))
    assert abs(got - 2.0 / 30 * hook) < 1e-10 * hook


def _tv_of_sharpened_routing(beta, tokens=4096):
    w = workload(2, tokens=tokens, sharpness=beta)
    counts = [np.bincount(O.route_topk(w.logits(l).numpy(), 2)[0].ravel(), minlength=16) for l in range(2)]
    return O.routing_divergence(np.stack(counts))[0, 1]


def test_sharpness_drives_layers_apart():
    tvs = [_tv_of_sharpened_routing(b) for b in (0.0, 0.25, 0.5)]
    assert tvs[0] < 0.05                      # same law in both layers: only sampling noise
    assert tvs[0] < tvs[1] < tvs[2]


def test_held_out_split_is_fresh_tokens_of_the_same_model():
    cal, test = workload(2, tokens=512), workload(2, tokens=512, split="test")
    assert not torch.equal(cal.x(0), test.x(0)) and not torch.equal(cal.logits(1), test.logits(1))
    for a, b in zip(cal.expert_weights(0, 4), test.expert_weights(0, 4)):
        assert torch.equal(a, b)
    sqd_c, us_c, _ = cal._cov_model(0, 1024)
    sqd_t, us_t, _ = test._cov_model(0, 1024)
    assert torch.equal(sqd_c, sqd_t) and all(torch.equal(a, b) for a, b in zip(us_c, us_t))
    # the knob leaves the calibration tokens themselves untouched
    assert torch.equal(workload(2, tokens=512, sharpness=0.5).x(0), cal.x(0))
