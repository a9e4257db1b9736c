"""Pins of the E-PMQ oracle (the E-PMQ page, section 2) against facts that do not come from the oracle
itself: closed forms, the normal equations, the completed square, limits of the anchor strength,
the raw-activation form of the objective, and the reduction to plain GPTQ."""
import numpy as np
import pytest

import oracle as O
from oracle import epmq_oracle as EP


def _setup(K=3, d_out=16, d=128, n=400, seed=0, spread=0.3):
    """Source experts W_i = W_base + tau_i, merged W_m = W_base + mean(tau) (simple averaging), and
    per-expert activations X_i [n, d] with different covariances."""
    g = np.random.default_rng(seed)
    W_base = g.normal(0, 0.02, (d_out, d))
    taus = [g.normal(0, 0.02 * spread, (d_out, d)) for _ in range(K)]
    W_src = [W_base + t for t in taus]
    W_m = W_base + sum(taus) / K
    X = [g.normal(0, 1, (n, d)) * (0.5 + g.random(d)) for _ in range(K)]
    H = [x.T @ x for x in X]
    return W_src, H, W_m, X


def test_identical_experts_give_the_merged_weight():
    W_src, H, W_m, _ = _setup()
    W_same = [W_m.copy() for _ in W_src]
    Hs, R, lam = EP.statistics(W_same, H, W_m)
    np.testing.assert_allclose(EP.target(Hs, R), W_m, rtol=0, atol=1e-13)


def test_normal_equations_and_completed_square():
    W_src, H, W_m, _ = _setup()
    Hs, R, lam = EP.statistics(W_src, H, W_m)
    W_star = EP.target(Hs, R)
    assert np.linalg.norm(W_star @ Hs - R) <= 1e-12 * np.linalg.norm(R)
    g = np.random.default_rng(9)
    J_star = EP.objective(W_star, W_src, H, W_m, lam)
    for _ in range(3):
        Q = W_star + g.normal(0, 0.01, W_star.shape)
        D = Q - W_star
        quad = float(np.sum((D @ Hs) * D))
        J = EP.objective(Q, W_src, H, W_m, lam)
        assert abs((J - J_star) - quad) <= 1e-9 * quad
        assert J > J_star


def test_objective_equals_raw_activation_form():
    W_src, H, W_m, X = _setup(K=2, d=128, n=300, seed=3)
    Hs, R, lam = EP.statistics(W_src, H, W_m)
    Q = W_m + np.random.default_rng(4).normal(0, 0.005, W_m.shape)
    direct = sum(np.linalg.norm(Q @ x.T - W @ x.T) ** 2 for W, x in zip(W_src, X)) + lam * np.linalg.norm(Q - W_m) ** 2
    assert abs(EP.objective(Q, W_src, H, W_m, lam) - direct) <= 1e-10 * direct


def test_anchor_limits():
    W_src, H, W_m, _ = _setup(K=1, n=600, seed=5)
    # strong anchor: the target is the merged weight
    Hs, R, _ = EP.statistics(W_src, H, W_m, damp_frac=1e9)
    np.testing.assert_allclose(EP.target(Hs, R), W_m, rtol=0, atol=1e-9)
    # no anchor with one full-rank expert: the target is that expert's weight
    Hs, R, _ = EP.statistics(W_src, H, W_m, damp_frac=1e-14)
    np.testing.assert_allclose(EP.target(Hs, R), W_src[0], rtol=0, atol=1e-10)


def test_reduces_to_gptq_of_the_merged_weight():
    W_src, H, W_m, _ = _setup(seed=7)
    same = [W_m.copy() for _ in W_src]
    r = EP.epmq(same, H, W_m, bits=3, group=128)
    Hs = r["H"]
    codes, scales, zeros, W_hat = O.gptq(W_m, O.factor(Hs), 3, 128)
    np.testing.assert_array_equal(r["codes"], codes)
    np.testing.assert_array_equal(r["scales"], scales)


def test_lambda_is_the_damped_activation_energy():
    W_src, H, W_m, X = _setup(seed=8)
    _, _, lam = EP.statistics(W_src, H, W_m, damp_frac=0.01)
    energy = sum(np.sum(x * x) for x in X)   # sum of squared activations = tr(sum H_i)
    assert lam == pytest.approx(0.01 * energy / W_m.shape[1], rel=1e-12)


def test_expert_targets_beat_plain_gptq_of_the_merged_weight():
    """The page's point: on merged weights that drift from their experts, quantizing toward the
    expert-driven target lowers the E-PMQ objective compared with quantizing W_m itself."""
    W_src, H, W_m, _ = _setup(K=4, d_out=32, d=256, n=800, seed=11, spread=1.0)
    r = EP.epmq(W_src, H, W_m, bits=3, group=128)
    _, _, _, W_hat_naive = O.gptq(W_m, O.factor(r["H"]), 3, 128)
    naive = EP.objective(W_hat_naive.astype(np.float64), W_src, H, W_m, r["lam"])
    assert r["objective"] < naive
