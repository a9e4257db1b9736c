"""Pins of the float64 oracle against facts fixed outside it: hand-worked golden values, closed forms,
textbook special cases, brute force on tiny inputs and identities of the mathematics.

Each test is chosen so that a plausible slip in the oracle (a dropped factor 2, a wrong alpha, a sign
or index error in the error feedback, a transposed factor, a wrong rounding mode) fails it.
"""
import itertools
import os

import numpy as np
import pytest
import scipy.linalg
import scipy.special
import torch

import oracle as O

RNG = np.random.default_rng(20240611)


def _golden_lines(path):
    with open(path) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.startswith("#")]


def _spd(d, rank=None, seed=0, damp=0.5):
    r = np.random.default_rng(seed)
    A = r.standard_normal((d, rank or d))
    return A @ A.T / (rank or d) + damp * np.eye(d)


# ------------------------------------------------------------------------------------ routing
def test_route_matches_python_loop_and_counts():
    r = np.random.default_rng(1)
    n, E, k = 37, 9, 3
    lg = r.standard_normal((n, E)).astype(np.float32)
    lg[5, 2] = lg[5, 7] = lg[5].max() + 1.0          # a tie at the top
    lg[6, :] = 0.25                                   # all tied
    ids, counts = O.route_topk(lg, k)
    for t in range(n):
        remaining = list(range(E))
        want = []
        for _ in range(k):
            best = remaining[0]
            for e in remaining[1:]:
                if lg[t, e] > lg[t, best]:           # strict: the lower index keeps a tie
                    best = e
            want.append(best)
            remaining.remove(best)
        assert list(ids[t]) == want
    assert counts.sum() == n * k
    assert list(ids[5][:2]) == [2, 7]
    assert list(ids[6]) == [0, 1, 2]
    for e in range(E):
        assert counts[e] == sum(e in list(ids[t]) for t in range(n))


def test_expert_token_lists_ascending_and_complete():
    r = np.random.default_rng(2)
    ids, counts = O.route_topk(r.standard_normal((50, 6)), 2)
    lists = O.expert_tokens(ids, 6)
    for e, t in enumerate(lists):
        assert len(t) == counts[e]
        assert np.all(np.diff(t) > 0)
    assert sorted(np.concatenate(lists).tolist()) == sorted(np.repeat(np.arange(50), 2).tolist())


# ------------------------------------------------------------------------------------ collection
def test_gram_is_sum_of_outer_products():
    X = RNG.standard_normal((7, 5))
    S = np.zeros((5, 5))
    for t in range(7):
        for i in range(5):
            for j in range(5):
                S[i, j] += X[t, i] * X[t, j]
    np.testing.assert_allclose(O.gram(X), S, rtol=1e-13, atol=1e-13)
    assert np.all(np.linalg.eigvalsh(O.gram(X)) > -1e-12)
    np.testing.assert_allclose(O.hessian(S, 7), 2.0 / 7 * S, rtol=1e-15)


def test_layer_tagged_accumulators_do_not_mix():
    """Layer-aware collection (CLHA page §2.4): one accumulator per layer. A hook-style shared
    accumulator mixes layers and equals neither the first layer's Hessian nor the equal-weight one."""
    Xa = RNG.standard_normal((40, 6))
    Xb = 3.0 * RNG.standard_normal((24, 6)) + 1.0
    Sa = O.gram(Xa)
    mixed = O.gram(np.vstack([Xa, Xb]))
    Ha = O.hessian(Sa, 40)
    Hmix = O.hessian(mixed, 64)
    Heq = O.aggregate([Sa, O.gram(Xb)], [40, 24], "eq")["H_comb"]
    assert np.linalg.norm(Hmix - Ha) > 0.1 * np.linalg.norm(Ha)
    assert np.linalg.norm(Hmix - Heq) > 1e-3 * np.linalg.norm(Heq)


# ------------------------------------------------------------------------------------ aggregation
def test_alpha_golden(golden_dir):
    (line,) = _golden_lines(os.path.join(golden_dir, "alpha_routing_frequency.txt"))
    na, nb, aa, ab = line.split()
    S = [np.eye(3), np.eye(3)]
    agg = O.aggregate(S, [int(na), int(nb)], "rt")
    np.testing.assert_allclose(agg["alpha"], [float(aa), float(ab)], rtol=1e-15)
    np.testing.assert_allclose(agg["alpha"] * (int(na) + int(nb)), [int(na), int(nb)], rtol=1e-14)


def test_routing_frequency_aggregate_is_pooled_hessian():
    """Closed form: with alpha_i = n_i/N and H_i = (2/n_i) S_i, sum_i alpha_i H_i = (2/N) sum_all x x^T,
    the Hessian of the pooled tokens."""
    Xs = [RNG.standard_normal((n, 8)) * (1 + i) for i, n in enumerate((13, 29, 5))]
    agg = O.aggregate([O.gram(X) for X in Xs], [13, 29, 5], "rt")
    pooled = np.vstack(Xs)
    want = 2.0 / pooled.shape[0] * (pooled.T @ pooled)
    np.testing.assert_allclose(agg["H_comb"], want, rtol=1e-13)
    lam = 0.01 * np.trace(want) / 8
    np.testing.assert_allclose(agg["lam"], lam, rtol=1e-13)
    np.testing.assert_allclose(agg["H_d"] - agg["H_comb"], lam * np.eye(8), atol=1e-15)


def test_equal_weights_and_rt_agree_on_equal_counts():
    Xa, Xb = RNG.standard_normal((20, 4)), RNG.standard_normal((20, 4))
    S = [O.gram(Xa), O.gram(Xb)]
    rt = O.aggregate(S, [20, 20], "rt")
    eq = O.aggregate(S, [20, 20], "eq")
    np.testing.assert_array_equal(rt["alpha"], [0.5, 0.5])
    np.testing.assert_allclose(rt["H_comb"], eq["H_comb"], rtol=1e-15)
    np.testing.assert_allclose(eq["H_comb"], 0.5 * (2 / 20 * S[0]) + 0.5 * (2 / 20 * S[1]), rtol=1e-15)


def test_identical_layers_reduce_to_single_layer_calibration():
    """X_b = X_a: H_comb = H_a for every weighting, so CLHA gives PLIC's codes exactly."""
    X = RNG.standard_normal((300, 128))
    W = 0.02 * RNG.standard_normal((16, 128))
    res = {m: O.calibrate_dense(W, [X, X], 2, 64, m) for m in ("rt", "eq")}
    plic = O.calibrate_dense(W, [X, X], 2, 64, "explicit", alpha=[1.0, 0.0])
    for m in res:
        np.testing.assert_allclose(res[m]["H_comb"], plic["H_comb"], rtol=1e-14)
        np.testing.assert_array_equal(res[m]["codes"], plic["codes"])


def test_proposition_1_loss_identity():
    """CLHA page §2.1 Proposition 1: sum_i alpha_i tr[D H_i D^T] = tr[D H_comb D^T]
    = sum_i alpha_i (2/n_i) ||D X_i^T||_F^2 for any D (the direct form carries the 2 of H = (2/n) S)."""
    d = 16
    Xs = [RNG.standard_normal((n, d)) @ RNG.standard_normal((d, d)) for n in (50, 70)]
    n = [50, 70]
    S = [O.gram(X) for X in Xs]
    Dl = RNG.standard_normal((5, d))
    for mode in ("rt", "eq"):
        agg = O.aggregate(S, n, mode)
        a = agg["alpha"]
        per_layer = sum(ai * O.loss(np.zeros_like(Dl), Dl, O.hessian(Si, ni)) for ai, Si, ni in zip(a, S, n))
        combined = O.loss(np.zeros_like(Dl), Dl, agg["H_comb"])
        direct = sum(ai * 2.0 / ni * np.sum((Dl @ X.T) ** 2) for ai, X, ni in zip(a, Xs, n))
        np.testing.assert_allclose(per_layer, combined, rtol=1e-12)
        np.testing.assert_allclose(direct, combined, rtol=1e-12)


def test_aggregate_rejects_empty():
    with pytest.raises(ValueError):
        O.aggregate([np.eye(2), np.eye(2)], [0, 0], "rt")


def test_empty_aggregate_as_identity():
    """No tokens at all, or none in the only weighted layer: H_comb = 0, lambda = 1, H_d = I, and GPTQ
    under it gives the codes of GPTQ under any diagonal Hessian (round to nearest, pinned below)."""
    d = 8
    S = [np.zeros((d, d)), 3.0 * np.eye(d)]
    for n, mode, alpha in (([0, 0], "rt", None), ([0, 0], "eq", None), ([0, 5], "explicit", (1.0, 0.0))):
        agg = O.aggregate(S, n, mode, alpha, empty="identity")
        np.testing.assert_array_equal(agg["H_comb"], 0.0)
        assert agg["lam"] == 1.0
        np.testing.assert_array_equal(agg["H_d"], np.eye(d))
    W = 0.02 * RNG.standard_normal((4, 128))
    S128 = [np.zeros((128, 128)), 3.0 * np.eye(128)]
    U = O.factor(O.aggregate(S128, [0, 5], "explicit", (1.0, 0.0), empty="identity")["H_d"])
    c_id = O.gptq(W, U, 3, 128)[0]
    c_diag = O.gptq(W, O.factor(np.diag(RNG.uniform(0.5, 2.0, 128))), 3, 128)[0]
    np.testing.assert_array_equal(c_id, c_diag)
    # with energy the policy changes nothing
    S2 = [_spd(d, seed=5), _spd(d, seed=6)]
    a, b = O.aggregate(S2, [7, 9], "rt"), O.aggregate(S2, [7, 9], "rt", empty="identity")
    np.testing.assert_array_equal(a["H_d"], b["H_d"])
    assert a["lam"] == b["lam"]


# ------------------------------------------------------------------------------------ factor
@pytest.mark.parametrize("d", [1, 5, 64])
def test_factor_inverse_cholesky(d):
    H = _spd(d, seed=d)
    U = O.factor(H)
    assert np.allclose(np.tril(U, -1), 0)
    assert np.all(np.diag(U) > 0)
    np.testing.assert_allclose(U.T @ U @ H, np.eye(d), atol=1e-10)
    np.testing.assert_allclose(U, scipy.linalg.cholesky(scipy.linalg.inv(H), lower=False), rtol=1e-9, atol=1e-12)
    # U is the inverse of the "reverse" (upper) Cholesky factor R of H = R R^T
    J = np.eye(d)[::-1]
    R = J @ np.linalg.cholesky(J @ H @ J) @ J
    assert np.allclose(np.tril(R, -1), 0)
    np.testing.assert_allclose(U, np.linalg.inv(R), rtol=1e-9, atol=1e-12)


@pytest.mark.parametrize("d,block", [(64, 16), (96, 32), (130, 64), (128, 128)])
def test_factor_block_scaled_gives_the_obs_lazy_update(d, block):
    """F against the textbook OBS recurrence, which holds no factor at all: quantize column j (any
    rounding rule will do), then move the remaining columns by -(w_j - w_hat_j) / [H_F^-1]_00 times the
    first row of H_F^-1, F the columns not yet quantized. At the start of every block the recurrence's
    current values equal W_b + (W - W_hat)_a F_ab, the earlier columns a < b entering only through
    F; inside a block F is U. A transposed F, a wrong sign, a block of R left unscaled or a diagonal
    block of R instead of U fails it."""
    H = _spd(d, rank=d // 2, seed=d + 7, damp=0.05)
    W = 0.02 * RNG.standard_normal((5, d))
    F = O.factor_block_scaled(H, block)
    assert np.allclose(np.tril(F, -1), 0)
    cur, W_hat = np.zeros_like(W), np.zeros_like(W)
    for r in range(W.shape[0]):
        w = W[r].copy()
        for j in range(d):
            if j % block == 0:
                cur[r, j:j + block] = w[j:j + block]
            W_hat[r, j] = np.round(w[j] * 64) / 64
            rest = np.arange(j, d)
            Hinv = np.linalg.inv(H[np.ix_(rest, rest)])
            w[j:] -= (w[j] - W_hat[r, j]) / Hinv[0, 0] * Hinv[0, :]
    D = W - W_hat
    U = O.factor(H)
    for b0 in range(0, d, block):
        b1 = min(d, b0 + block)
        np.testing.assert_allclose(W[:, b0:b1] + D[:, :b0] @ F[:b0, b0:b1], cur[:, b0:b1], rtol=0, atol=1e-12)
        np.testing.assert_allclose(F[b0:b1, b0:b1], U[b0:b1, b0:b1], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(O.factor_block_scaled(H, d), U, rtol=1e-9, atol=1e-12)   # one block: F = U


# ------------------------------------------------------------------------------------ grid + GPTQ
def test_grid_golden(golden_dir):
    for line in _golden_lines(os.path.join(golden_dir, "grid_minmax_examples.txt")):
        _, bits, w, s, z, q, wq = [f.strip() for f in line.split("|")]
        bits = int(bits)
        w = np.array([float(v) for v in w.split()])[None, :]
        gs, gz = O.grid_fp32(w, bits)
        assert gs[0] == np.float32(float(s)) and gz[0] == np.float32(float(z))
        gq, gwq = O.quantize_fp32(w[0], gs, gz, bits)
        np.testing.assert_array_equal(gq, [float(v) for v in q.split()])
        np.testing.assert_array_equal(gwq, np.array([float(v) for v in wq.split()], np.float32))


def test_grid_all_zero_group_maps_to_zero():
    s, z = O.grid_fp32(np.zeros((1, 8)), 2)
    q, wq = O.quantize_fp32(np.zeros(8), s, z, 2)
    np.testing.assert_array_equal(wq, 0.0)
    np.testing.assert_array_equal(q, z[0])


def test_gptq_diagonal_hessian_is_round_to_nearest():
    """H diagonal => U diagonal => no error feedback: GPTQ is per-group round-to-nearest exactly."""
    W = 0.02 * RNG.standard_normal((12, 256))
    H = np.diag(RNG.uniform(0.5, 2.0, 256))
    for bits in (2, 3, 4):
        codes, scales, zeros, W_hat = O.gptq(W, O.factor(H), bits, 128)
        for g in range(2):
            blk = W[:, g * 128:(g + 1) * 128]
            xmin = np.minimum(0, blk.astype(np.float32).min(1))
            xmax = np.maximum(0, blk.astype(np.float32).max(1))
            np.testing.assert_array_equal(scales[:, g], ((xmax - xmin) / np.float32(2 ** bits - 1)).astype(np.float32))
            q = np.clip(np.rint(blk.astype(np.float32) / scales[:, g:g + 1]) + zeros[:, g:g + 1], 0, 2 ** bits - 1)
            np.testing.assert_array_equal(codes[:, g * 128:(g + 1) * 128], q)


def _obs_gptq(W, H, bits, group):
    """Optimal-brain-surgeon form (explicit inverse of the remaining columns after each step)."""
    W = np.array(W, dtype=np.float64)
    d_out, d_in = W.shape
    codes = np.zeros((d_out, d_in), np.uint8)
    W_hat = np.zeros((d_out, d_in), np.float32)
    for r in range(d_out):
        w = W[r].copy()
        for j in range(d_in):
            if j % group == 0:
                s, z = O.grid_fp32(w[None, j:j + group], bits)
            q, wq = O.quantize_fp32(w[j:j + 1], s, z, bits)
            codes[r, j], W_hat[r, j] = q[0], wq[0]
            F = np.arange(j, d_in)
            Finv = np.linalg.inv(H[np.ix_(F, F)])
            w[j:] -= (w[j] - np.float64(wq[0])) / Finv[0, 0] * Finv[0, :]
    return codes, W_hat


@pytest.mark.parametrize("d,group,bits", [(16, 8, 2), (64, 32, 3), (48, 16, 4)])
def test_gptq_equals_obs_form(d, group, bits):
    H = _spd(d, rank=d // 2, seed=d, damp=0.05)
    W = 0.02 * RNG.standard_normal((6, d))
    codes, _, _, W_hat = O.gptq(W, O.factor(H), bits, group)
    c2, w2 = _obs_gptq(W, H, bits, group)
    np.testing.assert_array_equal(codes, c2)
    np.testing.assert_allclose(W_hat, w2, rtol=0, atol=0)


def test_gptq_two_columns_closed_form():
    """d = 2: after rounding column 0 the best continuous value of column 1 is w1 + (w0 - q0) H01/H11
    (minimise the 2x2 quadratic over w1 with q0 fixed)."""
    H = np.array([[2.0, 0.7], [0.7, 1.5]])
    W = np.array([[0.3, -0.2], [0.11, 0.05], [-0.4, 0.6]])
    _, _, _, W_hat = O.gptq(W, O.factor(H), 4, 2)
    s, z = O.grid_fp32(W, 4)
    q0, wq0 = O.quantize_fp32(W[:, 0], s, z, 4)
    w1 = W[:, 1] + (W[:, 0] - wq0.astype(np.float64)) * H[0, 1] / H[1, 1]
    _, wq1 = O.quantize_fp32(w1, s, z, 4)
    np.testing.assert_array_equal(W_hat[:, 0], wq0)
    np.testing.assert_array_equal(W_hat[:, 1], wq1)


@pytest.mark.parametrize("block", [1, 8, 32, 128])
def test_gptq_blocking_does_not_change_codes(block):
    d = 256
    H = _spd(d, rank=64, seed=3, damp=0.02)
    U = O.factor(H)
    W = 0.02 * RNG.standard_normal((8, d))
    codes, scales, zeros, W_hat = O.gptq(W, U, 3, 128)
    cb, sb, zb, wb, mb = O.gptq(W, U, 3, 128, block=block, margins=True)
    np.testing.assert_array_equal(cb, codes)
    np.testing.assert_array_equal(sb, scales)
    np.testing.assert_array_equal(zb, zeros)
    np.testing.assert_array_equal(wb, W_hat)
    assert mb["code"].shape == codes.shape and np.all((mb["code"] >= 0) & (mb["code"] <= 0.5))


def test_gptq_margins_are_distances_to_the_rounding_boundary():
    """With H = I (round to nearest) the code margin of w is |(|w/s - rint(w/s)|) - 1/2|, worked by
    hand on values placed at known offsets from the grid: a value on a grid point has margin 1/2, one
    a quarter step past a boundary has margin 1/4; the zero point's margin is that of -xmin/s."""
    # one row, one group of 128: xmin = -0.3 and xmax = 0.4 fix s = 0.7/7 = 0.1 (3 bits) and z = 3
    w = np.zeros(128)
    w[0], w[1] = -0.3, 0.4
    w[2] = 0.15 + 0.025          # a quarter step past the boundary 1.5 s: code 3 + 2 = 5
    w[3] = 0.2                   # on the grid point 2 s: code 5
    w[4] = -0.05 - 0.0125        # an eighth of a step past the boundary -0.5 s: code 3 - 1 = 2
    codes, scales, zeros, _, m = O.gptq(w[None], np.eye(128), 3, 128, margins=True)
    assert scales[0, 0] == np.float32(np.float32(np.float32(0.4) - np.float32(-0.3)) / np.float32(7)) and zeros[0, 0] == 3
    np.testing.assert_allclose(m["code"][0, :5], [0.5, 0.5, 0.25, 0.5, 0.125], atol=1e-5)
    assert list(codes[0, :5]) == [0, 7, 5, 5, 2]
    np.testing.assert_allclose(m["zero"][0, 0], 0.5, atol=1e-5)     # -xmin/s = 3
    np.testing.assert_allclose(O.boundary_distance([0.5, 1.0, 2.25, -0.75]), [0.0, 0.5, 0.25, 0.25])


def test_brute_force_lower_bounds_gptq():
    """4x8 weight, one group: every code vector on the same grid is a candidate, so the exhaustive
    minimum of the loss is at most GPTQ's; GPTQ must also beat plain rounding here on average."""
    H = _spd(8, rank=3, seed=11, damp=0.01)
    W = 0.02 * RNG.standard_normal((4, 8))
    bits = 2
    U = O.factor(H)
    codes, scales, zeros, W_hat = O.gptq(W, U, bits, 8)
    grid = np.array(list(itertools.product(range(4), repeat=8)), dtype=np.float64)   # 65536 x 8
    rtn_total = gptq_total = best_total = 0.0
    for r in range(4):
        vals = scales[r, 0] * (grid - zeros[r, 0])
        D = vals - W[r]
        losses = np.einsum("ij,jk,ik->i", D, H, D)
        g_loss = O.loss(W[r:r + 1], W_hat[r:r + 1], H)
        assert losses.min() <= g_loss * (1 + 1e-12)
        assert losses.min() >= 0
        q_rtn, wq_rtn = O.quantize_fp32(W[r], scales[r:r + 1, 0], zeros[r:r + 1, 0].astype(np.float32), bits)
        rtn_total += O.loss(W[r:r + 1], wq_rtn[None, :], H)
        gptq_total += g_loss
        best_total += losses.min()
    assert best_total <= gptq_total <= rtn_total


def test_gptq_codes_scale_invariant():
    d = 128
    H = _spd(d, rank=20, seed=5, damp=0.01)
    W = 0.02 * RNG.standard_normal((4, d))
    agg1 = O.aggregate([H], [2], "rt")
    agg4 = O.aggregate([4.0 * H], [2], "rt")
    c1, *_ = O.gptq(W, O.factor(agg1["H_d"]), 3, 64)
    c4, *_ = O.gptq(W, O.factor(agg4["H_d"]), 3, 64)
    np.testing.assert_array_equal(c1, c4)


def test_gptq_beats_rtn_on_correlated_inputs():
    """With strongly correlated inputs the error feedback must lower tr[D H D^T] well below plain
    rounding on the same grids (a sign or index slip in the feedback makes it worse, not better)."""
    d = 256
    X = RNG.standard_normal((2000, 16)) @ RNG.standard_normal((16, d)) + 0.3 * RNG.standard_normal((2000, d))
    H = O.aggregate([O.gram(X)], [2000], "rt")
    W = 0.02 * RNG.standard_normal((32, d))
    codes, scales, zeros, W_hat = O.gptq(W, O.factor(H["H_d"]), 3, 128)
    Hd = O.hessian(O.gram(X), 2000)
    rtn = np.zeros_like(W_hat)
    for g in range(2):
        blk = W[:, g * 128:(g + 1) * 128]
        s, z = O.grid_fp32(blk, 3)
        _, rtn[:, g * 128:(g + 1) * 128] = O.quantize_fp32(blk, s[:, None], z[:, None], 3)
    assert O.loss(W, W_hat, Hd) < 0.7 * O.loss(W, rtn, Hd)


# ------------------------------------------------------------------------------------ FFN act
def test_bf16_round_golden_and_library(golden_dir):
    for line in _golden_lines(os.path.join(golden_dir, "bf16_rounding.txt")):
        x, y = (float(v) for v in line.split())
        assert O.bf16_round(np.array([x]))[0] == y
        assert O.bf16_round(np.array([-x]))[0] == -y
    v = (RNG.standard_normal(100000) * np.exp(RNG.uniform(-20, 20, 100000))).astype(np.float32)
    lib = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    np.testing.assert_array_equal(O.bf16_round(v.astype(np.float64)), lib)


def test_silu_and_ffn_act():
    a = np.linspace(-60, 60, 1001)
    np.testing.assert_allclose(O.silu(a), a * scipy.special.expit(a), rtol=1e-14, atol=1e-300)
    X = RNG.standard_normal((5, 16))
    Wg, Wu = RNG.standard_normal((3, 16)), RNG.standard_normal((3, 16))
    h = O.ffn_act(X, Wg, Wu)
    for t in range(5):
        for f in range(3):
            g = sum(X[t, i] * Wg[f, i] for i in range(16))
            u = sum(X[t, i] * Wu[f, i] for i in range(16))
            want = g / (1 + np.exp(-g)) * u
            assert abs(h[t, f] - want) <= 2.0 ** -8 * abs(want) + 1e-300
            assert O.bf16_round(np.array([h[t, f]]))[0] == h[t, f]


# ------------------------------------------------------------------------------ deployable codes
def _golden_packed(golden_dir):
    rows = []
    with open(f"{golden_dir}/packed_codes_examples.txt") as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            b, codes, words = [p.strip() for p in line.split("|")]
            rows.append((int(b), [int(c) for c in codes.split(",")], [int(w, 16) for w in words.split(",")]))
    return rows


def test_pack_codes_matches_hand_worked_words(golden_dir):
    cases = _golden_packed(golden_dir)
    assert len(cases) == 4
    for bits, codes, words in cases:
        got = O.pack_codes(np.array([codes], np.uint8), bits)
        assert got.tolist() == [words], (bits, [hex(w) for w in got[0]])
        np.testing.assert_array_equal(O.unpack_codes(got, bits, len(codes))[0], codes)


@pytest.mark.parametrize("bits", [2, 3, 4, 5, 6, 7, 8])
def test_pack_roundtrip(bits):
    g = np.random.default_rng(bits)
    codes = g.integers(0, 2 ** bits, size=(5, 256), dtype=np.uint8)
    packed = O.pack_codes(codes, bits)
    assert packed.shape == (5, 256 * bits // 32)
    np.testing.assert_array_equal(O.unpack_codes(packed, bits, 256), codes)


def test_dequantized_codes_are_gptq_w_hat_and_the_layer_output():
    g = np.random.default_rng(3)
    W = g.normal(0, 0.02, (8, 256))
    A = g.normal(0, 1, (256, 300))
    H = A @ A.T / 300 + 0.01 * np.eye(256)
    codes, scales, zeros, W_hat = O.gptq(W, O.factor(H), 3, 128)
    np.testing.assert_array_equal(O.dequantize(codes, scales, zeros, 128), W_hat)
    X = g.normal(0, 1, (7, 256))
    packed = O.pack_codes(codes, 3)
    np.testing.assert_allclose(O.dequant_matmul(X, packed, scales, zeros, 3, 128), X @ W_hat.astype(np.float64).T,
                               rtol=1e-15, atol=1e-15)


def test_bf16_margin_hand_worked():
    """bfloat16 has 8 significant bits: in [1, 2) the step is 2^-7. 1 is on the grid (margin 1/2),
    1 + 2^-8 is a midpoint (0), 1 + 3 * 2^-10 lies 3/8 of a step above 1, 1/8 below the midpoint 1 + 2^-8
    (margin 1/8); in [4, 8) the step is 2^-5, so 4 + 2^-7 is a quarter step past 4 (margin 1/4)."""
    got = O.bf16_margin([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -10, 4.0 + 2 ** -7, -(1.0 + 2 ** -8)])
    np.testing.assert_allclose(got, [0.5, 0.0, 0.125, 0.25, 0.0], atol=1e-12)
    # a value rounds to its neighbour exactly when the margin sign flips: nudging a midpoint
    v = 1.0 + 2 ** -8
    assert O.bf16_round(v - 1e-9) == 1.0 and O.bf16_round(v + 1e-9) == 1.0 + 2 ** -7
