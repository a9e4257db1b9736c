"""Full-size parity on the large workloads, where the float64 oracle cannot redo everything:

* the 12-pair stack (24 layers, E16 top-2 + 2 always-active experts, 131072 tokens per layer): the GPU
  calibrates every pair with both weightings; the oracle checks every layer's routing counts and, on
  one pair of every drift class (0, 0.3, 0.6, 1.0), the least- and the most-routed routed expert and
  both always-active (3-bit) experts end to end: Hessians, codes, loss;
* the E64 top-6 pair with two always-active experts at 32768 tokens per layer: routing of both
  layers; the 8 least-routed and the 8 most-routed routed experts (most of the former see fewer
  tokens than d_model, so their Hessians are rank-deficient up to the damping) and both
  always-active experts end to end;
* the dense stress shape (W 8192 x 28672 bf16 shared by 4 layers of 65536 tokens, 4-bit): the oracle
  checks a random 512-channel principal block of every layer's Gram matrix and of the aggregate;
  the factor's trailing 2048 x 2048 block against the oracle's factor of the damped aggregate's
  trailing block (with H_d = R R^T, R upper, U = R^-1 has the block R22^-1, and R22 R22^T is the
  trailing block of H_d: that block of U depends on nothing else), plus U^T U H_d = I on sampled
  vectors; GPTQ stage-wise: the oracle's GPTQ of 16 sampled rows under the GPU's factor (checked as
  above) against the GPU's codes; the in-kernel loss equals the trace computed directly.
Codes: at least 99.9 % equal, and every row that differs starts with a certified rounding-boundary
flip (helpers.certify_codes).
"""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import (CONFIG_BAR, H_INPUT_BAR, MATRIX_BAR, CodeTally, assert_codes, certify_h, check_loss,
                     rel_fro, sym_from_upper, to64)
from post_quantization_expert_b200.clha import FACTOR_BLOCK_CHOL
from post_quantization_expert_b200.pipeline import DenseCalibration, MoECalibration, stack_weights
from synth import workload

pytestmark = [pytest.mark.gpu, pytest.mark.slow]
DEV = "cuda:0"


def _check_experts(ref, out, S_accs, E, what, tally, weights, h_gpu=None):
    """Hessians, certified codes and losses of every expert in an oracle result against the GPU's.
    S_accs: (S_in, S_dn, S_sdn) accumulator buffers; the always-active experts share input slot E.
    weights: (kind, e) -> (Wg, Wu, Wd) as float64 arrays, for the loss bar (check_loss).
    A down-projection Hessian more than 1e-4 from the oracle's is accepted only when h_gpu (the GPU's
    h of that routed expert and layer) shows why: its Gram equals the GPU's Hessian to 1e-4, every h
    element that differs from the oracle's is one bf16 step away and at most 0.1 % differ, and the
    difference stays under 1e-3 (a sparse expert, where one such difference on a large h moves the
    Gram by ~1e-4). The codes of such a down projection are held to H_INPUT_BAR."""
    S_in, S_dn, S_sdn = S_accs
    for (kind, e), r in ref["experts"].items():
        h_moved = False
        for j in range(len(r["n"])):
            s_in = S_in[j, e] if kind == "r" else S_in[j, E]
            s_dn = S_dn[j, e] if kind == "r" else S_sdn[j, e]
            assert rel_fro(sym_from_upper(s_in.double().cpu().numpy()), r["H_in"]["S"][j]) < 1e-4, (what, kind, e, j)
            got_dn = sym_from_upper(s_dn.double().cpu().numpy())
            rel_dn = rel_fro(got_dn, r["H_down"]["S"][j])
            if rel_dn >= 1e-4:
                assert h_gpu is not None and (kind, e, j) in h_gpu, (what, kind, e, j, rel_dn)
                hg = h_gpu[(kind, e, j)]
                assert rel_fro(got_dn, O.gram(hg)) < 1e-4, (what, kind, e, j)
                frac, worst = certify_h(hg, r["h"][j], r["h_margin"][j], (what, kind, e, j))
                assert rel_dn < 1e-3, (what, kind, e, j, rel_dn)
                h_moved = True
                print("H_down", what, kind, e, j, f"{rel_dn:.3g} from one-step h differences "
                      f"({frac:.2e} of h, largest rounding margin {worst:.3g})")
        qs = ({"gate": out.qg, "up": out.qu, "down": out.qd} if kind == "r" else
              {"gate": out.sg, "up": out.su, "down": out.sd})
        for wi, (name, q) in enumerate(qs.items()):
            bar = H_INPUT_BAR if name == "down" and h_moved else MATRIX_BAR
            codes, zeros = q.codes[e].cpu().numpy(), q.zeros[e].cpu().numpy()
            tally.add(codes, zeros, r[name], (what, kind, e, name, r["n"]), bar)
            H = r["H_down" if name == "down" else "H_in"]["H_comb"]
            check_loss(q.loss[e], weights[(kind, e)][wi], to64(q.W_hat[e]), codes, zeros, r[name], H,
                       (what, kind, e, name))


def test_stack_of_12_pairs_full_size(ctx):
    wl = workload(4, DEV)
    s = wl.spec
    checked_pairs = {}                       # first pair of each drift class
    for gi, dr in enumerate(s.drifts):
        checked_pairs.setdefault(dr, gi)
    checked_pairs = sorted(checked_pairs.values())
    assert len(checked_pairs) == 4
    tally = CodeTally("stack")
    for gi, (la, lb) in enumerate(s.group_of_layers):
        routed = [wl.expert_weights(gi, e) for e in range(s.E)]
        shared = [wl.expert_weights(gi, i, shared=True) for i in range(s.n_shared)]
        w = stack_weights((routed, shared), DEV)
        cal = MoECalibration(ctx, 2, s.tokens[la], s.E, s.k, s.d_model, s.d_ff, s.n_shared, s.shared_dff,
                             s.bits_routed, s.bits_shared, s.damp_frac, modes=s.alpha_modes)
        lgs = [wl.logits(la), wl.logits(lb)]
        for j, layer in enumerate((la, lb)):
            cal.collect(j, wl.x(layer, cache=False), lgs[j], w)
        cal.quantize(w, s.alpha_modes)
        torch.cuda.synchronize()
        routes = [O.route_topk(lg.cpu().numpy(), s.k) for lg in lgs]
        for j in range(2):
            np.testing.assert_array_equal(cal.counts[j].cpu().numpy(), routes[j][1])
        for r in cal.res.values():
            assert np.all(np.isfinite(r.expert_loss())) and np.all(r.expert_loss() > 0)
        if gi not in checked_pairs:
            continue
        total = routes[0][1] + routes[1][1]
        experts = sorted({int(np.argmin(total)), int(np.argmax(total))})
        X64 = [to64(wl.x(la, cache=False)), to64(wl.x(lb, cache=False))]
        S_accs = (cal.acc_in.buffers()[0], cal.acc_dn.buffers()[0], cal.acc_sdn.buffers()[0])
        for mode in s.alpha_modes:
            ref = O.calibrate_moe_group(X64, [lg.cpu().numpy() for lg in lgs], s.k,
                                        [tuple(to64(t) for t in r) if e in experts else None
                                         for e, r in enumerate(routed)],
                                        [tuple(to64(t) for t in sh) for sh in shared], experts,
                                        s.bits_routed, s.bits_shared, s.group, mode, s.damp_frac)
            wts = {("r", e): tuple(to64(t) for t in routed[e]) for e in experts}
            wts.update({("s", i): tuple(to64(t) for t in sh) for i, sh in enumerate(shared)})
            _check_experts(ref, cal.res[mode], S_accs, s.E, (gi, s.drifts[gi], mode), tally, wts)
        del cal, w
        torch.cuda.empty_cache()
    tally.check()


def test_moe_E64_top6_shared_full_size(ctx):
    """The E64 top-6 shape at full size (32768 tokens per layer, two always-active experts with one
    more bit, Zipf-skewed routing, x20 outlier channels): routing counts of both layers bit-exact;
    the 8 least-routed and the 8 most-routed routed experts and both always-active experts end to end
    against the oracle (Hessians, codes with flip certification, loss). Many of the least-routed
    experts see fewer tokens than d_model in a layer: their Hessians are rank-deficient up to the
    damping, the hardest case for the code bar, and their down-projection Hessians are sums of ~70
    outer products, where a single certified bf16 rounding flip of h counts. The activation runs on
    the tensor cores with the x20 channels taken out of the tensor-core sums."""
    from post_quantization_expert_b200 import clha as L
    wl = workload(3, "cpu")
    s = wl.spec
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    shared = [wl.expert_weights(0, i, shared=True) for i in range(s.n_shared)]
    w = stack_weights((routed, shared), DEV)
    cal = MoECalibration(ctx, 2, max(s.tokens), s.E, s.k, s.d_model, s.d_ff, s.n_shared, s.shared_dff,
                         s.bits_routed, s.bits_shared, s.damp_frac, modes=("rt",))
    Xs = [wl.x(l) for l in range(2)]
    lgs = [wl.logits(l) for l in range(2)]
    routes = [O.route_topk(lg.numpy(), s.k) for lg in lgs]
    total = routes[0][1] + routes[1][1]
    order = [int(e) for e in np.argsort(total, kind="stable")]
    checked = sorted(set(order[:8] + order[-8:]))
    h_gpu = {}
    for l in range(2):
        cal.collect(l, Xs[l].to(DEV), lgs[l].to(DEV), w)
        assert L.clha_last_act_kernel(ctx) == L.ACT_TENSOR     # outlier channels taken out of the sums
        seg = cal.seg[l].cpu().numpy()
        for e in checked:                                      # this layer's h of the checked experts
            h_gpu[("r", e, l)] = cal.hp[seg[e]:seg[e] + routes[l][1][e]].double().cpu().numpy()
    cal.quantize(w, ("rt",))
    torch.cuda.synchronize()
    for l in range(2):
        np.testing.assert_array_equal(cal.counts[l].cpu().numpy(), routes[l][1])
    least = np.minimum(routes[0][1], routes[1][1])
    assert (least[order[:8]] < s.d_model).sum() >= 4          # rank-deficient per-layer Hessians included
    X64 = [to64(X) for X in Xs]
    routed64 = [tuple(to64(t) for t in routed[e]) if e in checked else None for e in range(s.E)]
    ref = O.calibrate_moe_group(X64, [lg.numpy() for lg in lgs], s.k, routed64,
                                [tuple(to64(t) for t in sh) for sh in shared], checked, s.bits_routed,
                                s.bits_shared, s.group, "rt", s.damp_frac)
    assert len(ref["experts"]) == 16 + s.n_shared
    S_accs = (cal.acc_in.buffers()[0], cal.acc_dn.buffers()[0], cal.acc_sdn.buffers()[0])
    tally = CodeTally("E64")
    wts = {("r", e): routed64[e] for e in checked}
    wts.update({("s", i): tuple(to64(t) for t in sh) for i, sh in enumerate(shared)})
    _check_experts(ref, cal.res["rt"], S_accs, s.E, "E64", tally, wts, h_gpu)
    tally.check()


def _gptq_consistency(W, W_hat, codes, scales, zeros, U, rows, bits):
    """Codes, grids and W_hat of sampled rows follow the GPTQ recurrence with this U: the errors
    E = (W - W_hat) U^-1 give each column's current value w_j = W_hat_j + E_j U_jj and each group's
    current values at its start; the float32 grid of those values and the rounding of w_j must
    reproduce the kernel's grid (scales to 1e-4 relative) and codes (boundary cases excepted)."""
    maxq = np.float32(2 ** bits - 1)
    d_in = W.shape[1]
    agree = total = grid_ok = groups = 0
    for r in rows:
        Wr = W[r].double()
        D = (Wr - W_hat[r].double())[None, :]
        E = torch.linalg.solve_triangular(U, D, upper=True, left=False)[0]           # D = E U
        cur = (W_hat[r].double() + E * torch.diagonal(U)).cpu().numpy()
        for g in range(d_in // 128):
            c0 = 128 * g
            start = (Wr[c0:c0 + 128] - E[:c0] @ U[:c0, c0:c0 + 128]).cpu().numpy().astype(np.float32)
            xmin = min(np.float32(0), start.min())
            xmax = max(np.float32(0), start.max())
            sg = np.float32(np.float32(xmax - xmin) / maxq)
            zg = np.float32(np.rint(np.float32(-xmin) / sg))
            groups += 1
            # the start values here come from a float64 solve, the kernel's from its own float32
            # accumulation of the same sums: scales agree to a few ulps, zero points exactly
            grid_ok += (abs(sg - scales[r, g].item()) <= 1e-4 * sg) and (zg == zeros[r, g].item())
            w32 = cur[c0:c0 + 128].astype(np.float32)
            s_k, z_k = np.float32(scales[r, g].item()), np.float32(zeros[r, g].item())
            q = np.clip(np.rint((w32 / s_k).astype(np.float32)) + z_k, 0, maxq)
            agree += int(np.sum(q == codes[r, c0:c0 + 128].cpu().numpy()))
            total += 128
    return agree / total, grid_ok / groups


def _r_from_f(F, block=128):
    """R (upper, H_d = R R^T) from the block-scaled factor F, in float64 on the device: the diagonal
    blocks of F are U's, U_bb = R_bb^-1, and F_ab = R_ab U_bb above them."""
    F = F.double()
    d = F.shape[0]
    R = torch.zeros_like(F)
    eye = torch.eye(block, dtype=torch.float64, device=F.device)
    for b0 in range(0, d, block):
        b1 = b0 + block
        Rbb = torch.linalg.solve_triangular(F[b0:b1, b0:b1], eye, upper=True)
        R[b0:b1, b0:b1] = Rbb
        R[:b0, b0:b1] = F[:b0, b0:b1] @ Rbb
    return R


def test_dense_stress_shape_full_size(ctx):
    wl = workload(5, DEV)
    s = wl.spec
    L, n, d = s.n_layers, s.tokens[0], s.d_model
    W = wl.dense_weight()
    cal = DenseCalibration(ctx, s.d_out, d, L, s.bits_routed, s.damp_frac)
    g = np.random.default_rng(5)
    J = np.sort(g.choice(d, 512, replace=False))
    Jt = torch.from_numpy(J).to(DEV)
    sub_ref = []
    for l in range(L):
        X = wl.x(l, cache=False)
        cal.collect(l, X)
        sub_ref.append(O.gram(to64(X[:, Jt])))
        del X
        torch.cuda.empty_cache()
    alpha, lam = cal.quantize(W, "rt", want_host=True)
    torch.cuda.synchronize()
    S, cnt = cal.acc.buffers()
    assert cnt[:, 0].tolist() == [n] * L
    np.testing.assert_allclose(alpha[0], [0.25] * 4, rtol=1e-15)
    for l in range(L):
        blk = S[l, 0][Jt][:, Jt].double().cpu().numpy()
        full_blk = np.where(J[:, None] <= J[None, :], blk, blk.T)          # upper triangle is authoritative
        assert rel_fro(full_blk, sub_ref[l]) < 1e-4, l
    agg_ref = O.aggregate(sub_ref, [n] * L, "rt")
    assert rel_fro(cal.H_comb[0][Jt][:, Jt].double().cpu().numpy(), agg_ref["H_comb"]) < 1e-4
    # factor (the block-scaled Cholesky factor F), trailing block: F[t:, t:] depends only on H_d[t:, t:]
    # (H_d = R R^T, R upper, so R[t:, t:] is the factor of H_d[t:, t:]; t a multiple of 128)
    assert cal.form == FACTOR_BLOCK_CHOL
    t = d - 2048
    Hd_tail = cal.H_d[0][t:, t:].double().cpu().numpy()
    assert rel_fro(cal.U[0][t:, t:].double().cpu().numpy(), O.factor_block_scaled(Hd_tail)) < 1e-6
    assert torch.count_nonzero(torch.tril(cal.U[0], -1)) == 0
    # R from F (float64 on the device): R_bb = F_bb^-1, R_ab = F_ab R_bb; then R R^T v = H_d v
    R = _r_from_f(cal.U[0])
    Hd = cal.H_d[0].double()
    v = torch.randn((d, 4), dtype=torch.float64, device=DEV, generator=torch.Generator(DEV).manual_seed(1))
    assert (torch.linalg.norm(R @ (R.T @ v) - Hd @ v) / torch.linalg.norm(Hd @ v)).item() < 1e-5
    # U = R^-1; U^T U H_d v = v (float32-rounded F, cond(H_d) ~ 1e4)
    U = torch.linalg.solve_triangular(R, torch.eye(d, dtype=torch.float64, device=DEV), upper=True)
    del R
    res = U.T @ (U @ (Hd @ v)) - v
    assert (torch.linalg.norm(res) / torch.linalg.norm(v)).item() < 1e-2
    assert torch.all(torch.diagonal(U) > 0)
    # GPTQ: sampled rows consistent with the recurrence
    rows = g.choice(s.d_out, 6, replace=False)
    agree, grid_ok = _gptq_consistency(W, cal.q.W_hat[0], cal.q.codes[0], cal.q.scales[0], cal.q.zeros[0], U, rows,
                                       s.bits_routed)
    assert agree >= 0.999 and grid_ok >= 0.99, (agree, grid_ok)
    U64 = U.cpu().numpy()
    del U, Hd
    torch.cuda.empty_cache()
    # GPTQ stage-wise: the oracle's GPTQ of 16 sampled rows under the GPU's factor (as U, rebuilt from F
    # in float64; rows are independent)
    rows = np.sort(g.choice(s.d_out, 16, replace=False))
    rt = torch.from_numpy(rows).to(DEV)
    wc, ws, wz, wh, wm = O.gptq(to64(W[rt]), U64, s.bits_routed, s.group, 128, margins=True)
    del U64
    c = assert_codes(cal.q.codes[0][rt].cpu().numpy(), cal.q.zeros[0][rt].cpu().numpy(),
                     dict(codes=wc, zeros=wz, margin=wm), "dense stress rows", bar=CONFIG_BAR)
    print("codes dense stress", c)
    # loss: in-kernel |E|^2 - lambda |W_hat - W|^2 equals the direct trace under H_comb
    Dl = (cal.q.W_hat[0].double() - W.double())
    direct = torch.sum((Dl @ cal.H_comb[0].double()) * Dl).item()
    assert abs(cal.q.loss[0] - direct) <= 1e-3 * direct
