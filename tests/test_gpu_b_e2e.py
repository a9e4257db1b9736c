"""End-to-end parity of the GPU calibration path with the float64 oracle on the seeded workloads:
routing counts bit-exact, Hessians within 1e-4 relative Frobenius error, codes agreeing on >= 99.9%
of entries with every differing row starting at a certified rounding-boundary flip, per-expert
reconstruction loss within 1e-3 relative. Where the oracle cannot afford a whole workload, it checks
every Hessian and a sample of experts' GPTQ end to end."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import CONFIG_BAR, CodeTally, assert_codes, rel_fro, sym_from_upper, to64
from post_quantization_expert_b200 import clha as L
from post_quantization_expert_b200.pipeline import DenseCalibration, MoECalibration, stack_weights
from synth import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _dense_case(ctx, cfg, form=L.FACTOR_BLOCK_CHOL, **over):
    wl = workload(cfg, "cpu", **over)
    s = wl.spec
    W = wl.dense_weight()
    Xs = [wl.x(l) for l in range(s.n_layers)]
    cal = DenseCalibration(ctx, s.d_out, s.d_model, s.n_layers, s.bits_routed, s.damp_frac, factor_form=form)
    for l, X in enumerate(Xs):
        cal.collect(l, X.to(DEV))
    alpha, lam = cal.quantize(W.to(DEV), "rt", want_host=True)
    torch.cuda.synchronize()
    want = O.calibrate_dense(to64(W), [to64(X) for X in Xs], s.bits_routed, s.group, "rt", None, s.damp_frac)
    return cal, want, alpha, lam, W


@pytest.mark.parametrize("form", ["block", "inv"])
def test_dense_two_layer_fp32_workload(ctx, form):
    """The dense fp32 workload: W 256x512 shared by two layers of 1000 and 1024 tokens, 2-bit; GPTQ with
    either factor form against the oracle's (the pages' recurrence with U)."""
    block = form == "block"
    cal, want, alpha, lam, W = _dense_case(ctx, 1, L.FACTOR_BLOCK_CHOL if block else L.FACTOR_INV_CHOL)
    S, cnt = cal.acc.buffers()
    assert cnt[:, 0].tolist() == [1000, 1024]
    for l in range(2):
        assert rel_fro(sym_from_upper(S[l, 0].double().cpu().numpy()), want["S"][l]) < 1e-4
    np.testing.assert_allclose(alpha[0], [1000 / 2024, 1024 / 2024], rtol=1e-15)
    np.testing.assert_allclose(lam[0], want["lam"], rtol=1e-5)
    assert rel_fro(cal.H_comb[0].double().cpu().numpy(), want["H_comb"]) < 1e-4
    want_factor = O.factor_block_scaled(want["H_d"]) if block else want["U"]
    assert rel_fro(cal.U[0].double().cpu().numpy(), want_factor) < 1e-4
    print("dense c1 codes", assert_codes(cal.q.codes[0].cpu().numpy(), cal.q.zeros[0].cpu().numpy(), want, "dense",
                                         bar=CONFIG_BAR))
    assert abs(cal.q.loss[0] - want["loss"]) <= 1e-3 * want["loss"]


def _moe_pair(ctx, cfg, experts_checked, modes, shared_checked=None, fused=False, act=None, **over):
    wl = workload(cfg, "cpu", **over)
    s = wl.spec
    Xs = [wl.x(l) for l in range(2)]
    lgs = [wl.logits(l) for l in range(2)]
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    shared = [wl.expert_weights(0, i, shared=True) for i in range(s.n_shared)]
    w = stack_weights((routed, shared), DEV)
    cal = MoECalibration(ctx, 2, max(s.tokens), s.E, s.k, s.d_model, s.d_ff, s.n_shared, s.shared_dff,
                         s.bits_routed, s.bits_shared, s.damp_frac, modes=modes, fused_gather=fused)
    for l in range(2):
        cal.collect(l, Xs[l].to(DEV), lgs[l].to(DEV), w)
        if act is not None:   # the kernel the default per-call choice took (last activation call)
            assert L.clha_last_act_kernel(ctx) == act
    torch.cuda.synchronize()
    X64 = [to64(X) for X in Xs]
    # routing counts: bit-exact
    routes = [O.route_topk(lg.numpy(), s.k) for lg in lgs]
    for l in range(2):
        np.testing.assert_array_equal(cal.counts[l].cpu().numpy(), routes[l][1])
    # every routed expert's input Hessian, both layers
    S_in, n_in = cal.acc_in.buffers()
    S_dn, _ = cal.acc_dn.buffers()
    toks = [O.expert_tokens(r[0], s.E) for r in routes]
    for l in range(2):
        for e in range(s.E):
            assert n_in[l, e].item() == len(toks[l][e])
            got = sym_from_upper(S_in[l, e].double().cpu().numpy())
            assert rel_fro(got, O.gram(X64[l][toks[l][e]])) < 1e-4
    if s.n_shared:
        for l in range(2):
            assert rel_fro(sym_from_upper(S_in[l, s.E].double().cpu().numpy()), O.gram(X64[l])) < 1e-4
    # sampled experts: down-projection Hessians and the whole GPTQ path, per weighting
    ref = {}
    tally = CodeTally((cfg, over.get("tokens")))
    cal.quantize(w, modes)           # every weighting in one pass (batched factorisation)
    torch.cuda.synchronize()
    for mode in modes:
        out = cal.res[mode]
        res = O.calibrate_moe_group(X64, [lg.numpy() for lg in lgs], s.k, [tuple(to64(t) for t in r) for r in routed],
                                    [tuple(to64(t) for t in sh) for sh in shared], experts_checked,
                                    s.bits_routed, s.bits_shared, s.group, mode, s.damp_frac, shared_checked)
        for key, r in res["experts"].items():
            kind, e = key
            if kind == "r":
                for l in range(2):
                    got = sym_from_upper(S_dn[l, e].double().cpu().numpy())
                    assert rel_fro(got, r["H_down"]["S"][l]) < 1e-4, (mode, key, l)
                qs = {"gate": out.qg, "up": out.qu, "down": out.qd}
            else:
                qs = {"gate": out.sg, "up": out.su, "down": out.sd}
            for name, q in qs.items():
                tally.add(q.codes[e].cpu().numpy(), q.zeros[e].cpu().numpy(), r[name], (mode, key, name))
            got_loss = sum(qs[n].loss[e] for n in ("gate", "up", "down"))
            assert abs(got_loss - r["loss"]) <= 1e-3 * r["loss"], (mode, key, got_loss, r["loss"])
        ref[mode] = res
    tally.check()
    return cal, ref


def test_moe_pair_E16_top2_full_size(ctx):
    """The E=16, top-2, d_model 1024, d_ff 512 layer pair at 8192 tokens per layer, 3-bit, both
    weightings: all Hessians and routing checked; GPTQ end to end on experts 0, 7 and 15. The packed
    path, where the activation runs on the tensor cores (no outlier channels here)."""
    _moe_pair(ctx, 2, [0, 7, 15], ("rt", "eq"), act=L.ACT_TENSOR)


def test_moe_pair_E64_top6_shared_reduced_tokens(ctx):
    """The E=64 top-6 shape with two always-active experts (CLHA-MP: routed 2-bit, shared 3-bit),
    Zipf-skewed routing and outlier channels, at 4096 tokens per layer. The fused path (the expert
    inputs read from X by TMA gather4, no packed copy; the routed experts' activation reads its rows
    through the permutation on the FMA kernel); the always-active experts' activation, the last of a
    collect, runs on the tensor cores with the outlier channels taken out of the tensor-core sums."""
    _moe_pair(ctx, 3, [0, 63], ("rt",), shared_checked=[1], fused=True, act=L.ACT_TENSOR, tokens=4096)


def test_unrouted_experts_are_round_to_nearest(ctx):
    """An expert the router never picks (expert 3) and, under per-layer calibration on layer 0, an
    expert picked only in layer 1 (expert 5): their aggregates have no energy, so both sides quantize
    them by round to nearest (H_d = I) with zero loss; a routed expert (0) alongside is unaffected."""
    wl = workload(2, "cpu", tokens=1024)
    s = wl.spec
    Xs = [wl.x(l) for l in range(2)]
    lgs = [wl.logits(l).clone() for l in range(2)]
    for lg in lgs:
        lg[:, 3] = -1.0e4
    lgs[0][:, 5] = -1.0e4
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    w = stack_weights((routed, []), DEV)
    modes = ("rt", "explicit")
    cal = MoECalibration(ctx, 2, 1024, s.E, s.k, s.d_model, s.d_ff, 0, 0, s.bits_routed, s.bits_shared,
                         s.damp_frac, modes=modes)
    for l in range(2):
        cal.collect(l, Xs[l].to(DEV), lgs[l].to(DEV), w)
    cal.quantize(w, modes, alpha=(1.0, 0.0))
    torch.cuda.synchronize()
    cnt = cal.counts.cpu().numpy()
    assert cnt[0, 3] == 0 and cnt[1, 3] == 0 and cnt[0, 5] == 0 and cnt[1, 5] > 0
    X64 = [to64(X) for X in Xs]
    W64 = [tuple(to64(t) for t in r) for r in routed]
    # expert 0 under alpha = (1, 0) sees only layer 0's ~128 tokens in 1024 dimensions: a Hessian
    # that is rank-deficient up to the damping, the hardest case for the code bar
    tally = CodeTally("unrouted")
    for mode, alpha, experts in (("rt", None, (3, 0)), ("explicit", (1.0, 0.0), (3, 5, 0))):
        ref = O.calibrate_moe_group(X64, [lg.numpy() for lg in lgs], s.k, W64, (), list(experts), s.bits_routed,
                                    s.bits_shared, s.group, mode, s.damp_frac, alpha=alpha, empty="identity")
        r = cal.res[mode]
        for e in experts:
            want = ref["experts"][("r", e)]
            for name, q in (("gate", r.qg), ("up", r.qu), ("down", r.qd)):
                tally.add(q.codes[e].cpu().numpy(), q.zeros[e].cpu().numpy(), want[name], (mode, e, name))
            got = r.expert_loss()[e]
            if e == 0:
                assert abs(got - want["loss"]) <= 1e-3 * want["loss"]
            else:
                # the in-kernel loss is |E|^2 - lambda |W_hat - W|^2 with E = W - W_hat here: zero up
                # to the float32 rounding of the two sums
                err2 = sum(float(((q.W_hat[e].double() - Wm.double().to(DEV)) ** 2).sum())
                           for q, Wm in ((r.qg, routed[e][0]), (r.qu, routed[e][1]), (r.qd, routed[e][2])))
                assert want["loss"] == 0.0 and abs(got) <= 1e-5 * err2, (mode, e, got, err2)
    tally.check()
