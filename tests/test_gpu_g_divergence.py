"""Routing divergence and the Calibration Hessian Error on the GPU against the oracle (the CLHA page,
section 4: calibration versus held-out error and the routing-sharpness experiment).

The divergence is integer arithmetic plus one float64 division, so it must match the oracle's
exactly rounded rational bit for bit. The Hessian error runs the collection, aggregation and loss
kernels on held-out (or calibration) tokens; both sides score the same seeded W_hat, so the check
is independent of GPTQ, and the bar is the per-expert loss tolerance, 1e-3 relative."""
from types import SimpleNamespace

import numpy as np
import pytest
import torch

import oracle as O
from helpers import to64
from post_quantization_expert_b200 import clha as L
from post_quantization_expert_b200.analysis import HessianError, mean_pairwise, routing_divergence
from post_quantization_expert_b200.pipeline import MoECalibration, stack_weights
from synth import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _tv_device(ctx, counts: np.ndarray, slot0: int, E: int) -> np.ndarray:
    c = torch.from_numpy(np.ascontiguousarray(counts, np.int64)).to(DEV)
    L_, ld = counts.shape
    tv = torch.full((L_, L_), -1.0, dtype=torch.float64, device=DEV)
    L.clha_routing_divergence(ctx, c, L_, ld, slot0, E, tv)
    L.clha_check(ctx)
    return tv.cpu().numpy()


@pytest.mark.parametrize("L_,E,ld,slot0,hi", [(2, 16, 16, 0, 5000), (5, 1, 3, 2, 100), (3, 300, 301, 1, 1000),
                                             (32, 64, 65, 0, 200000), (4, 7, 7, 0, 3), (2, 1000, 1000, 0, 90000)])
def test_divergence_bit_exact(ctx, L_, E, ld, slot0, hi):
    """Ragged expert counts around the block width, one expert, a stride and offset, 32 layers, and
    totals up to ~9e7 tokens per layer (2 N_a N_b near 2^53)."""
    rng = np.random.default_rng(L_ * 1000 + E)
    counts = rng.integers(0, hi, size=(L_, ld)).astype(np.int64)
    counts[:, slot0] += 1                      # every layer has tokens
    counts[0, slot0:slot0 + E] = 0
    counts[0, slot0 + E - 1] = 9               # a layer routed to one expert only
    got = _tv_device(ctx, counts, slot0, E)
    want = O.routing_divergence(counts[:, slot0:slot0 + E])
    assert np.array_equal(got, want)


def test_divergence_errors_leave_the_context_usable(ctx):
    good = np.array([[3, 1, 0, 0], [1, 1, 1, 1]], np.int64)
    for bad, status in ((np.array([[1, 2, 0, 0], [0, 0, 0, 0]]), L.ERR_EMPTY),
                        (np.array([[1, -2, 5, 0], [1, 1, 1, 1]]), L.ERR_INVALID_ARG),
                        (np.array([[1, 2, 1 << 31, 0], [1, 1, 1, 1]]), L.ERR_INVALID_ARG)):
        with pytest.raises(L.ClhaError) as ei:
            _tv_device(ctx, bad, 0, 4)
        assert ei.value.status == status
    np.testing.assert_array_equal(_tv_device(ctx, good, 0, 4), [[0, 0.5], [0.5, 0]])


def _collected(ctx, wl, w, s, tokens):
    cal = MoECalibration(ctx, 2, tokens, s.E, s.k, s.d_model, s.d_ff, s.n_shared, s.shared_dff,
                         s.bits_routed, s.bits_shared, s.damp_frac)
    for l in range(2):
        cal.collect(l, wl.x(l).to(DEV), wl.logits(l).to(DEV), w)
    return cal


def _oracle_grams(wl, s, routed):
    """Per routed expert: per-layer Gram sums of its inputs and of its down-projection inputs, and
    token counts, from the oracle's own routing."""
    Xs = [to64(wl.x(l)) for l in range(2)]
    routes = [O.route_topk(wl.logits(l).numpy(), s.k) for l in range(2)]
    toks = [O.expert_tokens(ids, s.E) for ids, _ in routes]
    out = []
    for e, (Wg, Wu, _) in enumerate(routed):
        Xe = [X[t[e]] for X, t in zip(Xs, toks)]
        he = [O.ffn_act(x, to64(Wg), to64(Wu)) for x in Xe]
        out.append(([O.gram(x) for x in Xe], [O.gram(h) for h in he], [len(t[e]) for t in toks]))
    return out, [c for _, c in routes]


@pytest.mark.parametrize("beta", [0.0, 0.5])
def test_divergence_and_hessian_error_of_collected_tokens(ctx, beta):
    """A sharpened top-2-of-16 pair (d_model 1024, d_ff 512) on calibration and held-out tokens: the
    divergence of the collected counts, and each expert's error under the held-out rt aggregate and
    under the calibration hook layer's own Hessian, for a seeded W_hat given to both sides."""
    n = 2048
    cal_wl = workload(2, tokens=n, sharpness=beta)
    test_wl = workload(2, tokens=n, sharpness=beta, split="test")
    s = cal_wl.spec
    routed = [cal_wl.expert_weights(0, e) for e in range(s.E)]
    w = stack_weights((routed, []), DEV)
    g = torch.Generator().manual_seed(77)
    Wgu_hat = (w.Wgu.float().cpu() + 2e-3 * torch.randn(w.Wgu.shape, generator=g)).contiguous()
    Wd_hat = (w.Wd.float().cpu() + 2e-3 * torch.randn(w.Wd.shape, generator=g)).contiguous()
    r = SimpleNamespace(qgu=SimpleNamespace(W_hat=Wgu_hat.to(DEV)), qd=SimpleNamespace(W_hat=Wd_hat.to(DEV)))
    he = HessianError(ctx, s.E, s.d_model, s.d_ff)
    for wl, mode, alpha in ((test_wl, "rt", None), (cal_wl, "explicit", (1.0, 0.0))):
        col = _collected(ctx, wl, w, s, n)
        got = he(col, w, r, mode, alpha)["routed"]
        grams, counts = _oracle_grams(wl, s, routed)
        tv = routing_divergence(ctx, col.acc_in, 0, s.E)
        assert np.array_equal(tv, O.routing_divergence(np.stack(counts)))
        if beta > 0:
            assert mean_pairwise(tv) > 0.3
        for e, (S_in, S_dn, ne) in enumerate(grams):
            Wg, Wu, Wd = (to64(m) for m in routed[e])
            want = (O.hessian_error(Wg, to64(Wgu_hat[e]), S_in, ne, mode, alpha)
                    + O.hessian_error(Wu, to64(Wgu_hat[s.E + e]), S_in, ne, mode, alpha)
                    + O.hessian_error(Wd, to64(Wd_hat[e]), S_dn, ne, mode, alpha))
            assert abs(got[e] - want) <= 1e-3 * want, (e, got[e], want)
