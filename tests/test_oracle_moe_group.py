"""Pins of the oracle's MoE composition, calibrate_moe_group (CLHA page §2.2 phases 1-3, §2.3 CLHA-MP,
§2.4 per-layer accumulators), on a tiny weight-sharing MoE: E = 4 routed experts, top-2, two
always-active experts, d_model = d_ff = 128, two layers of 300 and 236 tokens.

Every output is rebuilt from the separately pinned step functions and from facts the pages fix:
  * a routed expert sees the tokens routed to it in each layer (ascending), an always-active expert
    every token of every layer; the routed counts of a layer sum to n k;
  * the gate and up projections share one input Hessian, the Gram of the expert's tokens x;
  * the down projection's Hessian is the Gram of h = SiLU(x Wg^T) (x Wu^T) (rounded to bf16), not of x;
  * routed experts get b bits, always-active ones b + 1 (CLHA-MP): codes of a shared expert use values
    above 2^b - 1, which no b-bit code can;
  * rt weighting of a layer pair is the pooled-token Hessian (closed form), eq weighting is 1/2 each;
  * an expert that no token reaches is an error, or round to nearest under the identity policy.
test_checker_catches_planted_slips plants, in a copy of the oracle's output, each slip that would
leave every step function's own pins green (the down-projection Gram built from x, the shared expert
given b bits, the shared expert given the routed token list) and checks that the checker fails.
"""
import copy

import numpy as np
import pytest

import oracle as O

E, K, DM, DFF, NSH = 4, 2, 128, 128, 2
TOKENS = (300, 236)
BITS_R, BITS_S = 2, 3


def _inputs(seed=11, dead_expert=None):
    g = np.random.default_rng(seed)
    Xs, lgs = [], []
    for l, n in enumerate(TOKENS):
        A = g.standard_normal((DM, 8)) * 0.4
        X = g.standard_normal((n, DM)) * np.sqrt(g.uniform(0.5, 2.0, DM)) + g.standard_normal((n, 8)) @ A.T
        Xs.append(O.bf16_round(X))
        lg = g.standard_normal((n, E))
        if dead_expert is not None:
            lg[:, dead_expert] = -50.0          # never among the top 2
        lgs.append(lg)
    w = lambda *shape: O.bf16_round(0.02 * g.standard_normal(shape))
    routed = [(w(DFF, DM), w(DFF, DM), w(DM, DFF)) for _ in range(E)]
    shared = [(w(DFF, DM), w(DFF, DM), w(DM, DFF)) for _ in range(NSH)]
    return Xs, lgs, routed, shared


def _check(out, Xs, lgs, routed, shared, mode, empty="error"):
    """Assert that calibrate_moe_group's output `out` is the composition of the pinned steps."""
    routes = out["routes"]
    for l, (X, lg) in enumerate(zip(Xs, lgs)):
        ids, counts = O.route_topk(lg, K)
        np.testing.assert_array_equal(routes[l][0], ids)
        np.testing.assert_array_equal(routes[l][1], counts)
        assert counts.sum() == X.shape[0] * K
    toks = [O.expert_tokens(O.route_topk(lg, K)[0], E) for lg in lgs]
    for (kind, e), r in out["experts"].items():
        Wg, Wu, Wd = (routed if kind == "r" else shared)[e]
        bits = BITS_R if kind == "r" else BITS_S
        tl = [t[e] for t in toks] if kind == "r" else [np.arange(X.shape[0]) for X in Xs]
        assert r["n"] == [len(t) for t in tl], (kind, e)
        Xe = [X[t] for X, t in zip(Xs, tl)]
        he = [O.ffn_act(x, Wg, Wu) for x in Xe]
        for l in range(len(Xs)):
            np.testing.assert_allclose(r["H_in"]["S"][l], O.gram(Xe[l]), rtol=1e-12, atol=1e-12)
            np.testing.assert_allclose(r["H_down"]["S"][l], O.gram(he[l]), rtol=1e-12, atol=1e-12)
            np.testing.assert_array_equal(r["h"][l], he[l])
        for hk, mats in (("H_in", (("gate", Wg), ("up", Wu))), ("H_down", (("down", Wd),))):
            agg = O.aggregate(r[hk]["S"], r["n"], mode, None, 0.01, empty)
            np.testing.assert_allclose(r[hk]["H_comb"], agg["H_comb"], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(r[hk]["lam"], agg["lam"], rtol=1e-12)
            U = O.factor(agg["H_d"])
            for name, Wm in mats:
                codes, scales, zeros, W_hat = O.gptq(Wm, U, bits, 128)
                np.testing.assert_array_equal(r[name]["codes"], codes, err_msg=f"{kind}{e} {name}")
                np.testing.assert_array_equal(r[name]["scales"], scales)
                np.testing.assert_array_equal(r[name]["zeros"], zeros)
                assert r[name]["codes"].max() <= 2 ** bits - 1
                np.testing.assert_allclose(r[name]["loss"], O.loss(Wm, W_hat, agg["H_comb"]), rtol=1e-12)
        assert r["loss"] == pytest.approx(r["gate"]["loss"] + r["up"]["loss"] + r["down"]["loss"], rel=1e-14)
        if kind == "s":
            # CLHA-MP: a 3-bit expert uses codes a 2-bit one cannot hold
            assert max(int(r[nm]["codes"].max()) for nm in ("gate", "up", "down")) > 2 ** BITS_R - 1
            # every token reaches it: its input Gram is the Gram of all of X
            for l, X in enumerate(Xs):
                np.testing.assert_allclose(r["H_in"]["S"][l], X.T @ X, rtol=1e-12, atol=1e-12)


@pytest.fixture(scope="module")
def tiny():
    return _inputs()


@pytest.mark.parametrize("mode", ["rt", "eq"])
def test_moe_group_is_the_composition_of_the_steps(tiny, mode):
    Xs, lgs, routed, shared = tiny
    out = O.calibrate_moe_group(Xs, lgs, K, routed, shared, None, BITS_R, BITS_S, 128, mode)
    assert sorted(out["experts"]) == [("r", e) for e in range(E)] + [("s", i) for i in range(NSH)]
    _check(out, Xs, lgs, routed, shared, mode)


def test_moe_group_weightings_closed_forms(tiny):
    """rt of a layer pair is the Hessian of the pooled tokens; eq is the plain mean of the per-layer
    Hessians (CLHA page §2.2 (2)); for an always-active expert rt = n_l / sum n."""
    Xs, lgs, routed, shared = tiny
    rt = O.calibrate_moe_group(Xs, lgs, K, routed, shared, [1], BITS_R, BITS_S, 128, "rt", shared_experts=[0])
    eq = O.calibrate_moe_group(Xs, lgs, K, routed, shared, [1], BITS_R, BITS_S, 128, "eq", shared_experts=[0])
    toks = [O.expert_tokens(O.route_topk(lg, K)[0], E)[1] for lg in lgs]
    pooled = np.concatenate([X[t] for X, t in zip(Xs, toks)])
    np.testing.assert_allclose(rt["experts"][("r", 1)]["H_in"]["H_comb"], 2.0 / len(pooled) * pooled.T @ pooled,
                               rtol=1e-12, atol=1e-12)
    per_layer = [2.0 / len(t) * X[t].T @ X[t] for X, t in zip(Xs, toks)]
    np.testing.assert_allclose(eq["experts"][("r", 1)]["H_in"]["H_comb"], 0.5 * (per_layer[0] + per_layer[1]),
                               rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(rt["experts"][("s", 0)]["H_in"]["alpha"], np.array(TOKENS) / sum(TOKENS), rtol=1e-15)
    allx = np.concatenate(Xs)
    np.testing.assert_allclose(rt["experts"][("s", 0)]["H_in"]["H_comb"], 2.0 / len(allx) * allx.T @ allx, rtol=1e-12,
                               atol=1e-12)


def test_moe_group_unrouted_expert_identity_policy():
    """An expert that no token reaches: an error by default, round to nearest (H_d = I, loss 0)
    under the identity policy; the other experts are unchanged by the policy."""
    Xs, lgs, routed, shared = _inputs(seed=12, dead_expert=3)
    with pytest.raises(ValueError):
        O.calibrate_moe_group(Xs, lgs, K, routed, (), [3], BITS_R, BITS_S, 128, "rt")
    out = O.calibrate_moe_group(Xs, lgs, K, routed, (), None, BITS_R, BITS_S, 128, "rt", empty="identity")
    r = out["experts"][("r", 3)]
    assert r["n"] == [0, 0]
    for hk in ("H_in", "H_down"):
        assert r[hk]["lam"] == 1.0
        np.testing.assert_array_equal(r[hk]["H_d"], np.eye(DM))
    for name in ("gate", "up", "down"):
        Wm = routed[3][("gate", "up", "down").index(name)]
        s, z = O.grid_fp32(Wm[:, :128], BITS_R)
        q, _ = O.quantize_fp32(Wm[:, :128], s[:, None], z[:, None], BITS_R)    # one group: plain RTN
        np.testing.assert_array_equal(r[name]["codes"], q.astype(np.uint8))
    assert r["loss"] == 0.0
    _check(out, Xs, lgs, routed, (), "rt", empty="identity")
    ref = O.calibrate_moe_group(Xs, lgs, K, routed, (), [0, 1, 2], BITS_R, BITS_S, 128, "rt")
    for e in range(3):
        np.testing.assert_array_equal(out["experts"][("r", e)]["gate"]["codes"], ref["experts"][("r", e)]["gate"]["codes"])


def test_checker_catches_planted_slips(tiny):
    """Each slip that the step functions' own pins cannot see, planted in a copy of the output, turns
    the composition check red."""
    Xs, lgs, routed, shared = tiny
    out = O.calibrate_moe_group(Xs, lgs, K, routed, shared, None, BITS_R, BITS_S, 128, "rt")
    _check(out, Xs, lgs, routed, shared, "rt")
    toks = [O.expert_tokens(O.route_topk(lg, K)[0], E) for lg in lgs]

    # 1. the down projection's Gram built from the expert's x instead of h
    bad = copy.deepcopy(out)
    r = bad["experts"][("r", 0)]
    r["H_down"]["S"] = [O.gram(X[t[0]]) for X, t in zip(Xs, toks)]
    with pytest.raises(AssertionError):
        _check(bad, Xs, lgs, routed, shared, "rt")

    # 2. an always-active expert quantized with the routed experts' bits
    bad = copy.deepcopy(out)
    r = bad["experts"][("s", 1)]
    U = O.factor(r["H_in"]["H_d"])
    for name, Wm in (("gate", shared[1][0]), ("up", shared[1][1])):
        codes, scales, zeros, W_hat = O.gptq(Wm, U, BITS_R, 128)
        r[name].update(codes=codes, scales=scales, zeros=zeros, loss=O.loss(Wm, W_hat, r["H_in"]["H_comb"]))
    Ud = O.factor(r["H_down"]["H_d"])
    codes, scales, zeros, W_hat = O.gptq(shared[1][2], Ud, BITS_R, 128)
    r["down"].update(codes=codes, scales=scales, zeros=zeros, loss=O.loss(shared[1][2], W_hat, r["H_down"]["H_comb"]))
    with pytest.raises(AssertionError):
        _check(bad, Xs, lgs, routed, shared, "rt")

    # 3. an always-active expert given a routed expert's token list
    bad = copy.deepcopy(out)
    r = bad["experts"][("s", 0)]
    r["n"] = [len(t[0]) for t in toks]
    r["H_in"]["S"] = [O.gram(X[t[0]]) for X, t in zip(Xs, toks)]
    with pytest.raises(AssertionError):
        _check(bad, Xs, lgs, routed, shared, "rt")
