"""E-PMQ on the GPU (the E-PMQ page, section 2) against the E-PMQ oracle: the plain-sum aggregation,
the target W* = (lambda W_m + sum_i W_i S_i) H^-1 from the same Gram matrices, and the whole path from
source-expert activations to codes."""
import numpy as np
import pytest
import torch

from helpers import CONFIG_BAR, assert_codes, rel_fro, to64
from oracle import epmq_oracle as EP
from post_quantization_expert_b200 import clha as L
from post_quantization_expert_b200.pipeline import EPMQCalibration

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _sources(K, d_out, d, n, seed, spread=1.0, dtype=torch.bfloat16):
    g = torch.Generator().manual_seed(seed)
    W_base = 0.02 * torch.randn((d_out, d), generator=g)
    taus = [0.02 * spread * torch.randn((d_out, d), generator=g) for _ in range(K)]
    W_src = torch.stack([W_base + t for t in taus]).to(dtype)
    W_m = (W_base + sum(taus) / K).to(dtype)
    X = [(torch.randn((n, d), generator=g) * (0.5 + torch.rand(d, generator=g))).to(torch.bfloat16) for _ in range(K)]
    return W_src, W_m, X


@pytest.mark.parametrize("K,d_out,d,wdt", [(3, 128, 256, torch.float32), (5, 256, 384, torch.bfloat16)])
def test_sum_aggregate_and_target_match_oracle(ctx, K, d_out, d, wdt):
    W_src, W_m, X = _sources(K, d_out, d, 3 * d, seed=K, dtype=wdt)
    S32 = np.stack([(to64(x).T @ to64(x)).astype(np.float32) for x in X])       # the Gram matrices, float32
    cal = EPMQCalibration(ctx, K, d_out, d, bits=3)
    L.clha_accum_import(ctx, cal.acc, S32[:, None], np.full((K, 1), 3 * d, np.int64))
    Wd, Wm = W_src.to(DEV).contiguous(), W_m.to(DEV).contiguous()
    cal.quantize(Wd, Wm)
    torch.cuda.synchronize()
    S64 = [s.astype(np.float64) for s in S32]
    H, R, lam = EP.statistics([to64(w) for w in W_src], S64, to64(W_m))
    assert abs(cal.lam.item() - lam) <= 1e-12 * lam
    assert rel_fro(cal.H[0].double().cpu().numpy(), H - lam * np.eye(d)) < 1e-6
    W_star = EP.target(H, R)
    # float64 products of float32 factor entries: the rounding of U (2^-24) grows with cond(H)
    assert rel_fro(cal.W_target.double().cpu().numpy(), W_star) < 1e-5
    o = EP.epmq([to64(w) for w in W_src], S64, to64(W_m), bits=3)
    assert_codes(cal.q.codes[0].cpu().numpy(), cal.q.zeros[0].cpu().numpy(), o, "epmq from Grams", bar=CONFIG_BAR)


def test_epmq_end_to_end_from_activations(ctx):
    K, d_out, d, n = 4, 256, 512, 2048
    W_src, W_m, X = _sources(K, d_out, d, n, seed=21)
    cal = EPMQCalibration(ctx, K, d_out, d, bits=3)
    for i, x in enumerate(X):
        cal.collect(i, x.to(DEV).contiguous())
    q = cal.quantize(W_src.to(DEV).contiguous(), W_m.to(DEV).contiguous())
    torch.cuda.synchronize()
    H_src = [to64(x).T @ to64(x) for x in X]
    o = EP.epmq([to64(w) for w in W_src], H_src, to64(W_m), bits=3)
    assert rel_fro(cal.W_target.double().cpu().numpy(), o["W_star"]) < 1e-4   # phase-1 Grams within 1e-4
    assert_codes(q.codes[0].cpu().numpy(), q.zeros[0].cpu().numpy(), o, "epmq from activations", bar=CONFIG_BAR)
    got = EP.objective(q.W_hat[0].double().cpu().numpy(), [to64(w) for w in W_src], H_src, to64(W_m), o["lam"])
    assert abs(got - o["objective"]) <= 1e-3 * o["objective"]
    # and the quantized weight is closer to the experts' outputs than GPTQ of the merged weight alone
    import oracle as O
    _, _, _, W_naive = O.gptq(to64(W_m), O.factor(o["H"]), 3, 128)
    assert got < EP.objective(W_naive.astype(np.float64), [to64(w) for w in W_src], H_src, to64(W_m), o["lam"])
