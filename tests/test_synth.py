"""The seeded input generator: determinism, shapes and the covariance model it promises."""
import math

import numpy as np
import torch

from synth import workload


def test_deterministic_and_shapes():
    a, b = workload(1), workload(1)
    for l in range(2):
        assert torch.equal(a.x(l), b.x(l))
    assert a.x(0).shape == (1000, 512) and a.x(1).shape == (1024, 512)
    assert a.x(0).dtype == torch.float32
    assert a.dense_weight().shape == (256, 512)
    w2 = workload(2, tokens=256)
    assert w2.x(0).dtype == torch.bfloat16 and w2.x(0).shape == (256, 1024)
    assert w2.logits(1).shape == (256, 16)
    wg, wu, wd = w2.expert_weights(0, 3)
    assert wg.shape == (512, 1024) and wd.shape == (1024, 512)
    assert not torch.equal(w2.x(0), w2.x(1))


def test_covariance_model_and_drift():
    w = workload(1, tokens=(20000, 20000))
    sqD, Us, _ = w._cov_model(0, 512)
    for l in range(2):
        X = w.x(l).double()
        C = X.T @ X / X.shape[0]
        want = torch.diag(sqD.double() ** 2) + Us[l].double() @ Us[l].double().T
        rel = torch.linalg.norm(C - want) / torch.linalg.norm(want)
        assert rel < 0.1          # sampling noise of a 20000-token estimate is about 0.05
    # drift 0.3: U_b = cos(0.15 pi) U_a + sin(0.15 pi) V
    Ua, Ub = Us
    c = math.cos(math.pi * 0.15)
    proj = (Ua * Ub).sum() / (Ua * Ua).sum()
    assert abs(proj.item() - c) < 0.1


def test_outliers_and_zipf():
    w = workload(3, tokens=2048)
    X = w.x(0).float()
    std = X.std(0)
    assert int((std > 8).sum()) == 20
    lg = w.logits(0)
    top1 = torch.bincount(lg.argmax(1), minlength=64).float()
    assert top1.max() > 8 * top1.median()
