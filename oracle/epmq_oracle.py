"""Plain float64 CPU oracle of E-PMQ: GPTQ of a merged layer toward its source experts' outputs.

TEST INFRASTRUCTURE ONLY (like the rest of this package): the tests call it, the CUDA library never
does, and it shares no code with it.

Source. "E-PMQ page" below is the technical summary "E-PMQ: Expert-Gestuurde Post-Merge Quantisatie
met Verankering van Gesmolten Gewichten" (gist.science, 2605.16882), section 2 (Methodologie):
  A  expert-driven targets: for source expert i with calibration activations X_i the target output
     is W_i X_i, and the quantized merged weight Q should reproduce it: minimise
     sum_i || Q X_i - W_i X_i ||_F^2;
  B  anchoring: add lambda || Q - W_m ||_F^2 toward the full-precision merged weight W_m, lambda
     adaptive and scaled with the layer's total activation energy;
  solver: GPTQ-style sequential rounding with the modified statistics H = sum_i H_i + lambda I and
     R = sum_i W_i H_i + lambda W_m.
The objective is a quadratic in Q: J(Q) = tr[Q H Q^T] - 2 tr[Q R^T] + const, so with the target
W* = R H^-1 it equals tr[(Q - W*) H (Q - W*)^T] + J(W*): GPTQ of W* under H minimises it.

Readings where the page is silent (also listed in the design notes):
  * H_i = X_i^T X_i with X_i [n_i, d] (rows are tokens), the unnormalised Gram matrix of the objective
    above (no 2/n factor: the objective sums over the calibration tokens);
  * lambda = damp_frac * tr(sum_i H_i) / d with damp_frac = 0.01, the GPTQ damping fraction applied to
    the layer's total activation energy tr(sum_i H_i) (the page gives no constant);
  * the GPTQ step (grid, rounding, column order, float32 decisions) is the CLHA oracle's;
  * X_i are given (the page collects them from the partially quantized model; that sequential
    collection is outside the path, as for CLHA).
"""
from __future__ import annotations

import numpy as np

from . import clha_oracle as _clha


def statistics(W_src, H_src, W_m, damp_frac: float = 0.01):
    """H = sum H_i + lambda I, R = sum W_i H_i + lambda W_m, lambda from the total activation energy.
    W_src: K arrays [d_out, d]; H_src: K arrays [d, d]; W_m [d_out, d]. float64 throughout."""
    H_sum = np.zeros_like(np.asarray(H_src[0], dtype=np.float64))
    R = np.zeros(np.asarray(W_m).shape, dtype=np.float64)
    for W_i, H_i in zip(W_src, H_src):
        H_i = np.asarray(H_i, dtype=np.float64)
        H_sum += H_i
        R += np.asarray(W_i, dtype=np.float64) @ H_i
    d = H_sum.shape[0]
    lam = damp_frac * np.trace(H_sum) / d
    H = H_sum + lam * np.eye(d)
    R += lam * np.asarray(W_m, dtype=np.float64)
    return H, R, lam


def target(H, R):
    """W* = R H^-1 (H symmetric positive definite), from the normal equations W* H = R."""
    return np.linalg.solve(H, R.T).T


def objective(Q, W_src, H_src, W_m, lam):
    """sum_i tr[(Q - W_i) H_i (Q - W_i)^T] + lambda || Q - W_m ||_F^2, the E-PMQ objective written with
    H_i = X_i^T X_i (|| (Q - W_i) X_i^T ||^2 = tr[(Q - W_i) H_i (Q - W_i)^T])."""
    Q = np.asarray(Q, dtype=np.float64)
    total = 0.0
    for W_i, H_i in zip(W_src, H_src):
        D = Q - np.asarray(W_i, dtype=np.float64)
        total += float(np.sum((D @ np.asarray(H_i, dtype=np.float64)) * D))
    Dm = Q - np.asarray(W_m, dtype=np.float64)
    return total + lam * float(np.sum(Dm * Dm))


def epmq(W_src, H_src, W_m, bits: int, group: int = 128, damp_frac: float = 0.01):
    """E-PMQ of one merged layer: statistics, target W* = R H^-1, GPTQ of W* under H (U = the upper
    Cholesky factor of H^-1). Returns the statistics, the target, the GPTQ outputs and the objective
    of the quantized weight (GPTQ in its lazy-batch form, with its rounding margins)."""
    H, R, lam = statistics(W_src, H_src, W_m, damp_frac)
    W_star = target(H, R)
    U = _clha.factor(H)
    codes, scales, zeros, W_hat, margin = _clha.gptq(W_star, U, bits, group, 128, margins=True)
    return {"H": H, "R": R, "lam": lam, "W_star": W_star, "U": U, "codes": codes, "scales": scales,
            "zeros": zeros, "W_hat": W_hat, "margin": margin,
            "objective": objective(W_hat.astype(np.float64), W_src, H_src, W_m, lam)}
