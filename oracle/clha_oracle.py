"""Plain, slow float64 CPU oracle of CLHA calibration (collect -> aggregate -> GPTQ).

TEST INFRASTRUCTURE ONLY: the tests, the package smoke check and the bench's CPU-baseline and
reference legs call this module; the CUDA library never does, and it shares no code with it.

Sources. "CLHA page" below is the technical summary "CLHA – Cross-Layer Hessian Aggregation voor
het kwantiseren van Weight-Shared Mixture-of-Experts Transformers" (gist.science, rs-10133806),
whose section 2 defines the method:
  §2.1   the shared-weight loss L(Wq) = sum_i alpha_i tr[(Wq - W) H_i (Wq - W)^T], alpha_i the share of
         tokens of layer i, and Proposition 1: minimising it is GPTQ with H_comb = sum_i alpha_i H_i;
  §2.2   the three phases: (1) collection of per-layer Hessians and token counts per active expert,
         (2) aggregation with alpha = n_a/(n_a+n_b) ("rt") or alpha = 0.5 ("eq"),
         (3) standard GPTQ column-sequential updates with H_comb;
  §2.3   CLHA-MP: b+1 bits for always-active shared experts;
  §2.4   layer-aware collection (one accumulator per (layer, expert), never mixed).
GPTQ itself is the published algorithm of Frantar, Ashkboos, Hoefler and Alistarh (2022), "GPTQ:
Accurate Post-Training Quantization for Generative Pre-trained Transformers", Algorithm 1; it is
restated here from its mathematics (damped Hessian, upper Cholesky factor of H^-1, column-by-column
rounding with the error fed forward along that factor's row).

Readings where the pages are silent (each also listed in the design notes):
  * H_l = (2/n_l) sum x x^T over the tokens routed to the expert in layer l; tokens are not weighted
    by their gate probability.
  * top-k ties go to the lower expert index; an expert's token list is in ascending token order.
  * the down-projection input is h = SiLU(x Wg^T) * (x Wu^T) of the full-precision weights, rounded
    to bfloat16 (round to nearest, ties to even) because that is the dtype h is stored in.
  * damping lambda = damp_frac * mean(diag H_comb) of the undamped aggregate; H_d = H_comb + lambda I.
  * the grid of a group is min-max asymmetric over the group's current (error-updated) values with 0
    included; an all-zero group uses [-1, 1].
  * the grid and the integer code are decided in binary32 (float32), the precision the kernel decides
    them in, so both sides take each rounding decision in the same precision; the error propagation
    around those decisions stays float64.
  * columns are quantized in natural order (no activation reordering).
  * a layer with no tokens contributes a zero Hessian; an expert with no tokens in any layer is an
    error (there is nothing to calibrate on), or, on request, is quantized by round to nearest
    (H_d = I), as is an expert whose weighted aggregate has no energy (per-layer calibration of an
    expert that the hook layer never routes to).
  * deployable codes are packed per row as one little-endian bit stream of 32-bit words, code j at
    bits [b*j, b*j + b) (the pages give no layout); W_hat = s (q - z) per group in float32.
  * cross-layer routing divergence (CLHA page §4-5: the gains grow with it; no formula is given) is
    the total-variation distance between two layers' expert frequencies p_l(e) = n_{l,e} / N_l.
  * the Calibration Hessian Error (CLHA page §4) of a quantized weight is the loss of §2.1 under a
    Hessian built from given tokens: on the calibration side the hook layer's own Hessian (the
    distribution per-layer calibration fits), on the test side the aggregate of fresh tokens of
    every layer sharing the weight (alpha by token share, the pooled distribution).
"""
from __future__ import annotations

from fractions import Fraction

import numpy as np

__all__ = [
    "route_topk", "expert_tokens", "gram", "hessian", "bf16_round", "bf16_margin", "silu", "ffn_act",
    "aggregate", "factor", "factor_block_scaled", "boundary_distance", "grid_fp32", "quantize_fp32", "gptq", "loss",
    "calibrate_dense", "calibrate_moe_group",
    "pack_codes", "unpack_codes", "dequantize", "dequant_matmul",
    "routing_divergence", "hessian_error",
]


# ----------------------------------------------------------------------------------- phase 1
def route_topk(logits, k: int):
    """Top-k routing of each token (CLHA page §2.2 (1): tokens reach their active experts).

    Returns ids [n, k] int32 (experts in descending logit order; ties -> lower expert index) and
    counts [E] int64 (tokens each expert receives).
    """
    lg = np.asarray(logits, dtype=np.float64)
    n, E = lg.shape
    if not (0 < k <= E):
        raise ValueError("k must be in 1..E")
    order = np.argsort(-lg, axis=1, kind="stable")
    ids = order[:, :k].astype(np.int32)
    counts = np.bincount(ids.ravel(), minlength=E).astype(np.int64)
    return ids, counts


def expert_tokens(ids, E: int):
    """Per expert, the ascending list of token indices routed to it."""
    ids = np.asarray(ids)
    return [np.nonzero((ids == e).any(axis=1))[0] for e in range(E)]


def gram(X):
    """S = sum over tokens of x x^T, in float64 from the exact stored values (CLHA page §2.2 (1))."""
    X = np.asarray(X, dtype=np.float64)
    return X.T @ X


def hessian(S, n: int):
    """H = (2/n) S; a layer without tokens contributes a zero Hessian."""
    S = np.asarray(S, dtype=np.float64)
    if n == 0:
        return np.zeros_like(S)
    return (2.0 / n) * S


def bf16_round(v):
    """Round float64 values to the nearest bfloat16 value (8 significant bits), ties to even."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    ulp_exp = np.maximum(ex - 8, -133)           # bfloat16 spacing; never finer than its subnormals
    r = np.ldexp(np.rint(np.ldexp(v, -ulp_exp)), ulp_exp)
    big = np.abs(r) >= 2.0 ** 128
    if np.any(big):
        r = np.where(big, np.copysign(np.inf, v), r)
    return r


def silu(a):
    """SiLU(a) = a * sigmoid(a), evaluated without overflow."""
    a = np.asarray(a, dtype=np.float64)
    out = np.empty_like(a)
    pos = a >= 0
    out[pos] = a[pos] / (1.0 + np.exp(-a[pos]))
    ea = np.exp(a[~pos])
    out[~pos] = a[~pos] * ea / (1.0 + ea)
    return out


def bf16_margin(v):
    """Distance of each value to the nearest rounding boundary of bf16_round (the midpoints between
    neighbouring bfloat16 values), in units of the bfloat16 step at the value: 0.5 for a value that
    is a bfloat16 number, 0 on a midpoint. A diagnostic of how close a rounding decision was."""
    v = np.asarray(v, dtype=np.float64)
    _, ex = np.frexp(v)
    return boundary_distance(np.ldexp(v, -np.maximum(ex - 8, -133)))


def ffn_act(Xe, Wg, Wu, return_margin: bool = False):
    """Input of an expert's down projection, h = SiLU(x Wg^T) * (x Wu^T), rounded to bfloat16;
    with return_margin also bf16_margin of the unrounded values."""
    Xe = np.asarray(Xe, dtype=np.float64)
    a = Xe @ np.asarray(Wg, dtype=np.float64).T
    b = Xe @ np.asarray(Wu, dtype=np.float64).T
    v = silu(a) * b
    if return_margin:
        return bf16_round(v), bf16_margin(v)
    return bf16_round(v)


# ----------------------------------------------------------------------------------- phase 2
def aggregate(S_list, n_list, mode: str = "rt", alpha=None, damp_frac: float = 0.01, empty: str = "error"):
    """Cross-layer aggregation (CLHA page §2.1 Proposition 1, §2.2 (2)) and damping.

    mode "rt": alpha_i = n_i / sum_j n_j; "eq": alpha_i = 1/L (0.5 for a pair);
    "explicit": alpha given (e.g. (1, 0) for per-layer calibration on the first layer only).
    Returns dict(alpha, H_comb, lam, H_d) with H_comb = sum_i alpha_i (2/n_i) S_i,
    lam = damp_frac * mean(diag H_comb), H_d = H_comb + lam I.
    empty: what an aggregate without energy (no tokens at all, or none in the layers that carry
    weight) becomes. "error" raises when no layer has tokens; "identity" gives H_comb = 0, lam = 1,
    H_d = I, under which GPTQ is round to nearest (a reading: the harness quantizes an expert that
    the calibration data never reach by RTN).
    """
    L = len(S_list)
    n = np.asarray(n_list, dtype=np.int64)
    if n.sum() == 0 and empty != "identity":
        raise ValueError("no tokens in any layer")
    if mode == "rt":
        a = n / n.sum() if n.sum() > 0 else np.zeros(L)
    elif mode == "eq":
        a = np.full(L, 1.0 / L)
    elif mode == "explicit":
        a = np.asarray(alpha, dtype=np.float64)
        if a.shape != (L,):
            raise ValueError("alpha must have one entry per layer")
    else:
        raise ValueError(mode)
    H_comb = np.zeros_like(np.asarray(S_list[0], dtype=np.float64))
    for ai, Si, ni in zip(a, S_list, n):
        H_comb += ai * hessian(Si, int(ni))
    lam = damp_frac * float(np.mean(np.diag(H_comb)))
    if empty == "identity" and np.trace(H_comb) == 0.0:
        lam = 1.0
    H_d = H_comb + lam * np.eye(H_comb.shape[0])
    return {"alpha": a, "H_comb": H_comb, "lam": lam, "H_d": H_d}


# ----------------------------------------------------------------------------------- phase 3
def factor(H_d):
    """U: the upper-triangular Cholesky factor of H_d^-1 (H_d^-1 = U^T U), by the plain route:
    H_d = L L^T, H_d^-1 = L^-T L^-1, then the Cholesky factorisation of that inverse."""
    H_d = np.asarray(H_d, dtype=np.float64)
    L = np.linalg.cholesky(H_d)
    Linv = np.linalg.inv(L)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T


def factor_block_scaled(H_d, block: int = 128):
    """F: the Cholesky factor of H_d scaled per column block, which GPTQ can use in place of U (a
    reformulation of GPTQ's lazy update, not a step of the pages).

    R is upper with H_d = R R^T (the Cholesky factorisation taken in reversed index order), and
    U = R^-1 is the same U as factor(H_d). A triangular matrix's inverse has the inverses of its
    diagonal blocks on its diagonal, so U_bb = R_bb^-1. F holds U_bb on each diagonal block b and
    R_ab U_bb on the blocks a < b above it, zeros below. With D = W - W_hat and GPTQ's scaled errors E
    (W - W_hat = E U, so E = D R and E_a U_aa = D_a), and U_ab = -U_aa R_ab U_bb, the lazy update
    W_b - E_a U_ab equals W_b + D_a F_ab. block = d gives F = U."""
    H_d = np.asarray(H_d, dtype=np.float64)
    d = H_d.shape[0]
    rev = np.arange(d)[::-1]
    R = np.linalg.cholesky(H_d[np.ix_(rev, rev)])[np.ix_(rev, rev)]   # upper, H_d = R R^T
    F = np.zeros_like(H_d)
    for b0 in range(0, d, block):
        b1 = min(d, b0 + block)
        Ubb = np.linalg.inv(R[b0:b1, b0:b1])
        F[b0:b1, b0:b1] = np.triu(Ubb)
        F[:b0, b0:b1] = R[:b0, b0:b1] @ Ubb
    return F


def boundary_distance(v):
    """Distance of each value to the nearest rounding boundary of round-to-nearest-integer (the
    half-integers): 0.5 for an integer, 0 exactly on a boundary. A diagnostic of how close a rounding
    decision was, not part of the method."""
    v = np.asarray(v, dtype=np.float64)
    return np.abs(np.abs(v - np.rint(v)) - 0.5)


def grid_fp32(wgrp, bits: int, return_margin: bool = False):
    """Asymmetric min-max grid of each row of a group, decided in binary32.

    wgrp: [rows, g] current values. Returns (s, z) float32 [rows]: step s = (xmax - xmin)/(2^b - 1)
    and integer zero point z = round(-xmin / s), with xmin <= 0 <= xmax (0 always on the grid) and
    [-1, 1] for an all-zero group. return_margin: also the boundary distance of -xmin / s, the value
    the zero point rounds.
    """
    w = np.asarray(wgrp, dtype=np.float64).astype(np.float32)
    maxq = np.float32(2 ** bits - 1)
    xmin = np.minimum(np.float32(0), w.min(axis=1))
    xmax = np.maximum(np.float32(0), w.max(axis=1))
    dead = (xmin == 0) & (xmax == 0)
    xmin = np.where(dead, np.float32(-1), xmin).astype(np.float32)
    xmax = np.where(dead, np.float32(1), xmax).astype(np.float32)
    s = ((xmax - xmin).astype(np.float32) / maxq).astype(np.float32)
    zv = ((-xmin).astype(np.float32) / s).astype(np.float32)
    z = np.rint(zv).astype(np.float32)
    if return_margin:
        return s, z, boundary_distance(zv)
    return s, z


def quantize_fp32(w, s, z, bits: int):
    """Code q = clamp(round(w/s) + z, 0, 2^b - 1) and value s (q - z), both in binary32."""
    w32 = np.asarray(w, dtype=np.float64).astype(np.float32)
    maxq = np.float32(2 ** bits - 1)
    q = np.clip(np.rint((w32 / s).astype(np.float32)) + z, np.float32(0), maxq).astype(np.float32)
    wq = (s * (q - z).astype(np.float32)).astype(np.float32)
    return q, wq


def gptq(W, U, bits: int, group: int, block: int | None = None, margins: bool = False):
    """GPTQ column-sequential quantization of W [d_out, d_in] with U = chol_upper(H_d^-1).

    For each column j in natural order: at a group start, fix each row's grid from the current
    values of that group; quantize the current value; e = (w_j - what_j) / U_jj; subtract e * U[j, k]
    from every later column k of the row. Rows are independent and are processed together.
    block=None applies every update at once (unblocked). block=B is GPTQ's lazy-batch form
    (Algorithm 1): inside a block of B columns the updates reach the block's own later columns column
    by column, and the later blocks receive the block's errors in one product E U[block, later] at
    its end: the same float64 updates in another order.
    Returns codes uint8 [d_out, d_in], scales float32 and zeros uint8 [d_out, d_in/group],
    W_hat float32 [d_out, d_in]; with margins=True also a dict of rounding margins, the boundary
    distance of each code's value w/s ("code", [d_out, d_in]) and of each zero point's -xmin/s
    ("zero", [d_out, d_in/group]): how far each integer decision was from flipping.
    """
    Wc = np.array(W, dtype=np.float64, copy=True)
    U = np.asarray(U, dtype=np.float64)
    d_out, d_in = Wc.shape
    if d_in % group:
        raise ValueError("d_in must be a multiple of the group size")
    B = d_in if block is None else int(block)
    codes = np.zeros((d_out, d_in), np.uint8)
    scales = np.zeros((d_out, d_in // group), np.float32)
    zeros = np.zeros((d_out, d_in // group), np.uint8)
    W_hat = np.zeros((d_out, d_in), np.float32)
    mc = np.zeros((d_out, d_in)) if margins else None
    mz = np.zeros((d_out, d_in // group)) if margins else None
    s = z = None
    for b0 in range(0, d_in, B):
        b1 = min(d_in, b0 + B)
        Err = np.zeros((d_out, b1 - b0))
        for j in range(b0, b1):
            if j % group == 0:
                s, z, zm = grid_fp32(Wc[:, j:j + group], bits, return_margin=True)
                scales[:, j // group] = s
                zeros[:, j // group] = z.astype(np.uint8)
                if margins:
                    mz[:, j // group] = zm
            q, wq = quantize_fp32(Wc[:, j], s, z, bits)
            if margins:
                mc[:, j] = boundary_distance((Wc[:, j].astype(np.float32) / s).astype(np.float32))
            codes[:, j] = q.astype(np.uint8)
            W_hat[:, j] = wq
            err = (Wc[:, j] - wq.astype(np.float64)) / U[j, j]
            Err[:, j - b0] = err
            Wc[:, j + 1:b1] -= np.outer(err, U[j, j + 1:b1])
        if b1 < d_in:
            Wc[:, b1:] -= Err @ U[b0:b1, b1:]
    if margins:
        return codes, scales, zeros, W_hat, {"code": mc, "zero": mz}
    return codes, scales, zeros, W_hat


def loss(W, W_hat, H):
    """tr[(W_hat - W) H (W_hat - W)^T] (CLHA page §2.1, one term of the shared-weight loss)."""
    D = np.asarray(W_hat, dtype=np.float64) - np.asarray(W, dtype=np.float64)
    return float(np.sum((D @ np.asarray(H, dtype=np.float64)) * D))


# ----------------------------------------------------------------------------------- pipelines
def calibrate_dense(W, X_list, bits: int, group: int = 128, mode: str = "rt", alpha=None,
                    damp_frac: float = 0.01, block: int | None = 128):
    """CLHA for one weight W [d_out, d_in] shared by the layers whose inputs are X_list (GPTQ in its
    lazy-batch form with `block` columns per batch; None: unblocked). "margin" holds GPTQ's rounding
    margins."""
    S = [gram(X) for X in X_list]
    n = [int(np.asarray(X).shape[0]) for X in X_list]
    agg = aggregate(S, n, mode, alpha, damp_frac)
    U = factor(agg["H_d"])
    codes, scales, zeros, W_hat, margin = gptq(W, U, bits, group, block, margins=True)
    return {"S": S, "n": n, **agg, "U": U, "codes": codes, "scales": scales, "zeros": zeros,
            "W_hat": W_hat, "margin": margin, "loss": loss(W, W_hat, agg["H_comb"]),
            "layer_loss": [loss(W, W_hat, hessian(Si, ni)) for Si, ni in zip(S, n)]}


def calibrate_moe_group(X_list, logits_list, k: int, routed, shared=(), experts=None,
                        bits_routed: int = 2, bits_shared: int = 3, group: int = 128,
                        mode: str = "rt", damp_frac: float = 0.01, shared_experts=None, alpha=None,
                        empty: str = "error", block: int | None = 128):
    """CLHA on one group of layers sharing routed experts `routed` [(Wg, Wu, Wd)] and always-active
    experts `shared` (CLHA page §2.2 phases 1-3, §2.3 mixed precision, §2.4 per-layer accumulators).

    experts / shared_experts: which routed / always-active experts to calibrate (default: all).
    Returns per-layer routing and, per expert key ("r", e) / ("s", e): token counts "n", the Hessian
    data "H_in" (gate/up inputs x) and "H_down" (down-projection inputs h), and the GPTQ results
    "gate", "up", "down" (with their rounding margins under "margin"), and the down projection's
    inputs "h" per layer with their bf16 rounding margins "h_margin". GPTQ runs in its lazy-batch
    form with `block` columns per batch (None: unblocked).
    """
    E = len(routed)
    if experts is None:
        experts = range(E)
    routes = [route_topk(lg, k) for lg in logits_list]
    toks = [expert_tokens(ids, E) for ids, _ in routes]
    out = {"routes": routes, "experts": {}}
    jobs = [(("r", e), routed[e], [t[e] for t in toks], bits_routed) for e in experts]
    if shared_experts is None:
        shared_experts = range(len(shared))
    jobs += [(("s", i), shared[i], [np.arange(np.asarray(X).shape[0]) for X in X_list], bits_shared)
             for i in shared_experts]
    for key, (Wg, Wu, Wd), tok_l, bits in jobs:
        Xe = [np.asarray(X, dtype=np.float64)[t] for X, t in zip(X_list, tok_l)]
        hm = [ffn_act(x, Wg, Wu, return_margin=True) for x in Xe]
        he = [h for h, _ in hm]
        n = [len(t) for t in tok_l]
        res = {"n": n}
        for kind, inputs, mats in (("H_in", Xe, (("gate", Wg), ("up", Wu))), ("H_down", he, (("down", Wd),))):
            S = [gram(x) for x in inputs]
            agg = aggregate(S, n, mode, alpha, damp_frac, empty)
            U = factor(agg["H_d"])
            res[kind] = {"S": S, **agg, "U": U}
            for name, Wm in mats:
                codes, scales, zeros, W_hat, margin = gptq(Wm, U, bits, group, block, margins=True)
                res[name] = {"codes": codes, "scales": scales, "zeros": zeros, "W_hat": W_hat, "margin": margin,
                             "loss": loss(Wm, W_hat, agg["H_comb"])}
        res["loss"] = res["gate"]["loss"] + res["up"]["loss"] + res["down"]["loss"]
        res["h"] = he
        res["h_margin"] = [m for _, m in hm]
        out["experts"][key] = res
    return out


# ------------------------------------------------------------------------------ deployable codes
def pack_codes(codes, bits: int):
    """Codes uint8 [rows, d_in] (values < 2^bits) -> uint32 [rows, d_in * bits / 32]: each row's codes
    as one little-endian bit stream, code j at bits [bits*j, bits*j + bits) (a code may straddle two
    words). The layout the deployable weights use; nothing in the pages fixes it."""
    codes = np.asarray(codes, dtype=np.uint64)
    rows, d_in = codes.shape
    if (d_in * bits) % 32:
        raise ValueError("d_in * bits must be a multiple of 32")
    words = np.zeros((rows, d_in * bits // 32), dtype=np.uint64)
    for j in range(d_in):
        bit = bits * j
        w, off = divmod(bit, 32)
        words[:, w] |= (codes[:, j] << np.uint64(off)) & np.uint64(0xFFFFFFFF)
        if off + bits > 32:
            words[:, w + 1] |= codes[:, j] >> np.uint64(32 - off)
    return words.astype(np.uint32)


def unpack_codes(packed, bits: int, d_in: int):
    """Inverse of pack_codes."""
    packed = np.asarray(packed, dtype=np.uint64)
    rows = packed.shape[0]
    out = np.zeros((rows, d_in), dtype=np.uint8)
    mask = np.uint64((1 << bits) - 1)
    for j in range(d_in):
        bit = bits * j
        w, off = divmod(bit, 32)
        v = packed[:, w] >> np.uint64(off)
        if off + bits > 32:
            v |= packed[:, w + 1] << np.uint64(32 - off)
        out[:, j] = (v & mask).astype(np.uint8)
    return out


def dequantize(codes, scales, zeros, group: int = 128):
    """W_hat = s (q - z) per group, in float32 (the same float32 operations GPTQ's W_hat uses)."""
    codes = np.asarray(codes)
    s = np.repeat(np.asarray(scales, np.float32), group, axis=1)
    z = np.repeat(np.asarray(zeros, np.float32), group, axis=1)
    return (s * (codes.astype(np.float32) - z)).astype(np.float32)


def dequant_matmul(X, packed, scales, zeros, bits: int, group: int = 128):
    """Y = X W_hat^T in float64 with W_hat decoded from the packed codes: the deployable layer's output."""
    d_in = np.asarray(X).shape[1]
    W_hat = dequantize(unpack_codes(packed, bits, d_in), scales, zeros, group)
    return np.asarray(X, dtype=np.float64) @ W_hat.astype(np.float64).T


# ------------------------------------------------------------------- divergence and held-out error
def routing_divergence(counts):
    """Total-variation distance between the expert frequencies of every pair of layers:
    TV[a][b] = 1/2 sum_e |n_{a,e}/N_a - n_{b,e}/N_b|, N_l = sum_e n_{l,e} (a reading: the CLHA page
    names cross-layer routing divergence without defining it). counts: integer [L, E]. Evaluated as
    an exact rational and rounded once to float64. A layer without tokens has no frequencies: error."""
    c = [[int(v) for v in row] for row in np.asarray(counts)]
    N = [sum(row) for row in c]
    if any(n <= 0 for n in N):
        raise ValueError("a layer without tokens has no expert frequencies")
    L = len(c)
    tv = np.zeros((L, L))
    for a in range(L):
        for b in range(L):
            tv[a, b] = float(sum(abs(Fraction(x, N[a]) - Fraction(y, N[b])) for x, y in zip(c[a], c[b])) / 2)
    return tv


def hessian_error(W, W_hat, S_list, n_list, mode: str = "rt", alpha=None):
    """The §2.1 loss of W_hat under the undamped aggregate of the given per-layer Gram sums: with
    alpha = (1, 0, ...) the hook layer's own Hessian, with "rt" the pooled Hessian of all layers."""
    return loss(W, W_hat, aggregate(S_list, n_list, mode, alpha)["H_comb"])
