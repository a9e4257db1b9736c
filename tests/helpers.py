"""Comparison helpers shared by the GPU parity tests (no method arithmetic here)."""
import numpy as np
import torch


def to64(t):
    """Exact float64 copy of a device tensor (bf16 / f32 values are exactly representable)."""
    return t.detach().float().cpu().double().numpy() if t.dtype != torch.float64 else t.cpu().numpy()


def sym_from_upper(S):
    """Full symmetric matrix from the authoritative upper triangle (incl. the diagonal)."""
    U = np.triu(S)
    return U + np.triu(S, 1).T


def rel_fro(a, b):
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def code_agreement(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return float(np.mean(a == b))


# A code mismatch is certified as a rounding-boundary flip when, at the first place its row parts
# ways with the oracle (the first mismatching code, or an earlier group whose zero point differs),
# the oracle's own value was within FLIP_TOL of a step from the rounding boundary. Before that place
# both sides made every decision alike, so their current values differ only by rounding order; a
# value that far from a boundary cannot flip. Later mismatches in the row follow from the first (the
# two runs then propagate different errors) and are not certified one by one.
FLIP_TOL = 1e-3


def certify_codes(got_codes, got_zeros, want, group=128, tol=FLIP_TOL):
    """Agreement of one matrix's codes with the oracle's (want: a GPTQ result with "codes", "zeros"
    and "margin") and the certification of every row that differs. Returns a dict: agree (fraction
    of equal codes), rows (rows that differ), certified (of those, rows whose first difference is a
    boundary flip), worst (largest margin, in steps, at a first difference)."""
    gc, wc = np.asarray(got_codes), np.asarray(want["codes"])
    gz, wz = np.asarray(got_zeros), np.asarray(want["zeros"])
    mism, zmism = gc != wc, gz != wz
    rows = np.nonzero(mism.any(1) | zmism.any(1))[0]
    worst, certified = 0.0, 0
    for r in rows:
        jc = int(np.argmax(mism[r])) if mism[r].any() else None
        jz = int(np.argmax(zmism[r])) if zmism[r].any() else None
        if jz is not None and (jc is None or jz * group <= jc):
            m = float(want["margin"]["zero"][r, jz])
        else:
            m = float(want["margin"]["code"][r, jc])
        worst = max(worst, m)
        certified += m <= tol
    return {"agree": 1.0 - float(mism.mean()), "rows": len(rows), "certified": int(certified), "worst": worst}


# The code bar (the reading of ">= 99.9 % of entries, rounding-boundary flips only"): the compared
# codes of a workload agree on at least CONFIG_BAR of their entries taken together; every single
# matrix on at least MATRIX_BAR; and every row that differs starts with a certified boundary flip.
# A matrix between the two bars is one whose Hessian is rank-deficient up to the damping (an expert
# with ~100 tokens in ~1000 dimensions), where the float32 rounding of the Hessian alone moves a few
# decisions across their boundaries and GPTQ carries each flip into the rest of its row.
CONFIG_BAR = 0.999
MATRIX_BAR = 0.998

# A down projection whose input h carries certified one-step bfloat16 differences (certify_h below)
# has a Hessian up to 1e-3 from the oracle's, not float32 rounding away, so many more of its decisions
# lie within reach of a flip, and GPTQ's error feedback carries each one along its row. Such a matrix
# is held to H_INPUT_BAR; every row that differs is still certified, and its codes still count toward
# the workload's CONFIG_BAR.
H_INPUT_BAR = 0.995


def assert_codes(got_codes, got_zeros, want, what, bar=MATRIX_BAR):
    """One matrix: at least `bar` of the codes equal the oracle's, and every row that differs starts
    with a certified rounding-boundary flip."""
    c = certify_codes(got_codes, got_zeros, want)
    assert c["agree"] >= bar and c["certified"] == c["rows"], (what, c)
    c["n"] = int(np.asarray(got_codes).size)
    return c


class CodeTally:
    """Per-workload tally of the code bar: add() checks one matrix (MATRIX_BAR, certification) and
    counts its codes; check() asserts the workload's agreement over every matrix added."""

    def __init__(self, what):
        self.what, self.equal, self.total, self.matrices = what, 0.0, 0, []

    def add(self, got_codes, got_zeros, want, what, bar=MATRIX_BAR):
        c = assert_codes(got_codes, got_zeros, want, what, bar)
        self.equal += c["agree"] * c["n"]
        self.total += c["n"]
        self.matrices.append((what, c))
        print("codes", self.what, what, c)
        return c

    def check(self):
        agree = self.equal / max(self.total, 1)
        print("codes total", self.what, f"{agree:.6f} over {len(self.matrices)} matrices, {self.total} codes")
        assert agree >= CONFIG_BAR, (self.what, agree)
        return agree


# h differences: the GPU and the oracle round h to bfloat16 from values that differ by float32-level
# errors in the pre-activations (the exact sums are float64 on the oracle's side). An element can
# then land on the other bfloat16 neighbour: near a rounding midpoint, or anywhere for a tiny h whose
# terms cancel. Such differences are one bfloat16 step each and rare (a wrong token, weight or
# expert would move most elements by far more); in an expert with ~100 tokens a single one on a large
# h moves the Gram of h by ~1e-4 relative.
H_DIFF_MAX = 1e-3


def certify_h(got_h, want_h, margin, what):
    """Every element of h that differs from the oracle's is one bfloat16 step away, or (a tiny h whose
    terms cancel) within 1e-5 of the largest |h| in absolute terms, and at most H_DIFF_MAX of the
    elements differ. Returns (fraction that differs, largest rounding margin of a differing element,
    in steps; near 0 for a flip at a midpoint)."""
    got_h, want_h, margin = np.asarray(got_h), np.asarray(want_h), np.asarray(margin)
    diff = got_h != want_h
    if not diff.any():
        return 0.0, 0.0
    _, ex = np.frexp(want_h[diff])
    step = np.ldexp(1.0, np.maximum(ex - 8, -133))
    gap = np.abs(got_h[diff] - want_h[diff])
    assert np.all((gap <= step * (1 + 1e-12)) | (gap <= 1e-5 * np.abs(want_h).max())), (what, float(gap.max()))
    frac = float(diff.mean())
    assert frac <= H_DIFF_MAX, (what, frac)
    return frac, float(margin[diff].max())


# The loss bar (the reading of "objective to 1e-3"): the kernel's in-kernel loss of its own W_hat is
# the trace of that W_hat under the oracle's H_comb to 1e-3 (the float32 Hessian and H_comb); and the
# GPU's objective is the oracle's to 1e-3, except that a row which parts ways with the oracle at a
# certified rounding-boundary flip follows another, equally valid rounding path: such a row's own
# term may take any value between the two runs' (its allowance is the larger of the two).
LOSS_REL = 1e-3


def row_losses(W, W_hat, H):
    """Per-row terms of tr[(W_hat - W) H (W_hat - W)^T], float64."""
    D = np.asarray(W_hat, np.float64) - np.asarray(W, np.float64)
    return np.einsum("rj,rj->r", D @ np.asarray(H, np.float64), D)


def check_loss(got_loss, W, got_W_hat, got_codes, got_zeros, want, H, what):
    """One matrix's loss against the oracle's GPTQ result `want` (codes, zeros, W_hat) under H."""
    lg, lo = row_losses(W, got_W_hat, H), row_losses(W, want["W_hat"], H)
    assert abs(got_loss - lg.sum()) <= LOSS_REL * lg.sum(), (what, got_loss, lg.sum())
    differ = (np.asarray(got_codes) != want["codes"]).any(1) | (np.asarray(got_zeros) != want["zeros"]).any(1)
    allow = LOSS_REL * lo.sum() + np.maximum(lg, lo)[differ].sum()
    assert abs(lg.sum() - lo.sum()) <= allow, (what, lg.sum(), lo.sum(), int(differ.sum()))
    return float(lg.sum() - lo.sum()) / lo.sum()
