"""The flip certification used by the GPU parity tests, on the CPU: a GPTQ run that parts ways with
the oracle only by small noise (the weights perturbed by a relative 1e-5, as rounding differences
would) has every differing row certified; a code changed where the oracle's value was far from a
boundary is not. (A uniform rescaling of W would flip nothing: GPTQ's grid scales with W.)"""
import numpy as np

import oracle as O
from helpers import FLIP_TOL, certify_codes


def _case(seed=5, d=256, rows=256, bits=4):
    g = np.random.default_rng(seed)
    A = g.standard_normal((d, 24))
    H = A @ A.T / 24 + 0.01 * np.eye(d)           # ill-conditioned: rank 24 plus a small ridge
    W = 0.02 * g.standard_normal((rows, d))
    U = O.factor(H)
    return W, U, bits


def test_rounding_only_differences_are_certified():
    W, U, bits = _case()
    want = dict(zip(("codes", "scales", "zeros", "W_hat", "margin"), O.gptq(W, U, bits, 128, margins=True)))
    noise = np.random.default_rng(99).standard_normal(W.shape)
    got = O.gptq(W * (1 + 1e-5 * noise), U, bits, 128)
    c = certify_codes(got[0], got[2], want)
    assert c["rows"] > 0, "the perturbation should flip some decision in this ill-conditioned case"
    assert c["certified"] == c["rows"] and c["worst"] <= FLIP_TOL, c


def test_a_planted_mismatch_is_not_certified():
    W, U, bits = _case(seed=6)
    want = dict(zip(("codes", "scales", "zeros", "W_hat", "margin"), O.gptq(W, U, bits, 128, margins=True)))
    codes = want["codes"].copy()
    r, j = np.unravel_index(np.argmax(want["margin"]["code"]), codes.shape)   # the safest decision
    codes[r, j] = (codes[r, j] + 1) % (2 ** bits)
    c = certify_codes(codes, want["zeros"], want)
    assert c["rows"] == 1 and c["certified"] == 0 and c["worst"] > 0.4, c
    zeros = want["zeros"].copy()
    zeros[3, 1] += 1                                  # a zero point far from its boundary
    c = certify_codes(want["codes"], zeros, want)
    assert c["rows"] == 1 and c["certified"] == (want["margin"]["zero"][3, 1] <= FLIP_TOL), c
