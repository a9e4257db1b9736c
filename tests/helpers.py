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
