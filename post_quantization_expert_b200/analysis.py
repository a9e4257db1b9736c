"""Cross-layer routing divergence and the Calibration Hessian Error of quantized experts, on the GPU.

The CLHA page, section 4, compares per-layer calibration (PLIC) with CLHA on the calibration tokens
and on held-out tokens (the Calibration Hessian Error), and sharpens the router to raise the
cross-layer routing divergence; section 5 ties CLHA's gains to that divergence. Both measurements
are calls of the library:
  divergence   clha_routing_divergence on an accumulator's token counts: the total-variation
               distance of two layers' expert frequencies (the pages give no formula; this is the
               reading);
  CHE          clha_aggregate (undamped H_comb of some weighting of collected Hessians) -> clha_loss
               of each expert's quantized weights: on the calibration side the hook layer's own
               Hessian (alpha = (1, 0), what PLIC fits), on the test side the token-share aggregate
               of fresh tokens of every layer that shares the expert.
"""
from __future__ import annotations

import numpy as np
import torch

from . import clha as L
from .pipeline import MODES, MoEResult, MoEWeights


def routing_divergence(ctx: L.Context, acc: L.Accum, slot0: int, E: int) -> np.ndarray:
    """[n_layers, n_layers] total-variation distances of the layers' expert frequencies over the
    accumulator slots [slot0, slot0 + E) (synchronises; raises on a layer without tokens)."""
    _, counts = acc.buffers()
    tv = torch.empty((acc.n_layers, acc.n_layers), dtype=torch.float64, device=counts.device)
    L.clha_routing_divergence(ctx, counts, acc.n_layers, acc.n_slots, slot0, E, tv)
    L.clha_check(ctx)
    return tv.cpu().numpy()


def mean_pairwise(tv: np.ndarray) -> float:
    """Mean of the off-diagonal divergences (the one pair's value for a layer pair)."""
    n = tv.shape[0]
    if n < 2:
        return 0.0
    return float(tv[~np.eye(n, dtype=bool)].mean())


class HessianError:
    """Per-expert loss tr[(W_hat - W) H_comb (W_hat - W)^T] (CLHA page §2.1) of quantized experts under
    an aggregate of the Hessians a MoECalibration (or any object with its accumulators acc_in, acc_dn
    and acc_sdn) has collected. Owns the aggregate buffers; one call per (accumulators, weighting)."""

    def __init__(self, ctx: L.Context, E: int, d_model: int, d_ff: int, n_shared: int = 0, shared_dff: int = 0):
        self.ctx, self.E, self.d_model, self.d_ff = ctx, E, d_model, d_ff
        self.n_shared, self.shared_dff = n_shared, shared_dff
        f32 = dict(dtype=torch.float32, device=torch.device("cuda", ctx.device))
        self.Hc_in = torch.empty((E, d_model, d_model), **f32)
        self.Hd_in = torch.empty_like(self.Hc_in)
        self.Hc_dn = torch.empty((E, d_ff, d_ff), **f32)
        self.Hd_dn = torch.empty_like(self.Hc_dn)
        if n_shared:
            self.Hc_sin = torch.empty((1, d_model, d_model), **f32)
            self.Hd_sin = torch.empty_like(self.Hc_sin)
            self.Hc_sdn = torch.empty((n_shared, shared_dff, shared_dff), **f32)
            self.Hd_sdn = torch.empty_like(self.Hc_sdn)

    def __call__(self, cal, w: MoEWeights, r: MoEResult, mode: str = "rt", alpha=None) -> dict:
        """{"routed": [E] gate + up + down losses, "shared": [n_shared] the same for the always-active
        experts} under the `mode` (alpha for "explicit") aggregate of cal's accumulators."""
        ctx, E, dm, dff = self.ctx, self.E, self.d_model, self.d_ff
        # the damped aggregate is scratch (only H_comb is scored); an expert without tokens scores 0
        m, dmp = MODES[mode] | L.AGG_EMPTY_IDENTITY, 0.01
        L.clha_aggregate(ctx, cal.acc_in, 0, E, m, alpha, dmp, self.Hc_in, self.Hd_in)
        L.clha_aggregate(ctx, cal.acc_dn, 0, E, m, alpha, dmp, self.Hc_dn, self.Hd_dn)
        gu = L.clha_loss(ctx, w.Wgu, r.qgu.W_hat, self.Hc_in, E, 2 * E, dff, dm)
        dn = L.clha_loss(ctx, w.Wd, r.qd.W_hat, self.Hc_dn, E, E, dm, dff)
        out = {"routed": gu[:E] + gu[E:] + dn, "shared": np.zeros(0)}
        ns, sdff = self.n_shared, self.shared_dff
        if ns:
            L.clha_aggregate(ctx, cal.acc_in, E, 1, m, alpha, dmp, self.Hc_sin, self.Hd_sin)
            L.clha_aggregate(ctx, cal.acc_sdn, 0, ns, m, alpha, dmp, self.Hc_sdn, self.Hd_sdn)
            sgu = L.clha_loss(ctx, w.Sgu, r.sgu.W_hat, self.Hc_sin, 1, 2 * ns, sdff, dm)
            sdn = L.clha_loss(ctx, w.Sd, r.sd.W_hat, self.Hc_sdn, ns, ns, dm, sdff)
            out["shared"] = sgu[:ns] + sgu[ns:] + sdn
        return out
