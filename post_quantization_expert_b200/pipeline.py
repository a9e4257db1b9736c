"""CLHA calibration of one weight group on the GPU, as a sequence of C-ABI calls.

This module only orders calls and owns device buffers; every step runs in libclha.so:
  collection   clha_route_topk -> clha_gather -> clha_collect (expert inputs)
               -> clha_expert_act -> clha_collect (down-projection inputs)       per layer
  aggregation  clha_aggregate (alpha, H_comb, damping)                            per weighting
  quantization clha_factor -> clha_quantize (gate, up share a factor) -> clha_loss
Always-active shared experts see every token: their gate/up input Hessian is one slot shared by
all of them, and they are quantized with one more bit (CLHA-MP).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np
import torch

from . import clha as L

MODES = {"rt": L.ALPHA_ROUTING, "eq": L.ALPHA_EQUAL, "explicit": L.ALPHA_EXPLICIT}


class PhaseTimer:
    """CUDA events around each call, per phase name, on the context's stream (measurement only)."""

    def __init__(self, stream: torch.cuda.Stream):
        self.stream = stream
        self.pending = []          # (name, start, end)
        self.totals = {}
        self.counts = {}
        self.enabled = True

    def span(self, name):
        timer = self

        class _Span:
            def __enter__(self_):
                if timer.enabled:
                    self_.a = torch.cuda.Event(enable_timing=True)
                    self_.a.record(timer.stream)

            def __exit__(self_, *exc):
                if timer.enabled:
                    b = torch.cuda.Event(enable_timing=True)
                    b.record(timer.stream)
                    timer.pending.append((name, self_.a, b))
        return _Span()

    def collect(self):
        """Fold finished spans into per-phase totals (ms); call after a synchronize."""
        for name, a, b in self.pending:
            self.totals[name] = self.totals.get(name, 0.0) + a.elapsed_time(b)
            self.counts[name] = self.counts.get(name, 0) + 1
        self.pending.clear()

    def reset(self):
        self.pending.clear()
        self.totals.clear()
        self.counts.clear()


class _NoTimer:
    enabled = False

    def span(self, name):
        class _S:
            def __enter__(self_):
                return None

            def __exit__(self_, *exc):
                return False
        return _S()


NO_TIMER = _NoTimer()


@dataclass
class QuantOut:
    codes: torch.Tensor
    scales: torch.Tensor
    zeros: torch.Tensor
    W_hat: torch.Tensor
    loss: np.ndarray | None = None


def _quant_buffers(batch, d_out, d_in, device):
    return QuantOut(torch.empty((batch, d_out, d_in), dtype=torch.uint8, device=device),
                    torch.empty((batch, d_out, d_in // 128), dtype=torch.float32, device=device),
                    torch.empty((batch, d_out, d_in // 128), dtype=torch.uint8, device=device),
                    torch.empty((batch, d_out, d_in), dtype=torch.float32, device=device))


class DenseCalibration:
    """One weight W [d_out, d_in] shared by n_layers layers (no routing)."""

    def __init__(self, ctx: L.Context, d_out: int, d_in: int, n_layers: int, bits: int, damp_frac: float = 0.01,
                 timer=NO_TIMER):
        self.ctx, self.d_out, self.d_in, self.n_layers, self.bits, self.damp = ctx, d_out, d_in, n_layers, bits, damp_frac
        self.timer = timer
        dev = torch.device("cuda", ctx.device)
        self.acc = L.Accum(ctx, d_in, n_layers, 1)
        self.H_comb = torch.empty((1, d_in, d_in), dtype=torch.float32, device=dev)
        self.H_d = torch.empty_like(self.H_comb)
        self.U = torch.empty_like(self.H_comb)
        self.q = _quant_buffers(1, d_out, d_in, dev)

    def reset(self):
        L.clha_accum_zero(self.ctx, self.acc)

    def collect(self, layer: int, X: torch.Tensor):
        with self.timer.span("hessian"):
            L.clha_collect(self.ctx, self.acc, layer, X, X.shape[0], self.d_in, None, 1, 0)

    def quantize(self, W: torch.Tensor, mode: str = "rt", alpha=None, with_loss: bool = True, want_host=False):
        t = self.timer
        with t.span("aggregate"):
            host = L.clha_aggregate(self.ctx, self.acc, 0, 1, MODES[mode], alpha, self.damp, self.H_comb, self.H_d,
                                    want_host=want_host)
        with t.span("factor"):
            L.clha_factor(self.ctx, self.H_d, 1, self.d_in, self.U)
        with t.span("gptq"):
            L.clha_quantize(self.ctx, self.U, 1, W, 1, self.d_out, self.d_in, self.bits, self.q.codes, self.q.scales,
                            self.q.zeros, self.q.W_hat)
        if with_loss:
            with t.span("loss"):
                self.q.loss = L.clha_loss(self.ctx, W, self.q.W_hat, self.H_comb, 1, 1, self.d_out, self.d_in)
        return host

    def columns(self) -> int:
        return self.d_in


@dataclass
class MoEWeights:
    """Stacked expert weights of one layer group: gate/up [E, d_ff, d_model], down [E, d_model, d_ff]."""
    Wg: torch.Tensor
    Wu: torch.Tensor
    Wd: torch.Tensor
    Sg: torch.Tensor | None = None   # always-active experts, [n_shared, shared_dff, d_model]
    Su: torch.Tensor | None = None
    Sd: torch.Tensor | None = None


class MoECalibration:
    """Routed experts (top-k of E) plus always-active shared experts of one weight-sharing group."""

    def __init__(self, ctx: L.Context, n_layers: int, max_tokens: int, E: int, k: int, d_model: int, d_ff: int,
                 n_shared: int = 0, shared_dff: int = 0, bits_routed: int = 2, bits_shared: int = 3,
                 damp_frac: float = 0.01, timer=NO_TIMER):
        self.ctx, self.n_layers, self.E, self.k = ctx, n_layers, E, k
        self.timer = timer
        self.d_model, self.d_ff, self.n_shared, self.shared_dff = d_model, d_ff, n_shared, shared_dff
        self.bits_routed, self.bits_shared, self.damp = bits_routed, bits_shared, damp_frac
        dev = self.dev = torch.device("cuda", ctx.device)
        self.P = L.clha_packed_rows(max_tokens, k, E)
        self.ids = torch.empty((max_tokens, k), dtype=torch.int32, device=dev)
        self.counts = torch.empty((n_layers, E), dtype=torch.int32, device=dev)
        self.Xp = torch.empty((self.P, d_model), dtype=torch.bfloat16, device=dev)
        self.hp = torch.empty((self.P, d_ff), dtype=torch.bfloat16, device=dev)
        self.seg = torch.empty((n_layers, 2 * E + 1), dtype=torch.int64, device=dev)
        # slots of the input accumulator: 0..E-1 routed, E the shared experts' common input
        self.acc_in = L.Accum(ctx, d_model, n_layers, E + (1 if n_shared else 0))
        self.acc_dn = L.Accum(ctx, d_ff, n_layers, E)
        if n_shared:
            self.hs = torch.empty((max_tokens, shared_dff), dtype=torch.bfloat16, device=dev)
            self.acc_sdn = L.Accum(ctx, shared_dff, n_layers, n_shared)
        f32 = dict(dtype=torch.float32, device=dev)
        self.Hc_in = torch.empty((E, d_model, d_model), **f32)
        self.Hd_in = torch.empty_like(self.Hc_in)
        self.U_in = torch.empty_like(self.Hc_in)
        self.Hc_dn = torch.empty((E, d_ff, d_ff), **f32)
        self.Hd_dn = torch.empty_like(self.Hc_dn)
        self.U_dn = torch.empty_like(self.Hc_dn)
        self.qg = _quant_buffers(E, d_ff, d_model, dev)
        self.qu = _quant_buffers(E, d_ff, d_model, dev)
        self.qd = _quant_buffers(E, d_model, d_ff, dev)
        if n_shared:
            self.Hc_sin = torch.empty((1, d_model, d_model), **f32)
            self.Hd_sin = torch.empty_like(self.Hc_sin)
            self.U_sin = torch.empty_like(self.Hc_sin)
            self.Hc_sdn = torch.empty((n_shared, shared_dff, shared_dff), **f32)
            self.Hd_sdn = torch.empty_like(self.Hc_sdn)
            self.U_sdn = torch.empty_like(self.Hc_sdn)
            self.sg = _quant_buffers(n_shared, shared_dff, d_model, dev)
            self.su = _quant_buffers(n_shared, shared_dff, d_model, dev)
            self.sd = _quant_buffers(n_shared, d_model, shared_dff, dev)

    def reset(self):
        for a in (self.acc_in, self.acc_dn) + ((self.acc_sdn,) if self.n_shared else ()):
            L.clha_accum_zero(self.ctx, a)

    # ------------------------------------------------------------------ phase 1
    def collect(self, layer: int, X: torch.Tensor, logits: torch.Tensor, w: MoEWeights):
        ctx, E, k, n, t = self.ctx, self.E, self.k, X.shape[0], self.timer
        ids = self.ids[:n]
        seg = self.seg[layer]
        with t.span("route"):
            L.clha_route_topk(ctx, logits, n, E, k, ids, self.counts[layer])
        with t.span("gather"):
            L.clha_gather(ctx, X, n, self.d_model, ids, k, E, self.Xp, self.P, seg)
        with t.span("hessian"):
            L.clha_collect(ctx, self.acc_in, layer, self.Xp, self.P, self.d_model, seg, E, 0)
        with t.span("act"):
            L.clha_expert_act(ctx, self.Xp, self.P, self.d_model, seg, E, w.Wg, w.Wu, self.d_ff, self.hp)
        with t.span("hessian"):
            L.clha_collect(ctx, self.acc_dn, layer, self.hp, self.P, self.d_ff, seg, E, 0)
        if self.n_shared:
            with t.span("hessian"):
                L.clha_collect(ctx, self.acc_in, layer, X, n, self.d_model, None, 1, E)
            hs = self.hs[:n]
            for i in range(self.n_shared):
                with t.span("act"):
                    L.clha_expert_act(ctx, X, n, self.d_model, None, 1, w.Sg[i], w.Su[i], self.shared_dff, hs)
                with t.span("hessian"):
                    L.clha_collect(ctx, self.acc_sdn, layer, hs, n, self.shared_dff, None, 1, i)

    # ------------------------------------------------------------------ phases 2 and 3
    def quantize(self, w: MoEWeights, mode: str = "rt", alpha=None, with_loss: bool = True):
        ctx, E, dm, dff, t = self.ctx, self.E, self.d_model, self.d_ff, self.timer
        m = MODES[mode]
        with t.span("aggregate"):
            L.clha_aggregate(ctx, self.acc_in, 0, E, m, alpha, self.damp, self.Hc_in, self.Hd_in)
        with t.span("factor"):
            L.clha_factor(ctx, self.Hd_in, E, dm, self.U_in)
        with t.span("aggregate"):
            L.clha_aggregate(ctx, self.acc_dn, 0, E, m, alpha, self.damp, self.Hc_dn, self.Hd_dn)
        with t.span("factor"):
            L.clha_factor(ctx, self.Hd_dn, E, dff, self.U_dn)
        br = self.bits_routed
        with t.span("gptq"):
            for W, q in ((w.Wg, self.qg), (w.Wu, self.qu)):
                L.clha_quantize(ctx, self.U_in, 1, W, E, dff, dm, br, q.codes, q.scales, q.zeros, q.W_hat)
            L.clha_quantize(ctx, self.U_dn, 1, w.Wd, E, dm, dff, br, self.qd.codes, self.qd.scales, self.qd.zeros,
                            self.qd.W_hat)
        if self.n_shared:
            ns, sdff, bs = self.n_shared, self.shared_dff, self.bits_shared
            with t.span("aggregate"):
                L.clha_aggregate(ctx, self.acc_in, E, 1, m, alpha, self.damp, self.Hc_sin, self.Hd_sin)
            with t.span("factor"):
                L.clha_factor(ctx, self.Hd_sin, 1, dm, self.U_sin)
            with t.span("aggregate"):
                L.clha_aggregate(ctx, self.acc_sdn, 0, ns, m, alpha, self.damp, self.Hc_sdn, self.Hd_sdn)
            with t.span("factor"):
                L.clha_factor(ctx, self.Hd_sdn, ns, sdff, self.U_sdn)
            with t.span("gptq"):
                for W, q in ((w.Sg, self.sg), (w.Su, self.su)):
                    L.clha_quantize(ctx, self.U_sin, ns, W, ns, sdff, dm, bs, q.codes, q.scales, q.zeros, q.W_hat)
                L.clha_quantize(ctx, self.U_sdn, 1, w.Sd, ns, dm, sdff, bs, self.sd.codes, self.sd.scales,
                                self.sd.zeros, self.sd.W_hat)
        if with_loss:
            with t.span("loss"):
                self.qg.loss = L.clha_loss(ctx, w.Wg, self.qg.W_hat, self.Hc_in, 1, E, dff, dm)
                self.qu.loss = L.clha_loss(ctx, w.Wu, self.qu.W_hat, self.Hc_in, 1, E, dff, dm)
                self.qd.loss = L.clha_loss(ctx, w.Wd, self.qd.W_hat, self.Hc_dn, 1, E, dm, dff)
                if self.n_shared:
                    ns, sdff = self.n_shared, self.shared_dff
                    self.sg.loss = L.clha_loss(ctx, w.Sg, self.sg.W_hat, self.Hc_sin, ns, ns, sdff, dm)
                    self.su.loss = L.clha_loss(ctx, w.Su, self.su.W_hat, self.Hc_sin, ns, ns, sdff, dm)
                    self.sd.loss = L.clha_loss(ctx, w.Sd, self.sd.W_hat, self.Hc_sdn, 1, ns, dm, sdff)

    def expert_loss(self) -> np.ndarray:
        """Per routed expert: loss(gate) + loss(up) + loss(down) under the undamped H_comb."""
        return self.qg.loss + self.qu.loss + self.qd.loss

    def columns(self) -> int:
        """Weight columns quantized per call of quantize()."""
        c = self.E * (2 * self.d_model + self.d_ff)
        if self.n_shared:
            c += self.n_shared * (2 * self.d_model + self.shared_dff)
        return c


def stack_weights(wl, device) -> MoEWeights:
    """MoEWeights from per-expert (Wg, Wu, Wd) lists (routed, and optionally shared)."""
    routed, shared = wl
    Wg = torch.stack([w[0] for w in routed]).to(device).contiguous()
    Wu = torch.stack([w[1] for w in routed]).to(device).contiguous()
    Wd = torch.stack([w[2] for w in routed]).to(device).contiguous()
    if shared:
        return MoEWeights(Wg, Wu, Wd, torch.stack([w[0] for w in shared]).to(device).contiguous(),
                          torch.stack([w[1] for w in shared]).to(device).contiguous(),
                          torch.stack([w[2] for w in shared]).to(device).contiguous())
    return MoEWeights(Wg, Wu, Wd)
