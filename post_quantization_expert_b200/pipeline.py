"""CLHA calibration of one weight group on the GPU, as a sequence of C-ABI calls.

This module only orders calls and owns device buffers; every step runs in libclha.so:
  collection   clha_route_topk -> clha_gather -> clha_collect (expert inputs)
               -> clha_expert_act -> clha_collect (down-projection inputs)       per layer
               (or, fused: clha_gather's permutation only -> clha_collect_gathered, which reads
               the routed rows from X by TMA gather4 -> clha_expert_act_gathered)
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

MODES = {"rt": L.ALPHA_ROUTING, "eq": L.ALPHA_EQUAL, "explicit": L.ALPHA_EXPLICIT, "sum": L.ALPHA_SUM}


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


def _halves(q: QuantOut, n: int):
    """Views of the first and second n problems of a stacked [2n] result (gate, then up)."""
    return (QuantOut(q.codes[:n], q.scales[:n], q.zeros[:n], q.W_hat[:n]),
            QuantOut(q.codes[n:], q.scales[n:], q.zeros[n:], q.W_hat[n:]))


class DenseCalibration:
    """One weight W [d_out, d_in] shared by n_layers layers (no routing)."""

    def __init__(self, ctx: L.Context, d_out: int, d_in: int, n_layers: int, bits: int, damp_frac: float = 0.01,
                 timer=NO_TIMER, keep_hcomb: bool = True, factor_form: int = L.FACTOR_BLOCK_CHOL):
        """keep_hcomb=False: the undamped aggregate is not written (GPTQ and its in-kernel loss need only
        the damped one and lambda). factor_form: what self.U holds, F (the block-scaled Cholesky factor
        of H_d, the default: half the factor's work) or U (H_d^-1 = U^T U)."""
        self.ctx, self.d_out, self.d_in, self.n_layers, self.bits, self.damp = ctx, d_out, d_in, n_layers, bits, damp_frac
        self.form = factor_form
        self.timer = timer
        self.dev = dev = torch.device("cuda", ctx.device)
        self.acc = L.Accum(ctx, d_in, n_layers, 1)
        self.H_d = torch.empty((1, d_in, d_in), dtype=torch.float32, device=dev)
        self.H_comb = torch.empty_like(self.H_d) if keep_hcomb else None
        self.U = torch.empty_like(self.H_d)
        self.q = _quant_buffers(1, d_out, d_in, dev)
        self.lam = torch.empty(1, dtype=torch.float64, device=dev)
        self.loss_dev = torch.empty(1, dtype=torch.float64, device=dev)

    def reset(self):
        L.clha_accum_zero(self.ctx, self.acc)

    def collect(self, layer: int, X: torch.Tensor):
        with self.timer.span("hessian"):
            L.clha_collect(self.ctx, self.acc, layer, X, X.shape[0], self.d_in, None, 1, 0)

    def quantize(self, W: torch.Tensor, mode: str = "rt", alpha=None, with_loss: bool = True, want_host=False,
                 read_loss: bool = True):
        """Aggregate, factor and GPTQ (with the in-kernel loss). read_loss=False leaves the loss in
        self.loss_dev (nothing synchronises)."""
        t = self.timer
        with t.span("aggregate"):
            host = L.clha_aggregate(self.ctx, self.acc, 0, 1, MODES[mode], alpha, self.damp, self.H_comb, self.H_d,
                                    want_host=want_host, lambda_dev=self.lam)
        with t.span("factor"):
            L.clha_factor_as(self.ctx, self.form, self.H_d, 1, self.d_in, self.U)
        with t.span("gptq"):
            L.clha_quantize(self.ctx, self.U, 1, W, 1, self.d_out, self.d_in, self.bits, self.q.codes, self.q.scales,
                            self.q.zeros, self.q.W_hat, lam=self.lam if with_loss else None,
                            loss=self.loss_dev if with_loss else None, form=self.form)
        if with_loss and read_loss:
            self.q.loss = self.loss_dev.cpu().numpy()
        return host

    def columns(self) -> int:
        return self.d_in


@dataclass
class MoEWeights:
    """Stacked expert weights of one layer group: Wgu [2E, d_ff, d_model] holds every gate then every
    up projection (Wg, Wu are its halves), Wd [E, d_model, d_ff]; Sgu / Sd the same for the
    always-active experts."""
    Wgu: torch.Tensor
    Wd: torch.Tensor
    Sgu: torch.Tensor | None = None
    Sd: torch.Tensor | None = None

    @property
    def Wg(self):
        return self.Wgu[: self.Wgu.shape[0] // 2]

    @property
    def Wu(self):
        return self.Wgu[self.Wgu.shape[0] // 2:]

    @property
    def Sg(self):
        return None if self.Sgu is None else self.Sgu[: self.Sgu.shape[0] // 2]

    @property
    def Su(self):
        return None if self.Sgu is None else self.Sgu[self.Sgu.shape[0] // 2:]


@dataclass
class MoEResult:
    """GPTQ outputs of one weighting: gate and up stacked [2E] (qg, qu are views), down [E], and the
    always-active experts' counterparts."""
    qgu: QuantOut
    qg: QuantOut
    qu: QuantOut
    qd: QuantOut
    sgu: QuantOut | None = None
    sg: QuantOut | None = None
    su: QuantOut | None = None
    sd: QuantOut | None = None

    def expert_loss(self) -> np.ndarray:
        """Per routed expert: loss(gate) + loss(up) + loss(down) under the undamped H_comb."""
        return self.qg.loss + self.qu.loss + self.qd.loss


class MoECalibration:
    """Routed experts (top-k of E) plus always-active shared experts of one weight-sharing group.

    quantize() takes one or several weightings; their aggregated Hessians are factored together in
    one batched call per Hessian kind, and each weighting keeps its own results (self.res[mode])."""

    def __init__(self, ctx: L.Context, n_layers: int, max_tokens: int, E: int, k: int, d_model: int, d_ff: int,
                 n_shared: int = 0, shared_dff: int = 0, bits_routed: int = 2, bits_shared: int = 3,
                 damp_frac: float = 0.01, timer=NO_TIMER, modes=("rt",), keep_hcomb: bool = False,
                 unrouted_rtn: bool = True, fused_gather: bool = False, factor_form: int = L.FACTOR_BLOCK_CHOL):
        """unrouted_rtn: an expert whose weighted Hessian aggregate is empty (never routed, or, for
        explicit alpha, never routed in the weighted layers) is quantized by round to nearest
        (H_d = I, loss 0) instead of failing. fused_gather: the expert inputs are read straight from
        the layer's X through the routing permutation (TMA gather4 in the Gram kernel, indexed rows
        in the activation) instead of from a packed copy (bf16 X only). Same results; off by
        default because four-row gather requests feed the tensor cores more slowly than the packed
        copy costs (the Hessian phase of the E16 pair: 0.41 ms against 0.16 ms plus a 0.03 ms copy).
        factor_form: what the U_* buffers hold, F (the block-scaled Cholesky factor of each H_d, the
        default) or U (H_d^-1 = U^T U)."""
        self.ctx, self.n_layers, self.E, self.k = ctx, n_layers, E, k
        self.form = factor_form
        self.agg_flag = L.AGG_EMPTY_IDENTITY if unrouted_rtn else 0
        self.fused_gather = fused_gather
        self.timer = timer
        self.d_model, self.d_ff, self.n_shared, self.shared_dff = d_model, d_ff, n_shared, shared_dff
        self.bits_routed, self.bits_shared, self.damp = bits_routed, bits_shared, damp_frac
        dev = self.dev = torch.device("cuda", ctx.device)
        self.P = L.clha_packed_rows(max_tokens, k, E)
        self.ids = torch.empty((max_tokens, k), dtype=torch.int32, device=dev)
        self.counts = torch.empty((n_layers, E), dtype=torch.int32, device=dev)
        self.Xp = None if fused_gather else torch.empty((self.P, d_model), dtype=torch.bfloat16, device=dev)
        self.perm = torch.empty(self.P, dtype=torch.int32, device=dev)
        self.hp = torch.empty((self.P, d_ff), dtype=torch.bfloat16, device=dev)
        self.seg = torch.empty((n_layers, 2 * E + 1), dtype=torch.int64, device=dev)
        # slots of the input accumulator: 0..E-1 routed, E the shared experts' common input
        self.acc_in = L.Accum(ctx, d_model, n_layers, E + (1 if n_shared else 0))
        self.acc_dn = L.Accum(ctx, d_ff, n_layers, E)
        if n_shared:
            self.hs = torch.empty((max_tokens, shared_dff), dtype=torch.bfloat16, device=dev)
            self.acc_sdn = L.Accum(ctx, shared_dff, n_layers, n_shared)
        self.modes = tuple(modes)
        nm = len(self.modes)
        f32 = dict(dtype=torch.float32, device=dev)
        # [weighting][expert] Hessians and factors; the undamped aggregates only on request (GPTQ and
        # its in-kernel loss need only the damped one and lambda)
        hc = (lambda shape: torch.empty(shape, **f32)) if keep_hcomb else (lambda shape: None)
        self.Hd_in = torch.empty((nm * E, d_model, d_model), **f32)
        self.Hc_in = hc(self.Hd_in.shape)
        self.U_in = torch.empty_like(self.Hd_in)
        self.Hd_dn = torch.empty((nm * E, d_ff, d_ff), **f32)
        self.Hc_dn = hc(self.Hd_dn.shape)
        self.U_dn = torch.empty_like(self.Hd_dn)
        if n_shared:
            self.Hd_sin = torch.empty((nm, d_model, d_model), **f32)
            self.Hc_sin = hc(self.Hd_sin.shape)
            self.U_sin = torch.empty_like(self.Hd_sin)
            self.Hd_sdn = torch.empty((nm * n_shared, shared_dff, shared_dff), **f32)
            self.Hc_sdn = hc(self.Hd_sdn.shape)
            self.U_sdn = torch.empty_like(self.Hd_sdn)
        f64 = dict(dtype=torch.float64, device=dev)
        self.lam_in = torch.empty(nm * E, **f64)
        self.lam_dn = torch.empty(nm * E, **f64)
        self.lam_sin = torch.empty(max(nm, 1), **f64)
        self.lam_sdn = torch.empty(max(nm * n_shared, 1), **f64)
        # per weighting: [gate E][up E][down E][shared gate][shared up][shared down]
        self.nloss = 3 * E + 3 * n_shared
        self.loss_dev = torch.empty((nm, self.nloss), **f64)
        self.res = {}
        for mode in self.modes:
            qgu = _quant_buffers(2 * E, d_ff, d_model, dev)
            r = MoEResult(qgu, *_halves(qgu, E), _quant_buffers(E, d_model, d_ff, dev))
            if n_shared:
                r.sgu = _quant_buffers(2 * n_shared, shared_dff, d_model, dev)
                r.sg, r.su = _halves(r.sgu, n_shared)
                r.sd = _quant_buffers(n_shared, d_model, shared_dff, dev)
            self.res[mode] = r
        self._last = self.res[self.modes[0]]

    # results of the most recent weighting (convenience for single-weighting callers)
    qgu = property(lambda self: self._last.qgu)
    qg = property(lambda self: self._last.qg)
    qu = property(lambda self: self._last.qu)
    qd = property(lambda self: self._last.qd)
    sgu = property(lambda self: self._last.sgu)
    sg = property(lambda self: self._last.sg)
    su = property(lambda self: self._last.su)
    sd = property(lambda self: self._last.sd)

    def reset(self):
        for a in (self.acc_in, self.acc_dn) + ((self.acc_sdn,) if self.n_shared else ()):
            L.clha_accum_zero(self.ctx, a)

    # ------------------------------------------------------------------ phase 1
    def collect(self, layer: int, X: torch.Tensor, logits: torch.Tensor, w: MoEWeights, before_act=None):
        """Phase 1 for one layer's tokens. before_act (optional) is called once the steps that need only
        X and the logits are queued, before the first that reads the weights (a caller copying the
        weights in on another stream makes the compute stream wait there)."""
        ctx, E, k, n, t = self.ctx, self.E, self.k, X.shape[0], self.timer
        ids = self.ids[:n]
        seg = self.seg[layer]
        with t.span("route"):
            L.clha_route_topk(ctx, logits, n, E, k, ids, self.counts[layer])
        fused = self.fused_gather and X.dtype == torch.bfloat16
        if not fused and self.Xp is None:
            self.Xp = torch.empty((self.P, self.d_model), dtype=X.dtype, device=self.dev)
        with t.span("gather"):
            L.clha_gather(ctx, X, n, self.d_model, ids, k, E, None if fused else self.Xp, self.P, seg,
                          self.perm if fused else None)
        with t.span("hessian"):
            if fused:
                L.clha_collect_gathered(ctx, self.acc_in, layer, X, n, self.d_model, self.perm, seg, E, 0)
            else:
                L.clha_collect(ctx, self.acc_in, layer, self.Xp, self.P, self.d_model, seg, E, 0)
            if self.n_shared:
                L.clha_collect(ctx, self.acc_in, layer, X, n, self.d_model, None, 1, E)
        if before_act is not None:
            before_act()
        with t.span("act"):
            if fused:
                L.clha_expert_act_gathered(ctx, X, n, self.d_model, self.perm, self.P, seg, E, w.Wg, w.Wu, self.d_ff,
                                           self.hp)
            else:
                L.clha_expert_act(ctx, self.Xp, self.P, self.d_model, seg, E, w.Wg, w.Wu, self.d_ff, self.hp)
        with t.span("hessian"):
            L.clha_collect(ctx, self.acc_dn, layer, self.hp, self.P, self.d_ff, seg, E, 0)
        if self.n_shared:
            hs = self.hs[:n]
            for i in range(self.n_shared):
                with t.span("act"):
                    L.clha_expert_act(ctx, X, n, self.d_model, None, 1, w.Sg[i], w.Su[i], self.shared_dff, hs)
                with t.span("hessian"):
                    L.clha_collect(ctx, self.acc_sdn, layer, hs, n, self.shared_dff, None, 1, i)

    # ------------------------------------------------------------------ phases 2 and 3
    def quantize(self, w: MoEWeights, modes=None, alpha=None, with_loss: bool = True, on_output=None,
                 read_loss: bool = True):
        """Aggregate, factor, GPTQ and score for each weighting in `modes` (a name or a tuple of the
        weightings given at construction; default all of them). on_output(mode, part) (optional) is
        called after each GPTQ call is queued, part one of "gu", "d", "sgu", "sd" (the QuantOut fields
        of self.res[mode]), so that a caller can start copying those outputs while the next call runs.
        read_loss=False leaves the losses in self.loss_dev (nothing synchronises) instead of reading
        them into the results."""
        notify = on_output if on_output is not None else (lambda mode, part: None)
        if modes is None:
            modes = self.modes
        if isinstance(modes, str):
            modes = (modes,)
        ctx, E, dm, dff, t = self.ctx, self.E, self.d_model, self.d_ff, self.timer
        ns, sdff = self.n_shared, self.shared_dff
        idx = [self.modes.index(m) for m in modes]
        opt = lambda h, sl: None if h is None else h[sl]
        with t.span("aggregate"):
            for i, m in zip(idx, modes):
                es, ss = slice(i * E, (i + 1) * E), slice(i * ns, (i + 1) * ns)
                am = MODES[m] | self.agg_flag
                L.clha_aggregate(ctx, self.acc_in, 0, E, am, alpha, self.damp, opt(self.Hc_in, es),
                                 self.Hd_in[es], lambda_dev=self.lam_in[es])
                L.clha_aggregate(ctx, self.acc_dn, 0, E, am, alpha, self.damp, opt(self.Hc_dn, es),
                                 self.Hd_dn[es], lambda_dev=self.lam_dn[es])
                if ns:
                    L.clha_aggregate(ctx, self.acc_in, E, 1, am, alpha, self.damp,
                                     opt(self.Hc_sin, slice(i, i + 1)), self.Hd_sin[i:i + 1],
                                     lambda_dev=self.lam_sin[i:i + 1])
                    L.clha_aggregate(ctx, self.acc_sdn, 0, ns, am, alpha, self.damp, opt(self.Hc_sdn, ss),
                                     self.Hd_sdn[ss], lambda_dev=self.lam_sdn[ss])
        # one batched factor per Hessian kind over every requested weighting (contiguous runs)
        lo, hi = min(idx), max(idx) + 1
        contiguous = sorted(idx) == list(range(lo, hi))
        runs = [(lo, hi)] if contiguous else [(i, i + 1) for i in idx]
        with t.span("factor"):   # one task-graph launch per run: routed in/down (+ shared in/down)
            for a, b in runs:
                groups = [(self.Hd_in[a * E:b * E], (b - a) * E, dm, self.U_in[a * E:b * E]),
                          (self.Hd_dn[a * E:b * E], (b - a) * E, dff, self.U_dn[a * E:b * E])]
                if ns:
                    groups += [(self.Hd_sin[a:b], b - a, dm, self.U_sin[a:b]),
                               (self.Hd_sdn[a * ns:b * ns], (b - a) * ns, sdff, self.U_sdn[a * ns:b * ns])]
                L.clha_factor_groups(ctx, groups, self.form)
        br, bs = self.bits_routed, self.bits_shared
        for i, m in zip(idx, modes):
            r = self.res[m]
            es, ss = slice(i * E, (i + 1) * E), slice(i * ns, (i + 1) * ns)
            lb = self.loss_dev[i]
            opt = ((lambda lam, lo: dict(lam=lam, loss=lo, form=self.form)) if with_loss else
                   (lambda lam, lo: dict(form=self.form)))
            with t.span("gptq"):
                q = r.qgu
                L.clha_quantize(ctx, self.U_in[es], E, w.Wgu, 2 * E, dff, dm, br, q.codes, q.scales, q.zeros, q.W_hat,
                                **opt(self.lam_in[es], lb[0:2 * E]))
                notify(m, "gu")
                L.clha_quantize(ctx, self.U_dn[es], E, w.Wd, E, dm, dff, br, r.qd.codes, r.qd.scales, r.qd.zeros,
                                r.qd.W_hat, **opt(self.lam_dn[es], lb[2 * E:3 * E]))
                notify(m, "d")
                if ns:
                    q = r.sgu
                    L.clha_quantize(ctx, self.U_sin[i:i + 1], 1, w.Sgu, 2 * ns, sdff, dm, bs, q.codes, q.scales,
                                    q.zeros, q.W_hat, **opt(self.lam_sin[i:i + 1], lb[3 * E:3 * E + 2 * ns]))
                    notify(m, "sgu")
                    L.clha_quantize(ctx, self.U_sdn[ss], ns, w.Sd, ns, dm, sdff, bs, r.sd.codes, r.sd.scales,
                                    r.sd.zeros, r.sd.W_hat, **opt(self.lam_sdn[ss], lb[3 * E + 2 * ns:]))
                    notify(m, "sd")
            self._last = r
        if with_loss and read_loss:      # one read of every weighting's losses
            host = self.loss_dev.cpu().numpy()
            for i, m in zip(idx, modes):
                r, h = self.res[m], host[i]
                r.qg.loss, r.qu.loss, r.qd.loss = h[:E], h[E:2 * E], h[2 * E:3 * E]
                if ns:
                    r.sg.loss, r.su.loss, r.sd.loss = h[3 * E:3 * E + ns], h[3 * E + ns:3 * E + 2 * ns], h[3 * E + 2 * ns:]

    def expert_loss(self) -> np.ndarray:
        """Per routed expert loss of the most recent weighting."""
        return self._last.expert_loss()

    def columns(self) -> int:
        """Weight columns quantized per weighting."""
        c = self.E * (2 * self.d_model + self.d_ff)
        if self.n_shared:
            c += self.n_shared * (2 * self.d_model + self.shared_dff)
        return c


def stack_weights(wl, device) -> MoEWeights:
    """MoEWeights from per-expert (Wg, Wu, Wd) lists (routed, and optionally shared)."""
    routed, shared = wl

    def gu(ws):
        return torch.stack([w[0] for w in ws] + [w[1] for w in ws]).to(device).contiguous()

    def dn(ws):
        return torch.stack([w[2] for w in ws]).to(device).contiguous()

    if shared:
        return MoEWeights(gu(routed), dn(routed), gu(shared), dn(shared))
    return MoEWeights(gu(routed), dn(routed))


PART_FIELDS = {"gu": "qgu", "d": "qd", "sgu": "sgu", "sd": "sd"}   # on_output part -> MoEResult field


class HostStep:
    """MoE calibration steps from pinned host memory to pinned host memory, the copies overlapped with
    the compute. Host→device copies run on an input stream in the order the compute needs them:
    layer 0's tokens and logits, the gate/up weights (the first step that reads weights is layer 0's
    expert activation), the other layers' tokens, then the down and always-active weights; the
    compute stream (the context's) waits on an event before each first use. Each GPTQ call's codes,
    scales and zeros, and at the end the losses, go back on an output stream as soon as the call is
    queued, while the compute goes on. The device copies of the inputs come in `n_sets` sets used in
    turn, so with two sets the next step's inputs are copied while the current step computes (a set
    is refilled once the step that last used it has finished; outputs are rewritten only after the
    previous step's copies of them are done). run() only queues work: nothing synchronises.
    """

    def __init__(self, cal: MoECalibration, x_shapes, logit_shapes, w_host: MoEWeights, x_dtype=torch.bfloat16,
                 n_sets: int = 2):
        self.cal = cal
        dev = cal.dev
        self.inp = torch.cuda.Stream(device=dev)
        self.out = torch.cuda.Stream(device=dev)
        like = lambda t: None if t is None else torch.empty(t.shape, dtype=t.dtype, device=dev)
        self.sets = []
        for _ in range(n_sets):
            self.sets.append(dict(
                X=[torch.empty(sh, dtype=x_dtype, device=dev) for sh in x_shapes],
                L=[torch.empty(sh, dtype=torch.float32, device=dev) for sh in logit_shapes],
                w=MoEWeights(like(w_host.Wgu), like(w_host.Wd), like(w_host.Sgu), like(w_host.Sd)),
                free=None))                      # event: the last step that used this set has finished
        self.step = 0
        self.outputs_copied = None               # event: the previous step's outputs are on the host

    def run(self, hX, hL, hW: MoEWeights, hout: dict, modes=None, alpha=None, hloss=None):
        """hX, hL: per-layer pinned host tokens and logits; hW: pinned host weights; hout[mode][part]
        = (codes, scales, zeros) pinned host tensors for the parts ("gu", "d", "sgu", "sd") to bring
        back; hloss (optional): pinned host float64 tensor shaped like the calibration's loss_dev.
        Everything is queued; the caller synchronises with the context's stream."""
        cal, comp = self.cal, self.cal.ctx.stream
        st = self.sets[self.step % len(self.sets)]
        self.step += 1
        ev = torch.cuda.Event
        if st["free"] is not None:
            self.inp.wait_event(st["free"])      # the step that last read this set is done
        ev_in, ev_gu, ev_rest = [], ev(), ev()
        w = st["w"]
        with torch.cuda.stream(self.inp):
            for l, (dx, dl, hx, hl) in enumerate(zip(st["X"], st["L"], hX, hL)):
                dx.copy_(hx, non_blocking=True)
                dl.copy_(hl, non_blocking=True)
                ev_in.append(ev())
                ev_in[-1].record(self.inp)
                if l == 0:
                    w.Wgu.copy_(hW.Wgu, non_blocking=True)
                    if hW.Sgu is not None:
                        w.Sgu.copy_(hW.Sgu, non_blocking=True)
                    ev_gu.record(self.inp)
            w.Wd.copy_(hW.Wd, non_blocking=True)
            if hW.Sd is not None:
                w.Sd.copy_(hW.Sd, non_blocking=True)
            ev_rest.record(self.inp)
        cal.reset()
        for l in range(len(st["X"])):
            comp.wait_event(ev_in[l])
            n = hX[l].shape[0]
            cal.collect(l, st["X"][l][:n], st["L"][l][:n], w,
                        before_act=(lambda: comp.wait_event(ev_gu)) if l == 0 else None)
        comp.wait_event(ev_rest)
        if self.outputs_copied is not None:
            comp.wait_event(self.outputs_copied)   # the previous step's outputs have left the device

        def on_output(mode, part):
            outs = hout.get(mode, {}).get(part)
            if outs is None:
                return
            ready = ev()
            ready.record(comp)
            self.out.wait_event(ready)
            q = getattr(cal.res[mode], PART_FIELDS[part])
            with torch.cuda.stream(self.out):
                for h, d in zip(outs, (q.codes, q.scales, q.zeros)):
                    h.copy_(d, non_blocking=True)

        cal.quantize(w, modes, alpha, on_output=on_output, read_loss=hloss is None)
        st["free"] = ev()
        st["free"].record(comp)
        if hloss is not None:
            self.out.wait_event(st["free"])
            with torch.cuda.stream(self.out):
                hloss.copy_(cal.loss_dev, non_blocking=True)
        done = ev()
        done.record(self.out)
        self.outputs_copied = done

    def join(self):
        """Make the context's stream wait for every copy queued so far (the outputs and losses of the
        last step included), so that an event recorded on it after this covers them."""
        if self.outputs_copied is not None:
            self.cal.ctx.stream.wait_event(self.outputs_copied)


class DenseHostStep:
    """Dense calibration steps (one weight shared by several layers) from pinned host memory to pinned
    host memory. Each layer's tokens, then the weight, go to the device on an input stream; the
    compute stream (the context's) collects a layer as soon as its tokens have arrived, so the
    copies of later layers overlap the Gram work of earlier ones. The device copies of the inputs
    come in `n_sets` sets used in turn: with two, the next step's inputs cross PCIe while this step
    aggregates, factors and quantizes. Codes, scales, zeros and the loss go back on an output stream.
    run() only queues work: nothing synchronises."""

    def __init__(self, cal: DenseCalibration, x_shapes, x_dtype, w_shape, w_dtype, n_sets: int = 2):
        self.cal = cal
        dev = cal.dev
        self.inp = torch.cuda.Stream(device=dev)
        self.out = torch.cuda.Stream(device=dev)
        self.sets = [dict(X=[torch.empty(sh, dtype=x_dtype, device=dev) for sh in x_shapes],
                          W=torch.empty(w_shape, dtype=w_dtype, device=dev), free=None) for _ in range(n_sets)]
        self.step = 0
        self.outputs_copied = None

    def run(self, hX, hW, hout, hloss=None, mode: str = "rt"):
        """hX: per-layer pinned host tokens; hW: pinned host weight; hout = (codes, scales, zeros)
        pinned host tensors shaped like cal.q's; hloss (optional): pinned float64 [1]."""
        cal, comp = self.cal, self.cal.ctx.stream
        st = self.sets[self.step % len(self.sets)]
        self.step += 1
        ev = torch.cuda.Event
        if st["free"] is not None:
            self.inp.wait_event(st["free"])
        ev_x, ev_w = [], ev()
        with torch.cuda.stream(self.inp):
            for dx, hx in zip(st["X"], hX):
                dx.copy_(hx, non_blocking=True)
                ev_x.append(ev())
                ev_x[-1].record(self.inp)
            st["W"].copy_(hW, non_blocking=True)
            ev_w.record(self.inp)
        cal.reset()
        for l, dx in enumerate(st["X"]):
            comp.wait_event(ev_x[l])
            cal.collect(l, dx)
        comp.wait_event(ev_w)
        if self.outputs_copied is not None:
            comp.wait_event(self.outputs_copied)
        cal.quantize(st["W"], mode, read_loss=hloss is None)
        st["free"] = ev()
        st["free"].record(comp)
        self.out.wait_event(st["free"])
        with torch.cuda.stream(self.out):
            for h, d in zip(hout, (cal.q.codes, cal.q.scales, cal.q.zeros)):
                h.copy_(d, non_blocking=True)
            if hloss is not None:
                hloss.copy_(cal.loss_dev, non_blocking=True)
        done = ev()
        done.record(self.out)
        self.outputs_copied = done

    def join(self):
        """Make the context's stream wait for every copy queued so far."""
        if self.outputs_copied is not None:
            self.cal.ctx.stream.wait_event(self.outputs_copied)


class EPMQCalibration:
    """E-PMQ of one merged linear layer (the E-PMQ page, section 2): the K source experts' calibration
    activations are collected as the K layers of one accumulator slot; quantize() forms
    H = sum_i S_i + lambda I (aggregation in the plain-sum weighting), factors it, computes the target
    W* = (lambda W_m + sum_i W_i S_i) H^-1 and runs GPTQ of W* under H."""

    def __init__(self, ctx: L.Context, K: int, d_out: int, d: int, bits: int, damp_frac: float = 0.01):
        self.ctx, self.K, self.d_out, self.d, self.bits, self.damp = ctx, K, d_out, d, bits, damp_frac
        dev = torch.device("cuda", ctx.device)
        self.acc = L.Accum(ctx, d, K, 1)
        f32 = dict(dtype=torch.float32, device=dev)
        self.H = torch.empty((1, d, d), **f32)       # sum_i S_i (undamped)
        self.H_d = torch.empty((1, d, d), **f32)     # + lambda I
        self.U = torch.empty((1, d, d), **f32)
        self.lam = torch.empty(1, dtype=torch.float64, device=dev)
        self.W_target = torch.empty((d_out, d), **f32)
        self.q = _quant_buffers(1, d_out, d, dev)

    def collect(self, i: int, X_i: torch.Tensor):
        """Activations of source expert i's calibration subset, [n_i, d] (bf16 or f32)."""
        L.clha_collect(self.ctx, self.acc, i, X_i, X_i.shape[0], self.d)

    def quantize(self, W_src: torch.Tensor, W_m: torch.Tensor):
        """W_src [K, d_out, d], W_m [d_out, d] (same dtype). Results in self.q (codes, scales, zeros,
        W_hat) and self.W_target."""
        ctx = self.ctx
        L.clha_aggregate(ctx, self.acc, 0, 1, L.ALPHA_SUM, None, self.damp, self.H, self.H_d, lambda_dev=self.lam)
        L.clha_factor(ctx, self.H_d, 1, self.d, self.U)
        L.clha_epmq_target(ctx, self.acc, 0, W_src, W_m, self.d_out, self.U, self.lam, self.W_target)
        q = self.q
        L.clha_quantize(ctx, self.U, 1, self.W_target, 1, self.d_out, self.d, self.bits, q.codes, q.scales, q.zeros,
                        q.W_hat)
        return q
