"""Token-sharded collection and expert-parallel quantization over several ranks (one process per GPU).

Phase 1 of CLHA (the CLHA page, §2.2 (1)) is a sum over calibration tokens, so it shards over
tokens: every rank routes, gathers, activates and collects its own contiguous share of each layer's
tokens into its own accumulators, and one all-reduce (sum) of the Gram matrices and token counts
gives every rank the Hessians of all the tokens. Phases 2 and 3 are independent per expert: each rank
aggregates, factors and quantizes its own contiguous range of experts (the always-active experts on
rank 0), and the results are gathered at the end. The all-reduce is the only exchange on the data
path; the kernels are the single-GPU ones.

The reduction is left to the caller, so the same code runs with torch.distributed (NCCL between
GPUs, gloo on CPU) or with the ranks simulated one after another in one process. Two forms:
  * all-reduce (`dist_reduce` or `simulated_reduce` on `reduce_tensors()`): every rank receives every
    slot's full d x d sums;
  * owner exchange (`exchange()` with `dist_reduce_scatter` or `simulated_reduce_scatter`): each rank
    packs the upper triangles of its partial sums into one buffer laid out by owner (`ExchangeLayout`),
    one reduce-scatter delivers to each rank the summed triangles of only the slots it quantizes, and
    the token counts (a few integers) are all-reduced. Against the all-reduce of full matrices that
    moves a quarter of the bytes: half for the triangles, half for reduce-scatter against all-reduce.
"""
from __future__ import annotations

from typing import Callable, Sequence

import torch

from . import clha as L
from .pipeline import MoECalibration, MoEWeights, NO_TIMER


def token_range(n: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced share [start, stop) of n tokens for `rank` of `world`."""
    base, extra = divmod(n, world)
    start = rank * base + min(rank, extra)
    return start, start + base + (1 if rank < extra else 0)


def expert_range(E: int, rank: int, world: int) -> tuple[int, int]:
    """Contiguous, balanced range [e0, e1) of the E routed experts quantized by `rank`."""
    return token_range(E, rank, world)


def accum_tensors(acc) -> list[torch.Tensor]:
    """The tensors of an accumulator that the token reduction sums: Gram matrices and token counts."""
    S, counts = acc.buffers()
    return [S, counts]


def dist_reduce(tensors: Sequence[torch.Tensor], group=None):
    """Sum every tensor over the ranks of `group`, in place (NCCL on GPUs)."""
    import torch.distributed as dist
    for t in tensors:
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)


def simulated_reduce(per_rank: Sequence[Sequence[torch.Tensor]]):
    """The same reduction for ranks simulated in one process: every rank's tensor i becomes the sum
    over ranks of tensor i."""
    for group in zip(*per_rank):
        total = group[0].clone()
        for t in group[1:]:
            total += t
        for t in group:
            t.copy_(total)


def packed_floats(d: int) -> int:
    """Floats of one packed upper triangle (d(d+1)/2)."""
    return d * (d + 1) // 2


class ExchangeLayout:
    """Which accumulator slots each rank owns, and where their packed triangles sit in the exchange
    buffer. Rank r owns the routed experts [e0, e1) of expert_range (their input slots in `in` and
    their down-projection slots in `dn`); rank 0 also owns the always-active experts (input slot E
    of `in`, every slot of `sdn`). Its chunk holds, part after part, each part's matrices in (layer,
    slot) order; every chunk is padded to the longest one, so the buffer is world * chunk floats."""

    def __init__(self, E: int, world: int, n_layers: int, d_model: int, d_ff: int, n_shared: int = 0,
                 shared_dff: int = 0):
        self.world, self.E = world, E
        dims = {"in": d_model, "dn": d_ff, "sdn": shared_dff}
        self.parts = []            # per rank: [(acc, slot0, nslots, d, offset in the chunk)]
        lens = []
        for r in range(world):
            e0, e1 = expert_range(E, r, world)
            spec = [("in", e0, e1 - e0), ("dn", e0, e1 - e0)]
            if r == 0 and n_shared:
                spec += [("in", E, 1), ("sdn", 0, n_shared)]
            off, parts = 0, []
            for acc, s0, ns in spec:
                parts.append((acc, s0, ns, dims[acc], off))
                off += n_layers * ns * packed_floats(dims[acc])
            self.parts.append(parts)
            lens.append(off)
        self.n_layers = n_layers
        self.chunk = max(lens)
        self.used = lens


def dist_reduce_scatter(out: torch.Tensor, inp: torch.Tensor, group=None):
    """Sum `inp` [world * chunk] over the ranks; this rank's chunk of the sum lands in `out`."""
    import torch.distributed as dist
    dist.reduce_scatter_tensor(out, inp, op=dist.ReduceOp.SUM, group=group)


def simulated_reduce_scatter(outs: Sequence[torch.Tensor], inps: Sequence[torch.Tensor]):
    """The same for ranks simulated in one process: out_r = sum over ranks (in rank order) of chunk r."""
    chunk = outs[0].numel()
    for r, out in enumerate(outs):
        total = inps[0][r * chunk:(r + 1) * chunk].clone()
        for inp in inps[1:]:
            total += inp[r * chunk:(r + 1) * chunk]
        out.copy_(total)


class ShardedMoECalibration:
    """One rank's part of a token-sharded, expert-parallel calibration of one weight-sharing group.

    collect() takes this rank's token share of a layer; after every layer is collected and the
    accumulators (self.reduce_tensors()) are summed over the ranks, quantize() runs this rank's
    experts [e0, e1) (plus the always-active experts on rank 0)."""

    def __init__(self, ctx: L.Context, rank: int, world: int, n_layers: int, max_tokens_per_rank: int, E: int,
                 k: int, d_model: int, d_ff: int, n_shared: int = 0, shared_dff: int = 0, bits_routed: int = 2,
                 bits_shared: int = 3, damp_frac: float = 0.01, timer=NO_TIMER, modes=("rt",)):
        if not 1 <= world <= E:
            raise ValueError(f"expert-parallel quantization needs 1 <= world ({world}) <= E ({E})")
        self.ctx, self.rank, self.world, self.E = ctx, rank, world, E
        self.e0, self.e1 = expert_range(E, rank, world)
        self.local_shared = n_shared if rank == 0 else 0
        # collection over every expert for this rank's tokens
        self.collector = MoECalibration(ctx, n_layers, max_tokens_per_rank, E, k, d_model, d_ff, n_shared, shared_dff,
                                        bits_routed, bits_shared, damp_frac, timer=timer, modes=modes)
        # quantization of this rank's experts (its own accumulators hold their summed Hessians)
        self.quantizer = MoECalibration(ctx, n_layers, 1, self.e1 - self.e0, k, d_model, d_ff,
                                        self.local_shared, shared_dff, bits_routed, bits_shared, damp_frac,
                                        timer=timer, modes=modes)
        self.exchanged = False
        self.layout = ExchangeLayout(E, world, n_layers, d_model, d_ff, n_shared, shared_dff)

    def reset(self):
        self.collector.reset()
        self.exchanged = False

    def collect(self, layer: int, X_shard: torch.Tensor, logits_shard: torch.Tensor, w: MoEWeights):
        self.collector.collect(layer, X_shard, logits_shard, w)

    def reduce_tensors(self) -> list[torch.Tensor]:
        c = self.collector
        accs = [c.acc_in, c.acc_dn] + ([c.acc_sdn] if c.n_shared else [])
        return [t for a in accs for t in accum_tensors(a)]

    def _accs(self, holder):
        accs = {"in": holder.acc_in, "dn": holder.acc_dn}
        if holder.n_shared:
            accs["sdn"] = holder.acc_sdn
        return accs

    def exchange_send(self, layout: ExchangeLayout) -> torch.Tensor:
        """This rank's send buffer [world * chunk]: for every owner rank, the packed upper triangles of
        this rank's partial sums of the slots that rank owns (padding zero)."""
        c = self.collector
        accs = self._accs(c)
        send = torch.zeros(layout.world * layout.chunk, dtype=torch.float32, device=c.dev)
        for r, parts in enumerate(layout.parts):
            for acc, s0, ns, d, off in parts:
                S, _ = accs[acc].buffers()
                if ns:
                    base = r * layout.chunk + off
                    L.clha_pack_upper(self.ctx, S, S.shape[0], S.shape[1], ns, d,
                                      send[base: base + S.shape[0] * ns * packed_floats(d)], first=s0)
        return send

    def exchange_receive(self, layout: ExchangeLayout, recv: torch.Tensor):
        """Unpack this rank's summed chunk into its quantizer's accumulators (the slots it owns, in the
        quantizer's own slot order) and take the token counts of those slots from the collector's
        (already summed) counts."""
        c, q = self.collector, self.quantizer
        qaccs, caccs = self._accs(q), self._accs(c)
        for acc, s0, ns, d, off in layout.parts[self.rank]:
            if not ns:
                continue
            Sq, cq = qaccs[acc].buffers()
            _, cc = caccs[acc].buffers()
            if acc == "sdn":
                q0 = 0                       # the always-active experts' down-projection slots
            elif s0 == self.E:
                q0 = Sq.shape[1] - 1         # the always-active experts' shared input slot (last)
            else:
                q0 = s0 - self.e0            # this rank's routed experts, from its slot 0
            L.clha_unpack_upper(self.ctx, recv[off: off + Sq.shape[0] * ns * packed_floats(d)], Sq.shape[0],
                                Sq.shape[1], ns, d, Sq, first=q0)
            cq[:, q0:q0 + ns].copy_(cc[:, s0:s0 + ns])
        self.exchanged = True

    def count_tensors(self) -> list[torch.Tensor]:
        """The token counts of every accumulator (all-reduced alongside the exchange: a few integers)."""
        return [a.buffers()[1] for a in self._accs(self.collector).values()]

    def local_weights(self, w: MoEWeights) -> MoEWeights:
        """This rank's experts' weights, stacked (gate of e0..e1-1, then up, then down)."""
        e0, e1, E = self.e0, self.e1, self.E
        Wgu = torch.cat([w.Wgu[e0:e1], w.Wgu[E + e0:E + e1]]).contiguous()
        out = MoEWeights(Wgu, w.Wd[e0:e1].contiguous())
        if self.local_shared:
            out.Sgu, out.Sd = w.Sgu, w.Sd
        return out

    def quantize(self, w_local: MoEWeights, modes=None):
        """After the reduction: copy this rank's summed Hessians into its own accumulators (unless the
        owner exchange already put them there), then aggregate, factor, GPTQ and score them (results
        in self.quantizer.res[mode])."""
        c, q, e0, e1 = self.collector, self.quantizer, self.e0, self.e1
        if self.exchanged:
            self.exchanged = False
            q.quantize(w_local, modes)
            return q.res
        S, cnt = c.acc_in.buffers()
        Sq, cq = q.acc_in.buffers()
        Sq[:, : e1 - e0].copy_(S[:, e0:e1])
        cq[:, : e1 - e0].copy_(cnt[:, e0:e1])
        S, cnt = c.acc_dn.buffers()
        Sq, cq = q.acc_dn.buffers()
        Sq.copy_(S[:, e0:e1])
        cq.copy_(cnt[:, e0:e1])
        if self.local_shared:
            S, cnt = c.acc_in.buffers()
            Sq, cq = q.acc_in.buffers()
            Sq[:, -1].copy_(S[:, c.E])
            cq[:, -1].copy_(cnt[:, c.E])
            S, cnt = c.acc_sdn.buffers()
            Sq, cq = q.acc_sdn.buffers()
            Sq.copy_(S)
            cq.copy_(cnt)
        q.quantize(w_local, modes)
        return q.res


def gather_expert_rows(local: torch.Tensor, E_local: int, E: int, world: int, group=None,
                       all_gather: Callable | None = None) -> torch.Tensor:
    """Reassemble per-expert results [E_local, ...] of every rank into [E, ...] in expert order (ranks
    hold contiguous, balanced ranges; shorter ranges are padded for the collective)."""
    import torch.distributed as dist
    e_max = -(-E // world)
    pad = torch.zeros((e_max,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:E_local].copy_(local[:E_local])
    parts = [torch.empty_like(pad) for _ in range(world)]
    if all_gather is None:
        dist.all_gather(parts, pad, group=group)
    else:
        all_gather(parts, pad)
    rows = []
    for r in range(world):
        e0, e1 = expert_range(E, r, world)
        rows.append(parts[r][: e1 - e0])
    return torch.cat(rows)


def exchange(ranks, reduce_scatter=None, all_reduce=None):
    """The owner exchange for the given rank objects (one per process under torch.distributed, or all
    of them when the ranks are simulated in one process): pack, reduce-scatter the triangles, all-reduce
    the counts, unpack into each rank's quantizer."""
    layout = ranks[0].layout
    sends = [rk.exchange_send(layout) for rk in ranks]
    recvs = [torch.empty(layout.chunk, dtype=torch.float32, device=s.device) for s in sends]
    if len(ranks) == 1 and reduce_scatter is not None:
        reduce_scatter(recvs[0], sends[0])
        all_reduce(ranks[0].count_tensors())
    else:
        simulated_reduce_scatter(recvs, sends)
        simulated_reduce([rk.count_tensors() for rk in ranks])
    for rk, recv in zip(ranks, recvs):
        rk.exchange_receive(layout, recv)
