"""Token-sharded collection and expert-parallel quantization over several ranks (one process per GPU).

Phase 1 of CLHA (the CLHA page, §2.2 (1)) is a sum over calibration tokens, so it shards over
tokens: every rank routes, gathers, activates and collects its own contiguous share of each layer's
tokens into its own accumulators, and one all-reduce (sum) of the Gram matrices and token counts
gives every rank the Hessians of all the tokens. Phases 2 and 3 are independent per expert: each rank
aggregates, factors and quantizes its own contiguous range of experts (the always-active experts on
rank 0), and the results are gathered at the end. The all-reduce is the only exchange on the data
path; the kernels are the single-GPU ones.

The reduction is left to the caller (`dist_reduce` or `simulated_reduce` on `reduce_tensors()`), so the
same code runs with torch.distributed (NCCL between GPUs, gloo on CPU) or with the ranks simulated
one after another in one process.
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

    def reset(self):
        self.collector.reset()

    def collect(self, layer: int, X_shard: torch.Tensor, logits_shard: torch.Tensor, w: MoEWeights):
        self.collector.collect(layer, X_shard, logits_shard, w)

    def reduce_tensors(self) -> list[torch.Tensor]:
        c = self.collector
        accs = [c.acc_in, c.acc_dn] + ([c.acc_sdn] if c.n_shared else [])
        return [t for a in accs for t in accum_tensors(a)]

    def local_weights(self, w: MoEWeights) -> MoEWeights:
        """This rank's experts' weights, stacked (gate of e0..e1-1, then up, then down)."""
        e0, e1, E = self.e0, self.e1, self.E
        Wgu = torch.cat([w.Wgu[e0:e1], w.Wgu[E + e0:E + e1]]).contiguous()
        out = MoEWeights(Wgu, w.Wd[e0:e1].contiguous())
        if self.local_shared:
            out.Sgu, out.Sd = w.Sgu, w.Sd
        return out

    def quantize(self, w_local: MoEWeights, modes=None):
        """After the reduction: copy this rank's summed Hessians into its own accumulators, then
        aggregate, factor, GPTQ and score them (results in self.quantizer.res[mode])."""
        c, q, e0, e1 = self.collector, self.quantizer, self.e0, self.e1
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
