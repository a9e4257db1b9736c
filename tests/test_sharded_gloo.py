"""Host logic of token-sharded collection and expert-parallel quantization on CPU: two gloo ranks run
the module's reduction and gather on CPU tensors (the oracle's Gram matrices stand in for the GPU
accumulators), plus the partitions themselves."""
import multiprocessing as mp
import os
import socket
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_partitions_cover_everything_once():
    from post_quantization_expert_b200.sharded import expert_range, token_range
    for n in (0, 1, 7, 8192, 131071):
        for world in (1, 2, 3, 8):
            parts = [token_range(n, r, world) for r in range(world)]
            assert parts[0][0] == 0 and parts[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
            sizes = [b - a for a, b in parts]
            assert max(sizes) - min(sizes) <= 1
    assert [expert_range(16, r, 3) for r in range(3)] == [(0, 6), (6, 11), (11, 16)]


class _FakeAccum:
    def __init__(self, S, counts):
        self.S, self.counts = S, counts

    def buffers(self):
        return self.S, self.counts


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
        from datetime import timedelta
        import torch
        import torch.distributed as dist
        import oracle as O
        from post_quantization_expert_b200 import sharded as SH
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
        g = np.random.default_rng(11)
        n, d, E = 1000, 64, 5
        X = g.standard_normal((n, d))
        t0, t1 = SH.token_range(n, rank, world)
        S = torch.from_numpy(O.gram(X[t0:t1]))[None, None].clone()          # [layers, slots, d, d]
        cnt = torch.tensor([[t1 - t0]], dtype=torch.int64)
        SH.dist_reduce(SH.accum_tensors(_FakeAccum(S, cnt)))
        ok_sum = bool(np.allclose(S[0, 0].numpy(), O.gram(X), rtol=1e-12, atol=1e-9)) and int(cnt[0, 0]) == n
        # expert results: every rank holds rows for its own experts; the gather puts them in order
        e0, e1 = SH.expert_range(E, rank, world)
        rows = torch.arange(e0, e1, dtype=torch.float64)[:, None] * torch.ones(3, dtype=torch.float64)
        full = SH.gather_expert_rows(rows, e1 - e0, E, world)
        ok_gather = full.shape == (E, 3) and bool(torch.equal(full[:, 0], torch.arange(E, dtype=torch.float64)))
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, ok_sum, ok_gather, ""))
    except Exception as e:
        q.put((rank, False, False, repr(e)))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_reduction_and_gather(world):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok_sum, ok_gather, err in res:
        assert not err, err
        assert ok_sum and ok_gather, (rank, ok_sum, ok_gather)


def _pack_np(mats):
    """Upper triangles of [n, d, d] matrices, row after row (the exchange's packed layout)."""
    d = mats.shape[-1]
    iu = np.triu_indices(d)
    return np.concatenate([m[iu] for m in mats])


def _exchange_rank_main(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
        from datetime import timedelta
        import torch
        import torch.distributed as dist
        import oracle as O
        from post_quantization_expert_b200 import sharded as SH
        dist.init_process_group("gloo", timeout=timedelta(seconds=60))
        E, Lyr, dm, dff, ns, n = 5, 2, 16, 8, 2, 600
        lay = SH.ExchangeLayout(E, world, Lyr, dm, dff, ns, dff)
        g = np.random.default_rng(7)
        # every "slot" of every accumulator gets its own token stream; this rank holds its token share
        X = {a: g.standard_normal((Lyr, slots, n, dim)) for a, slots, dim in
             (("in", E + 1, dm), ("dn", E, dff), ("sdn", ns, dff))}
        t0, t1 = SH.token_range(n, rank, world)
        part = {a: np.einsum("lsnd,lsne->lsde", x[:, :, t0:t1], x[:, :, t0:t1]) for a, x in X.items()}
        full = {a: np.einsum("lsnd,lsne->lsde", x, x) for a, x in X.items()}
        send = np.zeros(world * lay.chunk, np.float32)
        for r, parts in enumerate(lay.parts):
            for acc, s0, k, d, off in parts:
                blk = part[acc][:, s0:s0 + k].reshape(-1, d, d)
                send[r * lay.chunk + off: r * lay.chunk + off + blk.shape[0] * SH.packed_floats(d)] = _pack_np(blk)
        recv = torch.empty(lay.chunk, dtype=torch.float32)
        SH.dist_reduce_scatter(recv, torch.from_numpy(send))
        ok, owned = True, 0
        for acc, s0, k, d, off in lay.parts[rank]:
            want = _pack_np(full[acc][:, s0:s0 + k].reshape(-1, d, d).astype(np.float32))
            got = recv[off: off + want.size].numpy()
            ok &= bool(np.allclose(got, want, rtol=1e-5, atol=1e-3))
            owned += k
        e0, e1 = SH.expert_range(E, rank, world)
        ok &= owned == 2 * (e1 - e0) + (1 + ns if rank == 0 else 0)
        ok &= lay.chunk >= max(lay.used) and lay.used[rank] <= lay.chunk
        dist.barrier()
        dist.destroy_process_group()
        q.put((rank, ok, ""))
    except Exception as e:
        q.put((rank, False, repr(e)))


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_owner_exchange_of_packed_triangles(world):
    """Each rank packs the upper triangles of its partial sums by owner; one reduce-scatter gives each
    rank exactly the summed triangles of the slots it quantizes (its routed experts' input and
    down-projection slots, and on rank 0 the always-active experts')."""
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, ok, err in res:
        assert not err, err
        assert ok, rank
