"""The multi-rank host logic of bench.py on CPU: two gloo ranks (one process each, spawned), the same
calls bench.py makes under torchrun — process-group setup, barrier, max over ranks of the step time,
the whole-job value under weak scaling, a distinct reproducible input per rank, and the reference arm
that only rank 0 runs."""
import multiprocessing as mp
import os
import socket
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    try:
        sys.path.insert(0, ROOT)
        os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                          LOCAL_RANK=str(rank))
        import torch
        import torch.distributed as dist
        import bench
        w, r, _ = bench.dist_setup(backend="gloo")
        bench.barrier(w)
        step_ms = 10.0 + 5.0 * r                      # rank 1 is the slow one
        ms = bench.max_over_ranks(step_ms, w)
        value = bench.job_value(81920, ms, w)
        from synth import workload
        x = workload(2, "cpu", seed=bench.rank_seed(r), tokens=256).x(0)
        digest = torch.tensor([float(x.float().sum())], dtype=torch.float64)
        got = [torch.zeros(1, dtype=torch.float64) for _ in range(w)]
        dist.all_gather(got, digest)

        class Args:
            warmup, steps = 3, 1
        ref_rc = bench.run_reference(Args, w, r) if r != 0 else None   # rank 0 would run the oracle
        bench.barrier(w)
        dist.destroy_process_group()
        q.put((r, ms, value, [float(t) for t in got], ref_rc))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, "error", repr(e), None, None))


def test_two_gloo_ranks_bench_logic():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    results = {}
    for _ in procs:
        r, ms, value, digests, ref_rc = q.get(timeout=240)
        assert ms != "error", value
        results[r] = (ms, value, digests, ref_rc)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    # the slowest rank sets the step time on every rank; value = all ranks' columns / that time
    for r in range(2):
        ms, value, digests, _ = results[r]
        assert ms == 15.0
        assert value == pytest.approx(2 * 81920 / 15e-3)
    # each rank's inputs are its own (distinct seeds) and reproducible in a single process
    d0, d1 = results[0][2]
    assert d0 != d1 and results[1][2] == [d0, d1]
    sys.path.insert(0, ROOT)
    import bench
    from synth import workload
    assert float(workload(2, "cpu", seed=bench.rank_seed(1), tokens=256).x(0).float().sum()) == d1
    # the reference arm: ranks other than 0 exit 0 without work
    assert results[1][3] == 0
