"""clha_gather_noalloc, the gather for callers that cannot allocate device memory (their memory
belongs to their own allocator, where a library's cudaMalloc can fail and its cudaFree stalls the
device). It must give exactly what clha_gather gives, call after call, although every call reuses
the same fixed scratch array; and it must refuse a gather too large for that array.

Kept in a file of its own that is collected last, so a failure here comes after every other test.
"""
import numpy as np
import pytest
import torch

from post_quantization_expert_b200 import clha as L

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _route(ctx, n, E, k, seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    lg = torch.randn((n, E), generator=g).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    return ids, g


def _gather(fn, ctx, X, ids, k, E):
    n, d = X.shape
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.full((P, d), -7.0, dtype=X.dtype, device=DEV)
    seg = torch.full((2 * E + 1,), -7, dtype=torch.int64, device=DEV)
    perm = torch.full((P,), -7, dtype=torch.int32, device=DEV)
    fn(ctx, X, n, d, ids, k, E, Xp, P, seg, perm)
    torch.cuda.synchronize()
    end = int(seg[E].item())
    return Xp[:end].cpu(), seg.cpu(), perm[:end].cpu()


@pytest.mark.parametrize("calls", [[(8192, 16, 2, 1024, 1), (3001, 64, 6, 256, 2)]])
def test_noalloc_gather_equals_gather_on_consecutive_calls(ctx, calls):
    # the second call is smaller than the first, so anything left in the shared array from the first
    # call would show up as wrong permutation entries or rows
    for n, E, k, d, seed in calls:
        ids, g = _route(ctx, n, E, k, seed)
        X = torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV)
        want = _gather(L.clha_gather, ctx, X, ids, k, E)
        got = _gather(L.clha_gather_noalloc, ctx, X, ids, k, E)
        assert torch.equal(got[1], want[1])           # segment starts and token counts
        assert torch.equal(got[2], want[2])           # token of every packed row, -1 for padding
        assert torch.equal(got[0], want[0])           # the packed rows, bit for bit
        L.clha_check(ctx)


def test_noalloc_gather_rejects_oversize(ctx):
    n, E, k, d = 600_000, 8, 2, 128      # about 1.2M packed rows: more scratch than the fixed array
    ids = torch.zeros((n, k), dtype=torch.int32, device=DEV)
    ids[:, 1] = 1
    X = torch.zeros((1, d), dtype=torch.bfloat16, device=DEV)   # never read: the call is refused first
    P = L.clha_packed_rows(n, k, E)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    launched = L.clha_kernel_launches(ctx)
    with pytest.raises(L.ClhaError) as ei:
        L.clha_gather_noalloc(ctx, X, n, d, ids, k, E, X, P, seg)
    assert ei.value.status == L.ERR_INVALID_ARG
    assert "scratch" in ei.value.message
    assert L.clha_kernel_launches(ctx) == launched
