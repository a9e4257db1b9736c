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


def _gather(fn, ctx, X, ids, k, E, with_perm=True):
    """Packed rows, segment table and (with_perm) the permutation of one gather call, on the host.
    Without a perm array the permutation lives in the gather's scratch, which for
    clha_gather_noalloc is the shared fixed array."""
    n, d = X.shape
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.full((P, d), -7.0, dtype=X.dtype, device=DEV)
    seg = torch.full((2 * E + 1,), -7, dtype=torch.int64, device=DEV)
    perm = torch.full((P,), -7, dtype=torch.int32, device=DEV) if with_perm else None
    fn(ctx, X, n, d, ids, k, E, Xp, P, seg, perm)
    torch.cuda.synchronize()
    end = int(seg[E].item())
    return Xp[:end].cpu(), seg.cpu(), (perm[:end].cpu() if with_perm else None)


@pytest.mark.parametrize("calls", [[(8192, 16, 2, 1024, 1), (3001, 64, 6, 256, 2), (777, 16, 2, 128, 3)]])
def test_noalloc_gather_equals_gather_on_consecutive_calls(ctx, calls):
    # each call is smaller than the one before, so a permutation or histogram left in the shared
    # array by an earlier call would show up as wrong rows, segments or permutation entries; every
    # call runs both with a caller-owned perm (histograms only in the array) and without one (the
    # permutation in the array too)
    for n, E, k, d, seed in calls:
        ids, g = _route(ctx, n, E, k, seed)
        X = torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV)
        for with_perm in (True, False):
            want = _gather(L.clha_gather, ctx, X, ids, k, E, with_perm)
            got = _gather(L.clha_gather_noalloc, ctx, X, ids, k, E, with_perm)
            assert torch.equal(got[1], want[1]), (n, with_perm)     # segment starts and token counts
            if with_perm:
                assert torch.equal(got[2], want[2]), n              # token of every packed row, -1 for padding
            assert torch.equal(got[0], want[0]), (n, with_perm)     # the packed rows, bit for bit
            L.clha_check(ctx)


def test_noalloc_gather_rejects_oversize(ctx):
    n, E, k, d = 600_000, 8, 2, 128      # about 1.2M packed rows: a permutation larger than the fixed array
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


def test_noalloc_gather_with_perm_takes_only_histograms(ctx):
    """With a caller-owned perm the fixed array holds only the block histograms, so a gather whose
    permutation alone would not fit (about 1.2M packed rows) runs, and equals clha_gather."""
    n, E, k, d = 600_000, 8, 2, 128
    ids, g = _route(ctx, n, E, k, 4)
    X = torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV)
    want = _gather(L.clha_gather, ctx, X, ids, k, E, True)
    got = _gather(L.clha_gather_noalloc, ctx, X, ids, k, E, True)
    for a, b in zip(got, want):
        assert torch.equal(a, b)
    L.clha_check(ctx)
