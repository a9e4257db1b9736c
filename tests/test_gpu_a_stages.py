"""Stage-wise parity of each CUDA step against the float64 oracle, each stage fed the same inputs as
the oracle so its own error is isolated. Sizes span several tiles and end on ragged tails."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import CONFIG_BAR, assert_codes, rel_fro, sym_from_upper, to64
from post_quantization_expert_b200 import clha as L

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gen(seed):
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


# ------------------------------------------------------------------------------------ routing
@pytest.mark.parametrize("n,E,k", [(1000, 16, 2), (4099, 64, 6), (37, 5, 5), (1, 1024, 8), (777, 33, 1)])
def test_route_bit_exact(ctx, n, E, k):
    g = _gen(n + E)
    lg = torch.randn((n, E), generator=g)
    lg[::7, 3 % E] = lg[::7, 0]                                  # ties between experts
    lg[::11] = torch.round(lg[::11] * 2) / 2                     # many exact ties
    lg = lg.to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    want_ids, want_counts = O.route_topk(lg.cpu().numpy(), k)
    np.testing.assert_array_equal(ids.cpu().numpy(), want_ids)
    np.testing.assert_array_equal(counts.cpu().numpy(), want_counts)


def test_route_empty_input(ctx):
    counts = torch.full((8,), 7, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, None, 0, 8, 2, None, counts)
    assert counts.sum().item() == 0


# ------------------------------------------------------------------------------------ gather
@pytest.mark.parametrize("n,E,k,d", [(1000, 16, 2, 256), (3001, 64, 6, 128), (5, 8, 2, 384)])
def test_gather_segments(ctx, n, E, k, d):
    g = _gen(n)
    lg = torch.randn((n, E), generator=g).to(DEV)
    X = torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.full((P, d), float("nan"), dtype=torch.bfloat16, device=DEV)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    perm = torch.empty(P, dtype=torch.int32, device=DEV)
    L.clha_gather(ctx, X, n, d, ids, k, E, Xp, P, seg, perm)
    seg, perm, Xp = seg.cpu().numpy(), perm.cpu().numpy(), Xp.cpu()
    want_ids, want_counts = O.route_topk(lg.cpu().numpy(), k)
    lists = O.expert_tokens(want_ids, E)
    np.testing.assert_array_equal(seg[E + 1:], want_counts)
    start = 0
    for e in range(E):
        assert seg[e] == start and seg[e] % 128 == 0
        np.testing.assert_array_equal(perm[seg[e]:seg[e] + want_counts[e]], lists[e])
        assert np.all(perm[seg[e] + want_counts[e]:seg[e] + (want_counts[e] + 127) // 128 * 128] == -1)
        rows = Xp[seg[e]:seg[e] + want_counts[e]]
        assert torch.equal(rows, X.cpu()[torch.from_numpy(lists[e]).long()])
        pad = Xp[seg[e] + want_counts[e]:seg[e] + (want_counts[e] + 127) // 128 * 128]
        assert torch.all(pad == 0)
        start += (want_counts[e] + 127) // 128 * 128
    assert seg[E] == start


# --------------------------------------------------------------------- gather fused into collection
@pytest.mark.parametrize("n,E,k,d,dff", [(2048, 16, 2, 1024, 512), (1000, 64, 6, 2048, 1408), (37, 8, 3, 384, 256),
                                        (80000, 16, 2, 256, 128)])
def test_gathered_collection_and_activation_equal_the_packed_path(ctx, act_kernel, n, E, k, d, dff):
    """Gram sums read from X by TMA gather4 through the routing permutation, and the activation read
    through it, are bit-identical to the same kernels on the packed copy (the same rows in the same
    order; padding rows are zeros either way). Sizes: ragged segments, 64 experts with 128-row
    padding, a few tokens per expert, and ~10k-token segments (two accumulation chunks per tile,
    whose fp32 additions into S may land in either order: equal to 1e-6 there). The gathered
    activation is the FMA kernel, so the packed one is held to it too."""
    act_kernel(L.ACT_FMA)
    g = _gen(n + E)
    lg = torch.randn((n, E), generator=g).to(DEV)
    X = (torch.randn((n, d), generator=g) * (0.5 + torch.rand(d, generator=g))).to(torch.bfloat16).to(DEV)
    Wg = (0.03 * torch.randn((E, dff, d), generator=g)).to(torch.bfloat16).to(DEV)
    Wu = (0.03 * torch.randn((E, dff, d), generator=g)).to(torch.bfloat16).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.empty((P, d), dtype=torch.bfloat16, device=DEV)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    perm = torch.empty(P, dtype=torch.int32, device=DEV)
    L.clha_gather(ctx, X, n, d, ids, k, E, Xp, P, seg, perm)
    seg2 = torch.empty_like(seg)
    perm2 = torch.empty_like(perm)
    L.clha_gather(ctx, X, n, d, ids, k, E, None, P, seg2, perm2)      # the permutation alone
    assert torch.equal(seg, seg2) and torch.equal(perm, perm2)
    a, b = L.Accum(ctx, d, 2, E), L.Accum(ctx, d, 2, E)
    for layer in (0, 1):   # twice into layer 1: the second pass accumulates onto the first
        for _ in range(1 + layer):
            L.clha_collect(ctx, a, layer, Xp, P, d, seg, E, 0)
            L.clha_collect_gathered(ctx, b, layer, X, n, d, perm, seg, E, 0)
    h1 = torch.full((P, dff), 7.0, dtype=torch.bfloat16, device=DEV)
    h2 = torch.full((P, dff), -7.0, dtype=torch.bfloat16, device=DEV)
    L.clha_expert_act(ctx, Xp, P, d, seg, E, Wg, Wu, dff, h1)
    L.clha_expert_act_gathered(ctx, X, n, d, perm, P, seg, E, Wg, Wu, dff, h2)
    L.clha_check(ctx)
    Sa, ca = a.buffers()
    Sb, cb = b.buffers()
    assert torch.equal(ca, cb)
    # the authoritative upper triangle is bit-identical
    iu = torch.triu_indices(d, d, device=DEV)
    multi_chunk = n * k // E > 8192
    for layer in (0, 1):
        for e in range(E):
            ua, ub = Sa[layer, e][iu[0], iu[1]], Sb[layer, e][iu[0], iu[1]]
            if multi_chunk:
                assert (ua - ub).norm() <= 1e-6 * ua.norm(), (layer, e)
            else:
                assert torch.equal(ua, ub), (layer, e)
    end = int(seg[E].item())
    assert torch.equal(h1[:end], h2[:end])


# ------------------------------------------------------------------------------------ collection
@pytest.mark.parametrize("n,d", [(1000, 512), (129, 1408), (1, 256), (4096, 1024), (777, 2048), (9000, 384),
                                 (65536, 256)])
def test_collect_dense_bf16(ctx, n, d):
    g = _gen(n * d)
    X = (torch.randn((n, d), generator=g) * (1 + torch.rand(d, generator=g))).to(torch.bfloat16).to(DEV)
    acc = L.Accum(ctx, d, 2, 1)
    L.clha_collect(ctx, acc, 1, X, n, d)
    S, cnt = acc.buffers()
    torch.cuda.synchronize()
    want = O.gram(to64(X))
    got = sym_from_upper(S[1, 0].double().cpu().numpy())
    assert rel_fro(got, want) < 1e-4
    assert cnt[1, 0].item() == n and cnt[0, 0].item() == 0
    assert torch.all(S[0] == 0)


@pytest.mark.parametrize("n,d", [(1100, 8192), (700, 8320), (5000, 4096), (6000, 4224)])
def test_collect_large_d(ctx, n, d):
    """One dense Gram at d >= 4096 runs on pairs of SMs (256 x 256 tiles, one tcgen05.mma over both
    CTAs' shared memory). Ragged token counts; 2048-token chunks below d = 8192 (5000 tokens: three
    chunks per tile) and 8192-token ones above; d = 8320 and 4224 are not multiples of 256, so the
    last tile's second row half lies past the matrix (computed on zero-filled operands, never
    written). The Gram equals the float64 one; a second call into another layer of the same
    accumulator, over a token range that starts mid-block, accumulates there and leaves the first
    layer alone."""
    g = _gen(n + d)
    X = (torch.randn((n, d), generator=g) * (1 + torch.rand(d, generator=g))).to(torch.bfloat16).to(DEV)
    acc = L.Accum(ctx, d, 2, 1)
    L.clha_collect(ctx, acc, 0, X, n, d)
    L.clha_collect(ctx, acc, 1, X[37:].contiguous(), n - 37, d)
    S, cnt = acc.buffers()
    torch.cuda.synchronize()
    X64 = to64(X)
    assert rel_fro(sym_from_upper(S[0, 0].double().cpu().numpy()), O.gram(X64)) < 1e-4
    assert rel_fro(sym_from_upper(S[1, 0].double().cpu().numpy()), O.gram(X64[37:])) < 1e-4
    assert cnt[0, 0].item() == n and cnt[1, 0].item() == n - 37


def test_collect_routed_bf16_and_accumulates(ctx):
    n, E, k, d = 3000, 16, 2, 1024
    g = _gen(7)
    lg = torch.randn((n, E), generator=g).to(DEV)
    X = torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.empty((P, d), dtype=torch.bfloat16, device=DEV)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    L.clha_gather(ctx, X, n, d, ids, k, E, Xp, P, seg)
    acc = L.Accum(ctx, d, 1, E + 2)
    L.clha_collect(ctx, acc, 0, Xp, P, d, seg, E, 2)     # slots 2..E+1
    L.clha_collect(ctx, acc, 0, Xp, P, d, seg, E, 2)     # a second batch accumulates
    S, cnt = acc.buffers()
    torch.cuda.synchronize()
    want_ids, want_counts = O.route_topk(lg.cpu().numpy(), k)
    lists = O.expert_tokens(want_ids, E)
    X64 = to64(X)
    np.testing.assert_array_equal(cnt[0, 2:].cpu().numpy(), 2 * want_counts)
    assert cnt[0, :2].sum().item() == 0
    for e in range(E):
        want = 2 * O.gram(X64[lists[e]])
        assert rel_fro(sym_from_upper(S[0, 2 + e].double().cpu().numpy()), want) < 1e-4


@pytest.mark.parametrize("n,d", [(1000, 512), (1024, 512), (33, 128)])
def test_collect_dense_f32(ctx, n, d):
    g = _gen(n + 3)
    X = torch.randn((n, d), generator=g).to(DEV)
    acc = L.Accum(ctx, d, 1, 1)
    L.clha_collect(ctx, acc, 0, X, n, d)
    S, _ = acc.buffers()
    torch.cuda.synchronize()
    assert rel_fro(sym_from_upper(S[0, 0].double().cpu().numpy()), O.gram(to64(X))) < 1e-4


def test_layer_tagged_collection_is_order_independent(ctx):
    """Layer-aware accumulators (CLHA page §2.4): interleaving the layers' calls in any order gives
    each layer exactly its own tokens' Gram matrix."""
    d = 256
    g = _gen(11)
    Xa1, Xa2, Xb = (torch.randn((n, d), generator=g).to(torch.bfloat16).to(DEV) for n in (300, 200, 500))
    acc1, acc2 = L.Accum(ctx, d, 2, 1), L.Accum(ctx, d, 2, 1)
    for layer, X in ((0, Xa1), (1, Xb), (0, Xa2)):
        L.clha_collect(ctx, acc1, layer, X, X.shape[0], d)
    for layer, X in ((1, Xb), (0, Xa2), (0, Xa1)):
        L.clha_collect(ctx, acc2, layer, X, X.shape[0], d)
    S1, c1 = acc1.buffers()
    S2, c2 = acc2.buffers()
    torch.cuda.synchronize()
    want_a = O.gram(np.vstack([to64(Xa1), to64(Xa2)]))
    want_b = O.gram(to64(Xb))
    for S in (S1, S2):
        assert rel_fro(sym_from_upper(S[0, 0].double().cpu().numpy()), want_a) < 1e-4
        assert rel_fro(sym_from_upper(S[1, 0].double().cpu().numpy()), want_b) < 1e-4
    assert c1.tolist() == c2.tolist() == [[500], [500]]


def test_accumulator_checkpoint_roundtrip(ctx):
    d = 128
    X = torch.randn((70, d), generator=_gen(5)).to(torch.bfloat16).to(DEV)
    acc = L.Accum(ctx, d, 2, 3)
    L.clha_collect(ctx, acc, 1, X, 70, d, None, 1, 2)
    S, cnt = L.clha_accum_export(ctx, acc)
    acc2 = L.Accum(ctx, d, 2, 3)
    L.clha_accum_import(ctx, acc2, S, cnt)
    L.clha_collect(ctx, acc2, 1, X, 70, d, None, 1, 2)     # resume: one more batch
    S2, cnt2 = L.clha_accum_export(ctx, acc2)
    np.testing.assert_array_equal(cnt2[1, 2], 140)
    np.testing.assert_allclose(np.triu(S2[1, 2]), 2 * np.triu(S[1, 2]), rtol=1e-6)


# ------------------------------------------------------------------------------------ FFN act
@pytest.fixture
def act_kernel(ctx):
    """Restores the default (per-call) activation kernel choice after a test that forces one."""
    yield lambda k: L.clha_set_act_kernel(ctx, k)
    L.clha_set_act_kernel(ctx, L.ACT_AUTO)


@pytest.mark.parametrize("kernel", [L.ACT_FMA, L.ACT_TENSOR])
@pytest.mark.parametrize("rows,dm,dff", [(300, 256, 384), (1000, 1024, 512), (4097, 2048, 1408)])
def test_expert_act_dense(ctx, act_kernel, kernel, rows, dm, dff):
    """Both activation kernels against the oracle on inputs without outlier channels: at least 99.9 %
    of h bit-exact, the rest one bf16 rounding away."""
    act_kernel(kernel)
    g = _gen(rows)
    X = torch.randn((rows, dm), generator=g).to(torch.bfloat16).to(DEV)
    Wg = (0.05 * torch.randn((1, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    Wu = (0.05 * torch.randn((1, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    h = torch.empty((rows, dff), dtype=torch.bfloat16, device=DEV)
    L.clha_expert_act(ctx, X, rows, dm, None, 1, Wg, Wu, dff, h)
    assert L.clha_last_act_kernel(ctx) == kernel
    want = O.ffn_act(to64(X), to64(Wg[0]), to64(Wu[0]))
    got = to64(h)
    exact = np.mean(got == want)
    assert exact >= 0.999
    np.testing.assert_allclose(got, want, rtol=2 ** -7, atol=1e-6)


def test_expert_act_choice_follows_channel_range(ctx):
    """The default choice, decided on the device per call: the tensor cores for channels of similar
    range; the tensor cores too when a few channels are ~20x the rest (the outlier-channel workload),
    with those channels' products taken out of the tensor-core sums (their weights zeroed in a masked
    copy) and added exactly in the epilogue; the FMA kernel when more than 64 channels are outliers.
    Each time at least 99.9 % of h equals the float64 result rounded once to bf16."""
    g = _gen(5)
    rows, dm, dff = 512, 1024, 256
    X = torch.randn((rows, dm), generator=g)
    Wg = (0.05 * torch.randn((1, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    Wu = (0.05 * torch.randn((1, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    h = torch.empty((rows, dff), dtype=torch.bfloat16, device=DEV)
    perm = torch.randperm(dm, generator=g)
    for n_out, kernel in ((0, L.ACT_TENSOR), (10, L.ACT_TENSOR), (64, L.ACT_TENSOR), (80, L.ACT_FMA)):
        Xo = X.clone()
        Xo[:, perm[:n_out]] *= 20.0
        Xo = Xo.to(torch.bfloat16).to(DEV)
        h.fill_(float("nan"))
        L.clha_expert_act(ctx, Xo, rows, dm, None, 1, Wg, Wu, dff, h)
        assert L.clha_last_act_kernel(ctx) == kernel, n_out
        want = O.ffn_act(to64(Xo), to64(Wg[0]), to64(Wu[0]))
        got = to64(h)
        assert np.mean(got == want) >= 0.999, n_out
        # the FMA kernel's 32-term fp32 chunks carry the x20 terms: a few h two bf16 steps away where
        # they nearly cancel; the tensor-core path sums the outlier products exactly
        rtol = 2 ** -7 if kernel == L.ACT_TENSOR else 2 ** -6
        np.testing.assert_allclose(got, want, rtol=rtol, atol=1e-6, err_msg=f"{n_out} outlier channels")


def test_expert_act_outliers_segments_on_tensor_cores(ctx):
    """The E64 input shape in miniature: routed segments of 8 experts, 1 % of the channels x20, on the
    tensor cores with the outlier channels taken out; every segment's h against the oracle (99.9 %
    bit-equal) and the padding rows zero."""
    n, E, k, dm, dff = 1500, 8, 2, 2048, 256
    g = _gen(19)
    lg = torch.randn((n, E), generator=g).to(DEV)
    Xf = torch.randn((n, dm), generator=g)
    Xf[:, torch.randperm(dm, generator=g)[:20]] *= 20.0
    X = Xf.to(torch.bfloat16).to(DEV)
    Wg = (0.02 * torch.randn((E, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    Wu = (0.02 * torch.randn((E, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.empty((P, dm), dtype=torch.bfloat16, device=DEV)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    L.clha_gather(ctx, X, n, dm, ids, k, E, Xp, P, seg)
    h = torch.full((P, dff), 3.0, dtype=torch.bfloat16, device=DEV)
    L.clha_expert_act(ctx, Xp, P, dm, seg, E, Wg, Wu, dff, h)
    assert L.clha_last_act_kernel(ctx) == L.ACT_TENSOR
    seg = seg.cpu().numpy()
    lists = O.expert_tokens(O.route_topk(lg.cpu().numpy(), k)[0], E)
    X64, hh = to64(X), to64(h)
    exact = total = 0
    for e in range(E):
        c = len(lists[e])
        want = O.ffn_act(X64[lists[e]], to64(Wg[e]), to64(Wu[e]))
        got = hh[seg[e]:seg[e] + c]
        np.testing.assert_allclose(got, want, rtol=2 ** -7, atol=1e-6)
        exact += int(np.sum(got == want))
        total += want.size
        assert np.all(hh[seg[e] + c:seg[e] + (c + 127) // 128 * 128] == 0)
    assert exact / total >= 0.999, exact / total


@pytest.mark.parametrize("kernel", [L.ACT_FMA, L.ACT_TENSOR])
def test_expert_act_segments_zero_padding(ctx, act_kernel, kernel):
    act_kernel(kernel)
    n, E, k, dm, dff = 600, 8, 2, 256, 128
    g = _gen(9)
    lg = torch.randn((n, E), generator=g).to(DEV)
    X = torch.randn((n, dm), generator=g).to(torch.bfloat16).to(DEV)
    Wg = (0.05 * torch.randn((E, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    Wu = (0.05 * torch.randn((E, dff, dm), generator=g)).to(torch.bfloat16).to(DEV)
    ids = torch.empty((n, k), dtype=torch.int32, device=DEV)
    counts = torch.empty(E, dtype=torch.int32, device=DEV)
    L.clha_route_topk(ctx, lg, n, E, k, ids, counts)
    P = L.clha_packed_rows(n, k, E)
    Xp = torch.empty((P, dm), dtype=torch.bfloat16, device=DEV)
    seg = torch.empty(2 * E + 1, dtype=torch.int64, device=DEV)
    L.clha_gather(ctx, X, n, dm, ids, k, E, Xp, P, seg)
    h = torch.full((P, dff), 3.0, dtype=torch.bfloat16, device=DEV)
    L.clha_expert_act(ctx, Xp, P, dm, seg, E, Wg, Wu, dff, h)
    seg = seg.cpu().numpy()
    lists = O.expert_tokens(O.route_topk(lg.cpu().numpy(), k)[0], E)
    X64 = to64(X)
    hh = to64(h)
    for e in range(E):
        c = len(lists[e])
        want = O.ffn_act(X64[lists[e]], to64(Wg[e]), to64(Wu[e]))
        np.testing.assert_allclose(hh[seg[e]:seg[e] + c], want, rtol=2 ** -7, atol=1e-6)
        assert np.all(hh[seg[e] + c:seg[e] + (c + 127) // 128 * 128] == 0)


# ------------------------------------------------------------------------------------ aggregation
@pytest.mark.parametrize("mode", ["rt", "eq", "explicit"])
def test_aggregate_matches_oracle(ctx, mode):
    d, Lyr, slots = 384, 3, 2
    g = _gen(21)
    Xs = [[torch.randn((n, d), generator=g).double().numpy() for n in (50 + 10 * s, 0 if s else 80, 120)]
          for s in range(slots)]
    S = np.zeros((Lyr, slots, d, d), np.float32)
    cnt = np.zeros((Lyr, slots), np.int64)
    for s in range(slots):
        for l in range(Lyr):
            S[l, s] = O.gram(Xs[s][l]).astype(np.float32)
            cnt[l, s] = Xs[s][l].shape[0]
    acc = L.Accum(ctx, d, Lyr, slots)
    L.clha_accum_import(ctx, acc, S, cnt)
    Hc = torch.empty((slots, d, d), device=DEV)
    Hd = torch.empty_like(Hc)
    alpha = [0.7, 0.2, 0.1] if mode == "explicit" else None
    a_out, l_out = L.clha_aggregate(ctx, acc, 0, slots, {"rt": 0, "eq": 1, "explicit": 2}[mode], alpha, 0.01, Hc, Hd,
                                    want_host=True)
    for s in range(slots):
        want = O.aggregate([S[l, s].astype(np.float64) for l in range(Lyr)], list(cnt[:, s]), mode, alpha, 0.01)
        np.testing.assert_allclose(a_out[s], want["alpha"], rtol=1e-15)
        np.testing.assert_allclose(l_out[s], want["lam"], rtol=1e-10)
        assert rel_fro(Hc[s].double().cpu().numpy(), want["H_comb"]) < 1e-6
        assert rel_fro(Hd[s].double().cpu().numpy(), want["H_d"]) < 1e-6
        assert torch.equal(Hd[s], Hd[s].T)


# ------------------------------------------------------------------------------------ factor
@pytest.mark.parametrize("d,batch", [(128, 1), (128, 5), (512, 3), (896, 2), (1408, 1)])
def test_factor_matches_oracle(ctx, d, batch):
    """Two tiles per side (one with an odd batch), 8, 14 and 22 tiles; every problem against the
    oracle's float64 inverse Cholesky."""
    g = _gen(d)
    Hs = []
    for b in range(batch):
        A = torch.randn((d, d // 4), generator=g).double()
        H = (A @ A.T / (d // 4) + 0.05 * torch.eye(d, dtype=torch.float64)).float()
        Hs.append(H)
    Hd = torch.stack(Hs).to(DEV)
    U = torch.full_like(Hd, float("nan"))
    L.clha_factor(ctx, Hd, batch, d, U)
    L.clha_check(ctx)
    for b in range(batch):
        want = O.factor(Hs[b].double().numpy())
        got = U[b].double().cpu().numpy()
        assert np.all(np.tril(got, -1) == 0)
        assert rel_fro(got, want) < 1e-6


@pytest.mark.parametrize("d,batch", [(128, 1), (256, 5), (512, 3), (896, 2), (1408, 1)])
def test_factor_block_form_matches_oracle(ctx, d, batch):
    """F, the block-scaled Cholesky factor: one 128-block (its X tile only), an odd batch, and 4, 7 and
    11 blocks; every problem against the oracle's float64 F (whose own pin is the OBS recurrence)."""
    g = _gen(d + 1)
    Hs = []
    for b in range(batch):
        A = torch.randn((d, d // 4), generator=g).double()
        Hs.append((A @ A.T / (d // 4) + 0.05 * torch.eye(d, dtype=torch.float64)).float())
    Hd = torch.stack(Hs).to(DEV)
    F = torch.full_like(Hd, float("nan"))
    L.clha_factor_as(ctx, L.FACTOR_BLOCK_CHOL, Hd, batch, d, F)
    L.clha_check(ctx)
    for b in range(batch):
        got = F[b].double().cpu().numpy()
        assert np.all(np.tril(got, -1) == 0)
        assert rel_fro(got, O.factor_block_scaled(Hs[b].double().numpy())) < 1e-6


def test_factor_block_form_groups(ctx):
    """Three groups of different sizes in one Cholesky-only graph launch, each problem against the
    oracle's F; an unknown form is rejected."""
    specs = [(384, 3), (128, 2), (640, 2)]
    groups, host = [], []
    for gi, (d, batch) in enumerate(specs):
        g = _gen(200 + gi)
        Hs = []
        for b in range(batch):
            A = torch.randn((d, d // 4), generator=g).double()
            Hs.append((A @ A.T / (d // 4) + 0.05 * torch.eye(d, dtype=torch.float64)).float())
        groups.append((torch.stack(Hs).to(DEV), batch, d, torch.full((batch, d, d), float("nan"), device=DEV)))
        host.append(Hs)
    L.clha_factor_groups(ctx, groups, L.FACTOR_BLOCK_CHOL)
    L.clha_check(ctx)
    for (Hd, batch, d, F), Hs in zip(groups, host):
        for b in range(batch):
            assert rel_fro(F[b].double().cpu().numpy(), O.factor_block_scaled(Hs[b].double().numpy())) < 1e-6
    with pytest.raises(L.ClhaError):
        L.clha_factor_groups(ctx, groups, 2)


def test_factor_groups_match_oracle_and_report_across_groups(ctx):
    """Three groups of different sizes in one graph launch; each problem against the oracle. Then a
    non-positive pivot in the last group's second problem: its index counts across the groups."""
    specs = [(384, 3), (128, 2), (640, 2)]
    groups, host = [], []
    for gi, (d, batch) in enumerate(specs):
        g = _gen(100 + gi)
        Hs = []
        for b in range(batch):
            A = torch.randn((d, d // 4), generator=g).double()
            Hs.append((A @ A.T / (d // 4) + 0.05 * torch.eye(d, dtype=torch.float64)).float())
        Hd = torch.stack(Hs).to(DEV)
        U = torch.full_like(Hd, float("nan"))
        groups.append((Hd, batch, d, U))
        host.append(Hs)
    L.clha_factor_groups(ctx, groups)
    L.clha_check(ctx)
    for (Hd, batch, d, U), Hs in zip(groups, host):
        for b in range(batch):
            got = U[b].double().cpu().numpy()
            assert np.all(np.tril(got, -1) == 0)
            assert rel_fro(got, O.factor(Hs[b].double().numpy())) < 1e-6
    # non-PD: problem 1 of group 2 = problem 3 + 2 + 1 = 6 across the groups, original column 70
    Hd2 = groups[2][0]
    Hd2[1] = torch.eye(640, device=DEV)
    Hd2[1, 70, 70] = -1.0
    L.clha_factor_groups(ctx, groups)
    with pytest.raises(L.ClhaError) as ei:
        L.clha_check(ctx)
    assert ei.value.status == L.ERR_NOT_PD
    assert "problem 6" in str(ei.value) and "index 70" in str(ei.value)
    L.clha_check(ctx)
    for b in range(3):   # the other problems are unaffected
        assert torch.isfinite(groups[0][3][b]).all()
    with pytest.raises(L.ClhaError):
        L.clha_factor_groups(ctx, groups * 2)   # more than FACTOR_MAX_GROUPS


def test_factor_non_pd_reports_column(ctx):
    d = 256
    H = torch.eye(d)
    H[200, 200] = -1.0
    Hd = H[None].to(DEV).contiguous()
    U = torch.empty_like(Hd)
    L.clha_factor(ctx, Hd, 1, d, U)
    with pytest.raises(L.ClhaError) as ei:
        L.clha_check(ctx)
    assert ei.value.status == L.ERR_NOT_PD
    assert "index 200" in str(ei.value)
    L.clha_check(ctx)   # the error is cleared


def test_factor_wait_limit_runs_out_and_context_recovers(ctx):
    """A bounded device wait that runs out (failure detection without a GPU fault): with a 1 us limit
    on the factor graph's dependency waits, the CTAs that wait for a diagonal task (about 30 us of
    work) give up, the graph aborts and returns, and the next synchronising call reports
    CLHA_ERR_TIMEOUT. With the default limit restored, the same context factors the same inputs
    correctly."""
    d, batch = 1024, 4
    g = _gen(7)
    Hs = []
    for b in range(batch):
        A = torch.randn((d, d // 4), generator=g).double()
        Hs.append((A @ A.T / (d // 4) + 0.05 * torch.eye(d, dtype=torch.float64)).float())
    Hd = torch.stack(Hs).to(DEV)
    U = torch.full_like(Hd, float("nan"))
    try:
        L.clha_set_factor_wait_limit(ctx, 1000)
        L.clha_factor(ctx, Hd, batch, d, U)
        with pytest.raises(L.ClhaError) as ei:
            L.clha_check(ctx)
        assert ei.value.status == L.ERR_TIMEOUT
        assert "clha_factor" in str(ei.value)
    finally:
        L.clha_set_factor_wait_limit(ctx, 0)
    L.clha_check(ctx)                      # the record was cleared
    U.fill_(float("nan"))
    L.clha_factor(ctx, Hd, batch, d, U)
    L.clha_check(ctx)
    for b in range(batch):
        got = U[b].double().cpu().numpy()
        assert np.all(np.tril(got, -1) == 0)
        assert rel_fro(got, O.factor(Hs[b].double().numpy())) < 1e-6


# ------------------------------------------------------------------------------------ GPTQ
def _H(d, seed, rank=None, damp=0.01):
    g = _gen(seed)
    A = torch.randn((d, rank or d // 2), generator=g).double()
    H = A @ A.T / A.shape[1] + torch.diag(torch.rand(d, generator=g).double() + 0.5)
    return H.numpy()


@pytest.mark.parametrize("form", ["inv", "block"])
@pytest.mark.parametrize("d_out,d_in,bits,wdt", [(256, 512, 2, torch.float32), (384, 1024, 3, torch.bfloat16),
                                                   (128, 128, 4, torch.bfloat16), (256, 256, 8, torch.float32),
                                                   (256, 1152, 4, torch.bfloat16)])
def test_quantize_matches_oracle_on_same_factor(ctx, d_out, d_in, bits, wdt, form):
    """GPTQ against the oracle's (the pages' recurrence with U). inv: both sides take the same float32 U.
    block: the kernel takes float32 F and runs the lazy and trailing updates on W_hat - W, the oracle
    the exact U. d_in = 1152: two full chunks of 512 columns and a ragged one of 128."""
    H = _H(d_in, d_in + bits)
    agg = O.aggregate([H], [2], "rt")
    U32 = np.ascontiguousarray(O.factor(agg["H_d"]), np.float32)
    W = (0.02 * torch.randn((d_out, d_in), generator=_gen(bits))).to(wdt)
    if form == "block":
        Ud = torch.from_numpy(np.ascontiguousarray(O.factor_block_scaled(agg["H_d"]), np.float32))[None].to(DEV)
        U_or = O.factor(agg["H_d"])
    else:
        Ud = torch.from_numpy(U32)[None].to(DEV)
        U_or = U32.astype(np.float64)
    fcode = L.FACTOR_BLOCK_CHOL if form == "block" else L.FACTOR_INV_CHOL
    Wd = W[None].to(DEV).contiguous()
    codes = torch.empty((1, d_out, d_in), dtype=torch.uint8, device=DEV)
    scales = torch.empty((1, d_out, d_in // 128), device=DEV)
    zeros = torch.empty((1, d_out, d_in // 128), dtype=torch.uint8, device=DEV)
    W_hat = torch.empty((1, d_out, d_in), device=DEV)
    lam = torch.tensor([agg["lam"]], dtype=torch.float64, device=DEV)
    loss = torch.full((1,), float("nan"), dtype=torch.float64, device=DEV)
    L.clha_quantize(ctx, Ud, 1, Wd, 1, d_out, d_in, bits, codes, scales, zeros, W_hat, lam=lam, loss=loss,
                    form=fcode)
    wc, ws, wz, wh, wm = O.gptq(to64(W), U_or, bits, 128, margins=True)
    print("codes", form, assert_codes(codes[0].cpu().numpy(), zeros[0].cpu().numpy(),
                                      dict(codes=wc, zeros=wz, margin=wm), (d_out, d_in, bits, form), bar=CONFIG_BAR))
    # first group of every row: identical inputs, so the grid is bit-identical
    np.testing.assert_array_equal(scales[0, :, 0].cpu().numpy(), ws[:, 0])
    np.testing.assert_array_equal(zeros[0, :, 0].cpu().numpy(), wz[:, 0])
    got_loss = O.loss(to64(W), to64(W_hat[0]), agg["H_comb"])
    want_loss = O.loss(to64(W), wh, agg["H_comb"])
    assert abs(got_loss - want_loss) <= 1e-3 * want_loss
    # the in-kernel loss (|E|^2 - lambda |W_hat - W|^2) is the trace of the same W_hat under H_comb
    assert abs(loss.item() - got_loss) <= 1e-5 * got_loss
    # W_hat is the dequantised code
    q = codes[0].float()
    s = scales[0].repeat_interleave(128, 1)
    z = zeros[0].float().repeat_interleave(128, 1)
    assert torch.equal(W_hat[0], s * (q - z))


@pytest.mark.parametrize("form", ["inv", "block"])
def test_quantize_diagonal_hessian_is_rtn_bit_exact(ctx, form):
    """A diagonal H makes U and F the same diagonal matrix: no column moves another, GPTQ is round to
    nearest in either form (d_in = 640: two chunks, so the trailing update adds exact zeros)."""
    d_out, d_in = 256, 640
    W = (0.02 * torch.randn((d_out, d_in), generator=_gen(3))).to(torch.bfloat16)
    H = np.diag(np.linspace(0.5, 2.0, d_in))
    Hd = O.aggregate([H], [2], "rt")["H_d"]
    U = O.factor(Hd)
    np.testing.assert_allclose(O.factor_block_scaled(Hd), U, rtol=1e-14)
    Ud = torch.from_numpy(np.ascontiguousarray(U, np.float32))[None].to(DEV)
    codes = torch.empty((1, d_out, d_in), dtype=torch.uint8, device=DEV)
    scales = torch.empty((1, d_out, d_in // 128), device=DEV)
    zeros = torch.empty((1, d_out, d_in // 128), dtype=torch.uint8, device=DEV)
    L.clha_quantize(ctx, Ud, 1, W[None].to(DEV).contiguous(), 1, d_out, d_in, 3, codes, scales, zeros, None,
                    form=L.FACTOR_BLOCK_CHOL if form == "block" else L.FACTOR_INV_CHOL)
    wc, ws, wz, _ = O.gptq(to64(W), U.astype(np.float32).astype(np.float64), 3, 128)
    np.testing.assert_array_equal(codes[0].cpu().numpy(), wc)
    np.testing.assert_array_equal(scales[0].cpu().numpy(), ws)
    np.testing.assert_array_equal(zeros[0].cpu().numpy(), wz)


@pytest.mark.parametrize("form", ["inv", "block"])
def test_quantize_batched_shared_factor(ctx, form):
    """n_u = 2: problems 0, 2 use factor 0 and problems 1, 3 factor 1 (gate and up stacked share one)."""
    d_out, d_in, bits = 128, 768, 3
    Hds = [O.aggregate([_H(d_in, s)], [2], "rt")["H_d"] for s in (1, 2)]
    Us = [np.ascontiguousarray(O.factor(h), np.float32) for h in Hds]
    W = (0.02 * torch.randn((4, d_out, d_in), generator=_gen(4))).to(torch.bfloat16)
    if form == "block":
        Ud = torch.from_numpy(np.stack([np.ascontiguousarray(O.factor_block_scaled(h), np.float32) for h in Hds]))
        Uor = [O.factor(h) for h in Hds]
    else:
        Ud = torch.from_numpy(np.stack(Us))
        Uor = [u.astype(np.float64) for u in Us]
    codes = torch.empty((4, d_out, d_in), dtype=torch.uint8, device=DEV)
    scales = torch.empty((4, d_out, d_in // 128), device=DEV)
    zeros = torch.empty((4, d_out, d_in // 128), dtype=torch.uint8, device=DEV)
    L.clha_quantize(ctx, Ud.to(DEV), 2, W.to(DEV), 4, d_out, d_in, bits, codes, scales, zeros, None,
                    form=L.FACTOR_BLOCK_CHOL if form == "block" else L.FACTOR_INV_CHOL)
    for b in range(4):
        wc, _, wz, _, wm = O.gptq(to64(W[b]), Uor[b % 2], bits, 128, margins=True)
        assert_codes(codes[b].cpu().numpy(), zeros[b].cpu().numpy(), dict(codes=wc, zeros=wz, margin=wm), b,
                     bar=CONFIG_BAR)


# ------------------------------------------------------------------------------------ loss
def test_loss_matches_oracle(ctx):
    d_out, d_in, batch = 256, 384, 3
    g = _gen(31)
    W = (0.02 * torch.randn((batch, d_out, d_in), generator=g)).to(torch.bfloat16)
    W_hat = (W.float() + 0.003 * torch.randn((batch, d_out, d_in), generator=g))
    Hs = [_H(d_in, s) for s in (5, 6)]
    H = torch.from_numpy(np.stack(Hs).astype(np.float32))
    got = L.clha_loss(ctx, W.to(DEV), W_hat.to(DEV), H.to(DEV), 2, batch, d_out, d_in)
    for b in range(batch):
        want = O.loss(to64(W[b]), to64(W_hat[b]), H[b % 2].double().numpy())
        assert abs(got[b] - want) <= 1e-5 * want
