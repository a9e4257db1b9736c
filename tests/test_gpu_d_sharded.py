"""Token-sharded collection + expert-parallel quantization, with the ranks simulated one after
another on one GPU (their kernels never wait on one another): the summed accumulators equal the
unsharded ones; each rank's first expert meets the oracle parity bar; every expert's codes agree with
the unsharded run up to the float32 summation order of the Hessians (GPTQ's column recurrence carries
a flipped code into the rest of its row, so two float32 runs differ by about as much as each differs
from the float64 oracle)."""
import numpy as np
import pytest
import torch

import oracle as O
from helpers import CodeTally, code_agreement, rel_fro, to64
from post_quantization_expert_b200 import clha as L
from post_quantization_expert_b200 import sharded as SH
from post_quantization_expert_b200.pipeline import MoECalibration, stack_weights
from synth import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_matches_unsharded(ctx, world):
    wl = workload(2, DEV)   # full size: 4096 tokens per layer leave each expert's Hessian nearly rank-deficient
    s = wl.spec
    n = s.tokens[0]
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    w = stack_weights((routed, []), DEV)
    X = [wl.x(l) for l in range(2)]
    lg = [wl.logits(l) for l in range(2)]
    modes = s.alpha_modes
    full = MoECalibration(ctx, 2, n, s.E, s.k, s.d_model, s.d_ff, 0, 0, s.bits_routed, s.bits_shared, s.damp_frac,
                          modes=modes)
    for l in range(2):
        full.collect(l, X[l], lg[l], w)
    full.quantize(w, modes)
    ranks = [SH.ShardedMoECalibration(ctx, r, world, 2, n // world + 1, s.E, s.k, s.d_model, s.d_ff,
                                      bits_routed=s.bits_routed, bits_shared=s.bits_shared, damp_frac=s.damp_frac,
                                      modes=modes) for r in range(world)]
    for r, rk in enumerate(ranks):
        t0, t1 = SH.token_range(n, r, world)
        for l in range(2):
            rk.collect(l, X[l][t0:t1].contiguous(), lg[l][t0:t1].contiguous(), w)
    SH.simulated_reduce([rk.reduce_tensors() for rk in ranks])
    torch.cuda.synchronize()
    for a_full, a_sh in ((full.acc_in, ranks[0].collector.acc_in), (full.acc_dn, ranks[-1].collector.acc_dn)):
        S_f, c_f = a_full.buffers()
        S_s, c_s = a_sh.buffers()
        assert torch.equal(c_f, c_s)
        # float32 sums taken in a different order (shards, then one add): ~1e-6 apart; a lost shard or
        # a wrong expert would be >= 1e-3 off
        assert rel_fro(torch.triu(S_s[1, 3]).double().cpu().numpy(), torch.triu(S_f[1, 3]).double().cpu().numpy()) < 1e-5
    X64 = [to64(x) for x in X]
    L64 = [l.cpu().numpy() for l in lg]
    tally = CodeTally(("sharded", world))
    for rk in ranks:
        res = rk.quantize(rk.local_weights(w), modes)
        e0, e1 = rk.e0, rk.e1
        for mode in modes:
            loc, ref = res[mode], full.res[mode]
            for name in ("qg", "qu", "qd"):
                got, want = getattr(loc, name), getattr(ref, name)
                for j, e in enumerate(range(e0, e1)):
                    assert code_agreement(got.codes[j].cpu().numpy(), want.codes[e].cpu().numpy()) >= 0.995
                np.testing.assert_allclose(got.loss, want.loss[e0:e1], rtol=1e-3)
            # the rank's first expert against the oracle on all tokens (the parity bar)
            only = [tuple(to64(t) for t in routed[e]) if e == e0 else None for e in range(s.E)]
            o = O.calibrate_moe_group(X64, L64, s.k, only, [], [e0], s.bits_routed, s.bits_shared, s.group, mode,
                                      s.damp_frac)
            r = o["experts"][("r", e0)]
            for name, q in (("gate", loc.qg), ("up", loc.qu), ("down", loc.qd)):
                tally.add(q.codes[0].cpu().numpy(), q.zeros[0].cpu().numpy(), r[name], (mode, e0, name))
            got_loss = loc.qg.loss[0] + loc.qu.loss[0] + loc.qd.loss[0]
            assert abs(got_loss - r["loss"]) <= 1e-3 * r["loss"]
    tally.check()
    # gathering each rank's gate codes in expert order reproduces the unsharded layout
    mode = modes[0]
    parts = [rk.quantizer.res[mode].qg.codes for rk in ranks]
    e_max = -(-s.E // world)

    def fake_all_gather(out, pad, _state={"i": 0}):
        for r in range(world):
            out[r].zero_()
            out[r][: parts[r].shape[0]].copy_(parts[r])

    got = SH.gather_expert_rows(parts[0], parts[0].shape[0], s.E, world, all_gather=fake_all_gather)
    assert got.shape[0] == s.E
    assert code_agreement(got.cpu().numpy(), full.res[mode].qg.codes.cpu().numpy()) >= 0.995


@pytest.mark.parametrize("world", [2, 3])
def test_owner_exchange_equals_all_reduce(ctx, world):
    """The owner exchange (packed upper triangles, reduce-scatter by owner, counts all-reduced) leaves
    in every rank's quantizer exactly the summed Hessians the all-reduce would: the E64 shape with two
    always-active experts (rank 0 owns them), ranks simulated one after another, sums in rank order on
    both paths, so the triangles are bit-identical; a quarter of the all-reduce's bytes cross."""
    wl = workload(3, DEV, tokens=1024)
    s = wl.spec
    n = s.tokens[0]
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    shared = [wl.expert_weights(0, i, shared=True) for i in range(s.n_shared)]
    w = stack_weights((routed, shared), DEV)
    X = [wl.x(l) for l in range(2)]
    lg = [wl.logits(l) for l in range(2)]
    ranks = [SH.ShardedMoECalibration(ctx, r, world, 2, n // world + 1, s.E, s.k, s.d_model, s.d_ff, s.n_shared,
                                      s.shared_dff, s.bits_routed, s.bits_shared, s.damp_frac) for r in range(world)]
    for r, rk in enumerate(ranks):
        t0, t1 = SH.token_range(n, r, world)
        for l in range(2):
            rk.collect(l, X[l][t0:t1].contiguous(), lg[l][t0:t1].contiguous(), w)
    launched = L.clha_kernel_launches(ctx)
    SH.exchange(ranks)
    assert L.clha_kernel_launches(ctx) > launched           # the packing runs in the library
    lay = ranks[0].layout
    full_bytes = sum(t.numel() * t.element_size() for t in ranks[0].reduce_tensors())
    # a reduce-scatter moves (world-1)/world of its buffer per rank, an all-reduce twice that
    assert world * lay.chunk * 4 < 0.55 * full_bytes
    # the all-reduce path on the collectors' Gram sums (counts were summed by the exchange already)
    SH.simulated_reduce([[rk.collector.acc_in.buffers()[0], rk.collector.acc_dn.buffers()[0],
                          rk.collector.acc_sdn.buffers()[0]] for rk in ranks])
    torch.cuda.synchronize()
    for rk in ranks:
        c, q = rk.collector, rk.quantizer
        e0, e1 = rk.e0, rk.e1
        pairs = [(q.acc_in, slice(0, e1 - e0), c.acc_in, slice(e0, e1)), (q.acc_dn, slice(0, e1 - e0), c.acc_dn, slice(e0, e1))]
        if rk.rank == 0:
            pairs += [(q.acc_in, slice(e1 - e0, e1 - e0 + 1), c.acc_in, slice(s.E, s.E + 1)),
                      (q.acc_sdn, slice(0, s.n_shared), c.acc_sdn, slice(0, s.n_shared))]
        for qa, qs, ca, cs in pairs:
            Sq, cq = qa.buffers()
            Sc, cc = ca.buffers()
            assert torch.equal(cq[:, qs], cc[:, cs])
            assert torch.equal(torch.triu(Sq[:, qs]), torch.triu(Sc[:, cs])), (rk.rank, qs, cs)
