"""The host-to-host calibration step (inputs copied in and outputs copied back on their own streams,
overlapped with the compute, inputs double-buffered) must give exactly what the same calls give on
resident inputs: the copies only move bytes, and every kernel on this small pair is deterministic
(each Gram tile takes one accumulation chunk, the factor applies its tile updates in a fixed order).
Oracle parity of the calibration itself is covered by the end-to-end tests."""
import pytest
import torch

from post_quantization_expert_b200.pipeline import PART_FIELDS, HostStep, MoECalibration, MoEWeights, stack_weights
from synth import workload

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.mark.parametrize("n_shared", [0, 2])
def test_host_step_matches_resident_path(ctx, n_shared):
    over = dict(tokens=2048)
    if n_shared:
        over.update(n_shared=n_shared, shared_dff=512)
    wl = workload(2, "cpu", **over)
    s = wl.spec
    X = [wl.x(l) for l in range(2)]
    lg = [wl.logits(l) for l in range(2)]
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    shared = [wl.expert_weights(0, i, shared=True) for i in range(s.n_shared)]
    modes = ("rt", "eq")
    mk = lambda: MoECalibration(ctx, 2, 2048, s.E, s.k, s.d_model, s.d_ff, s.n_shared, s.shared_dff,
                                s.bits_routed, s.bits_shared, s.damp_frac, modes=modes)
    # resident inputs
    w = stack_weights((routed, shared), DEV)
    ref = mk()
    for l in range(2):
        ref.collect(l, X[l].to(DEV), lg[l].to(DEV), w)
    ref.quantize(w, modes)
    # host inputs, host outputs, run twice (the second run reuses every buffer)
    wh = stack_weights((routed, shared), "cpu")
    pin = lambda t: None if t is None else t.pin_memory()
    hW = MoEWeights(pin(wh.Wgu), pin(wh.Wd), pin(wh.Sgu), pin(wh.Sd))
    hX, hL = [pin(x) for x in X], [pin(l) for l in lg]
    cal = mk()
    parts = ("gu", "d") + (("sgu", "sd") if n_shared else ())
    out = lambda m, p: getattr(ref.res[m], PART_FIELDS[p])
    hout = {m: {p: tuple(pin(torch.zeros_like(t, device="cpu"))
                         for t in (out(m, p).codes, out(m, p).scales, out(m, p).zeros))
                for p in parts} for m in modes}
    step = HostStep(cal, [x.shape for x in X], [l.shape for l in lg], hW)
    hloss = pin(torch.zeros(cal.loss_dev.shape, dtype=torch.float64))
    ref_loss = ref.loss_dev.cpu()
    for it in range(3):   # both input sets, then the first again; the losses read synchronously or not
        for m in modes:
            for trip in hout[m].values():
                for t in trip:
                    t.zero_()
        hloss.zero_()
        step.run(hX, hL, hW, hout, modes, hloss=hloss if it != 1 else None)
        step.join()
        torch.cuda.synchronize()
        if it != 1:
            assert (hloss - ref_loss).abs().max() <= 1e-12 * ref_loss.abs().max()
        for m in modes:
            for p in parts:
                q = out(m, p)
                for h, d in zip(hout[m][p], (q.codes, q.scales, q.zeros)):
                    assert torch.equal(h, d.cpu()), (m, p)
            # the in-kernel loss adds per-CTA float64 partial sums atomically: equal up to their order
            if it == 1:
                for a, b in ((cal.res[m].qg.loss, ref.res[m].qg.loss), (cal.res[m].qd.loss, ref.res[m].qd.loss)):
                    assert abs(a - b).max() <= 1e-12 * abs(b).max()
