"""Throughput of CLHA calibration on B200: weight columns quantized per second, end to end.

Default workload (the largest one that fits one GPU): one weight W [8192, 28672] bf16 shared by 4
layers, 65536 calibration tokens per layer (d_in 28672, rank-64 covariance plus diagonal, drift 0.3
between consecutive layers), routing-frequency alpha, 4-bit, group 128. One step = the whole hot
path: zero the accumulators, Gram of each layer's tokens (4 x 53.9 TFLOP), aggregate and damp,
inverse-Cholesky factor (15.7 TFLOP in float64), GPTQ of W (28672 columns) with its in-kernel loss.
Inputs are synthetic (seeded), resident in HBM (15 GB of X per step, far larger than L2; a 512 MB
flush write before every timed step as well).

  python bench.py [--gpus N --steps K --warmup W] [--impl ours|reference]

The MoE layer pair (E=16 routed experts, top-2, d_model 1024, d_ff 512, 8192 tokens per layer,
3-bit; route -> gather -> Hessians -> expert activation -> down-projection Hessians per layer, then
for both weightings aggregate -> factor -> GPTQ of gate, up and down -> loss):
  python bench.py --workload moe-e16 [--parallel replicas|tokens]

Kernel-level workloads (one JSON line per shape; used for the profiles and the roofline tables):
  python bench.py --workload act --shape 18432x1024x512 ...   expert activation, dense bf16 X [n, d_model]
  python bench.py --workload hessian --shape 65536x4096 ...   Gram accumulation of dense bf16 X [n, d]
  python bench.py --workload gptq --shape 32x512x1024 ...     GPTQ of [batch, d_out, d_in] bf16 weights
  python bench.py --workload factor --shape 32x1024 ...       inverse-Cholesky factor of [batch, d, d]
  python bench.py --workload epmq --shape 8x4096x4096 ...     E-PMQ target W* = R H^-1 of K source experts
  python bench.py --workload dequant --shape 8192x4096x4096   deployable layer from 3-bit packed codes

Routing-sharpness sweep (not a throughput line; one JSON line per sharpness):
  python bench.py --workload sweep [--sharpness 0 0.1 ...]   the layer pair above at rising cross-layer
      routing divergence: per-layer calibration (alpha = (1, 0)) against CLHA rt and eq, each scored on
      the calibration hook layer and on fresh held-out tokens of both layers

With N > 1 (torchrun, one process per GPU) every rank calibrates its own independent weight (or
layer pair): weak scaling, no data-path collective; the step time is the max over ranks. With
--workload moe-e16 --parallel tokens the ranks share one layer pair instead: each collects its share
of the tokens, one NCCL reduce-scatter sums the packed upper triangles of the Hessian accumulators
onto the rank that quantizes each expert, and each quantizes its own range of experts (strong
scaling).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "sm_max_mhz": 1965.0}
N_SMS = 148
METRIC = "expert weight columns quantized/sec (CLHA-GPTQ end to end)"
DENSE_CPU_CHANNELS = 2560     # the oracle's bounded sample of the dense workload: this principal block


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


FORMS = {"inv": 0, "block": 1}   # clha_factor_form: CLHA_FACTOR_INV_CHOL, CLHA_FACTOR_BLOCK_CHOL


def factor_work(d: int, form: int) -> int:
    """Algorithmic flops of one factor: U takes the Cholesky and the triangular inverse (2d^3/3); F the
    Cholesky (d^3/3) and the block scaling, F_ab = R_ab U_bb above the diagonal blocks: per 64 rows of a
    128-column block three 64^3 tile products (L_ip D_p + L_i,p+1 X and L_i,p+1 D_p+1), 192 flops per
    element of the upper triangle, 96 d^2."""
    return 2 * d ** 3 // 3 if form == FORMS["inv"] else d ** 3 // 3 + 96 * d * d


def gram_kernel(d: int) -> str:
    """The kernel of one dense Gram: pairs of SMs from d = 4096 (the library's threshold)."""
    if d >= 4096:
        return "syrk_bf16_pair (tcgen05 kind::f16, cta_group::2: 256x256 tiles on SM pairs)"
    return "syrk_bf16_tc (tcgen05 kind::f16)"


def factor_kernels(form: int) -> str:
    if form == FORMS["inv"]:
        return "fac_load + fac_dag + fac_store (fp64 tile-task graph, mma.sync m8n8k4 f64)"
    return "fac_load + fac_dag (Cholesky only) + fac_pair + fac_store_f (fp64, mma.sync m8n8k4 f64)"


def alu_peaks(peaks):
    """Nominal SIMT peaks at the maximum SM clock (128 FP32 and 64 FP64 FMA lanes per SM), and the
    3xTF32 product rate: the tf32 tensor peak (the measured bf16 peak times the nominal tf32/bf16
    ratio, 1.1 / 2.25 PFLOP/s) divided by the three tf32 products of each float32-class product."""
    mhz = peaks.get("sm_max_mhz", 1965.0)
    tf32 = peaks["bf16_tflops"] * 1.1 / 2.25
    return {"fp32_tflops": N_SMS * 128 * 2 * mhz * 1e6 / 1e12, "fp64_tflops": N_SMS * 64 * 2 * mhz * 1e6 / 1e12,
            "tf32x3_tflops": tf32 / 3}


class ClockSampler:
    """nvidia-smi clock / throttle-reason samples (every 20 ms, with timestamps); only those taken
    inside the timed region's host-time window count."""
    Q = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.dev = device_index
        self.proc = None
        self.path = None
        self.window = None

    def start(self):
        """Start sampling and wait (up to 5 s) until the first sample is written."""
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.dev), f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "20"],
                                         stdout=self.f, stderr=subprocess.DEVNULL)
            t0 = time.time()
            while time.time() - t0 < 5.0 and os.path.getsize(self.path) == 0:
                time.sleep(0.01)
        except Exception:
            self.proc = None

    def mark(self, t_begin: float, t_end: float):
        """Host-time window of the timed region."""
        self.window = (t_begin, t_end)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.f.close()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    ts = time.mktime(time.strptime(parts[0].split(".")[0], "%Y/%m/%d %H:%M:%S"))
                    ts += float("0." + parts[0].split(".")[1]) if "." in parts[0] else 0.0
                    rows.append((ts, float(parts[2]), float(parts[3]), parts[6:10]))
                except (ValueError, IndexError):
                    continue
        os.unlink(self.path)
        if not rows:
            return None
        inside = rows
        if self.window:
            a, b = self.window
            sel = [r for r in rows if a - 0.025 <= r[0] <= b + 0.025]
            if sel:
                inside = sel
        reasons = set()
        for r in inside:
            for n, v in zip(names, r[3]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": inside[-1][2],
                "reasons": sorted(reasons), "samples": len(inside),
                "window": "timed region" if inside is not rows else "whole run (no sample inside the timed region)"}


def dist_setup(backend: str | None = None):
    """One process per GPU under torchrun (RANK / LOCAL_RANK / WORLD_SIZE / MASTER_* from the env).
    NCCL on GPUs; gloo when asked for (the CPU tests of this multi-rank logic). The process group
    has a short timeout so ranks that wait for a missing peer end with an error."""
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import torch
        import torch.distributed as dist
        from datetime import timedelta
        backend = backend or "nccl"
        if backend == "nccl":
            torch.cuda.set_device(local)
            dist.init_process_group("nccl", timeout=timedelta(seconds=120), device_id=torch.device("cuda", local))
        else:
            dist.init_process_group(backend, timeout=timedelta(seconds=120))
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's figure (the job's time is set by it)."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(units_per_step_per_rank: float, ms_max: float, world: int) -> float:
    """Whole-job throughput under weak scaling: every rank processes its own units each step, and
    the step takes as long as the slowest rank."""
    return world * units_per_step_per_rank / (ms_max / 1e3)


def rank_seed(rank: int, base: int = 1235) -> int:
    """Each rank calibrates its own independent problem: a distinct, reproducible input seed (rank 0
    keeps the workload's own seed)."""
    return base + 7919 * rank


KERNEL_SOURCES = {"act": ("ffn_act.cu", "ffn_act_tc.cu"), "gptq": ("gptq.cu",), "hessian": ("hessian.cu",),
                  "aggregate": ("aggregate.cu",), "factor": ("factor.cu",)}


def source_hash(phase: str) -> str:
    """sha1 prefix of the phase's kernel source file(s), concatenated in order."""
    import hashlib
    h = hashlib.sha1()
    for name in KERNEL_SOURCES[phase]:
        with open(os.path.join(ROOT, "post_quantization_expert_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()[:12]


def measured_traffic(phase: str, workload: str):
    """DRAM bytes per step of a phase from profiles/dram_traffic.txt, only while the kernel source is
    the one the counters were taken on (its hash is recorded beside the figure)."""
    path = os.path.join(ROOT, "profiles", "dram_traffic.txt")
    if not os.path.exists(path):
        return None
    cur = source_hash(phase)
    with open(path) as f:
        for line in f:
            parts = line.split()
            if len(parts) >= 4 and not line.startswith("#") and parts[0] == phase and parts[1] == workload \
                    and parts[2] == cur:
                return float(parts[3])
    return None


def blas_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        return max(n) if n else 1
    except Exception:
        return os.cpu_count() or 1


# ------------------------------------------------------------------------------------------ workload
MOE_CONFIGS = {"moe-e16": 2, "moe-e64": 3}   # the E16 top-2 pair; the E64 top-6 pair with 2 always-active experts


def make_inputs(rank: int, cfg: int = 2):
    from synth import workload
    wl = workload(cfg, "cpu", seed=rank_seed(rank))
    s = wl.spec
    X = [wl.x(l) for l in range(2)]
    lg = [wl.logits(l) for l in range(2)]
    routed = [wl.expert_weights(0, e) for e in range(s.E)]
    shared = [wl.expert_weights(0, i, shared=True) for i in range(s.n_shared)]
    return wl, X, lg, routed, shared


def moe_sample_experts(spec, first: int = 0):
    """The routed experts of one bounded oracle sample (about 10 s of host work): 8 of the E16 pair's,
    4 of the E64 pair's."""
    n = 8 if spec.E <= 16 else 4
    return [(first + j) % spec.E for j in range(n)]


def oracle_sample(X, lg, routed, spec, experts):
    """The float64 oracle on a bounded sample of the workload: the listed routed experts' full paths,
    every weighting (routing of both layers is computed in full)."""
    import oracle as O
    X64 = [x.double().numpy() for x in X]
    L64 = [l.numpy() for l in lg]
    W64 = {e: tuple(t.double().numpy() for t in routed[e]) for e in experts}
    cols = 0
    for mode in spec.alpha_modes:
        O.calibrate_moe_group(X64, L64, spec.k, [W64.get(e) for e in range(spec.E)], (), list(experts),
                              spec.bits_routed, spec.bits_shared, spec.group, mode, spec.damp_frac)
        cols += len(experts) * (2 * spec.d_model + spec.d_ff)
    return cols


def run_reference(args, world, rank):
    if rank != 0:
        return 0
    wl, X, lg, routed, _ = make_inputs(0, MOE_CONFIGS[args.workload])
    s = wl.spec
    n_ex = len(moe_sample_experts(s))
    for i in range(args.warmup):
        oracle_sample(X, lg, routed, s, moe_sample_experts(s, i * n_ex))
    times, cols = [], 0
    for i in range(args.steps):
        t0 = time.perf_counter()
        cols = oracle_sample(X, lg, routed, s, moe_sample_experts(s, (args.warmup + i) * n_ex))
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = cols / (ms / 1e3)
    sample = (f"{n_ex} routed experts per step (gate, up, down) through route, gather, Hessians, aggregate, "
              f"factor, GPTQ and loss, weightings {'/'.join(s.alpha_modes)}")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "columns/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": s.name, "columns_per_step": cols, "l2": "n/a (host)"},
            "cpu_baseline": {"value": value, "unit": "columns/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "columns/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_ours(args, world, rank, local):
    import numpy as np
    import torch
    from post_quantization_expert_b200 import clha as L
    from post_quantization_expert_b200.pipeline import MoECalibration, PhaseTimer, stack_weights

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    sharded = args.parallel == "tokens"
    # replicas: every rank calibrates its own pair; tokens: one pair, tokens and experts split over ranks
    wl, X, lg, routed, shared = make_inputs(0 if sharded else rank, MOE_CONFIGS[args.workload])
    s = wl.spec
    ns, sdff = s.n_shared, s.shared_dff
    ctx = L.Context(local)
    timer = PhaseTimer(ctx.stream)
    w = stack_weights((routed, shared), dev)
    modes = s.alpha_modes
    if sharded:
        from post_quantization_expert_b200 import sharded as SH
        t0, t1 = SH.token_range(s.tokens[0], rank, world)
        X, lg = [x[t0:t1].contiguous() for x in X], [l[t0:t1].contiguous() for l in lg]
        sh = SH.ShardedMoECalibration(ctx, rank, world, 2, t1 - t0, s.E, s.k, s.d_model, s.d_ff,
                                      bits_routed=s.bits_routed, bits_shared=s.bits_shared, damp_frac=s.damp_frac,
                                      timer=timer, modes=modes)
        cal, qcal, wq = sh.collector, sh.quantizer, sh.local_weights(w)
        cols_per_step = cal.columns() * len(modes) / world      # the pair's columns, per rank on average
    else:
        cal = qcal = MoECalibration(ctx, 2, max(s.tokens), s.E, s.k, s.d_model, s.d_ff, ns, sdff, s.bits_routed,
                                    s.bits_shared, s.damp_frac, timer=timer, modes=modes,
                                    factor_form=FORMS[args.factor_form])
        wq = w
        cols_per_step = cal.columns() * len(modes)
    Xd = [x.to(dev) for x in X]
    Ld = [l.to(dev) for l in lg]
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def calibrate():
        cal.reset()
        for l in range(2):
            cal.collect(l, Xd[l], Ld[l], w)
        if sharded:
            if world > 1:   # packed upper triangles reduce-scattered to their owners, counts all-reduced
                with timer.span("exchange"):
                    SH.exchange([sh], SH.dist_reduce_scatter, SH.dist_reduce)
            sh.quantize(wq, modes)
        else:
            cal.quantize(w, modes)

    def step():
        calibrate()

    timer.enabled = False
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    timer.enabled = True
    timer.reset()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = L.clha_kernel_launches(ctx)
    ev = []
    stream = ctx.stream
    t_begin = time.time()
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    clocks.mark(t_begin, time.time())
    launches = L.clha_kernel_launches(ctx) - launches0
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    timer.collect()
    ms = max_over_ranks(statistics.mean(step_ms), world)
    value = job_value(cols_per_step, ms, world)

    # ---- end to end through the public API with host buffers (pinned), copies inside the timed region
    pin = lambda t: t.pin_memory()
    hX, hL = [pin(x) for x in X], [pin(l) for l in lg]
    hW = [pin(w.Wgu.cpu()), pin(w.Wd.cpu())] + ([pin(w.Sgu.cpu()), pin(w.Sd.cpu())] if ns else [])
    outs = {m: {"gu": qcal.res[m].qgu, "d": qcal.res[m].qd} for m in modes}
    if ns:
        for m in modes:
            outs[m].update({"sgu": qcal.res[m].sgu, "sd": qcal.res[m].sd})
    hout = {m: {k: (pin(torch.empty_like(q.codes, device="cpu")), pin(torch.empty_like(q.scales, device="cpu")),
                    pin(torch.empty_like(q.zeros, device="cpu"))) for k, q in outs[m].items()} for m in modes}
    h2d = sum(t.numel() * t.element_size() for t in hX + hL + hW)
    d2h = sum(t.numel() * t.element_size() for m in modes for trip in hout[m].values() for t in trip)
    timer.enabled = False
    if not sharded:
        from post_quantization_expert_b200.pipeline import HostStep, MoEWeights
        host_step = HostStep(cal, [x.shape for x in X], [l.shape for l in lg], MoEWeights(*hW))
        hloss = pin(torch.empty(cal.loss_dev.shape, dtype=torch.float64))
        d2h += hloss.numel() * hloss.element_size()

    def e2e_step():
        if not sharded:     # copies on their own streams, overlapped with this step's and the next's compute
            host_step.run(hX, hL, MoEWeights(*hW), hout, modes, hloss=hloss)
            return
        with torch.cuda.stream(stream):
            for d_, h_ in zip(Xd + Ld + [w.Wgu, w.Wd], hX + hL + hW):
                d_.copy_(h_, non_blocking=True)
            wq.Wgu.copy_(torch.cat([w.Wgu[sh.e0:sh.e1], w.Wgu[s.E + sh.e0:s.E + sh.e1]]))
            wq.Wd.copy_(w.Wd[sh.e0:sh.e1])
            calibrate()
            for m in modes:
                for k, (hc, hs, hz) in hout[m].items():
                    q = outs[m][k]
                    hc.copy_(q.codes, non_blocking=True)
                    hs.copy_(q.scales, non_blocking=True)
                    hz.copy_(q.zeros, non_blocking=True)

    for _ in range(2):
        e2e_step()
    if not sharded:
        host_step.join()
    torch.cuda.synchronize()
    barrier(world)
    # one event pair around all K steps: a step's input copies overlap the previous step's compute
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        flush.zero_()
        e2e_step()
    if not sharded:
        host_step.join()
    b.record(stream)
    torch.cuda.synchronize()
    clk = clocks.stop()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, world)

    # ---- per-phase timing and the roofline of the dominant kernel
    K = args.steps
    phase_ms = {k: v / K for k, v in timer.totals.items()}
    phase_calls = {k: v // K for k, v in timer.counts.items()}
    counts = [cal.counts[l].cpu().numpy().astype(np.int64) for l in range(2)]
    dm, dff, E = s.d_model, s.d_ff, s.E
    hess_flops = sum(int(c.sum()) * (dm * (dm + 1) + dff * (dff + 1)) for c in counts)
    act_flops = sum(int(c.sum()) * 4 * dm * dff for c in counts)
    Eq = (sh.e1 - sh.e0) if sharded else E                  # experts this rank quantizes
    mats = [(dff, dm)] * (2 * Eq) + [(dm, dff)] * Eq        # gate, up, down per weighting
    factor_flops = len(modes) * Eq * (factor_work(dm, cal.form) + factor_work(dff, cal.form))
    # per slot and weighting: both layers' upper triangles of S read, the damped aggregate written (full)
    agg = lambda d: 2 * (d * (d + 1) // 2) * 4 + d * d * 4
    agg_bytes = len(modes) * Eq * (agg(dm) + agg(dff))
    if ns:   # always-active experts: every token, one shared input Gram, one down Gram each
        for n_l in s.tokens[:2]:
            hess_flops += n_l * (dm * (dm + 1) + ns * sdff * (sdff + 1))
            act_flops += n_l * ns * 4 * dm * sdff
        mats += [(sdff, dm)] * (2 * ns) + [(dm, sdff)] * ns
        factor_flops += len(modes) * (factor_work(dm, cal.form) + ns * factor_work(sdff, cal.form))
        agg_bytes += len(modes) * (agg(dm) + ns * agg(sdff))
    gptq_flops = len(modes) * sum(o * i * i for o, i in mats)
    loss_flops = len(modes) * sum(2 * o * i * i for o, i in mats)
    peaks, src = load_peaks()
    alu = alu_peaks(peaks)
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    act_tc = L.clha_last_act_kernel(ctx) == L.ACT_TENSOR   # the activation kernel the steps took
    kernels = {
        "hessian": ("tensor", hess_flops / 1e12, sustained, "TFLOP/s", "syrk_bf16_tc (tcgen05 kind::f16)"),
        "gptq": ("tensor", gptq_flops / 1e12, alu["tf32x3_tflops"], "TFLOP/s",
                 "gptq_tc + gptq_trail (column sweep in fp32; lazy and trailing updates on tcgen05 kind::tf32, "
                 "3xTF32; peak: tf32 / 3)"),
        "factor": ("alu", factor_flops / 1e12, alu["fp64_tflops"], "TFLOP/s", factor_kernels(cal.form)),
        "loss": ("alu", loss_flops / 1e12, alu["fp32_tflops"], "TFLOP/s", "loss_simt (fp32 FMA)"),
        "act": (("tensor", act_flops / 1e12, sustained, "TFLOP/s", "expert_act_tc (tcgen05 kind::f16)") if act_tc else
                ("alu", act_flops / 1e12, alu["fp32_tflops"], "TFLOP/s", "expert_act_simt (fp32 FMA)")),
        "aggregate": ("hbm", agg_bytes / 1e9, peaks["hbm_gbs"], "GB/s", "agg_combine"),
    }
    # the dominant kernel: the phase that takes longest per step (each is one kernel per call, the
    # factor one graph kernel between a load and a store); traffic is DRAM bytes per call
    single = ("act", "gptq", "hessian", "aggregate", "factor")
    dom = max((k for k in phase_ms if k in single), key=lambda k: phase_ms[k])
    bound, work, peak, unit, kname = kernels[dom]
    achieved = work / (phase_ms[dom] / 1e3)
    step_bytes = measured_traffic(dom, "moe-E16" if s.E == 16 else s.name)   # per step; per timed call
    traffic = step_bytes / phase_calls[dom] if step_bytes is not None and phase_calls.get(dom) else None
    phases = {k: {"ms": round(v, 4)} for k, v in sorted(phase_ms.items(), key=lambda kv: -kv[1])}
    for k, v in phases.items():
        if k in kernels:
            b_, wk, pk, un, _ = kernels[k]
            v["achieved"] = round(wk / (phase_ms[k] / 1e3), 3)
            v["unit"] = un
            v["frac"] = round(v["achieved"] / pk, 4)
    hess_tflops = hess_flops / 1e12 / (phase_ms["hessian"] / 1e3)

    # ---- the oracle on the host cores, bounded sample (rank 0, N = 1 only)
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        t0 = time.perf_counter()
        ex = moe_sample_experts(s)
        c = oracle_sample(X, lg, routed, s, ex)
        dt = time.perf_counter() - t0
        cpu = {"value": c / dt, "unit": "columns/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"routed experts {ex[0]}..{ex[-1]} of the layer pair (gate, up, down; weightings "
                         f"{'/'.join(modes)}; {c} columns) in {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "columns/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "strong" if sharded else "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": s.name, "global_batch": world * sum(s.tokens), "tokens_per_layer": s.tokens[0],
                       "E": E, "top_k": s.k, "d_model": dm, "d_ff": dff, "bits": s.bits_routed,
                       "always_active": ns, "always_active_d_ff": sdff, "always_active_bits": s.bits_shared if ns else None,
                       "weightings": list(modes), "columns_per_step_per_gpu": cols_per_step,
                       "parallelism": (f"tokens{world}+experts{world} (NCCL reduce-scatter of packed S triangles to owners)" if sharded
                                       else f"replicas{world}") if world > 1 else "single",
                       "l2": "flushed (512 MB write) before every timed step"},
            "weights_per_s": value * 3 * (E + ns) / cal.columns(),   # matrices: gate, up, down of every expert
            "hessian_tflops": hess_tflops,
            "hessian_frac_of_bf16_peak": hess_tflops / sustained,
            "roofline": {"kernel": kname, "phase": dom, "bound": bound, "achieved": achieved, "peak": peak,
                         "unit": unit, "frac": achieved / peak, "traffic": traffic,
                         "calls_per_step": phase_calls.get(dom),
                         "peak_source": src if bound in ("tensor", "hbm") else "derived (SM count x lanes x max clock)"},
            "phases_ms_per_step": phases,
            "e2e": {"value": job_value(cols_per_step, e2e_ms, world), "unit": "columns/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    ctx.close()
    return 0


# ------------------------------------------------------------------------------ dense stress workload
def dense_oracle_sample(Xs, W, spec, channels: int = DENSE_CPU_CHANNELS):
    """The float64 oracle on a bounded sample of the dense workload: the same calibration restricted to
    the first `channels` input channels (each layer's Gram over all its tokens on that principal block,
    routing-frequency aggregate and damping, factor, GPTQ of every row of W on those columns, loss).
    Returns the columns quantized."""
    import numpy as np
    import oracle as O
    X64 = [np.ascontiguousarray(x[:, :channels].double().cpu().numpy()) for x in Xs]
    W64 = W[:, :channels].double().cpu().numpy()
    O.calibrate_dense(W64, X64, spec.bits_routed, spec.group, "rt", None, spec.damp_frac)
    return channels


def dense_inputs(rank: int, device):
    from synth import workload
    wl = workload(5, device)
    wl = workload(5, device, seed=rank_seed(rank, wl.spec.seed))
    return wl


def run_reference_dense(args, world, rank):
    """The oracle arm: each step the float64 oracle on the bounded sample of the dense workload."""
    if rank != 0:
        return 0
    import torch
    dev = "cuda" if torch.cuda.is_available() else "cpu"   # inputs drawn where the GPU arm draws them
    wl = dense_inputs(0, dev)
    s = wl.spec
    C = DENSE_CPU_CHANNELS
    Xs = [wl.x(l, cache=False)[:, :C].cpu() for l in range(s.n_layers)]
    W = wl.dense_weight().cpu()
    for _ in range(args.warmup):
        dense_oracle_sample(Xs, W, s)
    times = []
    for _ in range(args.steps):
        t0 = time.perf_counter()
        cols = dense_oracle_sample(Xs, W, s)
        times.append(time.perf_counter() - t0)
    ms = 1e3 * statistics.mean(times)
    value = cols / (ms / 1e3)
    sample = (f"the calibration restricted to the first {C} of {s.d_model} input channels: Gram of all "
              f"{s.n_layers} x {s.tokens[0]} tokens on that block, aggregate, factor, GPTQ of all {s.d_out} rows "
              f"on those {C} columns, loss")
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "columns/s", "n_gpus": 1,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": s.name, "columns_per_step": cols, "l2": "n/a (host)"},
            "cpu_baseline": {"value": value, "unit": "columns/s", "cores": blas_threads(), "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "columns/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))
    return 0


def run_dense(args, world, rank, local):
    """One weight shared by 4 layers (the largest single-GPU workload): every rank calibrates its own."""
    import torch
    from post_quantization_expert_b200 import clha as L
    from post_quantization_expert_b200.pipeline import DenseCalibration, DenseHostStep, PhaseTimer

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    wl = dense_inputs(rank, dev)
    s = wl.spec
    nl, n, d, d_out = s.n_layers, s.tokens[0], s.d_model, s.d_out
    ctx = L.Context(local)
    timer = PhaseTimer(ctx.stream)
    cal = DenseCalibration(ctx, d_out, d, nl, s.bits_routed, s.damp_frac, timer=timer, keep_hcomb=False,
                           factor_form=FORMS[args.factor_form])
    W = wl.dense_weight()
    Xd = [wl.x(l, cache=False) for l in range(nl)]
    torch.cuda.synchronize()
    flush = torch.empty(512 << 20, dtype=torch.uint8, device=dev)
    cols_per_step = d

    def step():
        cal.reset()
        for l in range(nl):
            cal.collect(l, Xd[l])
        cal.quantize(W, "rt", read_loss=False)

    timer.enabled = False
    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    L.clha_check(ctx)
    timer.enabled = True
    timer.reset()
    barrier(world)
    torch.cuda.synchronize()
    clocks = ClockSampler(local)
    clocks.start()
    launches0 = L.clha_kernel_launches(ctx)
    ev = []
    stream = ctx.stream
    t_begin = time.time()
    for _ in range(args.steps):
        flush.zero_()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        step()
        b.record(stream)
        ev.append((a, b))
    torch.cuda.synchronize()
    t_end = time.time()
    launches = L.clha_kernel_launches(ctx) - launches0
    L.clha_check(ctx)
    barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    timer.collect()
    ms = max_over_ranks(statistics.mean(step_ms), world)
    value = job_value(cols_per_step, ms, world)
    loss_dev = float(cal.loss_dev[0].item())

    # ---- end to end through the public API: pinned host X and W in, codes / scales / zeros / loss out
    timer.enabled = False
    hX = [x.cpu().pin_memory() for x in Xd]
    hW = W.cpu().pin_memory()
    del Xd
    torch.cuda.empty_cache()
    q = cal.q
    hout = tuple(torch.empty(t.shape, dtype=t.dtype).pin_memory() for t in (q.codes, q.scales, q.zeros))
    hloss = torch.empty(1, dtype=torch.float64).pin_memory()
    h2d = sum(t.numel() * t.element_size() for t in hX) + hW.numel() * hW.element_size()
    d2h = sum(t.numel() * t.element_size() for t in hout) + 8
    hs = DenseHostStep(cal, [x.shape for x in hX], hX[0].dtype, hW.shape, hW.dtype)
    for _ in range(2):
        hs.run(hX, hW, hout, hloss)
    hs.join()
    torch.cuda.synchronize()
    barrier(world)
    clocks.mark(t_begin, t_end)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(stream)
    for _ in range(args.steps):
        flush.zero_()
        hs.run(hX, hW, hout, hloss)
    hs.join()
    b.record(stream)
    torch.cuda.synchronize()
    L.clha_check(ctx)
    clk = clocks.stop()
    e2e_ms = max_over_ranks(a.elapsed_time(b) / args.steps, world)
    assert abs(float(hloss[0]) - loss_dev) <= 1e-9 * abs(loss_dev), (float(hloss[0]), loss_dev)   # same inputs

    # ---- per-phase rates and the roofline of the dominant kernel
    K = args.steps
    phase_ms = {k: v / K for k, v in timer.totals.items()}
    phase_calls = {k: v // K for k, v in timer.counts.items()}
    peaks, src = load_peaks()
    alu = alu_peaks(peaks)
    sustained = peaks.get("bf16_tflops_sustained", peaks["bf16_tflops"])
    hess_flops = nl * n * d * (d + 1)
    factor_flops = factor_work(d, cal.form)
    gptq_flops = d_out * d * d
    agg_bytes = nl * (d * (d + 1) // 2) * 4 + d * d * 4     # every layer's upper triangle read, H_d written
    kernels = {
        "hessian": ("tensor", hess_flops / 1e12, sustained, "TFLOP/s", gram_kernel(d)),
        "factor": ("alu", factor_flops / 1e12, alu["fp64_tflops"], "TFLOP/s", factor_kernels(cal.form)),
        "gptq": ("tensor", gptq_flops / 1e12, alu["tf32x3_tflops"], "TFLOP/s",
                 "gptq_tc + gptq_trail (column sweep in fp32; lazy and trailing updates on tcgen05 kind::tf32, "
                 "3xTF32; peak: tf32 / 3)"),
        "aggregate": ("hbm", agg_bytes / 1e9, peaks["hbm_gbs"], "GB/s", "agg_combine"),
    }
    dom = max((k for k in phase_ms if k in kernels), key=lambda k: phase_ms[k])
    bound, work, peak, unit, kname = kernels[dom]
    achieved = work / (phase_ms[dom] / 1e3)
    step_bytes = measured_traffic(dom, "dense-stress")
    traffic = step_bytes / phase_calls[dom] if step_bytes is not None and phase_calls.get(dom) else None
    phases = {k: {"ms": round(v, 3)} for k, v in sorted(phase_ms.items(), key=lambda kv: -kv[1])}
    for k, v in phases.items():
        if k in kernels:
            _, wk, pk, un, _ = kernels[k]
            v["achieved"] = round(wk / (phase_ms[k] / 1e3), 3)
            v["unit"] = un
            v["frac"] = round(v["achieved"] / pk, 4)
    hess_tflops = hess_flops / 1e12 / (phase_ms["hessian"] / 1e3)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        C = DENSE_CPU_CHANNELS
        Xs = [wl.x(l, cache=False)[:, :C].cpu() for l in range(nl)]
        t0 = time.perf_counter()
        c = dense_oracle_sample(Xs, W.cpu(), s)
        dt = time.perf_counter() - t0
        cpu = {"value": c / dt, "unit": "columns/s", "cores": blas_threads(), "kind": "oracle",
               "sample": f"the calibration restricted to the first {C} of {d} input channels (Gram of all "
                         f"{nl} x {n} tokens on that block, aggregate, factor, GPTQ of all {d_out} rows on "
                         f"those columns, loss): {c} columns in {dt:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "columns/s", "n_gpus": world, "steps": K,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": s.name, "global_batch": world * nl * n, "tokens_per_layer": n,
                       "layers": nl, "d_out": d_out, "d_in": d, "bits": s.bits_routed, "group": s.group,
                       "weighting": "rt", "columns_per_step_per_gpu": cols_per_step,
                       "parallelism": f"replicas{world}" if world > 1 else "single",
                       "l2": "inputs larger than L2 (15 GB of X read per step) and a 512 MB flush write "
                             "before every timed step"},
            "weights_per_s": value / d,   # one weight [d_out, d] per step per GPU
            "hessian_tflops": hess_tflops,
            "hessian_frac_of_bf16_peak": hess_tflops / sustained,
            "hessian_peak": "bf16 sustained (the step lasts about a second)",
            "roofline": {"kernel": kname, "phase": dom, "bound": bound, "achieved": achieved, "peak": peak,
                         "unit": unit, "frac": achieved / peak, "traffic": traffic,
                         "calls_per_step": phase_calls.get(dom),
                         "peak_source": src if bound in ("tensor", "hbm") else "derived (SM count x lanes x max clock)"},
            "phases_ms_per_step": phases,
            "e2e": {"value": job_value(cols_per_step, e2e_ms, world), "unit": "columns/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
            "gpu_launches": int(launches),
            "clocks": clk,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    ctx.close()
    return 0


def run_sweep(args):
    """Calibration- and test-side Hessian error of per-layer calibration (PLIC) and CLHA (rt, eq) as
    the per-layer expert preference sharpens (the CLHA page, section 4). Synthetic tokens and weights:
    the pages' numbers are perplexities of a trained model, which this does not reproduce."""
    import numpy as np
    import torch
    from synth import workload
    from post_quantization_expert_b200 import clha as L
    from post_quantization_expert_b200.analysis import HessianError, mean_pairwise, routing_divergence
    from post_quantization_expert_b200.pipeline import MoECalibration, stack_weights
    ctx = L.Context(0)
    rows = []
    for beta in args.sharpness:
        cal_wl = workload(2, "cpu", sharpness=beta)
        test_wl = workload(2, "cpu", sharpness=beta, split="test")
        s = cal_wl.spec
        w = stack_weights(([cal_wl.expert_weights(0, e) for e in range(s.E)], []), "cuda")
        mk = lambda modes: MoECalibration(ctx, 2, max(s.tokens), s.E, s.k, s.d_model, s.d_ff, 0, 0, s.bits_routed,
                                          s.bits_shared, s.damp_frac, modes=modes)
        cal, held = mk(("explicit", "rt", "eq")), mk(("rt",))
        for col, wl in ((cal, cal_wl), (held, test_wl)):
            for l in range(2):
                col.collect(l, wl.x(l).to("cuda"), wl.logits(l).to("cuda"), w)
        counts = cal.acc_in.buffers()[1][:, : s.E].cpu().numpy()
        hook = (1.0, 0.0)
        cal.quantize(w, alpha=hook)
        he = HessianError(ctx, s.E, s.d_model, s.d_ff)
        che_cal, che_test = {}, {}
        for name, mode in (("plic", "explicit"), ("clha_rt", "rt"), ("clha_eq", "eq")):
            r = cal.res[mode]
            che_cal[name] = float(he(cal, w, r, "explicit", hook)["routed"].sum())
            che_test[name] = float(he(held, w, r, "rt")["routed"].sum())
        row = {"workload": "routing-sharpness sweep", "sharpness": beta,
               "divergence_tv": mean_pairwise(routing_divergence(ctx, cal.acc_in, 0, s.E)),
               "divergence_tv_test": mean_pairwise(routing_divergence(ctx, held.acc_in, 0, s.E)),
               "min_expert_tokens_per_layer": [int(c) for c in counts.min(1)],
               "che_cal": che_cal, "che_test": che_test,
               "test_gain_rt_vs_plic": 1.0 - che_test["clha_rt"] / che_test["plic"],
               "test_gain_eq_vs_plic": 1.0 - che_test["clha_eq"] / che_test["plic"],
               "config": {"workload": s.name, "tokens_per_layer": s.tokens[0], "held_out_tokens_per_layer":
                          test_wl.spec.tokens[0], "bits": s.bits_routed, "data": "synthetic"}}
        rows.append(row)
        print(json.dumps(row), flush=True)
        del cal, held, he, w
        torch.cuda.empty_cache()
    if rows:
        base = rows[0]["che_test"]
        print(json.dumps({"workload": "routing-sharpness sweep summary",
                          "sharpness": [r["sharpness"] for r in rows],
                          "divergence_tv": [r["divergence_tv"] for r in rows],
                          "test_error_vs_first": {k: [r["che_test"][k] / base[k] for r in rows] for k in base},
                          "test_gain_rt_vs_plic": [r["test_gain_rt_vs_plic"] for r in rows]}), flush=True)
    ctx.close()
    return 0


def run_kernel(args):
    """Kernel-level timing: CUDA events around `steps` launches after `warmup`, inputs resident."""
    import torch
    from post_quantization_expert_b200 import clha as L
    ctx = L.Context(0)
    peaks, src = load_peaks()
    alu = alu_peaks(peaks)
    g = torch.Generator(device="cuda")
    g.manual_seed(0)
    flush = torch.empty(512 << 20, dtype=torch.uint8, device="cuda")
    for shape in args.shape:
        dims = [int(v) for v in shape.split("x")]
        if args.workload == "act":
            n, dm, dff = dims
            X = torch.randn((n, dm), device="cuda", generator=g).to(torch.bfloat16)
            Wg = (0.03 * torch.randn((dff, dm), device="cuda", generator=g)).to(torch.bfloat16)
            Wu = (0.03 * torch.randn((dff, dm), device="cuda", generator=g)).to(torch.bfloat16)
            hbuf = torch.empty((n, dff), device="cuda", dtype=torch.bfloat16)
            fn = lambda: L.clha_expert_act(ctx, X, n, dm, None, 1, Wg, Wu, dff, hbuf)
            work, unit, bound, peak = 4 * n * dm * dff / 1e12, "TFLOP/s", "alu", alu["fp32_tflops"]
            kname = "expert_act_simt (fp32 FMA)"
        elif args.workload == "dequant":
            n, d_out, d_in = dims
            bits = 3
            X = torch.randn((n, d_in), device="cuda", generator=g).to(torch.bfloat16)
            codes = torch.randint(0, 2 ** bits, (d_out, d_in), device="cuda", generator=g, dtype=torch.uint8)
            packed = torch.empty((d_out, d_in * bits // 32), dtype=torch.int32, device="cuda")
            L.clha_pack_codes(ctx, codes, d_out, d_in, bits, packed)
            sc = 0.01 * torch.rand((d_out, d_in // 128), device="cuda", generator=g)
            zs = torch.full((d_out, d_in // 128), 3, dtype=torch.uint8, device="cuda")
            Y = torch.empty((n, d_out), device="cuda")
            fn = lambda: L.clha_dequant_matmul(ctx, X, n, packed, sc, zs, d_out, d_in, bits, Y)
            work, unit, bound, peak = 2 * n * d_out * d_in / 1e12, "TFLOP/s", "alu", alu["fp32_tflops"]
            kname = "dequant_matmul_kernel (3-bit packed codes, fp32 FMA)"
        elif args.workload == "epmq":
            Ksrc, d_out, d = dims
            Xs = torch.randn((Ksrc, 2 * d, d), device="cuda", generator=g).to(torch.bfloat16)
            acc = L.Accum(ctx, d, Ksrc, 1)
            for i in range(Ksrc):
                L.clha_collect(ctx, acc, i, Xs[i], 2 * d, d)
            del Xs
            Hc = torch.empty((1, d, d), device="cuda")
            Hd = torch.empty_like(Hc)
            U = torch.empty_like(Hc)
            lam = torch.empty(1, dtype=torch.float64, device="cuda")
            L.clha_aggregate(ctx, acc, 0, 1, L.ALPHA_SUM, None, 0.01, Hc, Hd, lambda_dev=lam)
            L.clha_factor(ctx, Hd, 1, d, U)
            W_src = (0.02 * torch.randn((Ksrc, d_out, d), device="cuda", generator=g)).to(torch.bfloat16)
            W_m = W_src.float().mean(0).to(torch.bfloat16)
            Wt = torch.empty((d_out, d), device="cuda")
            fn = lambda: L.clha_epmq_target(ctx, acc, 0, W_src, W_m, d_out, U, lam, Wt)
            work = (2 * Ksrc * d_out * d * d + 2 * d ** 3 + 2 * d_out * d * d) / 1e12
            unit, bound, peak = "TFLOP/s", "alu", alu["fp64_tflops"]
            kname = "epmq_gemm x3 (fp64, mma.sync m8n8k4 f64)"
        elif args.workload == "hessian":
            n, d = dims
            X = torch.randn((n, d), device="cuda", generator=g).to(torch.bfloat16)
            acc = L.Accum(ctx, d, 1, 1)
            fn = lambda: L.clha_collect(ctx, acc, 0, X, n, d)
            work, unit, bound, peak = n * d * (d + 1) / 1e12, "TFLOP/s", "tensor", peaks["bf16_tflops"]
            kname = gram_kernel(d)
        else:
            if args.workload == "gptq":
                B, d_out, d = dims
            else:
                B, d = dims
            A = torch.randn((B, d, d // 2), device="cuda", generator=g)
            H = (A @ A.transpose(1, 2) / (d // 2) + 0.05 * torch.eye(d, device="cuda")).contiguous()
            del A
            U = torch.empty_like(H)
            form = FORMS[args.factor_form]
            if args.workload == "factor":
                fn = lambda: L.clha_factor_as(ctx, form, H, B, d, U)
                work, unit, bound, peak = B * factor_work(d, form) / 1e12, "TFLOP/s", "alu", alu["fp64_tflops"]
                kname = factor_kernels(form)
            else:
                L.clha_factor_as(ctx, form, H, B, d, U)
                W = (0.02 * torch.randn((B, d_out, d), device="cuda", generator=g)).to(torch.bfloat16)
                codes = torch.empty((B, d_out, d), dtype=torch.uint8, device="cuda")
                sc = torch.empty((B, d_out, d // 128), device="cuda")
                zs = torch.empty((B, d_out, d // 128), dtype=torch.uint8, device="cuda")
                Wh = torch.empty((B, d_out, d), device="cuda")
                fn = lambda: L.clha_quantize(ctx, U, B, W, B, d_out, d, 3, codes, sc, zs, Wh, form=form)
                work, unit, bound, peak = B * d_out * d * d / 1e12, "TFLOP/s", "tensor", alu["tf32x3_tflops"]
                kname = "gptq_tc + gptq_trail (3xTF32; peak: tf32 / 3)"
        for _ in range(args.warmup):
            fn()
        torch.cuda.synchronize()
        clocks = ClockSampler(0)
        clocks.start()
        evs = []
        t_begin = time.time()
        for _ in range(args.steps):   # L2 flushed before every timed launch, each launch timed alone
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record(ctx.stream)
            fn()
            b.record(ctx.stream)
            evs.append((a, b))
        torch.cuda.synchronize()
        clocks.mark(t_begin, time.time())
        clk = clocks.stop()
        L.clha_check(ctx)
        if args.workload == "act" and L.clha_last_act_kernel(ctx) == L.ACT_TENSOR:   # the kernel that ran
            bound, peak, kname = "tensor", peaks["bf16_tflops"], "expert_act_tc (tcgen05 kind::f16)"
        ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
        achieved = work / (ms / 1e3)
        print(json.dumps({"workload": args.workload, "shape": shape, "kernel": kname, "ms": ms, "achieved": achieved,
                          "unit": unit, "bound": bound, "peak": peak, "frac": achieved / peak,
                          "peak_source": (src if bound == "tensor" and args.workload != "gptq" else
                                          "derived (measured bf16 x nominal tf32/bf16, / 3)" if bound == "tensor" else
                                          "derived (SM count x lanes x max clock)"),
                          "l2": "flushed (512 MB write) before every timed launch", "clocks": clk}))
        torch.cuda.empty_cache()
    ctx.close()
    return 0


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--parallel", choices=("replicas", "tokens"), default="replicas",
                    help="replicas (default): each rank calibrates its own layer pair (weak scaling); tokens: "
                         "one pair, its tokens sharded over the ranks with one reduce-scatter of the packed Hessian sums to their owners, "
                         "its experts quantized in parallel (strong scaling)")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the timed oracle sample")
    ap.add_argument("--workload", choices=("dense", "moe-e16", "moe-e64", "act", "hessian", "gptq", "factor", "epmq", "dequant",
                                           "sweep"),
                    default="dense",
                    help="dense: the end-to-end calibration step of the 8192x28672 weight shared by 4 layers "
                         "(default); moe-e16: the E16 MoE layer pair; sweep: the routing-sharpness "
                         "experiment; others: one kernel family")
    ap.add_argument("--sharpness", type=float, nargs="+", default=[0.0, 0.1, 0.2, 0.3, 0.5, 0.75, 1.0],
                    help="sweep: strengths of the per-layer expert preference")
    ap.add_argument("--shape", nargs="+", default=[], help="kernel workload shapes, e.g. 65536x4096")
    ap.add_argument("--factor-form", choices=tuple(FORMS), default="block",
                    help="GPTQ's factor: U (inv) or the block-scaled Cholesky factor of H (block, the default)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.workload == "sweep":
        return run_sweep(args)
    if args.workload not in ("dense", "moe-e16", "moe-e64"):
        if not args.shape:
            ap.error("--shape is required for kernel workloads")
        return run_kernel(args)
    if args.parallel == "tokens" and args.workload != "moe-e16":
        ap.error("--parallel tokens applies to --workload moe-e16")
    world, rank, local = dist_setup()
    try:
        if args.workload == "dense":
            if args.impl == "reference":
                return run_reference_dense(args, world, rank)
            return run_dense(args, world, rank, local)
        if args.impl == "reference":
            return run_reference(args, world, rank)
        return run_ours(args, world, rank, local)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    sys.exit(main())
