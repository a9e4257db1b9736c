"""The five calibration workloads, drawn from seeded torch generators.

Every draw comes from a torch.Generator seeded from (workload seed, tag), so a given
(workload, device, overrides) always yields the same bytes. Values drawn on "cpu" and on "cuda"
differ (different generator families); a test or a bench run reads both the oracle's and the
CUDA path's inputs from the one device it asked for.

Input model (CLHA technical summary, section 2.1: each layer sees its own activation distribution):
  x = D^{1/2} z1 + U z2,  z1 ~ N(0, I_d), z2 ~ N(0, I_r)   so   Cov(x) = D + U U^T
  D = diag(U(0.5, 2)),  U_ij ~ N(0, 0.3^2)
  drift delta between layers sharing a weight: U_next = cos(pi*delta/2) U + sin(pi*delta/2) V,
  V an independent draw of U's distribution (delta = 0: same subspace, delta = 1: independent).
Router logits are N(0, 1) per token and expert, plus log p_e for Zipf-skewed routing
(p_e proportional to rank_e^-s over a seeded permutation of the experts), plus, for the routing
sharpness sweep, beta * (-1)^j * v_e: a per-group expert preference v ~ N(0, I_E) that layer j of
the group follows with alternating sign, so that raising beta concentrates each layer on its own
experts and drives the layers' expert frequencies apart (a top-k choice is unchanged by a plain
temperature on the logits, so sharpening acts on this preference).
A split other than "cal" draws fresh tokens (X and logits) from the same per-layer laws and the
same weights: the held-out data of the test-side reconstruction error.
Outlier channels (a seeded 1% of channels) are multiplied by 20 before rounding to bf16.
Weights are N(0, 0.02^2).
"""
from __future__ import annotations

import math
import zlib
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Spec:
    """Shape and policy of one workload (sizes in elements)."""
    name: str
    seed: int
    kind: str                      # "dense": one weight W; "moe": routed experts (+ always-active ones)
    dtype: torch.dtype             # storage dtype of X and W
    n_layers: int                  # layers in the whole stack
    group_of_layers: tuple         # tuple of tuples: layer indices that share one set of weights
    tokens: tuple                  # tokens per layer (len n_layers)
    d_model: int                   # d_in of the dense W, or the MoE model width
    d_out: int = 0                 # rows of the dense W
    d_ff: int = 0                  # routed expert hidden width
    E: int = 0                     # routed experts per layer
    k: int = 0                     # top-k
    n_shared: int = 0              # always-active experts per layer
    shared_dff: int = 0
    rank: int = 8
    drifts: tuple = (0.3,)         # drift applied to each group's later layers (per group)
    outlier_frac: float = 0.0
    zipf_s: float = 0.0            # 0: plain N(0,1) logits
    bits_routed: int = 4
    bits_shared: int = 4
    group: int = 128
    block: int = 128
    damp_frac: float = 0.01
    alpha_modes: tuple = ("rt",)
    chunk_tokens: int = 8192       # draw X in chunks of this many tokens (bounds temporaries)
    split: str = "cal"             # "cal": calibration tokens; any other name: fresh tokens of the same law
    sharpness: float = 0.0         # strength of the per-layer expert preference added to the logits


def _spec_c1():
    return Spec(name="dense-256x512-fp32-2layers", seed=1234, kind="dense", dtype=torch.float32,
                n_layers=2, group_of_layers=((0, 1),), tokens=(1000, 1024), d_model=512, d_out=256,
                rank=8, drifts=(0.3,), bits_routed=2, bits_shared=2, alpha_modes=("rt",))


def _spec_c2():
    return Spec(name="moe-E16-top2-d1024-ff512-8k", seed=1235, kind="moe", dtype=torch.bfloat16,
                n_layers=2, group_of_layers=((0, 1),), tokens=(8192, 8192), d_model=1024, d_ff=512,
                E=16, k=2, rank=32, drifts=(0.3,), bits_routed=3, bits_shared=3,
                alpha_modes=("rt", "eq"))


def _spec_c3():
    return Spec(name="moe-E64-top6-d2048-ff1408-2shared-32k", seed=1236, kind="moe",
                dtype=torch.bfloat16, n_layers=2, group_of_layers=((0, 1),), tokens=(32768, 32768),
                d_model=2048, d_ff=1408, E=64, k=6, n_shared=2, shared_dff=1408, rank=32,
                drifts=(0.3,), outlier_frac=0.01, zipf_s=1.1, bits_routed=2, bits_shared=3,
                alpha_modes=("rt",))


def _spec_c4():
    pairs = tuple((2 * p, 2 * p + 1) for p in range(12))
    sweep = (0.0, 0.3, 0.6, 1.0)
    return Spec(name="moe-stack12pairs-E16-top2-d1024-ff512-2shared-128k", seed=1237, kind="moe",
                dtype=torch.bfloat16, n_layers=24, group_of_layers=pairs, tokens=(131072,) * 24,
                d_model=1024, d_ff=512, E=16, k=2, n_shared=2, shared_dff=512, rank=32,
                drifts=tuple(sweep[p % 4] for p in range(12)), bits_routed=2, bits_shared=3,
                alpha_modes=("rt", "eq"))


def _spec_c5():
    return Spec(name="dense-8192x28672-bf16-4layers-64k", seed=1238, kind="dense",
                dtype=torch.bfloat16, n_layers=4, group_of_layers=((0, 1, 2, 3),),
                tokens=(65536,) * 4, d_model=28672, d_out=8192, rank=64, drifts=(0.3,),
                bits_routed=4, bits_shared=4, alpha_modes=("rt",))


WORKLOADS = {1: _spec_c1, 2: _spec_c2, 3: _spec_c3, 4: _spec_c4, 5: _spec_c5}


def _tag_seed(seed: int, *tag) -> int:
    return (seed * 1_000_003 + zlib.crc32(repr(tag).encode())) % (2 ** 62)


class Workload:
    """Lazily drawn inputs of one workload on one torch device.

    Layers that share weights form a group (a layer pair for CLWS-MoE, four layers for the dense
    stress case); within a group the low-rank covariance factor drifts from layer to layer.
    """

    def __init__(self, spec: Spec, device="cpu"):
        self.spec = spec
        self.device = torch.device(device)
        self._cov = {}
        self._x = {}
        self._split = () if spec.split == "cal" else (spec.split,)   # calibration draws keep their tags

    # ------------------------------------------------------------------ generators
    def _gen(self, *tag) -> torch.Generator:
        g = torch.Generator(device=self.device)
        g.manual_seed(_tag_seed(self.spec.seed, *tag))
        return g

    def _randn(self, shape, *tag, std=1.0, dtype=torch.float32):
        t = torch.randn(shape, generator=self._gen(*tag), device=self.device, dtype=torch.float32)
        if std != 1.0:
            t.mul_(std)
        return t.to(dtype)

    def group_index(self, layer: int) -> int:
        for gi, g in enumerate(self.spec.group_of_layers):
            if layer in g:
                return gi
        raise IndexError(layer)

    # ------------------------------------------------------------------ covariance model
    def _cov_model(self, gi: int, d: int):
        """(sqrt(D), [U per layer of the group], outlier channel mask) for group gi."""
        key = (gi, d)
        if key in self._cov:
            return self._cov[key]
        s = self.spec
        g = self._gen("D", gi, d)
        Dg = torch.rand(d, generator=g, device=self.device) * 1.5 + 0.5
        layers = s.group_of_layers[gi]
        delta = s.drifts[gi] if len(s.drifts) > gi else s.drifts[0]
        c, sn = math.cos(math.pi * delta / 2), math.sin(math.pi * delta / 2)
        Us = [self._randn((d, s.rank), "U", gi, d, 0, std=0.3)]
        for j in range(1, len(layers)):
            V = self._randn((d, s.rank), "U", gi, d, j, std=0.3)
            Us.append(c * Us[-1] + sn * V)
        scale = torch.ones(d, device=self.device)
        if s.outlier_frac > 0:
            n_out = int(round(s.outlier_frac * d))
            perm = torch.randperm(d, generator=self._gen("outliers", gi, d), device=self.device)
            scale[perm[:n_out]] = 20.0
        self._cov[key] = (Dg.sqrt(), Us, scale)
        return self._cov[key]

    def x(self, layer: int, cache: bool = True) -> torch.Tensor:
        """Activations entering the weight(s) of `layer`: [tokens, d_model] in the storage dtype."""
        if layer in self._x:
            return self._x[layer]
        s = self.spec
        gi = self.group_index(layer)
        j = s.group_of_layers[gi].index(layer)
        sqD, Us, scale = self._cov_model(gi, s.d_model)
        U = Us[j]
        n = s.tokens[layer]
        out = torch.empty((n, s.d_model), dtype=s.dtype, device=self.device)
        for c0 in range(0, n, s.chunk_tokens):
            c1 = min(n, c0 + s.chunk_tokens)
            z1 = self._randn((c1 - c0, s.d_model), "z1", layer, c0, *self._split)
            z2 = self._randn((c1 - c0, s.rank), "z2", layer, c0, *self._split)
            xc = z1.mul_(sqD).addmm_(z2, U.t())
            if s.outlier_frac > 0:
                xc.mul_(scale)
            out[c0:c1] = xc.to(s.dtype)
            del z1, z2, xc
        if cache:
            self._x[layer] = out
        return out

    def drop(self, layer: int):
        self._x.pop(layer, None)

    def logits(self, layer: int) -> torch.Tensor:
        """Router logits [tokens, E] float32 for a MoE layer."""
        s = self.spec
        assert s.kind == "moe"
        lg = self._randn((s.tokens[layer], s.E), "logits", layer, *self._split)
        if s.zipf_s > 0:
            gi = self.group_index(layer)
            perm = torch.randperm(s.E, generator=self._gen("zipf", gi), device=self.device)
            ranks = torch.empty(s.E, device=self.device)
            ranks[perm] = torch.arange(1, s.E + 1, device=self.device, dtype=torch.float32)
            logp = -s.zipf_s * torch.log(ranks)
            logp = logp - torch.logsumexp(logp, 0)
            lg = lg + logp[None, :]
        if s.sharpness != 0.0:
            gi = self.group_index(layer)
            j = s.group_of_layers[gi].index(layer)
            v = self._randn((s.E,), "pref", gi)
            lg = lg + (s.sharpness * (-1.0) ** j) * v[None, :]
        return lg.contiguous()

    # ------------------------------------------------------------------ weights
    def dense_weight(self) -> torch.Tensor:
        s = self.spec
        assert s.kind == "dense"
        return self._randn((s.d_out, s.d_model), "W", std=0.02, dtype=s.dtype)

    def expert_weights(self, gi: int, e: int, shared: bool = False):
        """(W_gate [d_ff, d_model], W_up [d_ff, d_model], W_down [d_model, d_ff]) of one expert.

        Routed experts are indexed 0..E-1, always-active ones 0..n_shared-1 with shared=True.
        """
        s = self.spec
        dff = s.shared_dff if shared else s.d_ff
        tag = ("shared" if shared else "routed", gi, e)
        wg = self._randn((dff, s.d_model), "Wg", *tag, std=0.02, dtype=s.dtype)
        wu = self._randn((dff, s.d_model), "Wu", *tag, std=0.02, dtype=s.dtype)
        wd = self._randn((s.d_model, dff), "Wd", *tag, std=0.02, dtype=s.dtype)
        return wg, wu, wd


def workload(cfg: int, device="cpu", **overrides) -> Workload:
    """Workload `cfg` (1..5) on `device`; keyword overrides replace Spec fields (e.g. tokens=(512,512))."""
    spec = WORKLOADS[cfg]()
    if overrides:
        if "tokens" in overrides and isinstance(overrides["tokens"], int):
            overrides["tokens"] = (overrides["tokens"],) * spec.n_layers
        spec = replace(spec, **overrides)
    return Workload(spec, device)
