"""ctypes binding of libclha.so: the C entry points under the same names, plus argument marshalling.

Every array argument is a torch tensor on the context's CUDA device (or None where the C call allows
NULL); host outputs (alpha, lambda, loss, checkpoints) are numpy arrays. Nothing here computes any
part of the method: each call forwards to the CUDA library and raises ClhaError on a non-zero status.
The library must have been built (python -m post_quantization_expert_b200.build); there is no
fallback.
"""
from __future__ import annotations

import ctypes as C
import os
import sys

import numpy as np
import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libclha.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED_SHAPE, ERR_NOT_PD, ERR_NONFINITE, ERR_EMPTY, ERR_OOM, ERR_CUDA, ERR_TIMEOUT = range(9)
STATUS_NAMES = ["OK", "INVALID_ARG", "UNSUPPORTED_SHAPE", "NOT_PD", "NONFINITE", "EMPTY", "OOM", "CUDA", "TIMEOUT"]
BF16, F32 = 0, 1
ALPHA_ROUTING, ALPHA_EQUAL, ALPHA_EXPLICIT, ALPHA_SUM = 0, 1, 2, 3
AGG_EMPTY_IDENTITY = 0x100   # or'ed into an alpha mode: an aggregate without energy becomes H_d = I
ACT_AUTO, ACT_FMA, ACT_TENSOR = 0, 1, 2   # activation kernel policy (clha_set_act_kernel)

# every symbol include/clha.h declares
SYMBOLS = [
    "clha_create", "clha_destroy", "clha_last_error", "clha_check", "clha_version", "clha_kernel_launches",
    "clha_route_topk", "clha_packed_rows", "clha_gather", "clha_gather_noalloc", "clha_expert_act",
    "clha_accum_create", "clha_accum_destroy", "clha_accum_zero", "clha_accum_buffers",
    "clha_accum_export", "clha_accum_import", "clha_collect",
    "clha_aggregate", "clha_factor", "clha_factor_groups", "clha_epmq_target", "clha_quantize", "clha_loss",
    "clha_pack_codes", "clha_dequantize", "clha_dequant_matmul", "clha_routing_divergence",
    "clha_collect_gathered", "clha_expert_act_gathered", "clha_set_act_kernel", "clha_last_act_kernel",
    "clha_set_factor_wait_limit", "clha_pack_upper", "clha_unpack_upper", "clha_factor_groups_as",
    "clha_quantize_as",
]
FACTOR_MAX_GROUPS = 4
# clha_factor_form: U with H_d^-1 = U^T U, or F, the block-scaled Cholesky factor of H_d (GPTQ only)
FACTOR_INV_CHOL, FACTOR_BLOCK_CHOL = 0, 1


class FactorGroup(C.Structure):
    _fields_ = [("H_damped", C.c_void_p), ("U", C.c_void_p), ("batch", C.c_int), ("d", C.c_int)]


class QuantParams(C.Structure):
    _fields_ = [("bits", C.c_int), ("group", C.c_int), ("block", C.c_int), ("damp_frac", C.c_float)]


class ClhaError(RuntimeError):
    def __init__(self, status: int, message: str):
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"CLHA_ERR_{name}: {message}")
        self.status = status
        self.message = message


_lib = None
vp, i32, i64, f32, f64 = C.c_void_p, C.c_int, C.c_int64, C.c_float, C.c_double


def load(path: str = LIB_PATH):
    """Load libclha.so (once). Raises if it is missing: the path has no fallback."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing; build it with `python -m post_quantization_expert_b200.build`")
    lib = C.CDLL(path)
    sig = {
        "clha_create": (i32, [i32, vp, C.POINTER(vp)]),
        "clha_destroy": (None, [vp]),
        "clha_last_error": (C.c_char_p, [vp]),
        "clha_check": (i32, [vp]),
        "clha_version": (i32, []),
        "clha_kernel_launches": (i64, [vp]),
        "clha_route_topk": (i32, [vp, vp, i64, i32, i32, vp, vp]),
        "clha_packed_rows": (i64, [i64, i32, i32]),
        "clha_gather": (i32, [vp, vp, i32, i64, i32, vp, i32, i32, vp, i64, vp, vp]),
        "clha_gather_noalloc": (i32, [vp, vp, i32, i64, i32, vp, i32, i32, vp, i64, vp, vp]),
        "clha_expert_act": (i32, [vp, vp, i64, i32, vp, i32, vp, vp, i32, vp]),
        "clha_accum_create": (i32, [vp, i32, i32, i32, C.POINTER(vp)]),
        "clha_accum_destroy": (i32, [vp]),
        "clha_accum_zero": (i32, [vp, vp]),
        "clha_accum_buffers": (i32, [vp, C.POINTER(vp), C.POINTER(vp)]),
        "clha_accum_export": (i32, [vp, vp, vp, vp]),
        "clha_accum_import": (i32, [vp, vp, vp, vp]),
        "clha_collect": (i32, [vp, vp, i32, vp, i32, i64, i32, vp, i32, i32]),
        "clha_aggregate": (i32, [vp, vp, i32, i32, i32, vp, f64, vp, vp, vp, vp, vp]),
        "clha_factor": (i32, [vp, vp, i32, i32, vp]),
        "clha_factor_groups": (i32, [vp, i32, vp]),
        "clha_factor_groups_as": (i32, [vp, i32, i32, vp]),
        "clha_epmq_target": (i32, [vp, vp, i32, vp, vp, i32, i32, vp, vp, vp]),
        "clha_pack_codes": (i32, [vp, vp, i64, i32, i32, vp]),
        "clha_dequantize": (i32, [vp, vp, vp, vp, i64, i32, i32, vp]),
        "clha_dequant_matmul": (i32, [vp, vp, i32, i64, vp, vp, vp, i32, i32, i32, vp]),
        "clha_quantize": (i32, [vp, vp, i32, vp, i32, i32, i32, i32, C.POINTER(QuantParams), vp, vp, vp, vp, vp,
                                vp]),
        "clha_quantize_as": (i32, [vp, i32, vp, i32, vp, i32, i32, i32, i32, C.POINTER(QuantParams), vp, vp, vp, vp,
                                   vp, vp]),
        "clha_loss": (i32, [vp, vp, i32, vp, vp, i32, i32, i32, i32, vp]),
        "clha_routing_divergence": (i32, [vp, vp, i32, i32, i32, i32, vp]),
        "clha_collect_gathered": (i32, [vp, vp, i32, vp, i64, i32, vp, vp, i32, i32]),
        "clha_expert_act_gathered": (i32, [vp, vp, i64, i32, vp, i64, vp, i32, vp, vp, i32, vp]),
        "clha_set_act_kernel": (i32, [vp, i32]),
        "clha_last_act_kernel": (i32, [vp]),
        "clha_set_factor_wait_limit": (i32, [vp, C.c_uint64]),
        "clha_pack_upper": (i32, [vp, vp, i64, i64, i64, i32, vp]),
        "clha_unpack_upper": (i32, [vp, vp, i64, i64, i64, i32, vp]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def _p(t):
    """Device (or host) pointer of a tensor / ndarray, or NULL for None."""
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        if not t.is_contiguous():
            raise ValueError("libclha takes dense row-major arrays; got a non-contiguous tensor")
        return t.data_ptr()
    if isinstance(t, np.ndarray):
        if not t.flags["C_CONTIGUOUS"]:
            raise ValueError("libclha takes dense row-major arrays; got a non-C-contiguous ndarray")
        return t.ctypes.data
    raise TypeError(type(t))


def _dtype(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t.dtype}")


class Context:
    """A clha_ctx bound to a CUDA device and stream (torch's current stream by default)."""

    def __init__(self, device: int = 0, stream: torch.cuda.Stream | None = None):
        lib = load()
        self.device = device
        self.stream = stream if stream is not None else torch.cuda.current_stream(device)
        h = vp()
        st = lib.clha_create(device, self.stream.cuda_stream, C.byref(h))
        if st != OK:
            raise ClhaError(st, "clha_create failed")
        self.handle = h

    def _check(self, st: int):
        if st != OK:
            raise ClhaError(st, load().clha_last_error(self.handle).decode())

    def close(self):
        if getattr(self, "handle", None):
            load().clha_destroy(self.handle)
            self.handle = None

    def __del__(self):
        if sys is not None and not sys.is_finalizing():
            self.close()


def clha_version() -> int:
    return load().clha_version()


def clha_kernel_launches(ctx: Context) -> int:
    return load().clha_kernel_launches(ctx.handle)


def clha_check(ctx: Context):
    ctx._check(load().clha_check(ctx.handle))


def clha_route_topk(ctx: Context, logits, n: int, E: int, k: int, ids, counts):
    ctx._check(load().clha_route_topk(ctx.handle, _p(logits), n, E, k, _p(ids), _p(counts)))


def clha_packed_rows(n: int, k: int, E: int) -> int:
    return load().clha_packed_rows(n, k, E)


def clha_gather(ctx: Context, X, n: int, d: int, ids, k: int, E: int, X_packed, packed_rows: int, seg, perm=None):
    ctx._check(load().clha_gather(ctx.handle, _p(X), _dtype(X), n, d, _p(ids), k, E, _p(X_packed), packed_rows,
                                  _p(seg), _p(perm)))


def clha_gather_noalloc(ctx: Context, X, n: int, d: int, ids, k: int, E: int, X_packed, packed_rows: int, seg,
                        perm=None):
    """clha_gather with its scratch in the library's fixed device array (no allocation)."""
    ctx._check(load().clha_gather_noalloc(ctx.handle, _p(X), _dtype(X), n, d, _p(ids), k, E, _p(X_packed),
                                          packed_rows, _p(seg), _p(perm)))


def clha_expert_act(ctx: Context, X, rows: int, d_model: int, seg, E: int, Wg, Wu, d_ff: int, h):
    ctx._check(load().clha_expert_act(ctx.handle, _p(X), rows, d_model, _p(seg), E, _p(Wg), _p(Wu), d_ff, _p(h)))


def clha_set_act_kernel(ctx: Context, kernel: int):
    ctx._check(load().clha_set_act_kernel(ctx.handle, kernel))


def clha_last_act_kernel(ctx: Context) -> int:
    return load().clha_last_act_kernel(ctx.handle)


def clha_expert_act_gathered(ctx: Context, X, n: int, d_model: int, perm, packed_rows: int, seg, E: int, Wg, Wu,
                             d_ff: int, h):
    """The expert activation with the segment rows read from X [n, d_model] through perm."""
    ctx._check(load().clha_expert_act_gathered(ctx.handle, _p(X), n, d_model, _p(perm), packed_rows, _p(seg), E,
                                               _p(Wg), _p(Wu), d_ff, _p(h)))


class Accum:
    """clha_accum: per-(layer, slot) Gram matrices and token counts."""

    def __init__(self, ctx: Context, d: int, n_layers: int, n_slots: int):
        self.ctx, self.d, self.n_layers, self.n_slots = ctx, d, n_layers, n_slots
        h = vp()
        ctx._check(load().clha_accum_create(ctx.handle, d, n_layers, n_slots, C.byref(h)))
        self.handle = h

    def buffers(self):
        """(S, counts) as torch views of the device buffers: [L, slots, d, d] f32 and [L, slots] i64."""
        s, c = vp(), vp()
        self.ctx._check(load().clha_accum_buffers(self.handle, C.byref(s), C.byref(c)))
        return (_wrap(s.value, (self.n_layers, self.n_slots, self.d, self.d), torch.float32, self.ctx.device),
                _wrap(c.value, (self.n_layers, self.n_slots), torch.int64, self.ctx.device))

    def close(self):
        if getattr(self, "handle", None):
            load().clha_accum_destroy(self.handle)
            self.handle = None

    def __del__(self):
        if sys is not None and not sys.is_finalizing():
            self.close()


def _wrap(ptr: int, shape, dtype, device):
    """A torch view of library-owned device memory (valid while the owner lives)."""
    n = int(np.prod(shape))
    esz = torch.empty((), dtype=dtype).element_size()

    class _Holder:
        __cuda_array_interface__ = {
            "shape": (n,), "typestr": {torch.float32: "<f4", torch.int64: "<i8"}[dtype],
            "data": (ptr, False), "version": 3, "strides": (esz,),
        }
    return torch.as_tensor(_Holder(), device=f"cuda:{device}").view(shape)


def clha_accum_create(ctx: Context, d: int, n_layers: int, n_slots: int) -> Accum:
    return Accum(ctx, d, n_layers, n_slots)


def clha_accum_destroy(acc: Accum):
    acc.close()


def clha_accum_zero(ctx: Context, acc: Accum):
    ctx._check(load().clha_accum_zero(ctx.handle, acc.handle))


def clha_accum_export(ctx: Context, acc: Accum):
    S = np.empty((acc.n_layers, acc.n_slots, acc.d, acc.d), np.float32)
    cnt = np.empty((acc.n_layers, acc.n_slots), np.int64)
    ctx._check(load().clha_accum_export(ctx.handle, acc.handle, _p(S), _p(cnt)))
    return S, cnt


def clha_accum_import(ctx: Context, acc: Accum, S: np.ndarray, counts: np.ndarray):
    S = np.ascontiguousarray(S, np.float32)
    counts = np.ascontiguousarray(counts, np.int64)
    ctx._check(load().clha_accum_import(ctx.handle, acc.handle, _p(S), _p(counts)))


def clha_collect(ctx: Context, acc: Accum, layer: int, X, rows: int, d: int, seg=None, E: int = 1, slot0: int = 0):
    ctx._check(load().clha_collect(ctx.handle, acc.handle, layer, _p(X), _dtype(X), rows, d, _p(seg), E, slot0))


def clha_collect_gathered(ctx: Context, acc: Accum, layer: int, X, n: int, d: int, perm, seg, E: int, slot0: int = 0):
    """Gram accumulation straight from X [n, d] bf16 through clha_gather's perm (TMA gather4)."""
    ctx._check(load().clha_collect_gathered(ctx.handle, acc.handle, layer, _p(X), n, d, _p(perm), _p(seg), E, slot0))


def clha_aggregate(ctx: Context, acc: Accum, slot0: int, n_slots: int, mode: int, alpha_in=None,
                   damp_frac: float = 0.01, H_comb=None, H_damped=None, want_host: bool = False, lambda_dev=None):
    """Returns (alpha [n_slots, L], lambda [n_slots]) as numpy when want_host, else None. lambda_dev
    (float64 device tensor [n_slots]) receives lambda without a synchronisation."""
    a_in = None if alpha_in is None else np.ascontiguousarray(alpha_in, np.float64)
    a_out = np.empty((n_slots, acc.n_layers), np.float64) if want_host else None
    l_out = np.empty(n_slots, np.float64) if want_host else None
    ctx._check(load().clha_aggregate(ctx.handle, acc.handle, slot0, n_slots, mode, _p(a_in), damp_frac, _p(H_comb),
                                     _p(H_damped), _p(a_out), _p(l_out), _p(lambda_dev)))
    return (a_out, l_out) if want_host else None


def clha_factor(ctx: Context, H_damped, batch: int, d: int, U):
    ctx._check(load().clha_factor(ctx.handle, _p(H_damped), batch, d, _p(U)))


def clha_set_factor_wait_limit(ctx: Context, ns: int):
    """Limit of each dependency wait in the factor graph, in ns (0: the default, 4 s)."""
    ctx._check(load().clha_set_factor_wait_limit(ctx.handle, ns))


def clha_factor_groups(ctx: Context, groups, form: int = FACTOR_INV_CHOL):
    """groups: sequence of (H_damped, batch, d, U), at most FACTOR_MAX_GROUPS; one graph launch.
    form FACTOR_BLOCK_CHOL writes F (for clha_quantize with the same form) in place of U."""
    arr = (FactorGroup * len(groups))(*[FactorGroup(_p(H), _p(U), b, d) for H, b, d, U in groups])
    if form == FACTOR_INV_CHOL:
        ctx._check(load().clha_factor_groups(ctx.handle, len(groups), C.cast(arr, C.c_void_p)))
    else:
        ctx._check(load().clha_factor_groups_as(ctx.handle, form, len(groups), C.cast(arr, C.c_void_p)))


def clha_factor_as(ctx: Context, form: int, H_damped, batch: int, d: int, F):
    """One group of clha_factor_groups in the given form."""
    clha_factor_groups(ctx, [(H_damped, batch, d, F)], form)


def clha_epmq_target(ctx: Context, acc: "Accum", slot: int, W_src, W_merged, d_out: int, U, lambda_dev, W_target):
    """W_target = (lambda W_m + sum_i W_i S_i) U^T U for the accumulator's K source experts."""
    ctx._check(load().clha_epmq_target(ctx.handle, acc.handle, slot, _p(W_src), _p(W_merged), _dtype(W_src), d_out,
                                       _p(U), _p(lambda_dev), _p(W_target)))


def clha_pack_codes(ctx: Context, codes, rows: int, d_in: int, bits: int, packed):
    ctx._check(load().clha_pack_codes(ctx.handle, _p(codes), rows, d_in, bits, _p(packed)))


def clha_dequantize(ctx: Context, packed, scales, zeros, rows: int, d_in: int, bits: int, W_hat):
    ctx._check(load().clha_dequantize(ctx.handle, _p(packed), _p(scales), _p(zeros), rows, d_in, bits, _p(W_hat)))


def clha_dequant_matmul(ctx: Context, X, n: int, packed, scales, zeros, d_out: int, d_in: int, bits: int, Y):
    ctx._check(load().clha_dequant_matmul(ctx.handle, _p(X), _dtype(X), n, _p(packed), _p(scales), _p(zeros), d_out,
                                          d_in, bits, _p(Y)))


def clha_routing_divergence(ctx: Context, counts, n_layers: int, ld: int, slot0: int, E: int, tv):
    """tv (float64 device [n_layers, n_layers]) = total-variation distance of the layers' expert
    frequencies over experts [slot0, slot0 + E) of counts (int64 device [n_layers, ld])."""
    ctx._check(load().clha_routing_divergence(ctx.handle, _p(counts), n_layers, ld, slot0, E, _p(tv)))


def clha_quantize(ctx: Context, U, n_u: int, W, batch: int, d_out: int, d_in: int, bits: int, codes, scales,
                  zeros, W_hat=None, group: int = 128, block: int = 128, damp_frac: float = 0.01, lam=None, loss=None,
                  form: int = FACTOR_INV_CHOL):
    """lam (float64 device [n_u]) and loss (float64 device [batch]) request the in-kernel loss; form: what
    U holds (FACTOR_BLOCK_CHOL: F from clha_factor_groups with that form)."""
    qp = QuantParams(bits, group, block, damp_frac)
    if form == FACTOR_INV_CHOL:
        ctx._check(load().clha_quantize(ctx.handle, _p(U), n_u, _p(W), _dtype(W), batch, d_out, d_in, C.byref(qp),
                                        _p(codes), _p(scales), _p(zeros), _p(W_hat), _p(lam), _p(loss)))
    else:
        ctx._check(load().clha_quantize_as(ctx.handle, form, _p(U), n_u, _p(W), _dtype(W), batch, d_out, d_in,
                                           C.byref(qp), _p(codes), _p(scales), _p(zeros), _p(W_hat), _p(lam),
                                           _p(loss)))


def clha_loss(ctx: Context, W, W_hat, H, n_h: int, batch: int, d_out: int, d_in: int) -> np.ndarray:
    out = np.empty(batch, np.float64)
    ctx._check(load().clha_loss(ctx.handle, _p(W), _dtype(W), _p(W_hat), _p(H), n_h, batch, d_out, d_in, _p(out)))
    return out


def _mat_ptr(S, first: int, n_outer: int, outer_stride: int, n_inner: int, d: int):
    """Address of matrix `first` of a contiguous stack of d x d float32 matrices, after checking that the
    strided batch (o * outer_stride + i, o < n_outer, i < n_inner, from `first`) stays inside it."""
    ptr = _p(S)
    if S.dtype != torch.float32 or S.numel() % (d * d):
        raise ValueError("expected a stack of d x d float32 matrices")
    last = first + (n_outer - 1) * outer_stride + n_inner if n_outer * n_inner else first
    if first < 0 or last * d * d > S.numel():
        raise ValueError("matrix batch outside the tensor")
    return ptr + first * d * d * 4 if ptr else ptr


def clha_pack_upper(ctx: Context, S, n_outer: int, outer_stride: int, n_inner: int, d: int, packed, first: int = 0):
    """Upper triangles of matrices first + o * outer_stride + i (o < n_outer, i < n_inner) of the
    contiguous stack S (e.g. an accumulator's S viewed as [layers * slots, d, d]) into packed."""
    ctx._check(load().clha_pack_upper(ctx.handle, _mat_ptr(S, first, n_outer, outer_stride, n_inner, d), n_outer,
                                      outer_stride, n_inner, d, _p(packed)))


def clha_unpack_upper(ctx: Context, packed, n_outer: int, outer_stride: int, n_inner: int, d: int, S, first: int = 0):
    """The inverse of clha_pack_upper on the upper triangles (the strict lower ones are left alone)."""
    ctx._check(load().clha_unpack_upper(ctx.handle, _p(packed), n_outer, outer_stride, n_inner, d,
                                        _mat_ptr(S, first, n_outer, outer_stride, n_inner, d)))
