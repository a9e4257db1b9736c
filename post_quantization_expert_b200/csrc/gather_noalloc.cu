// clha_gather_noalloc: the routed-token gather without any device allocation.
//
// clha_gather takes its scratch (per-block expert histograms and the token permutation) from the
// context's workspace, which grows with cudaMalloc/cudaFree. This variant takes the same scratch
// from a fixed array that lives in the library's device image instead, for callers that must not
// see a library allocate: processes whose device memory is handed out by their own allocator (a
// framework's caching allocator, a fixed arena) where a cudaMalloc can fail after the arena took
// the memory and a cudaFree synchronises the whole device.
//
// The array is a file-scope __device__ object, so every GPU that loads libclha.so holds it until
// the process exits. In host code its name only stands for the symbol; its device address comes
// from cudaGetSymbolAddress, looked up on every call with the call's device current (a cheap
// lookup, and one that stays right if the context is reset and the module loaded again at another
// address). All calls share the array and it keeps the last call's contents: the gather rewrites
// every histogram entry it reads and resets a permutation kept in the array to -1 before
// scattering, and calls that overlap on the GPU (different streams, different contexts) race on it.
//
// Scratch per call: the per-block expert histograms, ceil(n/256)*E int32 entries (256 tokens per block), and, only when
// the caller passes no perm array, the token permutation, packed_rows int32 entries (each part
// rounded up to 256 bytes).
#include "clha_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(4) << 20;  // 4 MiB
static __device__ __align__(256) unsigned char g_gather_scratch[kScratchBytes];

// Bytes of the fixed array this gather uses: what launch_gather carves out of it.
size_t noalloc_scratch_bytes(int64_t n, int E, int64_t packed_rows, bool perm_given) {
    int64_t nblk = (n + kGatherBlockTokens - 1) / kGatherBlockTokens;
    if (nblk < 1) nblk = 1;
    size_t b = clha_round_up((size_t)nblk * E * sizeof(int));
    if (!perm_given) b += clha_round_up((size_t)packed_rows * sizeof(int32_t));
    return b;
}

}  // namespace

extern "C" clha_status clha_gather_noalloc(clha_ctx* ctx, const void* X, clha_dtype dtype, int64_t n, int d,
                                           const int32_t* ids, int k, int E, void* X_packed, int64_t packed_rows,
                                           int64_t* seg, int32_t* perm) {
    if (!ctx) return CLHA_ERR_INVALID_ARG;
    const int es = dtype == CLHA_BF16 ? 2 : (dtype == CLHA_F32 ? 4 : 0);
    if (!es) return clha_fail(ctx, CLHA_ERR_INVALID_ARG, "clha_gather_noalloc: unknown dtype");
    if (n < 0 || d <= 0) return clha_fail(ctx, CLHA_ERR_INVALID_ARG, "clha_gather_noalloc: bad sizes");
    if (E < 1 || E > 1024 || k < 1 || k > E)
        return clha_fail(ctx, CLHA_ERR_INVALID_ARG, "clha_gather_noalloc: need 1 <= k <= E <= 1024");
    if (d % 128 != 0)
        return clha_fail(ctx, CLHA_ERR_UNSUPPORTED_SHAPE, "clha_gather_noalloc: d=%d is not a multiple of 128", d);
    if (packed_rows < clha_packed_rows(n, k, E))
        return clha_fail(ctx, CLHA_ERR_INVALID_ARG, "clha_gather_noalloc: packed_rows %lld < %lld",
                         (long long)packed_rows, (long long)clha_packed_rows(n, k, E));
    if (!seg || (!X_packed && !perm) || (n > 0 && !ids) || (X_packed && n > 0 && !X))
        return clha_fail(ctx, CLHA_ERR_INVALID_ARG, "clha_gather_noalloc: null pointer");
    const size_t need = noalloc_scratch_bytes(n, E, packed_rows, perm != nullptr);
    if (need > kScratchBytes)
        return clha_fail(ctx, CLHA_ERR_INVALID_ARG,
                         "clha_gather_noalloc: this gather needs %zu bytes of scratch but the fixed array holds %zu "
                         "(4 MiB); use clha_gather, pass a perm array, or fewer tokens / experts per call",
                         need, kScratchBytes);
    cudaError_t e = cudaSetDevice(ctx->device);
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, "clha_gather_noalloc: cudaSetDevice");
    void* scratch = nullptr;
    e = cudaGetSymbolAddress(&scratch, g_gather_scratch);
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, "clha_gather_noalloc: cudaGetSymbolAddress");
    const int64_t l0 = clha_total_launches();
    e = launch_gather(ctx->stream, X, es, n, d, ids, k, E, X_packed, packed_rows, seg, perm, scratch, kScratchBytes,
                      ctx->d_err);
    ctx->launches += clha_total_launches() - l0;
    if (e != cudaSuccess) return clha_cuda_check(ctx, e, "clha_gather_noalloc");
    return CLHA_OK;
}
