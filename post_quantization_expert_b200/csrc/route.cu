// Top-k routing of tokens to experts (the CLHA page, §2.2 (1): statistics are gathered per active
// expert; §2.3: a routed expert sees K of E slots per token).
//
// One warp per token. Each lane holds E/32 logits (coalesced loads). k rounds of a warp-wide
// arg-max over (value, expert index) pairs pick the experts in descending logit order; equal logits
// go to the lower expert index. Counts go through a shared-memory histogram per block, then one
// global atomic per (block, expert).
#include "clha_internal.h"

namespace {

constexpr int kWarps = 8;

template <int VPL>  // values per lane: E <= 32 * VPL
__global__ void __launch_bounds__(kWarps * 32)
route_topk_kernel(const float* __restrict__ logits, int64_t n, int E, int k, int32_t* __restrict__ ids,
                  int32_t* __restrict__ counts, int* err) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    const int lane = threadIdx.x & 31;
    const int64_t warp_global = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
    const int64_t warp_stride = (int64_t)gridDim.x * kWarps;
    for (int64_t t = warp_global; t < n; t += warp_stride) {
        float v[VPL];
        bool live[VPL];
        bool bad = false;
#pragma unroll
        for (int i = 0; i < VPL; ++i) {
            int e = lane + 32 * i;
            live[i] = e < E;
            v[i] = live[i] ? logits[t * E + e] : 0.f;
            if (live[i] && !isfinite(v[i])) bad = true;
        }
        if (__any_sync(0xffffffffu, bad)) {
            if (lane == 0) clha_record_error(err, CLHA_ERR_NONFINITE, (int)(t & 0x7fffffff), 0, KID_ROUTE);
        }
        for (int r = 0; r < k; ++r) {
            // best live entry of this lane: larger value wins, equal values -> lower index
            float bv = 0.f;
            int bi = 0x7fffffff;
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                int e = lane + 32 * i;
                if (live[i] && (bi == 0x7fffffff || v[i] > bv)) { bv = v[i]; bi = e; }
            }
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) {
                float ov = __shfl_xor_sync(0xffffffffu, bv, off);
                int oi = __shfl_xor_sync(0xffffffffu, bi, off);
                bool take = (oi != 0x7fffffff) &&
                            (bi == 0x7fffffff || ov > bv || (ov == bv && oi < bi));
                if (take) { bv = ov; bi = oi; }
            }
            // the owner retires the winner
#pragma unroll
            for (int i = 0; i < VPL; ++i)
                if (lane + 32 * i == bi) live[i] = false;
            if (lane == 0) {
                ids[t * k + r] = bi;
                atomicAdd(&hist[bi], 1);
            }
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x)
        if (hist[e]) atomicAdd(&counts[e], hist[e]);
}

template <int VPL>
cudaError_t launch_v(cudaStream_t s, const float* logits, int64_t n, int E, int k, int32_t* ids,
                     int32_t* counts, int* err) {
    int64_t blocks = (n + kWarps - 1) / kWarps;
    if (blocks > 148 * 16) blocks = 148 * 16;
    if (blocks < 1) blocks = 1;
    route_topk_kernel<VPL><<<(unsigned)blocks, kWarps * 32, E * sizeof(int), s>>>(logits, n, E, k, ids, counts, err);
    clha_note_launches(1);
    return cudaGetLastError();
}

}  // namespace

cudaError_t launch_route_topk(cudaStream_t s, const float* logits, int64_t n, int E, int k, int32_t* ids,
                              int32_t* counts, int* err) {
    cudaError_t e = cudaMemsetAsync(counts, 0, E * sizeof(int32_t), s);
    if (e != cudaSuccess || n == 0) return e;
    if (E <= 32) return launch_v<1>(s, logits, n, E, k, ids, counts, err);
    if (E <= 64) return launch_v<2>(s, logits, n, E, k, ids, counts, err);
    if (E <= 128) return launch_v<4>(s, logits, n, E, k, ids, counts, err);
    if (E <= 256) return launch_v<8>(s, logits, n, E, k, ids, counts, err);
    if (E <= 512) return launch_v<16>(s, logits, n, E, k, ids, counts, err);
    return launch_v<32>(s, logits, n, E, k, ids, counts, err);
}
