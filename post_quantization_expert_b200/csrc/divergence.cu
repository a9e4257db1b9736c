// Cross-layer routing divergence (the CLHA page, sections 4-5, ties CLHA's gains to it without a
// formula; read as the total-variation distance of two layers' expert frequencies):
//   TV[a][b] = 1/2 sum_e |n_{a,e} / N_a - n_{b,e} / N_b|,   N_l = sum_e n_{l,e}.
// One block per (a, b): the totals and sum_e |n_{a,e} N_b - n_{b,e} N_a| are exact 64-bit integer
// sums (counts below 2^31 per layer keep every product and the sum below 2^63), then one float64
// division by 2 N_a N_b, which is the correctly rounded quotient while both integers are exact in
// float64 (2 N_a N_b <= 2^53).
#include "clha_internal.h"

namespace {

constexpr int THREADS = 256;

// Sum over the block (every thread gets the total); `red` holds one slot per warp.
__device__ __forceinline__ long long block_sum(long long v, long long* red) {
    for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    __syncthreads();   // a previous call's readers are done with `red`
    if (lane == 0) red[warp] = v;
    __syncthreads();
    long long t = 0;
#pragma unroll
    for (int w = 0; w < THREADS / 32; ++w) t += red[w];
    return t;
}

__global__ void __launch_bounds__(THREADS) tv_kernel(const int64_t* __restrict__ counts, int L, int ld, int slot0,
                                                     int E, double* __restrict__ tv, int* err) {
    __shared__ long long red[THREADS / 32];
    const int a = blockIdx.x / L, b = blockIdx.x % L;
    const int64_t* ca = counts + (int64_t)a * ld + slot0;
    const int64_t* cb = counts + (int64_t)b * ld + slot0;
    // every count in [0, 2^31) keeps the partial totals below 2^62 (no wrap-around to trust)
    const long long LIM = 1ll << 31;
    long long na = 0, nb = 0, bad = 0;
    for (int e = threadIdx.x; e < E; e += THREADS) {
        const long long x = ca[e], y = cb[e];
        const bool ok = x >= 0 && x < LIM && y >= 0 && y < LIM;
        na += ok ? x : 0;
        nb += ok ? y : 0;
        bad += !ok;
    }
    bad = block_sum(bad, red);
    na = block_sum(na, red);
    nb = block_sum(nb, red);
    if (bad != 0 || na <= 0 || nb <= 0 || na >= LIM || nb >= LIM) {
        if (threadIdx.x == 0) {
            const bool empty = bad == 0 && (na == 0 || nb == 0);
            clha_record_error(err, empty ? CLHA_ERR_EMPTY : CLHA_ERR_INVALID_ARG, na <= 0 || na >= LIM ? a : b, 0,
                              KID_DIVERGENCE);
            tv[(int64_t)a * L + b] = __longlong_as_double(0x7ff8000000000000ll);   // NaN
        }
        return;
    }
    long long num = 0;
    for (int e = threadIdx.x; e < E; e += THREADS) {
        const long long x = ca[e] * nb - cb[e] * na;
        num += x < 0 ? -x : x;
    }
    num = block_sum(num, red);
    if (threadIdx.x == 0) tv[(int64_t)a * L + b] = (double)num / (double)(2 * na * nb);
}

}  // namespace

cudaError_t launch_routing_divergence(cudaStream_t s, const int64_t* counts, int L, int ld, int slot0, int E,
                                      double* tv, int* err) {
    tv_kernel<<<L * L, THREADS, 0, s>>>(counts, L, ld, slot0, E, tv, err);
    clha_note_launches(1);
    return cudaGetLastError();
}
