// Packing of Gram accumulators for the token-sharded collection's exchange between GPUs.
//
// Phase 1 of CLHA (the CLHA page, §2.2 (1)) is a sum over tokens, so with the tokens split over
// several GPUs each holds partial Gram sums S; the expert that owns a slot needs the sum over GPUs.
// S is symmetric and only its upper triangle is authoritative, so the exchange moves the packed
// upper triangles (d(d+1)/2 floats per matrix instead of d^2), and a reduce-scatter delivers to each
// GPU only the slots it quantizes. These two kernels pack a batch of matrices into that layout and
// unpack the summed result; both are plain coalesced copies, one warp per matrix row.
//
// Packed layout of one d x d matrix: row i holds entries (i, i .. d-1), rows in order, so row i
// starts at i*d - i*(i-1)/2. A batch of matrices m = o * outer_stride + i (o < n_outer, i < n_inner,
// in units of matrices from the base pointer) is packed in (o, i) order, one after the other.
#include "clha_internal.h"

namespace {

__device__ __forceinline__ int64_t row_start(int64_t i, int64_t d) { return i * d - i * (i - 1) / 2; }

__global__ void __launch_bounds__(256) pack_upper_k(const float* __restrict__ S, int64_t n_outer, int64_t outer_stride,
                                                    int64_t n_inner, int d, float* __restrict__ P) {
    const int64_t rows = n_outer * n_inner * d;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t i = r % d, mi = r / d;                 // row, packed matrix index (o * n_inner + inner)
    const int64_t o = mi / n_inner, in = mi - o * n_inner;
    const float* src = S + ((o * outer_stride + in) * d + i) * d;
    float* dst = P + mi * ((int64_t)d * (d + 1) / 2) + row_start(i, d) - i;
    for (int64_t j = i + lane; j < d; j += 32) dst[j] = __ldg(src + j);
}

__global__ void __launch_bounds__(256) unpack_upper_k(const float* __restrict__ P, int64_t n_outer,
                                                      int64_t outer_stride, int64_t n_inner, int d,
                                                      float* __restrict__ S) {
    const int64_t rows = n_outer * n_inner * d;
    const int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
    if (r >= rows) return;
    const int lane = threadIdx.x & 31;
    const int64_t i = r % d, mi = r / d;
    const int64_t o = mi / n_inner, in = mi - o * n_inner;
    float* dst = S + ((o * outer_stride + in) * d + i) * d;
    const float* src = P + mi * ((int64_t)d * (d + 1) / 2) + row_start(i, d) - i;
    for (int64_t j = i + lane; j < d; j += 32) dst[j] = __ldg(src + j);
}

}  // namespace

cudaError_t launch_pack_upper(cudaStream_t s, const float* S, int64_t n_outer, int64_t outer_stride, int64_t n_inner,
                              int d, float* P) {
    const int64_t rows = n_outer * n_inner * d;
    if (rows == 0) return cudaSuccess;
    pack_upper_k<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(S, n_outer, outer_stride, n_inner, d, P);
    clha_note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_unpack_upper(cudaStream_t s, const float* P, int64_t n_outer, int64_t outer_stride,
                                int64_t n_inner, int d, float* S) {
    const int64_t rows = n_outer * n_inner * d;
    if (rows == 0) return cudaSuccess;
    unpack_upper_k<<<(unsigned)((rows + 7) / 8), 256, 0, s>>>(P, n_outer, outer_stride, n_inner, d, S);
    clha_note_launches(1);
    return cudaGetLastError();
}
