// Expert FFN activation h = SiLU(x Wg^T) * (x Wu^T) for every row of every expert segment: the input
// of the expert's down projection, whose Hessian phase 1 collects. fp32 accumulation, bf16 output
// (round to nearest even). Padding rows of a segment are written as zero, so h has exactly the
// segment layout of its input and can be collected the same way.
//
// Shared-memory tiled FMA kernel: a 64-row x 64-column output tile computes the gate and the up
// tile together (two accumulators per thread), so the SiLU-times-up epilogue needs no second pass.
// Products of bf16 values are exact in fp32; each 32-term chunk is summed in fp32 and the chunk sums
// in fp64, which keeps the rounding of h to bf16 at the correctly rounded value far more often than
// one long fp32 sum would (inputs with outlier channels cancel heavily); the SiLU product is
// evaluated in fp64 and rounded once to bf16.
#include "clha_internal.h"

namespace {

constexpr int TM = 64, TN = 64, TK = 32;

__device__ __forceinline__ int find_segment(const int64_t* seg, int E, int64_t row) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // last e with seg[e] <= row
        int mid = (lo + hi + 1) >> 1;
        if (seg[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__global__ void __launch_bounds__(256) expert_act_simt(const __nv_bfloat16* __restrict__ X, int64_t rows, int dm,
                                                       const int64_t* __restrict__ seg, int E,
                                                       const __nv_bfloat16* __restrict__ Wg,
                                                       const __nv_bfloat16* __restrict__ Wu, int dff,
                                                       __nv_bfloat16* __restrict__ h) {
    const int64_t m0 = (int64_t)blockIdx.x * TM;
    const int n0 = blockIdx.y * TN;
    int e = 0;
    int64_t valid_end = rows;
    if (seg) {
        if (m0 >= seg[E]) return;
        e = find_segment(seg, E, m0);
        valid_end = seg[e] + seg[E + 1 + e];
    }
    const __nv_bfloat16* wg = Wg + (size_t)e * dff * dm;
    const __nv_bfloat16* wu = Wu + (size_t)e * dff * dm;
    __shared__ float As[TK][TM + 4];
    __shared__ float Gs[TK][TN + 4];
    __shared__ float Us[TK][TN + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double ag[4][4] = {}, au[4][4] = {};
    for (int k0 = 0; k0 < dm; k0 += TK) {
        for (int i = threadIdx.x; i < TM * TK; i += 256) {
            int m = i / TK, kk = i % TK;
            int64_t row = m0 + m;
            As[kk][m] = (row < valid_end) ? __bfloat162float(X[row * dm + k0 + kk]) : 0.f;
            Gs[kk][m] = __bfloat162float(wg[(size_t)(n0 + m) * dm + k0 + kk]);
            Us[kk][m] = __bfloat162float(wu[(size_t)(n0 + m) * dm + k0 + kk]);
        }
        __syncthreads();
        float pg[4][4] = {}, pu[4][4] = {};
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], g[4], u[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                g[i] = Gs[kk][tx * 4 + i];
                u[i] = Us[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    pg[i][j] = fmaf(a[i], g[j], pg[i][j]);
                    pu[i][j] = fmaf(a[i], u[j], pu[i][j]);
                }
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                ag[i][j] += (double)pg[i][j];
                au[i][j] += (double)pu[i][j];
            }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        int64_t row = m0 + ty * 4 + i;
        if (row >= rows) continue;
        bool valid = row < valid_end;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const double g = ag[i][j];
            const double v = valid ? g / (1.0 + exp(-g)) * au[i][j] : 0.0;
            h[row * dff + n0 + tx * 4 + j] = __double2bfloat16(v);
        }
    }
}

}  // namespace

cudaError_t launch_expert_act(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d_model,
                              const int64_t* seg, int E, const __nv_bfloat16* Wg, const __nv_bfloat16* Wu, int d_ff,
                              __nv_bfloat16* h, int* err) {
    (void)num_sms;
    (void)err;
    dim3 grid((unsigned)((rows + TM - 1) / TM), d_ff / TN);
    expert_act_simt<<<grid, 256, 0, s>>>(X, rows, d_model, seg, E, Wg, Wu, d_ff, h);
    clha_note_launches(1);
    return cudaGetLastError();
}
