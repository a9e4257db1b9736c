// Phase 2 of CLHA (the CLHA page, §2.1 Proposition 1 and §2.2 (2)): H_comb = sum_i alpha_i H_i with
// H_i = (2 / n_i) S_i, routing-frequency (alpha_i = n_i / sum n), equal (1/L) or explicit weights,
// or the plain Gram sum (alpha_i = n_i / 2, H_comb = sum S_i: the E-PMQ statistics), then GPTQ
// damping H_d = H_comb + lambda I, lambda = damp_frac * mean(diag H_comb); on request a slot without
// energy (tr H_comb = 0) gets lambda = 1, so H_d = I and GPTQ under it is round to nearest.
//
// Two kernels per call, both HBM-bound:
//   agg_scalars  one block per slot: alpha (float64), lambda from the diagonals (float64 reduction),
//                empty-slot and non-finite checks;
//   agg_combine  one block per 64x64 upper tile pair: reads each layer's upper tile of S once (16-byte
//                loads) and writes both the tile and its mirror image (through shared memory, coalesced
//                16-byte stores).
#include "clha_internal.h"

namespace {

__device__ __forceinline__ double layer_coef(const double* alpha, const int64_t* cnt, int l) {
    int64_t n = cnt[l];
    return n > 0 ? alpha[l] * 2.0 / (double)n : 0.0;
}

__global__ void __launch_bounds__(256) agg_scalars(const float* __restrict__ S, const int64_t* __restrict__ counts,
                                                   int d, int L, int n_slots_total, int slot0, clha_alpha_args a,
                                                   double damp_frac, double* __restrict__ d_alpha,
                                                   double* __restrict__ d_lambda, int* err) {
    const int sl = blockIdx.x;
    const int slot = slot0 + sl;
    __shared__ double alpha[CLHA_MAX_LAYERS];
    __shared__ int64_t cnt[CLHA_MAX_LAYERS];
    __shared__ double red[256];
    const int amode = a.mode & 0xff;
    const bool identity = (a.mode & CLHA_AGG_EMPTY_IDENTITY) != 0;
    if (threadIdx.x == 0) {
        int64_t tot = 0;
        for (int l = 0; l < L; ++l) {
            cnt[l] = counts[(size_t)l * n_slots_total + slot];
            tot += cnt[l];
        }
        for (int l = 0; l < L; ++l) {
            double al;
            if (amode == CLHA_ALPHA_ROUTING) al = tot > 0 ? (double)cnt[l] / (double)tot : 0.0;
            else if (amode == CLHA_ALPHA_EQUAL) al = 1.0 / L;
            else if (amode == CLHA_ALPHA_SUM) al = (double)cnt[l] / 2.0;
            else al = a.alpha[l];
            alpha[l] = al;
            d_alpha[(size_t)sl * L + l] = al;
        }
        if (tot == 0 && !identity) clha_record_error(err, CLHA_ERR_EMPTY, slot, 0, KID_AGGREGATE);
    }
    __syncthreads();
    double acc = 0.0;
    for (int i = threadIdx.x; i < d; i += blockDim.x) {
        double v = 0.0;
        for (int l = 0; l < L; ++l) {
            double c = layer_coef(alpha, cnt, l);
            if (c != 0.0) v += c * (double)S[(((size_t)l * n_slots_total + slot) * d + i) * d + i];
        }
        acc += v;
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int off = 128; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        double lam = damp_frac * red[0] / d;
        if (identity && red[0] == 0.0) lam = 1.0;   // no energy: H_d = I (round to nearest)
        d_lambda[sl] = lam;
        if (!isfinite(red[0])) clha_record_error(err, CLHA_ERR_NONFINITE, slot, -1, KID_AGGREGATE);
    }
}

// One block per 64x64 upper tile pair (bi <= bj) of one slot: each thread combines 4 rows x 4 columns
// of the upper tile from 16-byte loads of every layer's S (v = sum_l coef_l S_l, fused multiply-adds in
// layer order), writes them with 16-byte stores, and the mirror tile (and, in a diagonal tile, the
// lower half) comes transposed through shared memory.
__global__ void __launch_bounds__(256) agg_combine(const float* __restrict__ S, const int64_t* __restrict__ counts,
                                                   int d, int L, int n_slots_total, int slot0,
                                                   const double* __restrict__ d_alpha,
                                                   const double* __restrict__ d_lambda, float* __restrict__ H_comb,
                                                   float* __restrict__ H_d, int* err) {
    constexpr int T = 64;
    const int sl = blockIdx.y;
    const int slot = slot0 + sl;
    const int nt = d / T;
    int t = blockIdx.x, bi = 0;
    while (t >= nt - bi) { t -= nt - bi; ++bi; }
    const int bj = bi + t;  // bi <= bj
    __shared__ float tile[T][T + 1];
    __shared__ float coef[CLHA_MAX_LAYERS];
    if (threadIdx.x < L) {
        int64_t n = counts[(size_t)threadIdx.x * n_slots_total + slot];
        coef[threadIdx.x] = n > 0 ? (float)(d_alpha[(size_t)sl * L + threadIdx.x] * 2.0 / (double)n) : 0.f;
    }
    __syncthreads();
    const float lam = (float)d_lambda[sl];
    const int c4 = (threadIdx.x & 15) * 4, r0 = threadIdx.x >> 4;   // rows r0, r0 + 16, r0 + 32, r0 + 48
    float v[4][4];
    bool bad = false;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int r = r0 + 16 * k;
        const size_t off = (size_t)(bi * T + r) * d + bj * T + c4;
#pragma unroll
        for (int q = 0; q < 4; ++q) v[k][q] = 0.f;
        for (int l = 0; l < L; ++l) {
            const float c = coef[l];
            if (c != 0.f) {
                const float4 sv = *reinterpret_cast<const float4*>(S + ((size_t)l * n_slots_total + slot) * d * d + off);
                v[k][0] = fmaf(c, sv.x, v[k][0]);
                v[k][1] = fmaf(c, sv.y, v[k][1]);
                v[k][2] = fmaf(c, sv.z, v[k][2]);
                v[k][3] = fmaf(c, sv.w, v[k][3]);
            }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            if (!isfinite(v[k][q])) bad = true;
            tile[r][c4 + q] = v[k][q];
        }
    }
    if (bad) clha_record_error(err, CLHA_ERR_NONFINITE, slot, bi * T, KID_AGGREGATE);
    __syncthreads();
    float* Hc = H_comb ? H_comb + (size_t)sl * d * d : nullptr;
    float* Hd = H_d + (size_t)sl * d * d;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
        const int r = r0 + 16 * k;
        // upper tile (bi, bj); inside a diagonal tile entries below the diagonal take the upper value
        float4 o;
        float* op = reinterpret_cast<float*>(&o);
#pragma unroll
        for (int q = 0; q < 4; ++q) op[q] = (bi == bj && r > c4 + q) ? tile[c4 + q][r] : v[k][q];
        const size_t up = (size_t)(bi * T + r) * d + bj * T + c4;
        if (Hc) *reinterpret_cast<float4*>(Hc + up) = o;
        if (bi == bj && r >= c4 && r < c4 + 4) op[r - c4] += lam;
        *reinterpret_cast<float4*>(Hd + up) = o;
        if (bi != bj) {   // mirror tile (bj, bi): entry (r, c) = upper (c, r)
            float4 m;
            float* mp = reinterpret_cast<float*>(&m);
#pragma unroll
            for (int q = 0; q < 4; ++q) mp[q] = tile[c4 + q][r];
            const size_t lo = (size_t)(bj * T + r) * d + bi * T + c4;
            if (Hc) *reinterpret_cast<float4*>(Hc + lo) = m;
            *reinterpret_cast<float4*>(Hd + lo) = m;
        }
    }
}

}  // namespace

cudaError_t launch_aggregate(cudaStream_t s, const float* S, const int64_t* counts, int d, int n_layers,
                             int n_slots_total, int slot0, int n_slots, clha_alpha_args a, double damp_frac,
                             float* H_comb, float* H_d, double* d_alpha, double* d_lambda, int* err) {
    agg_scalars<<<n_slots, 256, 0, s>>>(S, counts, d, n_layers, n_slots_total, slot0, a, damp_frac, d_alpha, d_lambda,
                                        err);
    clha_note_launches(1);
    int nt = d / 64;
    dim3 grid(nt * (nt + 1) / 2, n_slots);
    agg_combine<<<grid, 256, 0, s>>>(S, counts, d, n_layers, n_slots_total, slot0, d_alpha, d_lambda, H_comb, H_d,
                                     err);
    clha_note_launches(1);
    return cudaGetLastError();
}
