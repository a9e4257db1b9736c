// E-PMQ's quantization target (the E-PMQ page, section 2, "Implementatie van de Oplosser"): with the
// statistics H = sum_i H_i + lambda I and R = sum_i W_i H_i + lambda W_m, the objective
// sum_i ||Q X_i - W_i X_i||^2 + lambda ||Q - W_m||^2 equals tr[(Q - W*) H (Q - W*)^T] + const with
// W* = R H^-1, so GPTQ of W* under H solves it. This file computes W* in float64 on the FP64 tensor
// path, from the accumulator's per-source Gram matrices S_i (= H_i), the damped aggregate's lambda
// and factor U (H^-1 = U^T U):
//   R    = lambda W_m + sum_i W_i S_i           (S_i read symmetrically from its upper triangle)
//   Hinv = U^T U
//   W*   = R Hinv                               (float32 out, the input of GPTQ)
// One kernel does all three: C (64x64 tile per CTA) = init + sum_b sum_k P_b[m][k] Q_b[n][k], the
// operands described by how their elements are stored (row-major, transposed, or symmetric with the
// upper triangle stored), each 64x64 tile loaded into padded shared memory as float64 with the
// thread mapping that keeps the global reads coalesced; products are mma.sync m8n8k4 f64.
#include "clha_internal.h"

namespace {

constexpr int NB = 64;
constexpr int LD = NB + 4;   // padded shared row (doubles): conflict-free fragment loads
constexpr int TILE_DOUBLES = NB * LD;

enum Kind { K_F32 = 0, K_BF16 = 1, K_F64 = 2, K_F32_T = 3, K_F32_SYMU = 4 };

struct Operand {
    const void* p;
    int kind;
    int64_t ld;        // row stride of the stored matrix (elements)
    int64_t bstride;   // stride between batch items (elements)
};

// Element (r, c) of batch item b of the logical matrix, as a double.
__device__ __forceinline__ double elem(const Operand& o, int b, int64_t r, int64_t c) {
    const int64_t base = (int64_t)b * o.bstride;
    switch (o.kind) {
        case K_F32: return (double)reinterpret_cast<const float*>(o.p)[base + r * o.ld + c];
        case K_BF16: return (double)__bfloat162float(reinterpret_cast<const __nv_bfloat16*>(o.p)[base + r * o.ld + c]);
        case K_F64: return reinterpret_cast<const double*>(o.p)[base + r * o.ld + c];
        case K_F32_T: return (double)reinterpret_cast<const float*>(o.p)[base + c * o.ld + r];
        default: {
            const int64_t lo = r < c ? r : c, hi = r < c ? c : r;
            return (double)reinterpret_cast<const float*>(o.p)[base + lo * o.ld + hi];
        }
    }
}

// 64x64 logical tile starting at (r0, c0) into shared memory. Memory is contiguous along c for
// row-major storage (and for the upper part of a symmetric one), along r for transposed storage
// (and the lower part): consecutive threads take consecutive addresses either way.
__device__ __forceinline__ void load_tile(double (*dst)[LD], const Operand& o, int b, int64_t r0, int64_t c0) {
    const bool along_r = o.kind == K_F32_T || (o.kind == K_F32_SYMU && r0 > c0);
#pragma unroll 4
    for (int e = threadIdx.x; e < NB * NB; e += 256) {
        const int a = e >> 6, f = e & 63;
        const int r = along_r ? f : a, c = along_r ? a : f;
        dst[r][c] = elem(o, b, r0 + r, c0 + c);
    }
}

__device__ __forceinline__ void dmma(double& c0, double& c1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(c0), "+d"(c1)
                 : "d"(a), "d"(b));
}

struct GemmArgs {
    Operand P, Q;       // C[m][n] = init + sum_b sum_k P_b[m][k] Q_b[n][k]
    int nb, K;
    Operand init;       // init[m][n] (batch 0), scaled by *init_scale; init.p null: zero
    const double* init_scale;
    double* out64;      // [M, N] row-major, or
    float* out32;
};

__global__ void __launch_bounds__(256) epmq_gemm(GemmArgs g) {
    extern __shared__ __align__(16) double esm[];
    double (*Ps)[LD] = reinterpret_cast<double (*)[LD]>(esm);
    double (*Qs)[LD] = reinterpret_cast<double (*)[LD]>(esm + TILE_DOUBLES);
    const int64_t n0 = (int64_t)blockIdx.x * NB, m0 = (int64_t)blockIdx.y * NB;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int gq = lane >> 2, tq = lane & 3;
    const int wm = warp >> 2, wn = warp & 3;   // warp block: rows 32 wm .., cols 16 wn ..
    double c[4][2][2] = {};
    for (int b = 0; b < g.nb; ++b) {
        for (int k0 = 0; k0 < g.K; k0 += NB) {
            __syncthreads();   // the previous tiles are consumed
            load_tile(Ps, g.P, b, m0, k0);
            load_tile(Qs, g.Q, b, n0, k0);
            __syncthreads();
#pragma unroll 4
            for (int kk = 0; kk < NB; kk += 4) {
                double a[4], bq[2];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi) a[mi] = Ps[32 * wm + 8 * mi + gq][kk + tq];
#pragma unroll
                for (int ni = 0; ni < 2; ++ni) bq[ni] = Qs[16 * wn + 8 * ni + gq][kk + tq];
#pragma unroll
                for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                    for (int ni = 0; ni < 2; ++ni) dmma(c[mi][ni][0], c[mi][ni][1], a[mi], bq[ni]);
            }
        }
    }
    const double scale = g.init.p ? *g.init_scale : 0.0;
    const int64_t N = (int64_t)gridDim.x * NB;
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 2; ++ni)
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                const int64_t m = m0 + 32 * wm + 8 * mi + gq, n = n0 + 16 * wn + 8 * ni + 2 * tq + h;
                double v = c[mi][ni][h];
                if (g.init.p) v += scale * elem(g.init, 0, m, n);
                if (g.out64) g.out64[m * N + n] = v;
                else g.out32[m * N + n] = (float)v;
            }
}

constexpr int SMEM = 2 * TILE_DOUBLES * sizeof(double);

cudaError_t run(cudaStream_t s, const GemmArgs& g, int M, int N) {
    // per call: the attribute belongs to the current device's context (a process may drive several)
    cudaError_t e = cudaFuncSetAttribute(epmq_gemm, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM);
    if (e != cudaSuccess) return e;
    epmq_gemm<<<dim3(N / NB, M / NB), 256, SMEM, s>>>(g);
    clha_note_launches(1);
    return cudaGetLastError();
}

}  // namespace

size_t epmq_workspace_bytes(int d_out, int d) {
    return clha_round_up((size_t)d_out * d * sizeof(double)) + clha_round_up((size_t)d * d * sizeof(double));
}

cudaError_t launch_epmq_target(cudaStream_t s, const float* S_slot, int64_t layer_stride, int K, const void* W_src,
                               int w_bf16, const void* W_m, int d_out, int d, const float* U, const double* lambda,
                               float* W_target, void* ws) {
    char* cur = (char*)ws;
    double* R = (double*)clha_carve(cur, (size_t)d_out * d * sizeof(double));
    double* Hinv = (double*)clha_carve(cur, (size_t)d * d * sizeof(double));
    const int wk = w_bf16 ? K_BF16 : K_F32;
    cudaError_t e;
    // R = lambda W_m + sum_i W_i S_i
    GemmArgs g1{};
    g1.P = Operand{W_src, wk, d, (int64_t)d_out * d};
    g1.Q = Operand{S_slot, K_F32_SYMU, d, layer_stride};
    g1.nb = K;
    g1.K = d;
    g1.init = Operand{W_m, wk, d, 0};
    g1.init_scale = lambda;
    g1.out64 = R;
    if ((e = run(s, g1, d_out, d)) != cudaSuccess) return e;
    // Hinv = U^T U: P[a][j] = U[j][a], Q[c][j] = U[j][c]
    GemmArgs g2{};
    g2.P = Operand{U, K_F32_T, d, 0};
    g2.Q = Operand{U, K_F32_T, d, 0};
    g2.nb = 1;
    g2.K = d;
    g2.out64 = Hinv;
    if ((e = run(s, g2, d, d)) != cudaSuccess) return e;
    // W* = R Hinv (Hinv symmetric: Q[n][k] = Hinv[k][n] = Hinv[n][k])
    GemmArgs g3{};
    g3.P = Operand{R, K_F64, d, 0};
    g3.Q = Operand{Hinv, K_F64, d, 0};
    g3.nb = 1;
    g3.K = d;
    g3.out32 = W_target;
    return run(s, g3, d_out, d);
}
