// Phase 3 of CLHA (the CLHA page, §2.2 (3)): GPTQ column-sequential quantization with the
// aggregated Hessian's factor U (H_d^-1 = U^T U), restated from GPTQ (Frantar et al. 2022, Alg. 1).
//
// One CTA owns 128 rows of one weight and walks the columns in 128-column blocks; one thread owns
// one row, so a row's whole block lives in that thread's registers and the column-by-column error
// feedback needs no communication at all. Per block:
//   1. lazy update, left-looking: the block's columns receive the errors of all earlier blocks at
//      once, w[:, blk] = W[:, blk] - E[:, :cb] U[:cb, blk], from the error rows this CTA wrote
//      earlier (shared-memory staged FMA);
//   2. grid of the group (group = block = 128 columns): min/max over the row's current values;
//   3. 128 sequential columns: q = clamp(round(w/s) + z), w_hat = s (q - z), e = (w - w_hat) / U_jj,
//      later columns of the block -= e * U[j, :] (broadcast from shared memory);
//   4. errors, codes and w_hat of the block go to memory.
// The grid and the code are decided with IEEE float32 operations (division and rounding to nearest
// even), so a kernel decision equals the float32 decision on the same current value.
#include "clha_internal.h"

namespace {

constexpr int R = 128;     // rows per CTA (one per thread)
constexpr int BLK = 128;   // columns per block and per group
constexpr int KC = 32;     // k-chunk of the left-looking update
constexpr int SMEM_BYTES = (BLK * BLK + BLK + KC * BLK + KC * (R + 1)) * sizeof(float);

__global__ void __launch_bounds__(R, 1) gptq_simt(const float* __restrict__ U, int w_per_u, const void* __restrict__ Wv,
                                                  int w_f32, int d_out, int d_in, int bits, uint8_t* __restrict__ codes,
                                                  float* __restrict__ scales, uint8_t* __restrict__ zeros,
                                                  float* __restrict__ W_hat, float* __restrict__ Escr) {
    extern __shared__ float sm[];
    float (*Ud)[BLK] = reinterpret_cast<float (*)[BLK]>(sm);
    float* uinv = sm + BLK * BLK;
    float (*Us)[BLK] = reinterpret_cast<float (*)[BLK]>(uinv + BLK);
    float (*Es)[R + 1] = reinterpret_cast<float (*)[R + 1]>(&Us[KC][0]);

    const int b = blockIdx.y;
    const int t = threadIdx.x;
    const int row = blockIdx.x * R + t;
    const size_t dd = (size_t)d_in * d_in;
    const float* Ub = U + (size_t)(b / w_per_u) * dd;
    const size_t wrow = ((size_t)b * d_out + row) * d_in;
    float* Erow = Escr + wrow;
    const float maxq = (float)((1 << bits) - 1);
    const int ngroups = d_in / BLK;

    for (int cb = 0; cb < d_in; cb += BLK) {
        float w[BLK];
#pragma unroll
        for (int c = 0; c < BLK; ++c) w[c] = 0.f;
        // 1. lazy update from all earlier blocks
        for (int k0 = 0; k0 < cb; k0 += KC) {
            __syncthreads();
            const float4* e4 = reinterpret_cast<const float4*>(Erow + k0);
#pragma unroll
            for (int i = 0; i < KC / 4; ++i) {
                float4 v = e4[i];
                Es[4 * i + 0][t] = v.x;
                Es[4 * i + 1][t] = v.y;
                Es[4 * i + 2][t] = v.z;
                Es[4 * i + 3][t] = v.w;
            }
#pragma unroll 4
            for (int kk = 0; kk < KC; ++kk) Us[kk][t] = Ub[(size_t)(k0 + kk) * d_in + cb + t];
            __syncthreads();
#pragma unroll 2
            for (int kk = 0; kk < KC; ++kk) {
                const float e = Es[kk][t];
#pragma unroll
                for (int c = 0; c < BLK; ++c) w[c] = fmaf(e, Us[kk][c], w[c]);
            }
        }
        __syncthreads();
        for (int i = 0; i < BLK; ++i) Ud[i][t] = Ub[(size_t)(cb + i) * d_in + cb + t];
        __syncthreads();
        uinv[t] = 1.0f / Ud[t][t];
        // current values of this row's block
        if (w_f32) {
            const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(Wv) + wrow + cb);
#pragma unroll
            for (int i = 0; i < BLK / 4; ++i) {
                float4 v = src[i];
                w[4 * i + 0] = v.x - w[4 * i + 0];
                w[4 * i + 1] = v.y - w[4 * i + 1];
                w[4 * i + 2] = v.z - w[4 * i + 2];
                w[4 * i + 3] = v.w - w[4 * i + 3];
            }
        } else {
            const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(Wv) + wrow + cb);
#pragma unroll
            for (int i = 0; i < BLK / 8; ++i) {
                uint4 v = src[i];
                const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    float2 f = __bfloat1622float2(h2[j]);
                    w[8 * i + 2 * j + 0] = f.x - w[8 * i + 2 * j + 0];
                    w[8 * i + 2 * j + 1] = f.y - w[8 * i + 2 * j + 1];
                }
            }
        }
        __syncthreads();
        // 2. grid of the group from the current values (0 always on the grid; [-1, 1] if all zero)
        float xmin = 0.f, xmax = 0.f;
#pragma unroll
        for (int c = 0; c < BLK; ++c) { xmin = fminf(xmin, w[c]); xmax = fmaxf(xmax, w[c]); }
        if (xmin == 0.f && xmax == 0.f) { xmin = -1.f; xmax = 1.f; }
        const float s = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
        const float z = rintf(__fdiv_rn(-xmin, s));
        const int g = cb / BLK;
        scales[((size_t)b * d_out + row) * ngroups + g] = s;
        zeros[((size_t)b * d_out + row) * ngroups + g] = (uint8_t)z;
        // 3. column-sequential quantization with error feedback inside the block
        uint32_t qp[BLK / 4];
#pragma unroll
        for (int i = 0; i < BLK / 4; ++i) qp[i] = 0u;
#pragma unroll
        for (int j = 0; j < BLK; ++j) {
            float q = __fadd_rn(rintf(__fdiv_rn(w[j], s)), z);
            q = fminf(fmaxf(q, 0.f), maxq);
            const float wh = __fmul_rn(s, __fsub_rn(q, z));
            const float err = (w[j] - wh) * uinv[j];
            w[j] = err;  // the register of a quantized column keeps its error
            qp[j >> 2] |= (uint32_t)q << (8 * (j & 3));
#pragma unroll
            for (int c = 0; c < BLK; ++c)
                if (c > j) w[c] = fmaf(-err, Ud[j][c], w[c]);
        }
        // 4. outputs
        float4* e4o = reinterpret_cast<float4*>(Erow + cb);
#pragma unroll
        for (int i = 0; i < BLK / 4; ++i) e4o[i] = make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
        uint4* co = reinterpret_cast<uint4*>(codes + wrow + cb);
#pragma unroll
        for (int i = 0; i < BLK / 16; ++i) co[i] = make_uint4(qp[4 * i], qp[4 * i + 1], qp[4 * i + 2], qp[4 * i + 3]);
        if (W_hat) {
            float4* wo = reinterpret_cast<float4*>(W_hat + wrow + cb);
#pragma unroll
            for (int i = 0; i < BLK / 4; ++i) {
                float v[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int c = 4 * i + j;
                    const float q = (float)((qp[c >> 2] >> (8 * (c & 3))) & 255u);
                    v[j] = __fmul_rn(s, __fsub_rn(q, z));
                }
                wo[i] = make_float4(v[0], v[1], v[2], v[3]);
            }
        }
    }
}

}  // namespace

size_t quantize_workspace_bytes(int batch, int d_out, int d_in) {
    return clha_round_up((size_t)batch * d_out * d_in * sizeof(float));
}

cudaError_t launch_quantize(cudaStream_t s, const float* U, int w_per_u, const void* W, int w_is_f32, int batch,
                            int d_out, int d_in, int bits, uint8_t* codes, float* scales, uint8_t* zeros,
                            float* W_hat, void* ws) {
    cudaError_t e = cudaFuncSetAttribute(gptq_simt, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    dim3 grid(d_out / R, batch);
    gptq_simt<<<grid, R, SMEM_BYTES, s>>>(U, w_per_u, W, w_is_f32, d_out, d_in, bits, codes, scales, zeros, W_hat,
                                           (float*)ws);
    clha_note_launches(1);
    return cudaGetLastError();
}
