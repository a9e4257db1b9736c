// One term of the shared-weight loss of the CLHA page (§2.1): tr[(W_hat - W) H (W_hat - W)^T],
// batched. A 64x64 tile of Y = D H (D = W_hat - W) is formed with shared-memory FMA and reduced
// against the same tile of D; tile sums are added in float64.
#include "clha_internal.h"

namespace {

constexpr int T = 64, KC = 32;

__device__ __forceinline__ float w_at(const void* W, int f32, size_t i) {
    return f32 ? reinterpret_cast<const float*>(W)[i] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[i]);
}

__global__ void __launch_bounds__(256) loss_simt(const void* __restrict__ W, int f32, const float* __restrict__ W_hat,
                                                 const float* __restrict__ H, int n_h, int d_out, int d_in,
                                                 double* __restrict__ out) {
    const int b = blockIdx.z;
    const int r0 = blockIdx.y * T, c0 = blockIdx.x * T;
    const size_t base = (size_t)b * d_out * d_in;
    const float* Hb = H + (size_t)(b % n_h) * d_in * d_in;
    __shared__ float Ds[KC][T + 4];
    __shared__ float Hs[KC][T + 4];
    __shared__ double red[256];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d_in; k0 += KC) {
        for (int i = threadIdx.x; i < T * KC; i += 256) {
            int m = i / KC, kk = i % KC;
            size_t idx = base + (size_t)(r0 + m) * d_in + k0 + kk;
            Ds[kk][m] = W_hat[idx] - w_at(W, f32, idx);
            int kr = i / T, n = i % T;
            Hs[kr][n] = Hb[(size_t)(k0 + kr) * d_in + c0 + n];
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < KC; ++kk) {
            float a[4], h[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = Ds[kk][ty * 4 + i]; h[i] = Hs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], h[j], acc[i][j]);
        }
        __syncthreads();
    }
    double part = 0.0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            size_t idx = base + (size_t)(r0 + ty * 4 + i) * d_in + c0 + tx * 4 + j;
            part += (double)acc[i][j] * (double)(W_hat[idx] - w_at(W, f32, idx));
        }
    red[threadIdx.x] = part;
    __syncthreads();
    for (int off = 128; off > 0; off >>= 1) {
        if (threadIdx.x < off) red[threadIdx.x] += red[threadIdx.x + off];
        __syncthreads();
    }
    if (threadIdx.x == 0) atomicAdd(&out[b], red[0]);
}

}  // namespace

cudaError_t launch_loss(cudaStream_t s, const void* W, int w_is_f32, const float* W_hat, const float* H, int n_h,
                        int batch, int d_out, int d_in, double* d_loss) {
    dim3 grid(d_in / T, d_out / T, batch);
    loss_simt<<<grid, 256, 0, s>>>(W, w_is_f32, W_hat, H, n_h, d_out, d_in, d_loss);
    clha_note_launches(1);
    return cudaGetLastError();
}
