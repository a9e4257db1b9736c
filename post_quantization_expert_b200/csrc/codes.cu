// Deployable codes: GPTQ's b-bit codes packed per row as one little-endian bit stream of 32-bit
// words (code j at bits [b*j, b*j + b), so a code may straddle two words), their dequantization
// W_hat = s (q - z) per 128-column group, and the deployable layer Y = X W_hat^T with the weights
// decoded from the packed words inside the product.
#include "clha_internal.h"

namespace {

constexpr int GROUP = 128;

// One output word per thread: the codes whose bits fall into word w of row r.
__global__ void __launch_bounds__(256) pack_codes_kernel(const uint8_t* __restrict__ codes, int64_t rows, int d_in,
                                                         int bits, uint32_t* __restrict__ packed) {
    const int64_t W = (int64_t)d_in * bits / 32;
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * W) return;
    const int64_t r = gid / W, w = gid % W;
    const int64_t b0 = 32 * w;
    const uint8_t* row = codes + r * d_in;
    uint32_t word = 0;
    for (int64_t j = b0 / bits; j <= (b0 + 31) / bits && j < d_in; ++j) {
        const int64_t off = (int64_t)bits * j - b0;
        const uint32_t c = row[j];
        word |= off >= 0 ? (c << off) : (c >> (-off));
    }
    packed[gid] = word;
}

// Code j of a packed row.
__device__ __forceinline__ uint32_t code_at(const uint32_t* __restrict__ row, int j, int bits) {
    const int bit = bits * j, w = bit >> 5, off = bit & 31;
    uint32_t v = row[w] >> off;
    if (off + bits > 32) v |= row[w + 1] << (32 - off);
    return v & ((1u << bits) - 1u);
}

// The same float32 operations clha_quantize forms W_hat with.
__device__ __forceinline__ float dequant(uint32_t q, float s, float z) { return __fmul_rn(s, __fsub_rn((float)q, z)); }

__global__ void __launch_bounds__(256) dequantize_kernel(const uint32_t* __restrict__ packed, const float* __restrict__ scales,
                                                         const uint8_t* __restrict__ zeros, int64_t rows, int d_in,
                                                         int bits, float* __restrict__ W_hat) {
    const int64_t gid = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (gid >= rows * d_in) return;
    const int64_t r = gid / d_in;
    const int j = (int)(gid % d_in);
    const int64_t W = (int64_t)d_in * bits / 32;
    const int64_t g = r * (d_in / GROUP) + j / GROUP;
    W_hat[gid] = dequant(code_at(packed + r * W, j, bits), scales[g], (float)zeros[g]);
}

// Y [n, d_out] = X [n, d_in] W_hat^T: 64 x 64 output tiles, 32-wide k steps, 4 x 4 outputs per thread
// in fp32 FMA; the weight tile is decoded from the packed words as it is staged.
constexpr int TM = 64, TN = 64, TK = 32;

__global__ void __launch_bounds__(256) dequant_matmul_kernel(const void* __restrict__ X, int x_bf16, int64_t n, int d_in,
                                                             const uint32_t* __restrict__ packed,
                                                             const float* __restrict__ scales,
                                                             const uint8_t* __restrict__ zeros, int d_out, int bits,
                                                             float* __restrict__ Y) {
    __shared__ float As[TK][TM + 4];
    __shared__ float Bs[TK][TN + 4];
    const int64_t m0 = (int64_t)blockIdx.x * TM;
    const int o0 = blockIdx.y * TN;
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int64_t W = (int64_t)d_in * bits / 32;
    const int ng = d_in / GROUP;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < d_in; k0 += TK) {
        for (int i = threadIdx.x; i < TM * TK; i += 256) {
            const int m = i / TK, kk = i % TK;
            const int64_t row = m0 + m;
            float xv = 0.f;
            if (row < n) {
                const int64_t o = row * d_in + k0 + kk;
                xv = x_bf16 ? __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(X)[o])
                            : reinterpret_cast<const float*>(X)[o];
            }
            As[kk][m] = xv;
            const int oc = o0 + m, j = k0 + kk;
            const int64_t g = (int64_t)oc * ng + j / GROUP;
            Bs[kk][m] = dequant(code_at(packed + (int64_t)oc * W, j, bits), scales[g], (float)zeros[g]);
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                a[i] = As[kk][ty * 4 + i];
                b[i] = Bs[kk][tx * 4 + i];
            }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        const int64_t row = m0 + ty * 4 + i;
        if (row >= n) continue;
#pragma unroll
        for (int j = 0; j < 4; ++j) Y[row * d_out + o0 + tx * 4 + j] = acc[i][j];
    }
}

}  // namespace

cudaError_t launch_pack_codes(cudaStream_t s, const uint8_t* codes, int64_t rows, int d_in, int bits,
                              uint32_t* packed) {
    const int64_t words = rows * ((int64_t)d_in * bits / 32);
    if (words == 0) return cudaSuccess;
    pack_codes_kernel<<<(unsigned)((words + 255) / 256), 256, 0, s>>>(codes, rows, d_in, bits, packed);
    clha_note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_dequantize(cudaStream_t s, const uint32_t* packed, const float* scales, const uint8_t* zeros,
                              int64_t rows, int d_in, int bits, float* W_hat) {
    const int64_t elems = rows * d_in;
    if (elems == 0) return cudaSuccess;
    dequantize_kernel<<<(unsigned)((elems + 255) / 256), 256, 0, s>>>(packed, scales, zeros, rows, d_in, bits, W_hat);
    clha_note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_dequant_matmul(cudaStream_t s, const void* X, int x_bf16, int64_t n, int d_in,
                                  const uint32_t* packed, const float* scales, const uint8_t* zeros, int d_out, int bits,
                                  float* Y) {
    if (n == 0) return cudaSuccess;
    dim3 grid((unsigned)((n + TM - 1) / TM), d_out / TN);
    dequant_matmul_kernel<<<grid, 256, 0, s>>>(X, x_bf16, n, d_in, packed, scales, zeros, d_out, bits, Y);
    clha_note_launches(1);
    return cudaGetLastError();
}
