// GPTQ's factor of the damped Hessian: U upper triangular with H_d^-1 = U^T U.
//
// With J the index reversal, let L be the lower Cholesky factor of J H_d J. Then R = J L J is upper
// with H_d = R R^T, and U = R^-1 = J L^-1 J is upper with U^T U = (R R^T)^-1 = H_d^-1; its diagonal
// is positive, so it is THE upper Cholesky factor of H_d^-1. This needs one Cholesky and one
// triangular inverse (no explicit inverse of H_d, no second factorisation).
//
// Float64 throughout, blocked with 64 x 64 tiles, batched over problems (grid.z / grid.y = problem):
//   fac_load      A = J H_d J in float64
//   per panel k:  fac_potrf   Cholesky of the diagonal tile in shared memory, plus its inverse
//                 fac_trsm    panel tiles A[i][k] <- A[i][k] L_kk^-T   (a GEMM with the inverse)
//                 fac_update  trailing lower tiles A[i][j] -= A[i][k] A[j][k]^T
//   fac_inv_band  X = L^-1, one band of block diagonals at a time:
//                 X[i][j] = -X[i][i] sum_{m=j}^{i-1} L[i][m] X[m][j]  (diagonal tiles come from potrf)
//   fac_store     U = J X J as float32 (strict lower triangle zero)
// A non-positive pivot is recorded (problem, original column) and the problem's factor is NaN.
#include "clha_internal.h"

namespace {

constexpr int NB = 64;

__global__ void fac_load(const float* __restrict__ H, int d, double* __restrict__ A) {
    const int b = blockIdx.y;
    const size_t dd = (size_t)d * d;
    for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < dd; idx += (size_t)gridDim.x * blockDim.x) {
        size_t i = idx / d, j = idx % d;
        A[b * dd + idx] = (double)H[b * dd + (size_t)(d - 1 - i) * d + (d - 1 - j)];
    }
}

// Cholesky of the 64x64 diagonal tile of panel k (lower), and its inverse into Dall[b][k].
__global__ void __launch_bounds__(256) fac_potrf(double* __restrict__ A, int d, int k, double* __restrict__ Dall,
                                                 int* err) {
    const int b = blockIdx.x;
    double* Ab = A + (size_t)b * d * d;
    extern __shared__ double dsm[];
    double (*T)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm);
    double (*X)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm + NB * (NB + 1));
    __shared__ int bad;
    const int k0 = k * NB;
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        T[r][c] = Ab[(size_t)(k0 + r) * d + k0 + c];
    }
    if (threadIdx.x == 0) bad = -1;
    __syncthreads();
    for (int c = 0; c < NB; ++c) {
        if (threadIdx.x == 0) {
            double p = T[c][c];
            if (!(p > 0.0) || !isfinite(p)) {
                if (bad < 0) bad = c;
                p = __longlong_as_double(0x7ff8000000000000ll);  // NaN propagates to the factor
            } else {
                p = sqrt(p);
            }
            T[c][c] = p;
        }
        __syncthreads();
        const double piv = T[c][c];
        for (int r = c + 1 + threadIdx.x; r < NB; r += blockDim.x) T[r][c] /= piv;
        __syncthreads();
        // trailing update of the tile (lower part)
        for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
            int r = i / NB, cc = i % NB;
            if (cc > c && r >= cc) T[r][cc] -= T[r][c] * T[cc][c];
        }
        __syncthreads();
    }
    if (threadIdx.x == 0 && bad >= 0)
        clha_record_error(err, CLHA_ERR_NOT_PD, b, d - 1 - (k0 + bad), KID_FACTOR);
    // inverse of the lower tile: column c of X solves T x = e_c (forward substitution)
    if (threadIdx.x < NB) {
        const int c = threadIdx.x;
        for (int r = 0; r < NB; ++r) {
            if (r < c) { X[r][c] = 0.0; continue; }
            double s = (r == c) ? 1.0 : 0.0;
            for (int m = c; m < r; ++m) s -= T[r][m] * X[m][c];
            X[r][c] = s / T[r][r];
        }
    }
    __syncthreads();
    double* Db = Dall + ((size_t)b * (d / NB) + k) * NB * NB;
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        Ab[(size_t)(k0 + r) * d + k0 + c] = (c <= r) ? T[r][c] : 0.0;
        Db[i] = X[r][c];
    }
}

// Panel tiles below the diagonal: A[i][k] <- A[i][k] * L_kk^-T, i.e. X[r][c] = sum_m B[r][m] Linv[c][m].
__global__ void __launch_bounds__(256) fac_trsm(double* __restrict__ A, int d, int k, const double* __restrict__ Dall) {
    const int b = blockIdx.y;
    const int ib = k + 1 + blockIdx.x;
    double* Ab = A + (size_t)b * d * d;
    const double* Db = Dall + ((size_t)b * (d / NB) + k) * NB * NB;
    extern __shared__ double dsm[];
    double (*Bs)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm);
    double (*Li)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm + NB * (NB + 1));
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        Bs[r][c] = Ab[(size_t)(ib * NB + r) * d + k * NB + c];
        Li[r][c] = Db[i];
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int m = 0; m < NB; ++m) {
        double a[4], l[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[i] = Bs[ty * 4 + i][m]; l[i] = Li[tx * 4 + i][m]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], l[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Ab[(size_t)(ib * NB + ty * 4 + i) * d + k * NB + tx * 4 + j] = acc[i][j];
}

// Trailing update of the lower tiles (i >= j > k): A[i][j] -= A[i][k] A[j][k]^T.
__global__ void __launch_bounds__(256) fac_update(double* __restrict__ A, int d, int k) {
    const int b = blockIdx.y;
    int t = blockIdx.x, jj = 0;
    const int m = d / NB - k - 1;  // trailing tiles per side
    // enumerate lower tiles column by column: column jj has m - jj tiles (rows jj..m-1)
    while (t >= m - jj) { t -= m - jj; ++jj; }
    const int ib = k + 1 + jj + t, jb = k + 1 + jj;
    double* Ab = A + (size_t)b * d * d;
    extern __shared__ double dsm[];
    double (*P)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm);
    double (*Q)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm + NB * (NB + 1));
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        P[r][c] = Ab[(size_t)(ib * NB + r) * d + k * NB + c];
        Q[r][c] = Ab[(size_t)(jb * NB + r) * d + k * NB + c];
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int q = 0; q < NB; ++q) {
        double a[4], c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[i] = P[ty * 4 + i][q]; c[i] = Q[tx * 4 + i][q]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], c[j], acc[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Ab[(size_t)(ib * NB + ty * 4 + i) * d + jb * NB + tx * 4 + j] -= acc[i][j];
}

// Copy the diagonal-tile inverses of all panels into X (they were produced panel by panel).
__global__ void fac_inv_diag(const double* __restrict__ Dall, int d, double* __restrict__ X) {
    const int b = blockIdx.y, kb = blockIdx.x;
    const double* Db = Dall + ((size_t)b * (d / NB) + kb) * NB * NB;
    double* Xb = X + (size_t)b * d * d;
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        Xb[(size_t)(kb * NB + r) * d + kb * NB + c] = Db[i];
    }
}

// Band delta of X = L^-1: tiles (ib, jb = ib - delta).
__global__ void __launch_bounds__(256) fac_inv_band(const double* __restrict__ L, int d, int delta,
                                                    double* __restrict__ X) {
    const int b = blockIdx.y;
    const int jb = blockIdx.x, ib = jb + delta;
    const double* Lb = L + (size_t)b * d * d;
    double* Xb = X + (size_t)b * d * d;
    extern __shared__ double dsm[];
    double (*P)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm);
    double (*Q)[NB + 1] = reinterpret_cast<double (*)[NB + 1]>(dsm + NB * (NB + 1));
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int mb = jb; mb < ib; ++mb) {  // T = sum L[ib][mb] X[mb][jb]
        __syncthreads();
        for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
            int r = i / NB, c = i % NB;
            P[r][c] = Lb[(size_t)(ib * NB + r) * d + mb * NB + c];
            Q[r][c] = Xb[(size_t)(mb * NB + r) * d + jb * NB + c];
        }
        __syncthreads();
        for (int q = 0; q < NB; ++q) {
            double a[4], c[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = P[ty * 4 + i][q]; c[i] = Q[q][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], c[j], acc[i][j]);
        }
    }
    // X[ib][jb] = -X[ib][ib] * T
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Q[ty * 4 + i][tx * 4 + j] = acc[i][j];
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        int r = i / NB, c = i % NB;
        P[r][c] = Xb[(size_t)(ib * NB + r) * d + ib * NB + c];
    }
    __syncthreads();
    double out[4][4] = {};
    for (int q = 0; q < NB; ++q) {
        double a[4], c[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) { a[i] = P[ty * 4 + i][q]; c[i] = Q[q][tx * 4 + i]; }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) out[i][j] = fma(a[i], c[j], out[i][j]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Xb[(size_t)(ib * NB + ty * 4 + i) * d + jb * NB + tx * 4 + j] = -out[i][j];
}

__global__ void fac_store(const double* __restrict__ X, int d, float* __restrict__ U) {
    const int b = blockIdx.y;
    const size_t dd = (size_t)d * d;
    for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < dd; idx += (size_t)gridDim.x * blockDim.x) {
        size_t i = idx / d, j = idx % d;
        U[b * dd + idx] = (j >= i) ? (float)X[b * dd + (size_t)(d - 1 - i) * d + (d - 1 - j)] : 0.f;
    }
}

}  // namespace

size_t factor_workspace_bytes(int batch, int d) {
    size_t dd = (size_t)d * d;
    return clha_round_up((size_t)batch * dd * sizeof(double)) * 2 +
           clha_round_up((size_t)batch * (d / NB) * NB * NB * sizeof(double));
}

cudaError_t launch_factor(cudaStream_t s, const float* H_d, int batch, int d, float* U, void* ws, int* err) {
    size_t dd = (size_t)d * d;
    char* cur = (char*)ws;
    double* A = (double*)clha_carve(cur, (size_t)batch * dd * sizeof(double));
    double* X = (double*)clha_carve(cur, (size_t)batch * dd * sizeof(double));
    double* Dall = (double*)clha_carve(cur, (size_t)batch * (d / NB) * NB * NB * sizeof(double));
    const int nbk = d / NB;
    const int smem = 2 * NB * (NB + 1) * sizeof(double);
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(fac_potrf, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fac_trsm, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fac_update, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fac_inv_band, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    unsigned eg = (unsigned)((dd + 255) / 256);
    if (eg > 148 * 64) eg = 148 * 64;
    fac_load<<<dim3(eg, batch), 256, 0, s>>>(H_d, d, A);
    clha_note_launches(1);
    e = cudaMemsetAsync(X, 0, (size_t)batch * dd * sizeof(double), s);
    if (e != cudaSuccess) return e;
    for (int k = 0; k < nbk; ++k) {
        fac_potrf<<<batch, 256, smem, s>>>(A, d, k, Dall, err);
        clha_note_launches(1);
        const int rem = nbk - k - 1;
        if (rem > 0) {
            fac_trsm<<<dim3(rem, batch), 256, smem, s>>>(A, d, k, Dall);
            clha_note_launches(1);
            fac_update<<<dim3(rem * (rem + 1) / 2, batch), 256, smem, s>>>(A, d, k);
            clha_note_launches(1);
        }
    }
    fac_inv_diag<<<dim3(nbk, batch), 256, 0, s>>>(Dall, d, X);
    clha_note_launches(1);
    for (int delta = 1; delta < nbk; ++delta) {
        fac_inv_band<<<dim3(nbk - delta, batch), 256, smem, s>>>(A, d, delta, X);
        clha_note_launches(1);
    }
    fac_store<<<dim3(eg, batch), 256, 0, s>>>(X, d, U);
    clha_note_launches(1);
    return cudaGetLastError();
}
