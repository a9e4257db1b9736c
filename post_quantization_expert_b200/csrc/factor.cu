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
//   X = L^-1, right-looking by block rows (diagonal tiles come from potrf; X starts as I):
//     fac_inv_row   X[i][j] <- Linv_ii X[i][j]           for j < i
//     fac_inv_upd   X[r][j] -= L[r][i] X[i][j]           for r > i, j <= i
//   so X[i][j] = Linv_ii (I - sum_{m<i} L[i][m] X[m][j]), every launch one 64^3 product per CTA.
//   fac_store     U = J X J as float32 (strict lower triangle zero)
// A non-positive pivot is recorded (problem, original column) and the problem's factor is NaN.
#include "clha_internal.h"

namespace {

constexpr int NB = 64;
constexpr int LD = NB + 2;   // shared-memory row length (doubles): 16-byte aligned rows, few bank conflicts
constexpr int TILE_DOUBLES = NB * LD;
constexpr int SMEM2 = 2 * TILE_DOUBLES * sizeof(double);

typedef double Tile[LD];

__global__ void fac_load(const float* __restrict__ H, int d, double* __restrict__ A) {
    const int b = blockIdx.y;
    const size_t dd = (size_t)d * d;
    for (size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x; idx < dd; idx += (size_t)gridDim.x * blockDim.x) {
        size_t i = idx / d, j = idx % d;
        A[b * dd + idx] = (double)H[b * dd + (size_t)(d - 1 - i) * d + (d - 1 - j)];
    }
}

// All kernels below run 256 threads; a 64x64 tile is 16 elements per thread. The loads of a tile
// are issued together (unrolled) so their latencies overlap.
constexpr int PER_THREAD = NB * NB / 256;

// dst[r][c] = src[r * ld + c]      (64x64 tile, rows already indexed by k)
__device__ __forceinline__ void load_tile(Tile* dst, const double* __restrict__ src, size_t ld) {
    double v[PER_THREAD];
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int i = it * 256 + threadIdx.x;
        v[it] = src[(size_t)(i >> 6) * ld + (i & 63)];
    }
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int i = it * 256 + threadIdx.x;
        dst[i >> 6][i & 63] = v[it];
    }
}
// dst[c][r] = src[r * ld + c]      (transpose: the tile's columns become the k index)
__device__ __forceinline__ void load_tile_t(Tile* dst, const double* __restrict__ src, size_t ld) {
    double v[PER_THREAD];
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int i = it * 256 + threadIdx.x;
        v[it] = src[(size_t)(i >> 6) * ld + (i & 63)];
    }
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int i = it * 256 + threadIdx.x;
        dst[i & 63][i >> 6] = v[it];
    }
}
// acc[i][j] += sum_k As[k][4ty+i] * Bs[k][4tx+j]  (k-major operands; 16-byte shared loads)
__device__ __forceinline__ void mma_tile(const Tile* As, const Tile* Bs, double (&acc)[4][4]) {
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll 4
    for (int k = 0; k < NB; ++k) {
        const double2 a0 = *reinterpret_cast<const double2*>(&As[k][4 * ty]);
        const double2 a1 = *reinterpret_cast<const double2*>(&As[k][4 * ty + 2]);
        const double2 b0 = *reinterpret_cast<const double2*>(&Bs[k][4 * tx]);
        const double2 b1 = *reinterpret_cast<const double2*>(&Bs[k][4 * tx + 2]);
        const double a[4] = {a0.x, a0.y, a1.x, a1.y};
        const double bb[4] = {b0.x, b0.y, b1.x, b1.y};
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) acc[i][j] = fma(a[i], bb[j], acc[i][j]);
    }
}

// Cholesky of the 64x64 diagonal tile of panel k (lower), and its inverse into Dall[b][k].
// Column loop with one barrier per column: column c of L goes to a separate tile (Lt) while the
// trailing update reads the unscaled column from T, so no thread writes what another reads in the
// same step. The inverse is built from 16x16 blocks: four warps invert the diagonal blocks by forward
// substitution in registers, then three bands X[i][j] = -X[i][i] (sum_m L[i][m] X[m][j]).
constexpr int SMEM3 = 3 * TILE_DOUBLES * sizeof(double) + NB * sizeof(double);

__global__ void __launch_bounds__(256) fac_potrf(double* __restrict__ A, int d, int k, double* __restrict__ Dall,
                                                 int* err) {
    const int b = blockIdx.x;
    double* Ab = A + (size_t)b * d * d;
    extern __shared__ double dsm[];
    Tile* T = reinterpret_cast<Tile*>(dsm);
    Tile* Lt = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    Tile* X = reinterpret_cast<Tile*>(dsm + 2 * TILE_DOUBLES);
    double* dinv = dsm + 3 * TILE_DOUBLES;           // 1 / L[c][c]
    const int tid = threadIdx.x;
    const int k0 = k * NB;
    load_tile(T, Ab + (size_t)k0 * d + k0, d);
    __syncthreads();
    int bad = -1;
    for (int c = 0; c < NB; ++c) {
        const double p = T[c][c];
        const bool ok = (p > 0.0) && isfinite(p);
        const double inv = ok ? rsqrt(p) : __longlong_as_double(0x7ff8000000000000ll);
        if (!ok && bad < 0) bad = c;
        if (tid > c && tid < NB) Lt[tid][c] = T[tid][c] * inv;
        if (tid == 0) { Lt[c][c] = p * inv; dinv[c] = inv; }
        const int cc = tid & 63;
        if (cc > c) {
            const double lcc = T[cc][c] * inv;
            for (int r = c + 1 + (tid >> 6); r < NB; r += 4)
                if (r >= cc) T[r][cc] -= (T[r][c] * inv) * lcc;
        }
        __syncthreads();
    }
    if (tid == 0 && bad >= 0) clha_record_error(err, CLHA_ERR_NOT_PD, b, d - 1 - (k0 + bad), KID_FACTOR);
    // (1) diagonal 16x16 blocks: warp i, lane j < 16 solves column j of block i
    const int warp = tid >> 5, lane = tid & 31;
    if (warp < 4 && lane < 16) {
        const int o = 16 * warp, j = lane;
        double x[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            double s = (r == j) ? 1.0 : 0.0;
#pragma unroll
            for (int m = 0; m < r; ++m) s -= (m >= j) ? Lt[o + r][o + m] * x[m] : 0.0;
            x[r] = (r >= j) ? s * dinv[o + r] : 0.0;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) X[o + r][o + j] = x[r];
    }
    // zero the strict upper blocks of X
    for (int i = tid; i < NB * NB; i += 256) {
        const int r = i >> 6, c = i & 63;
        if ((c >> 4) > (r >> 4)) X[r][c] = 0.0;
    }
    __syncthreads();
    // (2) bands: T holds the partial products (T is free now)
    for (int delta = 1; delta < 4; ++delta) {
        const int nblk = 4 - delta;
        for (int e = tid; e < nblk * 256; e += 256) {       // Tp = sum_{m in blocks j..i-1} L[i][m] X[m][j]
            const int j = e >> 8, i = j + delta, r = (e >> 4) & 15, s = e & 15;
            double acc = 0.0;
            for (int m = 16 * j; m < 16 * i; ++m) acc = fma(Lt[16 * i + r][m], X[m][16 * j + s], acc);
            T[16 * i + r][16 * j + s] = acc;
        }
        __syncthreads();
        for (int e = tid; e < nblk * 256; e += 256) {       // X[i][j] = -X[i][i] Tp
            const int j = e >> 8, i = j + delta, r = (e >> 4) & 15, s = e & 15;
            double acc = 0.0;
#pragma unroll
            for (int q = 0; q < 16; ++q) acc = fma(X[16 * i + r][16 * i + q], T[16 * i + q][16 * j + s], acc);
            X[16 * i + r][16 * j + s] = -acc;
        }
        __syncthreads();
    }
    double* Db = Dall + ((size_t)b * (d / NB) + k) * NB * NB;
#pragma unroll
    for (int it = 0; it < PER_THREAD; ++it) {
        const int i = it * 256 + tid;
        const int r = i >> 6, c = i & 63;
        Ab[(size_t)(k0 + r) * d + k0 + c] = (c <= r) ? Lt[r][c] : 0.0;
        Db[i] = X[r][c];
    }
}

// Panel tiles below the diagonal: A[i][k] <- A[i][k] L_kk^-T, i.e. out[r][c] = sum_m B[r][m] Linv[c][m].
__global__ void __launch_bounds__(256) fac_trsm(double* __restrict__ A, int d, int k, const double* __restrict__ Dall) {
    const int b = blockIdx.y;
    const int ib = k + 1 + blockIdx.x;
    double* Ab = A + (size_t)b * d * d;
    const double* Db = Dall + ((size_t)b * (d / NB) + k) * NB * NB;
    extern __shared__ double dsm[];
    Tile* As = reinterpret_cast<Tile*>(dsm);
    Tile* Bs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    double* blk = Ab + (size_t)(ib * NB) * d + k * NB;
    load_tile_t(As, blk, d);          // As[m][r] = B[r][m]
    load_tile_t(Bs, Db, NB);          // Bs[m][c] = Linv[c][m]
    __syncthreads();
    double acc[4][4] = {};
    mma_tile(As, Bs, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) blk[(size_t)(ty * 4 + i) * d + tx * 4 + j] = acc[i][j];
}

// Trailing update of the lower tiles (i >= j > k): A[i][j] -= A[i][k] A[j][k]^T.
__global__ void __launch_bounds__(256) fac_update(double* __restrict__ A, int d, int k) {
    const int b = blockIdx.y;
    int t = blockIdx.x, jj = 0;
    const int m = d / NB - k - 1;  // trailing tiles per side
    while (t >= m - jj) { t -= m - jj; ++jj; }   // column jj holds m - jj tiles (rows jj..m-1)
    const int ib = k + 1 + jj + t, jb = k + 1 + jj;
    double* Ab = A + (size_t)b * d * d;
    extern __shared__ double dsm[];
    Tile* As = reinterpret_cast<Tile*>(dsm);
    Tile* Bs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    load_tile_t(As, Ab + (size_t)(ib * NB) * d + k * NB, d);   // As[q][r] = A[ib][k][r][q]
    load_tile_t(Bs, Ab + (size_t)(jb * NB) * d + k * NB, d);   // Bs[q][s] = A[jb][k][s][q]
    __syncthreads();
    double acc[4][4] = {};
    mma_tile(As, Bs, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double* out = Ab + (size_t)(ib * NB) * d + jb * NB;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) out[(size_t)(ty * 4 + i) * d + tx * 4 + j] -= acc[i][j];
}

// Copy the diagonal-tile inverses of all panels into X (they were produced panel by panel).
__global__ void fac_inv_diag(const double* __restrict__ Dall, int d, double* __restrict__ X) {
    const int b = blockIdx.y, kb = blockIdx.x;
    const double* Db = Dall + ((size_t)b * (d / NB) + kb) * NB * NB;
    double* Xb = X + (size_t)b * d * d;
    for (int i = threadIdx.x; i < NB * NB; i += blockDim.x) {
        const int r = i >> 6, c = i & 63;
        Xb[(size_t)(kb * NB + r) * d + kb * NB + c] = Db[i];
    }
}

// X[i][j] <- Linv_ii X[i][j] for the j < i tiles of block row i (in place).
__global__ void __launch_bounds__(256) fac_inv_row(const double* __restrict__ Dall, int d, int i,
                                                   double* __restrict__ X) {
    const int b = blockIdx.y, jb = blockIdx.x;
    double* Xt = X + (size_t)b * d * d + (size_t)(i * NB) * d + jb * NB;
    extern __shared__ double dsm[];
    Tile* As = reinterpret_cast<Tile*>(dsm);
    Tile* Bs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    load_tile_t(As, Dall + ((size_t)b * (d / NB) + i) * NB * NB, NB);   // As[q][r] = Linv_ii[r][q]
    load_tile(Bs, Xt, d);                                              // Bs[q][s] = X[i][jb][q][s]
    __syncthreads();
    double acc[4][4] = {};
    mma_tile(As, Bs, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) Xt[(size_t)(ty * 4 + a) * d + tx * 4 + c] = acc[a][c];
}

// X[r][j] -= L[r][i] X[i][j] for r > i, j <= i.
__global__ void __launch_bounds__(256) fac_inv_upd(const double* __restrict__ L, int d, int i,
                                                   double* __restrict__ X) {
    const int b = blockIdx.y;
    const int rb = i + 1 + blockIdx.x / (i + 1), jb = blockIdx.x % (i + 1);
    const double* Lb = L + (size_t)b * d * d;
    double* Xb = X + (size_t)b * d * d;
    extern __shared__ double dsm[];
    Tile* As = reinterpret_cast<Tile*>(dsm);
    Tile* Bs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    load_tile_t(As, Lb + (size_t)(rb * NB) * d + i * NB, d);     // As[q][r] = L[rb][i][r][q]
    load_tile(Bs, Xb + (size_t)(i * NB) * d + jb * NB, d);       // Bs[q][s] = X[i][jb][q][s]
    __syncthreads();
    double acc[4][4] = {};
    mma_tile(As, Bs, acc);
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double* out = Xb + (size_t)(rb * NB) * d + jb * NB;
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
        for (int c = 0; c < 4; ++c) out[(size_t)(ty * 4 + a) * d + tx * 4 + c] -= acc[a][c];
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
    const int smem = SMEM2;
    cudaError_t e;
    if ((e = cudaFuncSetAttribute(fac_potrf, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM3)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(fac_trsm, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fac_update, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess) return e;
    if ((e = cudaFuncSetAttribute(fac_inv_row, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(fac_inv_upd, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
        return e;
    unsigned eg = (unsigned)((dd + 255) / 256);
    if (eg > 148 * 64) eg = 148 * 64;
    fac_load<<<dim3(eg, batch), 256, 0, s>>>(H_d, d, A);
    clha_note_launches(1);
    e = cudaMemsetAsync(X, 0, (size_t)batch * dd * sizeof(double), s);
    if (e != cudaSuccess) return e;
    for (int k = 0; k < nbk; ++k) {
        fac_potrf<<<batch, 256, SMEM3, s>>>(A, d, k, Dall, err);
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
    for (int i = 0; i < nbk; ++i) {
        if (i > 0) {
            fac_inv_row<<<dim3(i, batch), 256, smem, s>>>(Dall, d, i, X);
            clha_note_launches(1);
        }
        if (i + 1 < nbk) {
            fac_inv_upd<<<dim3((nbk - 1 - i) * (i + 1), batch), 256, smem, s>>>(A, d, i, X);
            clha_note_launches(1);
        }
    }
    fac_store<<<dim3(eg, batch), 256, 0, s>>>(X, d, U);
    clha_note_launches(1);
    return cudaGetLastError();
}
