// Routed-token gather: a stable counting sort of (token, slot) pairs by expert, then a row copy into
// per-expert segments aligned to 128 rows (zero rows between segments). The Hessian and FFN kernels
// read whole 128-row tiles from these segments, so a tile never mixes experts and the zero padding
// adds nothing to a Gram matrix.
//
// Passes (all HBM- or latency-bound):
//   1. per block of 256 tokens, a histogram of expert ids                       (hist)
//   2. one block: per expert, exclusive scan of the block histograms; segment
//      starts = exclusive scan of counts rounded up to 128                       (scan)
//   3. per block: each (token, slot) finds its rank among earlier tokens of the
//      block routed to the same expert and writes its token index to perm       (scatter)
//   4. one warp per packed row: 16-byte vector copy of the token's row, or zeros (copy)
#include "clha_internal.h"

namespace {

constexpr int kTB = kGatherBlockTokens;  // tokens per block in passes 1 and 3

__global__ void gather_hist(const int32_t* __restrict__ ids, int64_t n, int k, int E, int* __restrict__ H,
                            int* err) {
    extern __shared__ int hist[];
    for (int e = threadIdx.x; e < E; e += blockDim.x) hist[e] = 0;
    __syncthreads();
    int64_t t = (int64_t)blockIdx.x * kTB + threadIdx.x;
    if (t < n) {
        for (int j = 0; j < k; ++j) {
            int e = ids[t * k + j];
            if (e < 0 || e >= E) {
                clha_record_error(err, CLHA_ERR_INVALID_ARG, (int)(t & 0x7fffffff), e, KID_GATHER);
                continue;
            }
            atomicAdd(&hist[e], 1);
        }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < E; e += blockDim.x) H[(size_t)blockIdx.x * E + e] = hist[e];
}

__global__ void __launch_bounds__(1024) gather_scan(int* __restrict__ H, int nblk, int E, int64_t* __restrict__ seg) {
    __shared__ int64_t sc[1024];
    const int e = threadIdx.x;
    int64_t cnt = 0;
    if (e < E) {
        for (int b = 0; b < nblk; ++b) {
            int v = H[(size_t)b * E + e];
            H[(size_t)b * E + e] = (int)cnt;
            cnt += v;
        }
    }
    int64_t padded = (e < E) ? ((cnt + 127) / 128) * 128 : 0;
    sc[e] = padded;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {  // inclusive Hillis-Steele scan
        int64_t v = (e >= off) ? sc[e - off] : 0;
        __syncthreads();
        sc[e] += v;
        __syncthreads();
    }
    int64_t start = sc[e] - padded;
    if (e < E) {
        seg[e] = start;
        seg[E + 1 + e] = cnt;
        for (int b = 0; b < nblk; ++b) H[(size_t)b * E + e] += (int)start;
    }
    if (e == E - 1) seg[E] = sc[e];
}

__global__ void __launch_bounds__(kTB) gather_scatter(const int32_t* __restrict__ ids, int64_t n, int k, int E,
                                                      const int* __restrict__ H, int32_t* __restrict__ perm) {
    extern __shared__ int sids[];  // [kTB * k]
    const int64_t t0 = (int64_t)blockIdx.x * kTB;
    const int nt = (n - t0 < kTB) ? (int)(n - t0) : kTB;
    for (int i = threadIdx.x; i < nt * k; i += blockDim.x) sids[i] = ids[t0 * k + i];
    __syncthreads();
    const int i = threadIdx.x;
    if (i >= nt) return;
    for (int j = 0; j < k; ++j) {
        int e = sids[i * k + j];
        if (e < 0 || e >= E) continue;
        int rank = 0;
        for (int q = 0; q < i * k; ++q) rank += (sids[q] == e);
        int64_t pos = (int64_t)H[(size_t)blockIdx.x * E + e] + rank;
        perm[pos] = (int32_t)(t0 + i);
    }
}

__global__ void gather_copy(const uint4* __restrict__ X, int64_t row_vecs, const int32_t* __restrict__ perm,
                            const int64_t* __restrict__ seg, int E, int64_t packed_rows, uint4* __restrict__ Xp) {
    const int lane = threadIdx.x & 31;
    const int64_t total = seg[E];
    const int64_t warps = (int64_t)gridDim.x * (blockDim.x >> 5);
    for (int64_t p = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); p < total && p < packed_rows;
         p += warps) {
        int32_t tok = perm[p];
        uint4* dst = Xp + p * row_vecs;
        if (tok >= 0) {
            const uint4* src = X + (int64_t)tok * row_vecs;
            for (int64_t v = lane; v < row_vecs; v += 32) dst[v] = __ldg(src + v);
        } else {
            for (int64_t v = lane; v < row_vecs; v += 32) dst[v] = make_uint4(0, 0, 0, 0);
        }
    }
}

}  // namespace

size_t gather_workspace_bytes(int64_t n, int k, int E, int64_t packed_rows) {
    int64_t nblk = (n + kTB - 1) / kTB;
    if (nblk < 1) nblk = 1;
    return clha_round_up((size_t)nblk * E * sizeof(int)) + clha_round_up((size_t)packed_rows * sizeof(int32_t));
}

cudaError_t launch_gather(cudaStream_t s, const void* X, int esize, int64_t n, int d, const int32_t* ids, int k,
                          int E, void* X_packed, int64_t packed_rows, int64_t* seg, int32_t* perm, void* ws,
                          size_t ws_bytes, int* err) {
    (void)ws_bytes;
    int64_t nblk = (n + kTB - 1) / kTB;
    char* cur = (char*)ws;
    int* H = (int*)clha_carve(cur, (size_t)(nblk < 1 ? 1 : nblk) * E * sizeof(int));
    int32_t* pm = perm ? perm : (int32_t*)clha_carve(cur, (size_t)packed_rows * sizeof(int32_t));
    cudaError_t e = cudaMemsetAsync(pm, 0xff, (size_t)packed_rows * sizeof(int32_t), s);
    if (e != cudaSuccess) return e;
    if (n == 0) {
        e = cudaMemsetAsync(seg, 0, (size_t)(2 * E + 1) * sizeof(int64_t), s);
        return e;
    }
    gather_hist<<<(unsigned)nblk, kTB, E * sizeof(int), s>>>(ids, n, k, E, H, err);
    clha_note_launches(1);
    gather_scan<<<1, 1024, 0, s>>>(H, (int)nblk, E, seg);
    clha_note_launches(1);
    gather_scatter<<<(unsigned)nblk, kTB, kTB * k * sizeof(int), s>>>(ids, n, k, E, H, pm);
    clha_note_launches(1);
    if (!X_packed) return cudaGetLastError();   // the permutation alone: the rows are read where they are
    int64_t row_vecs = (int64_t)d * esize / 16;
    int64_t warps = packed_rows;
    int64_t blocks = (warps + 7) / 8;
    if (blocks > 148 * 32) blocks = 148 * 32;
    gather_copy<<<(unsigned)blocks, 256, 0, s>>>((const uint4*)X, row_vecs, pm, seg, E, packed_rows, (uint4*)X_packed);
    clha_note_launches(1);
    return cudaGetLastError();
}
