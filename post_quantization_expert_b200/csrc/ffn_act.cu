// Expert FFN activation on the fp32 FMA pipes (and the choice between it and the tensor-core kernel
// of ffn_act_tc.cu): h = SiLU(x Wg^T) * (x Wu^T) for every row of every expert segment: the input
// of the expert's down projection, whose Hessian phase 1 collects. fp32 accumulation, bf16 output
// (round to nearest even). Padding rows of a segment are written as zero, so h has exactly the
// segment layout of its input and can be collected the same way. The rows are read either from a
// packed copy (row q of the segment layout) or straight from the token matrix through the gather's
// permutation (row q is token perm[q]), so the routed rows need not be copied.
//
// Shared-memory tiled FMA kernel: a 64-row x 64-column output tile computes the gate and the up
// tile together (two accumulators per thread), so the SiLU-times-up epilogue needs no second pass.
// Products of bf16 values are exact in fp32; each 32-term chunk is summed in fp32 and the chunk sums
// in fp64, which keeps the rounding of h to bf16 at the correctly rounded value far more often than
// one long fp32 sum would (inputs with outlier channels cancel heavily); the SiLU product is
// evaluated in fp64 and rounded once to bf16.
// Data movement: 16-byte cp.async copies of the bf16 tiles into a double-buffered staging area
// (rows past the segment's end are zero-filled), one conversion pass per 32-wide k-tile into
// double-buffered fp32 tiles laid out k-major for the inner loop, one barrier per k-tile; the copy
// of tile t+2 and the conversion of tile t+1 overlap the FMAs of tile t. The copy gives each row to
// four lanes (coalesced); the conversion gives a warp 32 rows, so its transposing stores and its
// reads of the padded staging rows are free of bank conflicts.
#include "clha_internal.h"

namespace {

constexpr int TM = 64, TN = 64, TK = 32;
constexpr int FLD = TM + 4;   // fp32 tile row (k-major): 16-byte aligned float4 reads

__device__ __forceinline__ int find_segment(const int64_t* seg, int E, int64_t row) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // last e with seg[e] <= row
        int mid = (lo + hi + 1) >> 1;
        if (seg[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

__device__ __forceinline__ void cp_async16_zfill(void* smem_dst, const void* gsrc, bool valid) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    const int n = valid ? 16 : 0;   // 0 source bytes: the 16 destination bytes are zero-filled
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(d), "l"(gsrc), "r"(n) : "memory");
}

constexpr int SLD = TK + 8;   // bf16 staging row: 80 B, so 8 rows' 16-byte chunks hit distinct banks
struct ActSmem {
    __nv_bfloat16 stage[2][3][TM][SLD];   // bf16 copies: X, Wg, Wu tiles (row-major)
    float f[2][3][TK][FLD];               // fp32, k-major
};

__global__ void __launch_bounds__(256, 2) expert_act_simt(const int* __restrict__ sel,
                                                          const __nv_bfloat16* __restrict__ X, int64_t rows, int dm,
                                                          const int32_t* __restrict__ perm,
                                                          const int64_t* __restrict__ seg, int E,
                                                          const __nv_bfloat16* __restrict__ Wg,
                                                          const __nv_bfloat16* __restrict__ Wu, int dff,
                                                          __nv_bfloat16* __restrict__ h) {
    if (sel && *sel != 0) return;   // the tensor-core kernel takes this call
    extern __shared__ __align__(16) uint8_t act_smem[];
    ActSmem& sm = *reinterpret_cast<ActSmem*>(act_smem);
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
    const int tid = threadIdx.x;
    const int lr = tid >> 2, lk = (tid & 3) * 8;       // this thread copies row lr, k lk..lk+7 (coalesced)
    const int cr = tid & 63, ck = (tid >> 6) * 8;      // and converts row cr, k ck..ck+7 (a warp: 32 rows)
    // packed row m0 + lr: row m0 + lr of X, or with perm the token perm[m0 + lr] (-1: padding, zeros)
    int64_t xrow = m0 + lr;
    bool row_ok = xrow < valid_end;
    if (perm && row_ok) {
        xrow = perm[xrow];
        row_ok = xrow >= 0;
    }
    const __nv_bfloat16* xsrc = X + (row_ok ? xrow * dm : 0) + lk;
    const __nv_bfloat16* gsrc = wg + (size_t)(n0 + lr) * dm + lk;
    const __nv_bfloat16* usrc = wu + (size_t)(n0 + lr) * dm + lk;
    const int nkt = dm / TK;

    auto issue = [&](int kt) {
        const int st = kt & 1, k0 = kt * TK;
        cp_async16_zfill(&sm.stage[st][0][lr][lk], xsrc + k0, row_ok);
        cp_async16_zfill(&sm.stage[st][1][lr][lk], gsrc + k0, true);
        cp_async16_zfill(&sm.stage[st][2][lr][lk], usrc + k0, true);
        asm volatile("cp.async.commit_group;" ::: "memory");
    };
    auto convert = [&](int kt) {
        const int st = kt & 1;
#pragma unroll
        for (int a = 0; a < 3; ++a) {
            const uint4 v = *reinterpret_cast<const uint4*>(&sm.stage[st][a][cr][ck]);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                sm.f[st][a][ck + 2 * q][cr] = __uint_as_float(w[q] << 16);
                sm.f[st][a][ck + 2 * q + 1][cr] = __uint_as_float(w[q] & 0xffff0000u);
            }
        }
    };

    const int tx = tid & 15, ty = tid >> 4;
    double ag[4][4] = {}, au[4][4] = {};
    issue(0);
    if (nkt > 1) issue(1);
    if (nkt > 1) asm volatile("cp.async.wait_group 1;" ::: "memory");
    else asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncthreads();
    convert(0);
    for (int kt = 0; kt < nkt; ++kt) {
        // tile kt+1 has landed (its copy was issued two steps ago); everyone is done with step kt-1
        if (kt + 1 < nkt) asm volatile("cp.async.wait_group 0;" ::: "memory");
        __syncthreads();
        if (kt + 1 < nkt) convert(kt + 1);
        if (kt + 2 < nkt) issue(kt + 2);
        const int st = kt & 1;
        float pg[4][4] = {}, pu[4][4] = {};
#pragma unroll 8
        for (int kk = 0; kk < TK; ++kk) {
            const float4 a4 = *reinterpret_cast<const float4*>(&sm.f[st][0][kk][ty * 4]);
            const float4 g4 = *reinterpret_cast<const float4*>(&sm.f[st][1][kk][tx * 4]);
            const float4 u4 = *reinterpret_cast<const float4*>(&sm.f[st][2][kk][tx * 4]);
            const float a[4] = {a4.x, a4.y, a4.z, a4.w}, g[4] = {g4.x, g4.y, g4.z, g4.w},
                        u[4] = {u4.x, u4.y, u4.z, u4.w};
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

// Per-channel max |x| over the rows (non-negative floats order like their bit patterns, so the
// maximum is an unsigned atomicMax). A block covers 256 channels and a 256-row slab: lane l of every
// warp reads channels 8l .. 8l+7 of a row with one 16-byte load, warp w takes the slab's rows w, w+8,
// .., and the eight warps' maxima meet in shared memory.
__global__ void __launch_bounds__(256) act_channel_max(const __nv_bfloat16* __restrict__ X, int64_t rows, int dm,
                                                       unsigned* __restrict__ chmax) {
    __shared__ float part[8][256];
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int c0 = blockIdx.x * 256 + lane * 8;            // dm is a multiple of 128; c0 + 7 < dm or c0 >= dm
    const int64_t r0 = (int64_t)blockIdx.y * 256, r1 = r0 + 256 < rows ? r0 + 256 : rows;
    float m[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    if (c0 < dm) {
        for (int64_t r = r0 + warp; r < r1; r += 8) {
            const uint4 v = *reinterpret_cast<const uint4*>(X + r * dm + c0);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                m[2 * q] = fmaxf(m[2 * q], fabsf(__uint_as_float(w[q] << 16)));
                m[2 * q + 1] = fmaxf(m[2 * q + 1], fabsf(__uint_as_float(w[q] & 0xffff0000u)));
            }
        }
    }
#pragma unroll
    for (int q = 0; q < 8; ++q) part[warp][lane * 8 + q] = m[q];
    __syncthreads();
    const int c = blockIdx.x * 256 + threadIdx.x;
    if (c < dm) {
        float v = part[0][threadIdx.x];
#pragma unroll
        for (int w = 1; w < 8; ++w) v = fmaxf(v, part[w][threadIdx.x]);
        atomicMax(chmax + c, __float_as_uint(v));
    }
}

// The choice, on the device, from the channels' max |x| over the rows: a channel is an outlier when
// its max is above kRangeRatio times the channels' mean. sel = 1 (tensor cores) when there is none;
// sel = 2 (tensor cores with the outlier channels taken out of the tensor-core sums and added in the
// epilogue) when there are at most kMaxOutliers, listed in ascending order in out_idx[0 .. *out_n);
// else sel = 0 (fp32 FMA). One block of 256 threads.
constexpr float kRangeRatio = 4.f;
__global__ void __launch_bounds__(256) act_select(const unsigned* __restrict__ chmax, int dm, int* __restrict__ sel,
                                                  int* __restrict__ out_n, int* __restrict__ out_idx) {
    __shared__ float smax[256], ssum[256];
    __shared__ int scount[257];
    float m = 0.f, sum = 0.f;
    for (int c = threadIdx.x; c < dm; c += 256) {
        const float v = __uint_as_float(chmax[c]);
        m = fmaxf(m, v);
        sum += v;
    }
    smax[threadIdx.x] = m;
    ssum[threadIdx.x] = sum;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if (threadIdx.x < o) {
            smax[threadIdx.x] = fmaxf(smax[threadIdx.x], smax[threadIdx.x + o]);
            ssum[threadIdx.x] += ssum[threadIdx.x + o];
        }
        __syncthreads();
    }
    const float limit = kRangeRatio * (ssum[0] / dm);
    if (smax[0] <= limit) {
        if (threadIdx.x == 0) { *sel = 1; *out_n = 0; }
        return;
    }
    // the outliers of each thread's contiguous channel range, then their places by a prefix sum
    const int per = (dm + 255) / 256, c0 = threadIdx.x * per, c1 = c0 + per < dm ? c0 + per : dm;
    int cnt = 0;
    for (int c = c0; c < c1; ++c) cnt += __uint_as_float(chmax[c]) > limit;
    scount[threadIdx.x + 1] = cnt;
    if (threadIdx.x == 0) scount[0] = 0;
    __syncthreads();
    if (threadIdx.x == 0)
        for (int t = 1; t <= 256; ++t) scount[t] += scount[t - 1];
    __syncthreads();
    const int total = scount[256];
    if (total > kMaxOutliers) {
        if (threadIdx.x == 0) { *sel = 0; *out_n = 0; }
        return;
    }
    int pos = scount[threadIdx.x];
    for (int c = c0; c < c1; ++c)
        if (__uint_as_float(chmax[c]) > limit) out_idx[pos++] = c;
    if (threadIdx.x == 0) { *sel = 2; *out_n = total; }
}

// sel == 2: the weights with the outlier channels zeroed (Wgm, Wum: what the tensor cores multiply),
// and the outlier channels' weights as float32, wo[e][0 gate | 1 up][o][f] (what the epilogue adds).
// One warp per weight row.
__global__ void __launch_bounds__(256) act_prep_weights(const int* __restrict__ sel, const int* __restrict__ out_n,
                                                        const int* __restrict__ out_idx,
                                                        const __nv_bfloat16* __restrict__ Wg,
                                                        const __nv_bfloat16* __restrict__ Wu, int E, int dff, int dm,
                                                        __nv_bfloat16* __restrict__ Wgm, __nv_bfloat16* __restrict__ Wum,
                                                        float* __restrict__ wo) {
    if (*sel != 2) return;
    const int n = *out_n;
    const int lane = threadIdx.x & 31;
    const int64_t nrows = 2LL * E * dff;
    for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < nrows;
         r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
        const int gu = r >= (int64_t)E * dff;
        const int64_t er = gu ? r - (int64_t)E * dff : r;
        const __nv_bfloat16* src = (gu ? Wu : Wg) + er * dm;
        __nv_bfloat16* dst = (gu ? Wum : Wgm) + er * dm;
        for (int c = lane * 8; c < dm; c += 256)
            *reinterpret_cast<uint4*>(dst + c) = __ldg(reinterpret_cast<const uint4*>(src + c));
        __syncwarp();
        const int e = (int)(er / dff), f = (int)(er - (int64_t)e * dff);
        for (int o = lane; o < n; o += 32) {
            const int c = out_idx[o];
            wo[((size_t)(2 * e + gu) * kMaxOutliers + o) * dff + f] = __bfloat162float(src[c]);
            dst[c] = __float2bfloat16(0.f);
        }
    }
}

// sel == 2: the outlier channels of every row as float32, xo[row][o].
__global__ void __launch_bounds__(256) act_prep_rows(const int* __restrict__ sel, const int* __restrict__ out_n,
                                                     const int* __restrict__ out_idx,
                                                     const __nv_bfloat16* __restrict__ X, int64_t rows, int dm,
                                                     float* __restrict__ xo) {
    if (*sel != 2) return;
    const int n = *out_n;
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < rows; r += (int64_t)gridDim.x * blockDim.x)
        for (int o = 0; o < n; ++o) xo[r * kMaxOutliers + o] = __bfloat162float(X[r * dm + out_idx[o]]);
}

}  // namespace

// Workspace: the channel maxima, the outlier list, and for the tensor-core path with outliers the
// masked weight copies, the outlier weights and the rows' outlier channels.
size_t expert_act_workspace_bytes(int d_model, int E, int d_ff, int64_t rows) {
    return clha_round_up((size_t)d_model * sizeof(unsigned)) + clha_round_up((kMaxOutliers + 1) * sizeof(int)) +
           2 * clha_round_up((size_t)E * d_ff * d_model * sizeof(__nv_bfloat16)) +
           clha_round_up((size_t)2 * E * kMaxOutliers * d_ff * sizeof(float)) +
           clha_round_up((size_t)rows * kMaxOutliers * sizeof(float));
}

// The fp32-FMA kernel always reads through a permutation (the tensor-core kernel's TMA loads take
// packed rows only). Otherwise `policy` picks: 1 fp32 FMA, 2 tensor cores, 0 per call on the device
// (act_select): the tensor cores when at most kMaxOutliers channels are outliers (their products then
// leave the tensor-core sums and are added in the epilogue), else the FMA kernel; every kernel is
// queued and the ones not chosen exit at once (no host round trip). ws: expert_act_workspace_bytes;
// sel: one device int.
cudaError_t launch_expert_act(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d_model,
                              const int32_t* perm, const int64_t* seg, int E, const __nv_bfloat16* Wg,
                              const __nv_bfloat16* Wu, int d_ff, __nv_bfloat16* h, int policy, void* ws, int* sel,
                              int* err) {
    {   // per call: the attribute belongs to the current device's context (a process may drive several)
        cudaError_t e = cudaFuncSetAttribute(expert_act_simt, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)sizeof(ActSmem));
        if (e != cudaSuccess) return e;
    }
    const bool simt_only = perm || policy == 1;
    const int* sel_dev = nullptr;
    if (!simt_only) {
        if (policy == 2) {
            return launch_expert_act_tc(s, num_sms, X, rows, d_model, seg, E, Wg, Wu, d_ff, h, nullptr, nullptr,
                                        nullptr, nullptr, nullptr, nullptr, err);
        }
        char* cur = (char*)ws;
        unsigned* chmax = (unsigned*)clha_carve(cur, (size_t)d_model * sizeof(unsigned));
        int* out_n = (int*)clha_carve(cur, (kMaxOutliers + 1) * sizeof(int));
        int* out_idx = out_n + 1;
        __nv_bfloat16* Wgm = (__nv_bfloat16*)clha_carve(cur, (size_t)E * d_ff * d_model * sizeof(__nv_bfloat16));
        __nv_bfloat16* Wum = (__nv_bfloat16*)clha_carve(cur, (size_t)E * d_ff * d_model * sizeof(__nv_bfloat16));
        float* wo = (float*)clha_carve(cur, (size_t)2 * E * kMaxOutliers * d_ff * sizeof(float));
        float* xo = (float*)clha_carve(cur, (size_t)rows * kMaxOutliers * sizeof(float));
        cudaError_t e = cudaMemsetAsync(chmax, 0, (size_t)d_model * sizeof(unsigned), s);
        if (e != cudaSuccess) return e;
        const int64_t slabs = (rows + 255) / 256;
        act_channel_max<<<dim3((unsigned)((d_model + 255) / 256), (unsigned)(slabs < 65535 ? slabs : 65535)), 256, 0,
                          s>>>(X, slabs < 65535 ? rows : 65535 * 256, d_model, chmax);
        act_select<<<1, 256, 0, s>>>(chmax, d_model, sel, out_n, out_idx);
        act_prep_weights<<<4 * num_sms, 256, 0, s>>>(sel, out_n, out_idx, Wg, Wu, E, d_ff, d_model, Wgm, Wum, wo);
        act_prep_rows<<<2 * num_sms, 256, 0, s>>>(sel, out_n, out_idx, X, rows, d_model, xo);
        clha_note_launches(4);
        if ((e = launch_expert_act_tc(s, num_sms, X, rows, d_model, seg, E, Wg, Wu, d_ff, h, sel, Wgm, Wum, out_n, xo,
                                      wo, err)) != cudaSuccess)
            return e;
        sel_dev = sel;
    }
    dim3 grid((unsigned)((rows + TM - 1) / TM), d_ff / TN);
    expert_act_simt<<<grid, 256, sizeof(ActSmem), s>>>(sel_dev, X, rows, d_model, perm, seg, E, Wg, Wu, d_ff, h);
    clha_note_launches(1);
    return cudaGetLastError();
}
