// Phase 3 of CLHA (the CLHA page, §2.2 (3)): GPTQ column-sequential quantization with the
// aggregated Hessian's factor U (H_d^-1 = U^T U), restated from GPTQ (Frantar et al. 2022, Alg. 1).
//
// One CTA owns 128 rows of one weight and walks the columns in 128-column blocks (the lazy-update
// block and the quantization group coincide). Warp roles:
//   warps 0-3  one thread per row: a row's whole block lives in its registers, so the column-by-
//              column error feedback inside a block needs no communication. Per block: take the lazy
//              update from TMEM, w = W[:, blk] - acc; fix the group's grid from the current values;
//              then for 128 columns q = clamp(round(w/s) + z), w_hat = s (q - z),
//              e = (w - w_hat) / U_jj and w[:, c > j] -= e U[j, c] (U's diagonal block in shared
//              memory). The block's errors go to global memory split into tf32 hi + lo parts.
//   warp 4     TMA producer: for block b+1 it streams E[:, :cb] (hi, lo) and the U panel U[:cb, blk]
//              (hi, lo, from a transposed copy so both operands are K-major) in 32-wide k steps;
//              the last 128 k (the errors of the block being quantized) only after the row warps
//              signal they are written.
//   warp 5     MMA issuer: acc = E[:, :cb] U[:cb, blk] with tcgen05.mma kind::tf32, M=128 N=128 K=8,
//              three products per step (hi*hi + hi*lo + lo*hi: float32-class accuracy from tf32
//              inputs), into one of two TMEM accumulators, so block b+1's update overlaps block b's
//              sequential columns.
// The grid and the code are decided with IEEE float32 operations (division and rounding to nearest
// even), the same operations a float32 reference takes on the same current value.
#include "clha_internal.h"
#include "tc_ptx.h"
#include "tmap.h"

namespace {

constexpr int R = 128;      // rows per CTA (one per row thread)
constexpr int BLK = 128;    // columns per lazy block and per group
constexpr int KS = 32;      // k per pipeline stage (one 128-byte row of fp32)
constexpr int STAGES = 2;
constexpr int A_BYTES = R * KS * 4;                       // 16 KB: E rows (hi or lo)
constexpr int B_BYTES = KS * BLK * 4;                     // 16 KB: U panel (hi or lo), K-major
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;    // 64 KB
constexpr int UD_OFF = STAGES * STAGE_BYTES;
constexpr int UINV_OFF = UD_OFF + BLK * BLK * 4;
constexpr int QROW = BLK + 4;                             // bytes per row of the code buffer (padded)
constexpr int CODES_OFF = UINV_OFF + BLK * 4;            // block codes, [row][QROW] bytes
constexpr int QE_OFF = CODES_OFF + R * QROW;             // one quarter's errors, [column][row] floats
constexpr int QW = 32;                                    // columns per quarter of a block
constexpr int BAR_OFF = QE_OFF + QW * R * 4;
constexpr int SMEM_BYTES = BAR_OFF + 128 + 1024;
constexpr int STG = 68;                                   // staging row (floats): 64 columns + pad
constexpr int kThreads = 192;
constexpr uint32_t IDESC = tc::idesc_f32acc(2 /*tf32*/, 0 /*A K-major*/, 0 /*B K-major*/, R, BLK);

struct GptqParams {
    const float* U;        // [n_u, d_in, d_in] (for the diagonal blocks)
    int n_u;               // problem b uses factor b % n_u
    const void* W;
    int w_f32;
    int d_out, d_in, bits;
    uint8_t* codes;
    float* scales;
    uint8_t* zeros;
    float* W_hat;
    float* Ehi;            // [batch, d_out, d_in]
    float* Elo;
    const double* lambda;  // [n_u] damping of each factor, or null
    double* loss;          // [batch] |E|^2 - lambda |W_hat - W|^2, or null
    int* err;
};

__device__ __forceinline__ float to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

__device__ __forceinline__ void row_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

// 16-byte asynchronous global -> shared copy (all of a thread's copies stay in flight together).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

__device__ __forceinline__ void fence_proxy_async_global() {
    asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Columns [32Q, 32Q+32) of the row's block, in order: quantize each, record its error and apply it
// to the rest of the quarter (unrolled; every index is a compile-time constant).
template <int Q>
__device__ __forceinline__ void quarter_sweep(float (&w)[BLK], float s, float z, float maxq, const float* uinv,
                                              const float (*Ud)[BLK], uint8_t (*qs)[QROW], float (*qe)[R], int t) {
#pragma unroll
    for (int jj = 0; jj < QW; ++jj) {
        const int j = Q * QW + jj;
        float q = __fadd_rn(rintf(__fdiv_rn(w[j], s)), z);
        q = fminf(fmaxf(q, 0.f), maxq);
        const float wh = __fmul_rn(s, __fsub_rn(q, z));
        const float e = (w[j] - wh) * uinv[j];
        w[j] = e;                                // a quantized column's register keeps its error
        qs[t][j] = (uint8_t)q;
        qe[jj][t] = e;
#pragma unroll
        for (int c = j + 1; c < (Q + 1) * QW; ++c) w[c] = fmaf(-e, Ud[j][c], w[c]);
    }
}

// The quarter's 32 errors applied, column by column, to every later column of the block: a rolled
// loop over the errors (read back from shared memory) keeps the code small.
template <int Q>
__device__ __forceinline__ void quarter_spill(float (&w)[BLK], const float (*Ud)[BLK], const float (*qe)[R], int t) {
#pragma unroll 2
    for (int jj = 0; jj < QW; ++jj) {
        const float e = qe[jj][t];
        const float4* u4 = reinterpret_cast<const float4*>(&Ud[Q * QW + jj][(Q + 1) * QW]);
#pragma unroll
        for (int c4 = 0; c4 < (BLK - (Q + 1) * QW) / 4; ++c4) {
            const float4 u = u4[c4];
            const int c = (Q + 1) * QW + 4 * c4;
            w[c] = fmaf(-e, u.x, w[c]);
            w[c + 1] = fmaf(-e, u.y, w[c + 1]);
            w[c + 2] = fmaf(-e, u.z, w[c + 2]);
            w[c + 3] = fmaf(-e, u.w, w[c + 3]);
        }
    }
}

__global__ void __launch_bounds__(kThreads, 1)
gptq_tc(const __grid_constant__ CUtensorMap tmEhi, const __grid_constant__ CUtensorMap tmElo,
        const __grid_constant__ CUtensorMap tmUhi, const __grid_constant__ CUtensorMap tmUlo, GptqParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float (*Ud)[BLK] = reinterpret_cast<float (*)[BLK]>(smem + UD_OFF);
    float* uinv = reinterpret_cast<float*>(smem + UINV_OFF);
    uint8_t (*qs)[QROW] = reinterpret_cast<uint8_t (*)[QROW]>(smem + CODES_OFF);
    float (*qe)[R] = reinterpret_cast<float (*)[R]>(smem + QE_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    const uint32_t full0 = tc::smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * STAGES;
    const uint32_t tfull0 = empty0 + 8 * STAGES;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t eready = tempty0 + 16;
    const uint32_t drain = eready + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BAR_OFF + 8 * (2 * STAGES + 6));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int r0 = blockIdx.x * R;
    const int u = b % p.n_u;
    const int nblk = p.d_in / BLK;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(full0 + 8 * s, 1);
            tc::mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tfull0 + 8 * a, 1);
            tc::mbar_init(tempty0 + 8 * a, R);
        }
        tc::mbar_init(eready, R);
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 5) tc::tmem_alloc(tc::smem_u32(tmem_slot), 256);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 4) {
        // ------------------------------------------------------------------ TMA producer
        if (lane == 0) {
            tc::prefetch_tmap(&tmEhi);
            tc::prefetch_tmap(&tmElo);
            tc::prefetch_tmap(&tmUhi);
            tc::prefetch_tmap(&tmUlo);
            int it = 0;
            bool ok = true;
            const int ey = b * p.d_out + r0;
            for (int bb = 1; bb < nblk && ok; ++bb) {
                const int cb = bb * BLK;
                for (int ks = 0; ks < cb / KS; ++ks) {
                    const int k0 = ks * KS;
                    if (k0 == cb - BLK) {   // errors of the previous block: wait until they are written
                        if (!tc::mbar_wait_bounded(eready, (bb - 1) & 1, abort_flag)) { ok = false; break; }
                    }
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t fb = full0 + 8 * s;
                    tc::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t st = tc::smem_u32(smem + s * STAGE_BYTES);
                    tc::tma_load_2d(st, &tmEhi, fb, k0, ey);
                    tc::tma_load_2d(st + A_BYTES, &tmElo, fb, k0, ey);
                    const int uy = u * p.d_in + cb;           // rows n of the transposed factor
                    tc::tma_load_2d(st + 2 * A_BYTES, &tmUhi, fb, k0, uy);
                    tc::tma_load_2d(st + 2 * A_BYTES + B_BYTES, &tmUlo, fb, k0, uy);
                    ++it;
                }
            }
            if (!ok) {
                for (int j = it - 1; j >= 0 && j >= it - STAGES; --j)
                    tc::mbar_wait_bounded(full0 + 8 * (j % STAGES), (j / STAGES) & 1, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 5) {
        // ------------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int bb = 1; bb < nblk && ok; ++bb) {
                const int tcount = bb - 1;
                const int acc = tcount & 1;
                if (!tc::mbar_wait_bounded(tempty0 + 8 * acc, ((tcount >> 1) & 1) ^ 1, abort_flag)) break;
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem + acc * BLK;
                const int nks = bb * BLK / KS;
                for (int ks = 0; ks < nks; ++ks, ++it) {
                    const int s = it % STAGES;
                    if (!tc::mbar_wait_bounded(full0 + 8 * s, (it / STAGES) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t ahi = tc::smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t alo = ahi + A_BYTES;
                    const uint32_t bhi = ahi + 2 * A_BYTES;
                    const uint32_t blo = bhi + B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KS / 8; ++kk) {
                        const uint64_t dah = tc::sw128_desc(ahi + kk * 32, 16, 1024);
                        const uint64_t dal = tc::sw128_desc(alo + kk * 32, 16, 1024);
                        const uint64_t dbh = tc::sw128_desc(bhi + kk * 32, 16, 1024);
                        const uint64_t dbl = tc::sw128_desc(blo + kk * 32, 16, 1024);
                        tc::mma_tf32(d_tmem, dah, dbh, IDESC, (ks | kk) != 0);
                        tc::mma_tf32(d_tmem, dah, dbl, IDESC, 1);
                        tc::mma_tf32(d_tmem, dal, dbh, IDESC, 1);
                    }
                    tc::mma_commit(empty0 + 8 * s);
                }
                if (!ok) break;
                tc::mma_commit(tfull0 + 8 * acc);
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ row threads
        const int t = threadIdx.x;
        const int row = r0 + t;
        const size_t dd = (size_t)p.d_in * p.d_in;
        const float* Ub = p.U + (size_t)u * dd;
        const size_t wrow = ((size_t)b * p.d_out + row) * p.d_in;
        const float maxq = (float)((1 << p.bits) - 1);
        const int ngroups = p.d_in / BLK;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        double e2 = 0.0, d2 = 0.0;   // this row's |E|^2 and |W_hat - W|^2
        for (int bb = 0; bb < nblk; ++bb) {
            const int cb = bb * BLK;
            row_bar();                                   // every row thread is done with the last Ud
            // U's diagonal block: 128 rows x 512 B; thread t copies 16 B pieces (t % 32) of rows t/32 + 4i
#pragma unroll 8
            for (int i = 0; i < BLK / 4; ++i) {
                const int r = (t >> 5) + 4 * i, c4 = (t & 31) * 4;
                cp_async16(&Ud[r][c4], Ub + (size_t)(cb + r) * p.d_in + cb + c4);
            }
            cp_async_wait_all();
            row_bar();
            uinv[t] = 1.0f / Ud[t][t];
            float w[BLK];
            if (p.w_f32) {
                const float4* src = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.W) + wrow + cb);
#pragma unroll
                for (int i = 0; i < BLK / 4; ++i) {
                    const float4 v = src[i];
                    w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
                }
            } else {
                const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.W) + wrow + cb);
#pragma unroll
                for (int i = 0; i < BLK / 8; ++i) {
                    const uint4 v = src[i];
                    const __nv_bfloat162* h2 = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const float2 f = __bfloat1622float2(h2[j]);
                        w[8 * i + 2 * j] = f.x;
                        w[8 * i + 2 * j + 1] = f.y;
                    }
                }
            }
            if (bb > 0 && ok) {    // lazy update of this block from all earlier blocks' errors
                const int tcount = bb - 1;
                const int acc = tcount & 1;
                if (!tc::mbar_wait_bounded(tfull0 + 8 * acc, (tcount >> 1) & 1, abort_flag)) ok = false;
                tc::fence_after_sync();
                if (ok) {
#pragma unroll
                    for (int ch = 0; ch < BLK / 32; ++ch) {
                        uint32_t v[32];
                        tc::tmem_ld_32x32b_x32(tmem + lane_base + acc * BLK + ch * 32, v);
                        tc::tmem_wait_ld();
#pragma unroll
                        for (int j = 0; j < 32; ++j) w[ch * 32 + j] -= __uint_as_float(v[j]);
                    }
                }
                tc::fence_before_sync();
                tc::mbar_arrive(tempty0 + 8 * acc);
            }
            row_bar();                                   // uinv complete
            // grid of the group from the current values (0 always on the grid; [-1, 1] if all zero)
            float xmin = 0.f, xmax = 0.f;
#pragma unroll
            for (int c = 0; c < BLK; ++c) { xmin = fminf(xmin, w[c]); xmax = fmaxf(xmax, w[c]); }
            if (xmin == 0.f && xmax == 0.f) { xmin = -1.f; xmax = 1.f; }
            const float s = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
            const float z = rintf(__fdiv_rn(-xmin, s));
            const int g = cb / BLK;
            p.scales[((size_t)b * p.d_out + row) * ngroups + g] = s;
            p.zeros[((size_t)b * p.d_out + row) * ngroups + g] = (uint8_t)z;
            // 128 columns in four quarters; each column still receives the errors of all earlier
            // columns in column order, exactly as in a single column-by-column sweep
            quarter_sweep<0>(w, s, z, maxq, uinv, Ud, qs, qe, t);
            quarter_spill<0>(w, Ud, qe, t);
            quarter_sweep<1>(w, s, z, maxq, uinv, Ud, qs, qe, t);
            quarter_spill<1>(w, Ud, qe, t);
            quarter_sweep<2>(w, s, z, maxq, uinv, Ud, qs, qe, t);
            quarter_spill<2>(w, Ud, qe, t);
            quarter_sweep<3>(w, s, z, maxq, uinv, Ud, qs, qe, t);
            if (p.loss) {
#pragma unroll
                for (int c = 0; c < BLK; ++c) e2 = fma((double)w[c], (double)w[c], e2);
            }
            // Outputs go through shared memory so that each warp writes whole rows (coalesced).
            // The U tile is no longer needed: its space stages the errors, 64 columns at a time.
            qe[0][t] = s;                                // the quarter-error buffer is free too:
            qe[1][t] = z;                                // it carries each row's grid to the writers
            float* stg = reinterpret_cast<float*>(smem + UD_OFF);
            const bool more = bb + 1 < nblk;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
                row_bar();                               // Ud reads finished / previous half written out
                if (more) {
#pragma unroll
                    for (int i = 0; i < 16; ++i)
                        *reinterpret_cast<float4*>(stg + t * STG + 4 * i) =
                            make_float4(w[64 * h + 4 * i], w[64 * h + 4 * i + 1], w[64 * h + 4 * i + 2],
                                        w[64 * h + 4 * i + 3]);
                }
                row_bar();
                if (more) {    // errors for the later blocks' lazy updates, as tf32 hi + lo
#pragma unroll 4
                    for (int rr = 0; rr < 32; rr += 2) {
                        const int r = warp * 32 + rr + (lane >> 4), c4 = (lane & 15) * 4;
                        const float4 v = *reinterpret_cast<const float4*>(stg + r * STG + c4);
                        const float hx = to_tf32(v.x), hy = to_tf32(v.y), hz = to_tf32(v.z), hw = to_tf32(v.w);
                        const size_t o = ((size_t)b * p.d_out + r0 + r) * p.d_in + cb + 64 * h + c4;
                        *reinterpret_cast<float4*>(p.Ehi + o) = make_float4(hx, hy, hz, hw);
                        *reinterpret_cast<float4*>(p.Elo + o) =
                            make_float4(to_tf32(v.x - hx), to_tf32(v.y - hy), to_tf32(v.z - hz), to_tf32(v.w - hw));
                    }
                }
            }
            if (more) {
                fence_proxy_async_global();
                tc::mbar_arrive(eready);
            }
            // codes, w_hat and |W_hat - W|^2 row by row: lane l owns columns 4l..4l+3
#pragma unroll 2
            for (int rr = 0; rr < 32; ++rr) {
                const int r = warp * 32 + rr;
                const size_t o = ((size_t)b * p.d_out + r0 + r) * p.d_in + cb + 4 * lane;
                const uint32_t cw = *reinterpret_cast<const uint32_t*>(&qs[r][4 * lane]);
                *reinterpret_cast<uint32_t*>(p.codes + o) = cw;
                const float sr = qe[0][r], zr = qe[1][r];
                float v[4];
#pragma unroll
                for (int m = 0; m < 4; ++m) v[m] = __fmul_rn(sr, __fsub_rn((float)((cw >> (8 * m)) & 255u), zr));
                if (p.W_hat) *reinterpret_cast<float4*>(p.W_hat + o) = make_float4(v[0], v[1], v[2], v[3]);
                if (p.loss) {
                    float wv[4];
                    if (p.w_f32) {
                        const float4 f = *reinterpret_cast<const float4*>(reinterpret_cast<const float*>(p.W) + o);
                        wv[0] = f.x; wv[1] = f.y; wv[2] = f.z; wv[3] = f.w;
                    } else {
                        const uint2 raw = *reinterpret_cast<const uint2*>(reinterpret_cast<const __nv_bfloat16*>(p.W) + o);
                        const float2 f0 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
                        const float2 f1 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
                        wv[0] = f0.x; wv[1] = f0.y; wv[2] = f1.x; wv[3] = f1.y;
                    }
#pragma unroll
                    for (int m = 0; m < 4; ++m) {
                        const double dv = (double)v[m] - (double)wv[m];
                        d2 = fma(dv, dv, d2);
                    }
                }
            }
        }
        if (p.loss) {
            double v = e2 - p.lambda[u] * d2;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
            if (lane == 0) atomicAdd(&p.loss[b], v);
        }
    }

    __syncthreads();
    if (warp == 5) {
        if (lane == 0) {
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, abort_flag, 100000000ull);
        }
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
    if (threadIdx.x == 0 && *abort_flag) clha_record_error(p.err, CLHA_ERR_TIMEOUT, b, r0, KID_QUANTIZE);
}

// U -> transposed (hi, lo) tf32 parts: hi_t[j][i] + lo_t[j][i] ~ U[i][j], so the lazy-update
// operand U[k][n] is read K-major (rows n, contiguous k). 32x32 tiles through shared memory.
__global__ void __launch_bounds__(256) gptq_split_t(const float* __restrict__ U, int d, float* __restrict__ hi,
                                                    float* __restrict__ lo) {
    __shared__ float tile[32][33];
    const size_t base = (size_t)blockIdx.z * d * d;
    const int i0 = blockIdx.y * 32, j0 = blockIdx.x * 32;
    const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
    for (int r = ty; r < 32; r += 8) tile[r][tx] = U[base + (size_t)(i0 + r) * d + j0 + tx];
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const float x = tile[tx][r];                       // U[i0 + tx][j0 + r]
        const float h = to_tf32(x);
        const size_t o = base + (size_t)(j0 + r) * d + i0 + tx;
        hi[o] = h;
        lo[o] = to_tf32(x - h);
    }
}

}  // namespace

size_t quantize_workspace_bytes(int batch, int d_out, int d_in) {
    const size_t e = clha_round_up((size_t)batch * d_out * d_in * sizeof(float));
    const size_t uu = clha_round_up((size_t)batch * d_in * d_in * sizeof(float));
    return 2 * e + 2 * uu;
}

cudaError_t launch_quantize(cudaStream_t s, const float* U, int n_u, const void* W, int w_is_f32, int batch,
                            int d_out, int d_in, int bits, uint8_t* codes, float* scales, uint8_t* zeros,
                            float* W_hat, const double* lambda, double* loss, void* ws, int* err) {
    char* cur = (char*)ws;
    float* Ehi = (float*)clha_carve(cur, (size_t)batch * d_out * d_in * sizeof(float));
    float* Elo = (float*)clha_carve(cur, (size_t)batch * d_out * d_in * sizeof(float));
    float* Uhi = (float*)clha_carve(cur, (size_t)batch * d_in * d_in * sizeof(float));
    float* Ulo = (float*)clha_carve(cur, (size_t)batch * d_in * d_in * sizeof(float));
    cudaError_t e;
    CUtensorMap tEhi, tElo, tUhi, tUlo;
    if ((e = make_tmap_2d(&tEhi, Ehi, (uint64_t)batch * d_out, d_in, 4, R, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tElo, Elo, (uint64_t)batch * d_out, d_in, 4, R, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tUhi, Uhi, (uint64_t)n_u * d_in, d_in, 4, BLK, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tUlo, Ulo, (uint64_t)n_u * d_in, d_in, 4, BLK, KS)) != cudaSuccess) return e;
    if (d_in > BLK) {
        gptq_split_t<<<dim3(d_in / 32, d_in / 32, n_u), 256, 0, s>>>(U, d_in, Uhi, Ulo);
        clha_note_launches(1);
    }
    if ((e = cudaFuncSetAttribute(gptq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
        return e;
    if (loss && (e = cudaMemsetAsync(loss, 0, (size_t)batch * sizeof(double), s)) != cudaSuccess) return e;
    GptqParams p{U, n_u, W, w_is_f32, d_out, d_in, bits, codes, scales, zeros, W_hat, Ehi, Elo, lambda, loss, err};
    dim3 grid(d_out / R, batch);
    gptq_tc<<<grid, kThreads, SMEM_BYTES, s>>>(tEhi, tElo, tUhi, tUlo, p);
    clha_note_launches(1);
    return cudaGetLastError();
}
