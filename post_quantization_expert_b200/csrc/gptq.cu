// Phase 3 of CLHA (the CLHA page, §2.2 (3)): GPTQ column-sequential quantization with the
// aggregated Hessian's factor U (H_d^-1 = U^T U), restated from GPTQ (Frantar et al. 2022, Alg. 1).
//
// One CTA owns 128 rows of one weight and walks the columns in 128-column blocks (the lazy-update
// block and the quantization group coincide), each block in four 32-column quarters. The column
// recurrence w[:, c] -= e_j U[j, c] (c > j) is split three ways:
//   * inside a quarter: fp32 FMAs in the row thread's registers (a row's 32 current values);
//   * from a quarter to the later quarters of its block: one small tensor-core product
//     acc[:, later] += E_q U[q, later], accumulated into the same TMEM columns that hold the block's
//     lazy update (the row threads read each quarter's columns only after it);
//   * from a block to all later blocks: the lazy update acc = E[:, :cb] U[:cb, blk], streamed while
//     the previous block is being swept.
// Products are tcgen05.mma kind::tf32 with operands split hi + lo and three products per step
// (hi*hi + hi*lo + lo*hi: float32-class accuracy). Warp roles:
//   warps 0-3  one thread per row: grid of the block from its current values, then per quarter: read
//              the quarter's update from TMEM, q = clamp(round(w/s) + z), w_hat = s (q - z),
//              e = (w - w_hat) / U_jj, in-quarter updates; write the quarter's errors as tf32 hi/lo
//              into shared memory in the 128-byte-swizzled K-major layout, which is both the A operand
//              of the quarter's product and the source of a TMA store of E to global memory (read
//              by the later blocks' lazy updates).
//   warp 4     TMA producer of the lazy update: E[:, :cb] (hi, lo) and the U panel U[:cb, blk] (hi,
//              lo, from a transposed copy so both operands are K-major) in 32-wide k steps; each of
//              the last four (the quarters of the block being swept) once that quarter is stored, so
//              that only the last quarter's step is left when the block ends.
//   warp 5     MMA issuer: the quarter products as soon as they are requested (the next quarter's
//              columns first, with their own completion signal, since they gate the row threads;
//              then the rest), between them the next block's lazy update (one step in the tensor
//              pipe at a time), into the other of two TMEM accumulators.
// The grid and the code are decided with IEEE float32 operations (division and rounding to nearest
// even), the same operations a float32 reference takes on the same current value.
//
// The factor may also be F, the block-scaled Cholesky factor of H_d (factor.cu): its diagonal blocks
// are U's, so everything inside a block is unchanged, and the later blocks' lazy updates (and the
// trailing updates) take W_hat - W of the earlier columns in place of their scaled errors e; the row
// threads write it over e in the same shared buffer once the quarter product has read e, and the TMA
// store takes it from there.
//
// Column chunks. The tensor core's fp32 accumulator does not round each addition to nearest, so a
// lazy update that sums the errors of many thousands of columns in TMEM drifts away from the exact
// sum (enough, on long rows, to flip rounding decisions that float32 arithmetic rounding to nearest
// would not). A launch therefore quantizes one chunk of at most CHUNK = 512 columns, its lazy updates
// summing only that chunk's errors, and gptq_trail then folds the chunk's errors into float32 running
// weights of every later column (a tcgen05 product over the chunk, subtracted by TMA reduce-add: fp32
// adds rounded to nearest). A weight with at most CHUNK columns takes one launch and no running copy.
#include "clha_internal.h"
#include "tc_ptx.h"
#include "tmap.h"

namespace {

constexpr int R = 128;      // rows per CTA (one per row thread)
constexpr int BLK = 128;    // columns per lazy block and per group
constexpr int QW = 32;      // columns per quarter
constexpr int KS = 32;      // k per lazy pipeline stage (one 128-byte row of fp32)
constexpr int STAGES = 2;
constexpr int A_BYTES = R * KS * 4;                       // 16 KB: E rows (hi or lo)
constexpr int B_BYTES = KS * BLK * 4;                     // 16 KB: U panel (hi or lo), K-major
constexpr int STAGE_BYTES = 2 * A_BYTES + 2 * B_BYTES;    // 64 KB
constexpr int SA_OFF = STAGES * STAGE_BYTES;              // quarter errors hi, lo: [128 rows][32 k]
constexpr int SA_BYTES = R * QW * 4;                      // 16 KB each
// U rows of a quarter's product (K-major [n][32 k], hi then lo), two buffers used alternately:
// quarters 0 and 2 (96 and 32 rows) in buffer 0, quarter 1 (64 rows) in buffer 1
constexpr int SB0_OFF = SA_OFF + 2 * SA_BYTES;
constexpr int SB0_HALF = 96 * QW * 4;                     // 12 KB
constexpr int SB1_OFF = SB0_OFF + 2 * SB0_HALF;
constexpr int SB1_HALF = 64 * QW * 4;                     // 8 KB
constexpr int UQ_OFF = SB1_OFF + 2 * SB1_HALF;            // the block's four diagonal 32x32 U blocks
constexpr int UINV_OFF = UQ_OFF + 4 * QW * QW * 4;
constexpr int BAR_OFF = UINV_OFF + BLK * 4;
constexpr int SMEM_BYTES = BAR_OFF + 256 + 1024;
constexpr int kThreads = 192;
constexpr uint32_t IDESC_LAZY = tc::idesc_f32acc(2 /*tf32*/, 0 /*A K-major*/, 0 /*B K-major*/, R, BLK);
static_assert(SA_OFF % 1024 == 0 && SB0_OFF % 1024 == 0 && (SB0_OFF + SB0_HALF) % 1024 == 0 && SB1_OFF % 1024 == 0 &&
                  (SB1_OFF + SB1_HALF) % 1024 == 0, "swizzle atoms");
static_assert(SMEM_BYTES <= 232448, "shared memory");

__host__ __device__ constexpr uint32_t idesc_spill(int n) {
    return tc::idesc_f32acc(2, 0, 0, R, (uint32_t)n);
}

struct GptqParams {
    const float* U;        // [n_u, d_in, d_in] (for the diagonal blocks)
    int n_u;               // problem b uses factor b % n_u
    const void* W;         // the original weights (the loss compares W_hat with them)
    int w_f32;
    const float* Wc;       // float32 running weights (W minus the earlier chunks' updates), or null: W
    int c0, c1;            // the column chunk this launch quantizes
    int d_out, d_in, bits;
    uint8_t* codes;
    float* scales;
    uint8_t* zeros;
    float* W_hat;
    const double* lambda;  // [n_u] damping of each factor, or null
    double* loss;          // [batch] |E|^2 - lambda |W_hat - W|^2, or null
    int* err;
    int blk;               // U holds F, the block-scaled Cholesky factor of H_d (lazy operand W_hat - W)
};

__device__ __forceinline__ float to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return __uint_as_float(r);
}

__device__ __forceinline__ void row_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(tc::smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void fence_proxy_async_global() { asm volatile("fence.proxy.async.global;" ::: "memory"); }

// This row's 32 current values of a quarter, in order: quantize each, keep its error in w[j] and
// apply it to the quarter's later columns (unrolled; every index a compile-time constant). The codes
// are packed four to a word.
__device__ __forceinline__ void quarter_sweep(float (&w)[QW], float s, float z, float maxq, const float* uinv,
                                              const float (*Uq)[QW], uint32_t (&codes)[QW / 4]) {
#pragma unroll
    for (int j = 0; j < QW; ++j) {
        float q = __fadd_rn(rintf(__fdiv_rn(w[j], s)), z);
        q = fminf(fmaxf(q, 0.f), maxq);
        const float wh = __fmul_rn(s, __fsub_rn(q, z));
        const float e = (w[j] - wh) * uinv[j];
        w[j] = e;
        if ((j & 3) == 0) codes[j >> 2] = 0u;
        codes[j >> 2] |= (uint32_t)q << (8 * (j & 3));
#pragma unroll
        for (int c = 1; c < QW; ++c)
            if (c > j) w[c] = fmaf(-e, Uq[j][c], w[c]);
    }
}

// W[row, c0 .. c0+31] as floats (bf16 or fp32 source); cur: the running weights when they exist.
__device__ __forceinline__ void load_w32(const GptqParams& p, size_t off, float (&w)[QW], bool cur = false) {
    if (p.w_f32 || (cur && p.Wc)) {
        const float4* src = reinterpret_cast<const float4*>((cur && p.Wc ? p.Wc : reinterpret_cast<const float*>(p.W)) + off);
#pragma unroll
        for (int i = 0; i < QW / 4; ++i) {
            const float4 v = src[i];
            w[4 * i] = v.x; w[4 * i + 1] = v.y; w[4 * i + 2] = v.z; w[4 * i + 3] = v.w;
        }
    } else {
        const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(p.W) + off);
#pragma unroll
        for (int i = 0; i < QW / 8; ++i) {
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
}

__global__ void __launch_bounds__(kThreads, 1)
gptq_tc(const __grid_constant__ CUtensorMap tmEhi, const __grid_constant__ CUtensorMap tmElo,
        const __grid_constant__ CUtensorMap tmUhi, const __grid_constant__ CUtensorMap tmUlo,
        const __grid_constant__ CUtensorMap tmQhi, const __grid_constant__ CUtensorMap tmQlo, GptqParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    float (*Uq)[QW][QW] = reinterpret_cast<float (*)[QW][QW]>(smem + UQ_OFF);
    float* uinv = reinterpret_cast<float*>(smem + UINV_OFF);
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + BAR_OFF);
    const uint32_t full0 = tc::smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * STAGES;
    const uint32_t tfull0 = empty0 + 8 * STAGES;   // lazy update of a block complete (per accumulator)
    const uint32_t tempty0 = tfull0 + 16;          // row threads done with an accumulator
    const uint32_t qready0 = tempty0 + 16;         // [4] quarter q of a block: its errors are in global memory
    const uint32_t sreq = qready0 + 32;            // a quarter's errors are in shared memory
    const uint32_t sbfull0 = sreq + 8;             // U rows of quarter 0 or 2's product in buffer 0 (twice a block)
    const uint32_t sbfull1 = sbfull0 + 8;          // U rows of quarter 1's product in buffer 1 (once a block)
    const uint32_t sdone = sbfull1 + 8;            // the quarter product's next-quarter columns are done
    const uint32_t sdone2 = sdone + 8;             // the whole quarter product is done (buffers free)
    const uint32_t drain = sdone2 + 8;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + BAR_OFF + 8 * (2 * STAGES + 14));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t sa_hi = tc::smem_u32(smem + SA_OFF), sa_lo = sa_hi + SA_BYTES;
    const uint32_t sb0 = tc::smem_u32(smem + SB0_OFF), sb1 = tc::smem_u32(smem + SB1_OFF);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int b = blockIdx.y;
    const int r0 = blockIdx.x * R;
    const int u = b % p.n_u;
    const int nblk = p.d_in / BLK;
    const int b_lo = p.c0 / BLK, b_hi = p.c1 / BLK;   // this launch's blocks; local index lb = bb - b_lo
    const int ey = b * p.d_out + r0;               // this CTA's rows in the [batch * d_out, d_in] E view
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(full0 + 8 * s, 1);
            tc::mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tfull0 + 8 * a, 1);
            tc::mbar_init(tempty0 + 8 * a, R);
        }
        for (int qq = 0; qq < 4; ++qq) tc::mbar_init(qready0 + 8 * qq, 1);
        tc::mbar_init(sreq, R);
        tc::mbar_init(sbfull0, 1);
        tc::mbar_init(sbfull1, 1);
        tc::mbar_init(sdone, 1);
        tc::mbar_init(sdone2, 1);
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
        // ------------------------------------------------------------------ TMA producer (lazy update)
        if (lane == 0) {
            tc::prefetch_tmap(&tmEhi);
            tc::prefetch_tmap(&tmElo);
            tc::prefetch_tmap(&tmUhi);
            tc::prefetch_tmap(&tmUlo);
            int it = 0;
            bool ok = true;
            for (int bb = b_lo + 1; bb < b_hi && ok; ++bb) {
                const int cb = bb * BLK;
                for (int ks = p.c0 / KS; ks < cb / KS; ++ks) {   // the chunk's earlier errors only
                    const int k0 = ks * KS;
                    if (k0 >= cb - BLK) {   // the previous block's errors: each quarter once it is stored, so
                                            // that only the last quarter's step remains at the block's end
                        const int qi = (k0 - (cb - BLK)) / KS;
                        if (!tc::mbar_wait_bounded(qready0 + 8 * qi, (bb - 1 - b_lo) & 1, abort_flag)) { ok = false; break; }
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
            int it = 0, nq = 0;   // lazy k steps consumed; quarter products issued
            bool ok = true;
            for (int bb = b_lo; bb < b_hi && ok; ++bb) {
                // block bb: its three quarter products (into acc lb & 1) and block bb+1's lazy update
                const int lb = bb - b_lo;
                const bool lazy = bb + 1 < b_hi;
                const int lacc = (lb + 1) & 1, pacc = lb & 1;
                const int nks = lazy ? ((bb + 1) * BLK - p.c0) / KS : 0;
                int ks = 0, q = 0;
                bool lazy_ready = !lazy;
                if (lazy && lb >= 1) {   // the row threads are done with block bb-1's accumulator
                    if (!tc::mbar_wait_bounded(tempty0 + 8 * lacc, ((lb - 1) >> 1) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                }
                lazy_ready = true;
                uint64_t t0 = tc::globaltimer_ns();
                uint32_t spins = 0;
                while (q < 3 || ks < nks) {
                    bool progressed = false;
                    const uint32_t sbf = (q & 1) ? sbfull1 : sbfull0;   // phases: 2 per block for buffer 0
                    const uint32_t sbp = (q & 1) ? (uint32_t)(lb & 1) : (uint32_t)((q >> 1) & 1);
                    if (q < 3 && tc::mbar_test_wait(sreq, nq & 1) && tc::mbar_test_wait(sbf, sbp)) {
                        tc::fence_after_sync();
                        const uint32_t sbh = (q & 1) ? sb1 : sb0;
                        const uint32_t sbl = sbh + ((q & 1) ? SB1_HALF : SB0_HALF);
                        // part 1: the next quarter's 32 columns; part 2: the later ones
                        for (int part = 0; part < 2; ++part) {
                            const int n = part == 0 ? QW : BLK - QW * (q + 2);
                            if (n > 0) {
                                const uint32_t d_tmem = tmem + pacc * BLK + QW * (q + 1) + part * QW;
                                const uint32_t id = idesc_spill(n);
                                const uint32_t boff = part * 4096;   // 32 rows of 128 B
#pragma unroll
                                for (int kk = 0; kk < QW / 8; ++kk) {
                                    const uint64_t dah = tc::sw128_desc(sa_hi + kk * 32, 16, 1024);
                                    const uint64_t dal = tc::sw128_desc(sa_lo + kk * 32, 16, 1024);
                                    const uint64_t dbh = tc::sw128_desc(sbh + boff + kk * 32, 16, 1024);
                                    const uint64_t dbl = tc::sw128_desc(sbl + boff + kk * 32, 16, 1024);
                                    tc::mma_tf32(d_tmem, dah, dbh, id, (lb > 0 || q > 0 || kk > 0) ? 1u : 0u);
                                    tc::mma_tf32(d_tmem, dah, dbl, id, 1);
                                    tc::mma_tf32(d_tmem, dal, dbh, id, 1);
                                }
                            }
                            tc::mma_commit(part == 0 ? sdone : sdone2);
                        }
                        ++q;
                        ++nq;
                        progressed = true;
                    }
                    // a lazy step only once the previous one has left the tensor pipe, so that a
                    // quarter product (which the row threads wait for) queues behind one step at most
                    const bool pipe_clear = it == 0 || tc::mbar_test_wait(empty0 + 8 * ((it - 1) % STAGES), ((it - 1) / STAGES) & 1);
                    if (lazy_ready && ks < nks && pipe_clear &&
                        tc::mbar_test_wait(full0 + 8 * (it % STAGES), (it / STAGES) & 1)) {
                        tc::fence_after_sync();
                        const int s = it % STAGES;
                        const uint32_t ahi = tc::smem_u32(smem + s * STAGE_BYTES);
                        const uint32_t alo = ahi + A_BYTES;
                        const uint32_t bhi = ahi + 2 * A_BYTES;
                        const uint32_t blo = bhi + B_BYTES;
                        const uint32_t d_tmem = tmem + lacc * BLK;
#pragma unroll
                        for (int kk = 0; kk < KS / 8; ++kk) {
                            const uint64_t dah = tc::sw128_desc(ahi + kk * 32, 16, 1024);
                            const uint64_t dal = tc::sw128_desc(alo + kk * 32, 16, 1024);
                            const uint64_t dbh = tc::sw128_desc(bhi + kk * 32, 16, 1024);
                            const uint64_t dbl = tc::sw128_desc(blo + kk * 32, 16, 1024);
                            tc::mma_tf32(d_tmem, dah, dbh, IDESC_LAZY, (ks | kk) != 0);
                            tc::mma_tf32(d_tmem, dah, dbl, IDESC_LAZY, 1);
                            tc::mma_tf32(d_tmem, dal, dbh, IDESC_LAZY, 1);
                        }
                        tc::mma_commit(empty0 + 8 * s);
                        ++ks;
                        ++it;
                        if (ks == nks) tc::mma_commit(tfull0 + 8 * lacc);
                        progressed = true;
                    }
                    if (progressed) {
                        t0 = tc::globaltimer_ns();
                        spins = 0;
                    } else if (((++spins) & 255u) == 0u) {
                        if (*abort_flag) { ok = false; break; }
                        if (tc::globaltimer_ns() - t0 > 2000000000ull) { *abort_flag = 1; ok = false; break; }
                    }
                }
            }
        }
        __syncwarp();
    } else {
        // ------------------------------------------------------------------ row threads
        const int t = threadIdx.x;
        const int row = r0 + t;
        const float* Ub = p.U + (size_t)u * p.d_in * p.d_in;
        const size_t wrow = ((size_t)b * p.d_out + row) * p.d_in;
        const float maxq = (float)((1 << p.bits) - 1);
        const int ngroups = p.d_in / BLK;
        const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
        bool ok = true;
        int nq = 0;                  // quarter products requested so far
        double e2 = 0.0, d2 = 0.0;   // this row's |E|^2 and |W_hat - W|^2
        auto load_sb = [&](int cb, int q) {   // the U rows of quarter q's product: n = later columns
            const int nbox = 3 - q;
            const uint32_t sbh = (q & 1) ? sb1 : sb0;
            const uint32_t sbl = sbh + ((q & 1) ? SB1_HALF : SB0_HALF);
            const uint32_t sbf = (q & 1) ? sbfull1 : sbfull0;
            tc::mbar_arrive_expect_tx(sbf, (uint32_t)(2 * nbox * 32 * QW * 4));
            for (int bx = 0; bx < nbox; ++bx) {
                const int n0 = u * p.d_in + cb + QW * (q + 1) + 32 * bx;
                tc::tma_load_2d(sbh + bx * 4096, &tmQhi, sbf, cb + QW * q, n0);
                tc::tma_load_2d(sbl + bx * 4096, &tmQlo, sbf, cb + QW * q, n0);
            }
        };
        auto load_uq = [&](int cb) {          // the block's four diagonal 32x32 blocks of U
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int e = i * R + t;          // 0 .. 1023: (quarter, row, 16-byte piece)
                const int qq = e >> 8, rr = (e >> 3) & 31, c4 = (e & 7) * 4;
                cp_async16(&Uq[qq][rr][c4], Ub + (size_t)(cb + QW * qq + rr) * p.d_in + cb + QW * qq + c4);
            }
        };
        // On a failed wait (abort) the row threads still run every step, so each reaches every named
        // barrier; their later waits return at once.
        load_uq(p.c0);
        for (int bb = b_lo; bb < b_hi; ++bb) {
            const int cb = bb * BLK;
            const int lb = bb - b_lo;
            const int acc = lb & 1;
            const bool more = bb + 1 < nblk;             // later blocks (of this chunk or later ones) need E
            const bool next_here = bb + 1 < b_hi;        // the next block is this launch's
            const size_t orow = ((size_t)b * p.d_out + row) * p.d_in + cb;   // this row's outputs
            row_bar();                                   // the last block's readers of Uq are done
            bool sb2_sent = false;                       // quarter 2's U rows (buffer 0, after quarter 0's product)
            if (t == 0) {                                // both buffers are free: the last block's products are done
                load_sb(cb, 0);
                load_sb(cb, 1);
            }
            cp_async_wait_all();                         // this block's Uq (issued during the last block)
            uinv[t] = 1.0f / __ldg(Ub + (size_t)(cb + t) * p.d_in + cb + t);
            if (lb > 0) {
                if (!tc::mbar_wait_bounded(tfull0 + 8 * acc, (lb - 1) >> 1 & 1, abort_flag)) ok = false;
                tc::fence_after_sync();
            }
            // grid of the group from the current values (0 always on the grid; [-1, 1] if all zero)
            float xmin = 0.f, xmax = 0.f;
            for (int ch = 0; ch < 4; ++ch) {
                float w[QW];
                load_w32(p, wrow + cb + QW * ch, w, true);
                if (lb > 0) {
                    uint32_t v[32];
                    tc::tmem_ld_32x32b_x32(tmem + lane_base + acc * BLK + ch * QW, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < QW; ++j) w[j] -= __uint_as_float(v[j]);
                }
#pragma unroll
                for (int j = 0; j < QW; ++j) { xmin = fminf(xmin, w[j]); xmax = fmaxf(xmax, w[j]); }
            }
            if (xmin == 0.f && xmax == 0.f) { xmin = -1.f; xmax = 1.f; }
            const float s = __fdiv_rn(__fsub_rn(xmax, xmin), maxq);
            const float z = rintf(__fdiv_rn(-xmin, s));
            p.scales[((size_t)b * p.d_out + row) * ngroups + bb] = s;
            p.zeros[((size_t)b * p.d_out + row) * ngroups + bb] = (uint8_t)z;
            row_bar();                                   // Uq, uinv visible to every row thread
            for (int q = 0; q < 4; ++q) {
                float w[QW];
                load_w32(p, wrow + cb + QW * q, w, true);
                if (q > 0) {                             // the previous quarter's product reached this quarter
                    if (!tc::mbar_wait_bounded(sdone, (nq - 1) & 1, abort_flag)) ok = false;
                    tc::fence_after_sync();
                }
                if (lb > 0 || q > 0) {
                    uint32_t v[32];
                    tc::tmem_ld_32x32b_x32(tmem + lane_base + acc * BLK + q * QW, v);
                    tc::tmem_wait_ld();
#pragma unroll
                    for (int j = 0; j < QW; ++j) w[j] -= __uint_as_float(v[j]);
                }
                if (q == 3) {                            // last read of this accumulator
                    tc::fence_before_sync();
                    tc::mbar_arrive(tempty0 + 8 * acc);
                }
                uint32_t codes[QW / 4];
                quarter_sweep(w, s, z, maxq, uinv + QW * q, Uq[q], codes);
                uint8_t* sah = smem + SA_OFF + t * 128;
                uint8_t* sal = sah + SA_BYTES;
                auto put_row = [&](const float (&v)[QW]) {   // row t, 16-byte piece c at c ^ (t % 8)
#pragma unroll
                    for (int c = 0; c < QW / 4; ++c) {
                        const float h0 = to_tf32(v[4 * c]), h1 = to_tf32(v[4 * c + 1]), h2 = to_tf32(v[4 * c + 2]),
                                    h3 = to_tf32(v[4 * c + 3]);
                        const int off = ((c ^ (t & 7)) << 4);
                        *reinterpret_cast<float4*>(sah + off) = make_float4(h0, h1, h2, h3);
                        *reinterpret_cast<float4*>(sal + off) =
                            make_float4(to_tf32(v[4 * c] - h0), to_tf32(v[4 * c + 1] - h1),
                                        to_tf32(v[4 * c + 2] - h2), to_tf32(v[4 * c + 3] - h3));
                    }
                    fence_proxy_async_smem();
                };
                float wo[QW];                                // the original weights of the quarter (issued
                if (p.loss || (p.blk && more)) load_w32(p, wrow + cb + QW * q, wo);   // before the handoff)
                // first the quarter's errors as tf32 hi/lo into the shared buffer and the request for the
                // quarter product, which gates the next quarter; the outputs below overlap that product.
                // The buffer is free once the last quarter's whole product and its store have read it.
                if (!(q == 3 && !more)) {
                    if (q > 0 && !tc::mbar_wait_bounded(sdone2, (nq - 1) & 1, abort_flag)) ok = false;
                    if (q == 1 && t == 0 && !sb2_sent) {     // quarter 0's product is done with buffer 0
                        load_sb(cb, 2);
                        sb2_sent = true;
                    }
                    if (t == 0) {
                        if (q > 0 && more) {                 // the previous quarter's store is complete: its
                            tc::bulk_wait_all();             // errors may feed the next block's lazy update
                            fence_proxy_async_global();
                            tc::mbar_arrive(qready0 + 8 * (q - 1));
                        } else {
                            tc::bulk_wait_read<0>();
                        }
                    }
                    row_bar();
                    if (q == 3 && next_here) load_uq(cb + BLK);   // every row is past its last use of Uq
                    if (!p.blk || q < 3) {                   // e: the quarter product's operand
                        put_row(w);
                        if (q < 3) {
                            tc::mbar_arrive(sreq);
                            ++nq;
                        }
                    }
                }
                // outputs of this quarter: codes (32 B) and w_hat (128 B) of this row, the loss terms
                uint4* cdst = reinterpret_cast<uint4*>(p.codes + orow + QW * q);
                cdst[0] = make_uint4(codes[0], codes[1], codes[2], codes[3]);
                cdst[1] = make_uint4(codes[4], codes[5], codes[6], codes[7]);
                if (p.W_hat || p.loss) {
                    double dq[4] = {0.0, 0.0, 0.0, 0.0};     // four independent chains: the fp64 FMA
#pragma unroll                                              // latency, not its rate, bounds one chain
                    for (int c = 0; c < QW / 4; ++c) {
                        float v[4];
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            v[m] = __fmul_rn(s, __fsub_rn((float)((codes[c] >> (8 * m)) & 255u), z));
                        if (p.W_hat)
                            *reinterpret_cast<float4*>(p.W_hat + orow + QW * q + 4 * c) = make_float4(v[0], v[1], v[2], v[3]);
                        if (p.loss) {
#pragma unroll
                            for (int m = 0; m < 4; ++m) {
                                const double dv = (double)v[m] - (double)wo[4 * c + m];
                                dq[m] = fma(dv, dv, dq[m]);
                            }
                        }
                    }
                    d2 += (dq[0] + dq[1]) + (dq[2] + dq[3]);
                }
                if (p.loss) {
                    double eq[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
                    for (int j = 0; j < QW; ++j) eq[j & 3] = fma((double)w[j], (double)w[j], eq[j & 3]);
                    e2 += (eq[0] + eq[1]) + (eq[2] + eq[3]);
                }
                if (more && p.blk) {
                    // the later blocks' lazy operand under F: W_hat - W of the quarter (original W), written
                    // over e once the quarter product has read it (a second buffer does not fit in shared
                    // memory; stores straight from registers to global memory measured slower)
#pragma unroll
                    for (int c = 0; c < QW / 4; ++c)
#pragma unroll
                        for (int m = 0; m < 4; ++m)
                            w[4 * c + m] = __fsub_rn(__fmul_rn(s, __fsub_rn((float)((codes[c] >> (8 * m)) & 255u), z)),
                                                     wo[4 * c + m]);
                    if (q < 3 && !tc::mbar_wait_bounded(sdone2, (nq - 1) & 1, abort_flag)) ok = false;
                    if (q == 0 && t == 0) {                  // quarter 0's product is done with buffer 0
                        load_sb(cb, 2);
                        sb2_sent = true;
                    }
                    put_row(w);
                }
                if (more) {
                    row_bar();                           // every row's errors are in the buffer
                    if (t == 0) {
                        tc::tma_store_2d(&tmEhi, sa_hi, cb + QW * q, ey);
                        tc::tma_store_2d(&tmElo, sa_lo, cb + QW * q, ey);
                        tc::bulk_commit();
                        if (q == 3) {
                            tc::bulk_wait_all();
                            fence_proxy_async_global();
                            tc::mbar_arrive(qready0 + 24);
                        }
                    }
                }
            }
            if (next_here) {   // this row's weights for the next block into L1
                const int es = (p.w_f32 || p.Wc) ? 4 : 2;
                const char* nxt = reinterpret_cast<const char*>(p.Wc ? (const void*)p.Wc : p.W) + (wrow + cb + BLK) * es;
                for (int o = 0; o < BLK * es; o += 128)
                    asm volatile("prefetch.global.L1 [%0];" ::"l"(nxt + o));
            }
        }
        if (t == 0) tc::bulk_wait_all();
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

// ------------------------------------------------------------------------------ trailing update
// The tensor core adds a product into its fp32 accumulator without rounding to nearest, so a long
// chain of accumulations drifts (for a lazy update over tens of thousands of columns, far enough to
// move GPTQ's rounding decisions). GPTQ therefore runs in column chunks of CHUNK columns: inside a
// chunk the lazy updates accumulate at most CHUNK columns of errors in TMEM, and at the end of a chunk
// this kernel folds the chunk's errors into the running weights of all later columns,
//   Wc[rows, n] -= sum_{k in chunk} E[rows, k] U[k, n],   n >= chunk end,
// as a 3xTF32 tcgen05 product (K = the chunk) whose fp32 result is subtracted by a TMA reduce-add (the
// L2's fp32 adds round to nearest). Persistent: tiles of 128 rows x 128 columns; warp 0 is the TMA
// producer, warp 1 the MMA issuer (two TMEM accumulators, so a tile's epilogue overlaps the next
// tile's products), warps 2-5 the epilogue (one TMEM lane quadrant each).
constexpr int CHUNK = 512;
constexpr int T_STAGES = 2;
constexpr int T_STG_OFF = T_STAGES * STAGE_BYTES;           // 128 KB of operand stages
constexpr int T_BAR_OFF = T_STG_OFF + 4 * 2 * 4096;          // + two 4 KB staging boxes per epilogue warp
constexpr int T_SMEM_BYTES = T_BAR_OFF + 256 + 1024;
static_assert(T_SMEM_BYTES <= 232448, "shared memory");

struct TrailParams {
    int d_out, d_in, n_u;
    int c0, c1;          // the chunk whose errors are folded; columns >= c1 are updated
    int n_rt, n_ct;      // row tiles (batch * d_out / 128) and column tiles ((d_in - c1) / 128)
    int* err;
};

__global__ void __launch_bounds__(kThreads, 1)
gptq_trail(const __grid_constant__ CUtensorMap tmEhi, const __grid_constant__ CUtensorMap tmElo,
           const __grid_constant__ CUtensorMap tmUhi, const __grid_constant__ CUtensorMap tmUlo,
           const __grid_constant__ CUtensorMap tmWc, TrailParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + T_BAR_OFF);
    const uint32_t full0 = tc::smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * T_STAGES;
    const uint32_t tfull0 = empty0 + 8 * T_STAGES;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t drain = tempty0 + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * T_STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int total = p.n_rt * p.n_ct;
    const int nk = (p.c1 - p.c0) / KS;
    if (threadIdx.x == 0) {
        for (int st = 0; st < T_STAGES; ++st) {
            tc::mbar_init(full0 + 8 * st, 1);
            tc::mbar_init(empty0 + 8 * st, 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tfull0 + 8 * a, 1);
            tc::mbar_init(tempty0 + 8 * a, 128);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), 256);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            tc::prefetch_tmap(&tmEhi);
            tc::prefetch_tmap(&tmElo);
            tc::prefetch_tmap(&tmUhi);
            tc::prefetch_tmap(&tmUlo);
            int it = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x) {
                const int rt = w % p.n_rt, ct = w / p.n_rt;
                const int row0 = rt * R;
                const int u = (row0 / p.d_out) % p.n_u;
                const int ny = u * p.d_in + p.c1 + ct * BLK;   // rows n of the transposed factor
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int st = it % T_STAGES;
                    const uint32_t ph = (it / T_STAGES) & 1;
                    if (!tc::mbar_wait_bounded(empty0 + 8 * st, ph ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t fb = full0 + 8 * st;
                    tc::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t sa = tc::smem_u32(smem + st * STAGE_BYTES);
                    const int k0 = p.c0 + ks * KS;
                    tc::tma_load_2d(sa, &tmEhi, fb, k0, row0);
                    tc::tma_load_2d(sa + A_BYTES, &tmElo, fb, k0, row0);
                    tc::tma_load_2d(sa + 2 * A_BYTES, &tmUhi, fb, k0, ny);
                    tc::tma_load_2d(sa + 2 * A_BYTES + B_BYTES, &tmUlo, fb, k0, ny);
                }
            }
            if (!ok) {   // let the copies already issued land before the CTA can exit
                for (int j = it - 1; j >= 0 && j >= it - T_STAGES; --j)
                    tc::mbar_wait_bounded(full0 + 8 * (j % T_STAGES), (j / T_STAGES) & 1, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < total && ok; w += gridDim.x, ++tcount) {
                const int acc = tcount & 1;
                if (!tc::mbar_wait_bounded(tempty0 + 8 * acc, ((tcount >> 1) & 1) ^ 1, abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                const uint32_t d_tmem = tmem + acc * BLK;
                for (int ks = 0; ks < nk; ++ks, ++it) {
                    const int st = it % T_STAGES;
                    if (!tc::mbar_wait_bounded(full0 + 8 * st, (it / T_STAGES) & 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t ahi = tc::smem_u32(smem + st * STAGE_BYTES);
                    const uint32_t alo = ahi + A_BYTES, bhi = ahi + 2 * A_BYTES, blo = bhi + B_BYTES;
#pragma unroll
                    for (int kk = 0; kk < KS / 8; ++kk) {
                        const uint64_t dah = tc::sw128_desc(ahi + kk * 32, 16, 1024);
                        const uint64_t dal = tc::sw128_desc(alo + kk * 32, 16, 1024);
                        const uint64_t dbh = tc::sw128_desc(bhi + kk * 32, 16, 1024);
                        const uint64_t dbl = tc::sw128_desc(blo + kk * 32, 16, 1024);
                        tc::mma_tf32(d_tmem, dah, dbh, IDESC_LAZY, (ks | kk) != 0);
                        tc::mma_tf32(d_tmem, dah, dbl, IDESC_LAZY, 1);
                        tc::mma_tf32(d_tmem, dal, dbh, IDESC_LAZY, 1);
                    }
                    tc::mma_commit(empty0 + 8 * st);
                }
                if (!ok) break;
                tc::mma_commit(tfull0 + 8 * acc);
            }
        }
        __syncwarp();
    } else {
        // epilogue: each warp's 32 rows, 32 columns at a time, negated, 128-byte-swizzled into a staging
        // box and added into Wc by TMA reduce-add
        const int q = warp & 3;
        const uint32_t stg = tc::smem_u32(smem + T_STG_OFF) + q * 8192;
        int sb = 0, tcount = 0;
        for (int w = blockIdx.x; w < total; w += gridDim.x, ++tcount) {
            const int rt = w % p.n_rt, ct = w / p.n_rt;
            const int wrow = rt * R + q * 32;
            const int n0 = p.c1 + ct * BLK;
            const int acc = tcount & 1;
            if (!tc::mbar_wait_bounded(tfull0 + 8 * acc, (tcount >> 1) & 1, abort_flag)) break;
            tc::fence_after_sync();
#pragma unroll 1
            for (int ch = 0; ch < BLK / 32; ++ch) {
                uint32_t v[32];
                tc::tmem_ld_32x32b_x32(tmem + acc * BLK + ch * 32 + ((uint32_t)(q * 32) << 16), v);
                tc::tmem_wait_ld();
                const uint32_t buf = stg + sb * 4096;
                if (lane == 0) tc::bulk_wait_read<1>();   // the reduce that last used buf has read it
                __syncwarp();
#pragma unroll
                for (int j = 0; j < 8; ++j)
                    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                 ::"r"(buf + lane * 128 + ((j ^ (lane & 7)) << 4)), "r"(v[4 * j] ^ 0x80000000u),
                                 "r"(v[4 * j + 1] ^ 0x80000000u), "r"(v[4 * j + 2] ^ 0x80000000u),
                                 "r"(v[4 * j + 3] ^ 0x80000000u) : "memory");
                tc::fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) {
                    tc::tma_reduce_add_2d(&tmWc, buf, n0 + ch * 32, wrow);
                    tc::bulk_commit();
                }
                sb ^= 1;
            }
            tc::fence_before_sync();
            tc::mbar_arrive(tempty0 + 8 * acc);
        }
        if (lane == 0) tc::bulk_wait_all();
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1) {
        if (lane == 0) {
            tc::mma_commit(drain);
            tc::mbar_wait_bounded(drain, 0, abort_flag, 100000000ull);
        }
        __syncwarp();
        tc::fence_after_sync();
        tc::tmem_dealloc(tmem, 256);
    }
    if (threadIdx.x == 0 && *abort_flag) clha_record_error(p.err, CLHA_ERR_TIMEOUT, blockIdx.x, 0, KID_QUANTIZE);
}

// The running weights start as the weights themselves (float32).
__global__ void gptq_init_wc(const void* __restrict__ W, int w_f32, size_t n, float* __restrict__ Wc) {
    for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        Wc[i] = w_f32 ? reinterpret_cast<const float*>(W)[i]
                      : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[i]);
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
    return 2 * e + 2 * uu + (d_in > CHUNK ? e : 0);   // E hi/lo, U^T hi/lo, the running weights
}

cudaError_t launch_quantize(cudaStream_t s, int num_sms, const float* U, int n_u, const void* W, int w_is_f32,
                            int batch, int d_out, int d_in, int bits, uint8_t* codes, float* scales, uint8_t* zeros,
                            float* W_hat, const double* lambda, double* loss, void* ws, int* err, int form) {
    if (form != 0 && form != 1) return cudaErrorInvalidValue;
    char* cur = (char*)ws;
    const size_t wsz = (size_t)batch * d_out * d_in;
    float* Ehi = (float*)clha_carve(cur, wsz * sizeof(float));
    float* Elo = (float*)clha_carve(cur, wsz * sizeof(float));
    float* Uhi = (float*)clha_carve(cur, (size_t)batch * d_in * d_in * sizeof(float));
    float* Ulo = (float*)clha_carve(cur, (size_t)batch * d_in * d_in * sizeof(float));
    const bool chunked = d_in > CHUNK;
    float* Wc = chunked ? (float*)clha_carve(cur, wsz * sizeof(float)) : nullptr;
    cudaError_t e;
    CUtensorMap tEhi, tElo, tUhi, tUlo, tQhi, tQlo, tWc;
    if ((e = make_tmap_2d(&tEhi, Ehi, (uint64_t)batch * d_out, d_in, 4, R, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tElo, Elo, (uint64_t)batch * d_out, d_in, 4, R, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tUhi, Uhi, (uint64_t)n_u * d_in, d_in, 4, BLK, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tUlo, Ulo, (uint64_t)n_u * d_in, d_in, 4, BLK, KS)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tQhi, Uhi, (uint64_t)n_u * d_in, d_in, 4, 32, QW)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tQlo, Ulo, (uint64_t)n_u * d_in, d_in, 4, 32, QW)) != cudaSuccess) return e;
    if (chunked && (e = make_tmap_2d(&tWc, Wc, (uint64_t)batch * d_out, d_in, 4, 32, 32)) != cudaSuccess) return e;
    gptq_split_t<<<dim3(d_in / 32, d_in / 32, n_u), 256, 0, s>>>(U, d_in, Uhi, Ulo);
    clha_note_launches(1);
    if ((e = cudaFuncSetAttribute(gptq_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) != cudaSuccess)
        return e;
    if (chunked &&
        (e = cudaFuncSetAttribute(gptq_trail, cudaFuncAttributeMaxDynamicSharedMemorySize, T_SMEM_BYTES)) != cudaSuccess)
        return e;
    if (loss && (e = cudaMemsetAsync(loss, 0, (size_t)batch * sizeof(double), s)) != cudaSuccess) return e;
    if (chunked) {
        gptq_init_wc<<<4 * num_sms, 256, 0, s>>>(W, w_is_f32, wsz, Wc);
        clha_note_launches(1);
    }
    const int n_rt = (int)((size_t)batch * d_out / R);
    for (int c0 = 0; c0 < d_in; c0 += CHUNK) {
        const int c1 = c0 + CHUNK < d_in ? c0 + CHUNK : d_in;
        GptqParams p{U, n_u, W, w_is_f32, Wc, c0, c1, d_out, d_in, bits, codes, scales, zeros, W_hat, lambda, loss,
                     err, form};
        gptq_tc<<<dim3(d_out / R, batch), kThreads, SMEM_BYTES, s>>>(tEhi, tElo, tUhi, tUlo, tQhi, tQlo, p);
        clha_note_launches(1);
        if (c1 < d_in) {   // fold this chunk's errors into the running weights of every later column
            TrailParams tp{d_out, d_in, n_u, c0, c1, n_rt, (d_in - c1) / BLK, err};
            const int tiles = tp.n_rt * tp.n_ct;
            gptq_trail<<<tiles < num_sms ? tiles : num_sms, kThreads, T_SMEM_BYTES, s>>>(tEhi, tElo, tUhi, tUlo, tWc,
                                                                                       tp);
            clha_note_launches(1);
        }
    }
    return cudaGetLastError();
}
