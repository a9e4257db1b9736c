// Phase 1 of CLHA (the CLHA page, §2.2 (1)): per (layer, expert) Gram matrices S += X_e^T X_e of the
// tokens routed to the expert, plus their token counts; H = (2/n) S is formed at aggregation.
//
// bf16 inputs: a persistent, warp-specialised tcgen05 kernel (one CTA per SM).
//   warp 0     TMA producer: for an output tile (rows i0..i0+127, cols j0..j0+255) streams the
//              token blocks X[t0:t0+64, i0:i0+128] and X[t0:t0+64, j0:j0+256] into a 4-stage ring
//              (128-byte swizzle; both operands are "M/N-major": one token row = 64 contiguous
//              channels, which is how X is laid out, so no transpose is ever materialised).
//   warp 1     MMA issuer: tcgen05.mma kind::f16 M=128 N=256 K=16, four per 64-token block,
//              accumulating in TMEM one chunk of at most 2048 (d < 8192) or 8192 tokens at a time; two accumulators
//              (512 TMEM columns) so the epilogue of one chunk overlaps the MMAs of the next.
//   warps 2-5  epilogue: tcgen05.ld of the fp32 chunk sum, one 32x32 sub-tile per warp at a time
//              written to a swizzled shared-memory buffer (two per warp) and added into S by a TMA
//              bulk reduce (the L2 performs the fp32 adds), so the epilogue never reads S.
// Why chunks: the tensor core's fp32 accumulation does not round to nearest, and over tens of
// thousands of tokens the Gram diagonal (a sum of positive terms) drifts low by a few 1e-4
// relative. Summing at most one chunk of tokens per accumulator and adding the chunk sums into S with
// round-to-nearest fp32 adds bounds that drift by the chunk length instead of the token count.
// Only tiles that touch the upper triangle are computed (rows tile r <= 2c+1 for column tile c);
// entries below the diagonal inside those tiles are correct values but the upper triangle is the
// authoritative one. Segments from the gather are 128-row aligned with zero padding, so a token
// block never mixes experts and padding adds nothing.
// float32 inputs: a plain shared-memory tiled FMA kernel (used by the small fp32 workload).
#include "clha_internal.h"
#include "tc_ptx.h"
#include "tmap.h"

namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int kPairMinD = 4096;   // one dense Gram with d at least this runs on pairs of SMs (syrk_bf16_pair)
// 64-token blocks per TMEM accumulation. The tensor core's fp32 accumulator does not round each add
// to nearest, so a long sum drifts (linearly in its length); chunk sums are added into S by TMA
// reduce-add, which rounds to nearest. Short chunks where the Hessian is small (an expert's d_model or
// d_ff: cheap extra epilogues, and the experts' Hessians feed GPTQ on rank-deficient, ill-conditioned
// problems), long ones for large d (each chunk's epilogue moves a whole 128x256 fp32 tile).
constexpr int KCHUNK_BLOCKS_SMALL_D = 32;     // 2048 tokens, d < 8192
constexpr int KCHUNK_BLOCKS_LARGE_D = 128;    // 8192 tokens, d >= 8192
__host__ __device__ constexpr int kchunk_blocks(int d) { return d < 8192 ? KCHUNK_BLOCKS_SMALL_D : KCHUNK_BLOCKS_LARGE_D; }
constexpr int A_BYTES = BM * BK * 2;
constexpr int B_BYTES = BN * BK * 2;
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int STG_OFF = STAGES * STAGE_BYTES + 1024;   // after the barriers, 1024-aligned for the swizzle
constexpr int STG_BYTES = 4 * 2 * 32 * 32 * 4;         // 4 epilogue warps x 2 buffers x 32x32 fp32
constexpr int SMEM_BYTES = STG_OFF + STG_BYTES + 1024;  // + alignment slack of the dynamic base
constexpr int kThreads = 192;
constexpr uint32_t IDESC = tc::idesc_f32acc(1 /*bf16*/, 1 /*A MN-major*/, 1 /*B MN-major*/, BM, BN);

struct SyrkParams {
    int d;
    int64_t rows;
    const int32_t* perm;   // gathered operands: token of each packed row (-1: padding), else null
    const int64_t* seg;
    int E;
    float* S;
    int tiles_per_slot;
    int nr, nc;
    int total_tiles;
    int* err;
};

__device__ __forceinline__ void decode_tile(int t, int nr, int nc, int& r, int& c) {
    r = 0;
    for (c = 0; c < nc; ++c) {
        int m = min(nr, 2 * c + 2);
        if (t < m) { r = t; return; }
        t -= m;
    }
}

__device__ __forceinline__ void slot_range(const SyrkParams& p, int e, int64_t& t0, int64_t& cnt) {
    if (p.seg) { t0 = p.seg[e]; cnt = p.seg[p.E + 1 + e]; }
    else { t0 = 0; cnt = p.rows; }
}

// kGather: the operands come straight from the token matrix X [rows, d]: packed row q of a segment is
// token perm[q], fetched four rows at a time by TMA gather4 (a padding row, perm -1, is a row index
// past the end and reads zeros), so the routed rows are never copied out of X.
template <bool kGather>
__global__ void __launch_bounds__(kThreads, 1) syrk_bf16_tc(const __grid_constant__ CUtensorMap tmX,
                                                            const __grid_constant__ CUtensorMap tmS, SyrkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    const uint32_t full0 = tc::smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * STAGES;
    const uint32_t tfull0 = full0 + 16 * STAGES;
    const uint32_t tempty0 = tfull0 + 16;
    const uint32_t drain = tfull0 + 32;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(full0 + 8 * s, 1);
            tc::mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tfull0 + 8 * a, 1);
            tc::mbar_init(tempty0 + 8 * a, 128);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&tmX);
        tc::prefetch_tmap(&tmS);
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0 && kGather) {
        // all 32 lanes issue: lane l fetches rows 4g .. 4g+3 (g = l % 16) of the 64-token block for
        // boxes l / 16, l / 16 + 2, l / 16 + 4 (boxes 0-1: the A columns, 2-5: the B columns)
        int it = 0;
        bool ok = true;
        const int g = lane & 15;
        const int oob = (int)p.rows;   // a row index past the end: zeros
        for (int w = blockIdx.x; w < p.total_tiles && ok; w += gridDim.x) {
            const int e = w / p.tiles_per_slot;
            int r, c;
            decode_tile(w % p.tiles_per_slot, p.nr, p.nc, r, c);
            int64_t t0, cnt;
            slot_range(p, e, t0, cnt);
            const int nk = (int)((cnt + BK - 1) / BK);
            // this lane's four token indices of blocks kb + 1 and kb + 2 are loaded ahead, so the
            // index loads overlap the wait for a free stage and the copies of block kb
            const int4* pq = reinterpret_cast<const int4*>(p.perm + t0 + 4 * g);
            int4 tk1 = nk > 0 ? pq[0] : make_int4(-1, -1, -1, -1);
            int4 tk2 = nk > 1 ? pq[BK / 4] : make_int4(-1, -1, -1, -1);
            for (int kb = 0; kb < nk; ++kb, ++it) {
                const int4 tk = tk1;
                tk1 = tk2;
                if (kb + 2 < nk) tk2 = pq[(int64_t)(kb + 2) * (BK / 4)];
                const int s = it % STAGES;
                const uint32_t ph = (it / STAGES) & 1;
                int got = 1;
                if (lane == 0) got = tc::mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag) ? 1 : 0;
                got = __shfl_sync(0xffffffffu, got, 0);
                if (!got) { ok = false; break; }
                const uint32_t fb = full0 + 8 * s;
                if (lane == 0) tc::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                __syncwarp();
                const uint32_t a_dst = tc::smem_u32(smem + s * STAGE_BYTES);
                const uint32_t b_dst = a_dst + A_BYTES;
                const int r0 = tk.x < 0 ? oob : tk.x, r1 = tk.y < 0 ? oob : tk.y;
                const int r2 = tk.z < 0 ? oob : tk.z, r3 = tk.w < 0 ? oob : tk.w;
#pragma unroll
                for (int hh = 0; hh < 3; ++hh) {
                    const int h = (lane >> 4) + 2 * hh;
                    const uint32_t dst = (h < 2 ? a_dst + h * 8192 : b_dst + (h - 2) * 8192) + g * 512;
                    const int x = h < 2 ? r * BM + h * 64 : c * BN + (h - 2) * 64;
                    tc::tma_gather4_2d(dst, &tmX, fb, x, r0, r1, r2, r3);
                }
            }
        }
        if (!ok && lane == 0) {  // let the copies already issued land before the CTA can exit
            for (int j = it - 1; j >= 0 && j >= it - STAGES; --j)
                tc::mbar_wait_bounded(full0 + 8 * (j % STAGES), (j / STAGES) & 1, abort_flag, 100000000ull);
        }
        __syncwarp();
    } else if (warp == 0) {
        if (lane == 0) {
            int it = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < p.total_tiles && ok; w += gridDim.x) {
                const int e = w / p.tiles_per_slot;
                int r, c;
                decode_tile(w % p.tiles_per_slot, p.nr, p.nc, r, c);
                int64_t t0, cnt;
                slot_range(p, e, t0, cnt);
                const int nk = (int)((cnt + BK - 1) / BK);
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    const uint32_t ph = (it / STAGES) & 1;
                    if (!tc::mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t fb = full0 + 8 * s;
                    tc::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t a_dst = tc::smem_u32(smem + s * STAGE_BYTES);
                    const uint32_t b_dst = a_dst + A_BYTES;
                    const int y = (int)(t0 + (int64_t)kb * BK);
#pragma unroll
                    for (int h = 0; h < BM / 64; ++h) tc::tma_load_2d(a_dst + h * 8192, &tmX, fb, r * BM + h * 64, y);
#pragma unroll
                    for (int h = 0; h < BN / 64; ++h) tc::tma_load_2d(b_dst + h * 8192, &tmX, fb, c * BN + h * 64, y);
                }
            }
            if (!ok) {  // let the copies already issued land before the CTA can exit
                for (int j = it - 1; j >= 0 && j >= it - STAGES; --j)
                    tc::mbar_wait_bounded(full0 + 8 * (j % STAGES), (j / STAGES) & 1, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true;
            for (int w = blockIdx.x; w < p.total_tiles && ok; w += gridDim.x) {
                const int e = w / p.tiles_per_slot;
                int64_t t0, cnt;
                slot_range(p, e, t0, cnt);
                const int nk = (int)((cnt + BK - 1) / BK);
                for (int kc = 0; kc < nk && ok; kc += kchunk_blocks(p.d)) {
                    const int kend = min(nk, kc + kchunk_blocks(p.d));
                    const int acc = tcount & 1;
                    const uint32_t aph = (tcount >> 1) & 1;
                    if (!tc::mbar_wait_bounded(tempty0 + 8 * acc, aph ^ 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t d_tmem = tmem + acc * BN;
                    for (int kb = kc; kb < kend; ++kb, ++it) {
                        const int s = it % STAGES;
                        const uint32_t ph = (it / STAGES) & 1;
                        if (!tc::mbar_wait_bounded(full0 + 8 * s, ph, abort_flag)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint32_t a_base = tc::smem_u32(smem + s * STAGE_BYTES);
                        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = tc::sw128_desc(a_base + kk * 2048, 8192, 1024);
                            const uint64_t bd = tc::sw128_desc(b_base + kk * 2048, 8192, 1024);
                            tc::mma_f16(d_tmem, ad, bd, IDESC, ((kb - kc) | kk) != 0);
                        }
                        tc::mma_commit(empty0 + 8 * s);
                    }
                    if (!ok) break;
                    tc::mma_commit(tfull0 + 8 * acc);
                    ++tcount;
                }
            }
        }
        __syncwarp();
    } else {
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const uint32_t stg = tc::smem_u32(smem + STG_OFF) + q * 8192;
        int sb = 0;
        int tcount = 0;
        for (int w = blockIdx.x; w < p.total_tiles; w += gridDim.x) {
            const int e = w / p.tiles_per_slot;
            int r, c;
            decode_tile(w % p.tiles_per_slot, p.nr, p.nc, r, c);
            int64_t t0, cnt;
            slot_range(p, e, t0, cnt);
            const int nk = (int)((cnt + BK - 1) / BK);
            const int warp_row_min = r * BM + q * 32;
            const int srow = e * p.d + warp_row_min;  // row of this warp's sub-tiles in the [E*d, d] view
            bool ok = true;
            for (int kc = 0; kc < nk; kc += kchunk_blocks(p.d)) {
                const int acc = tcount & 1;
                const uint32_t aph = (tcount >> 1) & 1;
                if (!tc::mbar_wait_bounded(tfull0 + 8 * acc, aph, abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll 1
                for (int ch = 0; ch < BN / 32; ++ch) {
                    const int col0 = c * BN + ch * 32;
                    if (col0 >= p.d) break;
                    if (col0 + 31 < warp_row_min) continue;  // whole sub-tile strictly below the diagonal
                    uint32_t v[32];
                    tc::tmem_ld_32x32b_x32(tmem + acc * BN + ch * 32 + ((uint32_t)(q * 32) << 16), v);
                    tc::tmem_wait_ld();
                    const uint32_t buf = stg + sb * 4096;
                    if (lane == 0) tc::bulk_wait_read<1>();  // the reduce that last used buf has read it
                    __syncwarp();
                    // row `lane` of the box; 16-byte chunk j sits at j ^ (row % 8) (128-byte swizzle)
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     ::"r"(buf + lane * 128 + ((j ^ (lane & 7)) << 4)), "r"(v[4 * j]),
                                     "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3]) : "memory");
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tc::tma_reduce_add_2d(&tmS, buf, col0, srow);
                        tc::bulk_commit();
                    }
                    sb ^= 1;
                }
                tc::fence_before_sync();
                tc::mbar_arrive(tempty0 + 8 * acc);
                ++tcount;
            }
            if (!ok) break;
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
        tc::tmem_dealloc(tmem, 512);
    }
    if (threadIdx.x == 0 && *abort_flag) clha_record_error(p.err, CLHA_ERR_TIMEOUT, blockIdx.x, 0, KID_COLLECT);
}

// ------------------------------------------------------------------------------ pairs of SMs
// The dense Gram at large d on CTA pairs (a cluster of two CTAs sharing each tcgen05.mma,
// cta_group::2): output tiles of 256 x 256, CTA k of a pair holding rows 128k .. 128k+127 of the tile
// (its half of A) and columns 128k .. 128k+127 (its half of B) in its shared memory, and its 128 rows
// of each accumulator in its TMEM. For the same tensor-core work a stage then carries 32 KB per SM
// instead of 48 KB, so six stages fit against four, and each SM's TMA traffic per flop falls by a
// third. Roles as in syrk_bf16_tc, on both CTAs, except that only the leader (rank 0) issues MMAs
// (M = 256, N = 256) and waits on the operand barriers, which count both CTAs' copies; its commits
// reach both CTAs' stage and accumulator barriers (multicast), and both CTAs' epilogue warps arrive
// on the leader's accumulator-empty barrier. Tile rows at or past d (the second half of the last row
// tile when d is not a multiple of 256) are computed on zero-filled operands and never written.
constexpr int P_STAGES = 6;
constexpr int P_HALF = 128;                      // rows of A and columns of B per CTA
constexpr int P_A_BYTES = P_HALF * BK * 2;       // 16 KB
constexpr int P_STAGE_BYTES = 2 * P_A_BYTES;     // A half + B half
constexpr int P_BAR_OFF = P_STAGES * P_STAGE_BYTES;
constexpr int P_STG_OFF = P_BAR_OFF + 1024;
constexpr int P_SMEM_BYTES = P_STG_OFF + STG_BYTES + 1024;
constexpr int P_TILE = 256;
constexpr uint32_t IDESC_PAIR = tc::idesc_f32acc(1 /*bf16*/, 1 /*A MN-major*/, 1 /*B MN-major*/, 256, 256);
static_assert(P_SMEM_BYTES <= 232448, "shared memory");

// Pair tiles in bands of 8 tile columns, row-major inside a band: the pairs working at one time share
// about sqrt(pairs) row blocks and 8 column blocks of X, so a block is read from DRAM once for several
// tiles (on 65536 x 28672, 163 GB of DRAM reads per call against 232 GB column after column).
__device__ __forceinline__ void decode_pair_tile(int t, int& R, int& C, int nC) {
    constexpr int WB = 8;
    int cmin = 0, cmax = 0;
    for (;;) {
        cmax = min(nC, cmin + WB) - 1;
        const int nb = (cmax + 1) * (cmax + 2) / 2 - cmin * (cmin + 1) / 2;
        if (t < nb) break;
        t -= nb;
        cmin += WB;
    }
    for (R = 0;; ++R) {
        const int c0 = max(R, cmin);
        const int cnt = cmax - c0 + 1;
        if (t < cnt) { C = c0 + t; return; }
        t -= cnt;
    }
}

__global__ void __launch_bounds__(kThreads, 1) syrk_bf16_pair(const __grid_constant__ CUtensorMap tmX,
                                                              const __grid_constant__ CUtensorMap tmS, SyrkParams p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + P_BAR_OFF);
    const uint32_t full0 = tc::smem_u32(bars);            // [P_STAGES] leader: both CTAs' copies of a stage
    const uint32_t empty0 = full0 + 8 * P_STAGES;         // [P_STAGES] each CTA: its stage may be refilled
    const uint32_t tfull0 = empty0 + 8 * P_STAGES;        // [2] each CTA: an accumulator holds a finished chunk
    const uint32_t tempty0 = tfull0 + 16;                 // [2] leader: both CTAs' epilogues are done with it
    const uint32_t drain = tempty0 + 16;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * P_STAGES + 5);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    const uint32_t rank = tc::cluster_ctarank();
    const bool leader = rank == 0;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
    const int nk = (int)((p.rows + BK - 1) / BK);
    const int kcb = kchunk_blocks(p.d);
    if (threadIdx.x == 0) {
        for (int s = 0; s < P_STAGES; ++s) {
            tc::mbar_init(full0 + 8 * s, 1);
            tc::mbar_init(empty0 + 8 * s, 1);
        }
        for (int a = 0; a < 2; ++a) {
            tc::mbar_init(tfull0 + 8 * a, 1);
            tc::mbar_init(tempty0 + 8 * a, 8);   // one arrival per epilogue warp of either CTA
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
        tc::prefetch_tmap(&tmX);
        tc::prefetch_tmap(&tmS);
    }
    if (warp == 1) tc::tmem_alloc_pair(tc::smem_u32(tmem_slot), 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::cluster_sync();   // both CTAs' barriers exist before any copy or arrival reaches them
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        if (lane == 0) {
            const uint32_t full_leader = tc::mapa_shared(full0, 0);
            int it = 0;
            bool ok = true;
            for (int w = pair; w < p.total_tiles && ok; w += npairs) {
                int R, C;
                decode_pair_tile(w, R, C, p.nc);
                const int ra = R * P_TILE + (int)rank * P_HALF, cb = C * P_TILE + (int)rank * P_HALF;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % P_STAGES;
                    const uint32_t ph = (it / P_STAGES) & 1;
                    if (!tc::mbar_wait_bounded(empty0 + 8 * s, ph ^ 1, abort_flag)) { ok = false; break; }
                    if (leader) tc::mbar_arrive_expect_tx(full0 + 8 * s, 2 * P_STAGE_BYTES);
                    const uint32_t fb = full_leader + 8 * s;
                    const uint32_t a_dst = tc::smem_u32(smem + s * P_STAGE_BYTES);
                    const uint32_t b_dst = a_dst + P_A_BYTES;
                    const int y = kb * BK;
#pragma unroll
                    for (int h = 0; h < P_HALF / 64; ++h) tc::tma_load_2d_pair(a_dst + h * 8192, &tmX, fb, ra + h * 64, y);
#pragma unroll
                    for (int h = 0; h < P_HALF / 64; ++h) tc::tma_load_2d_pair(b_dst + h * 8192, &tmX, fb, cb + h * 64, y);
                }
            }
            if (!ok && leader) {  // the copies already issued (both CTAs') land before either CTA can exit
                for (int j = it - 1; j >= 0 && j >= it - P_STAGES; --j)
                    tc::mbar_wait_bounded(full0 + 8 * (j % P_STAGES), (j / P_STAGES) & 1, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0 && leader) {
            int it = 0, tcount = 0;
            bool ok = true;
            for (int w = pair; w < p.total_tiles && ok; w += npairs) {
                for (int kc = 0; kc < nk && ok; kc += kcb) {
                    const int kend = min(nk, kc + kcb);
                    const int acc = tcount & 1;
                    const uint32_t aph = (tcount >> 1) & 1;
                    if (!tc::mbar_wait_bounded(tempty0 + 8 * acc, aph ^ 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t d_tmem = tmem + acc * P_TILE;
                    for (int kb = kc; kb < kend; ++kb, ++it) {
                        const int s = it % P_STAGES;
                        const uint32_t ph = (it / P_STAGES) & 1;
                        if (!tc::mbar_wait_bounded(full0 + 8 * s, ph, abort_flag)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint32_t a_base = tc::smem_u32(smem + s * P_STAGE_BYTES);
                        const uint32_t b_base = a_base + P_A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = tc::sw128_desc(a_base + kk * 2048, 8192, 1024);
                            const uint64_t bd = tc::sw128_desc(b_base + kk * 2048, 8192, 1024);
                            tc::mma_f16_pair(d_tmem, ad, bd, IDESC_PAIR, ((kb - kc) | kk) != 0);
                        }
                        tc::mma_commit_pair(empty0 + 8 * s, 0x3);
                    }
                    if (!ok) break;
                    tc::mma_commit_pair(tfull0 + 8 * acc, 0x3);
                    ++tcount;
                }
            }
        }
        __syncwarp();
    } else {
        const int q = warp & 3;  // TMEM lane quadrant this warp may access
        const uint32_t stg = tc::smem_u32(smem + P_STG_OFF) + q * 8192;
        const uint32_t tempty_leader = tc::mapa_shared(tempty0, 0);
        int sb = 0;
        int tcount = 0;
        for (int w = pair; w < p.total_tiles; w += npairs) {
            int R, C;
            decode_pair_tile(w, R, C, p.nc);
            const int warp_row_min = R * P_TILE + (int)rank * P_HALF + q * 32;
            bool ok = true;
            for (int kc = 0; kc < nk; kc += kcb) {
                const int acc = tcount & 1;
                const uint32_t aph = (tcount >> 1) & 1;
                if (!tc::mbar_wait_bounded(tfull0 + 8 * acc, aph, abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
#pragma unroll 1
                for (int ch = 0; ch < P_TILE / 32 && warp_row_min < p.d; ++ch) {
                    const int col0 = C * P_TILE + ch * 32;
                    if (col0 >= p.d) break;
                    if (col0 + 31 < warp_row_min) continue;  // whole sub-tile strictly below the diagonal
                    uint32_t v[32];
                    tc::tmem_ld_32x32b_x32(tmem + acc * P_TILE + ch * 32 + ((uint32_t)(q * 32) << 16), v);
                    tc::tmem_wait_ld();
                    const uint32_t buf = stg + sb * 4096;
                    if (lane == 0) tc::bulk_wait_read<1>();  // the reduce that last used buf has read it
                    __syncwarp();
#pragma unroll
                    for (int j = 0; j < 8; ++j)
                        asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};"
                                     ::"r"(buf + lane * 128 + ((j ^ (lane & 7)) << 4)), "r"(v[4 * j]),
                                     "r"(v[4 * j + 1]), "r"(v[4 * j + 2]), "r"(v[4 * j + 3]) : "memory");
                    tc::fence_proxy_async_smem();
                    __syncwarp();
                    if (lane == 0) {
                        tc::tma_reduce_add_2d(&tmS, buf, col0, warp_row_min);
                        tc::bulk_commit();
                    }
                    sb ^= 1;
                }
                tc::fence_before_sync();
                __syncwarp();
                if (lane == 0) tc::mbar_arrive_cluster(tempty_leader + 8 * acc);
                ++tcount;
            }
            if (!ok) break;
        }
        if (lane == 0) tc::bulk_wait_all();
        __syncwarp();
    }

    __syncthreads();
    if (warp == 1 && leader) {
        if (lane == 0) {
            tc::mma_commit_pair(drain, 0x1);
            tc::mbar_wait_bounded(drain, 0, abort_flag, 100000000ull);
        }
        __syncwarp();
    }
    tc::fence_before_sync();
    tc::cluster_sync();   // the leader's last products (which read both CTAs' shared memory) are done
    tc::fence_after_sync();
    if (warp == 1) tc::tmem_dealloc_pair(tmem, 512);
    if (threadIdx.x == 0 && *abort_flag) clha_record_error(p.err, CLHA_ERR_TIMEOUT, blockIdx.x, 0, KID_COLLECT);
}

__global__ void add_counts(int64_t* counts, const int64_t* seg, int E, int64_t rows) {
    int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < E) counts[e] += seg ? seg[E + 1 + e] : rows;
}

// ------------------------------------------------------------------------------ float32 inputs
constexpr int FT = 64, FK = 32;

__global__ void __launch_bounds__(256) syrk_f32_simt(const float* __restrict__ X, int64_t rows, int d,
                                                     const int64_t* __restrict__ seg, int E, float* __restrict__ S) {
    // blockIdx.x: upper tile index (r <= c) in row-major order over the tile grid; blockIdx.y: slot
    const int nt = d / FT;
    int t = blockIdx.x, r = 0;
    while (t >= nt - r) { t -= nt - r; ++r; }
    const int c = r + t;
    const int e = blockIdx.y;
    int64_t t0 = 0, cnt = rows;
    if (seg) { t0 = seg[e]; cnt = seg[E + 1 + e]; }
    __shared__ float As[FK][FT + 4];
    __shared__ float Bs[FK][FT + 4];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    float acc[4][4] = {};
    for (int64_t k0 = 0; k0 < cnt; k0 += FK) {
        for (int i = threadIdx.x; i < FK * FT; i += 256) {
            int kk = i / FT, m = i % FT;
            bool in = k0 + kk < cnt;
            const float* xr = X + (t0 + k0 + kk) * (int64_t)d;
            As[kk][m] = in ? xr[r * FT + m] : 0.f;
            Bs[kk][m] = in ? xr[c * FT + m] : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < FK; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; b[i] = Bs[kk][tx * 4 + i]; }
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
        }
        __syncthreads();
    }
    float* Se = S + (size_t)e * d * d;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) Se[(size_t)(r * FT + ty * 4 + i) * d + c * FT + tx * 4 + j] += acc[i][j];
}

}  // namespace

cudaError_t launch_collect_bf16(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d,
                                const int64_t* seg, int E, float* S_base, int64_t* counts_base, int* err) {
    CUtensorMap tm, tmS;
    cudaError_t e = make_tmap_2d(&tm, X, (uint64_t)rows, (uint64_t)d, 2, 64, 64);
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&tmS, S_base, (uint64_t)E * d, (uint64_t)d, 4, 32, 32);
    if (e != cudaSuccess) return e;
    // per call: the attribute belongs to the current device's context (a process may drive several)
    e = cudaFuncSetAttribute(syrk_bf16_tc<false>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    SyrkParams p;
    p.d = d;
    p.rows = rows;
    p.perm = nullptr;
    p.seg = seg;
    p.E = E;
    p.S = S_base;
    p.err = err;
    if (!seg && E == 1 && d >= kPairMinD) {   // one dense Gram at large d: pairs of SMs
        e = cudaFuncSetAttribute(syrk_bf16_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, P_SMEM_BYTES);
        if (e != cudaSuccess) return e;
        const int nC = (d + P_TILE - 1) / P_TILE;
        p.nr = p.nc = nC;
        p.tiles_per_slot = p.total_tiles = nC * (nC + 1) / 2;
        int npairs = num_sms / 2;
        if (npairs > p.total_tiles) npairs = p.total_tiles;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3((unsigned)(2 * npairs));
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = P_SMEM_BYTES;
        cfg.stream = s;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int max_clusters = 0;
        if (cudaOccupancyMaxActiveClusters(&max_clusters, syrk_bf16_pair, &cfg) == cudaSuccess && max_clusters > 0 &&
            max_clusters < npairs) {
            npairs = max_clusters;
            cfg.gridDim = dim3((unsigned)(2 * npairs));
        }
        e = cudaLaunchKernelEx(&cfg, syrk_bf16_pair, tm, tmS, p);
        if (e != cudaSuccess) return e;
        clha_note_launches(1);
    } else {
        p.nr = d / BM;
        p.nc = (d + BN - 1) / BN;
        p.tiles_per_slot = 0;
        for (int c = 0; c < p.nc; ++c) p.tiles_per_slot += (p.nr < 2 * c + 2) ? p.nr : 2 * c + 2;
        p.total_tiles = p.tiles_per_slot * E;
        int grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
        syrk_bf16_tc<false><<<grid, kThreads, SMEM_BYTES, s>>>(tm, tmS, p);
        clha_note_launches(1);
    }
    add_counts<<<(E + 255) / 256, 256, 0, s>>>(counts_base, seg, E, rows);
    clha_note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_collect_bf16_gathered(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t n, int d,
                                         const int32_t* perm, const int64_t* seg, int E, float* S_base,
                                         int64_t* counts_base, int* err) {
    CUtensorMap tm, tmS;
    cudaError_t e = make_tmap_2d(&tm, X, (uint64_t)n, (uint64_t)d, 2, 1, 64);   // gather4: one-row box
    if (e != cudaSuccess) return e;
    e = make_tmap_2d(&tmS, S_base, (uint64_t)E * d, (uint64_t)d, 4, 32, 32);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(syrk_bf16_tc<true>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    SyrkParams p;
    p.d = d;
    p.rows = n;
    p.perm = perm;
    p.seg = seg;
    p.E = E;
    p.S = S_base;
    p.nr = d / BM;
    p.nc = (d + BN - 1) / BN;
    p.tiles_per_slot = 0;
    for (int c = 0; c < p.nc; ++c) p.tiles_per_slot += (p.nr < 2 * c + 2) ? p.nr : 2 * c + 2;
    p.total_tiles = p.tiles_per_slot * E;
    p.err = err;
    int grid = p.total_tiles < num_sms ? p.total_tiles : num_sms;
    syrk_bf16_tc<true><<<grid, kThreads, SMEM_BYTES, s>>>(tm, tmS, p);
    clha_note_launches(1);
    add_counts<<<(E + 255) / 256, 256, 0, s>>>(counts_base, seg, E, n);
    clha_note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_collect_f32(cudaStream_t s, const float* X, int64_t rows, int d, const int64_t* seg, int E,
                               float* S_base, int64_t* counts_base) {
    int nt = d / FT;
    dim3 grid(nt * (nt + 1) / 2, E);
    syrk_f32_simt<<<grid, 256, 0, s>>>(X, rows, d, seg, E, S_base);
    clha_note_launches(1);
    add_counts<<<(E + 255) / 256, 256, 0, s>>>(counts_base, seg, E, rows);
    clha_note_launches(1);
    return cudaGetLastError();
}
