// Expert FFN activation on the tensor cores: h = SiLU(x Wg^T) * (x Wu^T), bf16 out, for inputs whose
// channels all have a similar dynamic range (clha_expert_act chooses this kernel or the fp32-FMA one
// per call from the rows' channel magnitudes; see launch_expert_act).
//
// A persistent, warp-specialised tcgen05 kernel (one CTA per SM); an output tile is 128 rows x 32
// h-columns:
//   warp 0     TMA producer: per 64-wide k step, the 128 token rows of X and the 32 gate rows plus the
//              32 up rows of the tile's expert (stacked into one 64-row operand), both K-major.
//   warp 1     MMA issuer: tcgen05.mma kind::f16 (bf16 in, fp32 accumulate) M=128 N=64 K=16, so one
//              MMA produces the gate and the up pre-activations side by side. K is cut into up to 8
//              chunks, each accumulated into its own 64 TMEM columns and handed over as soon as it is
//              done, so the epilogue reads chunk c while chunk c+1 runs.
//   warps 2-17 epilogue, four warps per TMEM lane quadrant, each a quarter of the tile's columns: the chunk
//              sums are added in fp64, h = SiLU(g) * u is evaluated in fp64 and rounded once to bf16
//              (as the fp32-FMA kernel does).
// Products of bf16 values are exact, but the tensor core adds a group's products after aligning them
// to the largest, so a group that holds a product from an outlier channel (tens of times the others)
// loses low bits of the rest: with such channels the bf16 rounding of h flips often enough to move the
// down-projection Hessian past 1e-4 relative, which is why the fp32-FMA kernel takes those inputs.
// A tile's expert comes from the segment table (segments are 128-row aligned, so a tile never mixes
// experts).
#include "clha_internal.h"
#include "tc_ptx.h"
#include "tmap.h"

namespace {

constexpr int BM = 128, BNH = 32, BK = 64, STAGES = 6, NCH = 8;
constexpr int A_BYTES = BM * BK * 2;            // 16 KB
constexpr int B_BYTES = 2 * BNH * BK * 2;       // 8 KB (gate rows then up rows)
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int BAR_BYTES = 8 * (2 * STAGES + 2 * NCH + 1) + 16;
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + 1024 + BAR_BYTES;
constexpr int kThreads = 576;                   // producer, MMA issuer, 16 epilogue warps
constexpr int EPI = 512;                         // epilogue threads
constexpr uint32_t IDESC = tc::idesc_f32acc(1 /*bf16*/, 0 /*K-major*/, 0 /*K-major*/, BM, 2 * BNH);

struct ActParams {
    const int* sel;        // null: run (no outlier channels taken out); else run when *sel is 1 or 2, and
                           // with *sel == 2 multiply the masked weights and add the outlier channels' terms
    int64_t rows;          // rows of X and h
    int dm, dff;
    const int64_t* seg;    // null: one expert, all rows valid
    int E;
    __nv_bfloat16* h;
    int n_tiles_n;         // dff / 32
    const int* out_n;      // outlier channels (sel == 2)
    const float* xo;       // [rows][kMaxOutliers] the rows' outlier channels
    const float* wo;       // [E][2][kMaxOutliers][dff] their gate and up weights
    int* err;
};

__device__ __forceinline__ int find_segment(const int64_t* seg, int E, int64_t row) {
    int lo = 0, hi = E - 1;
    while (lo < hi) {  // last e with seg[e] <= row
        int mid = (lo + hi + 1) >> 1;
        if (seg[mid] <= row) lo = mid; else hi = mid - 1;
    }
    return lo;
}

// (m-tile, n-tile, expert, end of the expert's valid rows) of work item w; false past the last tile
__device__ __forceinline__ bool decode(const ActParams& p, int64_t m_tiles, int64_t w, int64_t& m0, int& n0, int& e,
                                       int64_t& vend) {
    if (w >= m_tiles * p.n_tiles_n) return false;
    m0 = (w / p.n_tiles_n) * BM;
    n0 = (int)(w % p.n_tiles_n) * BNH;
    if (p.seg) {
        e = find_segment(p.seg, p.E, m0);
        vend = p.seg[e] + p.seg[p.E + 1 + e];
    } else {
        e = 0;
        vend = p.rows;
    }
    return true;
}

__global__ void __launch_bounds__(kThreads, 1)
expert_act_tc(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmWg,
       const __grid_constant__ CUtensorMap tmWu, const __grid_constant__ CUtensorMap tmWgm,
       const __grid_constant__ CUtensorMap tmWum, ActParams p) {
    const int selv = p.sel ? *p.sel : 1;
    if (selv == 0) return;              // the fp32-FMA kernel takes this call (uniform: before any setup)
    const bool masked = selv == 2;      // outlier channels: zeroed in the weights the tensor cores read
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES);
    const uint32_t full0 = tc::smem_u32(bars);
    const uint32_t empty0 = full0 + 8 * STAGES;
    const uint32_t cfull0 = empty0 + 8 * STAGES;      // chunk c of the accumulator is complete
    const uint32_t cempty0 = cfull0 + 8 * NCH;        // chunk c has been read by the epilogue
    const uint32_t drain = cempty0 + 8 * NCH;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 2 * NCH + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < STAGES; ++s) {
            tc::mbar_init(full0 + 8 * s, 1);
            tc::mbar_init(empty0 + 8 * s, 1);
        }
        for (int c = 0; c < NCH; ++c) {
            tc::mbar_init(cfull0 + 8 * c, 1);
            tc::mbar_init(cempty0 + 8 * c, EPI);
        }
        tc::mbar_init(drain, 1);
        *abort_flag = 0;
        tc::fence_barrier_init();
    }
    if (warp == 1) tc::tmem_alloc(tc::smem_u32(tmem_slot), 512);
    tc::fence_before_sync();
    __syncthreads();
    tc::fence_after_sync();
    const uint32_t tmem = *tmem_slot;

    const int64_t used_rows = p.seg ? p.seg[p.E] : p.rows;
    const int64_t m_tiles = (used_rows + BM - 1) / BM;
    const int nk = p.dm / BK;                      // >= 2
    const int nch = nk < NCH ? nk : NCH;           // chunks per tile
    // chunk c covers k steps [c*nk/nch, (c+1)*nk/nch)

    if (warp == 0) {
        if (lane == 0) {
            const CUtensorMap* mg = masked ? &tmWgm : &tmWg;
            const CUtensorMap* mu = masked ? &tmWum : &tmWu;
            tc::prefetch_tmap(&tmX);
            tc::prefetch_tmap(mg);
            tc::prefetch_tmap(mu);
            int it = 0;
            bool ok = true;
            int64_t m0, vend;
            int n0, e;
            for (int64_t w = blockIdx.x; ok && decode(p, m_tiles, w, m0, n0, e, vend); w += gridDim.x) {
                const int wy = e * p.dff + n0;
                for (int kb = 0; kb < nk; ++kb, ++it) {
                    const int s = it % STAGES;
                    if (!tc::mbar_wait_bounded(empty0 + 8 * s, ((it / STAGES) & 1) ^ 1, abort_flag)) { ok = false; break; }
                    const uint32_t fb = full0 + 8 * s;
                    tc::mbar_arrive_expect_tx(fb, STAGE_BYTES);
                    const uint32_t a_dst = tc::smem_u32(smem + s * STAGE_BYTES);
                    tc::tma_load_2d(a_dst, &tmX, fb, kb * BK, (int)m0);
                    tc::tma_load_2d(a_dst + A_BYTES, mg, fb, kb * BK, wy);
                    tc::tma_load_2d(a_dst + A_BYTES + B_BYTES / 2, mu, fb, kb * BK, wy);
                }
            }
            if (!ok) {
                for (int j = it - 1; j >= 0 && j >= it - STAGES; --j)
                    tc::mbar_wait_bounded(full0 + 8 * (j % STAGES), (j / STAGES) & 1, abort_flag, 100000000ull);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            int it = 0, tcount = 0;
            bool ok = true;
            int64_t m0, vend;
            int n0, e;
            for (int64_t w = blockIdx.x; ok && decode(p, m_tiles, w, m0, n0, e, vend); w += gridDim.x) {
                for (int c = 0; c < nch && ok; ++c) {
                    if (!tc::mbar_wait_bounded(cempty0 + 8 * c, (tcount & 1) ^ 1, abort_flag)) { ok = false; break; }
                    tc::fence_after_sync();
                    const uint32_t d_tmem = tmem + c * (2 * BNH);
                    const int k_lo = c * nk / nch, k_hi = (c + 1) * nk / nch;
                    for (int kb = k_lo; kb < k_hi; ++kb, ++it) {
                        const int s = it % STAGES;
                        if (!tc::mbar_wait_bounded(full0 + 8 * s, (it / STAGES) & 1, abort_flag)) { ok = false; break; }
                        tc::fence_after_sync();
                        const uint32_t a_base = tc::smem_u32(smem + s * STAGE_BYTES);
                        const uint32_t b_base = a_base + A_BYTES;
#pragma unroll
                        for (int kk = 0; kk < BK / 16; ++kk) {
                            const uint64_t ad = tc::sw128_desc(a_base + kk * 32, 16, 1024);
                            const uint64_t bd = tc::sw128_desc(b_base + kk * 32, 16, 1024);
                            tc::mma_f16(d_tmem, ad, bd, IDESC, (kb != k_lo) || kk != 0);
                        }
                        tc::mma_commit(empty0 + 8 * s);
                    }
                    if (ok) tc::mma_commit(cfull0 + 8 * c);
                }
                ++tcount;
            }
        }
        __syncwarp();
    } else {
        // warps 2-17: warp w reads TMEM lanes 32 (w % 4) .. (its quadrant) and quarter (w - 2) / 4 of
        // the tile's 32 h-columns (8 gate and 8 up values per row and chunk)
        const int q = warp & 3, quarter = (warp - 2) >> 2;
        constexpr int HW = BNH / 4;
        static_assert(HW == 8, "the outlier terms below are written out for 8 columns");
        int tcount = 0;
        int64_t m0, vend;
        int n0, e;
        bool ok = true;
        for (int64_t w = blockIdx.x; ok && decode(p, m_tiles, w, m0, n0, e, vend); w += gridDim.x) {
            const int64_t row = m0 + q * 32 + lane;
            const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + quarter * HW;
            double g[HW], u[HW];
#pragma unroll
            for (int j = 0; j < HW; ++j) { g[j] = 0.0; u[j] = 0.0; }
            for (int c = 0; c < nch; ++c) {
                if (!tc::mbar_wait_bounded(cfull0 + 8 * c, tcount & 1, abort_flag)) { ok = false; break; }
                tc::fence_after_sync();
                uint32_t vg[HW], vu[HW];
                tc::tmem_ld_32x32b_x8(tb + c * (2 * BNH), vg);           // gate pre-activation, chunk c
                tc::tmem_ld_32x32b_x8(tb + c * (2 * BNH) + BNH, vu);     // up pre-activation, chunk c
                tc::tmem_wait_ld();
                tc::fence_before_sync();
                tc::mbar_arrive(cempty0 + 8 * c);
#pragma unroll
                for (int j = 0; j < HW; ++j) {
                    g[j] += (double)__uint_as_float(vg[j]);
                    u[j] += (double)__uint_as_float(vu[j]);
                }
            }
            if (!ok) break;
            if (masked && row < vend) {   // the outlier channels' terms: bf16 products (exact in fp32) summed in fp64
                const int no = *p.out_n;
                const float* xr = p.xo + row * kMaxOutliers;
                const float* wg = p.wo + (size_t)(2 * e) * kMaxOutliers * p.dff + n0 + quarter * HW;
                const float* wu = wg + (size_t)kMaxOutliers * p.dff;
                for (int o = 0; o < no; ++o) {
                    const float x = __ldg(xr + o);
                    const float4 g0 = __ldg(reinterpret_cast<const float4*>(wg + (size_t)o * p.dff));
                    const float4 g1 = __ldg(reinterpret_cast<const float4*>(wg + (size_t)o * p.dff + 4));
                    const float4 u0 = __ldg(reinterpret_cast<const float4*>(wu + (size_t)o * p.dff));
                    const float4 u1 = __ldg(reinterpret_cast<const float4*>(wu + (size_t)o * p.dff + 4));
                    g[0] += (double)(x * g0.x); g[1] += (double)(x * g0.y); g[2] += (double)(x * g0.z);
                    g[3] += (double)(x * g0.w); g[4] += (double)(x * g1.x); g[5] += (double)(x * g1.y);
                    g[6] += (double)(x * g1.z); g[7] += (double)(x * g1.w);
                    u[0] += (double)(x * u0.x); u[1] += (double)(x * u0.y); u[2] += (double)(x * u0.z);
                    u[3] += (double)(x * u0.w); u[4] += (double)(x * u1.x); u[5] += (double)(x * u1.y);
                    u[6] += (double)(x * u1.z); u[7] += (double)(x * u1.w);
                }
            }
            if (row < p.rows) {
                const bool valid = row < vend;
                uint32_t out[HW / 2];
#pragma unroll
                for (int j = 0; j < HW; j += 2) {
                    const double h0 = valid ? g[j] / (1.0 + exp(-g[j])) * u[j] : 0.0;
                    const double h1 = valid ? g[j + 1] / (1.0 + exp(-g[j + 1])) * u[j + 1] : 0.0;
                    out[j / 2] = (uint32_t)__bfloat16_as_ushort(__double2bfloat16(h0)) |
                                 ((uint32_t)__bfloat16_as_ushort(__double2bfloat16(h1)) << 16);
                }
                uint4* dst = reinterpret_cast<uint4*>(p.h + row * p.dff + n0 + quarter * HW);
                dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
            }
            ++tcount;
        }
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
    if (threadIdx.x == 0 && *abort_flag) clha_record_error(p.err, CLHA_ERR_TIMEOUT, blockIdx.x, 0, KID_ACT);
}

}  // namespace

cudaError_t launch_expert_act_tc(cudaStream_t s, int num_sms, const __nv_bfloat16* X, int64_t rows, int d_model,
                                 const int64_t* seg, int E, const __nv_bfloat16* Wg, const __nv_bfloat16* Wu, int d_ff,
                                 __nv_bfloat16* h, const int* sel, const __nv_bfloat16* Wgm, const __nv_bfloat16* Wum,
                                 const int* out_n, const float* xo, const float* wo, int* err) {
    CUtensorMap tX, tG, tU, tGm, tUm;
    cudaError_t e;
    if ((e = make_tmap_2d(&tX, X, (uint64_t)rows, (uint64_t)d_model, 2, BM, BK)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tG, Wg, (uint64_t)E * d_ff, (uint64_t)d_model, 2, BNH, BK)) != cudaSuccess) return e;
    if ((e = make_tmap_2d(&tU, Wu, (uint64_t)E * d_ff, (uint64_t)d_model, 2, BNH, BK)) != cudaSuccess) return e;
    // the masked copies (outlier channels zeroed); without them the unmasked weights stand in (unused)
    if ((e = make_tmap_2d(&tGm, Wgm ? Wgm : Wg, (uint64_t)E * d_ff, (uint64_t)d_model, 2, BNH, BK)) != cudaSuccess)
        return e;
    if ((e = make_tmap_2d(&tUm, Wum ? Wum : Wu, (uint64_t)E * d_ff, (uint64_t)d_model, 2, BNH, BK)) != cudaSuccess)
        return e;
    // per call: the attribute belongs to the current device's context (a process may drive several)
    if ((e = cudaFuncSetAttribute(expert_act_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES)) !=
        cudaSuccess)
        return e;
    ActParams p{sel, rows, d_model, d_ff, seg, E, h, d_ff / BNH, out_n, xo, wo, err};
    expert_act_tc<<<num_sms, kThreads, SMEM_BYTES, s>>>(tX, tG, tU, tGm, tUm, p);
    clha_note_launches(1);
    return cudaGetLastError();
}
