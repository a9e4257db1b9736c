// GPTQ's factor of the damped Hessian, in one of two forms:
//   U (CLHA_FACTOR_INV_CHOL)    upper triangular with H_d^-1 = U^T U;
//   F (CLHA_FACTOR_BLOCK_CHOL)  the Cholesky factor of H_d itself, scaled per 128-column block.
//
// With J the index reversal, let L be the lower Cholesky factor of J H_d J. Then R = J L J is upper
// with H_d = R R^T, and U = R^-1 = J L^-1 J is upper with U^T U = (R R^T)^-1 = H_d^-1; its diagonal
// is positive, so it is THE upper Cholesky factor of H_d^-1. U needs one Cholesky and one triangular
// inverse (no explicit inverse of H_d, no second factorisation).
//
// F needs the Cholesky only. U's diagonal blocks are the inverses of R's (U_bb = R_bb^-1), and
// U_ab = -U_aa R_ab U_bb above them. F holds U_bb on the diagonal blocks and F_ab = R_ab U_bb (a < b)
// above them. GPTQ's lazy update of block b, W_b - E_a U_ab with E = (W - W_hat) R the scaled errors
// of the earlier columns a, then equals W_b + (W_a - W_hat_a) F_ab, since E_a U_aa = W_a - W_hat_a.
// So F serves GPTQ in place of U at half the factor's flops: the inverse terms (F and Q tasks below)
// drop out, and the block scaling is one small product per tile, done by the store. In J order a
// 128-block b of F is the pair of 64-tiles (p, p+1), p even, of L, and J F J = L blockdiag(L_bb^-1):
//   L_bb^-1 = [[D_p, 0], [X, D_{p+1}]],   X = -D_{p+1} L_{p+1,p} D_p,
// so the tiles of J F J are D_p, X, D_{p+1} on the diagonal block, L_ip D_p + L_{i,p+1} X and
// L_{i,p+1} D_{p+1} below it (i >= p + 2).
//
// Float64 throughout, on 64 x 64 tiles (nt = d / 64 per side), batched over problems, in up to four
// groups of different d that share one graph launch (the small groups' short critical paths then
// overlap the large groups' bulk work):
//   fac_load    A = J H_d J, lower tiles, tile-major float64 (each tile 32 KB contiguous); per group
//   fac_dag     one persistent kernel that runs the whole blocked Cholesky and the blocked inverse
//               of every problem of every group as a graph of tile tasks (below)
//   fac_store   U = J Y^T J as float32, strict lower triangle zero; per group
// and for F, the graph without its inverse tasks, then
//   fac_pair    X^T of every 128-block (two tile products, kept in the otherwise unused tile Y_{p,p+1})
//   fac_store_f F = J (L blockdiag(L_bb^-1)) J as float32, the products on the FP64 tensor path
//
// Tile tasks. The inverse is kept transposed, Y = L^-T (upper), so that every product has the form
// C <- alpha C + beta P Q^T with row-major tiles P and Q:
//   P(m)        L_mm = chol(A_mm), D_m = L_mm^-1, Y_mm = D_m^T                 (one CTA, in shared memory)
//   S(i,m)      L_im = A_im D_m^T                                                i > m
//   G(i,j,m)    A_ij -= L_im L_jm^T                                              i >= j > m
//   Q(j,i,m)    R_ji += Y_jm L_im^T         (R_ji accumulates in Y_ji; first term m = j overwrites)
//   F(j,m)      Y_jm = -R_jm D_m^T                                               j < m
// since L X = I with X = L^-1 = Y^T gives X_ij = -D_i sum_{m=j}^{i-1} L_im X_mj for i > j.
//
// Scheduling: tasks are numbered in a topological order (stages with a one-panel lookahead, see
// stage_counts; within a stage group after group, problems interleaved inside each class) and CTAs
// take numbers from a global counter. Every tile has a monotone state counter: A_ij counts the
// updates applied (j + 1 once L_ij is final); Y_ji counts the Q terms applied (i - j + 1 once final).
// Each CTA has 8 compute warps and a scheduler warp: the scheduler takes the next number, decodes
// it, prefetches its tiles into L2 and checks (acquire loads, bounded by a time limit) that its
// inputs have reached the states it needs while the compute warps run the current task (each wait
// bounded by the context's limit, 4 s by default; one that runs out aborts the whole graph and
// records CLHA_ERR_TIMEOUT); after the
// barrier that ends a task it publishes the output tile's new state with a release store. Any task
// waited on has a smaller number and is running or finished (a finished task is released before the
// scheduler waits on anything): the schedule cannot deadlock however many CTAs are resident. Tile
// data moves through L2 only (cp.async.cg and ld.global.cg), never through a stale L1 line.
//
// Products run on the FP64 tensor-core path (mma.sync m8n8k4 f64): 8 warps, each a 32 x 16 block
// of the 64 x 64 output, operands in padded shared memory; the diagonal task's inner products are
// 8 x 8 blocks on the same path.
// A non-positive pivot is recorded (problem, original column) and the problem's factor is NaN.
#include "clha_internal.h"

namespace {

constexpr int NB = 64;
constexpr int LD = NB + 8;   // padded shared row (doubles): the 16-byte fragment loads of two adjacent
                             // rows fall in opposite halves of the banks (conflict-free)
constexpr int TILE_DOUBLES = NB * LD;
constexpr int TILE_ELEMS = NB * NB;

typedef double Tile[LD];

// Barrier of the graph kernel's 256 compute threads (the scheduler warp does not take part).
__device__ __forceinline__ void cbar() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

__device__ __forceinline__ uint64_t gtimer() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ int ld_acquire(const int* p) {
    int v;
    asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}
__device__ __forceinline__ void st_release(int* p, int v) {
    asm volatile("st.release.gpu.global.b32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
    const uint32_t d = (uint32_t)__cvta_generic_to_shared(smem_dst);
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d), "l"(gsrc) : "memory");
}
// Bring a contiguous, 16-byte aligned range (a multiple of 16 bytes) into L2 (no completion to wait for).
__device__ __forceinline__ void prefetch_l2(const void* p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}
__device__ __forceinline__ void dmma(double& c0, double& c1, double a, double b) {
    asm volatile("mma.sync.aligned.m8n8k4.row.col.f64.f64.f64.f64 {%0, %1}, {%2}, {%3}, {%0, %1};"
                 : "+d"(c0), "+d"(c1)
                 : "d"(a), "d"(b));
}

// ------------------------------------------------------------------------------ load / store
// A tile (i, j), i >= j: A[r][c] = H[d-1-(64i+r)][d-1-(64j+c)]. One CTA per tile.
__global__ void __launch_bounds__(256) fac_load(const float* __restrict__ H, int d, int nt, double* __restrict__ A) {
    const int b = blockIdx.y;
    int t = blockIdx.x, i = 0;
    while (t > i) { t -= i + 1; ++i; }   // lower tiles, row-major: row i holds i + 1 tiles
    const int j = t;
    const float* Hb = H + (size_t)b * d * d;
    double* At = A + (((size_t)b * nt + i) * nt + j) * TILE_ELEMS;
    const size_t r0 = (size_t)d - 1 - (size_t)NB * i, c0 = (size_t)d - 1 - (size_t)NB * j;
#pragma unroll 4
    for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) {
        const int r = e >> 6, c = e & 63;
        At[e] = (double)Hb[(r0 - r) * d + (c0 - c)];
    }
}

// U tile (ta, tc): zero below the diagonal, else U[ra][rc] = Y_{jt,it}[63-rc][63-ra] with
// jt = nt-1-tc, it = nt-1-ta (Y upper, so jt <= it). Transposed through shared memory.
__global__ void __launch_bounds__(256) fac_store(const double* __restrict__ Y, int d, int nt, float* __restrict__ U) {
    __shared__ double s[NB][NB + 1];
    const int b = blockIdx.y;
    const int ta = blockIdx.x / nt, tc = blockIdx.x % nt;
    float* Ub = U + (size_t)b * d * d;
    if (ta > tc) {
        for (int e = threadIdx.x; e < TILE_ELEMS; e += 256)
            Ub[(size_t)(NB * ta + (e >> 6)) * d + NB * tc + (e & 63)] = 0.f;
        return;
    }
    const int jt = nt - 1 - tc, it = nt - 1 - ta;
    const double* Yt = Y + (((size_t)b * nt + jt) * nt + it) * TILE_ELEMS;
    for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) s[e >> 6][e & 63] = __ldcg(Yt + e);
    __syncthreads();
    for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) {
        const int ra = e >> 6, rc = e & 63;
        const float v = (ta == tc && ra > rc) ? 0.f : (float)s[63 - rc][63 - ra];
        Ub[(size_t)(NB * ta + ra) * d + NB * tc + rc] = v;
    }
}

// ------------------------------------------------------------------------------ tile primitives
// Contiguous 64x64 global tile -> padded shared tile (cp.async through L2).
__device__ __forceinline__ void tile_to_smem(Tile* dst, const double* __restrict__ src) {
#pragma unroll
    for (int it = 0; it < 8; ++it) {
        const int q = it * 256 + threadIdx.x;   // 16-byte chunk: row q / 32, doubles 2 (q % 32) ..
        cp_async16(&dst[q >> 5][2 * (q & 31)], src + 2 * q);
    }
}

// C (row-major 64x64, row pitch ldc; global, or shared when !load_c) <- (load_c ? C : 0) +
// sign * (P1 Q1^T [+ P2 Q2^T]): one or two
// operand pairs (a two-level task applies two panels' updates to its output tile with one read and
// one write of C). The first pair's copies into shared memory and the loads of this thread's C
// fragments are in flight together; a second pair is copied after every warp has finished with the
// first. A negative sign is applied to C on the way in and out (C - PQ^T = -(-C + PQ^T)), not to every
// operand fragment. Each 16-byte shared load feeds two k-steps: in the k-block k0..k0+7 lane tq
// supplies k0+2tq to the first m8n8k4 product and k0+2tq+1 to the second (the same k for its A and B
// fragments), so the two products together cover the block.
__device__ __forceinline__ void tile_gemm_nt(const double* __restrict__ Pg, const double* __restrict__ Qg, Tile* Ps,
                                             Tile* Qs, double* C, bool load_c, bool negate,
                                             const double* __restrict__ Pg2 = nullptr,
                                             const double* __restrict__ Qg2 = nullptr, int ldc = NB) {
    tile_to_smem(Ps, Pg);
    tile_to_smem(Qs, Qg);
    asm volatile("cp.async.commit_group;" ::: "memory");
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int wm = warp >> 2, wn = warp & 3;   // warp block: rows 32 wm .., cols 16 wn ..
    double c[4][2][2];
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 2; ++ni) {
            if (load_c) {
                const double2 v = __ldcg(reinterpret_cast<const double2*>(
                    C + (32 * wm + 8 * mi + g) * NB + 16 * wn + 8 * ni + 2 * tq));
                c[mi][ni][0] = negate ? -v.x : v.x;
                c[mi][ni][1] = negate ? -v.y : v.y;
            } else {
                c[mi][ni][0] = c[mi][ni][1] = 0.0;
            }
        }
    const int npairs = Pg2 ? 2 : 1;
#pragma unroll 1
    for (int pr = 0; pr < npairs; ++pr) {
        if (pr == 1) {           // every warp is done with the first pair's tiles
            cbar();
            tile_to_smem(Ps, Pg2);
            tile_to_smem(Qs, Qg2);
            asm volatile("cp.async.commit_group;" ::: "memory");
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");
        cbar();
#pragma unroll 2
        for (int k0 = 0; k0 < NB; k0 += 8) {
            double2 a[4], bq[2];
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
                a[mi] = *reinterpret_cast<const double2*>(&Ps[32 * wm + 8 * mi + g][k0 + 2 * tq]);
#pragma unroll
            for (int ni = 0; ni < 2; ++ni)
                bq[ni] = *reinterpret_cast<const double2*>(&Qs[16 * wn + 8 * ni + g][k0 + 2 * tq]);
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                for (int ni = 0; ni < 2; ++ni) dmma(c[mi][ni][0], c[mi][ni][1], a[mi].x, bq[ni].x);
#pragma unroll
            for (int mi = 0; mi < 4; ++mi)
#pragma unroll
                for (int ni = 0; ni < 2; ++ni) dmma(c[mi][ni][0], c[mi][ni][1], a[mi].y, bq[ni].y);
        }
    }
#pragma unroll
    for (int mi = 0; mi < 4; ++mi)
#pragma unroll
        for (int ni = 0; ni < 2; ++ni)
            *reinterpret_cast<double2*>(C + (32 * wm + 8 * mi + g) * ldc + 16 * wn + 8 * ni + 2 * tq) =
                negate ? make_double2(-c[mi][ni][0], -c[mi][ni][1]) : make_double2(c[mi][ni][0], c[mi][ni][1]);
}

// Cholesky of the 64x64 tile in T (lower, in place) and its inverse X = L^-1 (lower, in Xs with
// row pitch XLD); writes L to Lg, X to Dg, X^T to Yg. Right-looking by blocks of 8 columns (o = 8 kb),
// three CTA barriers per block:
//   1. warp 0 factors the 8x8 diagonal block in registers, every lane the whole block (no shuffles
//      on the pivot chain; two 4-column stages keep the live values few), and lane j < 8 solves
//      column j of its inverse X_bb. Meanwhile warps 1-7
//      form S = L_b,<o X_<o,<o, the sums that the block row of the inverse needs: with L X = I,
//      L_bb X_bj + S_bj = 0, so X_bj = -X_bb S_bj.
//   2. the panel below, L_ib = A_ib X_bb^T (kept transposed in PT), and X_bj = -X_bb S_bj.
//   3. the rank-8 update of the trailing lower triangle, A_ij -= L_ib L_jb^T, and L_ib into T.
// The products of steps 1-3 are 8x8 blocks on the FP64 tensor path (m8n8k4, k = 8 in two steps), one
// block per warp at a time; only the pivot chain of step 1 runs as scalar fp64 arithmetic.
// The inverse's column reads use Xs's odd pitch (65 doubles), so they are conflict-free.
constexpr int XLD = NB + 1;
constexpr int PLD = NB + 8;             // row pitch of S and PT (the fragment loads of rows k and k+1
                                        // fall in opposite halves of the banks)
constexpr int P_SCRATCH = 2 * 8 * PLD;  // S [8][PLD] and PT [8][PLD]

__device__ __forceinline__ constexpr int pk(int r, int c) { return r * (r + 1) / 2 + c; }   // packed lower

// In-register Cholesky of a 4x4 block (packed lower, in place) with the reciprocals of its diagonal;
// the first non-positive pivot's column (col0 + c) goes to `bad`, and the factor turns NaN from there.
__device__ __forceinline__ void chol4(double (&a)[10], double (&inv)[4], int& bad, int col0, double qnan) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
        const double p = a[pk(c, c)];
        const bool ok = (p > 0.0) && isfinite(p);
        if (!ok && bad < 0) bad = col0 + c;
        inv[c] = ok ? rsqrt(p) : qnan;
        a[pk(c, c)] = p * inv[c];
#pragma unroll
        for (int r = c + 1; r < 4; ++r) a[pk(r, c)] *= inv[c];
#pragma unroll
        for (int r = c + 1; r < 4; ++r)
#pragma unroll
            for (int k = c + 1; k <= r; ++k) a[pk(r, k)] = fma(-a[pk(r, c)], a[pk(k, c)], a[pk(r, k)]);
    }
}

__device__ void tile_potrf_inv(Tile* T, double* Xs, double* scr, double* Lg, double* Dg, double* Yg, int* err, int b,
                               int col_base, int d) {
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const double qnan = __longlong_as_double(0x7ff8000000000000ll);
    double* S = scr;              // S[r][j]  = sum_{m < o} L[o+r][m] X[m][j],   j < o
    double* PT = scr + 8 * PLD;   // PT[c][i] = L[i][o+c],                      i >= o + 8
    const int g = lane >> 2, tq = lane & 3;   // m8n8k4 fragment coordinates
    int bad = -1;   // first non-positive pivot (warp 0)
    for (int kb = 0; kb < 8; ++kb) {
        const int o = 8 * kb;
        if (warp == 0) {
            // two 4-column stages, so that at most ~30 of the block's values are live at once:
            // L11 = chol(A11); L21 = A21 L11^-T; A22 -= L21 L21^T; L22 = chol(A22)
            double* dinv = PT;   // 1 / L_cc of this block (PT is free until step 2)
            double a11[10], inv[4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c <= r; ++c) a11[pk(r, c)] = T[o + r][o + c];
            chol4(a11, inv, bad, o, qnan);
            double l21[4][4];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    double v = T[o + 4 + r][o + c];
#pragma unroll
                    for (int k = 0; k < c; ++k) v = fma(-l21[r][k], a11[pk(c, k)], v);
                    l21[r][c] = v * inv[c];
                }
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    dinv[r] = inv[r];
#pragma unroll
                    for (int c = 0; c <= r; ++c) T[o + r][o + c] = a11[pk(r, c)];
                }
            }
            double a22[10];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
                for (int c = 0; c <= r; ++c) {
                    double v = T[o + 4 + r][o + 4 + c];
#pragma unroll
                    for (int k = 0; k < 4; ++k) v = fma(-l21[r][k], l21[c][k], v);
                    a22[pk(r, c)] = v;
                }
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < 4; ++r)
#pragma unroll
                    for (int c = 0; c < 4; ++c) T[o + 4 + r][o + c] = l21[r][c];
            }
            chol4(a22, inv, bad, o + 4, qnan);
            if (lane == 0) {
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    dinv[4 + r] = inv[r];
#pragma unroll
                    for (int c = 0; c <= r; ++c) T[o + 4 + r][o + 4 + c] = a22[pk(r, c)];
                }
            }
            __syncwarp();
            if (lane < 8) {   // column j of X_bb: L_bb x = e_j, L_bb read back from T (broadcasts);
                              // right-looking, so that the dependent chain is one multiply and one
                              // fma per row
                const int j = lane;
                double acc[8];
#pragma unroll
                for (int r = 0; r < 8; ++r) acc[r] = (r == j) ? 1.0 : 0.0;
#pragma unroll
                for (int m = 0; m < 8; ++m) {
                    const double x = (m >= j) ? acc[m] * dinv[m] : 0.0;
                    Xs[(o + m) * XLD + o + j] = x;
#pragma unroll
                    for (int r = m + 1; r < 8; ++r) acc[r] = fma(-T[o + r][o + m], x, acc[r]);
                }
            }
        } else if (warp - 1 < kb) {
            // block jb = warp - 1 of S: the sum over the blocks mb = jb .. kb-1 of L_{b,mb} X_{mb,jb}
            // (the diagonal block X_{jb,jb} holds zeros above its diagonal)
            const int jb = warp - 1;
            double c0 = 0.0, c1 = 0.0;
            for (int mb = jb; mb < kb; ++mb) {
#pragma unroll
                for (int s4 = 0; s4 < 8; s4 += 4)
                    dmma(c0, c1, T[o + g][8 * mb + s4 + tq], Xs[(8 * mb + s4 + tq) * XLD + 8 * jb + g]);
            }
            S[g * PLD + 8 * jb + 2 * tq] = c0;
            S[g * PLD + 8 * jb + 2 * tq + 1] = c1;
        }
        cbar();
        // warps 0 .. 6-kb: panel block row bi = kb+1+warp, L_{bi,b} = A_{bi,b} X_bb^T, kept transposed;
        // the next kb warps: block jb of the block row of the inverse, X_{b,jb} = -X_bb S_{b,jb}
        if (warp < 7 - kb) {
            const int bi = kb + 1 + warp;
            double c0 = 0.0, c1 = 0.0;
#pragma unroll
            for (int s4 = 0; s4 < 8; s4 += 4)
                dmma(c0, c1, T[8 * bi + g][o + s4 + tq], Xs[(o + g) * XLD + o + s4 + tq]);
            PT[(2 * tq) * PLD + 8 * bi + g] = c0;
            PT[(2 * tq + 1) * PLD + 8 * bi + g] = c1;
        } else if (warp < 7) {
            const int jb = warp - (7 - kb);
            double c0 = 0.0, c1 = 0.0;
#pragma unroll
            for (int s4 = 0; s4 < 8; s4 += 4)
                dmma(c0, c1, Xs[(o + g) * XLD + o + s4 + tq], S[(s4 + tq) * PLD + 8 * jb + g]);
            Xs[(o + g) * XLD + 8 * jb + 2 * tq] = -c0;
            Xs[(o + g) * XLD + 8 * jb + 2 * tq + 1] = -c1;
        }
        cbar();
        {   // trailing blocks (bi, bj), kb < bj <= bi: A_{bi,bj} -= L_{bi,b} L_{bj,b}^T (whole 8x8 blocks;
            // above the diagonal of a diagonal block nothing is read), as -(-A + L L^T)
            const int nb = 7 - kb;
            for (int e = warp; e < nb * (nb + 1) / 2; e += 8) {
                int bi = 0, bj = e;
                while (bj > bi) { bj -= bi + 1; ++bi; }
                bi += kb + 1;
                bj += kb + 1;
                double2* cp = reinterpret_cast<double2*>(&T[8 * bi + g][8 * bj + 2 * tq]);
                const double2 cv = *cp;
                double c0 = -cv.x, c1 = -cv.y;
#pragma unroll
                for (int s4 = 0; s4 < 8; s4 += 4)
                    dmma(c0, c1, PT[(s4 + tq) * PLD + 8 * bi + g], PT[(s4 + tq) * PLD + 8 * bj + g]);
                *cp = make_double2(-c0, -c1);
            }
            for (int e = tid; e < (56 - o) * 8; e += 256) {   // the panel into T
                const int i = o + 8 + (e >> 3), c = e & 7;
                T[i][o + c] = PT[c * PLD + i];
            }
        }
        cbar();
    }
    if (tid == 0 && bad >= 0) clha_record_error(err, CLHA_ERR_NOT_PD, b, d - 1 - (col_base + bad), KID_FACTOR);
#pragma unroll 4
    for (int e = tid; e < TILE_ELEMS; e += 256) {
        const int r = e >> 6, c = e & 63;
        Lg[e] = (c <= r) ? T[r][c] : 0.0;
        Dg[e] = (c <= r) ? Xs[r * XLD + c] : 0.0;
        Yg[e] = (r <= c) ? Xs[c * XLD + r] : 0.0;
    }
}

// ------------------------------------------------------------------------------ the task graph
constexpr int MAX_GROUPS = 4;
constexpr int CW = 256;                 // compute threads (8 warps)
constexpr int DAG_THREADS = CW + 32;    // + the scheduler warp

// One group: `batch` problems of the same size d (nt = d / 64 tiles per side), its own workspace.
struct Grp {
    double* A;   // [batch][nt][nt] tiles, lower used: A, then L in place
    double* Y;   // [batch][nt][nt] tiles, upper used: R accumulators, then Y = L^-T
    double* D;   // [batch][nt] tiles: D_m = L_mm^-1
    int* stA;    // [batch][nt][nt]
    int* stY;    // [batch][nt][nt]
    int nt, batch, d;
    int pbase;   // index of the group's first problem across all groups (error reports)
};

struct Dag {
    Grp grp[MAX_GROUPS];
    int ng, max_nt;
    unsigned long long* ticket;
    int* abort_flag;
    int* err;
    unsigned long long total;
    uint64_t wait_ns;   // time limit of one dependency wait
    int inv;            // 1: Cholesky and inverse (U); 0: Cholesky only (F)
};

__device__ __forceinline__ double* tile(double* base, const Grp& g, int b, int i, int j) {
    return base + (((size_t)b * g.nt + i) * g.nt + j) * TILE_ELEMS;
}
__device__ __forceinline__ int* st(int* base, const Grp& g, int b, int i, int j) {
    return base + ((size_t)b * g.nt + i) * g.nt + j;
}

// One thread: wait until *p >= target (acquire). False when the graph was aborted or the wait ran out of time.
__device__ bool wait_ge(const int* p, int target, const Dag& g, int problem) {
    if (ld_acquire(p) >= target) return true;
    const uint64_t t0 = gtimer();
    unsigned ns = 32;
    for (;;) {
        __nanosleep(ns);
        if (ns < 512) ns <<= 1;
        if (ld_acquire(p) >= target) return true;
        if (*reinterpret_cast<volatile int*>(g.abort_flag)) return false;
        if (gtimer() - t0 > g.wait_ns) {
            atomicExch(g.abort_flag, 1);
            clha_record_error(g.err, CLHA_ERR_TIMEOUT, problem, 0, KID_FACTOR);
            return false;
        }
    }
}

// Tasks per problem in stage s, by class. Stage 0 holds P(0) and S(i,0); stage s >= 1 (m = s - 1)
// holds, in this order:
//   0  G(i,m+1,m)          the next panel's update (lookahead): P(m+1) can start once it is done
//   1  P(m+1)
//   2  F(j,m)              j < m
//   3  Q(j,i,m)            one level: for even m every j <= m with i = m+1, m+2; for odd m every
//                          j <= m with i = m+1, and j = m with i >= m+2
//   4  FQ(j,i,{m-1,m})     odd m, j <= m-1, i >= m+2: the terms of levels m-1 and m in one task
//   5  even m: G(i,m+2,m)  the column after the lookahead, one level;
//      odd m: FG(i,j,{m-1,m}) for m+2 <= j <= i: levels m-1 and m in one task
//   6  S(i,m+1)
// Levels pair up (even m, m+1): an even level updates only the two columns after its panel and
// leaves the rest of its trailing matrix (and of its inverse terms) to the next, odd level, whose
// bulk tasks apply both. A bulk task then reads and writes its output tile once per two panels and
// pays its scheduling once, and the lookahead chain P(m) -> S(m+1,m) -> G(m+1,m+1,m) -> P(m+1) keeps
// its one-level tasks. Every task waits only on tasks with smaller numbers (a CPU model of this
// numbering checks that, and that each update is applied once, for every tile count up to 39).
// Without the inverse (the F form) classes 2, 3 and 4 are empty and the rest keep their numbers'
// order and dependencies, which never involve Y.
__host__ __device__ __forceinline__ void stage_counts(int nt, int s, long long (&n)[7], bool inv = true) {
    for (int c = 0; c < 7; ++c) n[c] = 0;
    if (s == 0) {
        n[1] = 1;
        n[6] = nt - 1;
        return;
    }
    const int m = s - 1;
    const long long R = nt - 1 - m;
    if (R < 0) return;
    const long long R1 = R >= 1 ? R - 1 : 0;
    n[0] = R;
    n[1] = R >= 1 ? 1 : 0;
    n[2] = m;
    if ((m & 1) == 0) {
        n[3] = (long long)(m + 1) * (R < 2 ? R : 2);
        n[5] = R1;
    } else {
        n[3] = (long long)(m + 1) * (R < 1 ? R : 1) + R1;
        n[4] = (long long)m * R1;
        n[5] = R >= 1 ? (R - 1) * R / 2 : 0;
    }
    n[6] = R1;
    if (!inv) n[2] = n[3] = n[4] = 0;
}
__host__ __device__ __forceinline__ unsigned long long stage_total(int nt, int s, bool inv = true) {
    if (s > nt) return 0;
    long long n[7];
    stage_counts(nt, s, n, inv);
    return (unsigned long long)(n[0] + n[1] + n[2] + n[3] + n[4] + n[5] + n[6]);
}

// A decoded task: class q (0 P, 1 S, 2/5 G, 3 F, 4 Q, 6 FG, 7 FQ), group k, problem b of the group, level m,
// tiles i, j; its inputs' states to wait for; its outputs' states once done.
struct Task {
    int q, k, b, m, i, j;
    int status;                   // READY, WAIT (its inputs were not all ready yet), STOP
};
constexpr int READY = 0, WAIT = 1, STOP = 2;
struct Deps {
    const int* wp[3];
    int wt[3];
    int* out;                     // output state and its new value
    int out_value;
    int* out2;                    // P(m) also completes Y_mm (state 1)
};

__device__ __forceinline__ void decode_task(const Dag& g, const unsigned long long* lvl, unsigned long long t, Task& d,
                                            Deps& dp) {
    const int S = g.max_nt;
    int lo = 0, hi = S;   // stage: last s with lvl[s] <= t
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (lvl[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int sg = lo;
    // within a stage every count fits in 32 bits (a stage holds at most batch x ~nt^2 tasks):
    // 32-bit arithmetic keeps the decode off the 64-bit division path
    uint32_t r = (uint32_t)(t - lvl[sg]);
    int k = 0;
    bool found = false;
#pragma unroll
    for (int kk = 0; kk < MAX_GROUPS; ++kk) {
        if (!found && kk < g.ng) {
            const uint32_t c = (uint32_t)stage_total(g.grp[kk].nt, sg, g.inv) * (uint32_t)g.grp[kk].batch;
            if (r < c) { k = kk; found = true; }
            else r -= c;
        }
    }
    const Grp& G = g.grp[k];
    const int nt = G.nt;
    const uint32_t batch = (uint32_t)G.batch;
    long long n[7];
    stage_counts(nt, sg, n, g.inv);
    int c = 0;
#pragma unroll
    for (int cq = 0; cq < 7; ++cq)
        if (c == cq && r >= (uint32_t)n[cq] * batch) { r -= (uint32_t)n[cq] * batch; ++c; }
    const uint32_t local = r / batch;
    const int b = (int)(r - local * batch);
    int q, m = sg - 1, i = 0, j = 0;
    const bool odd = (m & 1) != 0;
    if (c == 0) { q = 2; i = m + 1 + (int)local; j = m + 1; }
    else if (c == 1) { q = 0; m = sg; }
    else if (c == 2) { q = 3; j = (int)local; }
    else if (c == 3) {
        q = 4;
        if (!odd) {
            const uint32_t ii = local / (uint32_t)(m + 1);
            i = m + 1 + (int)ii;
            j = (int)(local - ii * (uint32_t)(m + 1));
        } else if (local < (uint32_t)(m + 1)) {
            i = m + 1;
            j = (int)local;
        } else {
            i = m + 2 + (int)(local - (uint32_t)(m + 1));
            j = m;
        }
    } else if (c == 4) {
        q = 7;
        const uint32_t ii = local / (uint32_t)m;
        i = m + 2 + (int)ii;
        j = (int)(local - ii * (uint32_t)m);
    } else if (c == 5) {
        if (!odd) {
            q = 5;
            i = m + 2 + (int)local;
            j = m + 2;
        } else {
            // FG(i, j) for m+2 <= j <= i < nt, column after column (nt - j tasks in column j): the
            // column k = j - (m+2) is the largest with cum(k) = k R2 - k(k-1)/2 <= local, R2 = nt - m - 2,
            // the smaller root of a quadratic, then a unit step either way for the rounding of the root
            q = 6;
            const long long R2 = nt - m - 2, B = 2 * R2 + 1, lc = (long long)local;
            long long k = (long long)((double)B - sqrt((double)(B * B - 8 * lc))) / 2;
            auto cum = [&](long long kk) { return kk * R2 - kk * (kk - 1) / 2; };
            while (k > 0 && cum(k) > lc) --k;
            while (cum(k + 1) <= lc) ++k;
            j = m + 2 + (int)k;
            i = j + (int)(lc - cum(k));
        }
    } else { q = 1; m = sg; i = m + 1 + (int)local; j = m; }
    d.q = q; d.k = k; d.b = b; d.m = m; d.i = i; d.j = j;
    dp.wp[0] = dp.wp[1] = dp.wp[2] = nullptr;
    dp.wt[0] = dp.wt[1] = dp.wt[2] = 0;
    dp.out2 = nullptr;
    if (q == 0) {            // P(m)
        dp.wp[0] = st(G.stA, G, b, m, m); dp.wt[0] = m;
        dp.out = st(G.stA, G, b, m, m); dp.out_value = m + 1;
        dp.out2 = st(G.stY, G, b, m, m);
    } else if (q == 1) {     // L_im = A_im D_m^T
        dp.wp[0] = st(G.stA, G, b, i, m); dp.wt[0] = m;
        dp.wp[1] = st(G.stA, G, b, m, m); dp.wt[1] = m + 1;
        dp.out = st(G.stA, G, b, i, m); dp.out_value = m + 1;
    } else if (q == 2 || q == 5 || q == 6) {   // A_ij -= L_im L_jm^T (FG: and level m-1's term)
        // L_im final implies L_{i,m-1} final (S(i,m) waited for every update of A_im)
        dp.wp[0] = st(G.stA, G, b, i, m); dp.wt[0] = m + 1;
        dp.wp[1] = st(G.stA, G, b, j, m); dp.wt[1] = m + 1;
        dp.wp[2] = st(G.stA, G, b, i, j); dp.wt[2] = q == 6 ? m - 1 : m;
        dp.out = st(G.stA, G, b, i, j); dp.out_value = m + 1;
    } else if (q == 3) {     // Y_jm = -R_jm D_m^T
        dp.wp[0] = st(G.stY, G, b, j, m); dp.wt[0] = m - j;
        dp.wp[1] = st(G.stA, G, b, m, m); dp.wt[1] = m + 1;
        dp.out = st(G.stY, G, b, j, m); dp.out_value = m - j + 1;
    } else {                 // R_ji (+)= Y_jm L_im^T (FQ: and level m-1's term)
        // Y_jm final implies Y_{j,m-1} final (F(j,m) waited for every term of R_jm)
        dp.wp[0] = st(G.stY, G, b, j, m); dp.wt[0] = m - j + 1;
        dp.wp[1] = st(G.stA, G, b, i, m); dp.wt[1] = m + 1;
        dp.wp[2] = st(G.stY, G, b, j, i); dp.wt[2] = q == 7 ? m - 1 - j : m - j;
        dp.out = st(G.stY, G, b, j, i); dp.out_value = m - j + 1;
    }
}

// Warps 0-7 run tasks; warp 8 schedules them. While the compute warps run task n - 1, the scheduler
// takes the next number, decodes it into task n and checks its inputs' states once, then meets the
// compute warps at the CTA barrier that ends task n - 1 (the task descriptors are double-buffered),
// and after it releases task n - 1's outputs (cumulative over the compute warps' stores, which the
// barrier orders before it). When an input was not ready, the descriptor says WAIT: the scheduler
// releases the finished task first, then waits for the inputs and meets the compute warps at a second
// barrier (READY or STOP). Releasing every finished task before any blocking wait keeps the schedule
// deadlock-free: tasks are taken in number order, every task waited on has a smaller number, and the
// smallest unfinished number is always either running or waiting only on finished, released tasks.
__global__ void __launch_bounds__(DAG_THREADS, 2) fac_dag(Dag g) {
    extern __shared__ double dsm[];
    Tile* T0 = reinterpret_cast<Tile*>(dsm);
    Tile* T1 = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    double* scr = dsm + 2 * TILE_DOUBLES;   // the diagonal task's S and PT
    unsigned long long* lvl = reinterpret_cast<unsigned long long*>(scr + P_SCRATCH);   // [max_nt + 2] stage starts
    __shared__ Task s_task[2];
    __shared__ int s_final[2];   // a WAIT task's final status (READY or STOP), read after the second barrier
    const int tid = threadIdx.x, lane = tid & 31;

    if (tid >= CW) {
        // ---------------------------------------------------------------- scheduler (warp 8)
        const int S = g.max_nt;
        if (lane == 0) {   // stage s holds, group after group, stage s of every group that has one
            unsigned long long acc = 0;
            for (int s = 0; s <= S; ++s) {
                lvl[s] = acc;
                for (int k = 0; k < g.ng; ++k) acc += stage_total(g.grp[k].nt, s, g.inv) * g.grp[k].batch;
            }
            lvl[S + 1] = acc;
        }
        __syncwarp();
        int* run_out = nullptr;   // outputs of the task the compute warps are running
        int* run_out2 = nullptr;
        int run_value = 0;
        int slot = 0;
        for (;;) {
            unsigned long long t = 0;
            if (lane == 0) t = atomicAdd(g.ticket, 1ull);
            t = __shfl_sync(0xffffffffu, t, 0);
            Task d;
            Deps dp;
            d.status = STOP;
            const int* wpl = nullptr;   // lane k < 3 checks input k
            int wtl = 0;
            if (t < g.total && !*reinterpret_cast<volatile int*>(g.abort_flag)) {
                decode_task(g, lvl, t, d, dp);
                if (lane < 5) {   // the task's tiles into L2 while the compute warps run the current one
                    const Grp& G = g.grp[d.k];
                    const double* Dm = G.D + ((size_t)d.b * G.nt + d.m) * TILE_ELEMS;
                    const double* pt = nullptr;
                    // lanes 3, 4: the earlier level's operands of a two-level task
                    const int ml = lane >= 3 ? d.m - 1 : d.m;
                    if (d.q == 0) pt = lane == 0 ? tile(G.A, G, d.b, d.m, d.m) : nullptr;
                    else if (d.q == 1) pt = lane == 0 ? tile(G.A, G, d.b, d.i, d.m) : lane == 1 ? Dm : nullptr;
                    else if (d.q == 2 || d.q == 5 || d.q == 6) {
                        if (lane < 3 || d.q == 6)
                            pt = tile(G.A, G, d.b, lane == 2 ? d.i : (lane == 1 || lane == 4) ? d.j : d.i,
                                      lane == 2 ? d.j : ml);
                    } else if (d.q == 3) pt = lane == 0 ? tile(G.Y, G, d.b, d.j, d.m) : lane == 1 ? Dm : nullptr;
                    else if (lane < 3 || d.q == 7)
                        pt = (lane == 0 || lane == 3) ? tile(G.Y, G, d.b, d.j, ml)
                             : (lane == 1 || lane == 4) ? tile(G.A, G, d.b, d.i, ml) : tile(G.Y, G, d.b, d.j, d.i);
                    if (pt) prefetch_l2(pt, TILE_ELEMS * sizeof(double));
                }
                if (lane < 3) {   // (selects, not an indexed local array)
                    wpl = lane == 0 ? dp.wp[0] : lane == 1 ? dp.wp[1] : dp.wp[2];
                    wtl = lane == 0 ? dp.wt[0] : lane == 1 ? dp.wt[1] : dp.wt[2];
                }
                const bool ready = !wpl || ld_acquire(wpl) >= wtl;
                d.status = __all_sync(0xffffffffu, ready) ? READY : WAIT;
            }
            if (lane == 0) s_task[slot] = d;
            __syncwarp();
            __syncthreads();   // end of the running task; the compute warps read s_task[slot]
            if (lane == 0 && run_out) {
                if (run_out2) st_release(run_out2, 1);
                st_release(run_out, run_value);
            }
            if (d.status == WAIT) {
                bool ok = !wpl || wait_ge(wpl, wtl, g, g.grp[d.k].pbase + d.b);
                ok = __all_sync(0xffffffffu, ok);
                if (lane == 0) s_final[slot] = ok ? READY : STOP;
                __syncwarp();
                __syncthreads();   // the compute warps read the final status
                if (!ok) break;
            } else if (d.status == STOP) {
                break;
            }
            run_out = dp.out;
            run_out2 = dp.out2;
            run_value = dp.out_value;
            slot ^= 1;
        }
        return;
    }

    // -------------------------------------------------------------------- compute (warps 0-7)
    int slot = 0;
    for (;;) {
        __syncthreads();   // the scheduler has published the next task
        Task d = s_task[slot];
        if (d.status == WAIT) {
            __syncthreads();
            d.status = s_final[slot];
        }
        if (d.status != READY) break;
        slot ^= 1;
        const Grp& G = g.grp[d.k];
        const int q = d.q, b = d.b, m = d.m, i = d.i, j = d.j;
        double* Dm = G.D + ((size_t)b * G.nt + m) * TILE_ELEMS;
        if (q == 0) {            // P(m)
            tile_to_smem(T0, tile(G.A, G, b, m, m));
            cp_async_wait_all();
            cbar();
            tile_potrf_inv(T0, reinterpret_cast<double*>(T1), scr, tile(G.A, G, b, m, m), Dm, tile(G.Y, G, b, m, m),
                           g.err, G.pbase + b, NB * m, G.d);
        } else if (q == 1) {     // L_im = A_im D_m^T
            tile_gemm_nt(tile(G.A, G, b, i, m), Dm, T0, T1, tile(G.A, G, b, i, m), false, false);
        } else if (q == 2 || q == 5) {   // A_ij -= L_im L_jm^T
            tile_gemm_nt(tile(G.A, G, b, i, m), tile(G.A, G, b, j, m), T0, T1, tile(G.A, G, b, i, j), true, true);
        } else if (q == 6) {     // A_ij -= L_{i,m-1} L_{j,m-1}^T + L_im L_jm^T
            tile_gemm_nt(tile(G.A, G, b, i, m - 1), tile(G.A, G, b, j, m - 1), T0, T1, tile(G.A, G, b, i, j), true,
                         true, tile(G.A, G, b, i, m), tile(G.A, G, b, j, m));
        } else if (q == 3) {     // Y_jm = -R_jm D_m^T
            tile_gemm_nt(tile(G.Y, G, b, j, m), Dm, T0, T1, tile(G.Y, G, b, j, m), false, true);
        } else if (q == 7) {     // R_ji (+)= Y_{j,m-1} L_{i,m-1}^T + Y_jm L_im^T (level j's term starts R_ji)
            tile_gemm_nt(tile(G.Y, G, b, j, m - 1), tile(G.A, G, b, i, m - 1), T0, T1, tile(G.Y, G, b, j, i),
                         m - 1 != j, false, tile(G.Y, G, b, j, m), tile(G.A, G, b, i, m));
        } else {                 // R_ji (+)= Y_jm L_im^T
            tile_gemm_nt(tile(G.Y, G, b, j, m), tile(G.A, G, b, i, m), T0, T1, tile(G.Y, G, b, j, i), m != j, false);
        }
        // the barrier at the top of the loop ends the task: every compute thread's stores are issued
        // before the scheduler's release, and the shared tiles are free for the next task's copies
    }
}

constexpr size_t dag_smem_bytes(int nt) {
    return (size_t)(2 * TILE_DOUBLES + P_SCRATCH) * sizeof(double) + (size_t)(nt + 2) * sizeof(unsigned long long);
}

// ------------------------------------------------------------------------------ the F form
// X^T of the 128-block (p, p+1), p = 2 blockIdx.x, into the tile Y_{p,p+1} (unused without the
// inverse): T = Y_pp L_{p+1,p}^T = (L_{p+1,p} D_p)^T, then Y_{p,p+1} = -T D_{p+1}^T = X^T.
constexpr size_t PAIR_SMEM = 2 * TILE_DOUBLES * sizeof(double);
__global__ void __launch_bounds__(256) fac_pair(Grp G) {
    extern __shared__ double dsm[];
    Tile* Ps = reinterpret_cast<Tile*>(dsm);
    Tile* Qs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    const int b = blockIdx.y, p = 2 * blockIdx.x;
    double* Yx = tile(G.Y, G, b, p, p + 1);
    tile_gemm_nt(tile(G.Y, G, b, p, p), tile(G.A, G, b, p + 1, p), Ps, Qs, Yx, false, false);
    __threadfence();   // T reaches L2, where the next product's copies read it
    cbar();
    tile_gemm_nt(Yx, G.D + ((size_t)b * G.nt + p + 1) * TILE_ELEMS, Ps, Qs, Yx, false, true);
}

// F tile (ta, tc), ta <= tc, is the 180-degree rotation of the tile (it, jt) = (nt-1-ta, nt-1-tc) of
// J F J = L blockdiag(L_bb^-1): D_jt on the diagonal; for even jt, X at it = jt + 1 and
// L_{it,jt} D_jt + L_{it,jt+1} X below; for odd jt, L_{it,jt} D_jt below. The tile is formed in shared
// memory (products on the FP64 tensor path) and written as float32; tiles below the diagonal are zero.
constexpr size_t STORE_F_SMEM = 3 * TILE_DOUBLES * sizeof(double);
__global__ void __launch_bounds__(256) fac_store_f(Grp G, float* __restrict__ F) {
    extern __shared__ double dsm[];
    Tile* Ps = reinterpret_cast<Tile*>(dsm);
    Tile* Qs = reinterpret_cast<Tile*>(dsm + TILE_DOUBLES);
    Tile* Os = reinterpret_cast<Tile*>(dsm + 2 * TILE_DOUBLES);
    const int b = blockIdx.y, nt = G.nt, d = G.d;
    const int ta = blockIdx.x / nt, tc = blockIdx.x % nt;
    float* Fb = F + (size_t)b * d * d;
    if (ta > tc) {
        for (int e = threadIdx.x; e < TILE_ELEMS; e += 256)
            Fb[(size_t)(NB * ta + (e >> 6)) * d + NB * tc + (e & 63)] = 0.f;
        return;
    }
    const int it = nt - 1 - ta, jt = nt - 1 - tc;
    const double* Yjj = tile(G.Y, G, b, jt, jt);   // D_jt^T
    if (it == jt) {
        const double* Dj = G.D + ((size_t)b * nt + jt) * TILE_ELEMS;
        for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) Os[e >> 6][e & 63] = __ldcg(Dj + e);
    } else if ((jt & 1) == 0 && it == jt + 1) {
        const double* Yx = tile(G.Y, G, b, jt, jt + 1);
        for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) Os[e & 63][e >> 6] = __ldcg(Yx + e);
    } else if ((jt & 1) == 0) {
        tile_gemm_nt(tile(G.A, G, b, it, jt), Yjj, Ps, Qs, &Os[0][0], false, false, tile(G.A, G, b, it, jt + 1),
                     tile(G.Y, G, b, jt, jt + 1), LD);
    } else {
        tile_gemm_nt(tile(G.A, G, b, it, jt), Yjj, Ps, Qs, &Os[0][0], false, false, nullptr, nullptr, LD);
    }
    __syncthreads();
    for (int e = threadIdx.x; e < TILE_ELEMS; e += 256) {
        const int ra = e >> 6, rc = e & 63;
        const float v = (ta == tc && ra > rc) ? 0.f : (float)Os[63 - ra][63 - rc];
        Fb[(size_t)(NB * ta + ra) * d + NB * tc + rc] = v;
    }
}

}  // namespace

namespace {
size_t group_bytes(const FactorGroup& gr, size_t* states) {
    const size_t nt = (size_t)gr.d / NB;
    const size_t tiles = (size_t)gr.batch * nt * nt;
    *states = 2 * tiles * sizeof(int);
    return 2 * clha_round_up(tiles * TILE_ELEMS * sizeof(double)) +
           clha_round_up((size_t)gr.batch * nt * TILE_ELEMS * sizeof(double));
}
}  // namespace

size_t factor_workspace_bytes(const FactorGroup* groups, int n) {
    size_t total = 0, states = 2 * sizeof(unsigned long long);
    for (int k = 0; k < n; ++k) {
        size_t s;
        total += group_bytes(groups[k], &s);
        states += s;
    }
    return total + clha_round_up(states);
}

cudaError_t launch_factor(cudaStream_t s, int num_sms, const FactorGroup* groups, int n, void* ws, int* err,
                          uint64_t wait_ns, int form) {
    if (n < 1 || n > MAX_GROUPS || (form != 0 && form != 1)) return cudaErrorInvalidValue;
    char* cur = (char*)ws;
    Dag g;
    g.ng = n;
    g.max_nt = 0;
    g.err = err;
    g.wait_ns = wait_ns;
    g.inv = form == 0;
    size_t state_bytes = 2 * sizeof(unsigned long long);
    int pbase = 0;
    for (int k = 0; k < n; ++k) {
        const FactorGroup& gr = groups[k];
        const int nt = gr.d / NB;
        const size_t tiles = (size_t)gr.batch * nt * nt;
        Grp& G = g.grp[k];
        G.A = (double*)clha_carve(cur, tiles * TILE_ELEMS * sizeof(double));
        G.Y = (double*)clha_carve(cur, tiles * TILE_ELEMS * sizeof(double));
        G.D = (double*)clha_carve(cur, (size_t)gr.batch * nt * TILE_ELEMS * sizeof(double));
        G.nt = nt;
        G.batch = gr.batch;
        G.d = gr.d;
        G.pbase = pbase;
        pbase += gr.batch;
        state_bytes += 2 * tiles * sizeof(int);
        if (nt > g.max_nt) g.max_nt = nt;
    }
    for (int k = n; k < MAX_GROUPS; ++k) g.grp[k] = g.grp[0];
    char* sts = (char*)clha_carve(cur, state_bytes);   // task counter, abort flag, every group's states
    g.ticket = (unsigned long long*)sts;
    g.abort_flag = (int*)(sts + sizeof(unsigned long long));
    int* st_cur = (int*)(sts + 2 * sizeof(unsigned long long));
    g.total = 0;
    for (int k = 0; k < n; ++k) {
        Grp& G = g.grp[k];
        const size_t tiles = (size_t)G.batch * G.nt * G.nt;
        G.stA = st_cur;
        G.stY = st_cur + tiles;
        st_cur += 2 * tiles;
        unsigned long long per = 0;
        for (int st = 0; st <= G.nt; ++st) per += stage_total(G.nt, st, g.inv);
        g.total += per * (unsigned long long)G.batch;
    }

    // the kernel decodes a task's place inside its stage in 32-bit arithmetic
    for (int st = 0; st <= g.max_nt; ++st) {
        unsigned long long tasks = 0;
        for (int k = 0; k < n; ++k) {
            const int nt = g.grp[k].nt;
            if (st > nt) continue;
            tasks += stage_total(nt, st, g.inv) * (unsigned long long)g.grp[k].batch;
        }
        if (tasks >= (1ull << 31)) return cudaErrorInvalidValue;
    }
    const size_t smem = dag_smem_bytes(g.max_nt);
    cudaError_t e = cudaFuncSetAttribute(fac_dag, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    if ((e = cudaMemsetAsync(sts, 0, state_bytes, s)) != cudaSuccess) return e;
    for (int k = 0; k < n; ++k) {
        const Grp& G = g.grp[k];
        fac_load<<<dim3((unsigned)(G.nt * (G.nt + 1) / 2), G.batch), 256, 0, s>>>(groups[k].H, G.d, G.nt, G.A);
        clha_note_launches(1);
    }
    unsigned long long grid = 2ull * (unsigned long long)num_sms;   // two resident CTAs per SM
    if (grid > g.total) grid = g.total;
    fac_dag<<<(unsigned)grid, DAG_THREADS, smem, s>>>(g);
    clha_note_launches(1);
    if (form == 0) {
        for (int k = 0; k < n; ++k) {
            const Grp& G = g.grp[k];
            fac_store<<<dim3((unsigned)(G.nt * G.nt), G.batch), 256, 0, s>>>(G.Y, G.d, G.nt, groups[k].U);
            clha_note_launches(1);
        }
        return cudaGetLastError();
    }
    if ((e = cudaFuncSetAttribute(fac_pair, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)PAIR_SMEM)) != cudaSuccess)
        return e;
    if ((e = cudaFuncSetAttribute(fac_store_f, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)STORE_F_SMEM)) !=
        cudaSuccess)
        return e;
    for (int k = 0; k < n; ++k) {   // d is a multiple of 128: nt is even
        const Grp& G = g.grp[k];
        fac_pair<<<dim3((unsigned)(G.nt / 2), G.batch), 256, PAIR_SMEM, s>>>(G);
        fac_store_f<<<dim3((unsigned)(G.nt * G.nt), G.batch), 256, STORE_F_SMEM, s>>>(G, groups[k].U);
        clha_note_launches(2);
    }
    return cudaGetLastError();
}
