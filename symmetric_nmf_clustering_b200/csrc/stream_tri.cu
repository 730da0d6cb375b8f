// Upper-triangle S-stream: Y = S X for a symmetric S, reading only the
// 128 x 128 tiles S[p, q] with p <= q (half of the n^2 entries).
//
// The scope of the hot path allows the S-stream to read only the upper
// triangle and exploit symmetry; the pages' S H product ([CaS] "Factorization
// at scale": the dominant S H multiplications) streams the full matrix.  Each
// tile S[p, q] read once feeds two products:
//     forward     Y_p += S[p, q] X_q
//     transposed  Y_q += S[p, q]^T X_p      (= S[q, p] X_p; skipped when p = q)
//
// Precision.  Both products run on the 5th-generation tensor cores (kind::tf32)
// with X entering as its exact split [X_hi; X_lo] (as in the full-matrix
// stream).  S enters rounded to the nearest TF32 value (the split warps add
// half a TF32 unit to the fp32 bit pattern, the tensor core drops the 13 low
// mantissa bits): an unbiased per-entry error of at most 2^-12 relative,
// which averages out over a row of S (measured on the |corr| and TPDM
// workloads: 3e-6 to 8e-6 relative in S X at n = 2,000 to 12,000); a
// matrix whose entries all round the same way sees up to 2^-12.  The full-
// matrix stream keeps the exact three-product split instead.
//
// Why the transposed tile goes through tensor memory.  The transposed product
// needs the tile with its column index as the MMA's M dimension.  A TF32
// operand in shared memory read M-major must use the 32-byte-atom swizzle,
// while the forward product reads the same tile K-major in the 16-byte-chunk
// 128-byte swizzle; one copy cannot serve both.  So the split warps write the
// rounded tile transposed into tensor memory (lane = column), the A operand
// of the transposed MMA, and round the shared-memory copy in place for the
// forward MMA.
//
// Work decomposition.  Row tiles are grouped in panels of TR_PANEL; a work
// item is one panel times a run of C column tiles q >= the panel's
// first row tile, visited q-outer, p-inner (p <= q).  Per tile pair both
// accumulators are drained into registers: forward rows accumulate over the
// item in registers (one partial slab per item and panel row), transposed
// rows over the panel's row tiles (one partial slab per panel and q).  A
// second kernel sums every slab of a row tile in a fixed order, so results are
// bitwise reproducible.  Persistent CTAs (one per SM) take items b, b + G, ...
//
// Per CTA (256 threads):
//   warp 0      TMA producer: the tile (4 boxes of 128 rows x 32 columns,
//               128-byte swizzle), the X_p operand (4 boxes of 2KP x 32) per
//               tile pair; the X_q operand once per column tile
//   warp 1      forward MMA issuer (A = the rounded tile, shared memory)
//   warp 2      tensor-memory allocator
//   warp 3      transposed MMA issuer (A = the rounded tile^T, tensor memory)
//   warps 4-7   warp 4 + s owns the tile's column box s: lane j reads column
//               j, rounds it, writes it back in place (forward operand) and
//               into tensor-memory lane 32 s + j (transposed operand); then
//               drains both accumulators of the previous
//               tile pair (thread r = accumulator lane r) and writes the
//               partial slabs
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "sm100.cuh"

namespace symnmf {

int make_map(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld,
             uint32_t box_rows);   // stream_tc.cu

// Test hook (symnmf_test_stall_pipeline): the producer issues no loads.
__device__ int g_tri_stall = 0;

constexpr int TR_BM = 128;         // tile edge
constexpr int TR_BK = 32;          // columns per TMA box (128 bytes of fp32)
constexpr int TR_PANEL = 4;        // row tiles per panel
constexpr int TR_CHUNK_MAX = 16;   // column tiles per work item (fewer when the items would be too few)
constexpr int TR_THREADS = 256;
#ifndef SYMNMF_TRI_PREFETCH
#define SYMNMF_TRI_PREFETCH 4
#endif
constexpr int TR_PREFETCH = SYMNMF_TRI_PREFETCH;   // tile pairs prefetched into L2 ahead of the loads
constexpr uint32_t TR_BOX = TR_BM * TR_BK * 4;    // 16 KB
constexpr uint32_t TR_TILE = 4 * TR_BOX;          // 64 KB

template <int KP>
struct TrCfg {
    static constexpr int N = 2 * KP;                          // [X_hi ; X_lo] rows
    static constexpr uint32_t XBOX = N * TR_BK * 4;           // one 2KP x 32 box
    static constexpr uint32_t XTILE = 4 * XBOX;               // 128 columns
    static constexpr uint32_t DCOLS = (N + 31) / 32 * 32;     // accumulator slot
    static constexpr uint32_t COL_DF = 0;                     // 2 forward accumulators
    static constexpr uint32_t COL_DT = 2 * DCOLS;             // 2 transposed accumulators
    static constexpr uint32_t COL_ST = 256;                   // 2 transposed tiles, 128 columns each
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t OFF_XQ = 2 * TR_TILE;
    static constexpr uint32_t OFF_XP = OFF_XQ + 2 * XTILE;
    static constexpr uint32_t SMEM = OFF_XP + 2 * XTILE + 1024;
    static_assert(4 * DCOLS <= COL_ST, "accumulators below the transposed tiles");
    static_assert(XBOX % 1024 == 0, "operand boxes stay 1024-byte aligned");
    static_assert(SMEM <= 232448 - 1024, "fits one CTA per SM");
};

// ---------------------------------------------------------------- schedule
__host__ __device__ __forceinline__ int tr_chunks(int T, int C, int P) {
    return (T - TR_PANEL * P + C - 1) / C;
}
// index of the transposed slab of panel P and column tile q (q >= TR_PANEL P):
// panels' slabs are stored one after another, panel P holding T - 4P of them
__host__ __device__ __forceinline__ int64_t tr_tslab(int T, int P, int q) {
    return (int64_t)P * T - (int64_t)(TR_PANEL / 2) * P * (P - 1) + (q - TR_PANEL * P);
}
__host__ __device__ __forceinline__ int tr_panels(int T) { return (T + TR_PANEL - 1) / TR_PANEL; }

// geometry of work item `item`; (P, pbase) advance monotonically over calls
// with increasing items
__device__ __forceinline__ void tr_item(int T, int C, int item, int& P, int& pbase, int& qa,
                                        int& qb, int& pr0, int& pr1) {
    while (item >= pbase + tr_chunks(T, C, P)) {
        pbase += tr_chunks(T, C, P);
        ++P;
    }
    qa = TR_PANEL * P + (item - pbase) * C;
    qb = min(T, qa + C);
    pr0 = TR_PANEL * P;
    pr1 = min(T, pr0 + TR_PANEL);
}

// A position in a CTA's sequence of tile pairs (items b, b + G, ...; q-outer,
// p-inner), advanced one tile pair at a time.
struct TrCursor {
    int T, C, items, stride, item, P, pbase, qa, qb, pr0, pr1, q, p;
    bool valid;
    __device__ __forceinline__ void start(int T_, int C_, int items_, int first, int stride_) {
        T = T_;
        C = C_;
        items = items_;
        stride = stride_;
        item = first;
        P = 0;
        pbase = 0;
        valid = item < items;
        if (valid) {
            tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
            q = qa;
            p = pr0;
        }
    }
    __device__ __forceinline__ void next() {
        if (++p < min(pr1, q + 1)) return;
        if (++q < qb) {
            p = pr0;
            return;
        }
        item += stride;
        valid = item < items;
        if (!valid) return;
        tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
        q = qa;
        p = pr0;
    }
};

__device__ __forceinline__ void tr_fail(int* err, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    if (err != nullptr) atomicExch(err, code);
}

// Shared-memory descriptor of a tile box read K-major (128-byte swizzle).
__device__ __forceinline__ uint64_t tr_desc(uint32_t saddr) { return sm100::umma_desc_sw128(saddr); }

template <int KP>
__global__ void __launch_bounds__(TR_THREADS, 1)
stream_tri_kernel(const __grid_constant__ CUtensorMap mapS, const __grid_constant__ CUtensorMap mapX,
                  int T, int C, int items, int k, float* __restrict__ tpart,
                  float* __restrict__ fpart, int* __restrict__ err, const FitState* st) {
    using Cfg = TrCfg<KP>;
    using namespace sm100;
    pdl_wait();
    if (st != nullptr && st->done) return;

    extern __shared__ uint8_t tr_smem_raw[];
    __shared__ __align__(8) uint64_t b_sfull[2], b_xqfull[2], b_ready[2], b_done_f[2], b_done_t[2];
    __shared__ __align__(8) uint64_t b_dfree_f[2], b_dfree_t[2], b_xqfree[2], b_fin[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(tr_smem_raw) + 1023) & ~uintptr_t(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    if (tid == 0) {
        for (int b = 0; b < 2; ++b) {
            mbar_init(&b_sfull[b], 1);
            mbar_init(&b_xqfull[b], 1);
            mbar_init(&b_ready[b], 4);      // one arrival per split warp
            mbar_init(&b_done_f[b], 1);
            mbar_init(&b_done_t[b], 1);
            mbar_init(&b_dfree_f[b], 4);
            mbar_init(&b_dfree_t[b], 4);
            mbar_init(&b_xqfree[b], 1);
            mbar_init(&b_fin[b], 1);
        }
        abort_sh = 0;
        fence_mbar_init();
        prefetch_tmap(&mapS);
        prefetch_tmap(&mapX);
    }
    if (warp == 2) {
        tmem_alloc(&tmem_base_sh, Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base_sh;

    if (warp == 0 && lane == 0 && *(volatile int*)&g_tri_stall == 0) {
        // ---------------------------------------------------------------- producer
        const uint64_t pol_s = policy_evict_first();
        const uint64_t pol_x = policy_evict_last();
        // the tiles TR_PREFETCH tile pairs ahead are prefetched into L2, so the
        // loads into the two shared-memory slots find them there: the HBM
        // latency is covered without more shared memory
        TrCursor ahead;
        ahead.start(T, C, items, blockIdx.x, gridDim.x);
        for (int d = 0; d < TR_PREFETCH && ahead.valid; ++d, ahead.next())
            for (int s = 0; s < 4; ++s) tma_prefetch_2d(&mapS, ahead.q * TR_BM + s * TR_BK, ahead.p * TR_BM);
        uint32_t u = 0, g = 0;   // tile pairs and column groups issued so far
        int P = 0, pbase = 0;
        for (int item = blockIdx.x; item < items && !abort_sh; item += gridDim.x) {
            int qa, qb, pr0, pr1;
            tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
            for (int q = qa; q < qb && !abort_sh; ++q) {
                const uint32_t xs = g & 1u;
                if (g >= 2 && !mbar_wait(&b_xqfree[xs], ((g - 2) >> 1) & 1u)) {
                    tr_fail(err, &abort_sh, 11);
                    break;
                }
                mbar_arrive_expect_tx(&b_xqfull[xs], Cfg::XTILE);
                for (int s = 0; s < 4; ++s)
                    tma_load_2d_hint(smem + Cfg::OFF_XQ + xs * Cfg::XTILE + s * Cfg::XBOX, &mapX,
                                     q * TR_BM + s * TR_BK, 0, &b_xqfull[xs], pol_x);
                ++g;
                const int pe = min(pr1, q + 1);
                for (int p = pr0; p < pe; ++p) {
                    const uint32_t ss = u & 1u;
                    if (u >= 2) {
                        const uint32_t ph = ((u - 2) >> 1) & 1u;
                        if (!(mbar_wait(&b_done_f[ss], ph) && mbar_wait(&b_done_t[ss], ph))) {
                            tr_fail(err, &abort_sh, 12);
                            break;
                        }
                    }
                    mbar_arrive_expect_tx(&b_sfull[ss], TR_TILE + Cfg::XTILE);
                    for (int s = 0; s < 4; ++s)
                        tma_load_2d_hint(smem + ss * TR_TILE + s * TR_BOX, &mapS, q * TR_BM + s * TR_BK,
                                         p * TR_BM, &b_sfull[ss], pol_s);
                    for (int s = 0; s < 4; ++s)
                        tma_load_2d_hint(smem + Cfg::OFF_XP + ss * Cfg::XTILE + s * Cfg::XBOX, &mapX,
                                         p * TR_BM + s * TR_BK, 0, &b_sfull[ss], pol_x);
                    if (ahead.valid) {
                        for (int s = 0; s < 4; ++s)
                            tma_prefetch_2d(&mapS, ahead.q * TR_BM + s * TR_BK, ahead.p * TR_BM);
                        ahead.next();
                    }
                    ++u;
                }
            }
        }
        if (abort_sh) {
            // let the copies already issued land before the CTA exits: the most
            // recent phase of each slot's barriers is the one still in flight
            for (uint32_t v = (u >= 2 ? u - 2 : 0); v < u; ++v)
                mbar_wait(&b_sfull[v & 1u], (v >> 1) & 1u);
            for (uint32_t h = (g >= 2 ? g - 2 : 0); h < g; ++h)
                mbar_wait(&b_xqfull[h & 1u], (h >> 1) & 1u);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------------------------------------------------------- forward MMAs
        constexpr uint32_t idF = idesc_tf32(TR_BM, Cfg::N);
        uint32_t u = 0, g = 0;
        int P = 0, pbase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            int qa, qb, pr0, pr1;
            tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
            for (int q = qa; q < qb && ok; ++q, ++g) {
                const uint32_t xs = g & 1u;
                const int pe = min(pr1, q + 1);
                for (int p = pr0; p < pe; ++p, ++u) {
                    const uint32_t ss = u & 1u, ph = (u >> 1) & 1u;
                    if (abort_sh) { ok = false; break; }
                    ok = mbar_wait(&b_sfull[ss], ph) && mbar_wait(&b_ready[ss], ph) &&
                         (p != pr0 || mbar_wait(&b_xqfull[xs], (g >> 1) & 1u)) &&
                         (u < 2 || mbar_wait(&b_dfree_f[ss], ((u - 2) >> 1) & 1u));
                    if (!ok) {
                        tr_fail(err, &abort_sh, 13);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t a0 = smem_u32(smem + ss * TR_TILE);
                    const uint32_t b0 = smem_u32(smem + Cfg::OFF_XQ + xs * Cfg::XTILE);
                    const uint32_t d = tbase + Cfg::COL_DF + ss * Cfg::DCOLS;
#pragma unroll
                    for (int s = 0; s < 4; ++s)
#pragma unroll
                        for (int kk = 0; kk < TR_BK / 8; ++kk)
                            umma_tf32_ss(d, tr_desc(a0 + s * TR_BOX + kk * 32),
                                         tr_desc(b0 + s * Cfg::XBOX + kk * 32), idF, (s | kk) ? 1u : 0u);
                    umma_commit(&b_done_f[ss]);
                    if (p == pe - 1) umma_commit(&b_xqfree[xs]);   // X_q no longer read
                }
            }
        }
        if (!ok) {   // MMAs in flight finish before tensor memory is freed
            umma_commit(&b_fin[0]);
            mbar_wait(&b_fin[0], 0);
        }
    } else if (warp == 3 && lane == 0) {
        // ---------------------------------------------------------------- transposed MMAs
        constexpr uint32_t idT = idesc_tf32(TR_BM, Cfg::N);
        uint32_t u = 0;
        int P = 0, pbase = 0;
        bool ok = true;
        for (int item = blockIdx.x; item < items && ok; item += gridDim.x) {
            int qa, qb, pr0, pr1;
            tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
            for (int q = qa; q < qb && ok; ++q) {
                const int pe = min(pr1, q + 1);
                for (int p = pr0; p < pe; ++p, ++u) {
                    const uint32_t ss = u & 1u, ph = (u >> 1) & 1u;
                    if (abort_sh) { ok = false; break; }
                    ok = mbar_wait(&b_sfull[ss], ph) && mbar_wait(&b_ready[ss], ph) &&
                         (u < 2 || mbar_wait(&b_dfree_t[ss], ((u - 2) >> 1) & 1u));
                    if (!ok) {
                        tr_fail(err, &abort_sh, 14);
                        break;
                    }
                    tc_fence_after();
                    const uint32_t b0 = smem_u32(smem + Cfg::OFF_XP + ss * Cfg::XTILE);
                    const uint32_t a = tbase + Cfg::COL_ST + ss * 128u;
                    const uint32_t d = tbase + Cfg::COL_DT + ss * Cfg::DCOLS;
#pragma unroll
                    for (int kk = 0; kk < TR_BM / 8; ++kk)
                        umma_tf32_ts(d, a + kk * 8u, tr_desc(b0 + (kk >> 2) * Cfg::XBOX + (kk & 3) * 32),
                                     idT, kk ? 1u : 0u);
                    umma_commit(&b_done_t[ss]);
                }
            }
        }
        if (!ok) {
            umma_commit(&b_fin[1]);
            mbar_wait(&b_fin[1], 0);
        }
    } else if (warp >= 4) {
        // ---------------------------------------------------------------- split + drain warps
        const int w4 = warp & 3;                   // tensor-memory lane quarter and column box
        const int r = w4 * 32 + lane;              // accumulator lane = row of the output tile
        const uint32_t lane_off = (uint32_t)(w4 * 32) << 16;
        float acc_f[TR_PANEL][KP], acc_t[KP];
#pragma unroll
        for (int a = 0; a < TR_PANEL; ++a)
#pragma unroll
            for (int c = 0; c < KP; ++c) acc_f[a][c] = 0.f;
#pragma unroll
        for (int c = 0; c < KP; ++c) acc_t[c] = 0.f;
        // swizzled byte offset of element (row i, column lane) of a box, for i mod 8 = b
        uint32_t col_off[8];
#pragma unroll
        for (int b = 0; b < 8; ++b) col_off[b] = (uint32_t)(b * 128 + ((((lane >> 2) ^ b) & 7) << 4) + (lane & 3) * 4);

        // previous tile pair (drained one step behind)
        bool have_prev = false;
        uint32_t pv_u = 0;
        int pv_p = 0, pv_q = 0, pv_pr0 = 0, pv_P = 0, pv_item = 0;
        bool pv_last_p = false, pv_last_item = false;
        bool alive = true;

        auto drain = [&]() -> bool {
            const uint32_t ss = pv_u & 1u, ph = (pv_u >> 1) & 1u;
            if (!__all_sync(0xffffffffu, mbar_wait(&b_done_f[ss], ph))) return false;
            tc_fence_after();
            uint32_t v[2 * KP / 8][8];
#pragma unroll
            for (int q8 = 0; q8 < 2 * KP / 8; ++q8)
                tmem_ld_32x32b_x8(tbase + lane_off + Cfg::COL_DF + ss * Cfg::DCOLS + q8 * 8u, v[q8]);
            tmem_wait_ld();
            const int pp = pv_p - pv_pr0;
#pragma unroll
            for (int a = 0; a < TR_PANEL; ++a)
                if (a == pp) {
#pragma unroll
                    for (int c = 0; c < KP; ++c)
                        acc_f[a][c] += __uint_as_float(v[c / 8][c % 8]) + __uint_as_float(v[(KP + c) / 8][c % 8]);
                }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_dfree_f[ss]);
            if (!__all_sync(0xffffffffu, mbar_wait(&b_done_t[ss], ph))) return false;
            tc_fence_after();
#pragma unroll
            for (int q8 = 0; q8 < 2 * KP / 8; ++q8)
                tmem_ld_32x32b_x8(tbase + lane_off + Cfg::COL_DT + ss * Cfg::DCOLS + q8 * 8u, v[q8]);
            tmem_wait_ld();
            if (pv_p < pv_q) {   // the diagonal tile contributes once, through the forward product
#pragma unroll
                for (int c = 0; c < KP; ++c)
                    acc_t[c] += __uint_as_float(v[c / 8][c % 8]) + __uint_as_float(v[(KP + c) / 8][c % 8]);
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&b_dfree_t[ss]);
            if (pv_last_p) {   // every row tile of the panel has met column tile q
                float* o = tpart + (tr_tslab(T, pv_P, pv_q) * TR_BM + r) * (int64_t)k;
#pragma unroll
                for (int c = 0; c < KP; ++c) {
                    if (c < k) o[c] = acc_t[c];
                    acc_t[c] = 0.f;
                }
            }
            if (pv_last_item) {   // the item's forward rows are complete
#pragma unroll
                for (int a = 0; a < TR_PANEL; ++a) {
                    float* o = fpart + (((int64_t)pv_item * TR_PANEL + a) * TR_BM + r) * (int64_t)k;
#pragma unroll
                    for (int c = 0; c < KP; ++c) {
                        if (c < k) o[c] = acc_f[a][c];
                        acc_f[a][c] = 0.f;
                    }
                }
            }
            return true;
        };

        uint32_t u = 0;
        int P = 0, pbase = 0;
        for (int item = blockIdx.x; item < items && alive; item += gridDim.x) {
            int qa, qb, pr0, pr1;
            tr_item(T, C, item, P, pbase, qa, qb, pr0, pr1);
            for (int q = qa; q < qb && alive; ++q) {
                const int pe = min(pr1, q + 1);
                for (int p = pr0; p < pe; ++p, ++u) {
                    const uint32_t ss = u & 1u;
                    if (__any_sync(0xffffffffu, abort_sh != 0)) {
                        alive = false;
                        break;
                    }
                    if (!__all_sync(0xffffffffu, mbar_wait(&b_sfull[ss], (u >> 1) & 1u))) {
                        if (lane == 0) tr_fail(err, &abort_sh, 15);
                        alive = false;
                        break;
                    }
                    // transposed copy of box w4: lane j = 32 w4 + lane of the MMA's
                    // M dimension gets column j over the tile's 128 rows, rounded;
                    // the same lane writes the rounded value back in place for the
                    // forward MMA (each element is read and written by one lane
                    // only).  A warp's access touches one 128-byte row: no bank
                    // conflicts.
                    const uint32_t tcol = tbase + lane_off + Cfg::COL_ST + ss * 128u;
                    uint32_t* boxp = reinterpret_cast<uint32_t*>(smem + ss * TR_TILE + w4 * TR_BOX);
#pragma unroll
                    for (int ic = 0; ic < 8; ++ic) {
                        // all sixteen loads go out before the first store
                        uint32_t x[16];
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int i = ic * 16 + t;
                            x[t] = boxp[((i >> 3) * 1024 + col_off[i & 7]) >> 2] + 0x1000u;
                        }
#pragma unroll
                        for (int t = 0; t < 16; ++t) {
                            const int i = ic * 16 + t;
                            boxp[((i >> 3) * 1024 + col_off[i & 7]) >> 2] = x[t];
                        }
                        tmem_st_32x32b_x16(tcol + ic * 16u, x);
                    }
                    tmem_wait_st();
                    fence_proxy_async_smem();
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive(&b_ready[ss]);
                    if (have_prev && !drain()) {
                        if (lane == 0) tr_fail(err, &abort_sh, 16);
                        alive = false;
                        break;
                    }
                    have_prev = true;
                    pv_u = u;
                    pv_p = p;
                    pv_q = q;
                    pv_pr0 = pr0;
                    pv_P = P;
                    pv_item = item;
                    pv_last_p = p == pe - 1;
                    pv_last_item = pv_last_p && q == qb - 1;
                }
            }
        }
        if (alive && have_prev && !drain()) {
            if (lane == 0) tr_fail(err, &abort_sh, 17);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, Cfg::TMEM_COLS);
    }
    pdl_trigger();
}

// ----------------------------------------------------------------------------
// Y[t] = sum of the forward slabs of t's panel (item order) + the transposed
// slabs of panels 0..P(t) (panel order).  Block (t, b): TR_RED_THREADS
// consecutive elements e of the row tile's 128 x k block (one thread each, so
// a warp reads 128 contiguous bytes of every slab); eight slabs' loads are in
// flight at once and are added in slab order.
// ----------------------------------------------------------------------------
constexpr int TR_RED_THREADS = 256;
constexpr int TR_RED_BATCH = 8;

__global__ void __launch_bounds__(TR_RED_THREADS)
tri_reduce_kernel(int T, int C, int64_t n, int k, const float* __restrict__ tpart,
                  const float* __restrict__ fpart, float* __restrict__ Y, const FitState* st) {
    pdl_wait();
    pdl_trigger();
    if (st != nullptr && st->done) return;
    const int t = blockIdx.x;
    const int e = blockIdx.y * TR_RED_THREADS + threadIdx.x;   // element of the 128 x k block
    const int rows = (int)min64(TR_BM, n - (int64_t)t * TR_BM);
    if (e >= rows * k) return;
    const int P = t / TR_PANEL, pp = t % TR_PANEL;
    int ib = 0;
    for (int Q = 0; Q < P; ++Q) ib += tr_chunks(T, C, Q);
    const int nf = tr_chunks(T, C, P), nt = P + 1, ns = nf + nt;
    const int64_t slab = (int64_t)TR_BM * k;
    // source of the s-th term: forward slabs first, then transposed slabs
    auto src = [&](int s2) -> const float* {
        return s2 < nf ? fpart + ((int64_t)(ib + s2) * TR_PANEL + pp) * slab + e
                       : tpart + tr_tslab(T, s2 - nf, t) * slab + e;
    };
    float acc = 0.f;
    int s2 = 0;
    for (; s2 + TR_RED_BATCH <= ns; s2 += TR_RED_BATCH) {
        float v[TR_RED_BATCH];
#pragma unroll
        for (int b = 0; b < TR_RED_BATCH; ++b) v[b] = __ldcs(src(s2 + b));
#pragma unroll
        for (int b = 0; b < TR_RED_BATCH; ++b) acc += v[b];
    }
    for (; s2 < ns; ++s2) acc += __ldcs(src(s2));
    Y[(int64_t)t * TR_BM * k + e] = acc;
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
TriPlan plan_stream_tri(const Dev& d, int64_t n, int k) {
    TriPlan p;
    p.n = n;
    p.k = k;
    p.KP = (k + 7) / 8 * 8;
    p.T = (int)((n + TR_BM - 1) / TR_BM);
    const int TP = tr_panels(p.T);
    // the widest items that still give every SM at least four of them
    auto count = [&](int C) {
        int64_t c = 0;
        for (int P = 0; P < TP; ++P) c += tr_chunks(p.T, C, P);
        return c;
    };
    p.C = TR_CHUNK_MAX;
    while (p.C > 1 && count(p.C) < 4 * (int64_t)d.sms) p.C /= 2;
    int64_t slabs = 0;
    for (int P = 0; P < TP; ++P) slabs += p.T - TR_PANEL * P;
    p.items = (int)count(p.C);
    p.tslabs = slabs;
    p.grid = (int)std::min<int64_t>(p.items, d.sms);
    return p;
}

size_t tri_tpart_floats(const TriPlan& p) { return (size_t)p.tslabs * TR_BM * p.k; }
size_t tri_fpart_floats(const TriPlan& p) { return (size_t)p.items * TR_PANEL * TR_BM * p.k; }
bool tri_supported(int k) { return k >= 1 && k <= 24; }

int launch_stream_tri(const TriPlan& p, const float* S, int64_t lds, const float* XT, int64_t ldxt,
                      float* tpart, float* fpart, int* err, const FitState* st, cudaStream_t s) {
    if (!tri_supported(p.k)) {
        set_error("the upper-triangle S-stream supports k <= 24 (k = %d)", p.k);
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    CUtensorMap mapS, mapX;
    SYMNMF_TRY(make_map(&mapS, S, p.n, p.n, lds, TR_BM));
    SYMNMF_TRY(make_map(&mapX, XT, p.n, 2 * p.KP, ldxt, (uint32_t)(2 * p.KP)));
#define SYMNMF_TRI(KP)                                                                        \
    do {                                                                                      \
        auto kern = stream_tri_kernel<KP>;                                                    \
        /* once per process (thread-safe static initialisation) */                            \
        static const cudaError_t attr_rc = cudaFuncSetAttribute(                              \
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TrCfg<KP>::SMEM);         \
        SYMNMF_CUDA_TRY(attr_rc);                                                             \
        SYMNMF_CUDA_TRY(launch_pdl(kern, dim3(p.grid), dim3(TR_THREADS), TrCfg<KP>::SMEM, s,  \
                                   mapS, mapX, p.T, p.C, p.items, p.k, tpart, fpart, err, st)); \
    } while (0)
    switch (p.KP) {
        case 8: SYMNMF_TRI(8); break;
        case 16: SYMNMF_TRI(16); break;
        default: SYMNMF_TRI(24); break;
    }
#undef SYMNMF_TRI
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_tri_reduce(const TriPlan& p, const float* tpart, const float* fpart, float* Y,
                      const FitState* st, cudaStream_t s) {
    const dim3 grid((unsigned)p.T, (unsigned)((TR_BM * p.k + TR_RED_THREADS - 1) / TR_RED_THREADS));
    SYMNMF_CUDA_TRY(launch_pdl(tri_reduce_kernel, grid, dim3(TR_RED_THREADS), 0, s, p.T, p.C, p.n,
                               p.k, tpart, fpart, Y, st));
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int tri_set_stall(int on) {
    const int v = on ? 1 : 0;
    SYMNMF_CUDA_TRY(cudaMemcpyToSymbol(g_tri_stall, &v, sizeof(int)));
    return SYMNMF_OK;
}

}  // namespace symnmf
