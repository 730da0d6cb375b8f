// Tensor-core S-stream: part[s] = S[:, J_s] X[J_s, :] on the 5th-generation
// tensor cores (tcgen05), fp32-accurate through an exact TF32 split.
//
// The pages' hot spot is the S H product that streams S once per iteration
// ([CaS] "Factorization at scale": the dominant S H multiplications).  At
// k = 24 that is 12 flop per byte of S: more fp32 FMA than the CUDA cores
// can issue at HBM speed, so the contraction runs on the tensor cores while
// the kernel stays bound by the HBM read of S.
//
// Accuracy.  TF32 keeps 10 explicit mantissa bits.  Every fp32 value is split
// exactly as x = hi + lo with hi = x with its low 13 mantissa bits cleared and
// lo = x - hi (exact, at most 13 significant bits), and
//     S X = S_hi X_hi + S_hi X_lo + S_lo X_hi + O(2^-22 |S| |X|),
// accumulated in fp32 in TMEM.  hi is a TF32 number, so the product does not
// depend on how the tensor core converts fp32 operands.
//
// Per CTA (256 threads, two CTAs per SM): a 128-row tile of S times the
// contraction range of its split, in stages of 32 columns (128 bytes):
//   warp 0      TMA producer: S tile (128 x 32, 128-byte swizzle) and the
//               matching [X_hi; X_lo] tile (2*KP x 32, K-major) per stage,
//               KP = k rounded up to 8
//   warps 1, 3  MMA issuers (one thread each, alternate chunks of TC_CHUNK
//               stages): per 8-column step, D[:, 0:2KP] += S_hi [X_hi;X_lo]
//               (A = the S tile in shared memory, truncated to TF32 by the
//               tensor core) and D[:, 0:KP] += S_lo X_hi (A = S_lo in TMEM).
//               Issuing a tcgen05 MMA or commit costs the issuing thread tens
//               of cycles, and one thread alone could not keep up with HBM.
//   warp 2      TMEM allocator
//   warps 4-7   split warps: thread r reads row r of the S tile from shared
//               memory, stores its lo plane into TMEM lane r, folds the
//               finished accumulator into fp32 registers every TC_CHUNK
//               stages and writes the partial row
//   all warps   in the last split CTA of the tile, the epilogue (epilogue.cuh):
//               the tile's split partials staged in shared memory by
//               cp.async, then loss terms, gradient, AdaGrad step, Gram
//
// Launch: with programmatic stream serialisation; every CTA waits for the
// previous kernel (griddepcontrol.wait) before it reads anything, and the
// epilogue CTAs, which no longer hold TMEM, let the next kernel be scheduled.
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "sm100.cuh"

namespace symnmf {

// Test hook (symnmf_test_stall_pipeline): when set, the TMA producer issues no
// loads, so the consumers' bounded waits run out and the launch returns its
// error word instead of a result.
__device__ int g_stall_producer = 0;

// Pipeline shape (compile-time).  SYMNMF_TC_A_SMEM = 1: the first MMA reads S
// straight from shared memory; the tensor core truncates fp32 operands to
// TF32, which is exactly S_hi (measured on B200: bit-identical results to
// storing S_hi in TMEM), so only S_lo goes through TMEM.
#ifndef SYMNMF_TC_NS
#define SYMNMF_TC_NS 5
#endif
#ifndef SYMNMF_TC_CHUNK
#define SYMNMF_TC_CHUNK 2
#endif
#ifndef SYMNMF_TC_A_SMEM
#define SYMNMF_TC_A_SMEM 1
#endif
#ifndef SYMNMF_TC_L2HINT   // 1: S loads evict-first, the reused X operand evict-last
#define SYMNMF_TC_L2HINT 1
#endif
constexpr int TC_BM = 128;                  // S rows per tile = TMEM lanes
constexpr int TC_BK = 32;                   // columns per stage (128 bytes of fp32)
constexpr int TC_NS = SYMNMF_TC_NS;         // shared-memory stages
constexpr bool TC_A_SMEM = SYMNMF_TC_A_SMEM != 0;
constexpr int TC_TSTAGE = TC_A_SMEM ? 32 : 64;   // TMEM columns per stage of the split S tile
constexpr int TC_NT = TC_A_SMEM ? 4 : 2;         // TMEM stages of the split S tile
constexpr int TC_CHUNK = SYMNMF_TC_CHUNK;   // stages accumulated in TMEM before a drain
// The two MMA issuers take alternate chunks.  An mbarrier wait checks phase
// parity, so a thread may only wait on a barrier whose phases between its own
// consecutive waits are all its own.  With TC_NT == 2 * TC_CHUNK each issuer
// owns half of the TMEM stage slots (and their tfull barriers); its wait on
// the shared full barrier of a stage comes after its tfull wait, by which
// point the split warps have consumed that phase and no later phase of the
// slot can complete before this issuer's own commit.
static_assert(TC_NT == 2 * TC_CHUNK, "each MMA issuer must own its TMEM stage slots");
// Completion of stage s's MMAs is signalled once, by one tcgen05.commit to
// bar_done[s % TC_NDONE]; the producer (shared-memory slot of stage s - TC_NS),
// the split warps (TMEM slot of stage s - TC_NT) and the drain (last stage of
// a chunk) all wait on it.  Each waiter visits stages in order, and TC_NDONE
// exceeds both ring depths, so no barrier completes a second phase before its
// waiters have seen the first; the split warps reach stage x + TC_NT only after
// stage x completed, so a barrier's phases complete in stage order even though
// two threads issue.
constexpr int TC_NDONE = TC_NS * TC_NT;   // a common multiple of both ring depths
static_assert(TC_NDONE > TC_NS && TC_NDONE > TC_NT && TC_NDONE % TC_NS == 0 && TC_NDONE % TC_NT == 0,
              "stage-completion barriers must outnumber both rings");
constexpr int TC_THREADS = 256;
constexpr uint32_t TC_A_BYTES = TC_BM * TC_BK * 4;

// TMEM columns: two accumulators D0, D1 of 2*KP columns each (32-column
// aligned), then the
// TC_NT stages of the split S tile (32 hi + 32 lo columns each).
template <int KP>
struct TcCfg {
    // An MMA with M = 128 and A in TMEM needs N to be a multiple of 16.  N1 = 2 KP
    // always is; N2 rounds KP up, and when it does the extra 8 rows of B are the
    // first 8 rows of X_lo, so D[:, KP:KP+8] also collects S_lo X_lo for those
    // columns -- a correct (smaller-order) term that the drain keeps.
    static constexpr int N1 = 2 * KP;                       // [X_hi ; X_lo]
    static constexpr int N2 = (KP + 15) / 16 * 16;          // X_hi (+ 8 rows of X_lo)
    static constexpr uint32_t B_BYTES = N1 * TC_BK * 4;     // multiple of 1024
    static constexpr uint32_t STAGE = TC_A_BYTES + B_BYTES;
    static constexpr uint32_t DSTRIDE = (N1 + 31) / 32 * 32;   // accumulator buffers 32-column aligned
    static constexpr uint32_t COL_A = 2 * DSTRIDE <= 128 ? 128u : 256u;
    static constexpr uint32_t TMEM_COLS = COL_A + TC_NT * TC_TSTAGE <= 256 ? 256u : 512u;
    // with 512 TMEM columns only one CTA may be resident: ask for enough smem
    static constexpr uint32_t SMEM_MIN = TMEM_COLS == 512u ? 120u * 1024u : 0u;
    static constexpr uint32_t SMEM_RAW = TC_NS * STAGE + 1024;
    static constexpr uint32_t SMEM = SMEM_RAW > SMEM_MIN ? SMEM_RAW : SMEM_MIN;
};

__device__ __forceinline__ void tc_fail(int* err, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    if (err != nullptr) atomicExch(err, code);
}

// Two CTAs per SM for k <= 32 (TMEM and shared memory allow it): registers
// are capped at 128 per thread; one CTA per SM above that.
template <int KP>
__global__ void __launch_bounds__(TC_THREADS, TcCfg<KP>::TMEM_COLS == 256u ? 2 : 1)
stream_tc_kernel(const __grid_constant__ CUtensorMap mapS, const __grid_constant__ CUtensorMap mapX,
                 int64_t n, int k, int64_t j0, int64_t j1, int64_t jspan,
                 float* __restrict__ part, int* __restrict__ err, const FitState* st,
                 const EpiArgs epi, int* __restrict__ counters) {
    using Cfg = TcCfg<KP>;
    using namespace sm100;
    pdl_wait();   // everything below may read what the previous kernel wrote
    if (st != nullptr && st->done) return;

    extern __shared__ uint8_t tc_smem_raw[];
    __shared__ __align__(8) uint64_t bar_full[TC_NS], bar_tfull[TC_NT], bar_done[TC_NDONE];
    __shared__ __align__(8) uint64_t bar_dempty[2], bar_fin[2];
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ int go_sh, last_sh;
    static_assert(epilogue_cta_floats<KP>() * sizeof(float) <= Cfg::SMEM - 1024,
                  "the epilogue tiles must fit in the pipeline's shared memory");

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smemA = smem;                                // [NS][128 rows][128 B]
    uint8_t* smemB = smem + TC_NS * TC_A_BYTES;           // [NS][N1 rows][128 B]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t i0 = (int64_t)blockIdx.x * TC_BM;
    const int split = blockIdx.y;
    const int64_t jb = j0 + (int64_t)split * jspan;
    const int64_t je = min64(j1, jb + jspan);
    const int ksteps = jb < je ? (int)((je - jb + TC_BK - 1) / TC_BK) : 0;
    const int nchunks = (ksteps + TC_CHUNK - 1) / TC_CHUNK;

    if (tid == 0) {
        for (int s = 0; s < TC_NS; ++s) {
            mbar_init(&bar_full[s], 1);
        }
        for (int t = 0; t < TC_NT; ++t) {
            mbar_init(&bar_tfull[t], 4);   // one arrival per split warp

        }
        for (int b = 0; b < 2; ++b) {

            mbar_init(&bar_dempty[b], 4);  // one arrival per split warp
        }
        for (int d = 0; d < TC_NDONE; ++d) mbar_init(&bar_done[d], 1);
        mbar_init(&bar_fin[0], 1);
        mbar_init(&bar_fin[1], 1);
        abort_sh = 0;
        last_sh = 0;
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

    if (warp == 0 && lane == 0 && ksteps > 0 && *(volatile int*)&g_stall_producer == 0) {
        // ---------------- TMA producer
        int issued = 0;
        const uint64_t pol_s = SYMNMF_TC_L2HINT ? policy_evict_first() : 0;
        const uint64_t pol_x = SYMNMF_TC_L2HINT ? policy_evict_last() : 0;
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % TC_NS;
            if (s >= TC_NS && !mbar_wait(&bar_done[(s - TC_NS) % TC_NDONE],
                                         (uint32_t)((s - TC_NS) / TC_NDONE) & 1u)) {
                tc_fail(err, &abort_sh, 1);
                break;
            }
            mbar_arrive_expect_tx(&bar_full[slot], Cfg::STAGE);
            const int32_t x = (int32_t)(jb + (int64_t)s * TC_BK);
            if (SYMNMF_TC_L2HINT) {
                tma_load_2d_hint(smemA + slot * TC_A_BYTES, &mapS, x, (int32_t)i0, &bar_full[slot], pol_s);
                tma_load_2d_hint(smemB + slot * Cfg::B_BYTES, &mapX, x, 0, &bar_full[slot], pol_x);
            } else {
                tma_load_2d(smemA + slot * TC_A_BYTES, &mapS, x, (int32_t)i0, &bar_full[slot]);
                tma_load_2d(smemB + slot * Cfg::B_BYTES, &mapX, x, 0, &bar_full[slot]);
            }
            ++issued;
        }
        if (abort_sh) {  // let the copies already issued land before the CTA exits
            for (int s = max(0, issued - TC_NS); s < issued; ++s)
                mbar_wait(&bar_full[s % TC_NS], (uint32_t)(s / TC_NS) & 1u);
        }
    } else if ((warp == 1 || warp == 3) && lane == 0 && ksteps > 0) {
        // ---------------- MMA issuers: chunk q accumulates into D[q % 2] and is
        // issued by warp 1 (q even) or warp 3 (q odd).  A tcgen05.commit tracks
        // the MMAs of its own thread, and each accumulator has one issuer, so
        // the two run independently; together they issue twice as fast as one.
        const int par = warp == 1 ? 0 : 1;
        constexpr uint32_t id1 = idesc_tf32(TC_BM, Cfg::N1);
        constexpr uint32_t id2 = idesc_tf32(TC_BM, Cfg::N2);
        for (int s = 0; s < ksteps; ++s) {
            if (((s / TC_CHUNK) & 1) != par) continue;
            if (abort_sh) break;
            const int slot = s % TC_NS;
            const uint32_t ph = (uint32_t)(s / TC_NS) & 1u;
            const int ts = s % TC_NT;
            const uint32_t tph = (uint32_t)(s / TC_NT) & 1u;
            const int q = s / TC_CHUNK, b = q & 1;
            const bool first = (s % TC_CHUNK) == 0;
            bool ok = mbar_wait(&bar_tfull[ts], tph) && mbar_wait(&bar_full[slot], ph);
            if (ok && first && q >= 2) ok = mbar_wait(&bar_dempty[b], (uint32_t)((q >> 1) - 1) & 1u);
            if (!ok) {
                tc_fail(err, &abort_sh, 2);
                break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(smemB + slot * Cfg::B_BYTES);
            const uint32_t a_base = smem_u32(smemA + slot * TC_A_BYTES);
            const uint32_t a_t = tbase + Cfg::COL_A + (uint32_t)ts * (uint32_t)TC_TSTAGE;
            const uint32_t d = tbase + (uint32_t)b * Cfg::DSTRIDE;
#pragma unroll
            for (int kk = 0; kk < TC_BK / 8; ++kk) {
                const uint64_t bd = umma_desc_sw128(b_base + (uint32_t)kk * 32u);
                const uint32_t acc0 = (first && kk == 0) ? 0u : 1u;
                if (TC_A_SMEM) {
                    umma_tf32_ss(d, umma_desc_sw128(a_base + (uint32_t)kk * 32u), bd, id1, acc0);
                    umma_tf32_ts(d, a_t + (uint32_t)kk * 8u, bd, id2, 1u);
                } else {
                    umma_tf32_ts(d, a_t + (uint32_t)kk * 8u, bd, id1, acc0);
                    umma_tf32_ts(d, a_t + 32u + (uint32_t)kk * 8u, bd, id2, 1u);
                }
            }
            umma_commit(&bar_done[s % TC_NDONE]);
        }
        if (abort_sh) {  // MMAs in flight finish before TMEM is freed
            umma_commit(&bar_fin[par]);
            mbar_wait(&bar_fin[par], 0);
        }
    } else if (warp >= 4) {
        // ---------------- split warps (TMEM lane quarter = warp % 4)
        const int wl = warp & 3;
        const int r = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        float acc[KP];
#pragma unroll
        for (int c = 0; c < KP; ++c) acc[c] = 0.f;
        bool alive = true;

        // fold accumulator D[q % 2] into acc (round-to-nearest fp32 adds); the
        // tensor-core accumulation itself carries a one-signed rounding error
        // per accumulate, so TMEM chains are kept to TC_CHUNK stages
        auto drain = [&](int q) -> bool {
            const int b = q & 1;
            const int ls = min(ksteps, (q + 1) * TC_CHUNK) - 1;   // last stage of chunk q
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_done[ls % TC_NDONE], (uint32_t)(ls / TC_NDONE) & 1u)))
                return false;
            tc_fence_after();
            const uint32_t dcol = tbase + lane_off + (uint32_t)b * Cfg::DSTRIDE;
            uint32_t v[2 * KP / 8][8];
#pragma unroll
            for (int g = 0; g < 2 * KP / 8; ++g) tmem_ld_32x32b_x8(dcol + (uint32_t)g * 8u, v[g]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < KP; ++c)
                acc[c] += __uint_as_float(v[c / 8][c % 8]) + __uint_as_float(v[(KP + c) / 8][c % 8]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_dempty[b]);
            return true;
        };

        // control flow stays warp-uniform: tcgen05.st/ld are .sync.aligned
        for (int s = 0; s < ksteps; ++s) {
            if (__any_sync(0xffffffffu, abort_sh != 0)) {
                alive = false;
                break;
            }
            const int slot = s % TC_NS;
            const uint32_t ph = (uint32_t)(s / TC_NS) & 1u;
            const int ts = s % TC_NT;
            const bool ok = mbar_wait(&bar_full[slot], ph) &&
                            (s < TC_NT || mbar_wait(&bar_done[(s - TC_NT) % TC_NDONE],
                                                    (uint32_t)((s - TC_NT) / TC_NDONE) & 1u));
            if (!__all_sync(0xffffffffu, ok)) {
                if (lane == 0) tc_fail(err, &abort_sh, 3);
                alive = false;
                break;
            }
            const uint8_t* rowp = smemA + slot * TC_A_BYTES + r * 128;
            uint32_t hi[32], lo[32];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const float4 v = *reinterpret_cast<const float4*>(rowp + ((c ^ (r & 7)) << 4));
                const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t hb = __float_as_uint(e[u]) & 0xFFFFE000u;
                    hi[c * 4 + u] = hb;
                    lo[c * 4 + u] = __float_as_uint(e[u] - __uint_as_float(hb));
                }
            }
            const uint32_t tcol = tbase + lane_off + Cfg::COL_A + (uint32_t)ts * (uint32_t)TC_TSTAGE;
            if (TC_A_SMEM) {
                tmem_st_32x32b_x32(tcol, lo);
            } else {
                tmem_st_32x32b_x32(tcol, hi);
                tmem_st_32x32b_x32(tcol + 32u, lo);
            }
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_tfull[ts]);
            // end of chunk q: fold the previous chunk, whose MMAs are done by now
            const int q = s / TC_CHUNK;
            if (((s % TC_CHUNK) == TC_CHUNK - 1 || s == ksteps - 1) && q >= 1) {
                if (!drain(q - 1)) {
                    if (lane == 0) tc_fail(err, &abort_sh, 4);
                    alive = false;
                    break;
                }
            }
        }
        if (alive && nchunks > 0 && !drain(nchunks - 1)) {
            if (lane == 0) tc_fail(err, &abort_sh, 5);
            alive = false;
        }
        // ---- tail of the split warps: one decision for all four of them
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (r == 0) go_sh = abort_sh == 0 ? 1 : 0;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool go = go_sh != 0;
        const int64_t i = i0 + r;
        if (go && i < n) {
            float* out = part + (int64_t)split * n * k + i * (int64_t)k;
#pragma unroll
            for (int c = 0; c < KP; ++c)
                if (c < k) out[c] = acc[c];
        }
        if (go && counters != nullptr) {
            // the last split CTA of this row tile runs the epilogue for it (no waiting:
            // whoever arrives last finds every partial in place)
            __threadfence();
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (r == 0) last_sh = atomicAdd(&counters[blockIdx.x], 1) == (int)gridDim.y - 1 ? 1 : 0;
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, Cfg::TMEM_COLS);
    }
    // every stage has landed and been consumed: the pipeline's shared memory is
    // free, and all eight warps run the tile's epilogue
    if (last_sh) {
        // this CTA holds no TMEM any more and the CTAs without an epilogue
        // have exited: the next kernel may be scheduled
        pdl_trigger();
        __threadfence();
        epilogue_tile_cta<KP>(epi, (int)blockIdx.x, tid, reinterpret_cast<float*>(smem),
                              (int)((Cfg::SMEM - 1024) / sizeof(float)));
        if (tid == 0) counters[blockIdx.x] = 0;   // ready for the next pass
    }
}

// ----------------------------------------------------------------------------
// [X_hi ; X_lo] in the K-major layout the MMA reads: XT[c][j] (c < KP) and
// XT[KP + c][j] for j in [jlo, jhi); X = Xa - Xb on rows [r0, r1) and zero
// on the other rows of the range; rows c in [k, KP) of each half are zero.
// ----------------------------------------------------------------------------
__global__ void split_kernel(const float* __restrict__ Xa, const float* __restrict__ Xb,
                             int64_t ldx, int k, int KP, int64_t r0, int64_t r1, int64_t jlo,
                             int64_t jhi, float* __restrict__ XT, int64_t ldxt) {
    const int64_t j = jlo + (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= jhi) return;
    const bool in = j >= r0 && j < r1;
    for (int c = 0; c < KP; ++c) {
        float x = 0.f;
        if (in && c < k) {
            x = Xa[j * ldx + c];
            if (Xb != nullptr) x -= Xb[j * ldx + c];
        }
        const float h = __uint_as_float(__float_as_uint(x) & 0xFFFFE000u);
        XT[(int64_t)c * ldxt + j] = h;
        XT[(int64_t)(KP + c) * ldxt + j] = x - h;
    }
}

int launch_split(const float* Xa, const float* Xb, int64_t ldx, int k, int64_t r0, int64_t r1,
                 int64_t jlo, int64_t jhi, float* XT, int64_t ldxt, cudaStream_t s) {
    if (jhi <= jlo) return SYMNMF_OK;
    const int KP = (k + 7) / 8 * 8;
    const int64_t len = jhi - jlo;
    split_kernel<<<(unsigned)((len + 255) / 256), 256, 0, s>>>(Xa, Xb, ldx, k, KP, r0, r1, jlo,
                                                              jhi, XT, ldxt);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// host side
// ----------------------------------------------------------------------------
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    // looked up once (thread-safe static initialisation)
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = []() -> PFN_cuTensorMapEncodeTiled_v12000 {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
        return nullptr;
    }();
    return fn;
}

// Row-major fp32 matrix (rows x cols, row pitch `ld` elements) as a 2-D TMA
// map with boxes of 32 columns x box_rows rows and 128-byte swizzle.
int make_map(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld,
             uint32_t box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)ld * sizeof(float)};
    cuuint32_t box[2] = {(cuuint32_t)TC_BK, box_rows};
    cuuint32_t estr[2] = {1, 1};
    CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims, strides,
                    box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

// CTAs of stream_tc_kernel<KP> resident on one SM: two while both the tensor
// memory (256 columns each) and the shared memory (228 KB an SM, 1 KB of it
// reserved per CTA) allow, else one.
template <int KP>
static int tc_resident_per_sm() {
    using Cfg = TcCfg<KP>;
    if (Cfg::TMEM_COLS != 256u) return 1;
    return 2 * (Cfg::SMEM + 1024) <= 228u * 1024u ? 2 : 1;
}
static int tc_resident(int KP) {
    switch (KP) {
        case 8: return tc_resident_per_sm<8>();
        case 16: return tc_resident_per_sm<16>();
        case 24: return tc_resident_per_sm<24>();
        case 32: return tc_resident_per_sm<32>();
        case 40: return tc_resident_per_sm<40>();
        case 48: return tc_resident_per_sm<48>();
        case 56: return tc_resident_per_sm<56>();
        default: return tc_resident_per_sm<64>();
    }
}

// Contraction splits of a pass over `tiles` row tiles and `steps` stages of
// 32 columns: the count that minimises a model of the pass time fitted to
// timings of Y = S X on B200 (k = 24; n = 10,000, 20,000 and 50,000 with
// every split count from 1 to 15, where it picks the fastest count of each).
// The CTAs run in waves of `resident`; a wave takes the longer of its HBM
// time (16 KB of S a stage at 6.5 TB/s) and one CTA's stage cadence (0.55 us
// a stage), plus 5 us of setup and tail; each split adds 1 us to the
// epilogue's partial sums.  Every split keeps at least 8 stages.  (The fp16
// stream passes its own stage size and cadence.)
int choose_splits(int64_t tiles, int64_t steps, int64_t resident, double kStageBytes,
                  double kCadence) {
    constexpr double kBW = 6.5e12, kWave = 5e-6, kSplit = 1e-6;
    int best = 1;
    double best_t = 1e30;
    for (int s = 1; s <= 32; ++s) {
        if (s > 1 && steps / s < 8) break;
        const int64_t per = (steps + s - 1) / s;
        int64_t left = tiles * s;
        double t = kSplit * s;
        while (left > 0) {
            const int64_t w = std::min(left, resident);
            left -= w;
            t += std::max((double)w * (double)per * kStageBytes / kBW, (double)per * kCadence) + kWave;
        }
        if (t < best_t - 1e-12) {
            best_t = t;
            best = s;
        }
    }
    return best;
}

TcPlan plan_stream_tc(const Dev& d, int64_t n, int k, int64_t j0, int64_t j1) {
    TcPlan p;
    p.n = n;
    p.ncols = n;
    p.k = k;
    p.KP = (k + 7) / 8 * 8;
    p.j0 = j0 / TC_BK * TC_BK;                                 // 128-byte aligned TMA x
    p.j1 = std::min<int64_t>(n, (j1 + TC_BK - 1) / TC_BK * TC_BK);
    p.tiles = (n + TC_BM - 1) / TC_BM;
    const int64_t steps = std::max<int64_t>(1, (p.j1 - p.j0 + TC_BK - 1) / TC_BK);
    p.splits = choose_splits(p.tiles, steps, (int64_t)d.sms * tc_resident(p.KP), 16384.0, 0.55e-6);
    p.jspan = (steps + p.splits - 1) / p.splits * TC_BK;
    return p;
}

TcPlan plan_stream_tc_rows(const Dev& d, int64_t rows, int64_t ncols, int k) {
    // the split choice depends on the row tiles and the contraction length only
    TcPlan p = plan_stream_tc(d, ncols, k, 0, ncols);
    p.n = rows;
    p.ncols = ncols;
    p.tiles = (rows + TC_BM - 1) / TC_BM;
    const int64_t steps = std::max<int64_t>(1, (p.j1 - p.j0 + TC_BK - 1) / TC_BK);
    p.splits = choose_splits(p.tiles, steps, (int64_t)d.sms * tc_resident(p.KP), 16384.0, 0.55e-6);
    p.jspan = (steps + p.splits - 1) / p.splits * TC_BK;
    return p;
}

size_t tc_partial_floats(const TcPlan& p) { return (size_t)p.splits * p.n * p.k; }

int launch_stream_tc(const TcPlan& p, const float* S, int64_t lds, const float* XT, int64_t ldxt,
                     float* part, int* err, const FitState* st, cudaStream_t s,
                     const EpiArgs* epi, int* counters) {
    EpiArgs none;
    std::memset(&none, 0, sizeof(none));
    none.mode = -1;
    const EpiArgs ea = epi != nullptr ? *epi : none;
    int* cnt = epi != nullptr ? counters : nullptr;
    CUtensorMap mapS, mapX;
    SYMNMF_TRY(make_map(&mapS, S, p.ncols, p.n, lds, TC_BM));
    SYMNMF_TRY(make_map(&mapX, XT, p.ncols, 2 * p.KP, ldxt, (uint32_t)(2 * p.KP)));
    dim3 grid((unsigned)p.tiles, (unsigned)p.splits);
#define SYMNMF_TC(KP)                                                                         \
    do {                                                                                      \
        auto kern = stream_tc_kernel<KP>;                                                     \
        /* once per process (thread-safe static initialisation): keeps graph capture clean */ \
        static const cudaError_t attr_rc = cudaFuncSetAttribute(                              \
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)TcCfg<KP>::SMEM);         \
        SYMNMF_CUDA_TRY(attr_rc);                                                             \
        SYMNMF_CUDA_TRY(launch_pdl(kern, grid, dim3(TC_THREADS), TcCfg<KP>::SMEM, s, mapS, mapX, \
                                   p.n, p.k, p.j0, p.j1, p.jspan, part, err, st, ea, cnt));   \
    } while (0)
    switch (p.KP) {
        case 8: SYMNMF_TC(8); break;
        case 16: SYMNMF_TC(16); break;
        case 24: SYMNMF_TC(24); break;
        case 32: SYMNMF_TC(32); break;
        case 40: SYMNMF_TC(40); break;
        case 48: SYMNMF_TC(48); break;
        case 56: SYMNMF_TC(56); break;
        default: SYMNMF_TC(64); break;
    }
#undef SYMNMF_TC
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf

extern "C" int symnmf_test_stall_pipeline(int on) {
    symnmf::clear_error();
    const int v = on ? 1 : 0;
    const cudaError_t e = cudaMemcpyToSymbol(symnmf::g_stall_producer, &v, sizeof(int));
    if (e != cudaSuccess) {
        symnmf::set_error("cudaMemcpyToSymbol failed: %s", cudaGetErrorString(e));
        return SYMNMF_ERR_CUDA;
    }
    SYMNMF_TRY(symnmf::h16_set_stall(v));
    return symnmf::tri_set_stall(v);
}
