// fp16 tensor-core S-stream of the full-batch loop: part[s] = S[:, J_s] X[J_s, :]
// with S and X each entering as a power-of-two scaled fp16 hi/lo pair.
//
// The pages' hot spot is the S H product that streams S once per iteration
// ([CaS] "Factorization at scale": the dominant S H multiplications).  The
// TF32 stream (stream_tc.cu) feeds the tensor core S straight from shared
// memory and its remainder through tensor memory; under the sustained power
// cap its pace is set by shared-memory traffic (about four bytes per byte of
// S).  Here both parts of S go through tensor memory as fp16, four bytes per
// element in all, so the tensor core reads only the small X operand from
// shared memory, and the kind::f16 MMAs do the three products at twice the
// TF32 rate.
//
// Accuracy.  With cS = st->sscale (cS max|S| < 2^14, from the statistics
// pass) and cX = st->xscale (the same for max|X|, from the previous pass's
// finalise step), each value v = c s enters as hi = rn16(v) (v to 11
// significant bits in fp16's normal range) and lo = rn16(v - hi):
// v = hi + lo to 2^-22 |v| where lo is a normal fp16 number, and to 2^-25 in
// absolute terms where it is not (more than 2^-22 |v| only for v below 2^-3,
// about 2^-16 of the largest).
// Then
//     cS cX S X = S_hi X_hi + S_hi X_lo + S_lo X_hi
// (+ S_lo X_lo on the columns c < N2 - KP), each entry to first order within
// 3 * 2^-22 sum_j |s_ij| |x_jc| + 2^-25 sum_j (|s_ij| + |x_jc|) in scaled units,
// accumulated in fp32 in tensor memory over each pair of stages, folded into
// registers with round-to-nearest fp32 adds, and scaled back by 1 / cS and
// 1 / cX (powers of two: exact) once the split's range is done.
//
// Per CTA (256 threads, two CTAs per SM): a 128-row tile of S times the
// contraction range of its split, in stages of 64 columns:
//   warp 0      TMA producer of S: the stage's two 128 x 32 fp32 boxes
//               (128-byte swizzle) into a 3-slot ring that the split warps
//               release once they have read a stage
//   warp 3      TMA producer of X: the [X_hi; X_lo] tile (2 KP rows of 64
//               fp16, K-major, 128-byte swizzle) into a 2-slot ring that the
//               MMAs release
//   warp 1      MMA issuer: per 16-column step, D[:, 0:2KP] += S_hi [X_hi; X_lo]
//               and D[:, 0:N2] += S_lo [X_hi; ...], A from tensor memory
//   warp 2      tensor-memory allocator
//   warps 4-7   split warps: thread r reads row r of the stage from shared
//               memory, scales and splits it, stores hi and lo into tensor
//               memory lane r, folds each pair of stages' accumulator
//   all warps   in the last split CTA of the tile, the epilogue (epilogue.cuh)
#include <cuda_fp16.h>
#include <cudaTypedefs.h>

#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"
#include "sm100.cuh"

namespace symnmf {

// the TF32 stream's map of S (stream_tc.cu): boxes of 32 columns x box_rows rows,
// 128-byte swizzle
int make_map(CUtensorMap* m, const float* base, int64_t cols, int64_t rows, int64_t ld,
             uint32_t box_rows);

// Test hook (symnmf_test_stall_pipeline): when set, the producer of S issues
// no loads, so the consumers' bounded waits run out and the pass reports its
// error word instead of a result.
__device__ int g_h16_stall = 0;

constexpr int H16_BM = 128;                    // S rows per tile = tensor-memory lanes
constexpr int H16_BK = 64;                     // columns per stage (two 32-column S boxes)
constexpr int H16_NSS = 3;                     // shared-memory slots of S
constexpr int H16_NSX = 2;                     // shared-memory slots of X
constexpr int H16_NT = 2;                      // A stages in tensor memory = accumulator sets (a pair each)
constexpr int H16_NDONE = 4;                   // stage-completion barriers: > both rings, a multiple of each
constexpr int H16_THREADS = 256;
constexpr uint32_t H16_BOX = H16_BM * 32 * 4;  // 16 KB: one 128 x 32 fp32 box of S
constexpr uint32_t H16_A_BYTES = 2 * H16_BOX;  // 32 KB of S per stage
static_assert(H16_NDONE > H16_NSX && H16_NDONE > H16_NT && H16_NDONE % H16_NSX == 0 &&
                  H16_NDONE % H16_NT == 0,
              "stage-completion barriers must outnumber the rings they release");

template <int KP>
struct H16Cfg {
    static constexpr int N1 = 2 * KP;                       // [X_hi ; X_lo]
    static constexpr int N2 = (KP + 15) / 16 * 16;          // X_hi (+ rows of X_lo)
    static constexpr uint32_t B_BYTES = N1 * 128;           // N1 rows of 64 fp16
    static constexpr uint32_t DSTRIDE = (N1 + 31) / 32 * 32;
    static constexpr uint32_t COL_A = 2 * DSTRIDE;          // after the two accumulators
    static constexpr uint32_t TSTAGE = 64;                  // 32 columns of hi, 32 of lo
    static constexpr uint32_t TMEM_COLS = 256;
    static constexpr uint32_t SMEM = H16_NSS * H16_A_BYTES + H16_NSX * B_BYTES + 1024;
    static_assert(COL_A + H16_NT * TSTAGE <= TMEM_COLS, "tensor memory of one CTA");
    static_assert(B_BYTES % 1024 == 0, "whole 8-row swizzle atoms");
    static_assert(2 * (SMEM + 1024 + 256) <= 228u * 1024u, "two CTAs per SM (with static shared memory)");
};

__device__ __forceinline__ void h16_fail(int* err, volatile int* abort_flag, int code) {
    *abort_flag = 1;
    if (err != nullptr) atomicExch(err, code);
}

// v = hi + lo with hi = rn16(v) and lo = rn16(v - hi), two values at a time:
// the packed conversion's rounding does the split.  The difference is exact in
// fp32 (v and hi are fp32 numbers less than half an fp16 ulp apart), and hi
// carries v to 11 significant bits wherever v is in fp16's normal range.
__device__ __forceinline__ void split_pair(float a, float b, uint32_t& hi, uint32_t& lo) {
    const __half2 h = __floats2half2_rn(a, b);
    const float2 f = __half22float2(h);
    const __half2 l = __floats2half2_rn(__fsub_rn(a, f.x), __fsub_rn(b, f.y));
    hi = *reinterpret_cast<const uint32_t*>(&h);
    lo = *reinterpret_cast<const uint32_t*>(&l);
}

// Four values q scaled by cs (a power of two: exact), each split as above;
// h0/l0 hold the fp16 hi/lo of q.x, q.y (low, high half), h1/l1 of q.z, q.w.
__device__ __forceinline__ void split_scaled4(const float4 q, float cs, uint32_t& h0, uint32_t& h1,
                                              uint32_t& l0, uint32_t& l1) {
    split_pair(q.x * cs, q.y * cs, h0, l0);
    split_pair(q.z * cs, q.w * cs, h1, l1);
}

template <int KP>
__global__ void __launch_bounds__(H16_THREADS, 2)
stream_h16_kernel(const __grid_constant__ CUtensorMap mapS, const __grid_constant__ CUtensorMap mapX,
                  int64_t n, int k, int64_t j0, int64_t j1, int64_t jspan,
                  float* __restrict__ part, int* __restrict__ err, const FitState* st,
                  const EpiArgs epi, int* __restrict__ counters) {
    using Cfg = H16Cfg<KP>;
    using namespace sm100;
    pdl_wait();   // everything below may read what the previous kernel wrote
    if (st->done) return;

    extern __shared__ uint8_t h16_smem_raw[];
    __shared__ __align__(8) uint64_t bar_sfull[H16_NSS], bar_sempty[H16_NSS], bar_xfull[H16_NSX];
    __shared__ __align__(8) uint64_t bar_tfull[H16_NT], bar_done[H16_NDONE], bar_dempty[H16_NT], bar_fin;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;
    __shared__ int go_sh, last_sh;
    static_assert(epilogue_cta_floats<KP>() * sizeof(float) <= Cfg::SMEM - 1024,
                  "the epilogue tiles must fit in the pipeline's shared memory");

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(h16_smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* smemA = smem;                                 // [NSS][2 boxes][128 rows][128 B]
    uint8_t* smemB = smem + H16_NSS * H16_A_BYTES;         // [NSX][N1 rows][128 B]

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int64_t i0 = (int64_t)blockIdx.x * H16_BM;
    const int split = blockIdx.y;
    const int64_t jb = j0 + (int64_t)split * jspan;
    const int64_t je = min64(j1, jb + jspan);
    const int ksteps = jb < je ? (int)((je - jb + H16_BK - 1) / H16_BK) : 0;

    if (tid == 0) {
        for (int s = 0; s < H16_NSS; ++s) {
            mbar_init(&bar_sfull[s], 1);
            mbar_init(&bar_sempty[s], 4);   // one arrival per split warp
        }
        for (int s = 0; s < H16_NSX; ++s) mbar_init(&bar_xfull[s], 1);
        for (int t = 0; t < H16_NT; ++t) {
            mbar_init(&bar_tfull[t], 4);    // one arrival per split warp
            mbar_init(&bar_dempty[t], 4);   // one arrival per split warp
        }
        for (int d = 0; d < H16_NDONE; ++d) mbar_init(&bar_done[d], 1);
        mbar_init(&bar_fin, 1);
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

    if (warp == 0 && lane == 0 && ksteps > 0 && *(volatile int*)&g_h16_stall == 0) {
        // ---------------- TMA producer of S: slot s % 3, free once the split
        // warps have read stage s - 3
        int issued = 0;
        const uint64_t pol_s = policy_evict_first();
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % H16_NSS;
            if (s >= H16_NSS &&
                !mbar_wait(&bar_sempty[slot], (uint32_t)((s - H16_NSS) / H16_NSS) & 1u)) {
                h16_fail(err, &abort_sh, 1);
                break;
            }
            mbar_arrive_expect_tx(&bar_sfull[slot], H16_A_BYTES);
            const int32_t x = (int32_t)(jb + (int64_t)s * H16_BK);
            uint8_t* a = smemA + slot * H16_A_BYTES;
            tma_load_2d_hint(a, &mapS, x, (int32_t)i0, &bar_sfull[slot], pol_s);
            tma_load_2d_hint(a + H16_BOX, &mapS, x + 32, (int32_t)i0, &bar_sfull[slot], pol_s);
            ++issued;
        }
        if (abort_sh) {  // let the copies already issued land before the CTA exits
            for (int s = max(0, issued - H16_NSS); s < issued; ++s)
                mbar_wait(&bar_sfull[s % H16_NSS], (uint32_t)(s / H16_NSS) & 1u);
        }
    } else if (warp == 3 && lane == 0 && ksteps > 0) {
        // ---------------- TMA producer of X: slot s % 2, free once the MMAs
        // of stage s - 2 are done
        int issued = 0;
        const uint64_t pol_x = policy_evict_last();
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % H16_NSX;
            if (s >= H16_NSX && !mbar_wait(&bar_done[(s - H16_NSX) % H16_NDONE],
                                           (uint32_t)((s - H16_NSX) / H16_NDONE) & 1u)) {
                h16_fail(err, &abort_sh, 6);
                break;
            }
            mbar_arrive_expect_tx(&bar_xfull[slot], Cfg::B_BYTES);
            const int32_t x = (int32_t)(jb + (int64_t)s * H16_BK);
            tma_load_2d_hint(smemB + slot * Cfg::B_BYTES, &mapX, x, 0, &bar_xfull[slot], pol_x);
            ++issued;
        }
        if (abort_sh) {
            for (int s = max(0, issued - H16_NSX); s < issued; ++s)
                mbar_wait(&bar_xfull[s % H16_NSX], (uint32_t)(s / H16_NSX) & 1u);
        }
    } else if (warp == 1 && lane == 0 && ksteps > 0) {
        // ---------------- MMA issuer: stage s accumulates into D[(s / 2) % 2]
        constexpr uint32_t id1 = idesc_f16(H16_BM, Cfg::N1);
        constexpr uint32_t id2 = idesc_f16(H16_BM, Cfg::N2);
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % H16_NSX;
            const int ts = s % H16_NT;
            // stages 2g and 2g + 1 accumulate into set g % 2, which the split
            // warps must have folded for pair g - 2 first
            const int g = s / 2;
            const int dset = g % H16_NT;
            const bool first = (s % 2) == 0;
            bool ok = mbar_wait(&bar_tfull[ts], (uint32_t)(s / H16_NT) & 1u) &&
                      mbar_wait(&bar_xfull[slot], (uint32_t)(s / H16_NSX) & 1u);
            if (ok && first && g >= H16_NT)
                ok = mbar_wait(&bar_dempty[dset], (uint32_t)((g / H16_NT) - 1) & 1u);
            if (!ok) {
                h16_fail(err, &abort_sh, 2);
                break;
            }
            tc_fence_after();
            const uint32_t b_base = smem_u32(smemB + slot * Cfg::B_BYTES);
            const uint32_t a_hi = tbase + Cfg::COL_A + (uint32_t)ts * Cfg::TSTAGE;
            const uint32_t a_lo = a_hi + 32u;
            const uint32_t d = tbase + (uint32_t)dset * Cfg::DSTRIDE;
#pragma unroll
            for (int kk = 0; kk < H16_BK / 16; ++kk) {
                const uint64_t bd = umma_desc_sw128(b_base + (uint32_t)kk * 32u);
                umma_f16_ts(d, a_hi + (uint32_t)kk * 8u, bd, id1, (kk == 0 && first) ? 0u : 1u);
                umma_f16_ts(d, a_lo + (uint32_t)kk * 8u, bd, id2, 1u);
            }
            umma_commit(&bar_done[s % H16_NDONE]);
        }
        if (abort_sh) {  // MMAs in flight finish before tensor memory is freed
            umma_commit(&bar_fin);
            mbar_wait(&bar_fin, 0);
        }
    } else if (warp >= 4) {
        // ---------------- split warps (tensor-memory lane quarter = warp % 4)
        const int wl = warp & 3;
        const int r = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const float cs = st->sscale;
        // powers of two: the products scale back exactly; applied one after the
        // other, since cS cX alone could overflow for tiny S and X
        const float inv_s = 1.f / st->sscale, inv_x = 1.f / st->xscale;
        float acc[KP];
#pragma unroll
        for (int c = 0; c < KP; ++c) acc[c] = 0.f;
        bool alive = true;

        // fold accumulator set dset, complete once the MMAs of stage s_last are
        // done, into acc (round-to-nearest fp32 adds)
        auto drain = [&](int s_last, int dset) -> bool {
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_done[s_last % H16_NDONE], (uint32_t)(s_last / H16_NDONE) & 1u)))
                return false;
            tc_fence_after();
            const uint32_t dcol = tbase + lane_off + (uint32_t)dset * Cfg::DSTRIDE;
            uint32_t v[2 * KP / 8][8];
#pragma unroll
            for (int g = 0; g < 2 * KP / 8; ++g) tmem_ld_32x32b_x8(dcol + (uint32_t)g * 8u, v[g]);
            tmem_wait_ld();
#pragma unroll
            for (int c = 0; c < KP; ++c)
                acc[c] += __uint_as_float(v[c / 8][c % 8]) + __uint_as_float(v[(KP + c) / 8][c % 8]);
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_dempty[dset]);
            return true;
        };

        // control flow stays warp-uniform: tcgen05.st/ld are .sync.aligned
        for (int s = 0; s < ksteps; ++s) {
            if (__any_sync(0xffffffffu, abort_sh != 0)) {
                alive = false;
                break;
            }
            const int slot = s % H16_NSS;
            const int ts = s % H16_NT;
            // the stage of S has landed
            if (!__all_sync(0xffffffffu, mbar_wait(&bar_sfull[slot], (uint32_t)(s / H16_NSS) & 1u))) {
                if (lane == 0) h16_fail(err, &abort_sh, 3);
                alive = false;
                break;
            }
            uint32_t hi[32], lo[32];
#pragma unroll
            for (int b = 0; b < 2; ++b) {
                const uint8_t* rowp = smemA + slot * H16_A_BYTES + b * H16_BOX + r * 128;
#pragma unroll
                for (int c = 0; c < 8; ++c) {
                    const float4 q = *reinterpret_cast<const float4*>(rowp + ((c ^ (r & 7)) << 4));
                    const int w = b * 16 + c * 2;   // column pair of elements 4c..4c+3 of box b
                    split_scaled4(q, cs, hi[w], hi[w + 1], lo[w], lo[w + 1]);
                }
            }
            // the stage of S is read: release the slot.  The next fill is an
            // async-proxy (TMA) write, which the mbarrier alone does not order
            // after these generic-proxy reads; without the proxy fence a fill
            // could land under reads still in flight (seen on B200 as fits that
            // differed from run to run once the grid ran in several waves).
            fence_proxy_async_smem();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_sempty[slot]);
            // the tensor-memory slot's previous MMAs are done
            if (!__all_sync(0xffffffffu, s < H16_NT || mbar_wait(&bar_done[(s - H16_NT) % H16_NDONE],
                                                                 (uint32_t)((s - H16_NT) / H16_NDONE) & 1u))) {
                if (lane == 0) h16_fail(err, &abort_sh, 3);
                alive = false;
                break;
            }
            const uint32_t tcol = tbase + lane_off + Cfg::COL_A + (uint32_t)ts * Cfg::TSTAGE;
            tmem_st_32x32b_x32(tcol, hi);
            tmem_st_32x32b_x32(tcol + 32u, lo);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&bar_tfull[ts]);
            // at the start of a pair, the previous pair's MMAs are done by now:
            // fold its accumulator set
            if (s >= 2 && s % 2 == 0 && !drain(s - 1, ((s - 1) / 2) % H16_NT)) {
                if (lane == 0) h16_fail(err, &abort_sh, 4);
                alive = false;
                break;
            }
        }
        if (alive && ksteps > 0 && !drain(ksteps - 1, ((ksteps - 1) / 2) % H16_NT)) {
            if (lane == 0) h16_fail(err, &abort_sh, 5);
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
                if (c < k) out[c] = acc[c] * inv_s * inv_x;
        }
        if (go && counters != nullptr) {
            // the last split CTA of this row tile runs the epilogue for it
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
    if (last_sh) {
        pdl_trigger();
        __threadfence();
        epilogue_tile_cta<KP>(epi, (int)blockIdx.x, tid, reinterpret_cast<float*>(smem),
                              (int)((Cfg::SMEM - 1024) / sizeof(float)));
        if (tid == 0) counters[blockIdx.x] = 0;   // ready for the next pass
    }
}

// ----------------------------------------------------------------------------
// [X_hi; X_lo] of x = cX H in fp16, K-major: XT16[c][j] = rn16(x_jc) and
// XT16[KP + c][j] = rn16(x_jc - XT16[c][j]) for j < n, zero rows c >= k.
// ----------------------------------------------------------------------------
__global__ void split16_kernel(const float* __restrict__ H, int64_t n, int k, int KP,
                               const FitState* st, __half* __restrict__ XT, int64_t ld) {
    pdl_wait();
    const int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (j >= n) return;
    const float cx = st->xscale;
    for (int c = 0; c < KP; ++c) {
        const float x = c < k ? H[j * k + c] * cx : 0.f;   // exact: cx is 2^m
        const __half h = __float2half_rn(x);
        XT[(int64_t)c * ld + j] = h;
        XT[(int64_t)(KP + c) * ld + j] = __float2half_rn(x - __half2float(h));
    }
}

bool h16_supported(int k) { return k >= 1 && k <= 24; }

int h16_set_stall(int on) {
    const int v = on ? 1 : 0;
    SYMNMF_CUDA_TRY(cudaMemcpyToSymbol(g_h16_stall, &v, sizeof(int)));
    return SYMNMF_OK;
}

int64_t h16_ld(int64_t n) { return (n + H16_BK - 1) / H16_BK * H16_BK; }

size_t h16_xt_halves(int64_t n, int k) { return (size_t)2 * ((k + 7) / 8 * 8) * h16_ld(n); }

int launch_split16(const float* H, int64_t n, int k, const FitState* st, uint16_t* XT16,
                   cudaStream_t s) {
    const int KP = (k + 7) / 8 * 8;
    const unsigned blocks = (unsigned)((n + 255) / 256);
    SYMNMF_CUDA_TRY(launch_pdl(split16_kernel, dim3(blocks), dim3(256), 0, s, H, n, k, KP, st,
                               reinterpret_cast<__half*>(XT16), h16_ld(n)));
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

static PFN_cuTensorMapEncodeTiled_v12000 h16_encode_fn() {
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

// [X_hi; X_lo] fp16 operand: 2 KP rows of n columns (row pitch ld halves), a
// box of 64 columns x 2 KP rows, 128-byte swizzle
static int h16_map_x(CUtensorMap* m, const uint16_t* XT, int64_t n, int KP, int64_t ld) {
    auto fn = h16_encode_fn();
    if (fn == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)(2 * KP)};
    cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    cuuint32_t box[2] = {(cuuint32_t)H16_BK, (cuuint32_t)(2 * KP)};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<uint16_t*>(XT), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled (fp16 operand) failed (%d)", (int)r);
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

// The split warps' arithmetic on a plain array (test hook): x[4i .. 4i+3] ->
// hi[2i], hi[2i+1], lo[2i], lo[2i+1], as split_scaled4 produces them.
__global__ void split_probe_kernel(const float4* __restrict__ x, int64_t quads, float cs,
                                   uint32_t* __restrict__ hi, uint32_t* __restrict__ lo) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= quads) return;
    split_scaled4(x[i], cs, hi[2 * i], hi[2 * i + 1], lo[2 * i], lo[2 * i + 1]);
}

int launch_split_probe(const float* x, int64_t n, float cs, uint32_t* hi, uint32_t* lo,
                       cudaStream_t s) {
    const int64_t quads = n / 4;
    if (quads <= 0) return SYMNMF_OK;
    split_probe_kernel<<<(unsigned)((quads + 255) / 256), 256, 0, s>>>(
        reinterpret_cast<const float4*>(x), quads, cs, hi, lo);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

TcPlan plan_stream_h16(const Dev& d, int64_t n, int k) {
    TcPlan p;
    p.n = n;
    p.ncols = n;
    p.k = k;
    p.KP = (k + 7) / 8 * 8;
    p.j0 = 0;
    p.j1 = n;
    p.tiles = (n + H16_BM - 1) / H16_BM;
    const int64_t steps = std::max<int64_t>(1, (n + H16_BK - 1) / H16_BK);
    // a stage is two TF32-stream stages' worth of S, at about their cadence
    p.splits = choose_splits(p.tiles, steps, (int64_t)d.sms * 2, 32768.0, 1.1e-6);
    p.jspan = (steps + p.splits - 1) / p.splits * H16_BK;
    return p;
}

int launch_stream_h16(const TcPlan& p, const float* S, int64_t lds, const uint16_t* XT16,
                      float* part, int* err, const FitState* st, cudaStream_t s,
                      const EpiArgs* epi, int* counters) {
    if (!h16_supported(p.k) || epi == nullptr || counters == nullptr || st == nullptr) {
        set_error("fp16 S-stream: k must be in [1, 24], with the fused epilogue and a fit state");
        return SYMNMF_ERR_INVALID_ARG;
    }
    CUtensorMap mapS, mapX;
    SYMNMF_TRY(make_map(&mapS, S, p.ncols, p.n, lds, H16_BM));
    SYMNMF_TRY(h16_map_x(&mapX, XT16, p.ncols, p.KP, h16_ld(p.ncols)));
    dim3 grid((unsigned)p.tiles, (unsigned)p.splits);
#define SYMNMF_H16(KP)                                                                        \
    do {                                                                                      \
        auto kern = stream_h16_kernel<KP>;                                                    \
        /* once per process (thread-safe static initialisation) */                            \
        static const cudaError_t attr_rc = cudaFuncSetAttribute(                              \
            kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)H16Cfg<KP>::SMEM);        \
        SYMNMF_CUDA_TRY(attr_rc);                                                             \
        SYMNMF_CUDA_TRY(launch_pdl(kern, grid, dim3(H16_THREADS), H16Cfg<KP>::SMEM, s, mapS,  \
                                   mapX, p.n, p.k, p.j0, p.j1, p.jspan, part, err, st, *epi,  \
                                   counters));                                                \
    } while (0)
    switch (p.KP) {
        case 8: SYMNMF_H16(8); break;
        case 16: SYMNMF_H16(16); break;
        default: SYMNMF_H16(24); break;
    }
#undef SYMNMF_H16
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf

extern "C" int symnmf_test_split16(const float* x, int64_t n, float scale, uint32_t* hi, uint32_t* lo,
                                   symnmf_stream_t stream) {
    symnmf::clear_error();
    if (n < 0 || n % 4 != 0 || (n > 0 && (x == nullptr || hi == nullptr || lo == nullptr)) ||
        (reinterpret_cast<uintptr_t>(x) & 15u) != 0 || (reinterpret_cast<uintptr_t>(hi) & 3u) != 0 ||
        (reinterpret_cast<uintptr_t>(lo) & 3u) != 0) {
        symnmf::set_error("symnmf_test_split16: n must be a multiple of 4 and x 16-byte aligned");
        return SYMNMF_ERR_INVALID_ARG;
    }
    return symnmf::launch_split_probe(x, n, scale, hi, lo, (cudaStream_t)stream);
}
