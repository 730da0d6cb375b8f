// Symmetric Gram of the builders on the tensor cores:
//     S_ij = epi( sum_t Z_ti Z_tj )
// with Z the normalised returns (|Pearson correlation|: epi = |.|, S_ii = 1)
// or the tail angular components (TPDM: epi = scale * .) -- [CaS] "Tracking
// stability through time with the Rand index"; the one dense contraction of
// the pipeline (2 n^2 T flop).
//
// Z enters transposed and K-major as two planes of n_pad x Kp, a hi part F and
// a remainder L with Z = F + L to about 2^-22, so that
//     Z^T Z = F.F + (F.L + L.F) + (L.L, dropped)
// accumulated in two TMEM accumulators (main and correction):
//   |corr|  fp16 planes of c z (c = 2^14, both parts rounded to nearest),
//           kind::f16 MMAs (K = 16) at twice the TF32 rate, the sum scaled
//           back by c^-2 (exact) in the epilogue
//   TPDM    fp32 planes: F the values (the tensor core reads their TF32 part),
//           L = w - trunc_tf32(w) exact; kind::tf32 MMAs (K = 8)
// A stage holds 128 bytes of each row in either case (64 fp16 or 32 fp32
// contraction columns), so the shared-memory layout and the descriptors'
// 32-byte steps are the same for both.
//
// Persistent: one CTA per SM walks its share of the 128 x 128 output tiles
// (I <= J, the upper triangle of tiles; each tile is also written
// transposed), 256 threads:
//   warp 0      TMA producer: per stage the rows I of F and L and, off the
//               diagonal, the rows J of F and L (16 KB each), one stage ring
//               across the CTA's tiles
//   warp 1      MMA issuer (M = N = 128, both operands in shared memory) into
//               one of two TMEM accumulator sets, so that a tile's epilogue
//               overlaps the next tile's loads and MMAs
//   warp 2      TMEM allocator
//   warps 4-7   epilogue: thread r owns row I0 + r, reads the accumulators in
//               32-column chunks, stages S[I-tile][chunk] (128-byte swizzle)
//               and its transpose in shared memory and writes both with TMA
//               bulk stores
#include <cudaTypedefs.h>

#include <cmath>

#include "common.cuh"
#include "sm100.cuh"

namespace symnmf {

constexpr int GT_BM = 128;                    // tile rows and columns
constexpr int GT_ROW_BYTES = 128;             // bytes of each operand row per stage
constexpr int GT_NS_MAX = 3;                  // pipeline stages (|corr|; TPDM uses 2)
constexpr int GT_THREADS = 256;
constexpr uint32_t GT_PLANE = GT_BM * GT_ROW_BYTES; // 16 KB: 128 rows x 128 B
constexpr uint32_t GT_STAGE = 4 * GT_PLANE;        // AF, AL, BF, BL
constexpr uint32_t GT_OUT = GT_BM * 32 * 4;        // 16 KB: one 32-column output chunk
// |corr| (long contraction): a 3-stage ring, one staging pair for the output;
// TPDM (2 stages per tile, bound by the writes): a 2-stage ring and two staging
// pairs, so a chunk is written while the previous chunk's stores still read
template <int MODE> struct GtShape;
constexpr uint32_t GT_ACC = 256;                   // one accumulator set: main [0,128), correction [128,256)
constexpr uint32_t GT_TMEM_COLS = 2 * GT_ACC;      // two sets: a tile drains while the next accumulates

enum GramTcMode { GT_CORR = 0, GT_TPDM = 1 };
// BK: contraction columns per stage (128 bytes of fp16 or fp32)
template <> struct GtShape<GT_CORR> { static constexpr int NS = 3, NOUT = 1, BK = 64; };
template <> struct GtShape<GT_TPDM> { static constexpr int NS = 2, NOUT = 2, BK = 32; };
template <int MODE>
constexpr uint32_t gt_smem() {
    return GtShape<MODE>::NS * GT_STAGE + GtShape<MODE>::NOUT * 2 * GT_OUT + 1024;
}

// (a, b), a <= b, from a linear index over an upper triangle, b-major
__device__ __forceinline__ void gt_tri(int64_t x, int64_t* a, int64_t* b) {
    int64_t j = (int64_t)((sqrt(8.0 * (double)x + 1.0) - 1.0) * 0.5);
    while ((j + 1) * (j + 2) / 2 <= x) ++j;
    while (j * (j + 1) / 2 > x) --j;
    *b = j;
    *a = x - j * (j + 1) / 2;
}

// The tiles are visited in groups of GT_GROUP x GT_GROUP (the tile grid padded
// to whole groups, groups column-major over the upper triangle), so that the
// CTAs running at the same time share GT_GROUP row blocks of each operand in
// L2 instead of each fetching its own.  Tiles in the padding are skipped, by
// every role alike.
constexpr int64_t GT_GROUP = 16;
constexpr int64_t GT_G2 = GT_GROUP * GT_GROUP, GT_GD = GT_GROUP * (GT_GROUP + 1) / 2;
__host__ __device__ __forceinline__ int64_t gt_before(int64_t c) {   // tiles in group columns < c
    return GT_G2 * c * (c - 1) / 2 + c * GT_GD;
}
int64_t gt_virtual_tiles(int64_t nt) { return gt_before((nt + GT_GROUP - 1) / GT_GROUP); }

// tile (I, J), I <= J, of virtual index v; false for a tile in the padding
__device__ __forceinline__ bool gt_tile(int64_t v, int64_t nt, int64_t* I, int64_t* J) {
    int64_t c = (int64_t)(sqrt(2.0 * (double)v) / (double)GT_GROUP);
    while (c > 0 && gt_before(c) > v) --c;
    while (gt_before(c + 1) <= v) ++c;
    const int64_t off = v - gt_before(c);
    if (off < c * GT_G2) {   // off-diagonal group (gi, c), gi < c
        const int64_t gi = off / GT_G2, l = off % GT_G2;
        *I = gi * GT_GROUP + l / GT_GROUP;
        *J = c * GT_GROUP + l % GT_GROUP;
    } else {                 // diagonal group (c, c)
        int64_t a, b;
        gt_tri(off - c * GT_G2, &a, &b);
        *I = c * GT_GROUP + a;
        *J = c * GT_GROUP + b;
    }
    return *J < nt;
}

// Persistent: CTA b takes the tiles b, b + grid, b + 2 grid, ...
template <int MODE>
__global__ void __launch_bounds__(GT_THREADS, 1)
gram_tc_kernel(const __grid_constant__ CUtensorMap mapF, const __grid_constant__ CUtensorMap mapL,
               const __grid_constant__ CUtensorMap mapD, const __grid_constant__ CUtensorMap mapT,
               int64_t n, int Kp, int64_t vtiles, float scale, int* __restrict__ err) {
    using namespace sm100;
    extern __shared__ uint8_t gt_smem_raw[];
    constexpr int GT_NS = GtShape<MODE>::NS, NOUT = GtShape<MODE>::NOUT;
    static_assert(gt_smem<MODE>() <= 227 * 1024, "shared memory per block");
    __shared__ __align__(8) uint64_t bar_full[GT_NS_MAX], bar_empty[GT_NS_MAX];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], bar_fin;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh, ep_fail_sh, go_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(gt_smem_raw) + 1023) & ~uintptr_t(1023));
    // staging pair p: outD(p) [128 rows][32] with 128-byte swizzle, then outT(p) [32 rows][128]
    float* outBase = reinterpret_cast<float*>(smem + GT_NS * GT_STAGE);

    constexpr int GT_BK = GtShape<MODE>::BK;
    const int ksteps = Kp / GT_BK;
    const int64_t nt = (n + GT_BM - 1) / GT_BM;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < GT_NS; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);   // one arrival per epilogue warp
        }
        mbar_init(&bar_fin, 1);
        abort_sh = 0;
        ep_fail_sh = 0;
        go_sh = 1;
        fence_mbar_init();
        prefetch_tmap(&mapF);
        prefetch_tmap(&mapL);
        prefetch_tmap(&mapD);
        prefetch_tmap(&mapT);
    }
    if (warp == 2) {
        tmem_alloc(&tmem_base_sh, GT_TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tbase = tmem_base_sh;

    auto plane = [&](int slot, int q) { return smem + slot * GT_STAGE + q * GT_PLANE; };

    if (warp == 0 && lane == 0) {
        // ---------------- TMA producer: one stage ring across all of this CTA's tiles
        int64_t g = 0;   // stages issued
        for (int64_t x = blockIdx.x; x < vtiles && !abort_sh; x += gridDim.x) {
            int64_t I, J;
            if (!gt_tile(x, nt, &I, &J)) continue;
            const bool diag = I == J;
            const uint32_t stage_bytes = diag ? 2 * GT_PLANE : 4 * GT_PLANE;
            for (int s = 0; s < ksteps; ++s, ++g) {
                if (abort_sh) break;
                const int slot = (int)(g % GT_NS);
                if (g >= GT_NS && !mbar_wait(&bar_empty[slot], (uint32_t)((g / GT_NS) & 1) ^ 1u)) {
                    abort_sh = 1;
                    atomicExch(err, 1);
                    break;
                }
                mbar_arrive_expect_tx(&bar_full[slot], stage_bytes);
                const int32_t xk = s * GT_BK;
                tma_load_2d(plane(slot, 0), &mapF, xk, (int32_t)(I * GT_BM), &bar_full[slot]);
                tma_load_2d(plane(slot, 1), &mapL, xk, (int32_t)(I * GT_BM), &bar_full[slot]);
                if (!diag) {
                    tma_load_2d(plane(slot, 2), &mapF, xk, (int32_t)(J * GT_BM), &bar_full[slot]);
                    tma_load_2d(plane(slot, 3), &mapL, xk, (int32_t)(J * GT_BM), &bar_full[slot]);
                }
            }
        }
        if (abort_sh) {   // let the copies already issued land before the CTA exits
            for (int64_t q = g > GT_NS ? g - GT_NS : 0; q < g; ++q)
                mbar_wait(&bar_full[q % GT_NS], (uint32_t)((q / GT_NS) & 1));
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer: tile u accumulates into set u % 2
        constexpr uint32_t id = MODE == GT_CORR ? idesc_f16(GT_BM, GT_BM) : idesc_tf32(GT_BM, GT_BM);
        int64_t g = 0;
        int u = 0;
        for (int64_t x = blockIdx.x; x < vtiles && !abort_sh; x += gridDim.x) {
            int64_t I, J;
            if (!gt_tile(x, nt, &I, &J)) continue;
            const bool diag = I == J;
            const int b = u & 1;
            if (u >= 2 && !mbar_wait(&acc_empty[b], (uint32_t)((u >> 1) - 1) & 1u)) {
                abort_sh = 1;
                atomicExch(err, 2);
                break;
            }
            tc_fence_after();
            const uint32_t dm = tbase + (uint32_t)b * GT_ACC, dc = dm + 128u;
            for (int s = 0; s < ksteps; ++s, ++g) {
                if (abort_sh) break;
                const int slot = (int)(g % GT_NS);
                if (!mbar_wait(&bar_full[slot], (uint32_t)((g / GT_NS) & 1))) {
                    abort_sh = 1;
                    atomicExch(err, 2);
                    break;
                }
                tc_fence_after();
                const uint32_t af = smem_u32(plane(slot, 0)), al = smem_u32(plane(slot, 1));
                const uint32_t bf = diag ? af : smem_u32(plane(slot, 2));
                const uint32_t bl = diag ? al : smem_u32(plane(slot, 3));
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {   // four MMAs of 32 bytes of K each
                    const uint32_t o = (uint32_t)kk * 32u;
                    const uint32_t acc = (s | kk) ? 1u : 0u;
                    if constexpr (MODE == GT_CORR) {
                        umma_f16_ss(dm, umma_desc_sw128(af + o), umma_desc_sw128(bf + o), id, acc);
                        umma_f16_ss(dc, umma_desc_sw128(af + o), umma_desc_sw128(bl + o), id, acc);
                        umma_f16_ss(dc, umma_desc_sw128(al + o), umma_desc_sw128(bf + o), id, 1u);
                    } else {
                        umma_tf32_ss(dm, umma_desc_sw128(af + o), umma_desc_sw128(bf + o), id, acc);
                        umma_tf32_ss(dc, umma_desc_sw128(af + o), umma_desc_sw128(bl + o), id, acc);
                        umma_tf32_ss(dc, umma_desc_sw128(al + o), umma_desc_sw128(bf + o), id, 1u);
                    }
                }
                umma_commit(&bar_empty[slot]);
            }
            if (abort_sh) break;
            umma_commit(&acc_full[b]);
            ++u;
        }
        umma_commit(&bar_fin);
        mbar_wait(&bar_fin, 0);   // every MMA has finished before TMEM is freed
    } else if (warp >= 4) {
        // ---------------- epilogue: thread r owns row I0 + r of the tile; the four
        // warps take every decision together (they share named barrier 1)
        const int wl = warp & 3;
        const int r = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        int u = 0, cq = 0;   // tiles and output chunks handled
        for (int64_t x = blockIdx.x; x < vtiles; x += gridDim.x) {
            int64_t I, J;
            if (!gt_tile(x, nt, &I, &J)) continue;
            const bool diag = I == J;
            const int b = u & 1;
            const uint32_t par = (uint32_t)(u >> 1) & 1u;   // this tile's use of set b
            ++u;
            const int64_t I0 = I * GT_BM, J0 = J * GT_BM;
            const bool w_ok = __all_sync(0xffffffffu, mbar_wait(&acc_full[b], par));
            if (lane == 0 && !w_ok) atomicOr(const_cast<int*>(&ep_fail_sh), 1);
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (r == 0) go_sh = (ep_fail_sh == 0 && abort_sh == 0) ? 1 : 0;
            asm volatile("bar.sync 1, 128;" ::: "memory");
            if (!go_sh) break;
            tc_fence_after();
            const int64_t i = I0 + r;
            const uint32_t acc_col = tbase + lane_off + (uint32_t)b * GT_ACC;
#pragma unroll 1
            for (int q = 0; q < GT_BM / 32; ++q) {
                uint32_t vm[32], vc[32];
                tmem_ld_32x32b_x32(acc_col + (uint32_t)q * 32u, vm);
                tmem_ld_32x32b_x32(acc_col + 128u + (uint32_t)q * 32u, vc);
                tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float z = __uint_as_float(vm[e]) + __uint_as_float(vc[e]);
                    if (MODE == GT_CORR) {
                        z = fabsf(z) * (1.f / (CORR_F16_SCALE * CORR_F16_SCALE));   // exact: 2^-28
                        if (i == J0 + q * 32 + e) z = 1.f;
                    } else {
                        z *= scale;
                    }
                    v[e] = z;
                }
                // the staging tiles are free once the last chunk's stores have read them
                float* outD = outBase + (size_t)(cq % NOUT) * 2 * GT_BM * 32;
                float* outT = outD + GT_BM * 32;
                ++cq;
                if (r == 0) {
                    if (NOUT == 2) bulk_wait_read_but_one();   // the pair written two chunks ago is free
                    else bulk_wait_read_all();
                }
                asm volatile("bar.sync 1, 128;" ::: "memory");
                float* rowp = outD + r * 32;   // row r: 16-byte chunk c sits at c ^ (r & 7)
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    *reinterpret_cast<float4*>(rowp + ((c ^ (r & 7)) << 2)) =
                        make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
                if (!diag) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) outT[e * GT_BM + r] = v[e];
                }
                fence_proxy_async_smem();
                asm volatile("bar.sync 1, 128;" ::: "memory");
                if (r == 0) {
                    if (J0 + q * 32 < n) {   // chunks wholly past the end are not stored
                        tma_store_2d(&mapD, outD, (int32_t)(J0 + q * 32), (int32_t)I0);
                        if (!diag) tma_store_2d(&mapT, outT, (int32_t)I0, (int32_t)(J0 + q * 32));
                    }
                    bulk_commit_group();   // one group per chunk (possibly empty): the waits count chunks
                }
            }
            // this accumulator set has been read: the MMA issuer may reuse it
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[b]);
        }
        if (r == 0 && (ep_fail_sh || !go_sh)) {
            if (ep_fail_sh) atomicExch(err, 3);
        }
        if (r == 0) bulk_wait_all();   // stores complete before the CTA's shared memory goes
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, GT_TMEM_COLS);
    }
}

static PFN_cuTensorMapEncodeTiled_v12000 gt_encode_fn() {
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

// Load map over an operand plane: rows x Kp elements of `esize` bytes, a box of
// 128 bytes x GT_BM rows.
static int gt_map(CUtensorMap* m, const void* base, int64_t Kp, int64_t rows, bool f16) {
    auto fn = gt_encode_fn();
    if (fn == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    const int esize = f16 ? 2 : 4;
    cuuint64_t dims[2] = {(cuuint64_t)Kp, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)Kp * esize};
    cuuint32_t box[2] = {(cuuint32_t)(GT_ROW_BYTES / esize), (cuuint32_t)GT_BM};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2,
                          const_cast<void*>(base), dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

// Store map over S (n x n, row stride lds floats) with a box of bx x by floats.
static int gt_store_map(CUtensorMap* m, float* S, int64_t n, int64_t lds, uint32_t bx, uint32_t by,
                        CUtensorMapSwizzle swz) {
    auto fn = gt_encode_fn();
    if (fn == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    cuuint64_t dims[2] = {(cuuint64_t)n, (cuuint64_t)n};
    cuuint64_t strides[1] = {(cuuint64_t)lds * sizeof(float)};
    cuuint32_t box[2] = {bx, by};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, S, dims, strides, box, estr,
                          CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled (store) failed (%d)", (int)r);
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

// F, L: n_pad x Kp (n_pad multiple of 128, zero padding); fp16 with Kp a
// multiple of 64 for |corr|, fp32 with Kp a multiple of 32 for TPDM.
int launch_gram_tc(const void* F, const void* L, int64_t n, int64_t n_pad, int64_t Kp,
                   bool corr, float scale, float* S, int64_t lds, int* err, cudaStream_t s) {
    if (n_pad % GT_BM != 0 || Kp % (corr ? GtShape<GT_CORR>::BK : GtShape<GT_TPDM>::BK) != 0) {
        set_error("tensor-core Gram: operand planes not padded to whole stages");
        return SYMNMF_ERR_INVALID_ARG;
    }
    CUtensorMap mapF, mapL, mapD, mapT;
    SYMNMF_TRY(gt_map(&mapF, F, Kp, n_pad, corr));
    SYMNMF_TRY(gt_map(&mapL, L, Kp, n_pad, corr));
    SYMNMF_TRY(gt_store_map(&mapD, S, n, lds, 32, GT_BM, CU_TENSOR_MAP_SWIZZLE_128B));
    SYMNMF_TRY(gt_store_map(&mapT, S, n, lds, GT_BM, 32, CU_TENSOR_MAP_SWIZZLE_NONE));
    const int64_t nt = n_pad / GT_BM;
    const int64_t vtiles = gt_virtual_tiles(nt);
    int dev = 0, sms = 148;
    SYMNMF_CUDA_TRY(cudaGetDevice(&dev));
    SYMNMF_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    const unsigned grid = (unsigned)std::min<int64_t>(nt * (nt + 1) / 2, sms);   // persistent, one CTA per SM
    if (corr) {
        // once per process (thread-safe static initialisation)
        static const cudaError_t attr = cudaFuncSetAttribute(
            gram_tc_kernel<GT_CORR>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gt_smem<GT_CORR>());
        SYMNMF_CUDA_TRY(attr);
        gram_tc_kernel<GT_CORR><<<grid, GT_THREADS, gt_smem<GT_CORR>(), s>>>(mapF, mapL, mapD, mapT, n, (int)Kp,
                                                                 vtiles, scale, err);
    } else {
        static const cudaError_t attr = cudaFuncSetAttribute(
            gram_tc_kernel<GT_TPDM>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)gt_smem<GT_TPDM>());
        SYMNMF_CUDA_TRY(attr);
        gram_tc_kernel<GT_TPDM><<<grid, GT_THREADS, gt_smem<GT_TPDM>(), s>>>(mapF, mapL, mapD, mapT, n, (int)Kp,
                                                                 vtiles, scale, err);
    }
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf
