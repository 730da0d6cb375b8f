// Symmetric Gram of the builders on the tensor cores:
//     S_ij = epi( sum_t Z_ti Z_tj )
// with Z the normalised returns (|Pearson correlation|: epi = |.|, S_ii = 1)
// or the tail angular components (TPDM: epi = scale * .) -- [CaS] "Tracking
// stability through time with the Rand index"; the one dense contraction of
// the pipeline (2 n^2 T flop).
//
// Z enters transposed and K-major as two planes of n_pad x Kp: ZF (the fp32
// values, which the tensor core truncates to their TF32 part) and ZL (the
// exact remainder z - trunc(z)), so
//     Z^T Z = ZF.ZF + (ZF.ZL + ZL.ZF) + O(2^-22)
// accumulated in two TMEM accumulators (main and correction).
//
// One CTA per 128 x 128 output tile (I <= J, upper triangle of tiles; the
// tile is also written transposed), 256 threads:
//   warp 0      TMA producer: per 32-column stage the rows I of ZF and ZL and,
//               off the diagonal, the rows J of ZF and ZL (16 KB each)
//   warp 1      MMA issuer (M = N = 128, K = 8, both operands in shared memory)
//   warp 2      TMEM allocator
//   warps 4-7   epilogue: thread r owns row I0 + r, reads the accumulators in
//               32-column chunks and writes S[i][J-tile] and S[J-tile][i]
#include <cudaTypedefs.h>

#include <cmath>

#include "common.cuh"
#include "sm100.cuh"

namespace symnmf {

constexpr int GT_BM = 128;                    // tile rows and columns
constexpr int GT_BK = 32;                     // contraction columns per stage
constexpr int GT_NS = 3;                      // pipeline stages
constexpr int GT_THREADS = 256;
constexpr uint32_t GT_PLANE = GT_BM * GT_BK * 4;   // 16 KB: 128 rows x 128 B
constexpr uint32_t GT_STAGE = 4 * GT_PLANE;        // AF, AL, BF, BL
constexpr uint32_t GT_SMEM = GT_NS * GT_STAGE + 1024;
constexpr uint32_t GT_TMEM_COLS = 256;             // main [0,128), correction [128,256)

enum GramTcMode { GT_CORR = 0, GT_TPDM = 1 };

template <int MODE>
__global__ void __launch_bounds__(GT_THREADS, 1)
gram_tc_kernel(const __grid_constant__ CUtensorMap mapF, const __grid_constant__ CUtensorMap mapL,
               int64_t n, int Kp, float scale, float* __restrict__ S, int64_t lds,
               int* __restrict__ err) {
    using namespace sm100;
    extern __shared__ uint8_t gt_smem_raw[];
    __shared__ __align__(8) uint64_t bar_full[GT_NS], bar_empty[GT_NS], bar_acc;
    __shared__ uint32_t tmem_base_sh;
    __shared__ volatile int abort_sh;

    uint8_t* smem = reinterpret_cast<uint8_t*>(
        (reinterpret_cast<uintptr_t>(gt_smem_raw) + 1023) & ~uintptr_t(1023));

    // tile (I, J), I <= J, from the linear index over the upper triangle
    const int64_t x = blockIdx.x;
    int64_t J = (int64_t)((sqrt(8.0 * (double)x + 1.0) - 1.0) * 0.5);
    while ((J + 1) * (J + 2) / 2 <= x) ++J;
    while (J * (J + 1) / 2 > x) --J;
    const int64_t I = x - J * (J + 1) / 2;
    const bool diag = I == J;
    const int64_t I0 = I * GT_BM, J0 = J * GT_BM;
    const int ksteps = Kp / GT_BK;
    const uint32_t stage_bytes = diag ? 2 * GT_PLANE : 4 * GT_PLANE;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    if (tid == 0) {
        for (int s = 0; s < GT_NS; ++s) {
            mbar_init(&bar_full[s], 1);
            mbar_init(&bar_empty[s], 1);
        }
        mbar_init(&bar_acc, 1);
        abort_sh = 0;
        fence_mbar_init();
        prefetch_tmap(&mapF);
        prefetch_tmap(&mapL);
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
        // ---------------- TMA producer
        int issued = 0;
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % GT_NS;
            const uint32_t ph = (uint32_t)(s / GT_NS) & 1u;
            if (s >= GT_NS && !mbar_wait(&bar_empty[slot], ph ^ 1u)) {
                abort_sh = 1;
                atomicExch(err, 1);
                break;
            }
            mbar_arrive_expect_tx(&bar_full[slot], stage_bytes);
            const int32_t xk = s * GT_BK;
            tma_load_2d(plane(slot, 0), &mapF, xk, (int32_t)I0, &bar_full[slot]);
            tma_load_2d(plane(slot, 1), &mapL, xk, (int32_t)I0, &bar_full[slot]);
            if (!diag) {
                tma_load_2d(plane(slot, 2), &mapF, xk, (int32_t)J0, &bar_full[slot]);
                tma_load_2d(plane(slot, 3), &mapL, xk, (int32_t)J0, &bar_full[slot]);
            }
            ++issued;
        }
        if (abort_sh) {
            for (int s = max(0, issued - GT_NS); s < issued; ++s)
                mbar_wait(&bar_full[s % GT_NS], (uint32_t)(s / GT_NS) & 1u);
        }
    } else if (warp == 1 && lane == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t id = idesc_tf32(GT_BM, GT_BM);
        for (int s = 0; s < ksteps; ++s) {
            if (abort_sh) break;
            const int slot = s % GT_NS;
            const uint32_t ph = (uint32_t)(s / GT_NS) & 1u;
            if (!mbar_wait(&bar_full[slot], ph)) {
                abort_sh = 1;
                atomicExch(err, 2);
                break;
            }
            tc_fence_after();
            const uint32_t af = smem_u32(plane(slot, 0)), al = smem_u32(plane(slot, 1));
            const uint32_t bf = diag ? af : smem_u32(plane(slot, 2));
            const uint32_t bl = diag ? al : smem_u32(plane(slot, 3));
#pragma unroll
            for (int kk = 0; kk < GT_BK / 8; ++kk) {
                const uint32_t o = (uint32_t)kk * 32u;
                const uint32_t acc = (s | kk) ? 1u : 0u;
                umma_tf32_ss(tbase, umma_desc_sw128(af + o), umma_desc_sw128(bf + o), id, acc);
                umma_tf32_ss(tbase + 128u, umma_desc_sw128(af + o), umma_desc_sw128(bl + o), id, acc);
                umma_tf32_ss(tbase + 128u, umma_desc_sw128(al + o), umma_desc_sw128(bf + o), id, 1u);
            }
            umma_commit(&bar_empty[slot]);
        }
        umma_commit(&bar_acc);
        mbar_wait(&bar_acc, 0);   // (also when aborting: MMAs finish before TMEM is freed)
    } else if (warp >= 4) {
        // ---------------- epilogue (control flow warp-uniform for tcgen05.ld)
        const int wl = warp & 3;
        const int r = wl * 32 + lane;
        const uint32_t lane_off = (uint32_t)(wl * 32) << 16;
        const bool ok = __all_sync(0xffffffffu, mbar_wait(&bar_acc, 0)) &&
                        !__any_sync(0xffffffffu, abort_sh != 0);
        if (!ok) {
            if (lane == 0) atomicExch(err, 3);
        } else {
            tc_fence_after();
            const int64_t i = I0 + r;
#pragma unroll 1
            for (int q = 0; q < GT_BM / 32; ++q) {
                uint32_t vm[32], vc[32];
                tmem_ld_32x32b_x32(tbase + lane_off + (uint32_t)q * 32u, vm);
                tmem_ld_32x32b_x32(tbase + lane_off + 128u + (uint32_t)q * 32u, vc);
                tmem_wait_ld();
                float v[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    float z = __uint_as_float(vm[e]) + __uint_as_float(vc[e]);
                    const int64_t j = J0 + q * 32 + e;
                    if (MODE == GT_CORR) {
                        z = fabsf(z);
                        if (i == j) z = 1.f;
                    } else {
                        z *= scale;
                    }
                    v[e] = z;
                }
                const int64_t j0 = J0 + q * 32;
                if (i < n) {
                    float* dst = S + i * lds + j0;
                    if (j0 + 32 <= n) {
#pragma unroll
                        for (int e = 0; e < 32; e += 4)
                            *reinterpret_cast<float4*>(dst + e) =
                                make_float4(v[e], v[e + 1], v[e + 2], v[e + 3]);
                    } else {
                        for (int e = 0; e < 32; ++e)
                            if (j0 + e < n) dst[e] = v[e];
                    }
                }
                if (!diag && i < n) {
                    // transposed block: lanes write consecutive i of row j (coalesced)
#pragma unroll
                    for (int e = 0; e < 32; ++e)
                        if (j0 + e < n) S[(j0 + e) * lds + i] = v[e];
                }
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tbase, GT_TMEM_COLS);
    }
}

static PFN_cuTensorMapEncodeTiled_v12000 gt_encode_fn() {
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    if (fn == nullptr) {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }
    return fn;
}

static int gt_map(CUtensorMap* m, const float* base, int64_t Kp, int64_t rows) {
    auto fn = gt_encode_fn();
    if (fn == nullptr) {
        set_error("cuTensorMapEncodeTiled is not available from the driver");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    cuuint64_t dims[2] = {(cuuint64_t)Kp, (cuuint64_t)rows};
    cuuint64_t strides[1] = {(cuuint64_t)Kp * sizeof(float)};
    cuuint32_t box[2] = {(cuuint32_t)GT_BK, (cuuint32_t)GT_BM};
    cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<float*>(base), dims,
                          strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                          CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        set_error("cuTensorMapEncodeTiled failed (%d)", (int)r);
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

// ZF, ZL: n_pad x Kp (n_pad multiple of 128, Kp multiple of 32, zero padding).
int launch_gram_tc(const float* ZF, const float* ZL, int64_t n, int64_t n_pad, int64_t Kp,
                   bool corr, float scale, float* S, int64_t lds, int* err, cudaStream_t s) {
    CUtensorMap mapF, mapL;
    SYMNMF_TRY(gt_map(&mapF, ZF, Kp, n_pad));
    SYMNMF_TRY(gt_map(&mapL, ZL, Kp, n_pad));
    const int64_t nt = n_pad / GT_BM;
    const int64_t pairs = nt * (nt + 1) / 2;
    if (pairs > 0x7fffffffLL) {
        set_error("n = %lld too large for the Gram tile grid", (long long)n);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (corr) {
        SYMNMF_CUDA_TRY(cudaFuncSetAttribute(gram_tc_kernel<GT_CORR>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GT_SMEM));
        gram_tc_kernel<GT_CORR><<<(unsigned)pairs, GT_THREADS, GT_SMEM, s>>>(mapF, mapL, n, (int)Kp,
                                                                            scale, S, lds, err);
    } else {
        SYMNMF_CUDA_TRY(cudaFuncSetAttribute(gram_tc_kernel<GT_TPDM>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)GT_SMEM));
        gram_tc_kernel<GT_TPDM><<<(unsigned)pairs, GT_THREADS, GT_SMEM, s>>>(mapF, mapL, n, (int)Kp,
                                                                            scale, S, lds, err);
    }
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf
