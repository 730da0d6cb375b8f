// S-stream kernels of the SymNMF fit.
//
// One full-batch iteration ([CaS] "Factorization at scale": the dominant S H
// products; [SMI] AdaptGrow sketch: g = 4 (H (H^T H) - S H), AdaGrad step):
//
//   stream_partial   part[s] = S[J_s, :]^T X[J_s, :]  (contraction split s)
//   epilogue         per row i: P_i = sum_s part[s]_i, tr partial, gradient,
//                    AdaGrad accumulator and projected step, Gram partial of
//                    the new rows, all in registers/shared memory
//   reduce_finalize  deterministic fp64 reduction of the Gram and trace
//                    partials; the last block evaluates the trace-identity
//                    loss f(H_t) = ||S||^2 - 2 tr(H^T S H) + ||H^T H||^2 and
//                    the stopping test
//
// S is symmetric with full storage, so column j of S is its row j: the
// contraction over j reads rows of S, each a contiguous, coalesced run of
// the output index i.  Every reduction has a fixed order, so results are
// bitwise reproducible run to run on a given device.
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"

namespace symnmf {

// ----------------------------------------------------------------------------
// S-stream partial product (CUDA cores)
// ----------------------------------------------------------------------------
constexpr int ST_THREADS = 128;
constexpr int ST_TILE = ST_THREADS * 4;  // output rows (instruments) per CTA
constexpr int ST_JCHUNK = 32;            // rows of X staged in shared memory at once

__device__ __forceinline__ float4 ld_stream(const float* p) {
    // S is read exactly once per pass: do not allocate it in L1.
    float4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                 : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
                 : "l"(p));
    return v;
}

template <int KP>
__global__ void __launch_bounds__(ST_THREADS)
stream_partial_kernel(const float* __restrict__ S, int64_t lds, int64_t n, int k,
                      int64_t j0, int64_t j1, int64_t jspan, int64_t ldx,
                      const float* __restrict__ Xa, const float* __restrict__ Xb,
                      float* __restrict__ part, const FitState* st) {
    if (st != nullptr && st->done) return;
    __shared__ __align__(16) float xs[ST_JCHUNK][KP];

    const int tid = threadIdx.x;
    const int64_t i0 = (int64_t)blockIdx.x * ST_TILE + tid * 4;
    const int split = blockIdx.y;
    const int c0 = blockIdx.z * KP;                 // first column of this group
    const int cw = min(KP, k - c0);                 // columns in this group
    const int64_t jb = j0 + (int64_t)split * jspan;
    const int64_t je = min(j1, jb + jspan);

    float acc[4][KP];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int c = 0; c < KP; ++c) acc[q][c] = 0.f;

    const bool active = i0 < n;
    const int tail = (int)min64(4, n - i0);  // valid lanes of the float4

    for (int64_t jc = jb; jc < je; jc += ST_JCHUNK) {
        const int cnt = (int)min64(ST_JCHUNK, je - jc);
        __syncthreads();
        for (int e = tid; e < ST_JCHUNK * KP; e += ST_THREADS) {
            const int r = e / KP, c = e % KP;
            float v = 0.f;
            if (r < cnt && c < cw) {
                const int64_t idx = (jc + r) * ldx + c0 + c;
                v = Xa[idx];
                if (Xb != nullptr) v -= Xb[idx];
            }
            xs[r][c] = v;
        }
        __syncthreads();
        if (!active) continue;
        const float* srow = S + jc * lds + i0;
#pragma unroll 4
        for (int r = 0; r < cnt; ++r) {
            float4 s4 = ld_stream(srow + (int64_t)r * lds);
            if (tail < 4) {
                if (tail < 2) s4.y = 0.f;
                if (tail < 3) s4.z = 0.f;
                s4.w = 0.f;
            }
#pragma unroll
            for (int c = 0; c < KP; c += 4) {
                const float4 x4 = *reinterpret_cast<const float4*>(&xs[r][c]);
                acc[0][c + 0] = fmaf(s4.x, x4.x, acc[0][c + 0]);
                acc[0][c + 1] = fmaf(s4.x, x4.y, acc[0][c + 1]);
                acc[0][c + 2] = fmaf(s4.x, x4.z, acc[0][c + 2]);
                acc[0][c + 3] = fmaf(s4.x, x4.w, acc[0][c + 3]);
                acc[1][c + 0] = fmaf(s4.y, x4.x, acc[1][c + 0]);
                acc[1][c + 1] = fmaf(s4.y, x4.y, acc[1][c + 1]);
                acc[1][c + 2] = fmaf(s4.y, x4.z, acc[1][c + 2]);
                acc[1][c + 3] = fmaf(s4.y, x4.w, acc[1][c + 3]);
                acc[2][c + 0] = fmaf(s4.z, x4.x, acc[2][c + 0]);
                acc[2][c + 1] = fmaf(s4.z, x4.y, acc[2][c + 1]);
                acc[2][c + 2] = fmaf(s4.z, x4.z, acc[2][c + 2]);
                acc[2][c + 3] = fmaf(s4.z, x4.w, acc[2][c + 3]);
                acc[3][c + 0] = fmaf(s4.w, x4.x, acc[3][c + 0]);
                acc[3][c + 1] = fmaf(s4.w, x4.y, acc[3][c + 1]);
                acc[3][c + 2] = fmaf(s4.w, x4.z, acc[3][c + 2]);
                acc[3][c + 3] = fmaf(s4.w, x4.w, acc[3][c + 3]);
            }
        }
    }
    if (!active) return;
    float* out = part + (int64_t)split * n * k;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        if (q >= tail) break;
        float* o = out + (i0 + q) * (int64_t)k + c0;
#pragma unroll
        for (int c = 0; c < KP; ++c)
            if (c < cw) o[c] = acc[q][c];
    }
}

StreamPlan plan_stream(const Dev& d, int64_t n, int k, int64_t j0, int64_t j1) {
    StreamPlan p;
    p.n = n;
    p.k = k;
    p.j0 = j0;
    p.j1 = j1;
    p.kp = k <= 8 ? 8 : k <= 16 ? 16 : k <= 24 ? 24 : 32;
    p.groups = (k + p.kp - 1) / p.kp;
    const int64_t tiles = (n + ST_TILE - 1) / ST_TILE;
    const int64_t target = (int64_t)d.sms * 4;  // resident CTAs we aim to fill
    int64_t splits = (target + tiles * p.groups - 1) / (tiles * p.groups);
    const int64_t len = j1 - j0;
    splits = std::max<int64_t>(1, min64(splits, (len + 63) / 64));
    p.splits = (int)min64(splits, 64);
    return p;
}

size_t stream_partial_floats(const StreamPlan& p) { return (size_t)p.splits * p.n * p.k; }

int launch_stream_partial(const StreamPlan& p, const float* S, int64_t lds,
                          const float* Xa, const float* Xb, int64_t ldx, float* part,
                          const FitState* st, cudaStream_t s) {
    const int64_t tiles = (p.n + ST_TILE - 1) / ST_TILE;
    const int64_t len = p.j1 - p.j0;
    const int64_t jspan = (len + p.splits - 1) / p.splits;
    dim3 grid((unsigned)tiles, (unsigned)p.splits, (unsigned)p.groups);
    switch (p.kp) {
        case 8:
            stream_partial_kernel<8><<<grid, ST_THREADS, 0, s>>>(S, lds, p.n, p.k, p.j0, p.j1, jspan, ldx, Xa, Xb, part, st);
            break;
        case 16:
            stream_partial_kernel<16><<<grid, ST_THREADS, 0, s>>>(S, lds, p.n, p.k, p.j0, p.j1, jspan, ldx, Xa, Xb, part, st);
            break;
        case 24:
            stream_partial_kernel<24><<<grid, ST_THREADS, 0, s>>>(S, lds, p.n, p.k, p.j0, p.j1, jspan, ldx, Xa, Xb, part, st);
            break;
        default:
            stream_partial_kernel<32><<<grid, ST_THREADS, 0, s>>>(S, lds, p.n, p.k, p.j0, p.j1, jspan, ldx, Xa, Xb, part, st);
            break;
    }
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// Epilogue: gradient, AdaGrad step and Gram partial per block of rows
// (standalone kernel around epilogue_tile; see epilogue.cuh)
// ----------------------------------------------------------------------------
int epilogue_blocks(int64_t n) { return (int)((n + EP_ROWS - 1) / EP_ROWS); }

template <int KE>
__global__ void __launch_bounds__(EP_ROWS) epilogue_kernel(const EpiArgs a) {
    if (a.st != nullptr && a.st->done) return;
    constexpr int SM_FLOATS = KE * KE > EP_ROWS * (KE + 1) ? KE * KE : EP_ROWS * (KE + 1);
    __shared__ float smem[SM_FLOATS];
    __shared__ double red[EP_ROWS / 32];
    epilogue_tile<KE>(a, blockIdx.x, threadIdx.x, smem, red);
}

int launch_epilogue(int mode, int64_t n, int k, const float* part, int splits,
                    const float* H, const float* G, float* Hn, float* Gn,
                    float* Psnap, float m_scale, float lr, float eps,
                    double* tr_part, double* gram_part, float* Y,
                    const FitState* st, cudaStream_t s, float* XT, int64_t ldxt,
                    float* hmax_part) {
    const int nb = epilogue_blocks(n);
    EpiArgs a;
    std::memset(&a, 0, sizeof(a));
    a.mode = mode;
    a.n = n;
    a.k = k;
    a.part = part;
    a.splits = splits;
    a.H = H;
    a.G = G;
    a.Hn = Hn;
    a.Gn = Gn;
    a.Psnap = Psnap;
    a.m_scale = m_scale;
    a.lr = lr;
    a.eps = eps;
    a.tr_part = tr_part;
    a.gram_part = gram_part;
    a.Y = Y;
    a.st = st;
    a.XT = XT;
    a.ldxt = ldxt;
    a.hmax_part = hmax_part;
#define SYMNMF_EP(KE) epilogue_kernel<KE><<<nb, EP_ROWS, 0, s>>>(a)
    if (k <= 8) SYMNMF_EP(8);
    else if (k <= 16) SYMNMF_EP(16);
    else if (k <= 24) SYMNMF_EP(24);
    else if (k <= 32) SYMNMF_EP(32);
    else if (k <= 48) SYMNMF_EP(48);
    else SYMNMF_EP(64);
#undef SYMNMF_EP
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// Deterministic reduction of the partials and loop bookkeeping
// ----------------------------------------------------------------------------
constexpr int RF_THREADS = 256;  // 8 warps x 32 entries per block

struct FinalScratch {
    double A_next[KMAX * KMAX];
    double tr;
    unsigned int arrived;
};

__global__ void __launch_bounds__(RF_THREADS)
reduce_finalize_kernel(int mode, int nblk, int k, const double* __restrict__ tr_part,
                       const double* __restrict__ gram_part, FitState* st,
                       FinalScratch* fs, double rel_tol, int max_evals,
                       double* history, int history_cap, const float* __restrict__ hmax_part) {
    pdl_wait();
    pdl_trigger();   // the next pass's CTAs may start their setup meanwhile
    if (st->done) return;
    if (st->kerr != 0) {   // the S-stream gave up waiting: stop the loop, no result this pass
        if (blockIdx.x == 0 && threadIdx.x == 0) st->done = 1;
        return;
    }
    __shared__ double sh[8][32];
    __shared__ bool last;
    const int kk = k * k;
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    const bool gram = mode != MODE_SNAPSHOT;
    const int gram_blocks = gram ? (kk + 31) / 32 : 0;

    if ((int)blockIdx.x < gram_blocks) {
        const int e = blockIdx.x * 32 + l;
        double a0 = 0.0, a1 = 0.0;
        if (e < kk) {
            int b = w;
            for (; b + 8 < nblk; b += 16) {
                a0 += gram_part[(int64_t)b * kk + e];
                a1 += gram_part[(int64_t)(b + 8) * kk + e];
            }
            if (b < nblk) a0 += gram_part[(int64_t)b * kk + e];
        }
        sh[w][l] = a0 + a1;
        __syncthreads();
        if (w == 0 && e < kk) {
            double t = 0.0;
#pragma unroll
            for (int q = 0; q < 8; ++q) t += sh[q][l];
            fs->A_next[e] = t;
        }
    } else {
        // trace block
        double a = 0.0;
        for (int b = threadIdx.x; b < nblk; b += RF_THREADS) a += tr_part[b];
        sh[w][l] = a;
        __syncthreads();
        if (threadIdx.x == 0) {
            double t = 0.0;
            for (int q = 0; q < 8; ++q)
                for (int r = 0; r < 32; ++r) t += sh[q][r];
            fs->tr = t;
        }
    }
    // last-arriving block does the scalar work (no waiting on other blocks)
    __threadfence();
    __syncthreads();
    if (threadIdx.x == 0) {
        const unsigned int prev = atomicAdd(&fs->arrived, 1u);
        last = prev == gridDim.x - 1;
    }
    __syncthreads();
    if (!last) return;
    __threadfence();

    if (threadIdx.x == 0) {
        finalize_scalar(mode, st, __ldcg(&fs->tr), rel_tol, max_evals, history, history_cap);
        fs->arrived = 0u;
    }
    __syncthreads();
    if (gram && !st->done) {
        double q = 0.0;
        for (int e = threadIdx.x; e < kk; e += RF_THREADS) {
            const double v = __ldcg(&fs->A_next[e]);
            st->A64[e] = v;
            st->A32[e] = (float)v;
            q = fma(v, v, q);
        }
        // ||A||^2 for the next evaluation, fixed-order block sum
        __shared__ double qs[RF_THREADS];
        qs[threadIdx.x] = q;
        __syncthreads();
        for (int o = RF_THREADS / 2; o > 0; o >>= 1) {
            if ((int)threadIdx.x < o) qs[threadIdx.x] += qs[threadIdx.x + o];
            __syncthreads();
        }
        if (threadIdx.x == 0) st->a_sqnorm = qs[0];
        // the next iterate's operand scale: max |H_{t+1}| over the tiles (exact in any order)
        if (hmax_part != nullptr) {
            __shared__ float mw[RF_THREADS / 32];
            float m = 0.f;
            for (int b = threadIdx.x; b < nblk; b += RF_THREADS) m = fmaxf(m, __ldcg(&hmax_part[b]));
#pragma unroll
            for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
            if ((threadIdx.x & 31) == 0) mw[threadIdx.x >> 5] = m;
            __syncthreads();
            if (threadIdx.x == 0) {
                float mm = 0.f;
                for (int w = 0; w < RF_THREADS / 32; ++w) mm = fmaxf(mm, mw[w]);
                st->xscale = pow2_scale_below_2_14((double)mm);
            }
        }
    }
}

int launch_finalize(int mode, int nblk, int k, const double* tr_part,
                    const double* gram_part, FitState* st, double rel_tol,
                    int max_evals, double* history, int history_cap,
                    cudaStream_t s, const float* hmax_part) {
    // FinalScratch lives right after the FitState (see fit planning).
    FinalScratch* fs = reinterpret_cast<FinalScratch*>(
        reinterpret_cast<char*>(st) + ((sizeof(FitState) + 255) & ~size_t(255)));
    const int kk = k * k;
    const int gram_blocks = mode != MODE_SNAPSHOT ? (kk + 31) / 32 : 0;
    const int grid = gram_blocks + 1;
    SYMNMF_CUDA_TRY(launch_pdl(reduce_finalize_kernel, dim3(grid), dim3(RF_THREADS), 0, s, mode, nblk, k,
                               tr_part, gram_part, st, fs, rel_tol, max_evals, history,
                               history_cap, hmax_part));
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

size_t fit_state_bytes() {
    return ((sizeof(FitState) + 255) & ~size_t(255)) + sizeof(FinalScratch);
}

}  // namespace symnmf
