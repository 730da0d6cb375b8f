// Dependence-matrix builders from a T x n returns window ([CaS] "Tracking
// stability through time with the Rand index": |Pearson correlation| for the
// body of the distribution, TPDM for co-movement in the tails).
//
// Both end in a symmetric Gram S = c * op(Z^T Z) over the day index, computed
// by one tiled kernel with the builder's epilogue (abs + unit diagonal for
// correlation, the n/N scale for TPDM).
#include <cuda_fp16.h>

#include <cstdlib>
#include <cstring>

#include "common.cuh"

namespace symnmf {

// Tensor-core Gram by default; SYMNMF_STREAM=cuda_core selects the CUDA-core one.
static bool builders_tc() {
    static const bool v = [] {   // read once (thread-safe static initialisation)
        const char* e = getenv("SYMNMF_STREAM");
        return !(e != nullptr && std::strcmp(e, "cuda_core") == 0);
    }();
    return v;
}
constexpr int TCB_ROWS = 128;   // row padding of the transposed operands
constexpr int TCB_K = 32;       // contraction padding of the transposed fp32 operands (TPDM)
constexpr int TCB_K16 = 64;     // contraction padding of the transposed fp16 operands (|corr|)

constexpr int GB = 128;   // Gram output tile (GB x GB)
constexpr int GK = 16;    // day-slab per stage
constexpr int GT = 256;   // threads, 8 x 8 outputs each

enum GramMode { GRAM_CORR = 0, GRAM_TPDM = 1 };

static int64_t round_up(int64_t a, int64_t b) { return (a + b - 1) / b * b; }

// S[i][j] = epi(sum_t Z[t][i] Z[t][j]) for the tile (blockIdx.y, blockIdx.x).
// Z is Kp x ldz (Kp multiple of GK, ldz multiple of GB, zero padded).
__global__ void __launch_bounds__(GT)
gram_kernel(const float* __restrict__ Z, int64_t ldz, int Kp, int64_t n,
            float* __restrict__ S, int64_t lds, int mode, float scale) {
    __shared__ __align__(16) float As[2][GK][GB];
    __shared__ __align__(16) float Bs[2][GK][GB];
    const int tid = threadIdx.x;
    const int64_t I0 = (int64_t)blockIdx.y * GB, J0 = (int64_t)blockIdx.x * GB;
    const int tx = tid % 16, ty = tid / 16;

    float acc[8][8];
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;

    // each thread moves 2 float4 of each operand per stage
    float4 ra[2], rb[2];
    auto load = [&](int k0) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int e = tid + q * GT;
            const int row = e / 32, c4 = e % 32;
            const float* base = Z + (int64_t)(k0 + row) * ldz;
            ra[q] = *reinterpret_cast<const float4*>(base + I0 + c4 * 4);
            rb[q] = *reinterpret_cast<const float4*>(base + J0 + c4 * 4);
        }
    };
    auto store = [&](int buf) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
            const int e = tid + q * GT;
            const int row = e / 32, c4 = e % 32;
            *reinterpret_cast<float4*>(&As[buf][row][c4 * 4]) = ra[q];
            *reinterpret_cast<float4*>(&Bs[buf][row][c4 * 4]) = rb[q];
        }
    };

    load(0);
    store(0);
    __syncthreads();
    int buf = 0;
    for (int k0 = 0; k0 < Kp; k0 += GK) {
        const bool more = k0 + GK < Kp;
        if (more) load(k0 + GK);
#pragma unroll
        for (int kk = 0; kk < GK; ++kk) {
            const float4 a0 = *reinterpret_cast<const float4*>(&As[buf][kk][ty * 4]);
            const float4 a1 = *reinterpret_cast<const float4*>(&As[buf][kk][64 + ty * 4]);
            const float4 b0 = *reinterpret_cast<const float4*>(&Bs[buf][kk][tx * 4]);
            const float4 b1 = *reinterpret_cast<const float4*>(&Bs[buf][kk][64 + tx * 4]);
            const float a[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
            const float b[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
            for (int r = 0; r < 8; ++r)
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(a[r], b[c], acc[r][c]);
        }
        if (more) {
            store(buf ^ 1);
            __syncthreads();
            buf ^= 1;
        }
    }

#pragma unroll
    for (int r = 0; r < 8; ++r) {
        const int64_t i = I0 + (r < 4 ? ty * 4 + r : 64 + ty * 4 + (r - 4));
        if (i >= n) continue;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
            const int64_t j = J0 + h * 64 + tx * 4;
            float v[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                float x = acc[r][h * 4 + u];
                if (mode == GRAM_CORR) {
                    x = fabsf(x);
                    if (i == j + u) x = 1.f;
                } else {
                    x *= scale;
                }
                v[u] = x;
            }
            float* dst = S + i * lds + j;
            if (j + 3 < n) {
                *reinterpret_cast<float4*>(dst) = make_float4(v[0], v[1], v[2], v[3]);
            } else {
                for (int u = 0; u < 4; ++u)
                    if (j + u < n) dst[u] = v[u];
            }
        }
    }
}

static int launch_gram(const float* Z, int64_t ldz, int Kp, int64_t n, float* S, int64_t lds,
                       int mode, float scale, cudaStream_t s) {
    const int64_t tiles = (n + GB - 1) / GB;
    if (tiles > 65535) {
        set_error("n = %lld too large for the Gram tile grid", (long long)n);
        return SYMNMF_ERR_INVALID_ARG;
    }
    dim3 grid((unsigned)tiles, (unsigned)tiles);
    gram_kernel<<<grid, GT, 0, s>>>(Z, ldz, Kp, n, S, lds, mode, scale);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// |Pearson correlation|
// ----------------------------------------------------------------------------
int corr_plan(Arena& a, int64_t T, int64_t n, double** mu, double** inv, float** Z,
              int64_t* ldz) {
    *ldz = round_up(n, GB);
    const int64_t Kp = round_up(T, GK);
    *mu = a.take<double>(n);
    *inv = a.take<double>(n);
    // CUDA-core layout: Z (Kp x ldz) floats; tensor-core layout: two fp16 Z^T
    // planes (n_pad x Kt) + err, counted in floats
    const size_t cc = (size_t)Kp * *ldz;
    const size_t tc = (size_t)round_up(n, TCB_ROWS) * round_up(T, TCB_K16) + 64;
    *Z = a.take<float>(std::max(cc, tc));
    return SYMNMF_OK;
}

// Column means and inverse norms of the centred columns, fp64 two-pass.
__global__ void colstats_kernel(const float* __restrict__ R, int64_t T, int64_t n,
                                int64_t ldr, double* __restrict__ mu,
                                double* __restrict__ inv) {
    const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    double s = 0.0;
    for (int64_t t = 0; t < T; ++t) s += (double)R[t * ldr + i];
    const double m = s / (double)T;
    double ss = 0.0;
    for (int64_t t = 0; t < T; ++t) {
        const double d = (double)R[t * ldr + i] - m;
        ss = fma(d, d, ss);
    }
    mu[i] = m;
    inv[i] = ss > 0.0 ? 1.0 / sqrt(ss) : 0.0;   // zero-variance column -> zero row of Z
}

// Z[t][i] = (R[t][i] - mu_i) / ||R_i - mu_i||, zero in the padding.
__global__ void normalize_kernel(const float* __restrict__ R, int64_t T, int64_t n,
                                 int64_t ldr, const double* __restrict__ mu,
                                 const double* __restrict__ inv, float* __restrict__ Z,
                                 int64_t ldz, int64_t Kp) {
    const int64_t total = Kp * ldz;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t t = e / ldz, i = e % ldz;
        float z = 0.f;
        if (t < T && i < n) z = (float)(((double)R[t * ldr + i] - mu[i]) * inv[i]);
        Z[e] = z;
    }
}

// Z^T planes for the tensor-core Gram, in fp16 and scaled by c = CORR_F16_SCALE:
// ZH[i][t] = rn16(c z_ti) and ZL[i][t] = rn16(c z_ti - ZH[i][t]), zero in the
// padding (i >= n, t >= T).  |c z| <= 2^14, so neither part overflows; the pair
// carries c z to within 2^-22 of its magnitude (each rounding to nearest loses
// at most 2^-11 of what it rounds, and the remainder is at most 2^-11 c |z|).
// 32 x 32 tiles through shared memory: coalesced reads of R rows, writes of ZT rows.
__global__ void normalize_t_kernel(const float* __restrict__ R, int64_t T, int64_t n,
                                   int64_t ldr, const double* __restrict__ mu,
                                   const double* __restrict__ inv, __half* __restrict__ ZH,
                                   __half* __restrict__ ZL, int64_t Kt) {
    __shared__ float tile[32][33];
    const int64_t t0 = (int64_t)blockIdx.y * 32, i0 = (int64_t)blockIdx.x * 32;
    const int tx = threadIdx.x, ty = threadIdx.y;     // 32 x 8
    for (int r = ty; r < 32; r += 8) {
        const int64_t t = t0 + r, i = i0 + tx;
        float z = 0.f;
        if (t < T && i < n) z = (float)(((double)R[t * ldr + i] - mu[i]) * inv[i]);
        tile[r][tx] = z;
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {
        const int64_t i = i0 + r, t = t0 + tx;
        const float zs = tile[tx][r] * CORR_F16_SCALE;     // exact: a power of two
        const __half hi = __float2half_rn(zs);
        ZH[i * Kt + t] = hi;
        ZL[i * Kt + t] = __float2half_rn(zs - __half2float(hi));   // the difference is exact in fp32
    }
}

// The tensor-core Gram reports a bounded device-side wait that gave up in its
// error word; read it (this synchronises the stream).
static int gram_status(const int* err, cudaStream_t s) {
    int h = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&h, err, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (h != 0) {
        set_error("a builder pipeline wait timed out on the device (code %d)", h);
        return SYMNMF_ERR_TIMEOUT;
    }
    return SYMNMF_OK;
}

int launch_corr(const float* R, int64_t T, int64_t n, int64_t ldr, float* S,
                int64_t lds, double* mu, double* inv, float* Z, int64_t ldz,
                cudaStream_t s) {
    colstats_kernel<<<(unsigned)((n + 255) / 256), 256, 0, s>>>(R, T, n, ldr, mu, inv);
    SYMNMF_LAUNCH_CHECK();
    if (builders_tc()) {
        const int64_t n_pad = round_up(n, TCB_ROWS), Kt = round_up(T, TCB_K16);
        __half* ZH = reinterpret_cast<__half*>(Z);
        __half* ZL = ZH + (size_t)n_pad * Kt;
        int* err = reinterpret_cast<int*>(ZL + (size_t)n_pad * Kt);
        SYMNMF_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), s));
        dim3 grid((unsigned)(n_pad / 32), (unsigned)(Kt / 32));
        normalize_t_kernel<<<grid, dim3(32, 8), 0, s>>>(R, T, n, ldr, mu, inv, ZH, ZL, Kt);
        SYMNMF_LAUNCH_CHECK();
        SYMNMF_TRY(launch_gram_tc(ZH, ZL, n, n_pad, Kt, true, 1.f, S, lds, err, s));
        return gram_status(err, s);
    }
    const int64_t Kp = round_up(T, GK);
    const int64_t total = Kp * ldz;
    const int64_t blocks = min64((total + 255) / 256, 8192);
    normalize_kernel<<<(unsigned)blocks, 256, 0, s>>>(R, T, n, ldr, mu, inv, Z, ldz, Kp);
    SYMNMF_LAUNCH_CHECK();
    return launch_gram(Z, ldz, (int)Kp, n, S, lds, GRAM_CORR, 1.f, s);
}

// ----------------------------------------------------------------------------
// TPDM
// ----------------------------------------------------------------------------
int tpdm_plan(Arena& a, int64_t T, int64_t n, int N, int32_t** ranks, double** phi,
              double** rho, int32_t** days, float** W, int64_t* ldw) {
    *ldw = round_up(n, GB);
    *ranks = a.take<int32_t>((size_t)T * n);
    *phi = a.take<double>((size_t)T + 1);
    *rho = a.take<double>((size_t)T);
    *days = a.take<int32_t>((size_t)N);
    const size_t cc = (size_t)round_up(N, GK) * *ldw;
    const size_t tc = 2 * (size_t)round_up(n, TCB_ROWS) * round_up(N, TCB_K) + 64;
    *W = a.take<float>(std::max(cc, tc));
    return SYMNMF_OK;
}

constexpr int RK_COLS = 32;                       // columns per block (one per lane)
constexpr int RK_THREADS = 256;
constexpr int64_t RK_SMEM_MAX = 200 * 1024;       // stage the columns in smem up to this

// r_ti = 1 + #{s : x_s < x_t} + #{s < t : x_s == x_t}, x = tail_sign * R[:, i]
template <bool SMEM>
__global__ void __launch_bounds__(RK_THREADS)
rank_kernel(const float* __restrict__ R, int64_t T, int64_t n, int64_t ldr, float sign,
            int32_t* __restrict__ ranks) {
    extern __shared__ float xs[];  // [T][32] when SMEM
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    const int64_t i = (int64_t)blockIdx.x * RK_COLS + lane;
    const bool valid = i < n;
    const int64_t ic = valid ? i : 0;
    if (SMEM) {
        for (int64_t t = w; t < T; t += RK_THREADS / 32)
            xs[t * RK_COLS + lane] = valid ? sign * R[t * ldr + ic] : 0.f;
        __syncthreads();
    }
    auto val = [&](int64_t t) -> float {
        return SMEM ? xs[t * RK_COLS + lane] : sign * __ldg(R + t * ldr + ic);
    };
    for (int64_t base = (int64_t)w * 4; base < T; base += 4 * (RK_THREADS / 32)) {
        float x[4];
        int cnt[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            x[q] = base + q < T ? val(base + q) : 0.f;
            cnt[q] = 0;
        }
        for (int64_t s2 = 0; s2 < T; ++s2) {
            const float v = val(s2);
#pragma unroll
            for (int q = 0; q < 4; ++q)
                cnt[q] += (v < x[q]) | ((v == x[q]) & (s2 < base + q));
        }
        if (valid) {
#pragma unroll
            for (int q = 0; q < 4; ++q)
                if (base + q < T) ranks[(base + q) * n + i] = cnt[q] + 1;
        }
    }
}

// The same ranks by sorting: the rank of x_t is its 1-based position when the
// column is ordered by the key (x_t, t), which breaks ties towards the earlier
// day exactly as the count above does.  Eight columns per block (one 32-byte
// sector per day on load and store), a bitonic sort of each column's P = 2^m
// >= T keys in shared memory (padding keys (+inf, t >= T) sort last), then the
// positions are scattered into a day-major tile and written out.
constexpr int RS_COLS = 8;
constexpr int RS_THREADS = 1024;
constexpr int RS_PER_COL = RS_THREADS / RS_COLS;
constexpr int64_t RS_MAX_P = 2048;

__device__ __forceinline__ bool rs_before(float va, int ta, float vb, int tb) {
    return va < vb || (va == vb && ta < tb);
}

__global__ void __launch_bounds__(RS_THREADS)
rank_sort_kernel(const float* __restrict__ R, int64_t T, int64_t n, int64_t ldr, float sign,
                 int P, int32_t* __restrict__ ranks) {
    extern __shared__ uint8_t rs_smem[];
    float* kv = reinterpret_cast<float*>(rs_smem);                 // [RS_COLS][P] values
    int* kt = reinterpret_cast<int*>(kv + (size_t)RS_COLS * P);     // [RS_COLS][P] days
    int* rt = kt + (size_t)RS_COLS * P;                             // [T][RS_COLS] ranks
    const int tid = threadIdx.x;
    const int64_t i0 = (int64_t)blockIdx.x * RS_COLS;
    const int cols = (int)min64(RS_COLS, n - i0);

    for (int e = tid; e < RS_COLS * P; e += RS_THREADS) {
        const int t = e / RS_COLS, c = e % RS_COLS;
        float v = __int_as_float(0x7f800000);                       // +inf
        if (t < T && c < cols) v = sign * R[(int64_t)t * ldr + i0 + c];
        kv[c * P + t] = v;
        kt[c * P + t] = t;
    }
    __syncthreads();

    const int c = tid / RS_PER_COL, lt = tid % RS_PER_COL;
    float* v = kv + c * P;
    int* tt = kt + c * P;
    for (int k = 2; k <= P; k <<= 1) {
        for (int j = k >> 1; j > 0; j >>= 1) {
            for (int q = lt; q < (P >> 1); q += RS_PER_COL) {
                const int a = (q / j) * 2 * j + (q % j), b = a + j;
                const bool up = (a & k) == 0;
                const float va = v[a], vb = v[b];
                const int ta = tt[a], tb = tt[b];
                if (rs_before(vb, tb, va, ta) == up) {   // out of order for this direction
                    v[a] = vb;
                    v[b] = va;
                    tt[a] = tb;
                    tt[b] = ta;
                }
            }
            __syncthreads();
        }
    }

    for (int p = lt; p < T; p += RS_PER_COL) rt[tt[p] * RS_COLS + c] = p + 1;
    __syncthreads();
    for (int e = tid; e < T * RS_COLS; e += RS_THREADS) {
        const int t = e / RS_COLS, cc = e % RS_COLS;
        if (cc < cols) ranks[(int64_t)t * n + i0 + cc] = rt[e];
    }
}

// The same ranks with the sort held in registers: one warp per column and
// RPL = P / 32 keys per lane, P = 2^m >= max(T, 32) <= 1024.  A key packs the
// day under an order-preserving image of the value (the float's bits, with
// -0 folded onto +0 so that the two stay a tie), so one unsigned 64-bit
// comparison orders by (x_t, t).  Key slot e = lane * RPL + r: bitonic steps
// of span < RPL swap registers inside a lane, wider ones trade with the lane
// at distance span / RPL by shuffle.  The keys enter in any order (each
// carries its day), so the load reads day r * 32 + lane from a day-major tile
// of the block's columns without bank conflicts; positions leave through
// the same tile.  Padding keys are all ones and sort last.
constexpr int RW_COLS = 8;                  // columns per block, one per warp
constexpr int RW_THREADS = 32 * RW_COLS;
constexpr int RW_LD = RW_COLS + 1;          // tile row stride (odd: no bank conflicts)
constexpr int64_t RW_MAX_P = 1024;

__device__ __forceinline__ uint64_t rw_key(float x, int t) {
    uint32_t u = __float_as_uint(x);
    if ((u & 0x7fffffffu) == 0u) u = 0u;                   // -0 -> +0
    u = (u & 0x80000000u) ? ~u : (u | 0x80000000u);        // monotone in x
    return ((uint64_t)u << 32) | (uint32_t)t;
}

template <int RPL>
__device__ __forceinline__ void rw_bitonic(uint64_t (&key)[RPL], int lane) {
#pragma unroll
    for (int k = 2; k <= 32 * RPL; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            if (j >= RPL) {
                // partner slot e ^ j lives in lane ^ (j / RPL), same register
                const int lm = j / RPL;
                const bool up = ((lane * RPL) & k) == 0;
                const bool keep_min = ((lane & lm) == 0) == up;
#pragma unroll
                for (int r = 0; r < RPL; ++r) {
                    const uint64_t o = __shfl_xor_sync(0xffffffffu, key[r], lm);
                    key[r] = ((o < key[r]) == keep_min) ? o : key[r];
                }
            } else {
#pragma unroll
                for (int r = 0; r < RPL; ++r) {
                    if (r & j) continue;
                    const bool up = ((lane * RPL + r) & k) == 0;
                    const uint64_t a = key[r], b = key[r + j];
                    const bool sw = (b < a) == up;
                    key[r] = sw ? b : a;
                    key[r + j] = sw ? a : b;
                }
            }
        }
    }
}

template <int RPL>
__global__ void __launch_bounds__(RW_THREADS)
rank_warp_kernel(const float* __restrict__ R, int64_t T, int64_t n, int64_t ldr, float sign,
                 int32_t* __restrict__ ranks) {
    __shared__ uint32_t tile[RW_MAX_P * RW_LD];             // [day][column]
    const int tid = threadIdx.x, lane = tid & 31, c = tid >> 5;
    const int64_t i0 = (int64_t)blockIdx.x * RW_COLS;
    const int cols = (int)min64(RW_COLS, n - i0);
    const int Ti = (int)T;

    for (int e = tid; e < Ti * RW_COLS; e += RW_THREADS) {
        const int t = e / RW_COLS, cc = e % RW_COLS;
        const float x = cc < cols ? sign * R[(int64_t)t * ldr + i0 + cc] : 0.f;
        tile[t * RW_LD + cc] = __float_as_uint(x);
    }
    __syncthreads();

    uint64_t key[RPL];
#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        const int t = r * 32 + lane;
        key[r] = t < Ti ? rw_key(__uint_as_float(tile[t * RW_LD + c]), t) : ~0ull;
    }
    __syncthreads();                                        // the tile now takes ranks

    rw_bitonic<RPL>(key, lane);

#pragma unroll
    for (int r = 0; r < RPL; ++r) {
        const uint32_t t = (uint32_t)key[r];                // padding: 0xffffffff
        if (t < (uint32_t)Ti) tile[t * RW_LD + c] = (uint32_t)(lane * RPL + r + 1);
    }
    __syncthreads();
    for (int e = tid; e < Ti * RW_COLS; e += RW_THREADS) {
        const int t = e / RW_COLS, cc = e % RW_COLS;
        if (cc < cols) ranks[(int64_t)t * n + i0 + cc] = (int32_t)tile[t * RW_LD + cc];
    }
}

// phi[r] = (-ln(r / (T+1)))^(-1/2): Frechet (alpha = 2) margin of rank r, fp64.
__global__ void phi_kernel(double* __restrict__ phi, int64_t T) {
    const int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (r > T) return;
    phi[r] = r == 0 ? 0.0 : 1.0 / sqrt(-log((double)r / (double)(T + 1)));
}

// rho_t = sqrt(sum_i phi[r_ti]^2), one block per day, fixed reduction order.
__global__ void rho_kernel(const int32_t* __restrict__ ranks, const double* __restrict__ phi,
                           int64_t n, double* __restrict__ rho) {
    __shared__ double red[256];
    const int64_t t = blockIdx.x;
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < n; i += blockDim.x) {
        const double x = phi[ranks[t * n + i]];
        s = fma(x, x, s);
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int o = 128; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) rho[t] = sqrt(red[0]);
}

// days[p] = the day of position p when days are ordered by decreasing rho,
// ties to the earlier day; only positions p < N are written.
__global__ void select_kernel(const double* __restrict__ rho, int64_t T, int N,
                              int32_t* __restrict__ days) {
    const int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (t >= T) return;
    const double r = rho[t];
    int64_t pos = 0;
    for (int64_t s2 = 0; s2 < T; ++s2) {
        const double q = rho[s2];
        pos += (q > r) | ((q == r) & (s2 < t));
    }
    if (pos < N) days[pos] = (int32_t)t;
}

// W[p][i] = phi[r_{days[p], i}] / rho_{days[p]}; zero padding to Np x ldw.
__global__ void gather_w_kernel(const int32_t* __restrict__ ranks, const double* __restrict__ phi,
                                const double* __restrict__ rho, const int32_t* __restrict__ days,
                                int N, int64_t n, float* __restrict__ W, int64_t ldw,
                                int64_t Np) {
    const int64_t total = Np * ldw;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t p = e / ldw, i = e % ldw;
        float v = 0.f;
        if (p < N && i < n) {
            const int64_t t = days[p];
            v = (float)(phi[ranks[t * n + i]] / rho[t]);
        }
        W[e] = v;
    }
}

// W^T planes: WF[i][p] = phi[r_{days[p], i}] / rho_{days[p]} (fp32) and
// WL = WF - trunc_tf32(WF); zero padding to n_pad x Kt.
__global__ void gather_wt_kernel(const int32_t* __restrict__ ranks, const double* __restrict__ phi,
                                 const double* __restrict__ rho, const int32_t* __restrict__ days,
                                 int N, int64_t n, float* __restrict__ WF, float* __restrict__ WL,
                                 int64_t n_pad, int64_t Kt) {
    const int64_t total = n_pad * Kt;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / Kt, p = e % Kt;
        float v = 0.f;
        if (p < N && i < n) {
            const int64_t t = days[p];
            v = (float)(phi[ranks[t * n + i]] / rho[t]);
        }
        WF[e] = v;
        WL[e] = v - __uint_as_float(__float_as_uint(v) & 0xFFFFE000u);
    }
}

int launch_tpdm(const float* R, int64_t T, int64_t n, int64_t ldr, int N,
                int tail_sign, float* S, int64_t lds, int32_t* ranks, double* phi,
                double* rho, int32_t* days, float* W, int64_t ldw, cudaStream_t s) {
    const unsigned rblocks = (unsigned)((n + RK_COLS - 1) / RK_COLS);
    const int64_t smem = T * RK_COLS * (int64_t)sizeof(float);
    const float sign = tail_sign < 0 ? -1.f : 1.f;
    int P = 2;
    while (P < T) P <<= 1;
    if (P <= RW_MAX_P) {
        const unsigned wblocks = (unsigned)((n + RW_COLS - 1) / RW_COLS);
        switch (P <= 32 ? 1 : P / 32) {
            case 1: rank_warp_kernel<1><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
            case 2: rank_warp_kernel<2><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
            case 4: rank_warp_kernel<4><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
            case 8: rank_warp_kernel<8><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
            case 16: rank_warp_kernel<16><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
            default: rank_warp_kernel<32><<<wblocks, RW_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks); break;
        }
    } else if (P <= RS_MAX_P) {
        const size_t rs_smem = (size_t)RS_COLS * P * 8 + (size_t)T * RS_COLS * 4;
        // once per process (thread-safe static initialisation)
        static const cudaError_t rs_attr = cudaFuncSetAttribute(
            rank_sort_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)(RS_COLS * RS_MAX_P * 12));
        SYMNMF_CUDA_TRY(rs_attr);
        rank_sort_kernel<<<(unsigned)((n + RS_COLS - 1) / RS_COLS), RS_THREADS, rs_smem, s>>>(
            R, T, n, ldr, sign, P, ranks);
    } else if (smem <= RK_SMEM_MAX) {
        SYMNMF_CUDA_TRY(cudaFuncSetAttribute(rank_kernel<true>,
                                             cudaFuncAttributeMaxDynamicSharedMemorySize,
                                             (int)RK_SMEM_MAX));
        rank_kernel<true><<<rblocks, RK_THREADS, (size_t)smem, s>>>(R, T, n, ldr, sign, ranks);
    } else {
        rank_kernel<false><<<rblocks, RK_THREADS, 0, s>>>(R, T, n, ldr, sign, ranks);
    }
    SYMNMF_LAUNCH_CHECK();
    phi_kernel<<<(unsigned)((T + 1 + 255) / 256), 256, 0, s>>>(phi, T);
    SYMNMF_LAUNCH_CHECK();
    rho_kernel<<<(unsigned)T, 256, 0, s>>>(ranks, phi, n, rho);
    SYMNMF_LAUNCH_CHECK();
    select_kernel<<<(unsigned)((T + 255) / 256), 256, 0, s>>>(rho, T, N, days);
    SYMNMF_LAUNCH_CHECK();
    const float scale = (float)((double)n / (double)N);
    if (builders_tc()) {
        const int64_t n_pad = round_up(n, TCB_ROWS), Kt = round_up(N, TCB_K);
        float* WF = W;
        float* WL = W + (size_t)n_pad * Kt;
        int* err = reinterpret_cast<int*>(WL + (size_t)n_pad * Kt);
        SYMNMF_CUDA_TRY(cudaMemsetAsync(err, 0, sizeof(int), s));
        const int64_t total = n_pad * Kt;
        const int64_t blocks = min64((total + 255) / 256, 8192);
        gather_wt_kernel<<<(unsigned)blocks, 256, 0, s>>>(ranks, phi, rho, days, N, n, WF, WL, n_pad, Kt);
        SYMNMF_LAUNCH_CHECK();
        SYMNMF_TRY(launch_gram_tc(WF, WL, n, n_pad, Kt, false, scale, S, lds, err, s));
        return gram_status(err, s);
    }
    const int64_t Np = round_up(N, GK);
    const int64_t total = Np * ldw;
    const int64_t blocks = min64((total + 255) / 256, 8192);
    gather_w_kernel<<<(unsigned)blocks, 256, 0, s>>>(ranks, phi, rho, days, N, n, W, ldw, Np);
    SYMNMF_LAUNCH_CHECK();
    return launch_gram(W, ldw, (int)Np, n, S, lds, GRAM_TPDM, scale, s);
}

}  // namespace symnmf
