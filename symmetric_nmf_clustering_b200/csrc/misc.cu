// Statistics pre-pass, seeded initialisation, argmax labels and the small
// dense helpers of the spectral probe.
#include "common.cuh"

namespace symnmf {

// ----------------------------------------------------------------------------
// splitmix64 (Steele, Lea & Flood, OOPSLA 2014): output function of the
// generator whose state advances by the golden-ratio increment.
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t sm64_mix(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}
constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

// c-th output (c = 0, 1, ...) of the generator seeded with `seed`, as a
// 24-bit uniform in [0, 1): exact in fp32.
__device__ __forceinline__ float sm64_uniform(uint64_t seed, uint64_t c) {
    const uint64_t z = sm64_mix(seed + (c + 1ull) * kGamma);
    return (float)(z >> 40) * 0x1p-24f;
}

// ----------------------------------------------------------------------------
// Statistics pre-pass: sum, sum of squares (fp64) and non-finite count of S.
// ----------------------------------------------------------------------------
constexpr int STATS_BLOCKS = 1184;  // fixed grid: same partition on every device
constexpr int STATS_THREADS = 256;

int stats_blocks() { return STATS_BLOCKS; }

__global__ void __launch_bounds__(STATS_THREADS)
stats_partial_kernel(const float* __restrict__ S, int64_t rows, int64_t n, int64_t lds,
                     double* __restrict__ part, float* __restrict__ amax_part) {
    double sum = 0.0, sq = 0.0, bad = 0.0;
    float amax = 0.f;   // max |S| over the finite entries
    const int64_t n4 = n >> 2;
    for (int64_t r = blockIdx.x; r < rows; r += gridDim.x) {
        const float4* row = reinterpret_cast<const float4*>(S + r * lds);
        constexpr int U = 4;  // loads in flight per thread
        for (int64_t q0 = threadIdx.x; q0 < n4; q0 += (int64_t)U * blockDim.x) {
            float4 v[U];
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const int64_t q = q0 + (int64_t)u * blockDim.x;
                if (q < n4)
                    asm volatile("ld.global.nc.L1::no_allocate.v4.f32 {%0,%1,%2,%3}, [%4];"
                                 : "=f"(v[u].x), "=f"(v[u].y), "=f"(v[u].z), "=f"(v[u].w)
                                 : "l"(row + q));
                else
                    v[u] = make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int u = 0; u < U; ++u) {
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                // all four normal (false for zero, subnormal, inf and NaN)
                bool normal = true;
#pragma unroll
                for (int w = 0; w < 4; ++w)
                    normal &= (fabsf(e[w]) >= 0x1p-126f) & (fabsf(e[w]) <= 0x1.fffffep127f);
                if (normal) {
                    // widen to fp64 by moving the bit fields, exact for normal
                    // floats: the arithmetic shift puts the sign in bits 31..28
                    // and the exponent in 27..20, the mask clears bits 30..28
                    // and the add rebiases the exponent by 1023 - 127 = 896
                    // (no carry reaches bit 31); the conversion instruction's
                    // throughput, not HBM, limited this pass
#pragma unroll
                    for (int w = 0; w < 4; ++w) amax = fmaxf(amax, fabsf(e[w]));
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        const uint32_t b = __float_as_uint(e[w]);
                        const uint32_t hi = ((uint32_t)((int32_t)b >> 3) & 0x8FFFFFFFu) + 0x38000000u;
                        const double d = __hiloint2double((int)hi, (int)(b << 29));
                        sum += d;
                        sq = fma(d, d, sq);
                    }
                } else {
#pragma unroll
                    for (int w = 0; w < 4; ++w) {
                        if (isfinite(e[w])) {
                            const double d = e[w];
                            sum += d;
                            sq = fma(d, d, sq);
                            amax = fmaxf(amax, fabsf(e[w]));
                        } else {
                            bad += 1.0;
                        }
                    }
                }
            }
        }
        for (int64_t c = n4 * 4 + threadIdx.x; c < n; c += blockDim.x) {
            const float e = S[r * lds + c];
            if (isfinite(e)) {
                sum += (double)e;
                sq = fma((double)e, (double)e, sq);
                amax = fmaxf(amax, fabsf(e));
            } else {
                bad += 1.0;
            }
        }
    }
    __shared__ double red[3][STATS_THREADS];
    red[0][threadIdx.x] = sum;
    red[1][threadIdx.x] = sq;
    red[2][threadIdx.x] = bad;
    __syncthreads();
    for (int o = STATS_THREADS / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o)
            for (int q = 0; q < 3; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x < 3) part[blockIdx.x * 3 + threadIdx.x] = red[threadIdx.x][0];
    if (amax_part != nullptr) {
        // max is exact in any order
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
        __shared__ float wmax[STATS_THREADS / 32];
        if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = amax;
        __syncthreads();
        if (threadIdx.x == 0) {
            float m = 0.f;
            for (int w = 0; w < STATS_THREADS / 32; ++w) m = fmaxf(m, wmax[w]);
            amax_part[blockIdx.x] = m;
        }
    }
}

__global__ void stats_final_kernel(const double* __restrict__ part, int nblk,
                                   double* __restrict__ out3, const float* __restrict__ amax_part,
                                   FitState* st) {
    __shared__ double red[3][STATS_THREADS];
    double a[3] = {0.0, 0.0, 0.0};
    for (int b = threadIdx.x; b < nblk; b += blockDim.x)
        for (int q = 0; q < 3; ++q) a[q] += part[b * 3 + q];
    for (int q = 0; q < 3; ++q) red[q][threadIdx.x] = a[q];
    __syncthreads();
    for (int o = STATS_THREADS / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o)
            for (int q = 0; q < 3; ++q) red[q][threadIdx.x] += red[q][threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x < 3) out3[threadIdx.x] = red[threadIdx.x][0];
    if (amax_part != nullptr && st != nullptr) {
        // max over the blocks (exact in any order): strided, then across the block
        float m = 0.f;
        for (int b = threadIdx.x; b < nblk; b += blockDim.x) m = fmaxf(m, amax_part[b]);
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        __shared__ float wmax[STATS_THREADS / 32];
        if ((threadIdx.x & 31) == 0) wmax[threadIdx.x >> 5] = m;
        __syncthreads();
        if (threadIdx.x == 0) {
            float mm = 0.f;
            for (int w = 0; w < STATS_THREADS / 32; ++w) mm = fmaxf(mm, wmax[w]);
            st->s_absmax = mm;
            st->sscale = pow2_scale_below_2_14((double)mm);
        }
    }
}

int launch_stats(const float* S, int64_t rows, int64_t n, int64_t lds, double* part, int nblk,
                 double* out3, cudaStream_t s, float* amax_part, FitState* st) {
    stats_partial_kernel<<<nblk, STATS_THREADS, 0, s>>>(S, rows, n, lds, part, amax_part);
    SYMNMF_LAUNCH_CHECK();
    stats_final_kernel<<<1, STATS_THREADS, 0, s>>>(part, nblk, out3, amax_part, st);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// Scale-matched seeded init: H0_ij = fl32(u_ij * fl32(sqrt(mean(S)/k))),
// u_ij the (i*k + j)-th output of the splitmix64 counter stream of `seed`.
// ----------------------------------------------------------------------------
__global__ void init_kernel(float* __restrict__ H, int64_t count, int k, int64_t n,
                            uint64_t seed, const FitState* st) {
    // mean(S) = sum(S) / n^2 (diagonal included), c = fl32(sqrt(mean / k))
    const double mean = st->s_sum / ((double)n * (double)n);
    const float c = (float)sqrt(fmax(mean, 0.0) / (double)k);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count;
         e += (int64_t)gridDim.x * blockDim.x)
        H[e] = sm64_uniform(seed, (uint64_t)e) * c;
}

// Same draw with the sum of S given by the caller (a row-sharded fit gets it
// from an all-reduce of every shard's statistics).
__global__ void init_sum_kernel(float* __restrict__ H, int64_t count, int k, int64_t n,
                                uint64_t seed, double s_sum) {
    const double mean = s_sum / ((double)n * (double)n);
    const float c = (float)sqrt(fmax(mean, 0.0) / (double)k);
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count;
         e += (int64_t)gridDim.x * blockDim.x)
        H[e] = sm64_uniform(seed, (uint64_t)e) * c;
}

int launch_init_sum(float* H, int64_t n, int k, uint64_t seed, double s_sum, cudaStream_t s) {
    const int64_t count = n * k;
    const int threads = 256;
    const int64_t blocks = min64((count + threads - 1) / threads, 4096);
    init_sum_kernel<<<(unsigned)blocks, threads, 0, s>>>(H, count, k, n, seed, s_sum);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_init(float* H, int64_t n, int k, uint64_t seed, const FitState* st,
                cudaStream_t s) {
    const int64_t count = n * k;
    const int threads = 256;
    const int64_t blocks = min64((count + threads - 1) / threads, 4096);
    init_kernel<<<(unsigned)blocks, threads, 0, s>>>(H, count, k, n, seed, st);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// Labels: row-wise argmax, lowest index on ties.
// ----------------------------------------------------------------------------
__global__ void labels_kernel(const float* __restrict__ H, int64_t n, int k,
                              int32_t* __restrict__ labels) {
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float* h = H + i * k;
        float best = h[0];
        int arg = 0;
        for (int c = 1; c < k; ++c) {
            const float v = h[c];
            if (v > best) {
                best = v;
                arg = c;
            }
        }
        labels[i] = arg;
    }
}

int launch_labels(const float* H, int64_t n, int k, int32_t* labels, cudaStream_t s) {
    const int threads = 256;
    const int64_t blocks = min64((n + threads - 1) / threads, 65535);
    labels_kernel<<<(unsigned)blocks, threads, 0, s>>>(H, n, k, labels);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// ----------------------------------------------------------------------------
// Spectral-probe helpers (tall-skinny products, fp64 accumulation)
// ----------------------------------------------------------------------------
__global__ void uniform_fill_kernel(float* X, int64_t count, uint64_t seed, float offset) {
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < count;
         e += (int64_t)gridDim.x * blockDim.x)
        X[e] = sm64_uniform(seed, (uint64_t)e) + offset;
}

int launch_uniform_fill(float* X, int64_t count, uint64_t seed, float offset,
                        cudaStream_t s) {
    const int threads = 256;
    const int64_t blocks = min64((count + threads - 1) / threads, 4096);
    uniform_fill_kernel<<<(unsigned)blocks, threads, 0, s>>>(X, count, seed, offset);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

constexpr int TN_ROWS = 256;        // rows of V and W per block of the V^T W partials
constexpr int TN_PER_THREAD = 16;   // entries per thread: cv * cw <= 16 * 256
int gemm_tn_blocks(int64_t n) { return (int)min64((n + TN_ROWS - 1) / TN_ROWS, 1024); }

// part[b][a][c] = sum over the rows of block b of V[r][a] W[r][c]
__global__ void gemm_tn_partial_kernel(const float* __restrict__ V, int64_t n, int64_t ldv,
                                       int cv, const float* __restrict__ W, int64_t ldw,
                                       int cw, double* __restrict__ part) {
    extern __shared__ float tn_smem[];
    float* vs = tn_smem;                 // [32][cv]
    float* ws = tn_smem + 32 * cv;       // [32][cw]
    const int entries = cv * cw;
    double acc[TN_PER_THREAD];
    for (int q = 0; q < TN_PER_THREAD; ++q) acc[q] = 0.0;
    for (int64_t r0 = (int64_t)blockIdx.x * 32; r0 < n; r0 += (int64_t)gridDim.x * 32) {
        const int rows = (int)min64(32, n - r0);
        __syncthreads();
        for (int e = threadIdx.x; e < 32 * cv; e += blockDim.x) {
            const int r = e / cv, a = e % cv;
            vs[e] = r < rows ? V[(r0 + r) * ldv + a] : 0.f;
        }
        for (int e = threadIdx.x; e < 32 * cw; e += blockDim.x) {
            const int r = e / cw, c = e % cw;
            ws[e] = r < rows ? W[(r0 + r) * ldw + c] : 0.f;
        }
        __syncthreads();
        for (int q = 0; q < TN_PER_THREAD; ++q) {
            const int e = threadIdx.x + q * blockDim.x;
            if (e >= entries) break;
            const int a = e / cw, c = e % cw;
            double s = 0.0;
            for (int r = 0; r < rows; ++r) s += (double)vs[r * cv + a] * (double)ws[r * cw + c];
            acc[q] += s;
        }
    }
    for (int q = 0; q < TN_PER_THREAD; ++q) {
        const int e = threadIdx.x + q * blockDim.x;
        if (e < entries) part[(int64_t)blockIdx.x * entries + e] = acc[q];
    }
}

__global__ void gemm_tn_reduce_kernel(const double* __restrict__ part, int nblk, int entries,
                                      double* __restrict__ C) {
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e >= entries) return;
    double s = 0.0;
    for (int b = 0; b < nblk; ++b) s += part[(int64_t)b * entries + e];
    C[e] = s;
}

// C (cv x cw, fp64, device) = V^T W with V n x cv, W n x cw.  cv * cw <= 4096.
int launch_gemm_tn(const float* V, int64_t n, int64_t ldv, int cv, const float* W,
                   int64_t ldw, int cw, double* C, double* part, int nblk,
                   cudaStream_t s) {
    const size_t smem = (size_t)32 * (cv + cw) * sizeof(float);
    gemm_tn_partial_kernel<<<nblk, 256, smem, s>>>(V, n, ldv, cv, W, ldw, cw, part);
    SYMNMF_LAUNCH_CHECK();
    const int entries = cv * cw;
    gemm_tn_reduce_kernel<<<(entries + 255) / 256, 256, 0, s>>>(part, nblk, entries, C);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// W[r][c] -= sum_a V[r][a] C[a][c]   (C cv x cw fp32, device)
__global__ void gemm_nn_sub_kernel(float* __restrict__ W, int64_t n, int64_t ldw, int cw,
                                   const float* __restrict__ V, int64_t ldv, int cv,
                                   const float* __restrict__ C) {
    extern __shared__ float cs[];
    for (int e = threadIdx.x; e < cv * cw; e += blockDim.x) cs[e] = C[e];
    __syncthreads();
    const int64_t total = n * cw;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t r = e / cw;
        const int c = (int)(e % cw);
        const float* v = V + r * ldv;
        float s = 0.f;
        for (int a = 0; a < cv; ++a) s = fmaf(v[a], cs[a * cw + c], s);
        W[r * ldw + c] -= s;
    }
}

int launch_gemm_nn_sub(float* W, int64_t n, int64_t ldw, int cw, const float* V,
                       int64_t ldv, int cv, const float* C, cudaStream_t s) {
    const size_t smem = (size_t)cv * cw * sizeof(float);
    const int64_t total = n * cw;
    const int64_t blocks = min64((total + 255) / 256, 4096);
    gemm_nn_sub_kernel<<<(unsigned)blocks, 256, smem, s>>>(W, n, ldw, cw, V, ldv, cv, C);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

// W <- W M for a cw x cw matrix M (fp32, device), in place row by row.
__global__ void right_mul_kernel(float* __restrict__ W, int64_t n, int64_t ldw, int cw,
                                 const float* __restrict__ M) {
    extern __shared__ float ms[];
    for (int e = threadIdx.x; e < cw * cw; e += blockDim.x) ms[e] = M[e];
    __syncthreads();
    for (int64_t r = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; r < n;
         r += (int64_t)gridDim.x * blockDim.x) {
        float row[64];
        float* w = W + r * ldw;
        for (int a = 0; a < cw; ++a) row[a] = w[a];
        for (int c = 0; c < cw; ++c) {
            float s = 0.f;
            for (int a = 0; a < cw; ++a) s = fmaf(row[a], ms[a * cw + c], s);
            w[c] = s;
        }
    }
}

int launch_trsm_right(float* W, int64_t n, int64_t ldw, int cw, const float* M,
                      cudaStream_t s) {
    const size_t smem = (size_t)cw * cw * sizeof(float);
    const int64_t blocks = min64((n + 127) / 128, 4096);
    right_mul_kernel<<<(unsigned)blocks, 128, smem, s>>>(W, n, ldw, cw, M);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf
