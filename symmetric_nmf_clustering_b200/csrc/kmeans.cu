// Kernels of the spherical k-means baseline ([CaS] "Spherical k-means for
// direct hard clustering": k-means with cosine similarity on the L2-normalised
// rows of S).  Both S-sized steps of an iteration are S-stream passes (see the
// driver in api.cu); these kernels are the O(n k) pieces around them.
#include "common.cuh"

namespace symnmf {

constexpr int KM_THREADS = 256;

// inv_norm[i] = 1 / ||S_i||_2 (0 for a zero row), fp64, fixed reduction order.
__global__ void __launch_bounds__(KM_THREADS)
rownorm_kernel(const float* __restrict__ S, int64_t n, int64_t lds, double* __restrict__ inv_norm) {
    __shared__ double red[KM_THREADS];
    for (int64_t r = blockIdx.x; r < n; r += gridDim.x) {
        const float* row = S + r * lds;
        double a0 = 0.0, a1 = 0.0;
        int64_t j = threadIdx.x;
        for (; j + KM_THREADS < n; j += 2 * KM_THREADS) {
            const double x0 = row[j], x1 = row[j + KM_THREADS];
            a0 = fma(x0, x0, a0);
            a1 = fma(x1, x1, a1);
        }
        if (j < n) a0 = fma((double)row[j], (double)row[j], a0);
        red[threadIdx.x] = a0 + a1;
        __syncthreads();
        for (int o = KM_THREADS / 2; o > 0; o >>= 1) {
            if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
            __syncthreads();
        }
        if (threadIdx.x == 0) inv_norm[r] = red[0] > 0.0 ? 1.0 / sqrt(red[0]) : 0.0;
        __syncthreads();
    }
}

// CT[j][c] = S[idx_c][j] / ||S_idx_c|| : the initial centroids as columns.
__global__ void init_centroids_kernel(const float* __restrict__ S, int64_t n, int64_t lds, int k,
                                      const int64_t* __restrict__ idx,
                                      const double* __restrict__ inv_norm, float* __restrict__ CT) {
    const int64_t total = n * k;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t j = e / k;
        const int c = (int)(e % k);
        const int64_t r = idx[c];
        CT[e] = (float)((double)S[r * lds + j] * inv_norm[r]);
    }
}

// X[i][c] = [label_i == c] / ||S_i||: S X sums the normalised member rows.
__global__ void member_kernel(const int32_t* __restrict__ lab, const double* __restrict__ inv_norm,
                              int64_t n, int k, float* __restrict__ X) {
    const int64_t total = n * k;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / k;
        const int c = (int)(e % k);
        X[e] = lab[i] == c ? (float)inv_norm[i] : 0.f;
    }
}

// part[b][c] = sum over the rows of block b of Z[j][c]^2 (fp64)
constexpr int KM_ROWS = 512;
__global__ void colsq_kernel(const float* __restrict__ Z, int64_t n, int k, double* __restrict__ part) {
    extern __shared__ double csq[];  // [KM_THREADS / k groups][k] handled by thread c + g*k
    const int64_t r0 = (int64_t)blockIdx.x * KM_ROWS;
    const int64_t r1 = min64(n, r0 + KM_ROWS);
    const int groups = KM_THREADS / k;
    const int c = threadIdx.x % k, g = threadIdx.x / k;
    double a = 0.0;
    if (g < groups)
        for (int64_t r = r0 + g; r < r1; r += groups) {
            const double z = Z[r * k + c];
            a = fma(z, z, a);
        }
    csq[threadIdx.x] = g < groups ? a : 0.0;
    __syncthreads();
    if (threadIdx.x < k) {
        double t = 0.0;
        for (int q = 0; q < groups; ++q) t += csq[q * k + threadIdx.x];
        part[(int64_t)blockIdx.x * k + threadIdx.x] = t;
    }
}

// CT[j][c] = Z[j][c] / ||Z[:, c]|| (a column with zero norm keeps its centroid)
__global__ void normalize_centroids_kernel(const float* __restrict__ Z, int64_t n, int k,
                                           const double* __restrict__ part, int nblk,
                                           float* __restrict__ CT) {
    __shared__ double inv[64];
    if (threadIdx.x < k) {
        double t = 0.0;
        for (int b = 0; b < nblk; ++b) t += part[(int64_t)b * k + threadIdx.x];
        inv[threadIdx.x] = t > 0.0 ? 1.0 / sqrt(t) : -1.0;
    }
    __syncthreads();
    const int64_t total = n * k;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total;
         e += (int64_t)gridDim.x * blockDim.x) {
        const int c = (int)(e % k);
        if (inv[c] > 0.0) CT[e] = (float)((double)Z[e] * inv[c]);
    }
}

// count[0] += #{i : lab[i] != old[i]}; old <- lab
__global__ void label_change_kernel(const int32_t* __restrict__ lab, int32_t* __restrict__ old,
                                    int64_t n, int* __restrict__ count) {
    int local = 0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        local += lab[i] != old[i];
        old[i] = lab[i];
    }
    for (int o = 16; o > 0; o >>= 1) local += __shfl_down_sync(0xffffffffu, local, o);
    if ((threadIdx.x & 31) == 0 && local) atomicAdd(count, local);
}

static unsigned blocks_for(int64_t total) {
    return (unsigned)std::min<int64_t>((total + KM_THREADS - 1) / KM_THREADS, 8192);
}

int km_colsq_blocks(int64_t n) { return (int)((n + KM_ROWS - 1) / KM_ROWS); }

int launch_rownorm(const float* S, int64_t n, int64_t lds, double* inv_norm, cudaStream_t s) {
    rownorm_kernel<<<(unsigned)std::min<int64_t>(n, 4096), KM_THREADS, 0, s>>>(S, n, lds, inv_norm);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_init_centroids(const float* S, int64_t n, int64_t lds, int k, const int64_t* idx,
                          const double* inv_norm, float* CT, cudaStream_t s) {
    init_centroids_kernel<<<blocks_for(n * k), KM_THREADS, 0, s>>>(S, n, lds, k, idx, inv_norm, CT);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_member(const int32_t* lab, const double* inv_norm, int64_t n, int k, float* X,
                  cudaStream_t s) {
    member_kernel<<<blocks_for(n * k), KM_THREADS, 0, s>>>(lab, inv_norm, n, k, X);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_normalize_centroids(const float* Z, int64_t n, int k, double* part, float* CT,
                               cudaStream_t s) {
    const int nblk = km_colsq_blocks(n);
    colsq_kernel<<<nblk, KM_THREADS, KM_THREADS * sizeof(double), s>>>(Z, n, k, part);
    SYMNMF_LAUNCH_CHECK();
    normalize_centroids_kernel<<<blocks_for(n * k), KM_THREADS, 0, s>>>(Z, n, k, part, nblk, CT);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

int launch_label_change(const int32_t* lab, int32_t* old, int64_t n, int* count, cudaStream_t s) {
    label_change_kernel<<<blocks_for(n), KM_THREADS, 0, s>>>(lab, old, n, count);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

}  // namespace symnmf
