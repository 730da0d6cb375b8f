// Per-rank pieces of the row-sharded fit.
//
// The pages scale the factorisation out by sharding S by rows across GPUs
// while every GPU keeps a replica of H; the S H products are formed locally
// and the ranks exchange O(n k) data per iteration ([CaS] "Factorization at
// scale", "Scale-out").  Here rank p holds the block of rows [r0, r0 + m) of
// S (all n columns) and the whole current iterate H_t.  One step on that
// rank is one pass over its rows with the fused epilogue of the full-batch
// fit restricted to its rows:
//     P = S[r0:r0+m, :] H_t                  (tensor-core S-stream)
//     tr_p = sum_{i in rows} H_t,i . P_i      (its part of tr(H^T S H))
//     g, G, H_{t+1} rows by the projected AdaGrad step with A = H_t^T H_t
//     Gram_p = sum_{i in rows} H_{t+1,i} H_{t+1,i}^T
// and returns (Gram_p, tr_p) in fp64.  The caller sums these over the ranks
// (an all-reduce of k^2 + 1 numbers), which gives the next Gram and the loss
// f(H_t) = ||S||^2 - 2 tr + ||A_t||^2, and gathers the new rows of H from
// every rank.  The collectives belong to the caller's communication library;
// nothing here waits on another rank.
#include <cstring>

#include "common.cuh"
#include "epilogue.cuh"

namespace symnmf {

// FitState fields the fused epilogue and the stream kernel read: the Gram of
// the current iterate (fp64 and its fp32 rounding), no stop, no error.
__global__ void shard_state_kernel(FitState* st, const double* __restrict__ A, int k) {
    for (int e = threadIdx.x; e < k * k; e += blockDim.x) {
        const double v = A[e];
        st->A64[e] = v;
        st->A32[e] = (float)v;
    }
    if (threadIdx.x == 0) {
        st->done = 0;
        st->kerr = 0;
    }
}

// out[e] = sum over tiles, in tile order, of gram_part[tile][e] (e < k^2);
// out[k^2] = sum of tr_part in tile order (when tr_part is given).
__global__ void shard_reduce_kernel(const double* __restrict__ tr_part,
                                    const double* __restrict__ gram_part, int tiles, int k,
                                    double* __restrict__ out) {
    const int kk = k * k;
    const int e = blockIdx.x * blockDim.x + threadIdx.x;
    if (e < kk) {
        double a = 0.0;
        for (int t = 0; t < tiles; ++t) a += gram_part[(int64_t)t * kk + e];
        out[e] = a;
    } else if (e == kk && tr_part != nullptr) {
        double a = 0.0;
        for (int t = 0; t < tiles; ++t) a += tr_part[t];
        out[kk] = a;
    }
}

static int launch_shard_reduce(const double* tr_part, const double* gram_part, int tiles, int k,
                               double* out, cudaStream_t s) {
    const int count = k * k + 1;
    shard_reduce_kernel<<<(count + 127) / 128, 128, 0, s>>>(tr_part, gram_part, tiles, k, out);
    SYMNMF_LAUNCH_CHECK();
    return SYMNMF_OK;
}

struct ShardLayout {
    FitState* st = nullptr;
    float* part = nullptr;
    float* XT = nullptr;
    int64_t ldxt = 0;
    int* counters = nullptr;
    double* tr_part = nullptr;
    double* gram_part = nullptr;
};

static void shard_plan(const Dev& d, Arena& a, int64_t rows, int64_t n, int k, ShardLayout* L) {
    const TcPlan p = plan_stream_tc_rows(d, rows, n, k);
    const int64_t tiles = epilogue_blocks(rows);
    L->st = reinterpret_cast<FitState*>(a.take<char>(fit_state_bytes()));
    L->part = a.take<float>(tc_partial_floats(p));
    L->ldxt = xt_ld(n);
    L->XT = a.take<float>((size_t)xt_rows(k) * L->ldxt);
    L->counters = a.take<int>((size_t)tiles);
    L->tr_part = a.take<double>((size_t)tiles);
    L->gram_part = a.take<double>((size_t)tiles * k * k);
}

static bool mul_fits(int64_t a, int64_t b) {
    return a >= 0 && b >= 0 && (a == 0 || b <= (int64_t(1) << 62) / a);
}

}  // namespace symnmf

using namespace symnmf;

#define SHARD_CHECK(cond, ...)                  \
    do {                                        \
        if (!(cond)) {                          \
            set_error(__VA_ARGS__);             \
            return SYMNMF_ERR_INVALID_ARG;      \
        }                                       \
    } while (0)

static int check_rows(const float* S, int64_t rows, int64_t n, int64_t lds) {
    SHARD_CHECK(n >= 1 && rows >= 1 && rows <= n, "need 1 <= rows <= n (rows = %lld, n = %lld)",
                (long long)rows, (long long)n);
    SHARD_CHECK(lds >= n && lds % 4 == 0, "lds = %lld must be >= n and a multiple of 4",
                (long long)lds);
    SHARD_CHECK(mul_fits(rows, lds), "rows * lds overflows");
    SHARD_CHECK(S != nullptr && (reinterpret_cast<uintptr_t>(S) & 15u) == 0,
                "S must be a non-null 16-byte aligned device pointer");
    return SYMNMF_OK;
}

extern "C" {

int symnmf_stats_rows(const float* S, int64_t rows, int64_t n, int64_t lds, double* out_dev,
                      void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_rows(S, rows, n, lds));
    SHARD_CHECK(out_dev != nullptr, "out_dev must not be NULL");
    SHARD_CHECK(ws != nullptr && ws_bytes >= (size_t)stats_blocks() * 3 * sizeof(double),
                "workspace too small: %zu given, %zu needed", ws_bytes,
                (size_t)stats_blocks() * 3 * sizeof(double));
    return launch_stats(S, rows, n, lds, static_cast<double*>(ws), stats_blocks(), out_dev,
                        (cudaStream_t)stream);
}

int symnmf_seeded_init(float* H, int64_t n, int k, uint64_t seed, double s_sum,
                       symnmf_stream_t stream) {
    clear_error();
    SHARD_CHECK(H != nullptr && (reinterpret_cast<uintptr_t>(H) & 3u) == 0, "H must be a device pointer");
    SHARD_CHECK(n >= 1 && k >= 1 && k <= KMAX, "need n >= 1 and 1 <= k <= %d", KMAX);
    SHARD_CHECK(mul_fits(n, k), "n * k overflows");
    return launch_init_sum(H, n, k, seed, s_sum, (cudaStream_t)stream);
}

int symnmf_gram(const float* H, int64_t rows, int k, double* A_dev, void* ws, size_t ws_bytes,
                symnmf_stream_t stream) {
    clear_error();
    SHARD_CHECK(H != nullptr && (reinterpret_cast<uintptr_t>(H) & 3u) == 0, "H must be a device pointer");
    SHARD_CHECK(rows >= 1 && k >= 1 && k <= KMAX, "need rows >= 1 and 1 <= k <= %d", KMAX);
    SHARD_CHECK(A_dev != nullptr, "A_dev must not be NULL");
    const int tiles = epilogue_blocks(rows);
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    double* tr = a.take<double>((size_t)tiles);
    double* gp = a.take<double>((size_t)tiles * k * k);
    if (ws == nullptr || !a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    cudaStream_t s = (cudaStream_t)stream;
    SYMNMF_TRY(launch_epilogue(MODE_GRAM, rows, k, nullptr, 0, H, nullptr, nullptr, nullptr, nullptr,
                               0.f, 0.f, 0.f, tr, gp, nullptr, nullptr, s));
    return launch_shard_reduce(nullptr, gp, tiles, k, A_dev, s);
}

int symnmf_shard_workspace_size(int64_t rows, int64_t n, int k, size_t* bytes) {
    clear_error();
    SHARD_CHECK(bytes != nullptr, "bytes must not be NULL");
    SHARD_CHECK(n >= 1 && rows >= 1 && rows <= n && k >= 1 && k <= KMAX, "bad sizes");
    Dev d;
    {
        int dev = 0, sms = 0;
        if (cudaGetDevice(&dev) == cudaSuccess &&
            cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && sms > 0)
            d.sms = sms;
        else
            cudaGetLastError();
    }
    Arena a;
    a.dry = true;
    ShardLayout L;
    shard_plan(d, a, rows, n, k, &L);
    *bytes = a.used + 256;
    return SYMNMF_OK;
}

int symnmf_shard_step(const float* S_rows, int64_t rows, int64_t n, int64_t lds, int64_t row0,
                      int k, const float* H, const double* A_dev, const float* G_rows, float lr,
                      float eps, float* H_rows_next, float* G_rows_next, double* partial_dev,
                      void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_rows(S_rows, rows, n, lds));
    SHARD_CHECK(row0 >= 0 && row0 + rows <= n, "rows [%lld, %lld) must lie in [0, n)", (long long)row0,
                (long long)(row0 + rows));
    SHARD_CHECK(k >= 1 && k <= KMAX, "k = %d must be in [1, %d]", k, KMAX);
    SHARD_CHECK(mul_fits(n, k), "n * k overflows");
    SHARD_CHECK(H && A_dev && G_rows && H_rows_next && G_rows_next && partial_dev,
                "device pointers must not be NULL");
    SHARD_CHECK(lr > 0.f && eps >= 0.f, "lr must be positive and eps >= 0");
    SHARD_CHECK(H_rows_next != H + row0 * k, "H_rows_next must not alias the rows of H being read");
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    ShardLayout L;
    shard_plan(d, a, rows, n, k, &L);
    if (ws == nullptr || !a.ok() || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        set_error("workspace too small or misaligned: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    cudaStream_t s = (cudaStream_t)stream;
    const int tiles = epilogue_blocks(rows);
    shard_state_kernel<<<1, 256, 0, s>>>(L.st, A_dev, k);
    SYMNMF_LAUNCH_CHECK();
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.counters, 0, (size_t)tiles * sizeof(int), s));
    // the split operand of the whole replicated iterate (every column of S is read)
    SYMNMF_TRY(launch_split(H, nullptr, k, k, 0, n, 0, n, L.XT, L.ldxt, s));
    const TcPlan p = plan_stream_tc_rows(d, rows, n, k);
    EpiArgs e;
    std::memset(&e, 0, sizeof(e));
    e.mode = MODE_FULL;
    e.n = rows;
    e.k = k;
    e.splits = p.splits;
    e.part = L.part;
    e.H = H + row0 * k;
    e.G = G_rows;
    e.Hn = H_rows_next;
    e.Gn = G_rows_next;
    e.lr = lr;
    e.eps = eps;
    e.tr_part = L.tr_part;
    e.gram_part = L.gram_part;
    e.st = L.st;
    e.XT = nullptr;
    SYMNMF_TRY(launch_stream_tc(p, S_rows, lds, L.XT, L.ldxt, L.part, &L.st->kerr, L.st, s, &e,
                                L.counters));
    SYMNMF_TRY(launch_shard_reduce(L.tr_part, L.gram_part, tiles, k, partial_dev, s));
    int kerr = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&kerr, &L.st->kerr, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (kerr != 0) {
        set_error("an S-stream pipeline wait timed out on the device (code %d)", kerr);
        return SYMNMF_ERR_TIMEOUT;
    }
    return SYMNMF_OK;
}

}  // extern "C"
