// The rolling-window study ("GPU-Accelerated Clustering for Financial
// Instruments at Scale", sections "The temporal setup", "Tracking stability
// through time", "The metric", "Stability and break detection"): per window
// and per dependence matrix a build, the cross-sector monitor, an independent
// seeded fit and argmax labels; the ARI series against the previous window
// and the window delta earlier; a 3-sigma control limit on the latter.
//
// The driver composes the library's own entry points (builders, fit, labels,
// S-stream product).  The windows are independent fits, each pass of which is
// latency-bound at the workload's size, so the driver runs up to four chains
// side by side -- two per dependence matrix, taking alternate windows -- each
// on its own stream and host thread with its own matrix and buffers; the ARI
// series follows from the stored labels.  This file adds the contingency-table
// kernel behind the ARI and the monitor's reduction kernels.
#include <cmath>
#include <cstring>
#include <cstdlib>
#include <limits>
#include <string>
#include <thread>
#include <vector>

#include "common.cuh"

namespace symnmf {

constexpr int RL_THREADS = 256;
constexpr int RL_MAX_STRESSED = 8;

struct StressedList {
    int g[RL_MAX_STRESSED];
    int count;
};

// ---------------------------------------------------------------- ARI

// table[a_t * k + b_t] += 1 over t; a label outside [0, k) raises *err.
// Per-block counts in shared memory (at most k*k <= 4096 entries), folded into
// the global int64 table with integer atomics: exact in any order.
__global__ void __launch_bounds__(RL_THREADS)
contingency_kernel(const int32_t* __restrict__ a, const int32_t* __restrict__ b, int64_t n, int k,
                   unsigned long long* __restrict__ table, int* __restrict__ err) {
    extern __shared__ unsigned int h[];
    const int kk = k * k;
    for (int i = threadIdx.x; i < kk; i += blockDim.x) h[i] = 0u;
    __syncthreads();
    int bad = 0;
    for (int64_t t = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; t < n;
         t += (int64_t)gridDim.x * blockDim.x) {
        const int x = a[t], y = b[t];
        if ((unsigned)x < (unsigned)k && (unsigned)y < (unsigned)k)
            atomicAdd(&h[x * k + y], 1u);
        else
            bad = 1;
    }
    if (bad) atomicOr(err, 1);
    __syncthreads();
    for (int i = threadIdx.x; i < kk; i += blockDim.x)
        if (h[i]) atomicAdd(&table[i], (unsigned long long)h[i]);
}

static int64_t comb2(int64_t x) { return x * (x - 1) / 2; }

// Hubert & Arabie from exact pair counts; float64 in a fixed order.
static double ari_from_table(const std::vector<int64_t>& t, int k) {
    int64_t n = 0, I = 0, A = 0, B = 0;
    for (int i = 0; i < k; ++i) {
        int64_t row = 0;
        for (int j = 0; j < k; ++j) {
            row += t[(size_t)i * k + j];
            I += comb2(t[(size_t)i * k + j]);
        }
        A += comb2(row);
        n += row;
    }
    for (int j = 0; j < k; ++j) {
        int64_t col = 0;
        for (int i = 0; i < k; ++i) col += t[(size_t)i * k + j];
        B += comb2(col);
    }
    const int64_t P = comb2(n);
    if (P == 0) return 1.0;
    const __int128 den = (__int128)(A + B) * P - (__int128)2 * A * B;
    if (den == 0) return 1.0;
    const double e = ((double)A * (double)B) / (double)P;
    const double m = ((double)A + (double)B) / 2.0;
    return ((double)I - e) / (m - e);
}

struct AriLayout {
    unsigned long long* table = nullptr;
    int* err = nullptr;
};

static void ari_plan(Arena& a, AriLayout* L) {
    L->table = a.take<unsigned long long>((size_t)KMAX * KMAX);
    L->err = a.take<int>(64);
}

static int ari_run(const Dev& d, const AriLayout& L, const int32_t* a, const int32_t* b, int64_t n,
                   int k, double* ari, std::vector<int64_t>* table, cudaStream_t s) {
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.table, 0, sizeof(unsigned long long) * k * k, s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.err, 0, sizeof(int), s));
    const int64_t want = (n + RL_THREADS - 1) / RL_THREADS;
    const int blocks = (int)std::max<int64_t>(1, std::min<int64_t>(want, 2 * d.sms));
    contingency_kernel<<<blocks, RL_THREADS, sizeof(unsigned int) * k * k, s>>>(a, b, n, k, L.table,
                                                                               L.err);
    SYMNMF_LAUNCH_CHECK();
    std::vector<int64_t> t((size_t)k * k);
    int err = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(t.data(), L.table, sizeof(int64_t) * k * k,
                                    cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&err, L.err, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (err) {
        set_error("a label lies outside [0, %d)", k);
        return SYMNMF_ERR_INVALID_ARG;
    }
    *ari = ari_from_table(t, k);
    if (table) *table = std::move(t);
    return SYMNMF_OK;
}

// ---------------------------------------------------------------- cross-sector monitor

// Z[i][g] = [groups_i == stressed_g]; counts[g] = members of stressed group g.
__global__ void stressed_indicator_kernel(const int32_t* __restrict__ groups, int64_t n,
                                          StressedList sl, float* __restrict__ Z,
                                          int* __restrict__ counts) {
    int local[RL_MAX_STRESSED] = {0};
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int gi = groups[i];
        for (int g = 0; g < sl.count; ++g) {
            const bool hit = gi == sl.g[g];
            Z[i * sl.count + g] = hit ? 1.f : 0.f;
            local[g] += hit;
        }
    }
    for (int g = 0; g < sl.count; ++g) {
        int v = local[g];
        for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
        if ((threadIdx.x & 31) == 0 && v) atomicAdd(&counts[g], v);
    }
}

// part[block] = sum over the block's rows i in stressed group a of
// sum_{b != a} Y[i][b], Y = S Z (fp64, fixed order per block).
__global__ void __launch_bounds__(RL_THREADS)
cross_partial_kernel(const float* __restrict__ Y, const float* __restrict__ Z, int64_t n, int G,
                     double* __restrict__ part) {
    __shared__ double red[RL_THREADS];
    double acc = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
         i += (int64_t)gridDim.x * blockDim.x) {
        const float* y = Y + i * G;
        const float* z = Z + i * G;
        double in_group = 0.0, total = 0.0;
        bool member = false;
        for (int g = 0; g < G; ++g) {
            total += (double)y[g];
            if (z[g] != 0.f) {
                in_group = (double)y[g];
                member = true;
            }
        }
        if (member) acc += total - in_group;
    }
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int o = RL_THREADS / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// out = sum(part) / ((sum c)^2 - sum c^2), one block, fixed order.
__global__ void cross_final_kernel(const double* __restrict__ part, int nblk,
                                   const int* __restrict__ counts, int G, double* __restrict__ out) {
    __shared__ double red[RL_THREADS];
    double acc = 0.0;
    for (int i = threadIdx.x; i < nblk; i += blockDim.x) acc += part[i];
    red[threadIdx.x] = acc;
    __syncthreads();
    for (int o = RL_THREADS / 2; o > 0; o >>= 1) {
        if ((int)threadIdx.x < o) red[threadIdx.x] += red[threadIdx.x + o];
        __syncthreads();
    }
    if (threadIdx.x == 0) {
        int64_t sum = 0, sq = 0;
        for (int g = 0; g < G; ++g) {
            sum += counts[g];
            sq += (int64_t)counts[g] * counts[g];
        }
        const int64_t pairs = sum * sum - sq;
        *out = pairs > 0 ? red[0] / (double)pairs : nan("");
    }
}

// ---------------------------------------------------------------- workspace

// One chain's buffers.  A chain runs every P-th window of one dependence
// matrix (build, monitor, fit, labels) on its own stream.
struct ChainLayout {
    void* shared = nullptr;      // builders, fit and the monitor's product take turns here
    size_t shared_bytes = 0;
    float* H = nullptr;
    float* Y = nullptr;          // n x 8 product S Z
    double* part = nullptr;
    double* cross = nullptr;     // the current window's monitor value
};

constexpr int RL_MAX_CHAINS = 4;    // two per kind

struct RollingLayout {
    ChainLayout chain[RL_MAX_CHAINS];
    float* S_own[RL_MAX_CHAINS] = {};   // matrices of chains 1.. (chain 0 uses the caller's S)
    int64_t lds_own = 0;
    int nchains = 1;
    float* Z = nullptr;          // n x 8 indicator of the stressed groups (read-only)
    int* counts = nullptr;
    AriLayout ari;               // the ARI series, computed after the fits
};

static int cross_blocks(const Dev& d) { return 2 * d.sms; }

static int sub_ws(int op, int64_t n, int k, int64_t T, const symnmf_fit_params* P, size_t* b) {
    return symnmf_workspace_size(op, n, k, T, P, b);
}

static void chain_plan(const Dev& d, Arena& a, int64_t n, int k, size_t shared_bytes,
                       ChainLayout* C) {
    C->shared_bytes = shared_bytes;
    C->shared = a.take<char>(shared_bytes);
    C->H = a.take<float>((size_t)n * k);
    C->Y = a.take<float>((size_t)n * RL_MAX_STRESSED);
    C->part = a.take<double>((size_t)cross_blocks(d));
    C->cross = a.take<double>(64);
}

// nchains chains: each after the first gets its own n x n matrix
int rolling_plan(const Dev& d, Arena& a, int64_t n, int k, int64_t T, const symnmf_fit_params& P,
                 int nchains, RollingLayout* L) {
    size_t b_corr = 0, b_tpdm = 0, b_fit = 0, b_sh = 0;
    SYMNMF_TRY(sub_ws(SYMNMF_OP_BUILD_CORR, n, k, T, &P, &b_corr));
    SYMNMF_TRY(sub_ws(SYMNMF_OP_BUILD_TPDM, n, k, T, &P, &b_tpdm));
    SYMNMF_TRY(sub_ws(SYMNMF_OP_FIT, n, k, T, &P, &b_fit));
    SYMNMF_TRY(sub_ws(SYMNMF_OP_SH, n, RL_MAX_STRESSED, T, &P, &b_sh));
    const size_t shared = std::max(std::max(b_corr, b_tpdm), std::max(b_fit, b_sh));
    L->nchains = nchains;
    L->Z = a.take<float>((size_t)n * RL_MAX_STRESSED);
    L->counts = a.take<int>(64);
    ari_plan(a, &L->ari);
    L->lds_own = (n + 3) / 4 * 4;
    for (int c = 0; c < nchains; ++c) {
        chain_plan(d, a, n, k, shared, &L->chain[c]);
        if (c > 0) L->S_own[c] = a.take<float>((size_t)n * (size_t)L->lds_own);
    }
    return SYMNMF_OK;
}

size_t ari_workspace_bytes() {
    Arena a;
    a.dry = true;
    AriLayout L;
    ari_plan(a, &L);
    return a.used + 256;
}

int rolling_workspace_bytes(const Dev& d, int64_t n, int k, int64_t T, const symnmf_fit_params& P,
                            size_t* bytes) {
    Arena a;
    a.dry = true;
    RollingLayout L;
    SYMNMF_TRY(rolling_plan(d, a, n, k, T, P, RL_MAX_CHAINS, &L));
    *bytes = a.used + 256;
    return SYMNMF_OK;
}

// ---------------------------------------------------------------- driver

struct EventPair {
    cudaEvent_t a = nullptr, b = nullptr;
    ~EventPair() {
        if (a) cudaEventDestroy(a);
        if (b) cudaEventDestroy(b);
    }
    int create() {
        SYMNMF_CUDA_TRY(cudaEventCreate(&a));
        SYMNMF_CUDA_TRY(cudaEventCreate(&b));
        return SYMNMF_OK;
    }
    // elapsed ms between a and b (both recorded and complete)
    double ms() const {
        float v = 0.f;
        return cudaEventElapsedTime(&v, a, b) == cudaSuccess ? (double)v : 0.0;
    }
};

// What one chain needs and what it reports.
struct ChainRun {
    int kind = 0;                // 0 = |corr|, 1 = TPDM
    int64_t first = 0, step = 1; // windows first, first + step, ...
    const ChainLayout* C = nullptr;
    float* S = nullptr;
    int64_t lds = 0;
    cudaStream_t s = nullptr;
    double build_ms = 0.0, fit_ms = 0.0;
    int launches = 0;
    int rc = SYMNMF_OK;
    std::string err;
};

struct StudyArgs {
    const Dev* d;
    const float* R;
    int64_t n, ldr, T, W;
    const symnmf_rolling_params* p;
    bool monitor;
    int G;
    const float* Z;
    const int* counts;
    symnmf_rolling_out* out;
};

// The chain's windows on r.s: build, monitor, fit, labels (the ARIs come after).
static int run_chain(const StudyArgs& A, ChainRun& r) {
    const symnmf_rolling_params& p = *A.p;
    const ChainLayout& L = *r.C;
    const int64_t n = A.n;
    const int c = r.kind;
    const double nan = std::numeric_limits<double>::quiet_NaN();
    EventPair ev_build, ev_fit;
    SYMNMF_TRY(ev_build.create());
    SYMNMF_TRY(ev_fit.create());
    auto count = [&]() {
        r.launches += launches();
        reset_launches();
    };
    reset_launches();
    for (int64_t w = r.first; w < A.W; w += r.step) {
        const float* Rw = A.R + (size_t)(w * p.stride) * (size_t)A.ldr;
        SYMNMF_CUDA_TRY(cudaEventRecord(ev_build.a, r.s));
        if (c == 0)
            SYMNMF_TRY(symnmf_build_corr(Rw, A.T, n, A.ldr, r.S, r.lds, L.shared, L.shared_bytes, r.s));
        else
            SYMNMF_TRY(symnmf_build_tpdm(Rw, A.T, n, A.ldr, p.tail_frac, p.tail_sign, r.S, r.lds,
                                         L.shared, L.shared_bytes, r.s));
        count();
        SYMNMF_CUDA_TRY(cudaEventRecord(ev_build.b, r.s));
        double cross = nan;
        if (A.monitor) {
            SYMNMF_TRY(symnmf_sh(r.S, n, r.lds, A.Z, A.G, L.Y, L.shared, L.shared_bytes, r.s));
            cross_partial_kernel<<<cross_blocks(*A.d), RL_THREADS, 0, r.s>>>(L.Y, A.Z, n, A.G, L.part);
            SYMNMF_LAUNCH_CHECK();
            cross_final_kernel<<<1, RL_THREADS, 0, r.s>>>(L.part, cross_blocks(*A.d), A.counts, A.G,
                                                          L.cross);
            SYMNMF_LAUNCH_CHECK();
            SYMNMF_CUDA_TRY(cudaMemcpyAsync(&cross, L.cross, sizeof(double), cudaMemcpyDeviceToHost,
                                            r.s));
            count();
        }
        SYMNMF_CUDA_TRY(cudaEventRecord(ev_fit.a, r.s));
        symnmf_fit_stats st;
        // every window from the seeded start, or with a warm start from the
        // chain's previous window (step 1); the AdaGrad accumulator starts at 0
        symnmf_fit_params fp = p.fit;
        fp.init = (p.warm_start && w > r.first) ? SYMNMF_INIT_USER : SYMNMF_INIT_SEEDED;
        fp.G_inout = nullptr;
        SYMNMF_TRY(symnmf_fit(r.S, n, r.lds, p.k, &fp, L.H, &st, L.shared, L.shared_bytes, r.s));
        count();
        int32_t* lab = A.out->labels[c] + (size_t)w * (size_t)n;
        SYMNMF_TRY(symnmf_labels(L.H, n, p.k, lab, r.s));
        count();
        SYMNMF_CUDA_TRY(cudaEventRecord(ev_fit.b, r.s));
        SYMNMF_CUDA_TRY(cudaStreamSynchronize(r.s));   // both event pairs complete, cross read
        r.build_ms += ev_build.ms();
        r.fit_ms += ev_fit.ms();
        if (A.out->cross[c]) A.out->cross[c][w] = cross;
        if (A.out->loss[c]) A.out->loss[c][w] = st.loss;
    }
    return SYMNMF_OK;
}

// Chains side by side unless SYMNMF_ROLLING_SERIAL=1 (read at each call).
static bool rolling_serial() {
    const char* e = getenv("SYMNMF_ROLLING_SERIAL");
    return e != nullptr && std::strcmp(e, "1") == 0;
}

// Runs run[1..nc-1] on their own host threads (each on its own stream,
// ordered after s) and run[0] on this thread and s; s then waits for them.
// A chain whose thread cannot be started runs here after run[0].
static int run_chains(const StudyArgs& A, ChainRun* run, int nc, cudaStream_t s) {
    int dev = 0;
    SYMNMF_CUDA_TRY(cudaGetDevice(&dev));
    cudaEvent_t e_in = nullptr;
    cudaStream_t streams[RL_MAX_CHAINS] = {};
    cudaEvent_t e_out[RL_MAX_CHAINS] = {};
    auto release = [&]() {
        if (e_in) cudaEventDestroy(e_in);
        for (int i = 1; i < nc; ++i) {
            if (e_out[i]) cudaEventDestroy(e_out[i]);
            if (streams[i]) cudaStreamDestroy(streams[i]);
        }
    };
    bool ok = cudaEventCreateWithFlags(&e_in, cudaEventDisableTiming) == cudaSuccess &&
              cudaEventRecord(e_in, s) == cudaSuccess;
    for (int i = 1; ok && i < nc; ++i)
        ok = cudaStreamCreateWithFlags(&streams[i], cudaStreamNonBlocking) == cudaSuccess &&
             cudaEventCreateWithFlags(&e_out[i], cudaEventDisableTiming) == cudaSuccess &&
             cudaStreamWaitEvent(streams[i], e_in, 0) == cudaSuccess;
    if (!ok) {
        release();
        set_error("could not set up the rolling study's streams");
        return SYMNMF_ERR_CUDA;
    }
    auto body = [&](int i) {
        ChainRun& r = run[i];
        if (cudaSetDevice(dev) != cudaSuccess) {
            r.rc = SYMNMF_ERR_CUDA;
            r.err = "cudaSetDevice failed in a rolling chain";
            return;
        }
        r.rc = run_chain(A, r);
        if (r.rc != SYMNMF_OK) r.err = symnmf_last_error();
    };
    std::thread workers[RL_MAX_CHAINS];
    bool threaded[RL_MAX_CHAINS] = {};
    for (int i = 1; i < nc; ++i) {
        run[i].s = streams[i];
        try {
            workers[i] = std::thread(body, i);
            threaded[i] = true;
        } catch (...) {   // no thread to be had: this chain runs here after chain 0
            threaded[i] = false;
        }
    }
    run[0].rc = run_chain(A, run[0]);
    if (run[0].rc != SYMNMF_OK) run[0].err = symnmf_last_error();
    for (int i = 1; i < nc; ++i) {
        if (threaded[i]) workers[i].join();
        else body(i);
    }
    bool joined = true;
    for (int i = 1; i < nc; ++i)
        joined = joined && cudaEventRecord(e_out[i], streams[i]) == cudaSuccess &&
                 cudaStreamWaitEvent(s, e_out[i], 0) == cudaSuccess;
    release();
    for (int i = 0; i < nc; ++i)
        if (run[i].rc != SYMNMF_OK) {
            set_error("%s", run[i].err.c_str());
            return run[i].rc;
        }
    if (!joined) {
        set_error("could not order the caller's stream after the rolling chains");
        return SYMNMF_ERR_CUDA;
    }
    return SYMNMF_OK;
}

static int rolling_impl(const float* R, int64_t days, int64_t n, int64_t ldr, const int32_t* groups,
                        float* S, int64_t lds, const symnmf_rolling_params& p,
                        symnmf_rolling_out* out, void* ws, size_t ws_bytes, cudaStream_t s) {
    Dev d;
    SYMNMF_TRY(device_info(&d));
    const int64_t T = p.window;
    const int64_t W = p.n_windows > 0 ? p.n_windows : (days - T) / p.stride + 1;
    if (W < 1 || (W - 1) * p.stride + T > days) {
        set_error("%lld windows of %lld days with stride %lld do not fit in %lld days",
                  (long long)W, (long long)T, (long long)p.stride, (long long)days);
        return SYMNMF_ERR_INVALID_ARG;
    }
    const bool kind_on[2] = {(p.kinds & SYMNMF_KIND_CORR) != 0, (p.kinds & SYMNMF_KIND_TPDM) != 0};
    for (int c = 0; c < 2; ++c)
        if (kind_on[c] && out->labels[c] == nullptr) {
            set_error("labels[%d] must be a device buffer of n_windows x n int32", c);
            return SYMNMF_ERR_INVALID_ARG;
        }
    int kinds[2], nk = 0;
    for (int c = 0; c < 2; ++c)
        if (kind_on[c]) kinds[nk++] = c;
    // chains: two per kind when the workspace holds them, else one per kind,
    // else a single chain that runs the kinds in turn
    RollingLayout L;
    int per_kind = 1, nc = 1;
    {
        const int tries[3][2] = {{2, 2 * nk}, {1, nk}, {1, 1}};
        bool fit = false;
        // a warm start needs each kind's windows in order on one chain
        for (int t = rolling_serial() ? 2 : (p.warm_start ? 1 : 0); t < 3 && !fit; ++t) {
            if (tries[t][1] > RL_MAX_CHAINS) continue;
            Arena a;
            a.base = static_cast<char*>(ws);
            a.cap = ws_bytes;
            L = RollingLayout();
            SYMNMF_TRY(rolling_plan(d, a, n, p.k, T, p.fit, tries[t][1], &L));
            if (a.ok()) {
                fit = true;
                per_kind = tries[t][0];
                nc = tries[t][1];
            } else if (t == 2) {
                set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
                return SYMNMF_ERR_WORKSPACE;
            }
        }
    }
    const bool monitor = p.n_stressed >= 2;
    const int G = p.n_stressed;
    StressedList sl{};
    sl.count = G;
    for (int g = 0; g < G; ++g) sl.g[g] = p.stressed[g];

    reset_launches();
    EventPair whole;
    SYMNMF_TRY(whole.create());
    SYMNMF_CUDA_TRY(cudaEventRecord(whole.a, s));
    if (monitor) {
        SYMNMF_CUDA_TRY(cudaMemsetAsync(L.counts, 0, sizeof(int) * RL_MAX_STRESSED, s));
        const int blocks = (int)std::max<int64_t>(
            1, std::min<int64_t>((n + RL_THREADS - 1) / RL_THREADS, 2 * d.sms));
        stressed_indicator_kernel<<<blocks, RL_THREADS, 0, s>>>(groups, n, sl, L.Z, L.counts);
        SYMNMF_LAUNCH_CHECK();
    }
    int launches_total = launches();
    reset_launches();

    const double nan = std::numeric_limits<double>::quiet_NaN();
    for (int c = 0; c < 2; ++c) {
        out->build_ms[c] = 0.0;
        out->fit_ms[c] = 0.0;
        out->mean[c] = out->std[c] = out->limit[c] = nan;
    }
    out->n_windows = W;
    StudyArgs A{&d, R, n, ldr, T, W, &p, monitor, G, L.Z, L.counts, out};
    ChainRun run[RL_MAX_CHAINS];
    for (int i = 0; i < nc; ++i) {
        run[i].C = &L.chain[i];
        run[i].S = i == 0 ? S : L.S_own[i];
        run[i].lds = i == 0 ? lds : L.lds_own;
        run[i].s = s;
    }
    if (nc == 1) {
        for (int q = 0; q < nk; ++q) {   // the kinds in turn on one chain
            run[0].kind = kinds[q];
            SYMNMF_TRY(run_chain(A, run[0]));
            out->build_ms[kinds[q]] = run[0].build_ms;
            out->fit_ms[kinds[q]] = run[0].fit_ms;
            launches_total += run[0].launches;
            run[0].build_ms = run[0].fit_ms = 0.0;
            run[0].launches = 0;
        }
    } else {
        for (int i = 0; i < nc; ++i) {
            run[i].kind = kinds[i / per_kind];
            run[i].first = i % per_kind;
            run[i].step = per_kind;
        }
        SYMNMF_TRY(run_chains(A, run, nc, s));
        for (int i = 0; i < nc; ++i) {
            out->build_ms[run[i].kind] += run[i].build_ms;
            out->fit_ms[run[i].kind] += run[i].fit_ms;
            launches_total += run[i].launches;
        }
    }

    // ARI(t - 1, t) and ARI(t - delta, t) from the stored labels
    std::vector<double> ari_delta[2];
    reset_launches();
    for (int c = 0; c < 2; ++c) {
        if (!kind_on[c]) continue;
        ari_delta[c].assign((size_t)W, nan);
        const int32_t* lab = out->labels[c];
        for (int64_t w = 0; w < W; ++w) {
            double prev = nan, dl = nan;
            const int32_t* lw = lab + (size_t)w * (size_t)n;
            if (w >= 1) SYMNMF_TRY(ari_run(d, L.ari, lw - n, lw, n, p.k, &prev, nullptr, s));
            if (w >= p.delta)
                SYMNMF_TRY(ari_run(d, L.ari, lw - (size_t)p.delta * n, lw, n, p.k, &dl, nullptr, s));
            ari_delta[c][(size_t)w] = dl;
            if (out->ari_prev[c]) out->ari_prev[c][w] = prev;
            if (out->ari_delta[c]) out->ari_delta[c][w] = dl;
        }
    }
    launches_total += launches();
    SYMNMF_CUDA_TRY(cudaEventRecord(whole.b, s));
    SYMNMF_CUDA_TRY(cudaEventSynchronize(whole.b));
    out->total_ms = whole.ms();

    // 3-sigma control limit on ARI(t - delta, t)
    const int64_t c0 = std::max<int64_t>(p.calib_begin, p.delta);
    const int64_t c1 = p.calib_end > 0 ? std::min<int64_t>(p.calib_end, W) : W;
    for (int c = 0; c < 2; ++c) {
        if (!kind_on[c]) continue;
        const std::vector<double>& ad = ari_delta[c];
        double sum = 0.0;
        int64_t m = 0;
        for (int64_t t = c0; t < c1; ++t)
            if (std::isfinite(ad[(size_t)t])) {
                sum += ad[(size_t)t];
                ++m;
            }
        if (m >= 2) {
            const double mu = sum / (double)m;
            double ss = 0.0;
            for (int64_t t = c0; t < c1; ++t)
                if (std::isfinite(ad[(size_t)t])) {
                    const double dv = ad[(size_t)t] - mu;
                    ss += dv * dv;
                }
            out->mean[c] = mu;
            out->std[c] = std::sqrt(ss / (double)(m - 1));
            out->limit[c] = mu - 3.0 * out->std[c];
        }
        if (out->flag[c])
            for (int64_t t = 0; t < W; ++t) {
                const double v = ad[(size_t)t];
                out->flag[c][t] = (std::isfinite(v) && std::isfinite(out->limit[c]) &&
                                   v < out->limit[c]) ? 1 : 0;
            }
    }
    out->kernel_launches = launches_total;
    return SYMNMF_OK;
}

}  // namespace symnmf

using namespace symnmf;

extern "C" {

int symnmf_ari(const int32_t* a, const int32_t* b, int64_t n, int k, double* ari_host,
               int64_t* table_host, void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    if (n < 1 || k < 1 || k > KMAX || a == nullptr || b == nullptr || ari_host == nullptr) {
        set_error("need n >= 1, 1 <= k <= %d and non-null a, b, ari_host", KMAX);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0) {
        set_error("ws must be a 256-byte aligned device buffer");
        return SYMNMF_ERR_INVALID_ARG;
    }
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena ar;
    ar.base = static_cast<char*>(ws);
    ar.cap = ws_bytes;
    AriLayout L;
    ari_plan(ar, &L);
    if (!ar.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, ar.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    std::vector<int64_t> t;
    SYMNMF_TRY(ari_run(d, L, a, b, n, k, ari_host, &t, (cudaStream_t)stream));
    if (table_host) std::copy(t.begin(), t.end(), table_host);
    return SYMNMF_OK;
}

void symnmf_rolling_params_default(symnmf_rolling_params* p) {
    if (p == nullptr) return;
    std::memset(p, 0, sizeof(*p));
    p->window = 250;
    p->stride = 1;
    p->n_windows = 0;
    p->k = 24;
    p->kinds = SYMNMF_KIND_CORR | SYMNMF_KIND_TPDM;
    p->tail_frac = 0.05;
    p->tail_sign = -1;
    p->delta = 50;
    p->calib_begin = 0;
    p->calib_end = 0;
    p->n_stressed = 0;
    p->warm_start = 0;
    symnmf_fit_params_default(&p->fit);
    p->fit.max_iters = 100;
    p->fit.rel_tol = 0.0;
}

int symnmf_rolling(const float* R, int64_t days, int64_t n, int64_t ldr, const int32_t* groups,
                   float* S, int64_t lds, const symnmf_rolling_params* params,
                   symnmf_rolling_out* out, void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    if (params == nullptr || out == nullptr) {
        set_error("params and out must not be NULL");
        return SYMNMF_ERR_INVALID_ARG;
    }
    const symnmf_rolling_params& p = *params;
    if (R == nullptr || (reinterpret_cast<uintptr_t>(R) & 15u) != 0 || ldr < n || ldr % 4 != 0) {
        set_error("R must be a 16-byte aligned device pointer with ldr >= n, ldr a multiple of 4");
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (p.window < 2 || p.stride < 1 || p.n_windows < 0 || p.delta < 1 || days < p.window) {
        set_error("need window >= 2, stride >= 1, n_windows >= 0, delta >= 1, days >= window");
        return SYMNMF_ERR_INVALID_ARG;
    }
    if ((p.kinds & (SYMNMF_KIND_CORR | SYMNMF_KIND_TPDM)) == 0 || (p.kinds & ~3) != 0) {
        set_error("kinds = %d: select SYMNMF_KIND_CORR and/or SYMNMF_KIND_TPDM", p.kinds);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (p.n_stressed != 0 && (p.n_stressed < 2 || p.n_stressed > RL_MAX_STRESSED || groups == nullptr)) {
        set_error("n_stressed = %d: 0, or 2..%d with a groups array", p.n_stressed, RL_MAX_STRESSED);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (p.warm_start != 0 && p.warm_start != 1) {
        set_error("warm_start = %d must be 0 or 1", p.warm_start);
        return SYMNMF_ERR_INVALID_ARG;
    }
    if (p.k < 1 || p.k > KMAX || p.k > n) {
        set_error("k = %d must be in [1, min(64, n)]", p.k);
        return SYMNMF_ERR_INVALID_ARG;
    }
    return rolling_impl(R, days, n, ldr, groups, S, lds, p, out, ws, ws_bytes,
                        (cudaStream_t)stream);
}

}  // extern "C"
