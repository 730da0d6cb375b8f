// extern "C" entry points of libsymnmf.so and the host-side drivers: the
// full-batch loop, Block-SVRG with AdaptGrow growth, AUTO solver selection
// and the block-Lanczos spectral probe.  Every arithmetic step on n-sized
// data runs in the kernels of stream.cu, misc.cu and builders.cu.
#include <chrono>
#include <cmath>
#include <cstdarg>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <unordered_map>
#include <vector>

#include "common.cuh"
#include "epilogue.cuh"
#include "hostla.h"

namespace symnmf {

// ---------------------------------------------------------------- errors
static thread_local std::string g_last_error;

void set_error(const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof buf, fmt, ap);
    va_end(ap);
    g_last_error = buf;
}
void clear_error() { g_last_error.clear(); }

static thread_local int g_launches = 0;
void note_launch() { ++g_launches; }
int launches() { return g_launches; }
void reset_launches() { g_launches = 0; }

#define SYMNMF_CHECK_ARG(cond, ...)                 \
    do {                                            \
        if (!(cond)) {                              \
            ::symnmf::set_error(__VA_ARGS__);       \
            return SYMNMF_ERR_INVALID_ARG;          \
        }                                           \
    } while (0)

// ---------------------------------------------------------------- device
int device_info(Dev* d) {
    int dev = 0;
    SYMNMF_CUDA_TRY(cudaGetDevice(&dev));
    int major = 0, sms = 0;
    SYMNMF_CUDA_TRY(cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev));
    SYMNMF_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
    d->cc_major = major;
    d->sms = sms;
    if (major != 10) {
        set_error("libsymnmf is built for sm_100a (B200); device %d has compute capability %d.x",
                  dev, major);
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    return SYMNMF_OK;
}

static bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
static bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }
static bool mul_ok(int64_t a, int64_t b) {
    return a >= 0 && b >= 0 && (a == 0 || b <= (int64_t(1) << 62) / a);
}

static int check_S(const float* S, int64_t n, int64_t lds) {
    SYMNMF_CHECK_ARG(n >= 1, "n = %lld must be >= 1", (long long)n);
    SYMNMF_CHECK_ARG(lds >= n, "lds = %lld must be >= n = %lld", (long long)lds, (long long)n);
    SYMNMF_CHECK_ARG(lds % 4 == 0, "lds = %lld must be a multiple of 4 (16-byte rows)", (long long)lds);
    SYMNMF_CHECK_ARG(mul_ok(n, lds), "n * lds overflows");
    SYMNMF_CHECK_ARG(S != nullptr && aligned16(S), "S must be a non-null 16-byte aligned device pointer");
    return SYMNMF_OK;
}

// ---------------------------------------------------------------- S-stream dispatch
// The tensor-core kernel is the S-stream; SYMNMF_STREAM=cuda_core selects the
// CUDA-core kernel instead (same result within fp32 rounding), for comparison.
static bool use_tc() {
    static const bool v = [] {   // read once (thread-safe static initialisation)
        const char* e = getenv("SYMNMF_STREAM");
        return !(e != nullptr && std::strcmp(e, "cuda_core") == 0);
    }();
    return v;
}

static size_t stream_partials(const Dev& d, int64_t n, int k, int64_t r0, int64_t r1) {
    return std::max(stream_partial_floats(plan_stream(d, n, k, r0, r1)),
                    tc_partial_floats(plan_stream_tc(d, n, k, r0, r1)));
}

struct StreamArgs {
    const float* S;
    int64_t n, lds;
    int k;
    float* part;
    float* XT;     // [X_hi; X_lo] operand buffer (tensor-core path)
    int64_t ldxt;
    int* err;
    int* counters; // one per 128-row tile, zero between passes (tensor-core path)
    const FitState* st;
    bool upper = false;       // full passes read only the tiles on or above the diagonal
    float* tpart = nullptr;   // their partial slabs
    float* fpart = nullptr;
};

// One pass over S: part[s] = S[:, r0:r1] X[r0:r1, :] with X = Xa - Xb (Xb may be
// NULL) on the rows [r0, r1), then the epilogue `epi` (fused into the stream
// kernel on the tensor-core path).  xt_ready: XT already holds the split of X.
static int stream_pass(const Dev& d, const StreamArgs& a, const float* Xa, const float* Xb,
                       int64_t ldx, int64_t r0, int64_t r1, bool xt_ready, EpiArgs epi,
                       cudaStream_t s, struct Timing* tm);

// ---------------------------------------------------------------- workspace plans
struct FitLayout {
    FitState* st = nullptr;
    float* H1 = nullptr;
    float* G0 = nullptr;
    float* G1 = nullptr;
    float* part = nullptr;
    double* tr_part = nullptr;
    double* gram_part = nullptr;
    double* stats_part = nullptr;
    double* hist = nullptr;
    float* Psnap = nullptr;
    float* Hsnap = nullptr;
    void* probe_ws = nullptr;
    size_t probe_bytes = 0;
    int hist_cap = 0;
    float* XT[2] = {nullptr, nullptr};   // split operand of Hb[0] / Hb[1]
    int64_t ldxt = 0;
    int* counters = nullptr;
    float* tpart = nullptr;              // upper-triangle partial slabs (upper_only = 1)
    float* fpart = nullptr;
    uint16_t* XT16 = nullptr;            // fp16 operand of the fp16 S-stream (k <= 24)
    float* hmax_part = nullptr;          // per-tile max |H_{t+1}| (fp16 S-stream)
    float* amax_part = nullptr;          // per-block max |S| of the statistics pass
};

static int64_t default_block_rows(int64_t n) {
    // power of two nearest n/10 on a log scale (see the oracle for the reading)
    int64_t b = 1;
    while (10 * (2 * b) <= n) b *= 2;
    if (10 * b <= n && 200.0 * (double)b * (double)b < (double)n * (double)n) b *= 2;
    return std::max<int64_t>(1, std::min<int64_t>(b, n));
}

static size_t probe_workspace(const Dev& d, int64_t n, int block, int max_iter, Arena* a,
                              struct ProbeLayout* L);

struct ProbeLayout {
    float* Q = nullptr;      // n x mtot basis, row-major (ld = mtot)
    float* W = nullptr;      // n x b product block
    float* part = nullptr;   // stream partials
    float* XT = nullptr;     // split operand of the tensor-core stream
    int64_t ldxt = 0;
    int* err = nullptr;
    int* counters = nullptr;
    double* tn_part = nullptr;
    double* C64 = nullptr;
    float* C32 = nullptr;
    float* M32 = nullptr;
    int mtot = 0;
};

static int64_t probe_mtot(int64_t n, int block, int max_iter) {
    int64_t m = (int64_t)block * (max_iter + 1);
    return std::min<int64_t>(m, (n / block) * block);
}

static size_t probe_workspace(const Dev& d, int64_t n, int block, int max_iter, Arena* a,
                              ProbeLayout* L) {
    const int64_t mtot = std::max<int64_t>(probe_mtot(n, block, max_iter), block);
    L->mtot = (int)mtot;
    L->Q = a->take<float>((size_t)n * mtot);
    L->W = a->take<float>((size_t)n * block);
    L->part = a->take<float>(stream_partials(d, n, block, 0, n));
    L->ldxt = xt_ld(n);
    L->XT = a->take<float>((size_t)xt_rows(block) * L->ldxt);
    L->err = a->take<int>(64);
    L->counters = a->take<int>((size_t)epilogue_blocks(n));
    L->tn_part = a->take<double>((size_t)gemm_tn_blocks(n) * 4096);
    L->C64 = a->take<double>((size_t)mtot * block);
    L->C32 = a->take<float>((size_t)mtot * block);
    L->M32 = a->take<float>((size_t)block * block);
    return a->used;
}

static int plan_fit(const Dev& d, Arena& a, int64_t n, int k, const symnmf_fit_params& P,
                    FitLayout* L) {
    L->st = reinterpret_cast<FitState*>(a.take<char>(fit_state_bytes()));
    L->H1 = a.take<float>((size_t)n * k);
    L->G0 = a.take<float>((size_t)n * k);
    L->G1 = a.take<float>((size_t)n * k);
    size_t pf = stream_partials(d, n, k, 0, n);
    const bool svrg = P.solver != SYMNMF_SOLVER_ADAGRAD;
    int64_t b = 0;
    if (svrg) {
        b = P.block_rows > 0 ? std::min<int64_t>(P.block_rows, n) : default_block_rows(n);
        // the block can grow: every power-of-two multiple up to n may be planned
        for (int64_t bb = b; bb < n; bb *= 2) {
            const int64_t m = (n + bb - 1) / bb;
            for (int64_t blk = 0; blk < m && blk < 2; ++blk) {
                const int64_t r0 = blk * bb, r1 = std::min(n, r0 + bb);
                pf = std::max(pf, stream_partials(d, n, k, r0, r1));
            }
        }
    }
    if (h16_supported(k)) pf = std::max(pf, tc_partial_floats(plan_stream_h16(d, n, k)));
    if (P.upper_only) {
        const TriPlan tp = plan_stream_tri(d, n, k);
        pf = std::max(pf, (size_t)n * k);   // the reduced product goes to part
        L->tpart = a.take<float>(tri_tpart_floats(tp));
        L->fpart = a.take<float>(tri_fpart_floats(tp));
    }
    L->part = a.take<float>(pf);
    L->ldxt = xt_ld(n);
    L->XT[0] = a.take<float>((size_t)xt_rows(k) * L->ldxt);
    L->XT[1] = a.take<float>((size_t)xt_rows(k) * L->ldxt);
    L->counters = a.take<int>((size_t)epilogue_blocks(n));
    const int nb = epilogue_blocks(n);
    L->tr_part = a.take<double>((size_t)nb);
    L->gram_part = a.take<double>((size_t)nb * k * k);
    L->stats_part = a.take<double>((size_t)stats_blocks() * 3);
    L->amax_part = a.take<float>((size_t)stats_blocks());
    if (h16_supported(k)) {
        L->XT16 = a.take<uint16_t>(h16_xt_halves(n, k));
        L->hmax_part = a.take<float>((size_t)nb);
    }
    L->hist_cap = std::max(1, P.max_iters + 1);
    L->hist = a.take<double>((size_t)L->hist_cap);
    if (svrg) {
        L->Psnap = a.take<float>((size_t)n * k);
        L->Hsnap = a.take<float>((size_t)n * k);
    }
    if (P.solver == SYMNMF_SOLVER_AUTO && !(P.eigvals != nullptr && P.n_eigvals >= k + 2)) {
        Arena sub;
        sub.dry = true;
        ProbeLayout pl;
        const size_t pb = probe_workspace(d, n, P.probe_block, P.probe_max_iter, &sub, &pl);
        L->probe_ws = a.take<char>(pb + 256);
        L->probe_bytes = pb + 256;
    }
    return SYMNMF_OK;
}

// The full-batch loop of the AdaGrad solver streams S through the fp16
// tensor-core kernel (stream_h16.cu) from n = 20,000 up (k <= 24, tensor-core
// path, full matrix); below that the TF32 kernel, which measured about as fast
// there (its passes need no extra launch for the operand split).
// SYMNMF_H16_MIN_N overrides the size (0: never).
static int64_t h16_min_n() {
    const char* e = getenv("SYMNMF_H16_MIN_N");   // read per call: tests switch it
    if (e != nullptr && *e != 0) return std::strtoll(e, nullptr, 10);
    return 20000;
}
static bool h16_path(int64_t n, int k, const symnmf_fit_params& P) {
    const int64_t m = h16_min_n();
    return use_tc() && h16_supported(k) && P.upper_only == 0 && m > 0 && n >= m;
}

static int check_params(const symnmf_fit_params& P, int64_t n, int k) {
    SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX, "k = %d must be in [1, %d]", k, KMAX);
    SYMNMF_CHECK_ARG(P.solver >= 0 && P.solver <= 2, "unknown solver %d", P.solver);
    SYMNMF_CHECK_ARG(P.init == SYMNMF_INIT_SEEDED || P.init == SYMNMF_INIT_USER, "unknown init %d", P.init);
    SYMNMF_CHECK_ARG(P.lr > 0.f && std::isfinite(P.lr), "lr must be positive and finite");
    SYMNMF_CHECK_ARG(P.eps >= 0.f && std::isfinite(P.eps), "eps must be >= 0");
    SYMNMF_CHECK_ARG(P.max_iters >= 0 && P.max_iters < (1 << 30), "max_iters must be >= 0");
    SYMNMF_CHECK_ARG(P.rel_tol >= 0.0, "rel_tol must be >= 0");
    SYMNMF_CHECK_ARG(P.block_rows >= 0, "block_rows must be >= 0");
    SYMNMF_CHECK_ARG(P.upper_only == 0 || P.upper_only == 1, "upper_only must be 0 or 1");
    SYMNMF_CHECK_ARG(!P.upper_only || tri_supported(k), "upper_only = 1 supports k <= 24 (k = %d)", k);
    SYMNMF_CHECK_ARG(P.check_every >= 1, "check_every must be >= 1");
    if (P.solver == SYMNMF_SOLVER_AUTO) {
        SYMNMF_CHECK_ARG(k + 2 <= n, "AUTO needs n >= k + 2 eigenvalues");
        SYMNMF_CHECK_ARG(P.probe_block >= 1 && P.probe_block <= KMAX, "probe_block must be in [1, 64]");
        SYMNMF_CHECK_ARG(P.probe_max_iter >= 1, "probe_max_iter must be >= 1");
    }
    SYMNMF_CHECK_ARG(P.loss_history == nullptr || P.loss_history_len >= 0, "loss_history_len < 0");
    return SYMNMF_OK;
}

// ---------------------------------------------------------------- fit drivers
struct Timing {
    bool on = false;
    bool capturing = false;       // inside graph capture: records become graph nodes
    std::vector<cudaEvent_t> ev;  // pairs
    int used = 0;
    double ms = 0.0;
    int launches = 0;
    std::vector<float> each;      // every timed launch, in order
    int record(cudaEvent_t e, cudaStream_t s) {
        if (capturing) SYMNMF_CUDA_TRY(cudaEventRecordWithFlags(e, s, cudaEventRecordExternal));
        else SYMNMF_CUDA_TRY(cudaEventRecord(e, s));
        return SYMNMF_OK;
    }
    // after a graph replay: the first `count` captured pairs did work
    int harvest_pairs(int count) {
        for (int i = 0; i < 2 * count && i + 1 < used; i += 2) {
            float ms1 = 0.f;
            SYMNMF_CUDA_TRY(cudaEventElapsedTime(&ms1, ev[i], ev[i + 1]));
            ms += ms1;
            each.push_back(ms1);
            ++launches;
        }
        return SYMNMF_OK;
    }
    ~Timing() {
        for (auto e : ev) cudaEventDestroy(e);
    }
    int begin(cudaStream_t s) {
        if (!on) return SYMNMF_OK;
        if (used + 2 > (int)ev.size()) {
            cudaEvent_t a, b;
            SYMNMF_CUDA_TRY(cudaEventCreate(&a));
            SYMNMF_CUDA_TRY(cudaEventCreate(&b));
            ev.push_back(a);
            ev.push_back(b);
        }
        return record(ev[used], s);
    }
    int end(cudaStream_t s) {
        if (!on) return SYMNMF_OK;
        SYMNMF_TRY(record(ev[used + 1], s));
        used += 2;
        return SYMNMF_OK;
    }
    int harvest() {  // after a stream synchronisation
        for (int i = 0; i < used; i += 2) {
            float ms1 = 0.f;
            SYMNMF_CUDA_TRY(cudaEventElapsedTime(&ms1, ev[i], ev[i + 1]));
            ms += ms1;
            each.push_back(ms1);
            ++launches;
        }
        used = 0;
        return SYMNMF_OK;
    }
};

struct HostState {
    double s_sum, s_sqnorm, s_bad, loss, loss_prev, rel;
    int t, t_stop, done, converged, nonfinite;
};

static int read_state(const FitState* st, HostState* h, cudaStream_t s) {
    FitState tmp;
    const size_t head = offsetof(FitState, A64);
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&tmp, st, head, cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&tmp.t, &st->t, sizeof(int) * 6, cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    h->s_sum = tmp.s_sum;
    h->s_sqnorm = tmp.s_sqnorm;
    h->s_bad = tmp.s_bad;
    h->loss = tmp.loss;
    h->loss_prev = tmp.loss_prev;
    h->rel = tmp.rel;
    h->t = tmp.t;
    h->t_stop = tmp.t_stop;
    h->done = tmp.done || tmp.kerr != 0;   // a pass that gave up waiting ends the loop
    h->converged = tmp.converged;
    h->nonfinite = tmp.nonfinite;
    return SYMNMF_OK;
}

static int stream_pass(const Dev& d, const StreamArgs& a, const float* Xa, const float* Xb,
                       int64_t ldx, int64_t r0, int64_t r1, bool xt_ready, EpiArgs epi,
                       cudaStream_t s, Timing* tm) {
    epi.part = a.part;
    if (a.upper && r0 == 0 && r1 == a.n) {
        // upper-triangle stream: S X into part (or straight into Y for a product),
        // then the standalone epilogue over that one partial
        const TriPlan p = plan_stream_tri(d, a.n, a.k);
        if (!xt_ready) SYMNMF_TRY(launch_split(Xa, Xb, ldx, a.k, 0, a.n, 0, a.n, a.XT, a.ldxt, s));
        if (tm) SYMNMF_TRY(tm->begin(s));
        SYMNMF_TRY(launch_stream_tri(p, a.S, a.lds, a.XT, a.ldxt, a.tpart, a.fpart, a.err, a.st, s));
        if (tm) SYMNMF_TRY(tm->end(s));
        const bool product = epi.mode == MODE_PRODUCT;
        SYMNMF_TRY(launch_tri_reduce(p, a.tpart, a.fpart, product ? epi.Y : a.part, a.st, s));
        if (product) return SYMNMF_OK;
        return launch_epilogue(epi.mode, epi.n, epi.k, a.part, 1, epi.H, epi.G, epi.Hn, epi.Gn,
                               epi.Psnap, epi.m_scale, epi.lr, epi.eps, epi.tr_part, epi.gram_part,
                               epi.Y, epi.st, s, epi.XT, epi.ldxt);
    }
    if (use_tc()) {
        const TcPlan p = plan_stream_tc(d, a.n, a.k, r0, r1);
        if (!xt_ready)
            SYMNMF_TRY(launch_split(Xa, Xb, ldx, a.k, r0, r1, p.j0, p.j1, a.XT, a.ldxt, s));
        epi.splits = p.splits;
        if (tm) SYMNMF_TRY(tm->begin(s));
        SYMNMF_TRY(launch_stream_tc(p, a.S, a.lds, a.XT, a.ldxt, a.part, a.err, a.st, s, &epi,
                                    a.counters));
        if (tm) SYMNMF_TRY(tm->end(s));
        return SYMNMF_OK;
    }
    const StreamPlan p = plan_stream(d, a.n, a.k, r0, r1);
    if (tm) SYMNMF_TRY(tm->begin(s));
    SYMNMF_TRY(launch_stream_partial(p, a.S, a.lds, Xa, Xb, ldx, a.part, a.st, s));
    if (tm) SYMNMF_TRY(tm->end(s));
    return launch_epilogue(epi.mode, epi.n, epi.k, a.part, p.splits, epi.H, epi.G, epi.Hn, epi.Gn,
                           epi.Psnap, epi.m_scale, epi.lr, epi.eps, epi.tr_part, epi.gram_part,
                           epi.Y, epi.st, s, epi.XT, epi.ldxt);
}

static EpiArgs epi_product(int64_t n, int k, float* Y) {
    EpiArgs e;
    std::memset(&e, 0, sizeof(e));
    e.mode = MODE_PRODUCT;
    e.n = n;
    e.k = k;
    e.Y = Y;
    return e;
}

struct FitCtx {
    Dev d;
    const float* S;
    int64_t n, lds;
    int k;
    const symnmf_fit_params* P;
    FitLayout L;
    float* Hb[2];
    float* Gb[2];
    int cur = 0;
    int iters = 0;     // updates applied along the way to the current iterate
    int epochs = 0;
    cudaStream_t s;
    Timing tm;
    bool h16 = false;  // full-batch passes on the fp16 S-stream
    StreamArgs args() const {
        StreamArgs a;
        a.S = S;
        a.n = n;
        a.lds = lds;
        a.k = k;
        a.part = L.part;
        a.XT = L.XT[cur];
        a.ldxt = L.ldxt;
        a.err = &L.st->kerr;
        a.counters = L.counters;
        a.st = L.st;
        a.upper = P->upper_only != 0;
        a.tpart = L.tpart;
        a.fpart = L.fpart;
        return a;
    }
    // epilogue arguments of a pass that reads Hb[cur] and writes Hb[cur ^ 1]
    EpiArgs epi(int mode, float m_scale, bool write_xt) const {
        EpiArgs e;
        std::memset(&e, 0, sizeof(e));
        e.mode = mode;
        e.n = n;
        e.k = k;
        e.H = Hb[cur];
        e.G = Gb[cur];
        e.Hn = Hb[cur ^ 1];
        e.Gn = Gb[cur ^ 1];
        e.Psnap = L.Psnap;
        e.m_scale = m_scale;
        e.lr = P->lr;
        e.eps = P->eps;
        e.tr_part = L.tr_part;
        e.gram_part = L.gram_part;
        e.st = L.st;
        e.XT = write_xt ? L.XT[cur ^ 1] : nullptr;
        e.ldxt = L.ldxt;
        return e;
    }
};

// One S pass + epilogue + finalise in `mode`, reading Hb[cur], writing Hb[cur^1].
// xt_ready: the split operand of Hb[cur] is already in XT (full-batch loop).
static int full_pass(FitCtx& c, int mode, int max_evals, bool xt_ready) {
    if (c.h16 && mode == MODE_FULL) {
        // fp16 S-stream with the fused epilogue (which reports max |H_{t+1}| per
        // tile instead of writing the TF32 split), the finalise step (which
        // turns those maxima into the next operand's scale), then the fp16
        // operand of H_{t+1}
        const TcPlan p = plan_stream_h16(c.d, c.n, c.k);
        EpiArgs e = c.epi(mode, 0.f, false);
        e.part = c.L.part;
        e.splits = p.splits;
        e.hmax_part = c.L.hmax_part;
        SYMNMF_TRY(c.tm.begin(c.s));
        SYMNMF_TRY(launch_stream_h16(p, c.S, c.lds, c.L.XT16, c.L.part, &c.L.st->kerr, c.L.st, c.s,
                                     &e, c.L.counters));
        SYMNMF_TRY(c.tm.end(c.s));
        SYMNMF_TRY(launch_finalize(mode, epilogue_blocks(c.n), c.k, c.L.tr_part, c.L.gram_part,
                                   c.L.st, c.P->rel_tol, max_evals, c.L.hist, c.L.hist_cap, c.s,
                                   c.L.hmax_part));
        return launch_split16(c.Hb[c.cur ^ 1], c.n, c.k, c.L.st, c.L.XT16, c.s);
    }
    SYMNMF_TRY(stream_pass(c.d, c.args(), c.Hb[c.cur], nullptr, c.k, 0, c.n, xt_ready,
                           c.epi(mode, 0.f, mode == MODE_FULL), c.s, &c.tm));
    return launch_finalize(mode, epilogue_blocks(c.n), c.k, c.L.tr_part, c.L.gram_part, c.L.st,
                           c.P->rel_tol, max_evals, c.L.hist, c.L.hist_cap, c.s);
}

// Replaying the full-batch loop as a CUDA graph is opt-in (SYMNMF_GRAPHS=1):
// each pass's kernels run for tens of microseconds or more, the loop is not
// launch-bound, and eager (programmatically serialised) launches measured as
// fast or faster on B200 (n = 5,000: 4.85 ms per 100 iterations eager, 5.2 ms
// replayed).
static bool use_graphs() {
    static const bool v = [] {   // read once (thread-safe static initialisation)
        const char* e = getenv("SYMNMF_GRAPHS");
        return e != nullptr && std::strcmp(e, "1") == 0;
    }();
    return v;
}

// Replays a captured graph of G full-batch passes on a private stream (ordered
// after the caller's stream) until the device raises the stop flag.  Returns
// SYMNMF_OK with *used = false when the graph could not be built; the caller
// then continues eagerly.
static int run_full_graph(FitCtx& c, int G, int max_evals, HostState* hs, bool* used) {
    *used = false;
    cudaStream_t user = c.s, cs = nullptr;
    cudaEvent_t dep = nullptr;
    cudaGraph_t graph = nullptr;
    cudaGraphExec_t exec = nullptr;
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess ||
        cudaEventCreateWithFlags(&dep, cudaEventDisableTiming) != cudaSuccess) {
        cudaGetLastError();
        if (cs) cudaStreamDestroy(cs);
        return SYMNMF_OK;
    }
    auto cleanup = [&]() {
        if (exec) cudaGraphExecDestroy(exec);
        if (graph) cudaGraphDestroy(graph);
        if (dep) cudaEventDestroy(dep);
        if (cs) cudaStreamDestroy(cs);
        c.s = user;
        c.tm.capturing = false;
    };
    // timing events for the captured passes, allocated before capture
    if (c.tm.on) {
        c.tm.used = 0;
        while ((int)c.tm.ev.size() < 2 * G) {
            cudaEvent_t a;
            if (cudaEventCreate(&a) != cudaSuccess) { cleanup(); return SYMNMF_ERR_CUDA; }
            c.tm.ev.push_back(a);
        }
    }
    const int cur0 = c.cur;
    const int launches_before = launches();   // captured launches are not real ones
    c.s = cs;
    c.tm.capturing = true;
    bool ok = cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) == cudaSuccess;
    for (int p = 0; ok && p < G; ++p) {
        ok = full_pass(c, MODE_FULL, max_evals, true) == SYMNMF_OK;
        c.cur ^= 1;
    }
    const bool ended = cudaStreamEndCapture(cs, &graph) == cudaSuccess;
    c.tm.capturing = false;
    c.cur = cur0;
    const int per_replay = launches() - launches_before;
    reset_launches();
    for (int i = 0; i < launches_before; ++i) note_launch();
    if (!ok || !ended || cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
        cudaGetLastError();
        clear_error();
        cleanup();
        if (c.tm.on) c.tm.used = 0;
        return SYMNMF_OK;
    }
    *used = true;
    SYMNMF_CUDA_TRY(cudaEventRecord(dep, user));
    SYMNMF_CUDA_TRY(cudaStreamWaitEvent(cs, dep, 0));
    int rc = SYMNMF_OK;
    for (;;) {
        const int t_before = hs->t;
        if (cudaGraphLaunch(exec, cs) != cudaSuccess) {
            set_error("cudaGraphLaunch failed: %s", cudaGetErrorString(cudaGetLastError()));
            rc = SYMNMF_ERR_CUDA;
            break;
        }
        for (int i = 0; i < per_replay; ++i) note_launch();
        if ((rc = read_state(c.L.st, hs, cs)) != SYMNMF_OK) break;
        if (c.tm.on && (rc = c.tm.harvest_pairs(std::min(G, hs->t - t_before))) != SYMNMF_OK) break;
        if (hs->done) break;
    }
    // the caller's stream continues after the replays
    if (rc == SYMNMF_OK) {
        if (cudaEventRecord(dep, cs) != cudaSuccess || cudaStreamWaitEvent(user, dep, 0) != cudaSuccess) {
            set_error("stream ordering after the graph failed");
            rc = SYMNMF_ERR_CUDA;
        }
    }
    if (c.tm.on) c.tm.used = 0;
    cleanup();
    return rc;
}

// Full-batch projected AdaGrad until the device-side stop flag is raised.
static int run_full(FitCtx& c, int max_evals, HostState* hs) {
    SYMNMF_TRY(read_state(c.L.st, hs, c.s));
    if (hs->done) return SYMNMF_OK;
    const int t_begin = hs->t;
    const int cur_begin = c.cur;
    const int iters_begin = c.iters;
    const int check = c.P->check_every;
    const int G = std::max(2, (check + 1) / 2 * 2);   // passes per graph: even, so parity returns
    // with rel_tol = 0 the loop cannot stop early (a non-finite loss turns the
    // remaining passes into no-ops on the device), so the host reads the state
    // only after the first pass and after the last
    const int poll = c.P->rel_tol > 0.0 ? check : std::max(check, max_evals);
    bool graphed = false;
    for (int launched = 0;; ++launched) {
        SYMNMF_TRY(full_pass(c, MODE_FULL, max_evals, true));
        c.cur ^= 1;
        const bool last = t_begin + launched + 1 >= max_evals;
        if ((launched + 1) % poll == 0 || last || launched == 0) {
            SYMNMF_TRY(read_state(c.L.st, hs, c.s));
            SYMNMF_TRY(c.tm.harvest());
            if (hs->done) break;
            if (launched + 1 >= max_evals + 2 * check) {   // the device should have stopped by now
                set_error("the full-batch loop did not stop after %d passes", launched + 1);
                return SYMNMF_ERR_CUDA;
            }
            // after the first (eager) pass, replay graphs while enough passes remain
            if (!graphed && use_graphs() && max_evals - hs->t > G) {
                bool used = false;
                SYMNMF_TRY(run_full_graph(c, G, max_evals, hs, &used));
                graphed = true;
                if (used) {
                    if (hs->done) break;
                    // the graph ran an even number of passes: parity is back where it was
                }
            }
        }
    }
    const int steps = hs->t_stop - t_begin;  // updates between the first and the returned evaluation
    c.cur = cur_begin ^ (steps & 1);
    c.iters = iters_begin + steps;
    return SYMNMF_OK;
}

static void epoch_permutation(int64_t m, uint64_t seed, int64_t epoch, std::vector<int64_t>& perm) {
    // Fisher-Yates driven by splitmix64 seeded with seed ^ (epoch+1) * C
    perm.resize(m);
    for (int64_t i = 0; i < m; ++i) perm[i] = i;
    uint64_t state = seed ^ ((uint64_t)(epoch + 1) * 0xD1B54A32D192ED03ull);
    for (int64_t i = m - 1; i >= 1; --i) {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        const int64_t j = (int64_t)(z % (uint64_t)(i + 1));
        std::swap(perm[i], perm[j]);
    }
}

static int run_svrg(FitCtx& c, int max_evals, HostState* hs, int64_t* block_final) {
    const int64_t n = c.n;
    int64_t b = c.P->block_rows > 0 ? std::min<int64_t>(c.P->block_rows, n) : default_block_rows(n);
    bool have_prev = false;
    double L_prev = 0.0;
    std::vector<int64_t> perm;
    for (int e = 0;; ++e) {
        // snapshot: P~ = S H~, f(H~), stopping test on consecutive evaluations
        SYMNMF_TRY(full_pass(c, MODE_SNAPSHOT, max_evals, false));
        SYMNMF_TRY(read_state(c.L.st, hs, c.s));
        SYMNMF_TRY(c.tm.harvest());
        if (hs->nonfinite || hs->converged) break;
        const double L = hs->loss;
        if (have_prev && c.P->grow && b < n && (L_prev - L) / L_prev < c.P->stall_tol)
            b = std::min<int64_t>(2 * b, n);
        if (hs->done) break;  // evaluation budget reached at this snapshot
        if (b >= n) {
            // grown to the full gradient: take the step from the stored P~, then full batch
            SYMNMF_TRY(launch_epilogue(MODE_STEP_SNAP, n, c.k, nullptr, 0, c.Hb[c.cur], c.Gb[c.cur],
                                       c.Hb[c.cur ^ 1], c.Gb[c.cur ^ 1], c.L.Psnap, 0.f, c.P->lr,
                                       c.P->eps, c.L.tr_part, c.L.gram_part, nullptr, c.L.st, c.s,
                                       c.L.XT[c.cur ^ 1], c.L.ldxt));
            SYMNMF_TRY(launch_finalize(MODE_STEP_SNAP, epilogue_blocks(n), c.k, c.L.tr_part,
                                       c.L.gram_part, c.L.st, c.P->rel_tol, max_evals, c.L.hist,
                                       c.L.hist_cap, c.s));
            c.cur ^= 1;
            c.iters += 1;
            SYMNMF_TRY(run_full(c, max_evals, hs));
            break;
        }
        const int64_t m = (n + b - 1) / b;
        epoch_permutation(m, c.P->seed, e, perm);
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(c.L.Hsnap, c.Hb[c.cur], (size_t)n * c.k * sizeof(float),
                                        cudaMemcpyDeviceToDevice, c.s));
        for (int64_t q = 0; q < m; ++q) {
            const int64_t r0 = perm[q] * b, r1 = std::min(n, r0 + b);
            SYMNMF_TRY(stream_pass(c.d, c.args(), c.Hb[c.cur], c.L.Hsnap, c.k, r0, r1, false,
                                   c.epi(MODE_SVRG_INNER, (float)m, false), c.s, &c.tm));
            SYMNMF_TRY(launch_finalize(MODE_SVRG_INNER, epilogue_blocks(n), c.k, c.L.tr_part,
                                       c.L.gram_part, c.L.st, c.P->rel_tol, max_evals, c.L.hist,
                                       c.L.hist_cap, c.s));
            c.cur ^= 1;
        }
        c.epochs += 1;
        have_prev = true;
        L_prev = L;
    }
    *block_final = b;
    return SYMNMF_OK;
}

static int probe_impl(const Dev& d, const float* S, int64_t n, int64_t lds, int n_eig, int b,
                      int max_iter, double tol, uint64_t seed, double* eig_out, void* ws,
                      size_t ws_bytes, cudaStream_t s);

static int fit_impl(const float* S, int64_t n, int64_t lds, int k, const symnmf_fit_params& P,
                    float* H, symnmf_fit_stats* out, void* ws, size_t ws_bytes, cudaStream_t s) {
    FitCtx c;
    reset_launches();
    SYMNMF_TRY(device_info(&c.d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    SYMNMF_TRY(plan_fit(c.d, a, n, k, P, &c.L));
    if (!a.ok()) {
        set_error("workspace too small: %zu bytes given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    c.S = S;
    c.n = n;
    c.lds = lds;
    c.k = k;
    c.P = &P;
    c.s = s;
    c.Hb[0] = H;
    c.Hb[1] = c.L.H1;
    c.Gb[0] = c.L.G0;
    c.Gb[1] = c.L.G1;
    c.tm.on = P.timing != 0;

    // statistics pre-pass into the state head
    SYMNMF_CUDA_TRY(cudaMemsetAsync(c.L.st, 0, fit_state_bytes(), s));
    SYMNMF_TRY(launch_stats(S, n, n, lds, c.L.stats_part, stats_blocks(), &c.L.st->s_sum, s,
                            c.L.amax_part, c.L.st));
    HostState hs;
    SYMNMF_TRY(read_state(c.L.st, &hs, s));
    if (hs.s_bad > 0.0) {
        set_error("S holds %.0f non-finite entries", hs.s_bad);
        return SYMNMF_ERR_NONFINITE;
    }

    int solver = P.solver;
    double gamma = std::numeric_limits<double>::quiet_NaN();
    if (solver == SYMNMF_SOLVER_AUTO) {
        std::vector<double> ev(k + 2);
        if (P.eigvals != nullptr && P.n_eigvals >= k + 2) {
            for (int i = 0; i < k + 2; ++i) ev[i] = P.eigvals[i];
        } else {
            SYMNMF_TRY(probe_impl(c.d, S, n, lds, k + 2, P.probe_block, P.probe_max_iter,
                                  P.probe_tol, P.seed, ev.data(), c.L.probe_ws, c.L.probe_bytes, s));
        }
        const double l1 = ev[k], l2 = ev[k + 1];
        gamma = l2 == 0.0 ? std::numeric_limits<double>::infinity() : l1 / std::fabs(l2);
        solver = gamma >= P.gap_threshold ? SYMNMF_SOLVER_ADAGRAD : SYMNMF_SOLVER_BLOCK_SVRG;
    }

    if (P.init == SYMNMF_INIT_SEEDED) SYMNMF_TRY(launch_init(H, n, k, P.seed, c.L.st, s));
    if (P.G_inout != nullptr)
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(c.L.G0, P.G_inout, (size_t)n * k * sizeof(float),
                                        cudaMemcpyDeviceToDevice, s));
    else
        SYMNMF_CUDA_TRY(cudaMemsetAsync(c.L.G0, 0, (size_t)n * k * sizeof(float), s));
    // Gram of H0 (also writes the split operand of H0; its padding rows stay zero)
    for (int b = 0; b < 2; ++b)
        SYMNMF_CUDA_TRY(cudaMemsetAsync(c.L.XT[b], 0, (size_t)xt_rows(k) * c.L.ldxt * sizeof(float), s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(c.L.counters, 0, (size_t)epilogue_blocks(n) * sizeof(int), s));
    c.h16 = solver == SYMNMF_SOLVER_ADAGRAD && h16_path(n, k, P);
    float* hmax = c.h16 ? c.L.hmax_part : nullptr;
    SYMNMF_TRY(launch_epilogue(MODE_GRAM, n, k, nullptr, 0, H, nullptr, nullptr, nullptr, nullptr,
                               0.f, 0.f, 0.f, c.L.tr_part, c.L.gram_part, nullptr, c.L.st, s,
                               c.L.XT[0], c.L.ldxt, hmax));
    SYMNMF_TRY(launch_finalize(MODE_GRAM, epilogue_blocks(n), k, c.L.tr_part, c.L.gram_part,
                               c.L.st, P.rel_tol, P.max_iters + 1, c.L.hist, c.L.hist_cap, s, hmax));
    if (c.h16) SYMNMF_TRY(launch_split16(H, n, k, c.L.st, c.L.XT16, s));   // the fp16 operand of H0

    cudaEvent_t e0 = nullptr, e1 = nullptr;
    if (c.tm.on) {
        SYMNMF_CUDA_TRY(cudaEventCreate(&e0));
        SYMNMF_CUDA_TRY(cudaEventCreate(&e1));
        SYMNMF_CUDA_TRY(cudaEventRecord(e0, s));
    }
    const int max_evals = P.max_iters + 1;
    int64_t block_final = n;
    if (solver == SYMNMF_SOLVER_ADAGRAD) SYMNMF_TRY(run_full(c, max_evals, &hs));
    else SYMNMF_TRY(run_svrg(c, max_evals, &hs, &block_final));
    double loop_ms = 0.0;
    if (c.tm.on) {
        SYMNMF_CUDA_TRY(cudaEventRecord(e1, s));
        SYMNMF_CUDA_TRY(cudaEventSynchronize(e1));
        float ms = 0.f;
        SYMNMF_CUDA_TRY(cudaEventElapsedTime(&ms, e0, e1));
        loop_ms = ms;
        cudaEventDestroy(e0);
        cudaEventDestroy(e1);
        SYMNMF_TRY(c.tm.harvest());
    }
    SYMNMF_TRY(read_state(c.L.st, &hs, s));

    // the returned iterate must end up in the caller's H
    if (c.Hb[c.cur] != H)
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(H, c.Hb[c.cur], (size_t)n * k * sizeof(float),
                                        cudaMemcpyDeviceToDevice, s));
    if (P.G_inout != nullptr)
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(P.G_inout, c.Gb[c.cur], (size_t)n * k * sizeof(float),
                                        cudaMemcpyDeviceToDevice, s));
    const int evals = std::min(hs.t, c.L.hist_cap);
    if (P.loss_history != nullptr && P.loss_history_len > 0 && evals > 0)
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(P.loss_history, c.L.hist,
                                        sizeof(double) * std::min(evals, P.loss_history_len),
                                        cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    {
        int kerr = 0;
        SYMNMF_CUDA_TRY(cudaMemcpy(&kerr, &c.L.st->kerr, sizeof(int), cudaMemcpyDeviceToHost));
        if (kerr != 0) {
            set_error("an S-stream pipeline wait timed out on the device (code %d)", kerr);
            return SYMNMF_ERR_TIMEOUT;
        }
    }
    if (hs.nonfinite) {
        set_error("the loss became non-finite at evaluation %d", hs.t_stop);
        return SYMNMF_ERR_NONFINITE;
    }
    if (out != nullptr) {
        out->iters = c.iters;
        out->epochs = c.epochs;
        out->converged = hs.converged;
        out->solver_used = solver;
        out->block_final = solver == SYMNMF_SOLVER_ADAGRAD ? n : block_final;
        out->loss = hs.loss;
        out->rel_change = hs.rel;
        out->gamma = gamma;
        out->s_mean = hs.s_sum / ((double)n * (double)n);
        out->s_sqnorm = hs.s_sqnorm;
        out->evaluations = hs.t;
        out->stream_launches = c.tm.launches;
        if (P.stream_ms_out != nullptr && P.stream_ms_len > 0)
            for (int i = 0; i < std::min<int>(P.stream_ms_len, (int)c.tm.each.size()); ++i)
                P.stream_ms_out[i] = c.tm.each[i];
        out->stream_ms = c.tm.ms;
        out->loop_ms = loop_ms;
        out->kernel_launches = launches();
        out->stream_kernel = c.h16 ? SYMNMF_STREAM_FP16
                             : P.upper_only ? SYMNMF_STREAM_UPPER
                             : use_tc() ? SYMNMF_STREAM_TF32 : SYMNMF_STREAM_CUDA_CORE;
    }
    return SYMNMF_OK;
}

// ---------------------------------------------------------------- spectral probe
// Orthonormalise the b columns of V (n x b, leading dimension ldv) in place:
// V_in = V_out B with B b x b.  Directions whose Gram eigenvalue falls below
// 1e-10 of the largest are replaced by fresh seeded random vectors orthogonal
// to the first `nq` columns of Q and to the kept directions (B rows zero).
static int orthonormalize(const ProbeLayout& L, float* V, int64_t n, int64_t ldv, int b,
                          const float* Q, int64_t ldq, int nq, uint64_t seed,
                          std::vector<double>& B, cudaStream_t s);

static int proj_out(const ProbeLayout& L, float* V, int64_t n, int64_t ldv, int b, const float* Q,
                    int64_t ldq, int nq, std::vector<double>* coef, cudaStream_t s) {
    // V -= Q[:, :nq] (Q[:, :nq]^T V); coef (nq x b, fp64) accumulates the coefficients.
    // One V^T W launch covers at most 4096 entries and 32 x (cv + cw) floats of smem (48 KB).
    const int chunk = std::max(1, std::min(4096 / b, 384 - b));
    const int nblk = gemm_tn_blocks(n);
    std::vector<double> C((size_t)nq * b);
    for (int a0 = 0; a0 < nq; a0 += chunk) {
        const int cv = std::min(chunk, nq - a0);
        SYMNMF_TRY(launch_gemm_tn(Q + a0, n, ldq, cv, V, ldv, b, L.C64 + (size_t)a0 * b, L.tn_part,
                                  nblk, s));
    }
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(C.data(), L.C64, C.size() * sizeof(double),
                                    cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    std::vector<float> C32(C.size());
    for (size_t i = 0; i < C.size(); ++i) C32[i] = (float)C[i];
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(L.C32, C32.data(), C32.size() * sizeof(float),
                                    cudaMemcpyHostToDevice, s));
    const int sub_chunk = std::max(1, 12288 / b);
    for (int a0 = 0; a0 < nq; a0 += sub_chunk) {
        const int cv = std::min(sub_chunk, nq - a0);
        SYMNMF_TRY(launch_gemm_nn_sub(V, n, ldv, b, Q + a0, ldq, cv, L.C32 + (size_t)a0 * b, s));
    }
    if (coef != nullptr) {
        coef->resize(C.size(), 0.0);
        for (size_t i = 0; i < C.size(); ++i) (*coef)[i] += C[i];
    }
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));  // C32 host buffer goes out of scope
    return SYMNMF_OK;
}

static int gram_host(const ProbeLayout& L, const float* V, int64_t n, int64_t ldv, int b,
                     std::vector<double>& M, cudaStream_t s) {
    SYMNMF_TRY(launch_gemm_tn(V, n, ldv, b, V, ldv, b, L.C64, L.tn_part, gemm_tn_blocks(n), s));
    M.resize((size_t)b * b);
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(M.data(), L.C64, M.size() * sizeof(double),
                                    cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < i; ++j) {
            const double v = 0.5 * (M[(size_t)i * b + j] + M[(size_t)j * b + i]);
            M[(size_t)i * b + j] = M[(size_t)j * b + i] = v;
        }
    return SYMNMF_OK;
}

static int right_mul(const ProbeLayout& L, float* V, int64_t n, int64_t ldv, int b,
                     const std::vector<double>& F, cudaStream_t s) {
    std::vector<float> F32(F.size());
    for (size_t i = 0; i < F.size(); ++i) F32[i] = (float)F[i];
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(L.M32, F32.data(), F32.size() * sizeof(float),
                                    cudaMemcpyHostToDevice, s));
    SYMNMF_TRY(launch_trsm_right(V, n, ldv, b, L.M32, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    return SYMNMF_OK;
}

// Symmetric orthonormalisation of a full-rank block: V <- V M^{-1/2}, B <- M^{1/2} B.
static int sym_orth(const ProbeLayout& L, float* V, int64_t n, int64_t ldv, int b,
                    std::vector<double>& B, cudaStream_t s, bool* ok) {
    std::vector<double> M, w, U;
    SYMNMF_TRY(gram_host(L, V, n, ldv, b, M, s));
    jacobi_eig(b, M, w, U);
    double wmax = 0.0;
    for (double x : w) wmax = std::max(wmax, x);
    *ok = true;
    for (double x : w)
        if (!(x > 1e-10 * wmax) || wmax <= 0.0) *ok = false;
    if (!*ok) return SYMNMF_OK;
    std::vector<double> F((size_t)b * b, 0.0), Mh((size_t)b * b, 0.0);
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double f = 0.0, h = 0.0;
            for (int q = 0; q < b; ++q) {
                const double u = U[(size_t)i * b + q] * U[(size_t)j * b + q];
                f += u / std::sqrt(w[q]);
                h += u * std::sqrt(w[q]);
            }
            F[(size_t)i * b + j] = f;
            Mh[(size_t)i * b + j] = h;
        }
    SYMNMF_TRY(right_mul(L, V, n, ldv, b, F, s));
    std::vector<double> NB((size_t)b * b, 0.0);
    for (int i = 0; i < b; ++i)
        for (int j = 0; j < b; ++j) {
            double v = 0.0;
            for (int q = 0; q < b; ++q) v += Mh[(size_t)i * b + q] * B[(size_t)q * b + j];
            NB[(size_t)i * b + j] = v;
        }
    B.swap(NB);
    return SYMNMF_OK;
}

static int orthonormalize(const ProbeLayout& L, float* V, int64_t n, int64_t ldv, int b,
                          const float* Q, int64_t ldq, int nq, uint64_t seed,
                          std::vector<double>& B, cudaStream_t s) {
    // B starts as the identity; directions are examined through M = V^T V = U diag(w) U^T
    B.assign((size_t)b * b, 0.0);
    for (int i = 0; i < b; ++i) B[(size_t)i * b + i] = 1.0;
    bool ok = false;
    SYMNMF_TRY(sym_orth(L, V, n, ldv, b, B, s, &ok));
    if (ok) {
        SYMNMF_TRY(sym_orth(L, V, n, ldv, b, B, s, &ok));  // second pass for orthogonality
        if (ok) return SYMNMF_OK;
    }
    // rank-deficient block: keep the strong directions, replace the rest
    std::vector<double> M, w, U;
    SYMNMF_TRY(gram_host(L, V, n, ldv, b, M, s));
    jacobi_eig(b, M, w, U);
    double wmax = 0.0;
    for (double x : w) wmax = std::max(wmax, x);
    std::vector<int> keep;
    for (int q = 0; q < b; ++q)
        if (wmax > 0.0 && w[q] > 1e-10 * wmax) keep.push_back(q);
    const int r = (int)keep.size();
    // F maps V onto [kept orthonormal directions | zeros]; B_new rows for them
    std::vector<double> F((size_t)b * b, 0.0), NB((size_t)b * b, 0.0);
    for (int c2 = 0; c2 < r; ++c2) {
        const int q = keep[c2];
        const double sq = std::sqrt(w[q]);
        for (int i = 0; i < b; ++i) F[(size_t)i * b + c2] = U[(size_t)i * b + q] / sq;
        for (int j = 0; j < b; ++j) {
            double v = 0.0;
            for (int i = 0; i < b; ++i) v += sq * U[(size_t)i * b + q] * B[(size_t)i * b + j];
            NB[(size_t)c2 * b + j] = v;
        }
    }
    SYMNMF_TRY(right_mul(L, V, n, ldv, b, F, s));
    // columns r..b-1 are zero now: fill them with seeded uniform noise, column by column
    if (r < b) {
        // generate on the device into the scratch block, then copy the columns over;
        // V sits at column nq of Q, so Q[:, :nq + r] holds the basis and the kept directions
        SYMNMF_TRY(launch_uniform_fill(L.W, n * (int64_t)b, seed, -0.5f, s));
        SYMNMF_CUDA_TRY(cudaMemcpy2DAsync(V + r, ldv * sizeof(float), L.W + r, b * sizeof(float),
                                          (size_t)(b - r) * sizeof(float), (size_t)n,
                                          cudaMemcpyDeviceToDevice, s));
        if (nq + r > 0)
            for (int pass = 0; pass < 2; ++pass)
                SYMNMF_TRY(proj_out(L, V + r, n, ldv, b - r, Q, ldq, nq + r, nullptr, s));
    }
    B.swap(NB);
    // final symmetric orthonormalisation of the whole block (now full rank)
    SYMNMF_TRY(sym_orth(L, V, n, ldv, b, B, s, &ok));
    if (ok) SYMNMF_TRY(sym_orth(L, V, n, ldv, b, B, s, &ok));
    if (!ok) {
        set_error("spectral probe: could not complete an orthonormal block (n too small?)");
        return SYMNMF_ERR_NOT_SUPPORTED;
    }
    return SYMNMF_OK;
}

// what the last probe on this host thread did (symnmf_probe_last_info)
static thread_local symnmf_probe_info g_probe_info = {0, 0, 0};

static int probe_impl(const Dev& d, const float* S, int64_t n, int64_t lds, int n_eig, int b,
                      int max_iter, double tol, uint64_t seed, double* eig_out, void* ws,
                      size_t ws_bytes, cudaStream_t s) {
    g_probe_info = symnmf_probe_info{0, 0, 0};
    const int launches0 = launches();
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    ProbeLayout L;
    probe_workspace(d, n, b, max_iter, &a, &L);
    if (!a.ok()) {
        set_error("workspace too small for the spectral probe: %zu given, %zu needed", ws_bytes,
                  a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    const int mtot = L.mtot;
    const int64_t ldq = mtot;
    const int steps = mtot / b;  // blocks the basis can hold
    StreamArgs sa;
    sa.S = S;
    sa.n = n;
    sa.lds = lds;
    sa.k = b;
    sa.part = L.part;
    sa.XT = L.XT;
    sa.ldxt = L.ldxt;
    sa.err = L.err;
    sa.counters = L.counters;
    sa.st = nullptr;
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.err, 0, sizeof(int), s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.counters, 0, (size_t)epilogue_blocks(n) * sizeof(int), s));
    std::vector<double> T((size_t)mtot * mtot, 0.0), B, coef, theta, prev;
    // start block: seeded uniform noise, orthonormalised
    SYMNMF_TRY(launch_uniform_fill(L.W, n * (int64_t)b, seed, -0.5f, s));
    SYMNMF_CUDA_TRY(cudaMemcpy2DAsync(L.Q, ldq * sizeof(float), L.W, b * sizeof(float),
                                      (size_t)b * sizeof(float), (size_t)n,
                                      cudaMemcpyDeviceToDevice, s));
    SYMNMF_TRY(orthonormalize(L, L.Q, n, ldq, b, L.Q, ldq, 0, seed + 1, B, s));
    bool converged = false;
    // The Rayleigh-Ritz step costs O(nq^3) on the host and overlaps the next
    // block's S pass.  While it is shorter than a block step it runs every
    // step; when it grows longer (large bases on small matrices), the check
    // is spaced out so that the host work stays within half of the block
    // steps' time.  The last step always computes it (it is the result).
    using clk = std::chrono::steady_clock;
    double rr_ms = 0.0, step_ms = 0.0;
    int next_check = 0;
    auto step_t0 = clk::now();
    // W = S Q_0 (one S pass)
    SYMNMF_TRY(stream_pass(d, sa, L.Q, nullptr, ldq, 0, n, false, epi_product(n, b, L.W), s, nullptr));
    g_probe_info.s_passes = 1;
    for (int j = 0; j < steps; ++j) {
        g_probe_info.block_steps = j + 1;
        // W holds S Q_j: full reorthogonalisation against Q_0..Q_j, twice; the
        // Q_j coefficients are A_j
        const int nq = (j + 1) * b;
        coef.assign((size_t)nq * b, 0.0);
        for (int pass = 0; pass < 2; ++pass)
            SYMNMF_TRY(proj_out(L, L.W, n, b, b, L.Q, ldq, nq, &coef, s));
        for (int r = 0; r < b; ++r)
            for (int c2 = 0; c2 < b; ++c2) {
                const double v = 0.5 * (coef[(size_t)(j * b + r) * b + c2] + coef[(size_t)(j * b + c2) * b + r]);
                T[(size_t)(j * b + r) * mtot + j * b + c2] = v;
            }
        // next block W = Q_{j+1} B_{j+1}, and its S pass goes out before the
        // Rayleigh-Ritz step below, so that the host's eigenvalue work runs
        // while the GPU streams S (one pass is wasted when this block
        // converges)
        const bool more = j + 1 < steps;
        if (more) {
            float* Qn = L.Q + (size_t)(j + 1) * b;
            SYMNMF_CUDA_TRY(cudaMemcpy2DAsync(Qn, ldq * sizeof(float), L.W, b * sizeof(float),
                                              (size_t)b * sizeof(float), (size_t)n,
                                              cudaMemcpyDeviceToDevice, s));
            SYMNMF_TRY(orthonormalize(L, Qn, n, ldq, b, L.Q, ldq, nq, seed + 2 + j, B, s));
            for (int r = 0; r < b; ++r)
                for (int c2 = 0; c2 < b; ++c2) {
                    const double v = B[(size_t)r * b + c2];
                    T[(size_t)((j + 1) * b + r) * mtot + j * b + c2] = v;
                    T[(size_t)(j * b + c2) * mtot + (j + 1) * b + r] = v;
                }
            SYMNMF_TRY(stream_pass(d, sa, Qn, nullptr, ldq, 0, n, false, epi_product(n, b, L.W), s,
                                   nullptr));
            g_probe_info.s_passes += 1;
        }
        // Rayleigh-Ritz on the leading nq x nq block of the block tridiagonal T
        const auto now = clk::now();
        step_ms = std::chrono::duration<double, std::milli>(now - step_t0).count();
        if (nq >= n_eig && (!more || j >= next_check)) {
            const auto r0 = clk::now();
            std::vector<double> sub((size_t)nq * nq);
            for (int r = 0; r < nq; ++r)
                for (int c2 = 0; c2 < nq; ++c2) sub[(size_t)r * nq + c2] = T[(size_t)r * mtot + c2];
            sym_top_eigvals(nq, sub, n_eig, theta);
            if (!prev.empty()) {
                double dmax = 0.0;
                for (int i = 0; i < n_eig; ++i) dmax = std::max(dmax, std::fabs(theta[i] - prev[i]));
                if (dmax <= tol * std::fabs(theta[0])) converged = true;
            }
            prev = theta;
            rr_ms = std::chrono::duration<double, std::milli>(clk::now() - r0).count();
            const int gap = step_ms > 0.0 ? (int)std::ceil(rr_ms / (0.5 * step_ms)) : 1;
            next_check = j + std::max(1, gap);
        }
        step_t0 = clk::now();
        if (converged || !more) break;
    }
    {
        int kerr = 0;
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(&kerr, L.err, sizeof(int), cudaMemcpyDeviceToHost, s));
        SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
        if (kerr != 0) {
            set_error("an S-stream pipeline wait timed out on the device (code %d)", kerr);
            return SYMNMF_ERR_TIMEOUT;
        }
    }
    if (theta.empty()) {
        set_error("spectral probe: basis of %d vectors is smaller than n_eig = %d", mtot, n_eig);
        return SYMNMF_ERR_INVALID_ARG;
    }
    for (int i = 0; i < n_eig; ++i) eig_out[i] = theta[i];
    g_probe_info.kernel_launches = launches() - launches0;
    return SYMNMF_OK;
}

}  // namespace symnmf

// =============================================================================
// extern "C"
// =============================================================================
using namespace symnmf;

// ---------------------------------------------------------------- spherical k-means
struct KmeansLayout {
    double* inv_norm = nullptr;  // 1 / ||S_i||
    float* CT = nullptr;         // centroids as columns (n x k), when the caller gives none
    float* Y = nullptr;          // S C^T, then S M
    float* M = nullptr;          // membership weights
    int32_t* old = nullptr;      // previous labels
    int64_t* idx = nullptr;      // starting rows
    double* colsq = nullptr;     // per-block column sums of squares
    int* count = nullptr;        // labels changed this step
    StreamArgs sa{};
};

static void kmeans_plan(const Dev& d, Arena& a, int64_t n, int k, bool own_centroids,
                        KmeansLayout* L) {
    L->inv_norm = a.take<double>((size_t)n);
    L->CT = own_centroids ? a.take<float>((size_t)n * k) : nullptr;
    L->Y = a.take<float>((size_t)n * k);
    L->M = a.take<float>((size_t)n * k);
    L->old = a.take<int32_t>((size_t)n);
    L->idx = a.take<int64_t>((size_t)k);
    L->colsq = a.take<double>((size_t)km_colsq_blocks(n) * k);
    L->count = a.take<int>(64);
    L->sa.part = a.take<float>(stream_partials(d, n, k, 0, n));
    L->sa.ldxt = xt_ld(n);
    L->sa.XT = a.take<float>((size_t)xt_rows(k) * L->sa.ldxt);
    L->sa.err = a.take<int>(64);
    L->sa.counters = a.take<int>((size_t)epilogue_blocks(n));
}

// The first k entries of a Fisher-Yates shuffle of 0..n-1 taken upwards,
// driven by splitmix64 seeded with seed ^ 0x5851F42D4C957F2D.
static void forgy_rows(int64_t n, int k, uint64_t seed, std::vector<int64_t>& out) {
    std::unordered_map<int64_t, int64_t> perm;  // sparse: only touched positions
    auto at = [&](int64_t q) {
        auto it = perm.find(q);
        return it == perm.end() ? q : it->second;
    };
    uint64_t state = seed ^ 0x5851F42D4C957F2Dull;
    out.resize(k);
    for (int q = 0; q < k; ++q) {
        state += 0x9E3779B97F4A7C15ull;
        uint64_t z = state;
        z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
        z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
        z ^= z >> 31;
        const int64_t j = q + (int64_t)(z % (uint64_t)(n - q));
        const int64_t vq = at(q), vj = at(j);
        perm[q] = vj;
        perm[j] = vq;
        out[q] = vj;
    }
}

static int kmeans_impl(const float* S, int64_t n, int64_t lds, int k, uint64_t seed,
                       int max_iters, int32_t* labels, float* centroids, int* steps_host,
                       int* converged_host, void* ws, size_t ws_bytes, cudaStream_t s) {
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    KmeansLayout L;
    kmeans_plan(d, a, n, k, centroids == nullptr, &L);
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    float* CT = centroids != nullptr ? centroids : L.CT;
    StreamArgs sa = L.sa;
    sa.S = S;
    sa.n = n;
    sa.lds = lds;
    sa.k = k;
    sa.st = nullptr;

    std::vector<int64_t> rows;
    forgy_rows(n, k, seed, rows);
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(L.idx, rows.data(), (size_t)k * sizeof(int64_t),
                                    cudaMemcpyHostToDevice, s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(sa.err, 0, sizeof(int), s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(sa.counters, 0, (size_t)epilogue_blocks(n) * sizeof(int), s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(L.old, 0xFF, (size_t)n * sizeof(int32_t), s));  // no label
    SYMNMF_TRY(launch_rownorm(S, n, lds, L.inv_norm, s));
    SYMNMF_TRY(launch_init_centroids(S, n, lds, k, L.idx, L.inv_norm, CT, s));

    int steps = 0, converged = 0;
    while (steps < max_iters) {
        // assignment: argmax_c of (S C^T)_ic = ||S_i|| <x_i, c_c>
        SYMNMF_TRY(stream_pass(d, sa, CT, nullptr, k, 0, n, false, epi_product(n, k, L.Y), s,
                               nullptr));
        SYMNMF_TRY(launch_labels(L.Y, n, k, labels, s));
        ++steps;
        SYMNMF_CUDA_TRY(cudaMemsetAsync(L.count, 0, sizeof(int), s));
        SYMNMF_TRY(launch_label_change(labels, L.old, n, L.count, s));
        int changed = 0, err = 0;
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(&changed, L.count, sizeof(int), cudaMemcpyDeviceToHost, s));
        SYMNMF_CUDA_TRY(cudaMemcpyAsync(&err, sa.err, sizeof(int), cudaMemcpyDeviceToHost, s));
        SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
        if (err != 0) {
            set_error("a bounded device-side wait of the S-stream gave up (code %d)", err);
            return SYMNMF_ERR_TIMEOUT;
        }
        if (changed == 0) {
            converged = 1;
            break;
        }
        // update: column c of S M is the sum of the normalised member rows
        SYMNMF_TRY(launch_member(labels, L.inv_norm, n, k, L.M, s));
        SYMNMF_TRY(stream_pass(d, sa, L.M, nullptr, k, 0, n, false, epi_product(n, k, L.Y), s,
                               nullptr));
        SYMNMF_TRY(launch_normalize_centroids(L.Y, n, k, L.colsq, CT, s));
    }
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (steps_host) *steps_host = steps;
    if (converged_host) *converged_host = converged;
    return SYMNMF_OK;
}

extern "C" {

void symnmf_fit_params_default(symnmf_fit_params* p) {
    if (p == nullptr) return;
    std::memset(p, 0, sizeof(*p));
    p->solver = SYMNMF_SOLVER_ADAGRAD;
    p->init = SYMNMF_INIT_SEEDED;
    p->seed = 0;
    p->lr = 0.1f;
    p->eps = 1e-10f;
    p->max_iters = 2000;
    p->rel_tol = 1e-5;
    p->block_rows = 0;
    p->grow = 1;
    p->stall_tol = 1e-4;
    p->gap_threshold = 5.0;
    p->upper_only = 0;
    p->G_inout = nullptr;
    p->loss_history = nullptr;
    p->loss_history_len = 0;
    p->eigvals = nullptr;
    p->n_eigvals = 0;
    p->probe_block = 16;
    p->probe_max_iter = 40;
    p->probe_tol = 1e-6;
    p->check_every = 16;
    p->timing = 0;
}

const char* symnmf_status_string(int status) {
    switch (status) {
        case SYMNMF_OK: return "ok";
        case SYMNMF_ERR_INVALID_ARG: return "invalid argument";
        case SYMNMF_ERR_NONFINITE: return "non-finite value";
        case SYMNMF_ERR_WORKSPACE: return "workspace too small";
        case SYMNMF_ERR_CUDA: return "CUDA error";
        case SYMNMF_ERR_TIMEOUT: return "device wait timed out";
        case SYMNMF_ERR_NOT_SUPPORTED: return "not supported";
        default: return "unknown status";
    }
}

const char* symnmf_last_error(void) { return g_last_error.c_str(); }

int symnmf_version(void) { return 100; }

int symnmf_workspace_size(int op, int64_t n, int k, int64_t T, const symnmf_fit_params* params,
                          size_t* bytes) {
    clear_error();
    SYMNMF_CHECK_ARG(bytes != nullptr, "bytes must not be NULL");
    SYMNMF_CHECK_ARG(n >= 1, "n must be >= 1");
    Dev d;  // sizes depend on the SM count of the current device when one is present
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
    symnmf_fit_params P;
    symnmf_fit_params_default(&P);
    if (params != nullptr) P = *params;
    switch (op) {
        case SYMNMF_OP_BUILD_CORR: {
            SYMNMF_CHECK_ARG(T >= 2, "T must be >= 2");
            double *mu, *inv;
            float* Z;
            int64_t ldz;
            corr_plan(a, T, n, &mu, &inv, &Z, &ldz);
            break;
        }
        case SYMNMF_OP_BUILD_TPDM: {
            SYMNMF_CHECK_ARG(T >= 1, "T must be >= 1");
            int32_t *ranks, *days;
            double *phi, *rho;
            float* W;
            int64_t ldw;
            tpdm_plan(a, T, n, (int)T, &ranks, &phi, &rho, &days, &W, &ldw);
            break;
        }
        case SYMNMF_OP_SPECTRAL_PROBE: {
            SYMNMF_CHECK_ARG(P.probe_block >= 1 && P.probe_block <= KMAX, "probe_block in [1, 64]");
            ProbeLayout L;
            probe_workspace(d, n, P.probe_block, P.probe_max_iter, &a, &L);
            break;
        }
        case SYMNMF_OP_FIT: {
            SYMNMF_TRY(check_params(P, n, k));
            FitLayout L;
            plan_fit(d, a, n, k, P, &L);
            break;
        }
        case SYMNMF_OP_SH: {
            SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX, "k must be in [1, 64]");
            a.take<float>(stream_partials(d, n, k, 0, n));
            a.take<float>((size_t)xt_rows(k) * xt_ld(n));
            a.take<int>(64);
            a.take<int>((size_t)epilogue_blocks(n));
            break;
        }
        case SYMNMF_OP_SH_UPPER: {
            SYMNMF_CHECK_ARG(tri_supported(k), "SYMNMF_OP_SH_UPPER supports 1 <= k <= 24");
            const TriPlan tp = plan_stream_tri(d, n, k);
            a.take<float>(tri_tpart_floats(tp));
            a.take<float>(tri_fpart_floats(tp));
            a.take<float>((size_t)xt_rows(k) * xt_ld(n));
            a.take<int>(64);
            break;
        }
        case SYMNMF_OP_STATS:
            a.take<double>((size_t)stats_blocks() * 3);
            break;
        case SYMNMF_OP_ARI:
            *bytes = ari_workspace_bytes();
            return SYMNMF_OK;
        case SYMNMF_OP_ROLLING: {
            SYMNMF_CHECK_ARG(T >= 2, "T (the window) must be >= 2");
            SYMNMF_TRY(check_params(P, n, k));
            return rolling_workspace_bytes(d, n, k, T, P, bytes);
        }
        case SYMNMF_OP_SPHERICAL_KMEANS: {
            SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX, "k must be in [1, 64]");
            KmeansLayout L;
            kmeans_plan(d, a, n, k, true, &L);   // sized for the internal centroid buffer
            break;
        }
        default:
            set_error("unknown op %d", op);
            return SYMNMF_ERR_INVALID_ARG;
    }
    *bytes = a.used + 256;
    return SYMNMF_OK;
}

static int check_ws(void* ws, size_t ws_bytes) {
    SYMNMF_CHECK_ARG(ws != nullptr || ws_bytes == 0, "ws is NULL");
    SYMNMF_CHECK_ARG((reinterpret_cast<uintptr_t>(ws) & 255u) == 0, "ws must be 256-byte aligned");
    return SYMNMF_OK;
}

int symnmf_build_corr(const float* R, int64_t T, int64_t n, int64_t ldr, float* S, int64_t lds,
                      void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_CHECK_ARG(T >= 2, "T = %lld must be >= 2", (long long)T);
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(ldr >= n && ldr % 4 == 0, "ldr must be >= n and a multiple of 4");
    SYMNMF_CHECK_ARG(R != nullptr && aligned16(R), "R must be a non-null 16-byte aligned device pointer");
    SYMNMF_CHECK_ARG(mul_ok(T, ldr), "T * ldr overflows");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    double *mu, *inv;
    float* Z;
    int64_t ldz;
    corr_plan(a, T, n, &mu, &inv, &Z, &ldz);
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    return launch_corr(R, T, n, ldr, S, lds, mu, inv, Z, ldz, (cudaStream_t)stream);
}

int symnmf_build_tpdm(const float* R, int64_t T, int64_t n, int64_t ldr, double tail_frac,
                      int tail_sign, float* S, int64_t lds, void* ws, size_t ws_bytes,
                      symnmf_stream_t stream) {
    clear_error();
    SYMNMF_CHECK_ARG(T >= 1, "T must be >= 1");
    SYMNMF_CHECK_ARG(tail_frac > 0.0 && tail_frac <= 1.0, "tail_frac must be in (0, 1]");
    SYMNMF_CHECK_ARG(tail_sign == 1 || tail_sign == -1, "tail_sign must be +1 or -1");
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(ldr >= n && ldr % 4 == 0, "ldr must be >= n and a multiple of 4");
    SYMNMF_CHECK_ARG(R != nullptr && aligned16(R), "R must be a non-null 16-byte aligned device pointer");
    SYMNMF_CHECK_ARG(mul_ok(T, ldr) && mul_ok(T, n), "T * n overflows");
    SYMNMF_CHECK_ARG(T < (int64_t(1) << 31), "T too large");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    const int N = (int)std::max<int64_t>(1, (int64_t)std::floor(tail_frac * (double)T));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    int32_t *ranks, *days;
    double *phi, *rho;
    float* W;
    int64_t ldw;
    tpdm_plan(a, T, n, N, &ranks, &phi, &rho, &days, &W, &ldw);
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    return launch_tpdm(R, T, n, ldr, N, tail_sign, S, lds, ranks, phi, rho, days, W, ldw,
                       (cudaStream_t)stream);
}

int symnmf_stats(const float* S, int64_t n, int64_t lds, double* out_dev, void* ws,
                 size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(out_dev != nullptr, "out_dev must not be NULL");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    double* part = a.take<double>((size_t)stats_blocks() * 3);
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    return launch_stats(S, n, n, lds, part, stats_blocks(), out_dev, (cudaStream_t)stream);
}

int symnmf_sh(const float* S, int64_t n, int64_t lds, const float* X, int k, float* Y, void* ws,
              size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX, "k = %d must be in [1, 64]", k);
    SYMNMF_CHECK_ARG(X != nullptr && Y != nullptr && aligned4(X) && aligned4(Y), "X and Y must be device pointers");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    StreamArgs sa;
    sa.S = S;
    sa.n = n;
    sa.lds = lds;
    sa.k = k;
    sa.part = a.take<float>(stream_partials(d, n, k, 0, n));
    sa.ldxt = xt_ld(n);
    sa.XT = a.take<float>((size_t)xt_rows(k) * sa.ldxt);
    sa.err = a.take<int>(64);
    sa.counters = a.take<int>((size_t)epilogue_blocks(n));
    sa.st = nullptr;
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    cudaStream_t s = (cudaStream_t)stream;
    SYMNMF_CUDA_TRY(cudaMemsetAsync(sa.err, 0, sizeof(int), s));
    SYMNMF_CUDA_TRY(cudaMemsetAsync(sa.counters, 0, (size_t)epilogue_blocks(n) * sizeof(int), s));
    SYMNMF_TRY(stream_pass(d, sa, X, nullptr, k, 0, n, false, epi_product(n, k, Y), s, nullptr));
    // a bounded device-side wait that gave up is reported in the error word
    int h = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&h, sa.err, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (h != 0) {
        set_error("an S-stream pipeline wait timed out on the device (code %d)", h);
        return SYMNMF_ERR_TIMEOUT;
    }
    return SYMNMF_OK;
}

int symnmf_sh_upper(const float* S, int64_t n, int64_t lds, const float* X, int k, float* Y,
                    void* ws, size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(tri_supported(k), "k = %d must be in [1, 24]", k);
    SYMNMF_CHECK_ARG(X != nullptr && Y != nullptr && aligned4(X) && aligned4(Y), "X and Y must be device pointers");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    Arena a;
    a.base = static_cast<char*>(ws);
    a.cap = ws_bytes;
    const TriPlan tp = plan_stream_tri(d, n, k);
    StreamArgs sa;
    sa.S = S;
    sa.n = n;
    sa.lds = lds;
    sa.k = k;
    sa.part = nullptr;
    sa.tpart = a.take<float>(tri_tpart_floats(tp));
    sa.fpart = a.take<float>(tri_fpart_floats(tp));
    sa.ldxt = xt_ld(n);
    sa.XT = a.take<float>((size_t)xt_rows(k) * sa.ldxt);
    sa.err = a.take<int>(64);
    sa.counters = nullptr;
    sa.st = nullptr;
    sa.upper = true;
    if (!a.ok()) {
        set_error("workspace too small: %zu given, %zu needed", ws_bytes, a.used);
        return SYMNMF_ERR_WORKSPACE;
    }
    cudaStream_t s = (cudaStream_t)stream;
    SYMNMF_CUDA_TRY(cudaMemsetAsync(sa.err, 0, sizeof(int), s));
    SYMNMF_TRY(stream_pass(d, sa, X, nullptr, k, 0, n, false, epi_product(n, k, Y), s, nullptr));
    int h = 0;
    SYMNMF_CUDA_TRY(cudaMemcpyAsync(&h, sa.err, sizeof(int), cudaMemcpyDeviceToHost, s));
    SYMNMF_CUDA_TRY(cudaStreamSynchronize(s));
    if (h != 0) {
        set_error("an S-stream pipeline wait timed out on the device (code %d)", h);
        return SYMNMF_ERR_TIMEOUT;
    }
    return SYMNMF_OK;
}

int symnmf_probe_last_info(symnmf_probe_info* out) {
    clear_error();
    SYMNMF_CHECK_ARG(out != nullptr, "out must not be NULL");
    *out = g_probe_info;
    return SYMNMF_OK;
}

int symnmf_spectral_probe(const float* S, int64_t n, int64_t lds, int n_eig, int block,
                          int max_iter, double tol, uint64_t seed, double* eigvals_host, void* ws,
                          size_t ws_bytes, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(block >= 1 && block <= KMAX, "block = %d must be in [1, 64]", block);
    SYMNMF_CHECK_ARG(n_eig >= 1 && n_eig <= n, "n_eig = %d must be in [1, n]", n_eig);
    SYMNMF_CHECK_ARG(max_iter >= 1, "max_iter must be >= 1");
    SYMNMF_CHECK_ARG(block <= n, "block must be <= n");
    SYMNMF_CHECK_ARG(tol >= 0.0, "tol must be >= 0");
    SYMNMF_CHECK_ARG(eigvals_host != nullptr, "eigvals_host must not be NULL");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    Dev d;
    SYMNMF_TRY(device_info(&d));
    return probe_impl(d, S, n, lds, n_eig, block, max_iter, tol, seed, eigvals_host, ws, ws_bytes,
                      (cudaStream_t)stream);
}

int symnmf_fit(const float* S, int64_t n, int64_t lds, int k, const symnmf_fit_params* params,
               float* H, symnmf_fit_stats* stats_host, void* ws, size_t ws_bytes,
               symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(params != nullptr, "params must not be NULL");
    SYMNMF_TRY(check_params(*params, n, k));
    SYMNMF_CHECK_ARG(H != nullptr && aligned4(H), "H must be a non-null device pointer");
    SYMNMF_CHECK_ARG(mul_ok(n, k), "n * k overflows");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    return fit_impl(S, n, lds, k, *params, H, stats_host, ws, ws_bytes, (cudaStream_t)stream);
}

int symnmf_labels(const float* H, int64_t n, int k, int32_t* labels, symnmf_stream_t stream) {
    clear_error();
    SYMNMF_CHECK_ARG(n >= 1, "n must be >= 1");
    SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX, "k = %d must be in [1, 64]", k);
    SYMNMF_CHECK_ARG(H != nullptr && labels != nullptr, "H and labels must not be NULL");
    SYMNMF_CHECK_ARG(mul_ok(n, k), "n * k overflows");
    Dev d;
    SYMNMF_TRY(device_info(&d));
    return launch_labels(H, n, k, labels, (cudaStream_t)stream);
}

int symnmf_spherical_kmeans(const float* S, int64_t n, int64_t lds, int k, uint64_t seed,
                            int max_iters, int32_t* labels, float* centroids, int* steps_host,
                            int* converged_host, void* ws, size_t ws_bytes,
                            symnmf_stream_t stream) {
    clear_error();
    SYMNMF_TRY(check_S(S, n, lds));
    SYMNMF_CHECK_ARG(k >= 1 && k <= KMAX && k <= n, "k = %d must be in [1, min(64, n)]", k);
    SYMNMF_CHECK_ARG(max_iters >= 1, "max_iters must be >= 1");
    SYMNMF_CHECK_ARG(labels != nullptr, "labels must not be NULL");
    SYMNMF_CHECK_ARG(centroids == nullptr || aligned4(centroids), "centroids must be a device pointer");
    SYMNMF_CHECK_ARG(mul_ok(n, k), "n * k overflows");
    SYMNMF_TRY(check_ws(ws, ws_bytes));
    return kmeans_impl(S, n, lds, k, seed, max_iters, labels, centroids, steps_host,
                       converged_host, ws, ws_bytes, (cudaStream_t)stream);
}

}  // extern "C"
