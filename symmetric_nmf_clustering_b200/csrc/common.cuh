// Internal declarations shared by the libsymnmf translation units.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <string>
#include <utility>

#include "symnmf.h"

namespace symnmf {

__host__ __device__ __forceinline__ int64_t min64(int64_t a, int64_t b) { return a < b ? a : b; }
__host__ __device__ __forceinline__ int64_t max64(int64_t a, int64_t b) { return a > b ? a : b; }

// ---------------------------------------------------------------- errors
void set_error(const char* fmt, ...);
void clear_error();

struct Status {
    int code = SYMNMF_OK;
};

#define SYMNMF_CUDA_TRY(expr)                                                     \
    do {                                                                          \
        cudaError_t e_ = (expr);                                                  \
        if (e_ != cudaSuccess) {                                                  \
            ::symnmf::set_error("%s failed: %s (%s:%d)", #expr,                   \
                                cudaGetErrorString(e_), __FILE__, __LINE__);      \
            return SYMNMF_ERR_CUDA;                                               \
        }                                                                         \
    } while (0)

// Kernels launched by the calling host thread (reset by the entry points).
void note_launch();
int launches();
void reset_launches();

#define SYMNMF_LAUNCH_CHECK()                                                     \
    do {                                                                          \
        ::symnmf::note_launch();                                                  \
        cudaError_t e_ = cudaGetLastError();                                      \
        if (e_ != cudaSuccess) {                                                  \
            ::symnmf::set_error("kernel launch failed: %s (%s:%d)",               \
                                cudaGetErrorString(e_), __FILE__, __LINE__);      \
            return SYMNMF_ERR_CUDA;                                               \
        }                                                                         \
    } while (0)

#define SYMNMF_TRY(expr)                                                          \
    do {                                                                          \
        int s_ = (expr);                                                          \
        if (s_ != SYMNMF_OK) return s_;                                           \
    } while (0)

// ---------------------------------------------------------------- workspace
// A bump allocator over the caller's workspace; every block 256-byte aligned.
struct Arena {
    char* base = nullptr;
    size_t cap = 0;
    size_t used = 0;
    bool dry = false;  // sizing pass: no base pointer
    template <class T>
    T* take(size_t count) {
        size_t off = (used + 255) & ~size_t(255);
        used = off + count * sizeof(T);
        if (dry || used > cap) return nullptr;
        return reinterpret_cast<T*>(base + off);
    }
    bool ok() const { return dry || used <= cap; }
};

// ---------------------------------------------------------------- device state
// Loop state of a fit, kept in the workspace and updated by the finalise kernel.
constexpr int KMAX = 64;
struct FitState {
    double s_sum, s_sqnorm, s_bad;     // statistics pre-pass
    double loss, loss_prev, rel;       // last evaluation
    double a_sqnorm;                   // ||A||_F^2 of the Gram below
    double A64[KMAX * KMAX];           // Gram H^T H of the current iterate (fp64)
    float A32[KMAX * KMAX];            // same, rounded to fp32 for the epilogue
    int t;                             // evaluations done
    int t_stop;                        // evaluation index of the returned iterate
    int done;                          // 1: stop issued (no further work)
    int converged;
    int nonfinite;
    int kerr;                          // device-side error code (bounded wait gave up)
    // fp16 S-stream of the full-batch loop (stream_h16.cu): max|S| over the
    // finite entries, and the power-of-two scales of S and of the current
    // iterate's operand (c |.| < 2^14 for every entry)
    double s_absmax;
    float sscale, xscale;
};

// Epilogue / finalise modes.
enum Mode : int {
    MODE_FULL = 0,        // evaluate f(H_t), full-gradient AdaGrad step, Gram of H_{t+1}
    MODE_SNAPSHOT = 1,    // Block-SVRG snapshot: store P~ = S H, evaluate f(H), no step
    MODE_SVRG_INNER = 2,  // Block-SVRG inner step: P = P~ + m Y, AdaGrad step, Gram
    MODE_GRAM = 3,        // Gram of the given H only
    MODE_PRODUCT = 4,     // store Y = S X
    MODE_STEP_SNAP = 5    // full-gradient step from the stored P~ (no S pass), Gram
};

// ---------------------------------------------------------------- kernels (launchers)
struct Dev {
    int sms = 148;
    int cc_major = 10;
};
int device_info(Dev* d);

// S-stream partial products part[s] = S[J_s, :]^T X[J_s, :] (see stream.cu)
struct StreamPlan {
    int64_t n;        // rows of the output (instruments)
    int k;            // columns of X
    int64_t j0, j1;   // contraction range (rows of S read, by symmetry)
    int splits;       // contraction splits
    int kp;           // padded column count of one pass (8, 16, 24, 32)
    int groups;       // column groups (k > 32)
};
StreamPlan plan_stream(const Dev& d, int64_t n, int k, int64_t j0, int64_t j1);
size_t stream_partial_floats(const StreamPlan& p);
int launch_stream_partial(const StreamPlan& p, const float* S, int64_t lds,
                          const float* Xa, const float* Xb, int64_t ldx, float* part,
                          const FitState* st, cudaStream_t s);
size_t fit_state_bytes();

// Contraction splits of an S-stream pass (stream_tc.cu): the count that
// minimises the pass-time model for `tiles` row tiles of `steps` stages of
// `stage_bytes` of S, `resident` CTAs at a time, `cadence` seconds a stage.
int choose_splits(int64_t tiles, int64_t steps, int64_t resident, double stage_bytes,
                  double cadence);

// Tensor-core S-stream (stream_tc.cu): X enters as its exact TF32 split
// XT = [X_hi; X_lo] stored K-major (2*KP rows of length ldxt, KP = k rounded up to 8).
struct TcPlan {
    int64_t n;        // rows of the output (rows of S read)
    int64_t ncols;    // columns of S (the contraction's extent)
    int k, KP;
    int64_t j0, j1;   // contraction range, j0 a multiple of 32
    int64_t tiles;    // 128-row tiles of the output
    int splits;       // contraction splits
    int64_t jspan;    // columns per split (multiple of 32)
};
TcPlan plan_stream_tc(const Dev& d, int64_t n, int k, int64_t j0, int64_t j1);
// a block of `rows` rows of S (all ncols columns): S[r0 + i, :] X for i < rows
TcPlan plan_stream_tc_rows(const Dev& d, int64_t rows, int64_t ncols, int k);
size_t tc_partial_floats(const TcPlan& p);
struct EpiArgs;
// epi != NULL: the last split CTA of each row tile runs the epilogue in place
// (`counters`: one int per 128-row tile, zero between passes).
int launch_stream_tc(const TcPlan& p, const float* S, int64_t lds, const float* XT, int64_t ldxt,
                     float* part, int* err, const FitState* st, cudaStream_t s,
                     const EpiArgs* epi = nullptr, int* counters = nullptr);
// Upper-triangle S-stream (stream_tri.cu): Y = S X from the tiles S[p, q], p <= q,
// S rounded to TF32; partial slabs in the workspace, reduced by a second kernel.
struct TriPlan {
    int64_t n;
    int k, KP;
    int T;            // 128-row tiles
    int C;            // column tiles per work item
    int items;        // work items (panel x run of column tiles)
    int grid;         // persistent CTAs
    int64_t tslabs;   // transposed partial slabs
};
TriPlan plan_stream_tri(const Dev& d, int64_t n, int k);
size_t tri_tpart_floats(const TriPlan& p);
size_t tri_fpart_floats(const TriPlan& p);
bool tri_supported(int k);
int launch_stream_tri(const TriPlan& p, const float* S, int64_t lds, const float* XT, int64_t ldxt,
                      float* tpart, float* fpart, int* err, const FitState* st, cudaStream_t s);
int launch_tri_reduce(const TriPlan& p, const float* tpart, const float* fpart, float* Y,
                      const FitState* st, cudaStream_t s);

// fp16 S-stream of the full-batch loop (stream_h16.cu): S and X as scaled fp16
// hi/lo pairs (scales st->sscale, st->xscale); its operand XT16 = [X_hi; X_lo]
// is 2 KP rows of h16_ld(n) halves, written by launch_split16 from H and
// st->xscale.  k <= 24, fused epilogue only.
bool h16_supported(int k);
int h16_set_stall(int on);   // test hook: the producer of S issues no loads
int64_t h16_ld(int64_t n);
size_t h16_xt_halves(int64_t n, int k);
int launch_split16(const float* H, int64_t n, int k, const FitState* st, uint16_t* XT16,
                   cudaStream_t s);
TcPlan plan_stream_h16(const Dev& d, int64_t n, int k);
int launch_stream_h16(const TcPlan& p, const float* S, int64_t lds, const uint16_t* XT16,
                      float* part, int* err, const FitState* st, cudaStream_t s,
                      const EpiArgs* epi, int* counters);
int tri_set_stall(int on);

int launch_split(const float* Xa, const float* Xb, int64_t ldx, int k, int64_t r0, int64_t r1,
                 int64_t jlo, int64_t jhi, float* XT, int64_t ldxt, cudaStream_t s);
inline int64_t xt_ld(int64_t n) { return (n + 31) / 32 * 32; }
inline int xt_kp(int k) { return (k + 7) / 8 * 8; }
inline int xt_rows(int k) { return 2 * xt_kp(k); }

int epilogue_blocks(int64_t n);
int launch_epilogue(int mode, int64_t n, int k, const float* part, int splits,
                    const float* H, const float* G, float* Hn, float* Gn,
                    float* Psnap, float m_scale, float lr, float eps,
                    double* tr_part, double* gram_part, float* Y,
                    const FitState* st, cudaStream_t s, float* XT = nullptr,
                    int64_t ldxt = 0, float* hmax_part = nullptr);
// hmax_part (FULL / GRAM passes of the fp16 stream): per-tile max |H_{t+1}|,
// reduced into st->xscale
int launch_finalize(int mode, int nblk, int k, const double* tr_part,
                    const double* gram_part, FitState* st, double rel_tol,
                    int max_evals, double* history, int history_cap,
                    cudaStream_t s, const float* hmax_part = nullptr);

// amax_part (stats_blocks() floats) and st: optional; with both, max|S| over
// the finite entries goes to st->s_absmax and its power-of-two scale to st->sscale
int launch_stats(const float* S, int64_t rows, int64_t n, int64_t lds, double* part, int nblk,
                 double* out3, cudaStream_t s, float* amax_part = nullptr, FitState* st = nullptr);
// 2^(14 - e) for m < 2^e (m > 0 finite), at most 2^63; 1 otherwise: c m < 2^14.
// The cap keeps 1/c a normal float (the fp16 stream scales its products back
// by 1/cS and 1/cX); it only matters for m below 2^-49, where c m still lands
// in fp16's normal range for every entry above 2^-77 m.
__host__ __device__ inline float pow2_scale_below_2_14(double m) {
    if (!(m > 0.0) || !(m <= 1.7976931348623157e308)) return 1.f;
    int e = 0;
    (void)frexp(m, &e);                 // m = f 2^e, f in [0.5, 1)
    const int sh = 14 - e > 63 ? 63 : 14 - e;
    return ldexpf(1.f, sh);
}
int stats_blocks();
int launch_init_sum(float* H, int64_t n, int k, uint64_t seed, double s_sum, cudaStream_t s);
int launch_init(float* H, int64_t n, int k, uint64_t seed, const FitState* st,
                cudaStream_t s);
int launch_labels(const float* H, int64_t n, int k, int32_t* labels, cudaStream_t s);
// rolling windows (rolling.cu)
size_t ari_workspace_bytes();
int rolling_workspace_bytes(const Dev& d, int64_t n, int k, int64_t T, const symnmf_fit_params& P,
                            size_t* bytes);
// spherical k-means pieces (kmeans.cu)
int km_colsq_blocks(int64_t n);
int launch_rownorm(const float* S, int64_t n, int64_t lds, double* inv_norm, cudaStream_t s);
int launch_init_centroids(const float* S, int64_t n, int64_t lds, int k, const int64_t* idx,
                          const double* inv_norm, float* CT, cudaStream_t s);
int launch_member(const int32_t* lab, const double* inv_norm, int64_t n, int k, float* X,
                  cudaStream_t s);
int launch_normalize_centroids(const float* Z, int64_t n, int k, double* part, float* CT,
                               cudaStream_t s);
int launch_label_change(const int32_t* lab, int32_t* old, int64_t n, int* count, cudaStream_t s);

// builders
// Tensor-core Gram (gram_tc.cu) of the K-major operand planes F (hi parts) and
// L (remainders), n_pad x Kp each.  |corr| (corr = true): fp16 planes holding
// z * CORR_F16_SCALE, Kp a multiple of 64; TPDM: fp32 planes (TF32 split), Kp a
// multiple of 32.  err: one device int, zero on entry.
constexpr float CORR_F16_SCALE = 16384.f;   // 2^14: |z| <= 1 stays far below the fp16 maximum
int launch_gram_tc(const void* F, const void* L, int64_t n, int64_t n_pad, int64_t Kp,
                   bool corr, float scale, float* S, int64_t lds, int* err, cudaStream_t s);
int corr_plan(Arena& a, int64_t T, int64_t n, double** mu, double** inv, float** Z,
              int64_t* ldz);
int launch_corr(const float* R, int64_t T, int64_t n, int64_t ldr, float* S,
                int64_t lds, double* mu, double* inv, float* Z, int64_t ldz,
                cudaStream_t s);
int tpdm_plan(Arena& a, int64_t T, int64_t n, int N, int32_t** ranks, double** phi,
              double** rho, int32_t** days, float** W, int64_t* ldw);
int launch_tpdm(const float* R, int64_t T, int64_t n, int64_t ldr, int N,
                int tail_sign, float* S, int64_t lds, int32_t* ranks, double* phi,
                double* rho, int32_t* days, float* W, int64_t ldw, cudaStream_t s);

// small dense helpers for the spectral probe
int launch_uniform_fill(float* X, int64_t count, uint64_t seed, float offset,
                        cudaStream_t s);
int launch_gemm_tn(const float* V, int64_t n, int64_t ldv, int cv, const float* W,
                   int64_t ldw, int cw, double* C, double* part, int nblk,
                   cudaStream_t s);
int gemm_tn_blocks(int64_t n);
int launch_gemm_nn_sub(float* W, int64_t n, int64_t ldw, int cw, const float* V,
                       int64_t ldv, int cv, const float* C, cudaStream_t s);
int launch_trsm_right(float* W, int64_t n, int64_t ldw, int cw, const float* Rinv,
                      cudaStream_t s);

// Programmatic dependent launch.  A kernel launched with programmatic stream
// serialization may start before the previous kernel in its stream has
// finished; it calls pdl_wait() before it reads anything that kernel wrote
// (a no-op when it was launched the ordinary way).  pdl_trigger() lets the
// next such kernel be scheduled once every CTA of this grid has triggered or
// exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Launches kern<<<grid, block, smem, s>>>(args...) with programmatic stream
// serialization.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace symnmf
