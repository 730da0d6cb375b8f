/*
 * symnmf.h -- C ABI of libsymnmf.so, the B200 (sm_100a) SymNMF clustering path.
 *
 * The method (sources cited by page title and section):
 *   [CaS] "GPU-Accelerated Clustering for Financial Instruments at Scale",
 *         NVIDIA technical blog: sections "Factorization at scale",
 *         "Choosing the rank k", "Factorizing with SymNMF", "Why this solver",
 *         "Tracking stability through time with the Rand index".
 *   [SMI] "GPU-Accelerated SymNMF Clustering Scales to a Million Financial
 *         Instruments" (English copy of the same post): AdaGrad update in
 *         LaTeX form and the AdaptGrow algorithm sketch.
 *   [LRD] abstract of "Low-Rank Dependence Decomposition via Accelerated
 *         Symmetric Non-negative Matrix Factorization": trace identity,
 *         Block-SVRG AdaptGrow.
 *
 * A dependence matrix S (n x n, |Pearson correlation| or TPDM of a T x n
 * returns window) is factorised as S ~ H H^T with H >= 0 (n x k) by
 * projected diagonal AdaGrad on f(H) = ||S||^2 - 2 tr(H^T S H) + ||H^T H||^2,
 * one pass over S per full-batch iteration; the row-wise argmax of H is the
 * hard cluster label.
 *
 * Conventions shared by every entry point
 *  - Pointers named S, R, H, G, X, Y, labels and ws are DEVICE pointers on the
 *    current CUDA device; pointers documented as "host" are host memory.
 *  - All matrices are row-major.  S is n x n with leading dimension lds >= n
 *    and FULL symmetric storage (both triangles hold the values; the library
 *    may read either one).  R is T x n (row = day) with leading dimension
 *    ldr >= n.  H, G, X, Y are n x k dense (leading dimension k).
 *  - Alignment: S and R must be 16-byte aligned and lds, ldr multiples of 4
 *    (16-byte rows), else SYMNMF_ERR_INVALID_ARG.  H, G, X, Y need 4-byte
 *    alignment.
 *  - Ownership: the caller allocates and frees everything.  The library
 *    allocates no device memory: entry points that need scratch take a
 *    caller-provided workspace `ws` of `ws_bytes` bytes (256-byte aligned),
 *    sized by symnmf_workspace_size(); too small gives SYMNMF_ERR_WORKSPACE.
 *  - Streams: work is issued on `stream` (NULL = the legacy default stream).
 *    symnmf_stats and symnmf_labels are asynchronous.  The tensor-core builders,
 *    symnmf_sh and symnmf_sh_noalloc synchronise `stream` at the end to read
 *    their device error word (SYMNMF_ERR_TIMEOUT when a bounded wait gave up).
 *    symnmf_fit and symnmf_spectral_probe write host outputs and synchronise
 *    `stream` before they return.
 *  - Errors: every call returns a symnmf_status; SYMNMF_OK = 0.  A failing
 *    call leaves a description in symnmf_last_error() (per host thread).
 *    Not converging within the budget is SYMNMF_OK with stats.converged = 0.
 *    Sizes: 1 <= n, n*lds and T*ldr below 2^62; 1 <= k <= 64.
 */
#ifndef SYMNMF_H
#define SYMNMF_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define SYMNMF_API __attribute__((visibility("default")))
#else
#define SYMNMF_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* symnmf_stream_t;

typedef enum {
    SYMNMF_OK = 0,
    SYMNMF_ERR_INVALID_ARG = 1,   /* bad size, pointer, alignment or parameter */
    SYMNMF_ERR_NONFINITE = 2,     /* S holds NaN/Inf, or the loss became non-finite */
    SYMNMF_ERR_WORKSPACE = 3,     /* ws_bytes smaller than symnmf_workspace_size() */
    SYMNMF_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
    SYMNMF_ERR_TIMEOUT = 5,       /* a bounded device-side wait gave up */
    SYMNMF_ERR_NOT_SUPPORTED = 6  /* no sm_100 device, or option not available */
} symnmf_status;

enum { SYMNMF_SOLVER_ADAGRAD = 0, SYMNMF_SOLVER_BLOCK_SVRG = 1, SYMNMF_SOLVER_AUTO = 2 };
enum { SYMNMF_INIT_SEEDED = 0, SYMNMF_INIT_USER = 1 };
enum {
    SYMNMF_OP_BUILD_CORR = 0,
    SYMNMF_OP_BUILD_TPDM = 1,
    SYMNMF_OP_SPECTRAL_PROBE = 2,
    SYMNMF_OP_FIT = 3,
    SYMNMF_OP_SH = 4,
    SYMNMF_OP_STATS = 5,
    SYMNMF_OP_SPHERICAL_KMEANS = 6,
    SYMNMF_OP_ARI = 7,
    SYMNMF_OP_ROLLING = 8,
    SYMNMF_OP_SH_UPPER = 9
};
enum { SYMNMF_KIND_CORR = 1, SYMNMF_KIND_TPDM = 2 };

/*
 * Parameters of symnmf_fit ([SMI] AdaptGrow sketch: adaptgrow(S, k, lr, phi,
 * steps, eps)).  Fill with symnmf_fit_params_default() and override.
 */
typedef struct {
    int solver;              /* SYMNMF_SOLVER_*; default ADAGRAD */
    int init;                /* SYMNMF_INIT_SEEDED (H0 = scale-matched seeded draw) or _USER (H holds H0) */
    uint64_t seed;           /* init stream seed and Block-SVRG permutation seed; default 0 */
    float lr;                /* AdaGrad step eta; default 0.1 */
    float eps;               /* AdaGrad epsilon (outside the root); default 1e-10 */
    int max_iters;           /* full-batch updates (ADAGRAD) or epochs (BLOCK_SVRG); default 2000 */
    double rel_tol;          /* stop when |f_t - f_{t-1}| / f_{t-1} < rel_tol; 0 = off; default 1e-5 */
    int64_t block_rows;      /* Block-SVRG block b; 0 = power of two nearest n/10 */
    int grow;                /* AdaptGrow: double b when an epoch stalls; default 1 */
    double stall_tol;        /* stall = relative snapshot-loss decrease below this; default 1e-4 */
    double gap_threshold;    /* AUTO: gamma_{k+1} >= this selects full batch; default 5.0 */
    int upper_only;          /* 1: full-batch passes and Block-SVRG snapshots read only the tiles on or
                                above the diagonal of S (symnmf_sh_upper; k <= 24, S rounded to TF32 in
                                the product); Block-SVRG block steps read their slab as usual. Default 0 */
    float* G_inout;          /* optional device n*k: AdaGrad accumulator in (resume) and out; NULL = start at 0 */
    double* loss_history;    /* optional host array: f(H_t) of every evaluation (snapshots for Block-SVRG) */
    int loss_history_len;    /* capacity of loss_history */
    const double* eigvals;   /* optional host, descending: AUTO uses these instead of running the probe */
    int n_eigvals;           /* length of eigvals (>= k+2 to be used) */
    int probe_block;         /* AUTO probe block size; default 16 */
    int probe_max_iter;      /* AUTO probe Lanczos block steps; default 40 */
    double probe_tol;        /* AUTO probe Ritz tolerance; default 1e-6 */
    int check_every;         /* host reads the stop flag every this many iterations; default 16 */
    int timing;              /* 1 = record CUDA-event time of the S-stream kernels in stats */
    double* stream_ms_out;   /* optional host array: with timing = 1, the CUDA-event time (ms) of each
                                S-stream launch, in launch order (at most stream_ms_len entries) */
    int stream_ms_len;       /* capacity of stream_ms_out */
} symnmf_fit_params;

typedef struct {
    int iters;               /* full-batch updates applied to reach the returned H */
    int epochs;              /* Block-SVRG epochs run */
    int converged;           /* 1 when rel_tol stopped the run */
    int solver_used;         /* SYMNMF_SOLVER_ADAGRAD or _BLOCK_SVRG (possibly grown to full batch) */
    int64_t block_final;     /* Block-SVRG block at exit (n when grown to full batch) */
    double loss;             /* f(H) of the returned H (trace identity, fp64) */
    double rel_change;       /* last relative loss change */
    double gamma;            /* post-rank gap ratio (AUTO), else NaN */
    double s_mean;           /* sum(S) / n^2 */
    double s_sqnorm;         /* ||S||_F^2 */
    int evaluations;         /* passes over S that evaluated the loss (loss_history entries written) */
    int stream_launches;     /* with timing = 1: S-stream kernel launches timed */
    double stream_ms;        /* with timing = 1: their summed CUDA-event time, ms */
    double loop_ms;          /* with timing = 1: CUDA-event time of the iteration loop, ms */
    int kernel_launches;     /* kernels this call launched */
    int stream_kernel;       /* S-stream of the full-batch passes: SYMNMF_STREAM_* */
} symnmf_fit_stats;

/* Which S-stream ran the full-batch passes of a fit (symnmf_fit_stats.stream_kernel):
 * TF32: the tensor-core stream with S and X as exact TF32 splits (the default
 *       below n = 20,000, for k > 24, and for Block-SVRG);
 * FP16: the tensor-core stream with S and X as power-of-two scaled fp16 hi/lo
 *       pairs (the AdaGrad solver from n = 20,000 up, k <= 24; the environment
 *       variable SYMNMF_H16_MIN_N moves the threshold, 0 turns it off);
 * UPPER: the upper-triangle stream (upper_only = 1);
 * CUDA_CORE: the CUDA-core stream (SYMNMF_STREAM=cuda_core). */
enum {
    SYMNMF_STREAM_TF32 = 0,
    SYMNMF_STREAM_FP16 = 1,
    SYMNMF_STREAM_UPPER = 2,
    SYMNMF_STREAM_CUDA_CORE = 3
};

/* Defaults listed in symnmf_fit_params. */
SYMNMF_API void symnmf_fit_params_default(symnmf_fit_params* params);

/* Static string for a status code. */
SYMNMF_API const char* symnmf_status_string(int status);

/* Detail of the last failing call on this host thread ("" if none). */
SYMNMF_API const char* symnmf_last_error(void);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
SYMNMF_API int symnmf_version(void);

/*
 * Workspace bytes needed by `op` (SYMNMF_OP_*) for the given sizes.
 * k: rank (FIT, SH) or n_eig (SPECTRAL_PROBE); T: days (builders);
 * params: FIT options (may be NULL = defaults) -- for SPECTRAL_PROBE only
 * probe_block and probe_max_iter are read.  Writes *bytes.
 */
SYMNMF_API int symnmf_workspace_size(int op, int64_t n, int k, int64_t T,
                          const symnmf_fit_params* params, size_t* bytes);

/*
 * S = |corr(R)|: absolute Pearson correlation of the n columns of the T x n
 * returns window R ([CaS] "Tracking stability through time...": correlation
 * captures co-movement over the body of the distribution).
 * S_ij = |sum_t z_ti z_tj| / sqrt(sum_t z_ti^2 sum_t z_tj^2) with z the
 * column-centred returns; S_ii = 1; a zero-variance column gives a zero row
 * and column apart from S_ii = 1.  Column means and norms in fp64.
 * Requires T >= 2.  Synchronises `stream` (reads the device error word).
 */
SYMNMF_API int symnmf_build_corr(const float* R, int64_t T, int64_t n, int64_t ldr,
                      float* S, int64_t lds, void* ws, size_t ws_bytes,
                      symnmf_stream_t stream);

/*
 * S = TPDM(R): tail pairwise dependence matrix ([CaS] "Tracking stability
 * through time...": co-movement conditional on extreme events).
 *   r_ti  = rank of tail_sign*R_ti within column i (1..T; ties -> earlier day)
 *   x_ti  = (-ln(r_ti/(T+1)))^(-1/2)         (Frechet, alpha = 2, fp64)
 *   rho_t = ||x_t||_2                         (fp64)
 *   E     = the N = max(1, floor(tail_frac*T)) days of largest rho (ties -> earlier day)
 *   S_ij  = (n/N) sum_{t in E} (x_ti/rho_t)(x_tj/rho_t)
 * tail_frac in (0, 1]; tail_sign = +1 or -1.  R must be finite.  Synchronises
 * `stream` (reads the device error word).
 */
SYMNMF_API int symnmf_build_tpdm(const float* R, int64_t T, int64_t n, int64_t ldr,
                      double tail_frac, int tail_sign, float* S, int64_t lds,
                      void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Statistics pre-pass: out_dev[0] = sum S_ij, out_dev[1] = ||S||_F^2 (fp64,
 * non-finite entries skipped), out_dev[2] = count of non-finite entries (as a
 * double).  out_dev is a device array of 3 doubles.  Asynchronous.
 * ([CaS] "Factorization at scale": ||S||^2 is the constant of the trace loss.)
 */
SYMNMF_API int symnmf_stats(const float* S, int64_t n, int64_t lds, double* out_dev,
                 void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Y = S X: one pass of the S-stream ([CaS] "Factorization at scale": the
 * dominant S H products) for X, Y n x k (1 <= k <= 64).  Synchronises `stream`
 * (reads the device error word).
 */
SYMNMF_API int symnmf_sh(const float* S, int64_t n, int64_t lds, const float* X, int k,
              float* Y, void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Y = S X like symnmf_sh, reading only the 128 x 128 tiles of S on or above
 * the diagonal and using symmetry for the rest: half of the n^2 entries.  The
 * scope of this hot path allows the S-stream to read only the upper triangle
 * and exploit symmetry; the pages stream the full matrix ([CaS]
 * "Factorization at scale").  Each tile S[p, q], p <= q, feeds Y_p += S[p, q] X_q
 * and, for p < q, Y_q += S[p, q]^T X_p; partial sums are reduced in a fixed
 * order (bitwise reproducible).  The entries below the diagonal tiles are
 * never read, so S must be symmetric there.
 *
 * Precision: X enters as its exact TF32 split (as in symnmf_sh); S enters
 * rounded to the nearest TF32 value, an unbiased per-entry error of at most
 * 2^-12 relative that averages out along a row (a few 1e-6 relative in Y on
 * the |corr| and TPDM workloads); a matrix whose entries all round in the same
 * direction sees up to 2^-12.  1 <= k <= 24.  Workspace: SYMNMF_OP_SH_UPPER
 * (partial slabs, about (n^2 / 256 + n * items) * 4 k bytes: 1.2 GB at
 * n = 100,000, k = 24).  Synchronises `stream` (reads the device error word).
 */
SYMNMF_API int symnmf_sh_upper(const float* S, int64_t n, int64_t lds, const float* X, int k,
                               float* Y, void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Leading eigenvalues of S by block Lanczos with full reorthogonalisation on
 * the S-stream ([CaS] "Choosing the rank k": inspect the leading eigenvalues
 * and pick k at the clearest gap; "Why this solver": gamma_{k+1}).
 * Writes the n_eig algebraically largest Ritz values, descending, into the
 * host array eigvals_host.  block (1..64) vectors per step, at most max_iter
 * block steps (basis <= block*max_iter <= n); stops when no wanted Ritz value
 * moved by more than tol * |theta_1| between two consecutive block steps.
 * The next block's S pass is issued before the host's Rayleigh-Ritz step (a
 * converging step leaves one pass unused).  Start block from the splitmix64
 * counter stream of `seed`.  Synchronises `stream`.
 */
SYMNMF_API int symnmf_spectral_probe(const float* S, int64_t n, int64_t lds, int n_eig,
                          int block, int max_iter, double tol, uint64_t seed,
                          double* eigvals_host, void* ws, size_t ws_bytes,
                          symnmf_stream_t stream);

/*
 * Row-sharded fit, per-rank pieces ([CaS] "Factorization at scale" and
 * "Scale-out": S sharded by rows across GPUs, H replicated, the S H products
 * local, O(n k) exchanged per iteration).  Rank p holds rows [row0, row0 + rows)
 * of S (rows x n, row pitch lds, a multiple of 4, 16-byte aligned) and the
 * whole current iterate H (n x k).  The caller runs the loop and the
 * collectives (symmetric_nmf_clustering_b200.sharded does it over
 * torch.distributed); these calls never wait on another rank.
 *
 * symnmf_stats_rows: out_dev[0..2] = (sum, squared norm, non-finite count) of
 *   the block, fp64, as symnmf_stats; summed over the ranks they are those of
 *   S.  Workspace: symnmf_workspace_size(SYMNMF_OP_STATS, ...).
 *   Asynchronous.
 * symnmf_seeded_init: H (n x k) = the scale-matched seeded start of
 *   symnmf_fit (INIT_SEEDED) for a matrix whose entries sum to s_sum.
 *   Every rank draws the same H.  Asynchronous.
 * symnmf_gram: A_dev (k x k, device, fp64) = H^T H over `rows` rows of H, a
 *   fixed-order sum (bitwise reproducible).  Workspace: (rows/128 + 1) *
 *   (k^2 + 1) doubles, rounded up.  Asynchronous.
 * symnmf_shard_step: one full-batch iteration restricted to the block, with
 *   A_dev = H^T H of the current iterate (the sum of every rank's Gram):
 *   P = S[rows, :] H; the rows of the projected AdaGrad step of symnmf_fit
 *   ([CaS] "Factorizing with SymNMF") go to H_rows_next and G_rows_next
 *   (rows x k each; G_rows is the accumulator of those rows before the step);
 *   partial_dev (k^2 + 1 doubles, device) = (Gram of the new rows, then
 *   sum_{i in rows} H_i . P_i).  Summed over the ranks, partial_dev gives the
 *   next Gram and tr(H^T S H), and f(H) = ||S||^2 - 2 tr + ||A||_F^2.  Reads
 *   the whole of H (its split operand); H_rows_next must not alias H.
 *   Workspace: symnmf_shard_workspace_size(rows, n, k).  Synchronises `stream`
 *   (reads the device error word: SYMNMF_ERR_TIMEOUT when a bounded wait gave up).
 */
SYMNMF_API int symnmf_stats_rows(const float* S, int64_t rows, int64_t n, int64_t lds,
                                 double* out_dev, void* ws, size_t ws_bytes,
                                 symnmf_stream_t stream);
SYMNMF_API int symnmf_seeded_init(float* H, int64_t n, int k, uint64_t seed, double s_sum,
                                  symnmf_stream_t stream);
SYMNMF_API int symnmf_gram(const float* H, int64_t rows, int k, double* A_dev, void* ws,
                           size_t ws_bytes, symnmf_stream_t stream);
SYMNMF_API int symnmf_shard_workspace_size(int64_t rows, int64_t n, int k, size_t* bytes);
SYMNMF_API int symnmf_shard_step(const float* S_rows, int64_t rows, int64_t n, int64_t lds,
                                 int64_t row0, int k, const float* H, const double* A_dev,
                                 const float* G_rows, float lr, float eps, float* H_rows_next,
                                 float* G_rows_next, double* partial_dev, void* ws,
                                 size_t ws_bytes, symnmf_stream_t stream);

/*
 * What the last symnmf_spectral_probe call on this host thread did: the
 * number of passes over S it launched (each reads the n x n matrix once,
 * with a block-wide operand) and the kernels it launched in all.  Lets a
 * caller put the probe's time on the HBM roofline (bytes = s_passes * 4 n^2).
 * Zeros before the first call.  Returns SYMNMF_OK, or SYMNMF_ERR_INVALID_ARG
 * for a NULL out.
 */
typedef struct {
    int s_passes;           /* S-stream passes (one per Krylov block, plus the start) */
    int block_steps;        /* Lanczos block steps taken */
    int kernel_launches;    /* kernels launched by the call */
} symnmf_probe_info;
SYMNMF_API int symnmf_probe_last_info(symnmf_probe_info* out);

/*
 * Factorise S ~ H H^T, H >= 0 ([SMI] AdaptGrow sketch; [CaS] "Factorizing
 * with SymNMF": G <- G + g*g, H <- max(H - lr g/(sqrt(G)+eps), 0)).
 *   ADAGRAD:    g = 4 (H (H^T H) - S H), one S pass per iteration; the pass
 *               that forms S H_t also evaluates f(H_t) and takes the update.
 *               Evaluation t = 0..max_iters; stops at the first t > 0 with
 *               relative loss change < rel_tol, or at t = max_iters, and
 *               returns H_t.
 *   BLOCK_SVRG: per epoch a snapshot pass (S H~, f(H~)), then one SVRG step
 *               per row block of b rows in a seeded order,
 *               g = 4 (H H^T H - S H~ - m S[:,B] (H_B - H~_B)), m = ceil(n/b);
 *               stalled epochs double b; at b = n it continues as ADAGRAD.
 *   AUTO:       gamma_{k+1} = lambda_{k+1}/|lambda_{k+2}| >= gap_threshold
 *               selects ADAGRAD, else BLOCK_SVRG.
 * H (n x k, device): output; with INIT_USER also the input H0.
 * stats_host may be NULL.  Synchronises `stream`.
 */
SYMNMF_API int symnmf_fit(const float* S, int64_t n, int64_t lds, int k,
               const symnmf_fit_params* params, float* H,
               symnmf_fit_stats* stats_host, void* ws, size_t ws_bytes,
               symnmf_stream_t stream);

/*
 * labels[i] = argmax_j H_ij, lowest j on ties ([CaS] "Factorizing with
 * SymNMF": the row-wise argmax is the hard cluster label).  H n x k, labels
 * n int32 (device).  Needs no workspace.  Asynchronous.
 */
SYMNMF_API int symnmf_labels(const float* H, int64_t n, int k, int32_t* labels,
                  symnmf_stream_t stream);

/*
 * Spherical k-means on the L2-normalised rows x_i = S_i / ||S_i|| of S, the
 * hard-label baseline of [CaS] "Spherical k-means for direct hard
 * clustering" (cosine similarity; a zero row stays zero).
 *   start:   centroid c = x_{r_c}, r_0..r_{k-1} the first k entries of a
 *            Fisher-Yates shuffle of 0..n-1 taken upwards (position q swaps
 *            with q + (z_q mod (n - q))), z_q the q-th splitmix64 output
 *            seeded with seed XOR 0x5851F42D4C957F2D;
 *   assign:  l_i = argmax_c <x_i, c_c>, lowest c on ties (one S pass:
 *            S C^T, whose row i is ||S_i|| times the cosine scores);
 *   stop:    when no label changed, or after max_iters assignment steps;
 *   update:  c_c = sum_{l_i = c} x_i / ||.||; an empty cluster keeps its
 *            centroid (one S pass: S M, M_ic = [l_i = c] / ||S_i||, by the
 *            symmetry of S).
 * S: n x n symmetric, 1 <= k <= min(64, n).  labels: n int32 (device), the
 * last assignment.  centroids: n x k row-major fp32 (device; column c is
 * centroid c) or NULL.  steps_host / converged_host (may be NULL): assignment
 * steps taken and whether the labels stopped changing.  Synchronises `stream`
 * once per step (to read the change count).
 */
SYMNMF_API int symnmf_spherical_kmeans(const float* S, int64_t n, int64_t lds, int k,
                                       uint64_t seed, int max_iters, int32_t* labels,
                                       float* centroids, int* steps_host, int* converged_host,
                                       void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Adjusted Rand index of two labelings ([CaS] "The metric": pair agreement
 * corrected for chance; Hubert & Arabie).  a, b: n int32 labels in [0, k)
 * (device), 1 <= k <= 64.  The k x k contingency table is counted on the GPU
 * in exact integers; from it I = sum C(n_ij,2), A = sum C(a_i,2),
 * B = sum C(b_j,2), P = C(n,2) (int64), then in float64 and in this order
 * e = A*B/P, m = (A+B)/2, ARI = (I-e)/(m-e); 1.0 when P = 0 or
 * (A+B)P - 2AB = 0.  Writes ari_host and, if not NULL, the table (k x k
 * int64, row = label of a) to table_host.  A label outside [0, k) gives
 * SYMNMF_ERR_INVALID_ARG.  Workspace: SYMNMF_OP_ARI.  Synchronises `stream`.
 */
SYMNMF_API int symnmf_ari(const int32_t* a, const int32_t* b, int64_t n, int k, double* ari_host,
                          int64_t* table_host, void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * The rolling-window study ([CaS] "The temporal setup", "Tracking stability
 * through time", "Stability and break detection").  Window w holds the days
 * [w*stride, w*stride + window) of the returns stream R (days x n fp32,
 * row = day, leading dimension ldr, device).  For every window and every
 * kind of dependence matrix selected in `kinds`, in this order: build S
 * (symnmf_build_corr / symnmf_build_tpdm) into an n x n buffer (the caller's
 * for the first chain, a chain's own matrix in the workspace otherwise);
 * the cross-sector monitor, when n_stressed >= 2: the mean of S_ij over the
 * pairs of instruments in two different stressed groups (group ids from
 * `groups`, n int32 device); an independent fit from the same seeded start
 * ("Factorizing with SymNMF": fixed-seed initialisation, no warm start) with
 * the `fit` parameters -- or, with warm_start = 1, the workload recipe's
 * warm start: window 0 from the seeded start and every later window from
 * the previous window's factor of the same kind, with the AdaGrad
 * accumulator reset; argmax labels into labels[kind] + w*n; ARI against
 * window w-1 and window w-delta.  Then the 3-sigma control limit of
 * ARI(t-delta, t): mean and sample standard deviation (n-1) over the
 * calibration windows [calib_begin, calib_end) where it is defined,
 * limit = mean - 3 std, and a flag on every window below the limit.
 * Kind index 0 is |corr|, 1 is TPDM.
 */
typedef struct {
    int64_t window;          /* T, days per window (>= 2); default 250 */
    int64_t stride;          /* days between window starts (>= 1); default 1 */
    int64_t n_windows;       /* windows to run; 0 = all that fit, (days - window)/stride + 1 */
    int k;                   /* rank (1..64); default 24 */
    int kinds;               /* SYMNMF_KIND_* bits; default both */
    double tail_frac;        /* TPDM tail fraction; default 0.05 */
    int tail_sign;           /* TPDM tail: -1 lower (joint crashes, default), +1 upper */
    int delta;               /* ARI(t - delta, t) spacing (>= 1); default 50 */
    int64_t calib_begin;     /* calibration windows [calib_begin, calib_end); */
    int64_t calib_end;       /*   default 0, 0 = every window with ARI(t - delta, t) */
    int n_stressed;          /* groups in the cross-sector monitor: 0 = off, else 2..8 */
    int stressed[8];         /* their group ids */
    int warm_start;          /* 0 (default): every window from the seeded start; 1: window
                                w > 0 from window w-1's H of the same kind, G reset to 0 */
    symnmf_fit_params fit;   /* per-window fit; default ADAGRAD, 100 iterations, rel_tol 0 */
} symnmf_rolling_params;

typedef struct {             /* caller-owned outputs, [0] = |corr|, [1] = TPDM */
    int32_t* labels[2];      /* device, n_windows x n: required for each selected kind */
    double* ari_prev[2];     /* host, n_windows (NaN at window 0) or NULL */
    double* ari_delta[2];    /* host, n_windows (NaN below delta) or NULL */
    double* cross[2];        /* host, n_windows (NaN with the monitor off) or NULL */
    double* loss[2];         /* host, n_windows: f(H) of each window's fit, or NULL */
    uint8_t* flag[2];        /* host, n_windows: ARI(t - delta, t) < limit, or NULL */
    double mean[2], std[2], limit[2];  /* written: the calibration (NaN if < 2 windows) */
    int64_t n_windows;       /* written: windows run */
    double build_ms[2];      /* written: CUDA-event time of the builders */
    double fit_ms[2];        /* written: CUDA-event time of the fits and labels */
    double total_ms;         /* written: CUDA-event time of the whole call */
    int kernel_launches;     /* written: kernels launched */
} symnmf_rolling_out;

SYMNMF_API void symnmf_rolling_params_default(symnmf_rolling_params* p);

/*
 * Runs the study above.  S: the caller's n x n fp32 buffer (lds a multiple of
 * 4), overwritten window by window.  groups may be NULL when n_stressed = 0.
 * Workspace: SYMNMF_OP_ROLLING with T = window and params = &p->fit.  That
 * size holds four chains: each selected kind's windows are split between two
 * chains (alternate windows), each chain after the first with its own n x n
 * matrix and buffers, running on a stream and host thread of its own (the
 * chains are ordered after `stream`'s earlier work and `stream` waits for
 * them before the call returns); the ARI series is computed from the stored
 * labels afterwards.  A smaller workspace runs one chain per kind, or a
 * single chain that takes the kinds in turn (also forced by the environment
 * variable SYMNMF_ROLLING_SERIAL=1); the results are the same.  Synchronises
 * the streams once per window and kind (the fit reads its state).
 */
SYMNMF_API int symnmf_rolling(const float* R, int64_t days, int64_t n, int64_t ldr,
                              const int32_t* groups, float* S, int64_t lds,
                              const symnmf_rolling_params* params, symnmf_rolling_out* out,
                              void* ws, size_t ws_bytes, symnmf_stream_t stream);

/*
 * Y = S X like symnmf_sh, for callers that cannot allocate device memory
 * when they call in: a runtime whose device memory is owned entirely by its
 * own pool or by another framework's caching allocator, where an outside
 * cudaMalloc would fragment the pool or break its budget, or a latency-
 * critical loop that cannot take cudaMalloc's implicit synchronisation.
 * The pages have no counterpart of this entry point; it is a packaging
 * variant of the S-stream.
 *
 * It takes no workspace and calls no allocating routine: its scratch (the
 * TF32 split of X and an error word) lives in a 4 MiB file-scope device array
 * that every GPU loading the library holds until exit.  Limit:
 * 2 * roundup(k, 8) * roundup(n, 32) + 64 <= 1,048,576 floats (for k = 24,
 * n <= 21,824); larger sizes return SYMNMF_ERR_INVALID_ARG.  Every call looks
 * up the array's device address (cudaGetSymbolAddress) with the calling
 * device current, so the address stays right after cudaDeviceReset or under
 * another context; the first call on a device also loads the library's
 * module there, so make that first call before any stream capture.
 * Every call shares the one array and it keeps the last call's contents:
 * calls that overlap on the GPU (on different streams, or from several host
 * threads without ordering) race on it.  S, X, Y as for symnmf_sh.
 * Synchronises `stream` at the end (reads the error word).
 */
SYMNMF_API int symnmf_sh_noalloc(const float* S, int64_t n, int64_t lds, const float* X, int k,
                                 float* Y, symnmf_stream_t stream);

/*
 * Test hook for failure detection (no counterpart on the pages).  on != 0:
 * the TMA producer of S in every S-stream kernel (TF32, fp16 and upper-
 * triangle) issues no loads on the current device,
 * so every bounded pipeline wait of the next S-stream launches runs out
 * (about 2 s) and those calls return SYMNMF_ERR_TIMEOUT with the CUDA context
 * intact; on = 0 restores normal operation.  Synchronous.
 */
SYMNMF_API int symnmf_test_stall_pipeline(int on);

/*
 * Test hook for the fp16 S-stream's operand split (no counterpart on the
 * pages): applies the split warps' arithmetic to the n values at x (device,
 * n a multiple of 4, x 16-byte aligned): v = scale * x (scale a power of two),
 * hi = v rounded to fp16, lo = v - hi (exact in fp32) rounded to fp16;
 * hi[i] and lo[i] (device, n / 2 words each) hold the fp16 bit patterns of
 * values 2i (low half) and 2i + 1 (high half).
 * Asynchronous on `stream`.
 */
SYMNMF_API int symnmf_test_split16(const float* x, int64_t n, float scale, uint32_t* hi,
                                   uint32_t* lo, symnmf_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* SYMNMF_H */
