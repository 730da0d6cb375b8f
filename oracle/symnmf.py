"""CPU fp64 oracle for the SymNMF clustering hot path.

TEST INFRASTRUCTURE.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module.  It shares no code
with the CUDA library; the only common input is ``synth``.

Sources (cited by page title and section):

[CaS]  "GPU-Accelerated Clustering for Financial Instruments at Scale"
       (NVIDIA technical blog, bilingual copy), sections "Factorization at
       scale", "Choosing the rank k", "Factorizing with SymNMF" (diagonal
       AdaGrad update), "Why this solver" (post-rank gap ratio), "Tracking
       stability through time with the Rand index", "The metric".
[SMI]  "GPU-Accelerated SymNMF Clustering Scales to a Million Financial
       Instruments" (English copy of the same post): the LaTeX form of the
       AdaGrad update and the AdaptGrow algorithm sketch.
[LRD]  abstract of "Low-Rank Dependence Decomposition via Accelerated
       Symmetric Non-negative Matrix Factorization" (trace-identity
       reformulation; Block-SVRG AdaptGrow).

Every floating-point step runs in float64.  Inputs arrive as float32 (the
library's storage type) and are widened exactly.  ``mirror=True`` in the
solvers rounds H and G to float32 after every step, the precision in which
the library stores them, so that trajectories stay comparable.

Where the pages leave a step open, the reading taken is stated at the
function.  Parity status per function is listed in ``PINS`` at the bottom.
Three such readings have nothing on the pages to check them against and are
parity unpinned (both sides implement the written reading, and GPU/oracle
parity is still tested): the Block-SVRG stall rule (``stall_tol`` on the
snapshot loss), the seeding of the starting block size (the power of two
nearest n/10), and the TPDM tail sign.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np

# ---------------------------------------------------------------------------
# dependence matrices
# ---------------------------------------------------------------------------


def corr_abs(R: np.ndarray) -> np.ndarray:
    """Absolute Pearson correlation of the columns of a T x n returns window.

    [CaS] "Tracking stability through time..." (correlation measures
    co-movement over the body of the distribution): S_ij = |corr(r_i, r_j)|.
    Reading for a zero-variance column i (not covered by the pages): row and
    column i are 0 except S_ii = 1.  Returns float64 n x n.
    """
    X = np.asarray(R, dtype=np.float64)
    T, n = X.shape
    mu = X.sum(axis=0) / T
    Z = X - mu
    ss = (Z * Z).sum(axis=0)
    C = Z.T @ Z
    ok = ss > 0.0
    denom = np.sqrt(np.outer(ss, ss))
    S = np.zeros((n, n), dtype=np.float64)
    both = np.outer(ok, ok)
    S[both] = np.abs(C[both]) / denom[both]
    np.fill_diagonal(S, 1.0)
    return S


def corr_abs_rows(R: np.ndarray, rows) -> np.ndarray:
    """Rows ``rows`` of ``corr_abs(R)`` without forming the n x n matrix."""
    X = np.asarray(R, dtype=np.float64)
    T, n = X.shape
    rows = np.asarray(rows)
    Z = X - X.sum(axis=0) / T
    ss = (Z * Z).sum(axis=0)
    ok = ss > 0.0
    Zn = np.where(ok, Z / np.sqrt(np.where(ok, ss, 1.0)), 0.0)
    out = np.abs(Zn[:, rows].T @ Zn)
    out[np.arange(len(rows)), rows] = 1.0
    return out


def tail_count(T: int, tail_frac: float) -> int:
    """N = max(1, floor(tail_frac * T)), evaluated in IEEE double."""
    return max(1, int(math.floor(tail_frac * float(T))))


def column_ranks(X: np.ndarray) -> np.ndarray:
    """Rank 1..T of every entry within its column; ties go to the earlier day."""
    T, n = X.shape
    order = np.argsort(X, axis=0, kind="stable")
    r = np.empty((T, n), dtype=np.int64)
    cols = np.arange(n)[None, :]
    r[order, cols] = np.arange(1, T + 1)[:, None]
    return r


def tpdm(R: np.ndarray, tail_frac: float = 0.05, tail_sign: int = 1,
         return_parts: bool = False):
    """Tail pairwise dependence matrix of a T x n returns window.

    [CaS] "Tracking stability through time..." (TPDM: co-movement
    conditional on extreme events).  The pages give the name only; the
    estimator follows the workload recipe (ranks mapped to Frechet alpha=2
    margins, average of w_i w_j over the days with the top tail_frac radii,
    scaled by n), which is the TPDM of Cooley & Thibaud (2019):

      1. r_ti  = rank of tail_sign * R_ti in column i (1..T, ties to earlier t)
      2. x_ti  = (-ln(r_ti / (T+1)))^(-1/2)
      3. rho_t = ||x_t||_2
      4. E     = the N = max(1, floor(tail_frac*T)) days of largest rho
                 (ties to the earlier day)
      5. w_ti  = x_ti / rho_t
      6. S_ij  = (n / N) * sum_{t in E} w_ti w_tj
    """
    X = tail_sign * np.asarray(R, dtype=np.float64)
    T, n = X.shape
    r = column_ranks(X)
    x = (-np.log(r / float(T + 1))) ** -0.5
    rho = np.sqrt((x * x).sum(axis=1))
    N = tail_count(T, tail_frac)
    days = np.lexsort((np.arange(T), -rho))[:N]      # largest rho first, then earlier t
    W = x[days] / rho[days, None]
    S = (float(n) / N) * (W.T @ W)
    if return_parts:
        return S, dict(ranks=r, x=x, rho=rho, days=days)
    return S


def tpdm_rows(R: np.ndarray, rows, tail_frac: float = 0.05, tail_sign: int = 1) -> np.ndarray:
    """Rows ``rows`` of ``tpdm(R, tail_frac, tail_sign)`` without the n x n matrix."""
    X = tail_sign * np.asarray(R, dtype=np.float64)
    T, n = X.shape
    r = column_ranks(X)
    x = (-np.log(r / float(T + 1))) ** -0.5
    rho = np.sqrt((x * x).sum(axis=1))
    N = tail_count(T, tail_frac)
    days = np.lexsort((np.arange(T), -rho))[:N]
    W = x[days] / rho[days, None]
    return (float(n) / N) * (W[:, np.asarray(rows)].T @ W)


# ---------------------------------------------------------------------------
# statistics pre-pass and seeded initialisation
# ---------------------------------------------------------------------------


def stats(S: np.ndarray):
    """(sum of all S_ij, ||S||_F^2, number of non-finite entries), fp64.

    The squared norm is the constant term of the trace-identity loss ([CaS]
    "Factorization at scale"); the mean feeds the scale-matched init.
    """
    X = np.asarray(S, dtype=np.float64)
    fin = np.isfinite(X)
    Xf = np.where(fin, X, 0.0)
    return float(Xf.sum()), float((Xf * Xf).sum()), int((~fin).sum())


MASK64 = (1 << 64) - 1
GOLDEN_GAMMA = 0x9E3779B97F4A7C15          # splitmix64 state increment
SVRG_STREAM = 0xD1B54A32D192ED03           # per-epoch stream separation constant


def splitmix64_mix(z):
    """The splitmix64 output function (Steele, Lea & Flood, OOPSLA 2014).

    Works on Python ints or numpy uint64 arrays (wrapping arithmetic).
    """
    if isinstance(z, np.ndarray):
        z = z.astype(np.uint64)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))
    z &= MASK64
    z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & MASK64
    z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & MASK64
    return z ^ (z >> 31)


def splitmix64_stream(state: int, count: int):
    """``count`` successive outputs of a splitmix64 generator seeded with ``state``."""
    out = []
    for _ in range(count):
        state = (state + GOLDEN_GAMMA) & MASK64
        out.append(splitmix64_mix(state))
    return out


def counter_uniform(seed: int, count: int) -> np.ndarray:
    """u_c = (mix(seed + (c+1)*gamma) >> 40) * 2^-24 for c = 0..count-1.

    The c-th output of a splitmix64 generator seeded with ``seed``, reduced to
    24 bits: an exact float32 in [0, 1).  Counter-addressed, so any element
    can be produced independently.
    """
    c = np.arange(1, count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed & MASK64) + c * np.uint64(GOLDEN_GAMMA)
    return (splitmix64_mix(z) >> np.uint64(40)).astype(np.float64) * 2.0 ** -24


def init_scale(s_sum: float, n: int, k: int) -> float:
    """c = fl32(sqrt(mean(S) / k)) with mean(S) = sum(S) / n^2 (diagonal included)."""
    mean = s_sum / (float(n) * float(n))
    return float(np.float32(math.sqrt(max(mean, 0.0) / k)))


def scale_matched_init(s_sum: float, n: int, k: int, seed: int) -> np.ndarray:
    """H0_ij = fl32(u_ij * c), u from ``counter_uniform`` with element index i*k + j.

    [SMI] AdaptGrow sketch calls ``scale_matched_init(S, k)`` with a fixed
    seed ([CaS] "Factorizing with SymNMF": same fixed-seed initialisation for
    every window) without defining it.  Reading: uniform entries scaled so
    that E[(H H^T)_ij] matches mean(S) in order of magnitude, the recipe of
    the small correlation workload.  Returns float32 n x k.
    """
    c = init_scale(s_sum, n, k)
    u = counter_uniform(seed, n * k).reshape(n, k)
    return (u * c).astype(np.float32)


# ---------------------------------------------------------------------------
# loss, gradient, update
# ---------------------------------------------------------------------------


def trace_loss(S_sqnorm: float, H: np.ndarray, P: np.ndarray) -> float:
    """f(H) = ||S||^2 - 2 tr(H^T S H) + ||H^T H||_F^2, with P = S H.

    [CaS] "Factorization at scale" / [LRD]: the trace form of
    ||S - H H^T||_F^2 that needs no n x n intermediate.
    """
    A = H.T @ H
    return S_sqnorm - 2.0 * float((H * P).sum()) + float((A * A).sum())


def gradient(H: np.ndarray, P: np.ndarray) -> np.ndarray:
    """g = 4 (H (H^T H) - S H), the gradient printed in the [SMI] sketch."""
    return 4.0 * (H @ (H.T @ H) - P)


def adagrad_step(H: np.ndarray, G: np.ndarray, g: np.ndarray, lr: float, eps: float):
    """Projected diagonal AdaGrad, elementwise ([CaS] "Factorizing with SymNMF"):

        G <- G + g * g
        H <- max(H - lr * g / (sqrt(G) + eps), 0)

    The accumulator is updated before the step and eps sits outside the root.
    """
    G = G + g * g
    H = np.maximum(H - lr * g / (np.sqrt(G) + eps), 0.0)
    return H, G


def rel_change(L: float, L_prev: float) -> float:
    if L_prev != 0.0:
        return abs(L - L_prev) / abs(L_prev)
    return 0.0 if L == L_prev else math.inf


@dataclass
class FitResult:
    H: np.ndarray                   # returned loadings (float64; float32 values when mirrored)
    G: np.ndarray                   # AdaGrad accumulator matching H
    iters: int                      # full-batch updates applied to reach H
    epochs: int = 0                 # Block-SVRG epochs run
    converged: bool = False
    loss: float = math.nan          # f(H) of the returned H
    rel: float = math.nan           # last relative loss change
    history: list = field(default_factory=list)     # f(H_t) for every evaluation
    solver_used: int = 0            # 0 full batch, 1 Block-SVRG (possibly grown to full)
    block_final: int = 0
    gamma: float = math.nan         # post-rank gap ratio (AdaptGrow only)


def _f32(a):
    return a.astype(np.float32).astype(np.float64)


def _operand(S):
    """S as the solvers use it.  Normally the matrix widened to float64.  An
    object that declares ``exact_float64_products = True`` is passed through
    unchanged: it supplies the two products the solvers form, ``S @ X`` and
    ``S[:, rows] @ D``, exactly in float64 (a matrix too large to widen at
    once, read in row chunks).  The solvers then need ``S_sqnorm`` given."""
    if getattr(S, "exact_float64_products", False):
        return S
    return np.asarray(S, dtype=np.float64)


def fit_adagrad(S, k, H0, lr=0.1, eps=1e-10, max_iters=200, rel_tol=0.0,
                G0=None, mirror=True, S_sqnorm=None, hook=None) -> FitResult:
    """Full-batch projected AdaGrad ([SMI] AdaptGrow sketch, phi >= 1 branch).

    Evaluation t (t = 0..max_iters) computes f(H_t).  The loop stops at the
    first t > 0 with |f_t - f_{t-1}| / f_{t-1} < rel_tol (rel_tol > 0) or at
    t = max_iters, and returns H_t; otherwise it takes the update of H_t.
    ``hook(t, H, P)`` (tests only) sees every evaluated iterate.
    """
    S = _operand(S)
    n = S.shape[0]
    H = np.asarray(H0, dtype=np.float64).reshape(n, k).copy()
    G = np.zeros_like(H) if G0 is None else np.asarray(G0, dtype=np.float64).copy()
    sq = float((S * S).sum()) if S_sqnorm is None else float(S_sqnorm)
    res = FitResult(H=H, G=G, iters=0)
    L_prev = None
    t = 0
    while True:
        P = S @ H
        L = trace_loss(sq, H, P)
        res.history.append(L)
        if hook is not None:
            hook(t, H, P)
        if L_prev is not None:
            res.rel = rel_change(L, L_prev)
            if rel_tol > 0.0 and res.rel < rel_tol:
                res.converged = True
                break
        if t == max_iters:
            break
        H, G = adagrad_step(H, G, gradient(H, P), lr, eps)
        if mirror:
            H, G = _f32(H), _f32(G)
        L_prev = L
        t += 1
    res.H, res.G, res.iters, res.loss = H, G, t, L
    return res


# ---------------------------------------------------------------------------
# Block-SVRG and AdaptGrow
# ---------------------------------------------------------------------------


def default_block_rows(n: int) -> int:
    """Starting block b0: the power of two nearest to n/10 on a log scale.

    The pages fix no rule; this one reproduces the blocks of both Block-SVRG
    workloads (2048 rows at n = 20,000 and 8192 at n = 100,000).  Exact
    integer form: b = largest power of two with 10 b <= n, doubled when
    b < (n/10) / sqrt(2), i.e. when 200 b^2 < n^2; clamped to [1, n].
    """
    b = 1
    while 10 * (2 * b) <= n:
        b *= 2
    if 10 * b <= n and 200 * b * b < n * n:
        b *= 2
    return max(1, min(b, n))


def epoch_permutation(m: int, seed: int, epoch: int) -> list:
    """Visiting order of the m row blocks in an epoch: Fisher-Yates driven by a
    splitmix64 stream seeded with seed XOR (epoch+1)*SVRG_STREAM; swap index
    r mod (i+1) for i = m-1 down to 1.
    """
    state = (seed ^ ((epoch + 1) * SVRG_STREAM)) & MASK64
    perm = list(range(m))
    draws = splitmix64_stream(state, max(m - 1, 0))
    for d, i in enumerate(range(m - 1, 0, -1)):
        j = draws[d] % (i + 1)
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def block_svrg_grad(S, H, H_snap, P_snap, rows: slice, m: int) -> np.ndarray:
    """Block-sampled SVRG estimate of the gradient on row block B.

    [CaS] "Factorizing with SymNMF" (block-sampled gradient corrected with
    SVRG); [SMI] sketch names ``block_svrg_grad(S, H, phi)`` without defining
    it.  Reading (Johnson & Zhang 2013 control variate on the S H term, with
    the unbiased 1/p = m weight for a uniformly drawn block of m):

        S H  ~  P_snap + m * S[:, B] (H_B - H_snap_B)
        g    =  4 (H (H^T H) - that estimate)

    S[:, B] (H_B - H_snap_B) equals (S[B, :])^T (...) for symmetric S: the
    "row block" of the pages.
    """
    D = H[rows] - H_snap[rows]
    est = P_snap + m * (S[:, rows] @ D)
    return 4.0 * (H @ (H.T @ H) - est)


def fit_block_svrg(S, k, H0, lr=0.1, eps=1e-10, max_epochs=50, rel_tol=0.0,
                   block_rows=0, grow=True, stall_tol=1e-4, seed=0, G0=None,
                   mirror=True, S_sqnorm=None) -> FitResult:
    """Block-SVRG with AdaptGrow growth of the block ([SMI] sketch, phi < 1 branch).

    Epoch e: snapshot H~ = H, P~ = S H~, f(H~) (the convergence test runs on
    consecutive snapshot losses); if growth is on and the snapshot loss fell
    by less than stall_tol (relative) since the previous snapshot, the block
    doubles (b <- min(2b, n)) -- "expands the sample toward the full gradient
    if progress stalls".  Then one pass over the m = ceil(n/b) contiguous row
    blocks in a seeded permutation, each an SVRG step with the AdaGrad update.
    Once b = n, the solver continues as full-batch AdaGrad with the same G
    ("same diagonal AdaGrad update either way"); each such iteration counts
    as one epoch of the budget.
    """
    S = _operand(S)
    n = S.shape[0]
    H = np.asarray(H0, dtype=np.float64).reshape(n, k).copy()
    G = np.zeros_like(H) if G0 is None else np.asarray(G0, dtype=np.float64).copy()
    sq = float((S * S).sum()) if S_sqnorm is None else float(S_sqnorm)
    b = default_block_rows(n) if block_rows <= 0 else min(int(block_rows), n)
    res = FitResult(H=H, G=G, iters=0, solver_used=1)
    L_prev = None
    e = 0
    while True:
        P = S @ H
        L = trace_loss(sq, H, P)
        res.history.append(L)
        if L_prev is not None:
            res.rel = rel_change(L, L_prev)
            if rel_tol > 0.0 and res.rel < rel_tol:
                res.converged = True
                break
            if grow and b < n and (L_prev - L) / L_prev < stall_tol:
                b = min(2 * b, n)
        if e == max_epochs:
            break
        if b >= n:
            # full gradient from here on, same accumulator
            H, G = adagrad_step(H, G, gradient(H, P), lr, eps)
            if mirror:
                H, G = _f32(H), _f32(G)
            res.iters += 1
        else:
            m = -(-n // b)
            H_snap = H.copy()
            for blk in epoch_permutation(m, seed, e):
                rows = slice(blk * b, min((blk + 1) * b, n))
                g = block_svrg_grad(S, H, H_snap, P, rows, m)
                H, G = adagrad_step(H, G, g, lr, eps)
                if mirror:
                    H, G = _f32(H), _f32(G)
            res.epochs += 1
        L_prev = L
        e += 1
    res.H, res.G, res.loss, res.block_final = H, G, L, b
    return res


def top_eigenvalues(S: np.ndarray, n_eig: int) -> np.ndarray:
    """The n_eig algebraically largest eigenvalues of symmetric S, descending (LAPACK)."""
    w = np.linalg.eigvalsh(np.asarray(S, dtype=np.float64))
    return w[::-1][:n_eig].copy()


def gap_ratio(eigvals_desc, k: int) -> float:
    """gamma_{k+1} = lambda_{k+1} / |lambda_{k+2}| (1-indexed, descending).

    [CaS] "Why this solver".  gamma = +inf when lambda_{k+2} = 0.
    """
    lam1 = float(eigvals_desc[k])
    lam2 = float(eigvals_desc[k + 1])
    if lam2 == 0.0:
        return math.inf
    return lam1 / abs(lam2)


def adaptgrow(S, k, lr=0.1, eps=1e-10, max_iters=2000, rel_tol=1e-5, seed=0,
              gap_threshold=5.0, block_rows=0, grow=True, stall_tol=1e-4,
              H0=None, eigvals=None, mirror=True) -> FitResult:
    """AdaptGrow ([SMI] sketch; [CaS] "Why this solver").

    gamma_{k+1} >= gap_threshold selects full-batch AdaGrad; otherwise the
    solver starts with Block-SVRG at b0 = ``default_block_rows(n)``.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    s_sum, sq, _ = stats(S)
    if H0 is None:
        H0 = scale_matched_init(s_sum, n, k, seed)
    if eigvals is None:
        eigvals = top_eigenvalues(S, k + 2)
    gamma = gap_ratio(eigvals, k)
    if gamma >= gap_threshold:
        r = fit_adagrad(S, k, H0, lr, eps, max_iters, rel_tol, mirror=mirror, S_sqnorm=sq)
        r.solver_used = 0
    else:
        r = fit_block_svrg(S, k, H0, lr, eps, max_iters, rel_tol, block_rows, grow,
                           stall_tol, seed, mirror=mirror, S_sqnorm=sq)
    r.gamma = gamma
    return r


# ---------------------------------------------------------------------------
# spherical k-means (hard-label baseline)
# ---------------------------------------------------------------------------

KMEANS_STREAM = 0x5851F42D4C957F2D   # splitmix64 stream separation for the initial centroids


def forgy_indices(n: int, k: int, seed: int) -> list:
    """k distinct row indices: the first k entries of a Fisher-Yates shuffle of
    0..n-1 driven upwards (position q swaps with q + r mod (n - q)) by the
    splitmix64 stream seeded with seed XOR KMEANS_STREAM."""
    state = (seed ^ KMEANS_STREAM) & MASK64
    draws = splitmix64_stream(state, k)
    perm = {}
    out = []
    for q in range(k):
        j = q + draws[q] % (n - q)
        vq, vj = perm.get(q, q), perm.get(j, j)
        perm[q], perm[j] = vj, vq
        out.append(perm[q])
    return out


@dataclass
class KMeansResult:
    labels: np.ndarray       # int32 [n], the last assignment
    centroids: np.ndarray    # [k, n], unit rows
    steps: int               # assignment steps taken
    converged: bool          # the labels stopped changing
    objective: list          # sum_i <x_i, c_{l_i}> at each assignment step
    min_gap: list            # smallest best-minus-second score over the rows, per step


def spherical_kmeans(S, k: int, seed: int = 0, max_iters: int = 100) -> KMeansResult:
    """Spherical k-means on the L2-normalised rows of S ([CaS] "Spherical
    k-means for direct hard clustering": cosine similarity on the normalised
    rows of S).

    x_i = S_i / ||S_i|| (a zero row stays zero); centroids start at the rows
    ``forgy_indices(n, k, seed)``; each step assigns l_i = argmax_c <x_i, c_c>
    (lowest index on ties) and stops when no label changed, else sets
    c_c = sum_{l_i = c} x_i / ||.|| (an empty cluster keeps its centroid).
    ``min_gap`` records how close each step came to a tie, so that a caller
    comparing against another precision knows whether the labels are decided.
    """
    S = np.asarray(S, dtype=np.float64)
    n = S.shape[0]
    norms = np.sqrt((S * S).sum(axis=1))
    X = np.where(norms[:, None] > 0, S / np.where(norms > 0, norms, 1.0)[:, None], 0.0)
    C = X[forgy_indices(n, k, seed)].copy()
    lab = None
    objective, min_gap = [], []
    steps = 0
    converged = False
    while steps < max_iters:
        scores = X @ C.T
        new = np.argmax(scores, axis=1).astype(np.int32)
        steps += 1
        objective.append(float(scores[np.arange(n), new].sum()))
        if k > 1:
            top2 = np.sort(scores, axis=1)[:, -2:]
            min_gap.append(float((top2[:, 1] - top2[:, 0]).min()))
        else:
            min_gap.append(float("inf"))
        if lab is not None and np.array_equal(new, lab):
            converged = True
            break
        lab = new
        for c in range(k):
            members = lab == c
            if members.any():
                v = X[members].sum(axis=0)
                nv = np.sqrt((v * v).sum())
                if nv > 0:
                    C[c] = v / nv
    return KMeansResult(lab, C, steps, converged, objective, min_gap)


# ---------------------------------------------------------------------------
# labels and agreement
# ---------------------------------------------------------------------------


def labels(H: np.ndarray) -> np.ndarray:
    """Hard label = row-wise argmax of H, lowest index on ties ([CaS]
    "Factorizing with SymNMF").  An all-zero row gets label 0."""
    return np.argmax(np.asarray(H), axis=1).astype(np.int32)


def contingency(a, b, ka: int, kb: int) -> np.ndarray:
    """n_ij = #{t : a_t = i, b_t = j} for labels a in [0, ka), b in [0, kb) (int64)."""
    a = np.asarray(a, dtype=np.int64).ravel()
    b = np.asarray(b, dtype=np.int64).ravel()
    if a.size and (a.min() < 0 or a.max() >= ka or b.min() < 0 or b.max() >= kb):
        raise ValueError("label out of range")
    table = np.zeros((ka, kb), dtype=np.int64)
    np.add.at(table, (a, b), 1)
    return table


def ari_from_table(table) -> float:
    """Adjusted Rand index (Hubert & Arabie 1985) from a contingency table.

    [CaS] "The metric": pair agreement corrected for chance, 1 for identical
    clusterings and about 0 for unrelated ones.  The pair counts
    I = sum C(n_ij, 2), A = sum C(a_i, 2), B = sum C(b_j, 2), P = C(n, 2) are
    exact integers; then, in float64 and in this order,
    e = (A * B) / P, m = (A + B) / 2, ARI = (I - e) / (m - e).
    Returns 1.0 when P = 0 or the exact denominator (A + B) P - 2 A B is 0
    (both labelings trivial).
    """
    t = np.asarray(table, dtype=np.int64)
    n = int(t.sum())
    comb = lambda x: sum(int(v) * (int(v) - 1) // 2 for v in np.asarray(x).ravel())
    I, A, B = comb(t), comb(t.sum(axis=1)), comb(t.sum(axis=0))
    P = n * (n - 1) // 2
    if P == 0 or (A + B) * P - 2 * A * B == 0:
        return 1.0
    e = (float(A) * float(B)) / float(P)
    m = (float(A) + float(B)) / 2.0
    return (float(I) - e) / (m - e)


def ari(a, b) -> float:
    """Adjusted Rand index of two labelings (any integer label values)."""
    a = np.asarray(a).ravel()
    b = np.asarray(b).ravel()
    _, ai = np.unique(a, return_inverse=True)
    _, bi = np.unique(b, return_inverse=True)
    if a.size == 0:
        return 1.0
    return ari_from_table(contingency(ai, bi, int(ai.max()) + 1, int(bi.max()) + 1))


# ---------------------------------------------------------------------------
# rolling windows: stability, the control limit, the cross-sector monitor
# ---------------------------------------------------------------------------

def cross_sector_mean(S, groups, stressed) -> float:
    """Mean of S_ij over the pairs (i, j) whose instruments sit in two
    different stressed groups ([CaS] "Stability and break detection": the
    cross-sector dependence among the stressed sectors, read off the
    off-diagonal blocks of S)."""
    S = np.asarray(S, dtype=np.float64)
    groups = np.asarray(groups)
    idx = [np.flatnonzero(groups == g) for g in stressed]
    total, count = 0.0, 0
    for a in range(len(idx)):
        for b in range(len(idx)):
            if a != b:
                total += float(S[np.ix_(idx[a], idx[b])].sum())
                count += len(idx[a]) * len(idx[b])
    return total / count if count else float("nan")


def control_limit(series, calib_windows):
    """Self-calibrating 3-sigma limit ([CaS] "Stability and break detection"):
    mean and sample standard deviation (ddof = 1) of the series over the calm
    calibration windows (NaNs skipped); limit = mean - 3 * std."""
    vals = np.array([series[t] for t in calib_windows if np.isfinite(series[t])], dtype=np.float64)
    if vals.size < 2:
        return float("nan"), float("nan"), float("nan")
    mu = float(vals.mean())
    sd = float(np.sqrt(((vals - mu) ** 2).sum() / (vals.size - 1)))
    return mu, sd, mu - 3.0 * sd


def rolling_pipeline(R, T: int, k: int, n_windows: int | None = None, stride: int = 1,
                     kinds=("corr", "tpdm"), tail_frac: float = 0.05, tail_sign: int = -1,
                     delta: int = 50, calib=None, groups=None, stressed=(), iters: int = 100,
                     lr: float = 0.1, eps: float = 1e-10, seed: int = 0, only=None,
                     keep_H: bool = False, warm_start: bool = False) -> dict:
    """The rolling-window study ([CaS] "The temporal setup", "Tracking
    stability through time", "Stability and break detection").

    Window w holds days [w * stride, w * stride + T).  For each window and
    each kind of dependence matrix: S = the matrix of that window (float64,
    rounded to float32 as stored); an independent fit from the same
    scale-matched seeded start ("Factorizing with SymNMF": fixed-seed
    initialisation, no warm start), ``iters`` full-batch AdaGrad updates;
    labels = row-wise argmax; ARI against the previous window and against
    the window ``delta`` earlier; the cross-sector mean over ``stressed``
    groups of ``groups``.  Then the 3-sigma limit of ARI(t - delta, t) over
    the windows ``calib`` (default: every window with ARI(t - delta, t)) and
    a flag on every window whose ARI(t - delta, t) falls below it.

    ``only`` (a set of window indices) restricts the work to those windows:
    the others keep label -1 and NaN entries, and an ARI needs both of its
    windows.  ``keep_H`` also returns each window's factor (float32).

    ``warm_start`` takes the workload recipe's reading instead ("warm-started
    100-iteration fit", AdaGrad accumulator reset per window): the first
    window starts from the seeded start, every later window from the
    previous window's factor of the same kind (rounded to float32 as the
    library stores it), with G = 0.  It needs every window, so not ``only``.
    """
    R = np.asarray(R)
    days, n = R.shape
    W = (days - T) // stride + 1 if n_windows is None else n_windows
    if W < 1 or (W - 1) * stride + T > days:
        raise ValueError("windows do not fit in the stream")
    if warm_start and only is not None:
        raise ValueError("a warm start needs every window")
    todo = set(range(W)) if only is None else {int(w) for w in only if 0 <= w < W}
    out = {}
    for kind in kinds:
        lab = np.full((W, n), -1, dtype=np.int32)
        loss = np.full(W, np.nan)
        cross = np.full(W, np.nan)
        smax = np.full(W, np.nan)
        Hs = {}
        H_prev = None
        for w in sorted(todo):
            Rw = R[w * stride: w * stride + T]
            if kind == "corr":
                S = corr_abs(Rw).astype(np.float32)
            else:
                S = tpdm(Rw, tail_frac, tail_sign).astype(np.float32)
            smax[w] = float(np.abs(S).max())
            if groups is not None and len(stressed) > 1:
                cross[w] = cross_sector_mean(S, groups, stressed)
            s_sum, sq, _ = stats(S)
            if warm_start and H_prev is not None:
                H0 = H_prev
            else:
                H0 = scale_matched_init(s_sum, n, k, seed)
            r = fit_adagrad(S, k, H0, lr=lr, eps=eps, max_iters=iters, rel_tol=0.0, S_sqnorm=sq)
            H_prev = _f32(r.H)
            lab[w] = labels(_f32(r.H))
            loss[w] = r.loss
            if keep_H:
                Hs[w] = _f32(r.H)
        ari_prev = np.full(W, np.nan)
        ari_delta = np.full(W, np.nan)
        for w in range(1, W):
            if w in todo and w - 1 in todo:
                ari_prev[w] = ari_from_table(contingency(lab[w - 1], lab[w], k, k))
            if w >= delta and w in todo and w - delta in todo:
                ari_delta[w] = ari_from_table(contingency(lab[w - delta], lab[w], k, k))
        cw = range(delta, W) if calib is None else range(max(calib[0], delta), min(calib[1], W))
        mu, sd, limit = control_limit(ari_delta, cw)
        flags = np.array([np.isfinite(x) and x < limit for x in ari_delta], dtype=bool)
        out[kind] = dict(labels=lab, loss=loss, cross=cross, smax=smax, ari_prev=ari_prev,
                         ari_delta=ari_delta, mean=mu, std=sd, limit=limit, flags=flags)
        if keep_H:
            out[kind]["H"] = Hs
    return out


# What pins each function in the CPU test suite (tests/test_oracle_*.py).
PINS = {
    "corr_abs": "numpy.corrcoef; T=2 closed form; symmetry, range, unit diagonal, affine invariance",
    "tpdm": "trace(S)=n; PSD of rank <= N; monotone invariance; day-permutation invariance; loop brute force",
    "corr_abs_rows / tpdm_rows": "equal the rows of corr_abs / tpdm",
    "stats": "math.fsum; planted block closed form",
    "counter_uniform": "published splitmix64 outputs (tests/golden); uniformity",
    "trace_loss": "brute-force ||S - H H^T||_F^2",
    "gradient": "central finite differences of the brute-force loss",
    "adagrad_step": "first-step closed form; H >= 0; G non-decreasing",
    "fit_adagrad": "k=1 rank-one recovery; planted blocks ARI = 1; permutation equivariance",
    "fit_block_svrg": ("b = n equals full batch; block unbiasedness identity; H >= 0; a two-block "
                       "epoch equals hand-applied steps with the snapshot frozen at the epoch start "
                       "(ragged block, masked full products); three epochs equal hand-applied epochs "
                       "in the epoch_permutation order, and differ in the reversed order; the stall "
                       "rule replayed on consecutive snapshot losses; planted noise-free blocks "
                       "recovered with ARI = 1 by b < n, growth off, from listed starts"),
    "epoch_permutation": "is a permutation; uniform over orders for small m",
    "top_eigenvalues": "block-of-ones closed form; sum = trace",
    "gap_ratio": "hand values",
    "labels": "hand cases with ties",
    "spherical_kmeans": "objective non-decreasing; unit centroids; brute-force assignment; planted blocks recovered",
    "forgy_indices": "distinct, in range; uniform first index",
    "ari": "sklearn.metrics.adjusted_rand_score; O(n^2) pair brute force",
    "contingency": "loop count; row and column sums",
    "cross_sector_mean": "pair loop brute force; planted constant blocks",
    "control_limit": "hand values",
    "rolling_pipeline": "windows equal standalone window runs; planted switch flagged, calm windows not",
    "stall rule, starting block size, TPDM tail sign": "parity unpinned (readings of silent passages)",
}
