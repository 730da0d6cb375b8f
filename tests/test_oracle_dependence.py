"""Pins of the oracle's dependence-matrix builders and statistics (CPU only).

Each check compares the oracle with something other than itself: a library
routine it does not call, a closed form, an invariant, or a loop brute force.
"""
import math

import numpy as np
import pytest

import oracle
import synth


def _returns(T, n, seed, dist="normal"):
    R, _, _ = synth.workload("corr_n2000_k8" if dist == "normal" else "tpdm_n20000_k24",
                             seed=seed, n=n, T=T)
    return R


# ----------------------------------------------------------------- correlation

def test_corr_matches_numpy_corrcoef():
    R = _returns(50, 300, 0)
    S = oracle.corr_abs(R)
    ref = np.abs(np.corrcoef(R.astype(np.float64), rowvar=False))
    np.testing.assert_allclose(S, ref, rtol=0, atol=1e-12)


def test_corr_two_days_is_one():
    # with T = 2 every non-constant pair of columns is perfectly (anti)correlated
    rng = np.random.default_rng(1)
    R = rng.standard_normal((2, 40)).astype(np.float32)
    S = oracle.corr_abs(R)
    np.testing.assert_allclose(S, np.ones((40, 40)), atol=1e-12)


def test_corr_invariants_and_affine_invariance():
    R = _returns(80, 120, 2)
    S = oracle.corr_abs(R)
    assert np.array_equal(S, S.T)
    assert S.min() >= 0.0 and S.max() <= 1.0 + 1e-15
    assert np.all(np.diag(S) == 1.0)
    rng = np.random.default_rng(3)
    a = rng.uniform(0.5, 2.0, 120) * rng.choice([-1.0, 1.0], 120)
    b = rng.standard_normal(120)
    R2 = (R.astype(np.float64) * a + b)
    np.testing.assert_allclose(oracle.corr_abs(R2), S, atol=1e-10)


def test_corr_zero_variance_column():
    R = _returns(30, 10, 4).astype(np.float64)
    R[:, 3] = 7.0
    S = oracle.corr_abs(R)
    assert S[3, 3] == 1.0
    assert np.all(S[3, np.arange(10) != 3] == 0.0)
    assert np.all(S[np.arange(10) != 3, 3] == 0.0)


# ------------------------------------------------------------------------ TPDM

def _tpdm_loops(R, tail_frac, tail_sign):
    """Brute force with explicit loops: counting ranks, scanning for the top days."""
    T, n = R.shape
    X = [[tail_sign * float(R[t, i]) for i in range(n)] for t in range(T)]
    x = [[0.0] * n for _ in range(T)]
    for i in range(n):
        for t in range(T):
            below = sum(1 for s in range(T) if X[s][i] < X[t][i])
            tied_before = sum(1 for s in range(t) if X[s][i] == X[t][i])
            r = 1 + below + tied_before
            x[t][i] = (-math.log(r / (T + 1))) ** -0.5
    rho = [math.sqrt(sum(v * v for v in x[t])) for t in range(T)]
    N = max(1, int(math.floor(tail_frac * T)))
    chosen = []
    remaining = list(range(T))
    for _ in range(N):
        best = remaining[0]
        for t in remaining[1:]:
            if rho[t] > rho[best]:
                best = t
        chosen.append(best)
        remaining.remove(best)
    S = [[0.0] * n for _ in range(n)]
    for i in range(n):
        for j in range(n):
            S[i][j] = (n / N) * sum((x[t][i] / rho[t]) * (x[t][j] / rho[t]) for t in chosen)
    return np.array(S), sorted(chosen)


@pytest.mark.parametrize("tail_sign", [1, -1])
def test_tpdm_matches_loop_brute_force(tail_sign):
    R = _returns(20, 2, 5, dist="t3")
    S, parts = oracle.tpdm(R, 0.1, tail_sign, return_parts=True)
    ref, days = _tpdm_loops(R, 0.1, tail_sign)
    assert sorted(parts["days"].tolist()) == days
    np.testing.assert_allclose(S, ref, rtol=1e-13, atol=0)


def test_tpdm_brute_force_with_ties():
    # integer-valued returns: many tied values inside a column and tied radii
    rng = np.random.default_rng(6)
    R = rng.integers(-2, 3, size=(24, 4)).astype(np.float32)
    S, parts = oracle.tpdm(R, 0.25, 1, return_parts=True)
    ref, days = _tpdm_loops(R, 0.25, 1)
    assert sorted(parts["days"].tolist()) == days
    np.testing.assert_allclose(S, ref, rtol=1e-13, atol=0)


def test_tpdm_trace_equals_n_and_psd_rank():
    R = _returns(200, 150, 7, dist="t3")
    S = oracle.tpdm(R, 0.05, 1)
    N = oracle.tail_count(200, 0.05)
    assert N == 10
    assert abs(np.trace(S) - 150) < 1e-10
    w = np.linalg.eigvalsh(S)
    assert w.min() > -1e-10
    assert np.sum(w > 1e-9 * w.max()) <= N
    assert np.array_equal(S, S.T)


def test_tpdm_monotone_invariance_is_exact():
    R = _returns(100, 30, 8, dist="t3").astype(np.float64)
    S = oracle.tpdm(R, 0.05, 1)
    R2 = R.copy()
    R2[:, 5] = np.exp(R2[:, 5])             # strictly increasing transform
    R2[:, 9] = 3.0 * R2[:, 9] + 11.0
    assert np.array_equal(oracle.tpdm(R2, 0.05, 1), S)


def test_tpdm_day_permutation_invariance():
    R = _returns(120, 40, 9, dist="t3")
    S = oracle.tpdm(R, 0.05, 1)
    perm = np.random.default_rng(10).permutation(120)
    np.testing.assert_allclose(oracle.tpdm(R[perm], 0.05, 1), S, rtol=1e-12, atol=1e-13)


def test_tail_count():
    assert oracle.tail_count(1000, 0.05) == 50
    assert oracle.tail_count(250, 0.05) == 12
    assert oracle.tail_count(10, 0.01) == 1


# ----------------------------------------------------------------------- stats

def test_stats_against_fsum_and_nonfinite():
    rng = np.random.default_rng(11)
    S = rng.random((37, 37)).astype(np.float32)
    S[3, 4] = np.nan
    S[5, 6] = np.inf
    s, sq, bad = oracle.stats(S)
    vals = [float(v) for v in S.ravel() if np.isfinite(v)]
    assert bad == 2
    assert abs(s - math.fsum(vals)) <= 1e-12 * abs(s)
    assert abs(sq - math.fsum(v * v for v in vals)) <= 1e-12 * sq


def test_stats_planted_blocks_closed_form():
    S, _ = synth.planted_block_matrix([5, 3, 2])
    s, sq, bad = oracle.stats(S)
    assert (s, sq, bad) == (25 + 9 + 4, 25 + 9 + 4, 0)


def test_row_sampled_builders_equal_full_rows():
    R = _returns(90, 150, 13, dist="t3").astype(np.float64)
    R[:, 4] = 2.0                                  # a zero-variance column
    rows = np.array([0, 4, 77, 149])
    np.testing.assert_allclose(oracle.corr_abs_rows(R, rows), oracle.corr_abs(R)[rows], atol=1e-13)
    for sign in (1, -1):
        np.testing.assert_allclose(oracle.tpdm_rows(R, rows, 0.05, sign),
                                   oracle.tpdm(R, 0.05, sign)[rows], rtol=1e-12, atol=1e-14)
