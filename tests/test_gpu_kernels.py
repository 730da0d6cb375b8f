"""GPU parity of the individual kernels against the CPU oracle.

Sizes span several tiles of every kernel plus a ragged tail; each case also
runs a degenerate size.  Tolerances:
  S H            relative Frobenius <= 1e-4 (fp32 products, fp32 accumulation)
  |corr| builder max |dS| <= 5e-6 (fp32 normalised window, fp32 accumulation)
  TPDM builder   max |dS| <= 1e-5 * max|S|; the selected days are exact
  stats          1e-12 relative (fp64 on both sides); non-finite count exact
  labels         bit-exact
  probe          top k+2 eigenvalues within 1e-5 relative to lambda_1
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import corr_problem, rel_fro, to_dev, tpdm_problem

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def m():
    import torch
    from symmetric_nmf_clustering_b200 import build
    build.build()
    import symmetric_nmf_clustering_b200 as m
    torch.cuda.init()
    return m


DEV = "cuda:0"


def test_labels_bit_exact_with_ties(m):
    rng = np.random.default_rng(0)
    for n, k in [(1, 1), (5, 3), (1000, 24), (4097, 64)]:
        H = rng.integers(0, 4, size=(n, k)).astype(np.float32)   # many ties
        H[0] = 0.0
        got = m.labels(to_dev(H, DEV)).cpu().numpy()
        assert np.array_equal(got, oracle.labels(H))


@pytest.mark.parametrize("n", [1, 7, 2000])
def test_stats_matches_oracle(m, n):
    rng = np.random.default_rng(n)
    S = rng.random((n, n)).astype(np.float32)
    if n > 5:
        S[1, 2] = np.nan
        S[3, 4] = -np.inf
    got = m.stats(to_dev(S, DEV, pad4=True)).cpu().numpy()
    s, sq, bad = oracle.stats(S)
    assert got[2] == bad
    assert abs(got[0] - s) <= 1e-12 * abs(s)
    assert abs(got[1] - sq) <= 1e-12 * sq


@pytest.mark.parametrize("n", [513, 1024])
def test_stats_full_float_range(m, n):
    # the pass widens a group of four values by moving bit fields when all four
    # are normal and through the conversion otherwise: mix every class into the
    # groups -- both signs over the whole normal range, the extreme normals,
    # signed zeros, subnormals, infinities and NaN (n = 513 adds a ragged tail)
    rng = np.random.default_rng(n)
    mag = 10.0 ** rng.uniform(-37.0, 37.0, size=(n, n))
    S = (rng.choice([-1.0, 1.0], size=(n, n)) * mag).astype(np.float32)
    specials = np.array([0.0, -0.0, 1e-40, -3e-42, 1.4e-45, np.float32(2.0 ** -126),
                         -np.float32(2.0 ** -126), np.finfo(np.float32).max,
                         -np.finfo(np.float32).max, np.inf, -np.inf, np.nan], dtype=np.float32)
    pick = rng.random((n, n)) < 0.05
    S[pick] = rng.choice(specials, size=int(pick.sum()))
    got = m.stats(to_dev(S, DEV, pad4=True)).cpu().numpy()
    s, sq, bad = oracle.stats(S)
    absum = float(np.abs(np.where(np.isfinite(S), S, 0.0).astype(np.float64)).sum())
    assert got[2] == bad
    assert abs(got[0] - s) <= 1e-12 * absum   # relative to sum |S|: the signs cancel
    assert abs(got[1] - sq) <= 1e-12 * sq


@pytest.mark.parametrize("n,k", [(2000, 24), (2000, 8), (1999, 7), (2001, 33), (1500, 64), (3, 1), (1, 1)])
def test_sh_matches_oracle(m, n, k):
    _, _, S = corr_problem(n, 60, seed=n)
    X = synth.uniform_h0(n, k, 0.5, seed=k)
    Y = m.sh(to_dev(S, DEV, pad4=True), to_dev(X, DEV)).cpu().numpy()
    ref = S.astype(np.float64) @ X.astype(np.float64)
    assert rel_fro(Y, ref) <= 1e-4
    assert rel_fro(Y, ref) <= 2e-6   # regression guard: fp32-class error, far inside the bound


def test_sh_partials_staged_in_several_batches(m):
    # k = 64 at n = 2,000: 7 contraction splits (one CTA per SM at this k),
    # while the epilogue's shared memory holds 5 partial tiles, so each
    # tile's partials arrive in two batches (summed in split order either way)
    rng = np.random.default_rng(5)
    A = rng.random((2000, 2000), dtype=np.float32)
    S = ((A + A.T) * np.float32(0.5)).astype(np.float32)
    X = synth.uniform_h0(2000, 64, 0.5, seed=3)
    Y = m.sh(to_dev(S, DEV), to_dev(X, DEV)).cpu().numpy()
    ref = S.astype(np.float64) @ X.astype(np.float64)
    assert rel_fro(Y, ref) <= 2e-6


# n = 4,100: 561 tiles, several per CTA of the persistent Gram (both TMEM
# accumulator sets and their barrier phases in use)
@pytest.mark.parametrize("T,n", [(250, 2000), (250, 1999), (2, 37), (17, 130), (1000, 600), (60, 4100)])
def test_corr_builder(m, T, n):
    R, _, _ = synth.workload("corr_n2000_k8", seed=T + n, n=n, T=T)
    S = m.build_corr(to_dev(R, DEV, pad4=True)).cpu().numpy()
    ref = oracle.corr_abs(R)
    assert np.max(np.abs(S - ref)) <= 5e-6
    assert np.all(np.diag(S) == 1.0)


def test_corr_builder_zero_variance_column(m):
    R, _, _ = synth.workload("corr_n2000_k8", seed=1, n=64, T=40)
    R[:, 5] = 3.25
    S = m.build_corr(to_dev(R, DEV)).cpu().numpy()
    ref = oracle.corr_abs(R)
    assert np.max(np.abs(S - ref)) <= 5e-6
    assert S[5, 5] == 1.0 and np.all(S[5, np.arange(64) != 5] == 0.0)


# T <= 1024 ranks by a sort held in registers (32 keys per lane at most;
# T = 20, 33, 400, 1024 fill 1, 2, 16, 32 keys per lane), T <= 2048 by a sort
# in shared memory, larger T by the counting kernel
@pytest.mark.parametrize("T,n,frac,sign", [(250, 2000, 0.05, 1), (1000, 1999, 0.05, 1),
                                           (100, 130, 0.1, -1), (20, 2, 0.1, 1), (1, 5, 1.0, 1),
                                           (33, 500, 0.1, -1), (400, 333, 0.05, 1),
                                           (1024, 300, 0.05, -1), (1025, 70, 0.05, 1),
                                           (2048, 45, 0.05, -1), (2100, 37, 0.05, 1),
                                           (80, 4100, 0.1, 1)])
def test_tpdm_builder(m, T, n, frac, sign):
    R, _, _ = synth.workload("tpdm_n20000_k24", seed=T + n, n=n, T=T)
    S = m.build_tpdm(to_dev(R, DEV, pad4=True), frac, sign).cpu().numpy()
    ref = oracle.tpdm(R, frac, sign)
    assert np.max(np.abs(S - ref)) <= 1e-5 * np.max(np.abs(ref))
    assert abs(np.trace(S.astype(np.float64)) - n) <= 1e-5 * n


@pytest.mark.parametrize("T,n,sign", [(64, 40, 1), (64, 40, -1), (1000, 24, -1), (1500, 16, 1)])
def test_tpdm_builder_with_ties(m, T, n, sign):
    # integer returns: long runs of equal values, ranked towards the earlier
    # day; a third of the zeros are -0.0, which ties with +0.0
    rng = np.random.default_rng(T + n)
    R = rng.integers(-3, 4, size=(T, n)).astype(np.float32)
    R[(R == 0) & (rng.random((T, n)) < 0.33)] = -0.0
    S = m.build_tpdm(to_dev(R, DEV), 0.125, sign).cpu().numpy()
    ref = oracle.tpdm(R, 0.125, sign)
    assert np.max(np.abs(S - ref)) <= 1e-5 * np.max(np.abs(ref))


@pytest.mark.parametrize("n,k,block", [(2000, 8, 16), (1999, 24, 16), (600, 6, 8)])
def test_spectral_probe_matches_lapack(m, n, k, block):
    _, _, S = corr_problem(n, 250, seed=n)
    ev = m.spectral_probe(to_dev(S, DEV, pad4=True), k + 2, block=block, max_iter=60, tol=1e-9)
    ref = oracle.top_eigenvalues(S, k + 2)
    assert np.max(np.abs(ev - ref)) <= 1e-5 * ref[0]
    assert (oracle.gap_ratio(ev, k) >= 5.0) == (oracle.gap_ratio(ref, k) >= 5.0)


def test_spectral_probe_64_eigenvalues_planted_rank_24(m):
    # the 64-eigenvalue probe on the planted rank-24 workload (24 groups, 10%
    # boundary instruments, T = 500), at a size LAPACK answers in seconds:
    # 24 leading eigenvalues and 40 from the noise bulk
    _, _, S = corr_problem(4000, 500, seed=11, name="corr_n20000_k24")
    ev = m.spectral_probe(to_dev(S, DEV, pad4=True), 64, block=16, max_iter=60, tol=1e-9)
    ref = oracle.top_eigenvalues(S, 64)
    assert np.max(np.abs(ev - ref)) <= 1e-5 * ref[0]
    assert (oracle.gap_ratio(ev, 24) >= 5.0) == (oracle.gap_ratio(ref, 24) >= 5.0)


def test_spectral_probe_low_rank_block_matrix(m):
    # rank 3 < block: the first Krylov block is rank deficient
    S, _ = synth.planted_block_matrix([50, 30, 20], order_seed=2)
    ev = m.spectral_probe(to_dev(S, DEV), 5, block=8, max_iter=10, tol=1e-9)
    np.testing.assert_allclose(ev, [50, 30, 20, 0, 0], atol=1e-4)


def test_sh_long_contraction_has_no_drift(m):
    # each CTA contracts ~4,000 columns: the tensor-core accumulator is folded
    # into round-to-nearest fp32 registers every few stages, so the error stays
    # at fp32 level however long the row
    n, k = 12000, 24
    rng = np.random.default_rng(12)
    A = rng.random((n, n), dtype=np.float32)
    S = (A + A.T) * np.float32(0.5)
    del A
    X = synth.uniform_h0(n, k, 0.5, seed=3)
    Y = m.sh(to_dev(S, DEV), to_dev(X, DEV)).cpu().numpy()
    ref = S.astype(np.float64) @ X.astype(np.float64)
    assert rel_fro(Y, ref) <= 2e-6
    # the one-signed part of the error does not grow with the row length
    assert abs(float(np.mean((Y - ref) / ref))) <= 2e-6
