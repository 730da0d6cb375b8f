"""GPU parity of symnmf_spherical_kmeans against the CPU oracle.

Both sides get the same float32 S (built by the oracle) and the same seed.
The labels are argmax decisions on scores the GPU forms in float32 and the
oracle in float64, so a row whose best and second-best cosine scores lie
within TIE of each other may legitimately go either way, after which the two
trajectories may part.  Hence:
  decided prefix  up to the first step at which the oracle saw a gap below
                  TIE: labels bit-equal, centroids relative Frobenius <= 1e-5,
                  same step count and convergence flag;
  the first near tie  labels equal on every row with an oracle gap >= TIE;
                  on the others the GPU label scores within TIE of the best;
  the end state   a fixed point checked in float64 on the host: every label
                  scores within TIE of its row's best under the returned
                  centroids, and each centroid is its members' normalised sum.
TIE = 1e-5 in cosine units: the S-stream product is float32-accurate (relative
error ~1e-6 of ||S_i|| ||c||) and the centroids are stored in float32.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import corr_problem, rel_fro, to_dev, tpdm_problem

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
TIE = 1e-5


@pytest.fixture(scope="module")
def m():
    import torch
    from symmetric_nmf_clustering_b200 import build
    build.build()
    import symmetric_nmf_clustering_b200 as m
    torch.cuda.init()
    return m


def _km(m, S, k, seed, max_iters):
    import torch
    Sd = to_dev(S, DEV, pad4=True)
    lab, cent, steps, conv = m.spherical_kmeans(Sd, k, seed=seed, max_iters=max_iters)
    torch.cuda.synchronize()
    return lab.cpu().numpy(), cent.cpu().numpy().T.astype(np.float64), steps, conv


def _unit_rows(S):
    S = S.astype(np.float64)
    nr = np.sqrt((S * S).sum(axis=1))
    return np.where(nr[:, None] > 0, S / np.where(nr > 0, nr, 1.0)[:, None], 0.0)


def _check_fixed_point(S, k, lab, C):
    """The returned state is a spherical k-means fixed point (float64 check)."""
    X = _unit_rows(S)
    scores = X @ C.T
    best = scores.max(axis=1)
    mine = scores[np.arange(len(lab)), lab]
    assert np.all(best - mine <= TIE), float((best - mine).max())
    for c in range(k):
        members = lab == c
        if members.any():
            v = X[members].sum(axis=0)
            if np.linalg.norm(v) > 0:
                assert rel_fro(C[c], v / np.linalg.norm(v)) <= 1e-5, c
    np.testing.assert_allclose(np.linalg.norm(C, axis=1), 1.0, atol=1e-5)


def _compare(m, S, k, seed, max_iters=100):
    ref = oracle.spherical_kmeans(S, k, seed=seed, max_iters=max_iters)
    lab, C, steps, conv = _km(m, S, k, seed, max_iters)
    near = [t for t, g in enumerate(ref.min_gap) if g < TIE]
    if not near:
        assert steps == ref.steps and conv == ref.converged
        assert np.array_equal(lab, ref.labels)
        assert rel_fro(C, ref.centroids) <= 1e-5
    else:
        t0 = near[0] + 1   # the step whose assignment met a near tie
        if t0 > 1:
            p = oracle.spherical_kmeans(S, k, seed=seed, max_iters=t0 - 1)
            lp, Cp, sp, _ = _km(m, S, k, seed, t0 - 1)
            assert sp == p.steps and np.array_equal(lp, p.labels)
            assert rel_fro(Cp, p.centroids) <= 1e-5
        # the step with the near tie, against the oracle's own scores
        p = oracle.spherical_kmeans(S, k, seed=seed, max_iters=t0 - 1) if t0 > 1 else None
        X = _unit_rows(S)
        Cprev = p.centroids if p is not None else X[oracle.forgy_indices(len(S), k, seed)]
        scores = X @ Cprev.T
        srt = np.sort(scores, axis=1)
        gap = srt[:, -1] - srt[:, -2]
        lt, _, _, _ = _km(m, S, k, seed, t0)
        decided = gap >= TIE
        assert np.array_equal(lt[decided], np.argmax(scores, axis=1)[decided])
        assert np.all(srt[:, -1] - scores[np.arange(len(lt)), lt] <= TIE)
    if conv:
        _check_fixed_point(S, k, lab, C)
    return ref, lab, steps, conv


@pytest.mark.parametrize("n,T,k,seed", [(2000, 250, 8, 7), (2000, 250, 8, 0), (1999, 120, 24, 1),
                                        (777, 80, 33, 2), (300, 60, 64, 3), (5, 20, 3, 5)])
def test_corr_parity(m, n, T, k, seed):
    _, _, S = corr_problem(n, T, seed)
    _compare(m, S, k, seed)


def test_tpdm_parity(m):
    _, _, S = tpdm_problem(1500, 400, 4)
    _compare(m, S, 12, 4)


def test_decided_run_is_exact(m):
    # this start meets no near tie on the way (oracle gap >= 6e-5 at every step)
    _, _, S = corr_problem(2000, 250, 7)
    ref = oracle.spherical_kmeans(S, 8, seed=7)
    assert min(ref.min_gap) >= TIE
    lab, C, steps, conv = _km(m, S, 8, 7, 100)
    assert (steps, conv) == (ref.steps, ref.converged)
    assert np.array_equal(lab, ref.labels)
    assert rel_fro(C, ref.centroids) <= 1e-5


@pytest.mark.parametrize("seed", [0, 1, 3, 4])
def test_planted_blocks(m, seed):
    S, planted = synth.planted_block_matrix([40, 35, 30, 25], order_seed=seed)
    lab, C, steps, conv = _km(m, S, 4, seed, 20)
    assert conv and oracle.ari(lab, planted) == 1.0
    ref = oracle.spherical_kmeans(S, 4, seed=seed, max_iters=20)
    assert np.array_equal(lab, ref.labels) and steps == ref.steps


def test_single_step_does_not_converge(m):
    _, _, S = corr_problem(500, 60, 9)
    lab, C, steps, conv = _km(m, S, 6, 9, 1)
    ref = oracle.spherical_kmeans(S, 6, seed=9, max_iters=1)
    assert steps == 1 and not conv and ref.steps == 1 and not ref.converged
    assert ref.min_gap[0] >= TIE
    assert np.array_equal(lab, ref.labels)
    assert rel_fro(C, ref.centroids) <= 1e-5


def test_n_equals_one_and_zero_row(m):
    S = np.array([[2.0]], dtype=np.float32)
    lab, C, steps, conv = _km(m, S, 1, 0, 10)
    assert list(lab) == [0] and steps == 2 and conv
    assert abs(C[0, 0] - 1.0) <= 1e-7
    S = np.array([[0, 0, 0], [0, 1, 0.1], [0, 0.1, 1]], dtype=np.float32)
    ref = oracle.spherical_kmeans(S, 2, seed=0, max_iters=5)
    lab, C, steps, conv = _km(m, S, 2, 0, 5)
    assert np.array_equal(lab, ref.labels) and lab[0] == 0


def test_deterministic(m):
    _, _, S = corr_problem(1999, 120, 1)
    a = _km(m, S, 24, 1, 100)
    b = _km(m, S, 24, 1, 100)
    assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1]) and a[2:] == b[2:]


def test_errors(m):
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    S = to_dev(np.eye(8, dtype=np.float32), DEV)
    for kw in [dict(k=0), dict(k=9), dict(k=65), dict(k=2, max_iters=0)]:
        k = kw.pop("k")
        with pytest.raises(L.SymNMFError):
            m.spherical_kmeans(S, k, **kw)
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(L.SymNMFError) as e:
        m.spherical_kmeans(S, 2, ws=ws)
    assert "workspace" in str(e.value)
