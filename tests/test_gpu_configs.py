"""Parity at the two n = 20,000 workloads' stated sizes.

  rank-24 |corr|  n = 20,000, T = 500, 24 planted groups with 10% boundary
                  instruments: 500 full-batch AdaGrad iterations (lr 0.1,
                  eps 1e-10) from the seeded start, and the 64 leading
                  eigenvalues by the spectral probe against LAPACK
  heavy tail      n = 20,000, T = 1,000, Student-t(3): the TPDM, 50 Block-SVRG
                  epochs at b = 2,048 with growth

Both sides start from the same float32 S (the oracle's), so builder error
does not enter the fit.  Tolerances: H 1e-3 relative Frobenius, loss history
1e-4 (1e-4 of the loss plus 1e-5 ||S||^2 where the fit explains nearly all
of ||S||^2 and the trace identity cancels), labels equal except on near-ties
the H difference explains; the eigenvalues within 1e-5 lambda_1.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_labels_differ_only_on_near_ties, rel_fro, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


@pytest.fixture(scope="module")
def m():
    import torch
    from symmetric_nmf_clustering_b200 import build
    build.build()
    import symmetric_nmf_clustering_b200 as m
    torch.cuda.init()
    return m


@pytest.fixture(scope="module")
def corr20k():
    R, planted, spec = synth.workload("corr_n20000_k24", seed=0)
    S = oracle.corr_abs(R).astype(np.float32)
    return S, planted, spec


def test_rank24_corr_n20000_500_iterations(m, corr20k):
    import torch
    S, planted, spec = corr20k
    n, k = spec["n"], spec["k"]
    s_sum, sq, _ = oracle.stats(S)
    Sd = to_dev(S, DEV, pad4=True)
    H, st = m.fit(Sd, k, seed=1000, max_iters=500, rel_tol=0.0, history=True)
    torch.cuda.synchronize()
    Hg = H.cpu().numpy()
    r = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 1000), max_iters=500,
                           S_sqnorm=sq)
    assert st["iters"] == 500
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    assert rel_fro(Hg, r.H) <= 1e-3
    lg = m.labels(H).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)
    # the planted recovery is the same on both sides
    assert abs(oracle.ari(lg, planted) - oracle.ari(oracle.labels(r.H), planted)) <= 1e-3


def test_rank24_corr_n20000_probe_64_eigenvalues(m, corr20k):
    import scipy.linalg
    S, _, spec = corr20k
    n = spec["n"]
    ev = m.spectral_probe(to_dev(S, DEV, pad4=True), 64, block=16, max_iter=60, tol=1e-9)
    ref = scipy.linalg.eigh(S.astype(np.float64), eigvals_only=True,
                            subset_by_index=[n - 64, n - 1])[::-1]
    err = float(np.max(np.abs(ev - ref)))
    print(f"64 leading eigenvalues: max deviation {err:.3g} (lambda_1 = {ref[0]:.6g})")
    assert err <= 1e-5 * ref[0]
    assert (oracle.gap_ratio(ev, 24) >= 5.0) == (oracle.gap_ratio(ref, 24) >= 5.0)


def test_heavy_tail_tpdm_n20000_block_svrg_50_epochs(m):
    import torch
    R, planted, spec = synth.workload("tpdm_n20000_k24", seed=0)
    n, k = spec["n"], spec["k"]
    S = oracle.tpdm(R, 0.05, 1).astype(np.float32)
    s_sum, sq, _ = oracle.stats(S)
    Sd = to_dev(S, DEV, pad4=True)
    H, st = m.fit(Sd, k, seed=5, solver="block_svrg", block_rows=2048, grow=True, max_iters=50,
                  rel_tol=0.0, history=True)
    torch.cuda.synchronize()
    Hg = H.cpu().numpy()
    r = oracle.fit_block_svrg(S, k, oracle.scale_matched_init(s_sum, n, k, 5), max_epochs=50,
                              block_rows=2048, grow=True, seed=5, S_sqnorm=sq)
    assert st["epochs"] == r.epochs and st["block_final"] == r.block_final
    assert st["iters"] == r.iters
    # the snapshot losses: 1e-4 of the loss plus the trace identity's
    # cancellation allowance 1e-5 ||S||^2 (the loss carries the absolute error
    # of ||S||^2 - 2 tr, and this fit explains about 98% of ||S||^2)
    dL = np.abs(np.asarray(st["history"]) - np.asarray(r.history))
    print(f"snapshot losses: max |dL| = {dL.max():.4g}, ||S||^2 = {sq:.6g}, "
          f"H rel = {rel_fro(Hg, r.H):.3g}")
    assert np.all(dL <= 1e-4 * np.asarray(r.history) + 1e-5 * sq)
    assert rel_fro(Hg, r.H) <= 1e-3
    lg = m.labels(H).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)
