"""Parity at the benchmark's full size (n = 100,000, k = 24, T = 1,000).

The oracle cannot hold a 100,000 x 100,000 fp64 matrix.  It computes
sampled rows one by one from the same returns window (rows of |corr| and of
the TPDM, the matching rows of S X, one AdaGrad step on those rows), and it
runs whole fits on the device's S read in row chunks (``DeviceRowChunks``):
three full-batch AdaGrad iterations on |corr| from the seeded start, and one
Block-SVRG epoch at the workload's block of 8,192 rows on the TPDM.  The
library runs exactly as bench.py times it (same builder, same S-stream
launch configuration).
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import DeviceRowChunks, assert_labels_differ_only_on_near_ties, rel_fro

pytestmark = pytest.mark.gpu
DEV = "cuda:0"
ROWS = np.array([0, 1, 2, 127, 128, 4095, 12345, 33333, 50000, 54321, 77777, 99872, 99998, 99999])


@pytest.fixture(scope="module")
def big():
    import torch
    from symmetric_nmf_clustering_b200 import build
    build.build()
    import symmetric_nmf_clustering_b200 as m
    R, planted, spec = synth.workload("corr_n100000_k24", seed=0)
    Rd = torch.from_numpy(R).to(DEV)
    S = m.alloc_S(spec["n"], DEV)
    yield m, R, Rd, S, spec
    del S, Rd
    torch.cuda.empty_cache()


def test_fullsize_corr_rows_sh_rows_and_one_step(big):
    import torch
    m, R, Rd, S, spec = big
    n, k = spec["n"], spec["k"]
    m.build_corr(Rd, out=S)
    torch.cuda.synchronize()
    # |corr| rows: the oracle's definition row by row (centred, normalised columns)
    S_rows_gpu = S[torch.as_tensor(ROWS, device=DEV)].cpu().numpy()
    S_rows = oracle.corr_abs_rows(R, ROWS)
    assert np.max(np.abs(S_rows_gpu - S_rows)) <= 5e-6

    # S X on the sampled rows
    X = synth.uniform_h0(n, k, 0.1, seed=5)
    Xd = torch.from_numpy(X).to(DEV)
    Y = m.sh(S, Xd)
    torch.cuda.synchronize()
    P_rows = S_rows @ X.astype(np.float64)
    assert rel_fro(Y[torch.as_tensor(ROWS, device=DEV)].cpu().numpy(), P_rows) <= 1e-4

    # one full-batch step from H0 = X, G0 = 0 on the sampled rows
    H, st = m.fit(S, k, H0=Xd, max_iters=1, rel_tol=0.0)
    torch.cuda.synchronize()
    X64 = X.astype(np.float64)
    A = X64.T @ X64
    g = 4.0 * (X64[ROWS] @ A - P_rows)
    H1, _ = oracle.adagrad_step(X64[ROWS], np.zeros_like(g), g, 0.1, 1e-10)
    assert rel_fro(H[torch.as_tensor(ROWS, device=DEV)].cpu().numpy(), H1) <= 1e-4
    assert st["iters"] == 1 and st["evaluations"] == 2


def test_fullsize_tpdm_rows(big):
    import torch
    m, _, _, S, spec = big
    n = spec["n"]
    R, _, _ = synth.workload("tpdm_n100000_k24", seed=0)
    Rd = torch.from_numpy(R).to(DEV)
    m.build_tpdm(Rd, 0.05, 1, out=S)
    torch.cuda.synchronize()
    S_rows = oracle.tpdm_rows(R, ROWS, 0.05, 1)
    got = S[torch.as_tensor(ROWS, device=DEV)].cpu().numpy()
    assert np.max(np.abs(got - S_rows)) <= 1e-5 * np.max(np.abs(S_rows))
    # the diagonal sums to n exactly in exact arithmetic
    diag = torch.diagonal(S).double().sum().item()
    assert abs(diag - n) <= 1e-4 * n


def test_fullsize_labels_bit_exact(big):
    import torch
    m, _, _, _, spec = big
    n, k = spec["n"], spec["k"]
    rng = np.random.default_rng(9)
    H = rng.integers(0, 50, size=(n, k)).astype(np.float32) / 7.0   # many ties
    got = m.labels(torch.from_numpy(H).to(DEV)).cpu().numpy()
    assert np.array_equal(got, oracle.labels(H))


def test_fullsize_adagrad_trajectory_against_streamed_oracle(big):
    # the benchmark's workload: |corr| at n = 100,000, k = 24, seeded start,
    # three full-batch iterations (four loss evaluations) on both sides
    import torch
    m, R, Rd, S, spec = big
    n, k = spec["n"], spec["k"]
    m.build_corr(Rd, out=S)
    torch.cuda.synchronize()
    X = DeviceRowChunks(S)
    s_sum, sq, bad = X.stats()
    assert bad == 0
    H0 = oracle.scale_matched_init(s_sum, n, k, 1000)
    H0g, st0 = m.fit(S, k, seed=1000, max_iters=0, rel_tol=0.0)
    assert np.array_equal(H0g.cpu().numpy(), H0)                 # seeded start bit-exact
    assert st0["s_sqnorm"] == pytest.approx(sq, rel=1e-12)
    Hg, st = m.fit(S, k, seed=1000, max_iters=3, rel_tol=0.0, history=True)
    r = oracle.fit_adagrad(X, k, H0, max_iters=3, S_sqnorm=sq)
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    Hg = Hg.cpu().numpy()
    assert rel_fro(Hg, r.H) <= 1e-3
    lg = m.labels(torch.from_numpy(Hg).to(DEV)).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)


def test_fullsize_block_svrg_epoch_against_streamed_oracle(big):
    # the heavy-tailed workload's TPDM at n = 100,000, one Block-SVRG epoch at
    # b = 8,192 (13 blocks, the last of 1,696 rows), growth off
    import torch
    m, _, _, S, spec = big
    n, k = spec["n"], spec["k"]
    R, _, _ = synth.workload("tpdm_n100000_k24", seed=0)
    Rd = torch.from_numpy(R).to(DEV)
    m.build_tpdm(Rd, 0.05, 1, out=S)
    torch.cuda.synchronize()
    del Rd
    X = DeviceRowChunks(S)
    s_sum, sq, _ = X.stats()
    H0 = oracle.scale_matched_init(s_sum, n, k, 1000)
    Hg, st = m.fit(S, k, seed=1000, solver="block_svrg", block_rows=8192, grow=False,
                   max_iters=1, rel_tol=0.0, history=True)
    r = oracle.fit_block_svrg(X, k, H0, max_epochs=1, block_rows=8192, grow=False, seed=1000,
                              S_sqnorm=sq)
    assert st["epochs"] == r.epochs == 1 and st["block_final"] == r.block_final == 8192
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    Hg = Hg.cpu().numpy()
    assert rel_fro(Hg, r.H) <= 1e-3
    lg = m.labels(torch.from_numpy(Hg).to(DEV)).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)
