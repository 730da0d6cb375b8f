"""GPU parity of symnmf_fit against the CPU oracle.

Both sides get the same float32 S (built by the oracle) and the same start.
  step parity        same H_t, G_t: one update; H, G relative 1e-4, loss 1e-5
  trajectory parity  same seeded H0, fixed iteration count: H relative
                     Frobenius <= 1e-3, loss history 1e-4, labels and ARI equal
  Block-SVRG         same permutation spec: H <= 1e-3, snapshot losses 1e-4
"""
import math

import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_labels_differ_only_on_near_ties, corr_problem, rel_fro, to_dev, tpdm_problem

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


def _fit(m, S, k, **kw):
    import torch
    Sd = to_dev(S, DEV, pad4=True)
    H0 = kw.pop("H0", None)
    G = kw.pop("G", None)
    Gd = to_dev(G.astype(np.float32), DEV) if G is not None else None
    H, st = m.fit(Sd, k, H0=to_dev(H0, DEV) if H0 is not None else None, G=Gd, history=True, **kw)
    torch.cuda.synchronize()
    out = H.cpu().numpy()
    return out, st, (Gd.cpu().numpy() if Gd is not None else None)


def test_seeded_init_is_bit_exact(m):
    _, _, S = corr_problem(2000, 250, seed=0)
    H, st, _ = _fit(m, S, 8, seed=1000, max_iters=0, rel_tol=0.0)
    s_sum, sq, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, 2000, 8, 1000)
    assert np.array_equal(H, H0)
    assert st["iters"] == 0 and st["evaluations"] == 1
    L0 = oracle.trace_loss(sq, H0.astype(np.float64), S.astype(np.float64) @ H0.astype(np.float64))
    assert abs(st["loss"] - L0) <= 1e-6 * L0
    assert st["s_sqnorm"] == pytest.approx(sq, rel=1e-12)
    assert st["s_mean"] == pytest.approx(s_sum / 2000 ** 2, rel=1e-12)


@pytest.mark.parametrize("n,k", [(2000, 8), (1999, 24), (777, 33), (300, 64), (5, 3), (1, 1)])
def test_one_step_parity(m, n, k):
    _, _, S = corr_problem(n, 80, seed=n + k)
    rng = np.random.default_rng(k)
    H = (rng.random((n, k)) * 0.3).astype(np.float32)
    G = (rng.random((n, k)) * 0.01).astype(np.float32)
    Hg, st, Gg = _fit(m, S, k, H0=H, G=G, max_iters=1, rel_tol=0.0)
    r = oracle.fit_adagrad(S, k, H, max_iters=1, G0=G)
    # the step divides g = 4(H A - S H) -- a near-cancellation -- by sqrt(G),
    # so S H's fp32-level error shows up amplified: per-iteration bar 1e-4
    assert rel_fro(Hg, r.H) <= 1e-4
    assert rel_fro(Gg, r.G) <= 1e-4
    assert np.all(Hg >= 0)
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-5)
    assert st["iters"] == 1 and st["evaluations"] == 2


def test_trajectory_parity_small_corr_workload(m):
    # 2,000 instruments, 8 planted groups, T = 250, 200 iterations (lr 0.1, eps 1e-10)
    R, planted, S = corr_problem(2000, 250, seed=0)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 8, seed=1000, max_iters=200, rel_tol=0.0)
    H0 = oracle.scale_matched_init(s_sum, 2000, 8, 1000)
    r = oracle.fit_adagrad(S, 8, H0, lr=0.1, eps=1e-10, max_iters=200, S_sqnorm=sq)
    assert rel_fro(Hg, r.H) <= 1e-3
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    lg = m.labels(to_dev(Hg, DEV)).cpu().numpy()      # the library's labels kernel
    lo = oracle.labels(r.H)                           # the oracle's labels of its own H
    assert np.array_equal(lg, lo)
    assert oracle.ari(lg, planted) == oracle.ari(lo, planted)


def test_trajectory_parity_rank24_boundary_workload(m):
    # 24 groups with 10% boundary instruments at a reduced n (same recipe)
    R, planted, S = corr_problem(4000, 500, seed=1, name="corr_n20000_k24")
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 24, seed=1001, max_iters=100, rel_tol=0.0)
    H0 = oracle.scale_matched_init(s_sum, 4000, 24, 1001)
    r = oracle.fit_adagrad(S, 24, H0, max_iters=100, S_sqnorm=sq)
    assert rel_fro(Hg, r.H) <= 1e-3
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    lg = m.labels(to_dev(Hg, DEV)).cpu().numpy()
    lo = oracle.labels(r.H)
    assert_labels_differ_only_on_near_ties(lg, lo, Hg, r.H)


def test_convergence_stop(m):
    _, _, S = corr_problem(1000, 120, seed=4)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 8, seed=7, max_iters=3000, rel_tol=1e-4, check_every=7)
    H0 = oracle.scale_matched_init(s_sum, 1000, 8, 7)
    r = oracle.fit_adagrad(S, 8, H0, max_iters=3000, rel_tol=1e-4, S_sqnorm=sq)
    assert st["converged"] == 1 and r.converged
    assert abs(st["iters"] - r.iters) <= 2
    assert st["rel_change"] < 1e-4
    assert rel_fro(Hg, r.H) <= 1e-3        # iterates near convergence barely move
    assert st["evaluations"] == st["iters"] + 1


def test_block_svrg_parity(m):
    # heavy-tailed TPDM workload at a reduced n, b = 256, growth on
    _, planted, S = tpdm_problem(2000, 1000, seed=0)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 24, solver="block_svrg", seed=5, max_iters=12, rel_tol=0.0,
                     block_rows=256, grow=True, stall_tol=1e-2)
    H0 = oracle.scale_matched_init(s_sum, 2000, 24, 5)
    r = oracle.fit_block_svrg(S, 24, H0, max_epochs=12, block_rows=256, grow=True,
                              stall_tol=1e-2, seed=5, S_sqnorm=sq)
    assert st["solver_used"] == 1
    assert st["block_final"] == r.block_final
    assert st["epochs"] == r.epochs and st["iters"] == r.iters
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    assert rel_fro(Hg, r.H) <= 1e-3


def test_block_svrg_grows_to_full_batch(m):
    _, _, S = corr_problem(600, 100, seed=9)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 6, solver="block_svrg", seed=3, max_iters=20, rel_tol=0.0,
                     block_rows=64, grow=True, stall_tol=10.0)
    H0 = oracle.scale_matched_init(s_sum, 600, 6, 3)
    r = oracle.fit_block_svrg(S, 6, H0, max_epochs=20, block_rows=64, grow=True,
                              stall_tol=10.0, seed=3, S_sqnorm=sq)
    assert r.block_final == 600 and st["block_final"] == 600
    assert (st["epochs"], st["iters"]) == (r.epochs, r.iters)
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    assert rel_fro(Hg, r.H) <= 1e-3


def test_auto_selects_solver_from_gap(m):
    _, _, S = corr_problem(1000, 250, seed=2)
    ev = oracle.top_eigenvalues(S, 10)
    _, st, _ = _fit(m, S, 8, solver="auto", eigvals=list(ev), max_iters=3, rel_tol=0.0)
    want = 0 if oracle.gap_ratio(ev, 8) >= 5.0 else 1
    assert st["solver_used"] == want
    assert st["gamma"] == pytest.approx(oracle.gap_ratio(ev, 8), rel=1e-12)
    # and with the built-in probe
    _, st2, _ = _fit(m, S, 8, solver="auto", max_iters=3, rel_tol=0.0, probe_max_iter=60,
                     probe_tol=1e-9)
    assert st2["solver_used"] == want
    assert st2["gamma"] == pytest.approx(oracle.gap_ratio(ev, 8), rel=1e-3)


def test_deterministic_bitwise(m):
    _, _, S = corr_problem(1500, 100, seed=11)
    a, sa, _ = _fit(m, S, 12, seed=3, max_iters=40, rel_tol=0.0)
    b, sb, _ = _fit(m, S, 12, seed=3, max_iters=40, rel_tol=0.0)
    assert np.array_equal(a, b)
    assert np.array_equal(sa["history"], sb["history"])


def test_resume_from_returned_h_and_g(m):
    # a fit resumed from the (H, G) another fit returned continues it exactly:
    # 40 updates, then 30 more from there, equal 70 updates in one call (the
    # Gram of the resumed iterate is recomputed in the same fixed order)
    n, k = 1200, 8
    _, _, S = corr_problem(n, 150, seed=21)
    zeros = np.zeros((n, k), np.float32)
    H70, s70, G70 = _fit(m, S, k, seed=9, G=zeros, max_iters=70, rel_tol=0.0)
    H40, s40, G40 = _fit(m, S, k, seed=9, G=zeros, max_iters=40, rel_tol=0.0)
    Hr, sr, Gr = _fit(m, S, k, H0=H40, G=G40, max_iters=30, rel_tol=0.0)
    assert np.array_equal(Hr, H70) and np.array_equal(Gr, G70)
    assert np.array_equal(sr["history"], s70["history"][40:])
    assert np.array_equal(s40["history"], s70["history"][:41])


def test_planted_blocks_recovered_on_gpu(m):
    S, planted = synth.planted_block_matrix([60] * 5, order_seed=3)
    Hg, st, _ = _fit(m, S, 5, seed=1003, max_iters=600, rel_tol=0.0)
    lg = m.labels(to_dev(Hg, DEV)).cpu().numpy()
    assert oracle.ari(lg, planted) == 1.0


def test_errors(m):
    import torch
    from symmetric_nmf_clustering_b200 import _lib
    S = np.ones((16, 16), dtype=np.float32)
    S[2, 3] = np.nan
    with pytest.raises(_lib.SymNMFError) as e:
        _fit(m, S, 2, max_iters=2)
    assert e.value.status == _lib.SYMNMF_ERR_NONFINITE
    Sd = to_dev(np.eye(16, dtype=np.float32), DEV)
    tiny = torch.empty(256, dtype=torch.uint8, device=DEV)
    with pytest.raises(_lib.SymNMFError) as e:
        m.fit(Sd, 2, ws=tiny)
    assert e.value.status == _lib.SYMNMF_ERR_WORKSPACE


_OTHER_MODE_SCRIPT = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[1])
import symmetric_nmf_clustering_b200 as m
S = torch.from_numpy(np.load(sys.argv[2])).cuda()
H, st = m.fit(S, 8, seed=5, max_iters=70, rel_tol=0.0, history=True)
np.save(sys.argv[3], H.cpu().numpy())
np.save(sys.argv[4], st["history"])
"""


def test_graph_replay_matches_eager_launches(m, tmp_path):
    # the default is eager launches; the subprocess replays the loop as a graph
    import os
    import subprocess
    import sys
    _, _, S = corr_problem(1200, 100, seed=13)
    Hg, st, _ = _fit(m, S, 8, seed=5, max_iters=70, rel_tol=0.0)
    np.save(tmp_path / "S.npy", S)
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, SYMNMF_GRAPHS="1")
    r = subprocess.run([sys.executable, "-c", _OTHER_MODE_SCRIPT, root, str(tmp_path / "S.npy"),
                        str(tmp_path / "H.npy"), str(tmp_path / "hist.npy")],
                       env=env, capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stderr
    assert np.array_equal(np.load(tmp_path / "H.npy"), Hg)
    assert np.array_equal(np.load(tmp_path / "hist.npy"), st["history"])
