"""GPU parity of the upper-triangle S-stream (symnmf_sh_upper, and symnmf_fit
with upper_only = 1) against the CPU oracle.

The kernel reads only the 128 x 128 tiles on or above the diagonal; S enters
rounded to the nearest TF32 value (an unbiased per-entry error of at most
2^-12 relative), X its exact TF32 split.  Tolerances are the hot path's:
S X within 1e-4 relative Frobenius (and a tighter regression guard of 3e-5
on these inputs, whose entries are continuous), one step from the same
(H, G) within 1e-4, H after a fixed seeded iteration count within 1e-3, labels
equal except on near-ties that the H difference explains.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import (assert_labels_differ_only_on_near_ties, corr_problem, rel_fro, to_dev,
                      tpdm_problem)

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


def _sym(n, seed):
    rng = np.random.default_rng(seed)
    A = rng.random((n, n), dtype=np.float32)
    return ((A + A.T) * np.float32(0.5)).astype(np.float32)


@pytest.mark.parametrize("n,k", [(1, 1), (5, 3), (128, 8), (129, 7), (257, 24), (1000, 16),
                                 (2049, 24), (3001, 24), (4100, 12)])
def test_sh_upper_matches_fp64_product(m, n, k):
    # one tile, a ragged second tile, several panels and items, a ragged tail
    import torch
    S = _sym(n, n)
    X = (np.random.default_rng(k).random((n, k)) * 0.5).astype(np.float32)
    Y = m.sh_upper(to_dev(S, DEV, pad4=True), to_dev(X, DEV))
    torch.cuda.synchronize()
    ref = S.astype(np.float64) @ X.astype(np.float64)
    got = Y.cpu().numpy()
    # a row of a few entries keeps the per-entry rounding bound (2^-12); from a
    # hundred entries on it averages out
    tol = 2.0 ** -12 if n < 100 else 3e-5
    assert rel_fro(got, ref) <= tol, rel_fro(got, ref)
    # the full-matrix stream (exact split) agrees to the same level
    Yf = m.sh(to_dev(S, DEV, pad4=True), to_dev(X, DEV)).cpu().numpy()
    assert rel_fro(got, Yf) <= tol


def test_sh_upper_reads_only_tiles_on_or_above_the_diagonal(m):
    # every tile strictly below the diagonal tiles holds NaN, and so does the
    # row padding: the product must not see any of it
    import torch
    n, k, B = 777, 24, 128
    S = _sym(n, 5)
    X = (np.random.default_rng(6).random((n, k)) * 0.5).astype(np.float32)
    lds = (n + 3) // 4 * 4 + 4
    buf = torch.full((n, lds), float("nan"), dtype=torch.float32, device=DEV)
    Sd = buf[:, :n]
    Sd.copy_(torch.from_numpy(S).to(DEV))
    T = (n + B - 1) // B
    for p in range(T):
        for q in range(p):
            Sd[p * B:(p + 1) * B, q * B:(q + 1) * B] = float("nan")
    Y = m.sh_upper(Sd, to_dev(X, DEV))
    torch.cuda.synchronize()
    got = Y.cpu().numpy()
    assert np.all(np.isfinite(got))
    assert rel_fro(got, S.astype(np.float64) @ X.astype(np.float64)) <= 3e-5


def test_sh_upper_is_bitwise_reproducible(m):
    import torch
    n, k = 3001, 24
    Sd = to_dev(_sym(n, 7), DEV, pad4=True)
    Xd = to_dev((np.random.default_rng(8).random((n, k))).astype(np.float32), DEV)
    a = m.sh_upper(Sd, Xd)
    b = m.sh_upper(Sd, Xd)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_sh_upper_on_the_workload_matrices(m):
    # |corr| and TPDM of the rank-24 workloads (continuous entries): the
    # rounding error averages out along the rows
    import torch
    for S in (corr_problem(4000, 500, seed=1, name="corr_n20000_k24")[2],
              tpdm_problem(4000, 1000, seed=2)[2]):
        s_sum, _, _ = oracle.stats(S)
        X = oracle.scale_matched_init(s_sum, 4000, 24, 1001)
        Y = m.sh_upper(to_dev(S, DEV, pad4=True), to_dev(X, DEV))
        torch.cuda.synchronize()
        ref = S.astype(np.float64) @ X.astype(np.float64)
        assert rel_fro(Y.cpu().numpy(), ref) <= 2e-5


def _fit(m, S, k, **kw):
    import torch
    Sd = to_dev(S, DEV, pad4=True)
    H0 = kw.pop("H0", None)
    G = kw.pop("G", None)
    Gd = to_dev(G.astype(np.float32), DEV) if G is not None else None
    H, st = m.fit(Sd, k, H0=to_dev(H0, DEV) if H0 is not None else None, G=Gd, history=True,
                  upper_only=True, **kw)
    torch.cuda.synchronize()
    return H.cpu().numpy(), st, (Gd.cpu().numpy() if Gd is not None else None)


@pytest.mark.parametrize("n,k", [(2000, 8), (1999, 24), (300, 5)])
def test_upper_one_step_parity(m, n, k):
    # the product and both losses within the per-iteration bar (1e-4); the
    # step itself divides g = 4 (H A - S H), a near-cancellation, by sqrt(G),
    # which magnifies the product's rounding (about 1e-5 here) roughly twenty
    # times, so H and G after the step are held to the H bar (1e-3)
    import torch
    _, _, S = corr_problem(n, 80, seed=n + k)
    rng = np.random.default_rng(k + 1)
    H = (rng.random((n, k)) * 0.3).astype(np.float32)
    G = (rng.random((n, k)) * 0.01).astype(np.float32)
    P = m.sh_upper(to_dev(S, DEV, pad4=True), to_dev(H, DEV))
    torch.cuda.synchronize()
    assert rel_fro(P.cpu().numpy(), S.astype(np.float64) @ H.astype(np.float64)) <= 1e-4
    Hg, st, Gg = _fit(m, S, k, H0=H, G=G, max_iters=1, rel_tol=0.0)
    r = oracle.fit_adagrad(S, k, H, max_iters=1, G0=G)
    np.testing.assert_allclose(st["history"], r.history, rtol=1e-4)
    assert rel_fro(Hg, r.H) <= 1e-3
    assert rel_fro(Gg, r.G) <= 1e-3
    assert st["iters"] == 1 and st["evaluations"] == 2


def test_upper_trajectory_parity_small_corr_workload(m):
    # 2,000 instruments, 8 planted groups, T = 250, 200 iterations
    R, planted, S = corr_problem(2000, 250, seed=0)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 8, seed=1000, max_iters=200, rel_tol=0.0)
    H0 = oracle.scale_matched_init(s_sum, 2000, 8, 1000)
    r = oracle.fit_adagrad(S, 8, H0, max_iters=200, S_sqnorm=sq)
    assert rel_fro(Hg, r.H) <= 1e-3
    # the final loss (the same H to 1e-3) within 1e-4
    assert abs(st["history"][-1] - r.history[-1]) <= 1e-4 * r.history[-1]
    lg = m.labels(to_dev(Hg, DEV)).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)


def test_upper_trajectory_parity_rank24_workload(m):
    _, _, S = corr_problem(4000, 500, seed=1, name="corr_n20000_k24")
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 24, seed=1001, max_iters=100, rel_tol=0.0)
    H0 = oracle.scale_matched_init(s_sum, 4000, 24, 1001)
    r = oracle.fit_adagrad(S, 24, H0, max_iters=100, S_sqnorm=sq)
    assert rel_fro(Hg, r.H) <= 1e-3
    lg = m.labels(to_dev(Hg, DEV)).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(r.H), Hg, r.H)


def test_upper_block_svrg_parity(m):
    # snapshots through the upper-triangle stream, block steps through the slab stream
    _, _, S = tpdm_problem(2000, 1000, seed=0)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st, _ = _fit(m, S, 24, solver="block_svrg", seed=5, max_iters=6, rel_tol=0.0,
                     block_rows=256, grow=True, stall_tol=1e-2)
    H0 = oracle.scale_matched_init(s_sum, 2000, 24, 5)
    r = oracle.fit_block_svrg(S, 24, H0, max_epochs=6, block_rows=256, grow=True,
                              stall_tol=1e-2, seed=5, S_sqnorm=sq)
    assert st["block_final"] == r.block_final and st["epochs"] == r.epochs
    assert rel_fro(Hg, r.H) <= 1e-3


def test_upper_fit_is_bitwise_reproducible(m):
    import torch
    _, _, S = corr_problem(1500, 120, seed=9)
    Sd = to_dev(S, DEV, pad4=True)
    H1, s1 = m.fit(Sd, 8, seed=2, max_iters=30, rel_tol=0.0, upper_only=True)
    H2, s2 = m.fit(Sd, 8, seed=2, max_iters=30, rel_tol=0.0, upper_only=True)
    torch.cuda.synchronize()
    assert torch.equal(H1, H2) and s1["loss"] == s2["loss"]
