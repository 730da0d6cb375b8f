"""GPU parity of the row-sharded fit's per-rank pieces (one process, one GPU).

The ranks' blocks are emulated one after another in this process: each block
is a separate symnmf_shard_step on its rows, and the exchange (the sum of the
partials, the concatenation of the new rows) is done here by hand.  No kernel
waits on another.  The collectives themselves are covered by the CPU gloo
tests; here the kernels are compared with the oracle and with symnmf_fit.
"""
import numpy as np
import pytest

import oracle
from gpu_util import corr_problem, rel_fro, to_dev

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


def test_rows_stats_init_and_gram(m):
    import torch
    from symmetric_nmf_clustering_b200.sharded import DeviceShardOps
    n, k = 1000, 8
    _, _, S = corr_problem(n, 120, seed=2)
    Sd = to_dev(S, DEV, pad4=True)
    ops = DeviceShardOps(DEV)
    parts = [ops.stats(Sd[a:b], n) for a, b in ((0, 384), (384, 1000))]
    tot = (parts[0] + parts[1]).cpu().numpy()
    s_sum, sq, bad = oracle.stats(S)
    assert abs(tot[0] - s_sum) <= 1e-12 * s_sum and abs(tot[1] - sq) <= 1e-12 * sq and tot[2] == 0
    H = ops.init(n, k, 77, s_sum)
    assert np.array_equal(H.cpu().numpy(), oracle.scale_matched_init(s_sum, n, k, 77))
    A = ops.gram(H)[: k * k].cpu().numpy().reshape(k, k)
    h = H.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(A, h.T @ h, rtol=1e-13)


def test_two_blocks_equal_one_full_step(m):
    # rows [0, 256) and [256, 999): one step on each, summed and concatenated,
    # against the oracle's step and the library's single-process step
    import torch
    from symmetric_nmf_clustering_b200.sharded import DeviceShardOps
    n, k = 999, 24
    _, _, S = corr_problem(n, 120, seed=3, name="corr_n20000_k24")
    Sd = to_dev(S, DEV, pad4=True)
    rng = np.random.default_rng(4)
    H0 = (rng.random((n, k)) * 0.2).astype(np.float32)
    G0 = (rng.random((n, k)) * 0.01).astype(np.float32)
    ops = DeviceShardOps(DEV)
    H = torch.from_numpy(H0).to(DEV)
    A = ops.gram(H)[: k * k].contiguous()
    Hn = torch.empty_like(H)
    Gn = torch.empty_like(H)
    tot = None
    for a, b in ((0, 256), (256, n)):
        Ga = torch.from_numpy(G0[a:b].copy()).to(DEV)
        hn = torch.empty((b - a, k), dtype=torch.float32, device=DEV)
        gn = torch.empty_like(hn)
        part = ops.step(Sd[a:b], a, H, A, Ga, 0.1, 1e-10, hn, gn, ops.workspace(b - a, n, k))
        Hn[a:b] = hn
        Gn[a:b] = gn
        tot = part if tot is None else tot + part
    torch.cuda.synchronize()
    r = oracle.fit_adagrad(S, k, H0, max_iters=1, G0=G0)
    assert rel_fro(Hn.cpu().numpy(), r.H) <= 1e-4
    assert rel_fro(Gn.cpu().numpy(), r.G) <= 1e-4
    s_sum, sq, _ = oracle.stats(S)
    h0 = H0.astype(np.float64)
    a2 = float(((h0.T @ h0) ** 2).sum())
    loss0 = sq - 2.0 * float(tot[k * k]) + a2
    assert abs(loss0 - r.history[0]) <= 1e-5 * r.history[0]
    gram1 = tot[: k * k].cpu().numpy().reshape(k, k)
    h1 = Hn.cpu().numpy().astype(np.float64)
    np.testing.assert_allclose(gram1, h1.T @ h1, rtol=1e-12)
    # and the library's own single-process step from the same (H, G)
    Hs, _ = m.fit(Sd, k, H0=to_dev(H0, DEV), G=to_dev(G0.copy(), DEV), max_iters=1, rel_tol=0.0)
    assert rel_fro(Hn.cpu().numpy(), Hs.cpu().numpy()) <= 1e-5


def test_fit_sharded_single_rank_equals_fit(m):
    # the driver on one rank (no process group): the same loop as symnmf_fit
    import torch
    from symmetric_nmf_clustering_b200.sharded import fit_sharded
    n, k = 2000, 8
    _, _, S = corr_problem(n, 250, seed=0)
    Sd = to_dev(S, DEV, pad4=True)
    Hs, st = fit_sharded(Sd, 0, n, k, seed=1000, max_iters=60, rel_tol=0.0)
    Hf, sf = m.fit(Sd, k, seed=1000, max_iters=60, rel_tol=0.0, history=True)
    torch.cuda.synchronize()
    assert st["iters"] == sf["iters"] == 60
    np.testing.assert_allclose(st["history"], sf["history"], rtol=1e-5)
    assert rel_fro(Hs.cpu().numpy(), Hf.cpu().numpy()) <= 1e-4
    # against the oracle as well
    s_sum, sq, _ = oracle.stats(S)
    ref = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 1000), max_iters=60,
                             S_sqnorm=sq)
    assert rel_fro(Hs.cpu().numpy(), ref.H) <= 1e-3
    np.testing.assert_allclose(st["history"], ref.history, rtol=1e-4)
