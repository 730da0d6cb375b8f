"""The row-chunked view of a matrix that the full-size GPU parity tests hand
to the oracle (``gpu_util.DeviceRowChunks``) gives the oracle's solvers the
same results as the matrix itself (CPU, on a torch CPU tensor)."""
import numpy as np
import torch

import oracle
import synth
from gpu_util import DeviceRowChunks


def _problem():
    R, _, _ = synth.workload("corr_n2000_k8", seed=3, n=203, T=80)
    S = oracle.corr_abs(R).astype(np.float32)
    # full storage with a row pitch wider than n, as on the device
    buf = torch.full((203, 208), float("nan"), dtype=torch.float32)
    buf[:, :203] = torch.from_numpy(S)
    return S, buf[:, :203]


def test_chunked_stats_and_adagrad_equal_the_matrix():
    S, St = _problem()
    X = DeviceRowChunks(St, rows_per_chunk=17)
    s_sum, sq, bad = oracle.stats(S)
    a, b, c = X.stats()
    assert c == bad == 0
    assert abs(a - s_sum) <= 1e-12 * s_sum and abs(b - sq) <= 1e-12 * sq
    H0 = oracle.scale_matched_init(s_sum, 203, 5, 9)
    r1 = oracle.fit_adagrad(S, 5, H0, max_iters=6, S_sqnorm=sq)
    r2 = oracle.fit_adagrad(X, 5, H0, max_iters=6, S_sqnorm=sq)
    np.testing.assert_allclose(r2.H, r1.H, rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(r2.history, r1.history, rtol=1e-12)


def test_chunked_block_svrg_equals_the_matrix():
    S, St = _problem()
    X = DeviceRowChunks(St, rows_per_chunk=50)
    s_sum, sq, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, 203, 5, 11)
    kw = dict(max_epochs=3, block_rows=40, grow=True, stall_tol=0.5, seed=11, S_sqnorm=sq)
    r1 = oracle.fit_block_svrg(S, 5, H0, **kw)
    r2 = oracle.fit_block_svrg(X, 5, H0, **kw)
    np.testing.assert_allclose(r2.H, r1.H, rtol=1e-11, atol=1e-14)
    np.testing.assert_allclose(r2.history, r1.history, rtol=1e-12)
    assert r2.block_final == r1.block_final
