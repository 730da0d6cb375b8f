"""Parity of the fp16 S-stream of the full-batch loop (stream_h16.cu).

The library runs the AdaGrad solver's full-batch passes through this kernel
from n = 20,000 up (k <= 24); SYMNMF_H16_MIN_N lowers the threshold so that
it runs at sizes the oracle follows (the variable is read on every call).
S and X enter as power-of-two scaled fp16 hi/lo pairs, so the tolerances are
those of the TF32 path: per-step H and G 1e-4, trajectories H 1e-3 and loss
history 1e-4, labels equal except near-ties.
"""
import os

import numpy as np
import pytest

import oracle
import synth
from gpu_util import assert_labels_differ_only_on_near_ties, corr_problem, rel_fro, to_dev

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


@pytest.fixture()
def h16_on():
    old = os.environ.get("SYMNMF_H16_MIN_N")
    os.environ["SYMNMF_H16_MIN_N"] = "1"
    yield
    if old is None:
        os.environ.pop("SYMNMF_H16_MIN_N", None)
    else:
        os.environ["SYMNMF_H16_MIN_N"] = old


def _fit(m, S, k, **kw):
    import torch
    H, st = m.fit(to_dev(S, DEV, pad4=True), k, history=True, **kw)
    torch.cuda.synchronize()
    return H.cpu().numpy(), st


@pytest.mark.parametrize("n,k", [(4000, 24), (3001, 8), (1000, 1), (257, 24)])
def test_h16_trajectory(m, h16_on, n, k):
    _, _, S = corr_problem(n, 200, seed=n + k)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st = _fit(m, S, k, seed=1000, max_iters=100, rel_tol=0.0)
    # three launches per pass (stream, finalise, operand split): the fp16 path ran
    assert st["kernel_launches"] >= 3 * 100
    ref = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 1000), max_iters=100,
                             S_sqnorm=sq)
    np.testing.assert_allclose(st["history"], ref.history, rtol=1e-4)
    assert rel_fro(Hg, ref.H) <= 1e-3
    import torch
    lg = m.labels(torch.from_numpy(Hg).to(DEV)).cpu().numpy()
    assert_labels_differ_only_on_near_ties(lg, oracle.labels(ref.H), Hg, ref.H)


@pytest.mark.parametrize("n,k", [(2000, 24), (1999, 16)])
def test_h16_one_step(m, h16_on, n, k):
    _, _, S = corr_problem(n, 120, seed=7)
    rng = np.random.default_rng(4)
    H0 = (rng.random((n, k)) * 0.2).astype(np.float32)
    G0 = (rng.random((n, k)) * 0.01).astype(np.float32)
    import torch
    G = to_dev(G0.copy(), DEV)
    H, st = m.fit(to_dev(S, DEV, pad4=True), k, H0=to_dev(H0, DEV), G=G, max_iters=1,
                  rel_tol=0.0, history=True)
    torch.cuda.synchronize()
    ref = oracle.fit_adagrad(S, k, H0, max_iters=1, G0=G0)
    assert rel_fro(H.cpu().numpy(), ref.H) <= 1e-4
    assert rel_fro(G.cpu().numpy(), ref.G) <= 1e-4
    np.testing.assert_allclose(st["history"], ref.history, rtol=1e-5)


def test_h16_wide_range_scales(m, h16_on):
    # entries spread over many binades and a large maximum: S = D |corr| D with
    # D_i = 2^(u_i), u_i in [0, 12) (max |S| near 2^24), so the scale of S is
    # far from 2^14 and small entries sit deep below the largest
    n, k = 1500, 12
    _, _, C = corr_problem(n, 150, seed=11)
    rng = np.random.default_rng(12)
    d = np.exp2(rng.random(n) * 12.0)
    S = (C.astype(np.float64) * d[:, None] * d[None, :]).astype(np.float32)
    s_sum, sq, _ = oracle.stats(S)
    Hg, st = _fit(m, S, k, seed=3, max_iters=40, rel_tol=0.0)
    ref = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 3), max_iters=40,
                             S_sqnorm=sq)
    np.testing.assert_allclose(st["history"], ref.history, rtol=1e-4)
    assert rel_fro(Hg, ref.H) <= 1e-3


def test_h16_bitwise_reproducible_over_several_waves(m, h16_on):
    # n = 12,000: the grid runs in several waves of CTAs (where a missing
    # proxy fence once made fits differ from run to run)
    _, _, S = corr_problem(12000, 200, seed=12000)
    Sd = to_dev(S, DEV, pad4=True)
    import torch
    outs = []
    for _ in range(3):
        H, st = m.fit(Sd, 24, seed=1000, max_iters=30, rel_tol=0.0, history=True)
        torch.cuda.synchronize()
        outs.append((H.cpu().numpy(), np.asarray(st["history"])))
    for H, h in outs[1:]:
        assert np.array_equal(H, outs[0][0]) and np.array_equal(h, outs[0][1])


def test_h16_path_selection(m):
    # below the threshold, for k > 24 at any size and for Block-SVRG the TF32
    # path runs (two launches per pass instead of three)
    from symmetric_nmf_clustering_b200 import _lib as L
    _, _, S = corr_problem(2000, 120, seed=5)
    old = os.environ.pop("SYMNMF_H16_MIN_N", None)
    try:
        _, st = _fit(m, S, 8, seed=1, max_iters=20, rel_tol=0.0)
        assert st["stream_kernel"] == L.STREAM_TF32 and st["kernel_launches"] < 3 * 20
        os.environ["SYMNMF_H16_MIN_N"] = "1"
        _, st = _fit(m, S, 8, seed=1, max_iters=20, rel_tol=0.0)
        assert st["stream_kernel"] == L.STREAM_FP16 and st["kernel_launches"] >= 3 * 20
        _, st = _fit(m, S, 32, seed=1, max_iters=20, rel_tol=0.0)
        assert st["stream_kernel"] == L.STREAM_TF32 and st["kernel_launches"] < 3 * 20
        _, st = _fit(m, S, 8, seed=1, solver="block_svrg", block_rows=512, max_iters=3,
                     rel_tol=0.0)
        assert st["stream_kernel"] == L.STREAM_TF32
    finally:
        if old is None:
            os.environ.pop("SYMNMF_H16_MIN_N", None)
        else:
            os.environ["SYMNMF_H16_MIN_N"] = old


def test_h16_split_arithmetic_is_exact_ieee(m):
    # the split warps' arithmetic, through its test entry point, against the same
    # steps in IEEE arithmetic on the host: v = x scale in float32, hi = rn16(v),
    # lo = rn16(v - hi) (the difference exact in float32), bit for bit.  (A split
    # that lost lo, or rounded differently, would still pass the fit tolerances
    # above: the tensor core's accumulation error is as large.)
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    lib = L.load()
    rng = np.random.default_rng(21)
    n = 1 << 16
    x = np.concatenate([rng.random(n // 2, dtype=np.float32),
                        (rng.random(n // 4, dtype=np.float32) * 1e-3).astype(np.float32),
                        np.exp2(rng.uniform(-20, 0, n // 4)).astype(np.float32)])
    for scale in (16384.0, 2.0 ** -6, 1.0):
        xd = torch.from_numpy(x).to(DEV)
        hi = torch.empty(n // 2, dtype=torch.int32, device=DEV)
        lo = torch.empty(n // 2, dtype=torch.int32, device=DEV)
        assert lib.symnmf_test_split16(xd.data_ptr(), n, scale, hi.data_ptr(), lo.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream) == 0
        torch.cuda.synchronize()
        v = (x * np.float32(scale)).astype(np.float32)
        h16 = v.astype(np.float16)
        h = h16.astype(np.float32)
        lo_f = (v - h).astype(np.float32)
        # the difference is exact: hi and v are float32 numbers less than half an
        # fp16 ulp apart (computed in float64 as well)
        assert np.array_equal(lo_f.astype(np.float64), v.astype(np.float64) - h.astype(np.float64))
        want_h = h16.view(np.uint16).astype(np.uint32)
        want_l = lo_f.astype(np.float16).view(np.uint16).astype(np.uint32)
        got = hi.cpu().numpy().view(np.uint32)
        got_l = lo.cpu().numpy().view(np.uint32)
        assert np.array_equal(got & 0xFFFF, want_h[0::2]) and np.array_equal(got >> 16, want_h[1::2])
        assert np.array_equal(got_l & 0xFFFF, want_l[0::2]) and np.array_equal(got_l >> 16, want_l[1::2])
        # where v is in fp16's normal range, hi + lo carries v to 2^-22 relative,
        # plus 2^-25 absolute where lo falls below fp16's normal range
        normal = np.abs(v) >= 2.0 ** -14
        got_sum = (np.asarray(want_h, np.uint16).view(np.float16).astype(np.float64) +
                   np.asarray(want_l, np.uint16).view(np.float16).astype(np.float64))
        err = np.abs(got_sum - v)[normal]
        assert np.all(err <= 2.0 ** -22 * np.abs(v[normal]) + 2.0 ** -25)


def test_per_launch_stream_times(m, h16_on):
    # stream_times: every S-stream launch's CUDA-event time, in order, summing
    # to the total the fit reports
    _, _, S = corr_problem(3000, 150, seed=8)
    _, st = _fit(m, S, 24, seed=1, max_iters=12, rel_tol=0.0, stream_times=True)
    each = st["stream_ms_each"]
    assert len(each) == st["stream_launches"] == 13
    assert all(x > 0 for x in each)
    assert abs(sum(each) - st["stream_ms"]) <= 1e-3 * st["stream_ms"] + 1e-3


def test_h16_tiny_matrix_and_iterate_scales_at_their_cap(m, h16_on):
    # S = 2^-60 |corr| and H0 near 2^-55: both operand scales reach their cap
    # (2^63; uncapped, cS cX would overflow fp32), and the products are scaled
    # back one scale at a time
    import torch
    n, k = 1000, 8
    _, _, C = corr_problem(n, 120, seed=13)
    S = (C.astype(np.float64) * 2.0 ** -60).astype(np.float32)
    rng = np.random.default_rng(14)
    H0 = (rng.random((n, k)) * 2.0 ** -55).astype(np.float32)
    s_sum, sq, _ = oracle.stats(S)
    H, st = m.fit(to_dev(S, DEV, pad4=True), k, H0=to_dev(H0, DEV), max_iters=5, rel_tol=0.0,
                  history=True)
    torch.cuda.synchronize()
    ref = oracle.fit_adagrad(S, k, H0, max_iters=5, S_sqnorm=sq)
    assert st["stream_kernel"] == 1   # STREAM_FP16
    np.testing.assert_allclose(st["history"], ref.history, rtol=1e-4)
    assert rel_fro(H.cpu().numpy(), ref.H) <= 1e-3
