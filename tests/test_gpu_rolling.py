"""GPU parity of symnmf_ari and symnmf_rolling against the CPU oracle.

ARI: the contingency table is integer work (bit-exact) and the index is the
same float64 expression on both sides, so the values must be bit-equal.

Rolling study: both sides get the same returns stream; the GPU builds its own
S, so the builders' rounding (per entry e_S = 5e-6 for |corr|, 1e-5 max|S|
for TPDM) enters the fit.  Per window: labels equal wherever the oracle's
top-two margin of H exceeds 1e-3 max|H| (the fit's H tolerance); loss within
1e-4 (the fit's loss tolerance) plus 2 sqrt(f) n e_S, the most an entrywise
perturbation of e_S moves f = ||S - H H^T||^2 to first order; cross-sector
mean within e_S plus 1e-6 relative; an ARI bit-equal whenever both of its
windows' label vectors are equal; the 3-sigma limit and flags equal when
every calibration ARI is.  Those cross-side checks run only where labels
agree, so each test also asserts how many of them ran, and checks in every
window that the library's ARI series, limit and flags are the oracle's
functions of the library's own labels.
"""
import numpy as np
import pytest

import oracle
import synth
from gpu_util import to_dev

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


@pytest.mark.parametrize("n,k,seed", [(1, 1, 0), (5, 3, 1), (1000, 7, 2), (100003, 24, 3),
                                      (4096, 64, 4)])
def test_ari_bit_exact(m, n, k, seed):
    rng = np.random.default_rng(seed)
    a = rng.integers(0, k, n).astype(np.int32)
    # b: a relabelled copy of a with a fraction of the rows redrawn
    b = np.random.default_rng(seed + 100).permutation(k).astype(np.int32)[a]
    flip = rng.random(n) < 0.2
    b[flip] = rng.integers(0, k, int(flip.sum()))
    v, table = m.ari(to_dev(a, DEV), to_dev(b, DEV), k)
    ref_table = oracle.contingency(a, b, k, k)
    assert np.array_equal(table, ref_table)
    assert v == oracle.ari_from_table(ref_table)


def test_ari_identical_and_trivial(m):
    a = np.arange(50, dtype=np.int32) % 5
    assert m.ari(to_dev(a, DEV), to_dev(a, DEV), 5)[0] == 1.0
    z = np.zeros(50, dtype=np.int32)
    assert m.ari(to_dev(z, DEV), to_dev(z, DEV), 5)[0] == 1.0
    assert m.ari(to_dev(z, DEV), to_dev(a, DEV), 5)[0] == oracle.ari_from_table(
        oracle.contingency(z, a, 5, 5))


def test_ari_rejects_out_of_range_labels(m):
    from symmetric_nmf_clustering_b200 import _lib as L
    a = np.array([0, 1, 2, 5], dtype=np.int32)
    with pytest.raises(L.SymNMFError) as e:
        m.ari(to_dev(a, DEV), to_dev(a, DEV), 4)
    assert "outside" in str(e.value)


def _compare_windows(got, ref, k, windows, H, kind):
    """Labels on the oracle's clear rows, loss, cross; returns windows whose
    label vectors are fully equal."""
    equal = set()
    lab = got["labels"].cpu().numpy()
    n = lab.shape[1]
    for w in windows:
        e_S = 5e-6 if kind == "corr" else 1e-5 * ref["smax"][w]
        Hw = H[w]
        srt = np.sort(Hw, axis=1)
        clear = (srt[:, -1] - srt[:, -2]) > 1e-3 * np.abs(Hw).max()
        assert np.array_equal(lab[w][clear], ref["labels"][w][clear]), w
        assert (~clear).sum() <= max(3, 0.05 * len(clear)), w
        if np.array_equal(lab[w], ref["labels"][w]):
            equal.add(w)
        f = ref["loss"][w]
        assert abs(got["loss"][w] - f) <= 1e-4 * f + 2.0 * np.sqrt(f) * n * e_S, w
        if np.isfinite(ref["cross"][w]):
            c = ref["cross"][w]
            assert abs(got["cross"][w] - c) <= e_S + 1e-6 * abs(c), w
    return equal


def _check_series_from_own_labels(g, k, delta, calib, kind):
    """The library's ARI(t-1, t), ARI(t-delta, t), 3-sigma limit and flags are
    the oracle's ARI and control limit applied to the library's own labels,
    in every window (no window is skipped, whatever the labels are)."""
    lab = g["labels"].cpu().numpy()
    W = lab.shape[0]
    for w in range(1, W):
        want = oracle.ari_from_table(oracle.contingency(lab[w - 1], lab[w], k, k))
        assert g["ari_prev"][w] == want, (kind, w)
        if w >= delta:
            want = oracle.ari_from_table(oracle.contingency(lab[w - delta], lab[w], k, k))
            assert g["ari_delta"][w] == want, (kind, w)
    cw = range(max(calib[0], delta), min(calib[1], W))
    mu, sd, lim = oracle.control_limit(np.asarray(g["ari_delta"], dtype=np.float64), cw)
    assert g["mean"] == pytest.approx(mu, rel=1e-12, abs=1e-15), kind
    assert g["std"] == pytest.approx(sd, rel=1e-12, abs=1e-15), kind
    assert g["limit"] == pytest.approx(lim, rel=1e-12, abs=1e-15), kind
    flags = np.array([np.isfinite(x) and x < g["limit"] for x in g["ari_delta"]], dtype=bool)
    assert np.array_equal(np.asarray(g["flags"], dtype=bool), flags), kind


def _stream_small():
    return synth.rolling_stream(seed=5, n=360, g=6, days=90, sigma=1.0, boundary=0.1,
                                switch_day=45, switch_frac=0.1, shock_days=(5, 9),
                                shock_groups=2, shock_scale=1.0)


def test_rolling_parity_small(m):
    st = _stream_small()
    T, k, delta, iters = 60, 6, 10, 60
    kw = dict(tail_frac=0.05, tail_sign=-1, delta=delta, calib=(10, 20), groups=st.groups_before,
              stressed=list(st.stressed), iters=iters, seed=3)
    ref = oracle.rolling_pipeline(st.R, T, k, keep_H=True, **kw)
    R = to_dev(st.R, DEV, pad4=True)
    groups = to_dev(st.groups_before.astype(np.int32), DEV)
    got = m.rolling(R, groups=groups, window=T, k=k, delta=delta, calib_begin=10, calib_end=20,
                    tail_frac=0.05, tail_sign=-1, stressed=list(st.stressed),
                    fit=dict(max_iters=iters, seed=3))
    W = 90 - T + 1
    assert got["n_windows"] == W
    for kind in ("corr", "tpdm"):
        g, r = got[kind], ref[kind]
        equal = _compare_windows(g, r, k, range(W), r["H"], kind)
        _check_series_from_own_labels(g, k, delta, (10, 20), kind)
        n_prev = n_delta = 0
        for w in range(1, W):
            if w in equal and w - 1 in equal:
                assert g["ari_prev"][w] == r["ari_prev"][w], (kind, w)
                n_prev += 1
            if w >= delta and w in equal and w - delta in equal:
                assert g["ari_delta"][w] == r["ari_delta"][w], (kind, w)
                n_delta += 1
        assert np.isnan(g["ari_prev"][0]) and np.all(np.isnan(g["ari_delta"][:delta]))
        calib_equal = all(w in equal and w - delta in equal for w in range(10, 20))
        if calib_equal:
            assert g["mean"] == r["mean"] and g["std"] == r["std"] and g["limit"] == r["limit"]
            assert np.array_equal(g["flags"], r["flags"])
        print(f"{kind}: {len(equal)} of {W} windows with equal labels; {n_prev} ARI(t-1,t) and "
              f"{n_delta} ARI(t-delta,t) compared with the oracle; calibration equal: {calib_equal}")
        # the cross-side comparisons above must have run on (nearly) every window:
        # on B200 all 31 windows of both kinds agree, calibration included
        assert len(equal) >= W - 2, (kind, len(equal))
        assert n_prev >= W - 5 and n_delta >= W - delta - 4, (kind, n_prev, n_delta)
        assert calib_equal, kind
        assert g["build_ms"] > 0 and g["fit_ms"] > 0
    assert got["launches"] > 0


def test_rolling_kinds_and_stride(m):
    st = _stream_small()
    R = to_dev(st.R, DEV, pad4=True)
    got = m.rolling(R, window=40, stride=7, k=6, kinds=1, delta=2, fit=dict(max_iters=20))
    assert "tpdm" not in got and got["n_windows"] == (90 - 40) // 7 + 1
    ref = oracle.rolling_pipeline(st.R, 40, 6, stride=7, kinds=("corr",), delta=2, iters=20,
                                  keep_H=True)
    _compare_windows(got["corr"], ref["corr"], 6, range(got["n_windows"]), ref["corr"]["H"], "corr")
    assert np.all(np.isnan(got["corr"]["cross"]))


def test_rolling_rejects_bad_arguments(m):
    from symmetric_nmf_clustering_b200 import _lib as L
    st = _stream_small()
    R = to_dev(st.R, DEV, pad4=True)
    for kw in [dict(window=100), dict(window=40, n_windows=60), dict(window=40, kinds=0),
               dict(window=40, stressed=[1]), dict(window=40, delta=0)]:
        with pytest.raises(L.SymNMFError):
            m.rolling(R, k=6, **kw)


def test_rolling_full_size_sampled_windows(m):
    # the rolling workload at its full size: n = 5,000, k = 24, 250 windows of
    # 250 days over 499 days, delta = 50; the oracle computes windows 0, 1,
    # 124, 125 and 174 (both kinds) and the GPU run is compared there
    st = synth.rolling_stream(seed=0)
    R = to_dev(st.R, DEV, pad4=True)
    groups = to_dev(st.groups_before.astype(np.int32), DEV)
    got = m.rolling(R, groups=groups, window=250, k=24, delta=50, calib_begin=50, calib_end=125,
                    tail_frac=0.05, tail_sign=-1, stressed=list(st.stressed))
    assert got["n_windows"] == 250
    sample = [0, 1, 124, 125, 174]
    ref = oracle.rolling_pipeline(st.R, 250, 24, tail_frac=0.05, tail_sign=-1, delta=50,
                                  groups=st.groups_before, stressed=list(st.stressed),
                                  only=sample, keep_H=True)
    for kind in ("corr", "tpdm"):
        equal = _compare_windows(got[kind], ref[kind], 24, sample, ref[kind]["H"], kind)
        _check_series_from_own_labels(got[kind], 24, 50, (50, 125), kind)
        compared = 0
        for w in (1, 125):
            if w in equal and w - 1 in equal:
                assert got[kind]["ari_prev"][w] == ref[kind]["ari_prev"][w]
                compared += 1
        if 174 in equal and 124 in equal:
            assert got[kind]["ari_delta"][174] == ref[kind]["ari_delta"][174]
            compared += 1
        print(f"{kind}: sampled windows with equal labels {sorted(equal)}; "
              f"{compared} of 3 ARIs compared with the oracle")
        assert len(equal) >= 4 and compared >= 2, (kind, sorted(equal), compared)
        a = got[kind]["ari_delta"]
        assert np.all(np.isnan(a[:50])) and np.all((a[50:] >= -1.0) & (a[50:] <= 1.0))


def _same(x, y):
    return np.array_equal(np.asarray(x), np.asarray(y), equal_nan=True)


def test_rolling_concurrent_chains_match_serial(m, monkeypatch):
    # the full workspace runs four chains (two per kind, alternate windows) on
    # their own streams and host threads; every output must equal the single-
    # chain run bit for bit, and so must a run whose workspace is one matrix
    # short of the full size (one chain per kind)
    import ctypes as C
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    st = _stream_small()
    R = to_dev(st.R, DEV, pad4=True)
    groups = to_dev(st.groups_before.astype(np.int32), DEV)
    kw = dict(groups=groups, window=60, k=6, delta=10, calib_begin=10, calib_end=20,
              tail_frac=0.05, tail_sign=-1, stressed=list(st.stressed),
              fit=dict(max_iters=60, seed=3))
    conc = m.rolling(R, **kw)
    monkeypatch.setenv("SYMNMF_ROLLING_SERIAL", "1")
    serial = m.rolling(R, **kw)
    monkeypatch.delenv("SYMNMF_ROLLING_SERIAL")
    n = st.R.shape[1]
    p = m.rolling_params(window=60, k=6, fit=dict(max_iters=60, seed=3))
    size = C.c_size_t(0)
    L.check("symnmf_workspace_size", L.load().symnmf_workspace_size(
        L.OP_ROLLING, n, p.k, p.window, C.byref(p.fit), C.byref(size)))
    short = size.value - n * ((n + 3) // 4 * 4) * 4
    small = m.rolling(R, ws=torch.empty(short, dtype=torch.uint8, device=DEV), **kw)
    for other in (serial, small):
        for kind in ("corr", "tpdm"):
            a, b = conc[kind], other[kind]
            assert torch.equal(a["labels"], b["labels"]), kind
            for key in ("loss", "cross", "ari_prev", "ari_delta", "flags"):
                assert _same(a[key], b[key]), (kind, key)
            for key in ("mean", "std", "limit"):
                assert _same(a[key], b[key]), (kind, key)


def test_rolling_error_in_the_second_chain_is_reported(m):
    # tail_frac is checked by the TPDM builder only: the TPDM chain (second
    # stream and host thread) fails at its first window while the |corr| chain
    # runs on, and the call reports the TPDM builder's error
    from symmetric_nmf_clustering_b200 import _lib as L
    st = _stream_small()
    R = to_dev(st.R, DEV, pad4=True)
    with pytest.raises(L.SymNMFError) as e:
        m.rolling(R, window=60, k=6, kinds=3, delta=5, tail_frac=0.0, fit=dict(max_iters=5))
    assert "tail_frac" in str(e.value)
    # the library is still usable afterwards
    ok = m.rolling(R, window=60, k=6, kinds=3, delta=5, n_windows=3, fit=dict(max_iters=5))
    assert ok["n_windows"] == 3


def test_rolling_warm_start_equals_chained_fits(m):
    # warm_start = 1: window 0 from the seeded start, window w from window
    # w-1's factor of the same kind, G reset -- the same as chaining the
    # public fit by hand on the same builders, bit for bit
    import torch
    st = _stream_small()
    R = to_dev(st.R, DEV, pad4=True)
    T, k, W, iters, seed = 60, 6, 5, 40, 3
    got = m.rolling(R, window=T, k=k, n_windows=W, delta=2, tail_frac=0.05, tail_sign=-1,
                    warm_start=1, fit=dict(max_iters=iters, seed=seed))
    for kind in ("corr", "tpdm"):
        H = None
        for w in range(W):
            Rw = R[w: w + T]
            S = m.build_corr(Rw) if kind == "corr" else m.build_tpdm(Rw, 0.05, -1)
            if H is None:
                H, stt = m.fit(S, k, seed=seed, max_iters=iters, rel_tol=0.0)
            else:
                H, stt = m.fit(S, k, H0=H, max_iters=iters, rel_tol=0.0)
            assert torch.equal(m.labels(H), got[kind]["labels"][w]), (kind, w)
            assert stt["loss"] == got[kind]["loss"][w], (kind, w)
    # Parity with the oracle's warm-started pipeline is not compared window by
    # window: each window starts from its own side's previous result, which
    # differs at the fit's 1e-3 level, and the difference compounds over the
    # windows of an unconverged fit.  The oracle's warm start is pinned against
    # its own chained fits, and each fit's parity is tested on its own.
    from symmetric_nmf_clustering_b200 import _lib as L
    with pytest.raises(L.SymNMFError):
        m.rolling(R, window=T, k=k, n_windows=2, warm_start=2)
