"""Pins of the oracle's generator, spectral pieces, labels and ARI (CPU only)."""
import os

import numpy as np
import pytest

import oracle
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_splitmix64_reference_outputs():
    with open(os.path.join(GOLDEN, "splitmix64_seed0.txt")) as f:
        want = [int(l, 16) for l in f if l.strip() and not l.startswith("#")]
    assert oracle.splitmix64_stream(0, len(want)) == want
    # counter form: element c is the (c+1)-th stream output
    u = oracle.counter_uniform(0, 3)
    assert np.array_equal(u, np.array([(w >> 40) * 2.0 ** -24 for w in want]))


def test_counter_uniform_range_and_uniformity():
    u = oracle.counter_uniform(42, 200000)
    assert u.min() >= 0.0 and u.max() < 1.0
    assert np.array_equal(u, u.astype(np.float32).astype(np.float64))
    hist, _ = np.histogram(u, bins=20, range=(0, 1))
    assert np.all(np.abs(hist - 10000) < 5 * 100)
    assert abs(u.mean() - 0.5) < 0.005


def test_scale_matched_init():
    S, _ = synth.planted_block_matrix([40] * 5)
    s_sum, _, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, 200, 5, 7)
    c = oracle.init_scale(s_sum, 200, 5)
    assert c == pytest.approx(np.sqrt(0.2 / 5), rel=1e-7)
    assert H0.dtype == np.float32 and H0.shape == (200, 5)
    assert H0.min() >= 0 and H0.max() < c
    assert abs(H0.mean() - c / 2) < 0.02 * c
    # element (i, j) uses counter i*k + j
    u = oracle.counter_uniform(7, 1000)
    assert H0[3, 2] == np.float32(u[3 * 5 + 2] * c)


def test_top_eigenvalues_block_of_ones():
    S, _ = synth.planted_block_matrix([5, 3, 2], order_seed=1)
    ev = oracle.top_eigenvalues(S, 5)
    np.testing.assert_allclose(ev, [5, 3, 2, 0, 0], atol=1e-12)


def test_eigenvalue_sum_is_trace():
    R, _, _ = synth.workload("corr_n2000_k8", seed=3, n=60, T=40)
    S = oracle.corr_abs(R)
    ev = oracle.top_eigenvalues(S, 60)
    assert abs(ev.sum() - 60.0) < 1e-9
    assert np.all(np.diff(ev) <= 0)


def test_gap_ratio_values():
    ev = [9.0, 8.0, 4.0, -2.0, 1.0]
    assert oracle.gap_ratio(ev, 2) == 2.0          # lambda_3 / |lambda_4|
    assert oracle.gap_ratio([3.0, 2.0, 0.0], 1) == float("inf")


def test_labels_ties_take_lowest_index():
    H = np.array([[0.1, 0.5, 0.5],
                  [0.0, 0.0, 0.0],
                  [2.0, 1.0, 3.0],
                  [1.0, 1.0, 0.0]], dtype=np.float32)
    assert oracle.labels(H).tolist() == [1, 0, 2, 0]


def _ari_pairs(a, b):
    n = len(a)
    ss = sd = ds = dd = 0
    for i in range(n):
        for j in range(i + 1, n):
            same_a, same_b = a[i] == a[j], b[i] == b[j]
            ss += same_a and same_b
            sd += same_a and not same_b
            ds += (not same_a) and same_b
            dd += (not same_a) and (not same_b)
    # Hubert-Arabie ARI from the four pair counts
    num = 2.0 * (ss * dd - sd * ds)
    den = (ss + sd) * (sd + dd) + (ss + ds) * (ds + dd)
    return 1.0 if den == 0 else num / den


def test_ari_against_sklearn_and_pair_counts():
    from sklearn.metrics import adjusted_rand_score
    rng = np.random.default_rng(5)
    for trial in range(5):
        a = rng.integers(0, 4, 150)
        b = np.where(rng.random(150) < 0.7, a, rng.integers(0, 5, 150))
        v = oracle.ari(a, b)
        assert v == pytest.approx(adjusted_rand_score(a, b), abs=1e-12)
        assert v == pytest.approx(_ari_pairs(a.tolist(), b.tolist()), abs=1e-12)


def test_ari_identity_and_label_permutation():
    a = np.random.default_rng(6).integers(0, 6, 300)
    assert oracle.ari(a, a) == 1.0
    relabel = np.array([3, 5, 0, 1, 4, 2])
    assert oracle.ari(a, relabel[a]) == 1.0
    assert oracle.ari(np.zeros(10), np.zeros(10)) == 1.0
