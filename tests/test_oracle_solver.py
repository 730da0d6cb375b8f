"""Pins of the oracle's factorisation steps and solvers (CPU only)."""
import math

import numpy as np
import pytest

import oracle
import synth


def _brute_loss(S, H):
    D = S - H @ H.T
    return float((D * D).sum())


def _small_problem(n, k, seed):
    R, _, _ = synth.workload("corr_n2000_k8", seed=seed, n=n, T=60)
    S = oracle.corr_abs(R)
    rng = np.random.default_rng(seed + 100)
    H = rng.random((n, k)) * 0.4
    return S, H


@pytest.mark.parametrize("n,k", [(1, 1), (7, 3), (64, 8)])
def test_trace_loss_equals_brute_force(n, k):
    S, H = _small_problem(n, k, n)
    sq = float((S * S).sum())
    L = oracle.trace_loss(sq, H, S @ H)
    ref = _brute_loss(S, H)
    assert abs(L - ref) <= 1e-12 * max(ref, sq)


def test_gradient_matches_central_differences():
    S, H = _small_problem(16, 4, 3)
    g = oracle.gradient(H, S @ H)
    h = 1e-6
    fd = np.zeros_like(H)
    for i in range(H.shape[0]):
        for j in range(H.shape[1]):
            Hp = H.copy(); Hp[i, j] += h
            Hm = H.copy(); Hm[i, j] -= h
            fd[i, j] = (_brute_loss(S, Hp) - _brute_loss(S, Hm)) / (2 * h)
    np.testing.assert_allclose(g, fd, rtol=1e-6, atol=1e-6 * np.abs(fd).max())


def test_first_step_closed_form():
    # G_1 = g_0^2, so H_1 = max(H_0 - lr * g_0 / (|g_0| + eps), 0) ~ max(H_0 - lr*sign(g_0), 0)
    S, H0 = _small_problem(12, 3, 4)
    h = 1e-6
    sign = np.zeros_like(H0)
    for i in range(12):
        for j in range(3):
            Hp = H0.copy(); Hp[i, j] += h
            Hm = H0.copy(); Hm[i, j] -= h
            sign[i, j] = np.sign(_brute_loss(S, Hp) - _brute_loss(S, Hm))
    H1, G1 = oracle.adagrad_step(H0, np.zeros_like(H0), oracle.gradient(H0, S @ H0), 0.1, 1e-10)
    np.testing.assert_allclose(H1, np.maximum(H0 - 0.1 * sign, 0.0), atol=1e-8)
    assert np.all(G1 >= 0)


def test_iterates_nonnegative_and_accumulator_monotone():
    S, H0 = _small_problem(50, 5, 5)
    seen = []

    def hook(t, H, P):
        seen.append(H.copy())

    r = oracle.fit_adagrad(S, 5, H0, max_iters=30, hook=hook)
    assert all(np.all(H >= 0) for H in seen)
    # G only grows: rerun step by step
    H, G = H0.copy(), np.zeros_like(H0)
    for _ in range(10):
        Hn, Gn = oracle.adagrad_step(H, G, oracle.gradient(H, S @ H), 0.1, 1e-10)
        assert np.all(Gn >= G)
        H, G = Hn, Gn
    assert r.iters == 30 and len(r.history) == 31


def test_rank_one_recovery():
    # S = v v^T with v > 0 and k = 1: the minimiser is H = v
    rng = np.random.default_rng(6)
    v = rng.uniform(0.2, 1.0, 40)
    S = np.outer(v, v)
    H0 = np.full((40, 1), 0.3)
    r = oracle.fit_adagrad(S, 1, H0, lr=0.05, max_iters=3000, mirror=False)
    np.testing.assert_allclose(r.H[:, 0], v, rtol=1e-3)


# SymNMF is non-convex: from some starts AdaGrad settles in a local minimum that
# merges two blocks (loss = one block's mass).  The listed starts are ones from
# which exact arithmetic reaches the planted optimum; a wrong sign, index or
# scale anywhere in the loop fails all of them.
@pytest.mark.parametrize("sizes,seed", [([60] * 5, s) for s in range(10)]
                         + [([50] * 8, s) for s in (0, 1, 3, 4, 7)])
def test_planted_blocks_recovered_with_ari_one(sizes, seed):
    S, planted = synth.planted_block_matrix(sizes, order_seed=seed)
    n, k = S.shape[0], len(sizes)
    s_sum, sq, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, n, k, 1000 + seed)
    r = oracle.fit_adagrad(S, k, H0, lr=0.1, eps=1e-10, max_iters=600, S_sqnorm=sq)
    assert oracle.ari(oracle.labels(r.H), planted) == 1.0
    assert r.loss < 1e-3 * sq


def test_joint_permutation_equivariance():
    S, H0 = _small_problem(60, 4, 7)
    perm = np.random.default_rng(8).permutation(60)
    a = oracle.fit_adagrad(S, 4, H0, max_iters=25, mirror=False)
    b = oracle.fit_adagrad(S[np.ix_(perm, perm)], 4, H0[perm], max_iters=25, mirror=False)
    np.testing.assert_allclose(b.H, a.H[perm], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(b.history, a.history, rtol=1e-11)


def test_convergence_returns_evaluated_iterate():
    S, H0 = _small_problem(40, 4, 9)
    r = oracle.fit_adagrad(S, 4, H0, max_iters=5000, rel_tol=1e-4)
    assert r.converged
    assert r.rel < 1e-4
    assert r.loss == r.history[-1] == r.history[r.iters]
    assert abs(r.loss - _brute_loss(S, r.H)) <= 1e-10 * float((S * S).sum())


# -------------------------------------------------------------------- Block-SVRG

def test_svrg_single_block_is_full_gradient():
    S, H = _small_problem(30, 3, 10)
    rng = np.random.default_rng(11)
    H_snap = H + rng.normal(0, 0.05, H.shape)
    g = oracle.block_svrg_grad(S, H, H_snap, S @ H_snap, slice(0, 30), 1)
    np.testing.assert_allclose(g, oracle.gradient(H, S @ H), rtol=1e-12, atol=1e-12)


def test_svrg_block_estimates_are_unbiased():
    S, H = _small_problem(33, 3, 12)
    D = np.random.default_rng(13).normal(size=H.shape)
    b, n = 8, 33
    m = -(-n // b)
    acc = np.zeros_like(H)
    for blk in range(m):
        rows = slice(blk * b, min((blk + 1) * b, n))
        acc += m * (S[:, rows] @ D[rows])
    np.testing.assert_allclose(acc / m, S @ D, rtol=1e-12, atol=1e-12)


def test_svrg_first_inner_step_has_no_correction():
    S, H = _small_problem(30, 3, 14)
    g = oracle.block_svrg_grad(S, H, H.copy(), S @ H, slice(8, 16), 4)
    np.testing.assert_allclose(g, oracle.gradient(H, S @ H), rtol=1e-12, atol=1e-12)


def test_svrg_fit_decreases_loss_and_stays_nonnegative():
    S, H0 = _small_problem(120, 6, 15)
    r = oracle.fit_block_svrg(S, 6, H0, max_epochs=15, block_rows=16, grow=True, seed=3)
    assert np.all(r.H >= 0)
    assert r.history[-1] < r.history[0]
    assert r.block_final >= 16


def test_svrg_growth_reaches_full_batch():
    S, H0 = _small_problem(64, 4, 16)
    r = oracle.fit_block_svrg(S, 4, H0, max_epochs=40, block_rows=8, grow=True,
                              stall_tol=10.0, seed=1)
    # stall_tol > 1 forces growth every epoch: 8 -> 16 -> 32 -> 64, then full batch
    assert r.block_final == 64
    assert r.epochs == 3 and r.iters == 40 - 3


def test_epoch_permutation_is_a_permutation():
    for m in [1, 2, 5, 13]:
        for e in range(4):
            p = oracle.epoch_permutation(m, 1234, e)
            assert sorted(p) == list(range(m))
    counts = {}
    for e in range(6000):
        key = tuple(oracle.epoch_permutation(3, 99, e))
        counts[key] = counts.get(key, 0) + 1
    assert len(counts) == 6
    assert min(counts.values()) > 850 and max(counts.values()) < 1150


def test_default_block_rows():
    assert oracle.default_block_rows(20000) == 2048
    assert oracle.default_block_rows(100000) == 8192
    assert oracle.default_block_rows(5) == 1
    assert oracle.default_block_rows(2000) == 256      # 200 -> nearest power of two 256
    assert oracle.default_block_rows(1400) == 128      # 140 -> 128


# -------------------------------------------------------------------- AdaptGrow

def test_adaptgrow_selects_solver_from_gap():
    sizes = [30] * 4
    S, _ = synth.planted_block_matrix(sizes, order_seed=0)
    ev = oracle.top_eigenvalues(S, 6)
    # block matrix: lambda_{k+1} = 30 and lambda_{k+2} = 0 (to rounding) for k = 3
    r = oracle.adaptgrow(S.astype(np.float64), 3, max_iters=5, eigvals=ev)
    assert r.gamma > 1e10 and r.solver_used == 0
    flat = np.array([10.0, 9.0, 8.0, 7.0, 6.0, 5.5])
    r2 = oracle.adaptgrow(S.astype(np.float64), 3, max_iters=2, eigvals=flat, block_rows=16)
    assert r2.gamma == pytest.approx(7.0 / 6.0) and r2.solver_used == 1


# ------------------------------------------------- Block-SVRG epoch loop, pinned
# [CaS] "Factorizing with SymNMF": block-sampled gradient corrected with the
# SVRG control variate, same AdaGrad update; [SMI] AdaptGrow sketch.  The
# pins below fix the loop around block_svrg_grad: which snapshot the blocks
# see, which rows a block holds, the visiting order, and the stall rule.

def _blocks_by_hand(n, b):
    """Row index sets of the contiguous blocks [jb, min((j+1)b, n)), built
    from index arrays rather than slices."""
    m = -(-n // b)
    return [np.arange(j * b, min((j + 1) * b, n)) for j in range(m)]


def _epoch_by_hand(S, H, G, b, order, lr=0.1, eps=1e-10):
    """One Block-SVRG epoch applied step by step: snapshot H~ and P~ = S H~
    frozen at the epoch start, then one AdaGrad step per block in `order`,
    each with the corrected block gradient.  The block product is formed as
    a full product against the difference masked to the block's rows."""
    n = S.shape[0]
    blocks = _blocks_by_hand(n, b)
    m = len(blocks)
    H_snap = H.copy()
    P_snap = np.einsum("ij,jc->ic", S, H_snap)
    for j in order:
        mask = np.zeros((n, 1))
        mask[blocks[j]] = 1.0
        est = P_snap + m * (S @ ((H - H_snap) * mask))
        g = 4.0 * (H @ (H.T @ H) - est)
        H, G = oracle.adagrad_step(H, G, g, lr, eps)
    return H, G


def test_svrg_two_block_epoch_equals_hand_applied_steps():
    # n = 37, b = 20: a full block and a ragged one (m = 2)
    S, H0 = _small_problem(37, 3, 21)
    for seed in (0, 1, 2, 5):
        order = oracle.epoch_permutation(2, seed, 0)
        r = oracle.fit_block_svrg(S, 3, H0, max_epochs=1, block_rows=20, grow=False,
                                  seed=seed, mirror=False)
        H1, G1 = _epoch_by_hand(S, H0.copy(), np.zeros_like(H0), 20, order)
        np.testing.assert_allclose(r.H, H1, rtol=1e-12, atol=1e-15)
        np.testing.assert_allclose(r.G, G1, rtol=1e-12, atol=1e-15)
        assert r.epochs == 1 and r.iters == 0
        # the two evaluations are the snapshot losses of H0 and of the epoch's result
        assert len(r.history) == 2
        assert abs(r.history[0] - _brute_loss(S, H0)) <= 1e-12 * _brute_loss(S, H0)
        assert abs(r.history[1] - _brute_loss(S, H1)) <= 1e-12 * _brute_loss(S, H0)


def test_svrg_visits_blocks_in_the_epoch_permutation_each_once():
    # n = 50, b = 17: blocks of 17, 17, 16; three epochs, every order distinct
    S, H0 = _small_problem(50, 4, 22)
    seed = 7
    orders = [oracle.epoch_permutation(3, seed, e) for e in range(3)]
    r = oracle.fit_block_svrg(S, 4, H0, max_epochs=3, block_rows=17, grow=False, seed=seed,
                              mirror=False)
    H, G = H0.copy(), np.zeros_like(H0)
    for o in orders:
        assert sorted(o) == [0, 1, 2]
        H, G = _epoch_by_hand(S, H, G, 17, o)
    np.testing.assert_allclose(r.H, H, rtol=1e-11, atol=1e-14)
    # the order matters: the same epochs with every order reversed end elsewhere
    Hx, Gx = H0.copy(), np.zeros_like(H0)
    for o in orders:
        Hx, Gx = _epoch_by_hand(S, Hx, Gx, 17, o[::-1])
    assert np.abs(Hx - r.H).max() > 1e-6


def test_svrg_stall_rule_doubles_on_consecutive_snapshots():
    # the block doubles after the epoch whose snapshot loss fell by less than
    # stall_tol relative to the previous snapshot (not the first one)
    S, H0 = _small_problem(96, 4, 23)
    seed, b0, stall = 3, 12, 0.02
    E = 8
    r = oracle.fit_block_svrg(S, 4, H0, max_epochs=E, block_rows=b0, grow=True,
                              stall_tol=stall, seed=seed, mirror=False)
    # replay: block schedule from the replay's own snapshot losses
    H, G, b = H0.copy(), np.zeros_like(H0), b0
    losses, schedule = [], []
    for e in range(E + 1):
        L = _brute_loss(S, H)
        if losses and (losses[-1] - L) / losses[-1] < stall:
            b = min(2 * b, 96)
        losses.append(L)
        if e == E:
            break
        schedule.append(b)
        if b >= 96:
            g = oracle.gradient(H, S @ H)
            H, G = oracle.adagrad_step(H, G, g, 0.1, 1e-10)
        else:
            H, G = _epoch_by_hand(S, H, G, b, oracle.epoch_permutation(-(-96 // b), seed, e))
    np.testing.assert_allclose(r.history, losses, rtol=1e-10)
    np.testing.assert_allclose(r.H, H, rtol=1e-10, atol=1e-13)
    assert r.block_final == b
    # the schedule grew at some epochs and not at others, so the rule was exercised
    assert b0 < b and len(set(schedule)) >= 3


@pytest.mark.parametrize("sizes,b,seed", [([60] * 5, 64, s) for s in range(6)]
                         + [([40] * 6, 48, s) for s in (0, 3, 7)]
                         + [([50] * 8, 64, s) for s in (1, 2, 4)])
def test_svrg_recovers_planted_blocks_with_growth_off(sizes, b, seed):
    # noise-free planted blocks, b < n and growth off: the sampled solver alone
    # reaches the planted factorisation (ARI = 1, loss ~ 0) from these starts
    S, planted = synth.planted_block_matrix(sizes, order_seed=seed)
    n, k = S.shape[0], len(sizes)
    s_sum, sq, _ = oracle.stats(S)
    H0 = oracle.scale_matched_init(s_sum, n, k, 1000 + seed)
    r = oracle.fit_block_svrg(S, k, H0, max_epochs=300, block_rows=b, grow=False, seed=seed,
                              S_sqnorm=sq)
    assert r.block_final == b and r.epochs == 300
    assert oracle.ari(oracle.labels(r.H), planted) == 1.0
    assert r.loss < 1e-9 * sq
