"""Seeded synthetic inputs for the SymNMF clustering hot path.

This module is the one piece shared by the CPU oracle (``oracle/``) and the
CUDA path (``symmetric_nmf_clustering_b200``): it only draws inputs and holds
none of the method's arithmetic (no correlation, no ranks, no factorisation).

The pages describe their data only in outline: a synthetic stream of daily
returns with planted groups, boundary instruments that load on two groups, a
membership-switch event and a joint tail shock ("GPU-Accelerated Clustering
for Financial Instruments at Scale", sections "The temporal setup" and
"Choosing the rank k": planted rank 24).  The recipe below fills in that
outline; every workload is

    r_t = B f_t + sigma * eps_t          (t = 1..T, r_t in R^n)

with B an n x g nonnegative loading matrix (one own group per instrument,
boundary instruments split over two groups), f_t in R^g the group factors and
eps_t idiosyncratic noise, both iid N(0,1) or Student-t(3).

All draws use numpy's PCG64 through ``numpy.random.default_rng(seed)``.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "planted_groups",
    "planted_loadings",
    "factor_returns",
    "workload",
    "uniform_h0",
    "planted_block_matrix",
    "rolling_stream",
    "RollingStream",
    "WORKLOADS",
]


def planted_groups(n: int, n_groups: int, rng: np.random.Generator) -> np.ndarray:
    """Equal-size planted groups in a seeded random order (int64 labels)."""
    labels = np.empty(n, dtype=np.int64)
    labels[rng.permutation(n)] = np.arange(n) % n_groups
    return labels


def planted_loadings(n: int, n_groups: int, boundary_frac: float,
                     rng: np.random.Generator, lo: float = 0.5, hi: float = 1.0):
    """Loading matrix B (n x g, float64) and the planted hard label per instrument.

    Every instrument loads c ~ U[lo, hi] on its own group.  A seeded subset of
    round(boundary_frac * n) boundary instruments instead loads c*w on its own
    group and c*(1-w) on a second group drawn uniformly from the others, with
    w ~ U[0.3, 0.7]; its planted label is the group with the larger loading.
    """
    own = planted_groups(n, n_groups, rng)
    c = rng.uniform(lo, hi, size=n)
    B = np.zeros((n, n_groups), dtype=np.float64)
    B[np.arange(n), own] = c
    label = own.copy()
    n_b = int(round(boundary_frac * n))
    if n_b > 0 and n_groups > 1:
        idx = rng.choice(n, size=n_b, replace=False)
        second = rng.integers(0, n_groups - 1, size=n_b)
        second = second + (second >= own[idx])          # uniform over the other groups
        w = rng.uniform(0.3, 0.7, size=n_b)
        B[idx, own[idx]] = c[idx] * w
        B[idx, second] = c[idx] * (1.0 - w)
        label[idx] = np.where(w >= 0.5, own[idx], second)
    return B, label


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    if dist == "normal":
        return rng.standard_normal(shape)
    if dist == "t3":
        return rng.standard_t(3.0, size=shape)
    raise ValueError(f"unknown distribution {dist!r}")


def factor_returns(B: np.ndarray, T: int, sigma: float, dist: str,
                   rng: np.random.Generator, chunk: int = 16384) -> np.ndarray:
    """Returns window R (T x n, float32, row = day): R = F B^T + sigma * E."""
    n, g = B.shape
    F = _draw(rng, (T, g), dist)
    R = np.empty((T, n), dtype=np.float32)
    for c0 in range(0, n, chunk):
        c1 = min(n, c0 + chunk)
        E = _draw(rng, (T, c1 - c0), dist)
        R[:, c0:c1] = (F @ B[c0:c1].T + sigma * E).astype(np.float32)
    return R


# The workloads the path is exercised and measured on.  Field meanings:
#   n instruments, g planted groups, T days, sigma noise scale, dist of f and
#   eps, boundary fraction; k is the factorisation rank used with it.
WORKLOADS = {
    # 8 disjoint groups, B_own ~ U[0.5, 1], sigma = 1 (small parity case)
    "corr_n2000_k8": dict(n=2000, g=8, T=250, sigma=1.0, dist="normal", boundary=0.0, k=8),
    # 24 groups with 10% boundary instruments, sigma = 1.5
    "corr_n20000_k24": dict(n=20000, g=24, T=500, sigma=1.5, dist="normal", boundary=0.1, k=24),
    # heavy tails (Student-t, 3 dof, unscaled) for the tail-dependence matrix
    "tpdm_n20000_k24": dict(n=20000, g=24, T=1000, sigma=1.5, dist="t3", boundary=0.1, k=24),
    # the single-GPU scale: 100,000 instruments, one trading-year-scale window
    "corr_n100000_k24": dict(n=100000, g=24, T=1000, sigma=1.5, dist="normal", boundary=0.1, k=24),
    "tpdm_n100000_k24": dict(n=100000, g=24, T=1000, sigma=1.5, dist="t3", boundary=0.1, k=24),
}


def workload(name: str, seed: int = 0, n: int | None = None, T: int | None = None):
    """Draw a named workload: returns (R float32 T x n, planted labels, spec).

    ``n`` / ``T`` override the sizes (same recipe, smaller draw) for tests.
    """
    spec = dict(WORKLOADS[name])
    if n is not None:
        spec["n"] = n
    if T is not None:
        spec["T"] = T
    rng = np.random.default_rng(seed)
    B, label = planted_loadings(spec["n"], spec["g"], spec["boundary"], rng)
    R = factor_returns(B, spec["T"], spec["sigma"], spec["dist"], rng)
    return R, label, spec


def uniform_h0(n: int, k: int, scale: float, seed: int) -> np.ndarray:
    """A user-supplied starting point H0 (n x k float32, entries U[0, scale))."""
    rng = np.random.default_rng(seed)
    return (rng.random((n, k)) * scale).astype(np.float32)


def planted_block_matrix(sizes, order_seed: int | None = None):
    """Noise-free planted block matrix S = Z Z^T (float32) and its labels.

    Z is the n x g indicator of the groups with the given sizes; with
    ``order_seed`` the instruments are put in a seeded random order.
    """
    n = int(sum(sizes))
    labels = np.repeat(np.arange(len(sizes)), sizes)
    if order_seed is not None:
        labels = labels[np.random.default_rng(order_seed).permutation(n)]
    S = (labels[:, None] == labels[None, :]).astype(np.float32)
    return S, labels


class RollingStream:
    """A synthetic daily return stream with a membership switch and a joint
    tail shock (fields below), for the rolling-window pipeline."""

    def __init__(self, R, groups_before, groups_after, switchers, stressed, spec):
        self.R = R                          # days x n float32, row = day
        self.groups_before = groups_before  # planted hard labels before the switch day
        self.groups_after = groups_after    # ... from the switch day on
        self.switchers = switchers          # instruments that change group
        self.stressed = stressed            # groups hit by the joint tail shock
        self.spec = spec


def rolling_stream(seed: int = 0, n: int = 5000, g: int = 24, days: int = 499,
                   sigma: float = 1.5, boundary: float = 0.1, switch_day: int = 250,
                   switch_frac: float = 0.05, shock_days=(180, 200), shock_groups: int = 3,
                   shock_scale: float = 1.0) -> RollingStream:
    """The rolling workload's stream ("The temporal setup": planted groups, some
    instruments changing group, several groups in a joint tail-stress episode
    without changing membership).

    r_d = B_d f_d + sigma * eps_d with f, eps iid N(0,1); B_d = B before
    ``switch_day`` and B' from it on, where B' moves a seeded set of
    round(switch_frac * n) instruments' whole loading onto another group drawn
    uniformly from the rest.  On the days shock_days[0]..shock_days[1]
    (inclusive) every member (planted label before the switch) of
    ``shock_groups`` seeded groups gets -shock_scale * |z_d| added, z_d one
    Student-t(2) draw per day shared by all of them: a joint crash, which
    sits in the lower tail of the returns.  With the defaults a
    250-day window starting at day w holds w post-switch days, so the labels
    turn over around window 125.
    """
    rng = np.random.default_rng(seed)
    B, before = planted_loadings(n, g, boundary, rng)
    n_sw = int(round(switch_frac * n))
    switchers = np.sort(rng.choice(n, size=n_sw, replace=False)) if n_sw else np.zeros(0, np.int64)
    shift = rng.integers(1, g, size=n_sw) if g > 1 else np.zeros(n_sw, np.int64)
    new_group = (before[switchers] + shift) % g
    B_after = B.copy()
    total = B[switchers].sum(axis=1)
    B_after[switchers] = 0.0
    B_after[switchers, new_group] = total
    after = before.copy()
    after[switchers] = new_group
    stressed = np.sort(rng.choice(g, size=min(shock_groups, g), replace=False))
    F = rng.standard_normal((days, g))
    E = rng.standard_normal((days, n))
    z = rng.standard_t(2.0, size=days)
    R = np.empty((days, n), dtype=np.float64)
    R[:switch_day] = F[:switch_day] @ B.T
    R[switch_day:] = F[switch_day:] @ B_after.T
    R += sigma * E
    members = np.isin(before, stressed)
    d0, d1 = shock_days
    for d in range(max(d0, 0), min(d1 + 1, days)):
        R[d, members] -= shock_scale * abs(z[d])
    spec = dict(seed=seed, n=n, g=g, days=days, sigma=sigma, boundary=boundary,
                switch_day=switch_day, switch_frac=switch_frac, shock_days=tuple(shock_days),
                shock_groups=shock_groups, shock_scale=shock_scale)
    return RollingStream(R.astype(np.float32), before, after, switchers, stressed, spec)

