"""The spectral probe's host eigen-solvers against LAPACK (numpy).

The block Lanczos probe reduces S to a block tridiagonal matrix T of at most a
few hundred rows and takes its leading eigenvalues on the host (reduction to
tridiagonal form: by bulge-chasing Givens rotations for a band matrix, by
Householder reflections otherwise; then Sturm bisection); Cholesky and cyclic Jacobi
orthonormalise each new block.  These run without a GPU: the test compiles
them with a small C shim and checks them against numpy.linalg.
"""
import ctypes as C
import os
import shutil
import subprocess

import numpy as np
import pytest

HERE = os.path.dirname(os.path.abspath(__file__))
CSRC = os.path.join(HERE, "..", "symmetric_nmf_clustering_b200", "csrc")


@pytest.fixture(scope="module")
def hl(tmp_path_factory):
    cxx = shutil.which("g++") or shutil.which("c++")
    if cxx is None:
        pytest.skip("no C++ compiler")
    out = str(tmp_path_factory.mktemp("hostla") / "libhostla.so")
    subprocess.run([cxx, "-O2", "-std=c++17", "-shared", "-fPIC", "-I", CSRC,
                    os.path.join(CSRC, "hostla.cpp"), os.path.join(HERE, "hostla_shim.cpp"),
                    "-o", out], check=True)
    lib = C.CDLL(out)
    dp = C.POINTER(C.c_double)
    lib.hl_top_eigvals.argtypes = [C.c_int, dp, C.c_int, dp]
    lib.hl_top_eigvals.restype = C.c_int
    lib.hl_jacobi.argtypes = [C.c_int, dp, dp, dp]
    lib.hl_cholesky_upper.argtypes = [C.c_int, dp, dp]
    lib.hl_cholesky_upper.restype = C.c_int
    return lib


def _p(a):
    return a.ctypes.data_as(C.POINTER(C.c_double))


def top(hl, A, count):
    A = np.ascontiguousarray(A, dtype=np.float64)
    out = np.zeros(max(count, 1))
    got = hl.hl_top_eigvals(A.shape[0], _p(A), count, _p(out))
    return out[:got]


def block_tridiagonal(rng, blocks, b):
    m = blocks * b
    T = np.zeros((m, m))
    for j in range(blocks):
        D = rng.standard_normal((b, b))
        T[j * b:(j + 1) * b, j * b:(j + 1) * b] = (D + D.T) / 2 + 5.0 * np.eye(b) * (blocks - j)
        if j + 1 < blocks:
            B = np.triu(rng.standard_normal((b, b)))
            T[(j + 1) * b:(j + 2) * b, j * b:(j + 1) * b] = B
            T[j * b:(j + 1) * b, (j + 1) * b:(j + 2) * b] = B.T
    return T


@pytest.mark.parametrize("m,count", [(1, 1), (2, 2), (3, 2), (17, 10), (64, 26), (192, 26)])
def test_top_eigenvalues_random_symmetric(hl, m, count):
    rng = np.random.default_rng(m)
    X = rng.standard_normal((m, m))
    A = (X + X.T) / 2
    ref = np.sort(np.linalg.eigvalsh(A))[::-1][:count]
    got = top(hl, A, count)
    assert got.shape == ref.shape
    assert np.max(np.abs(got - ref)) <= 1e-11 * max(1.0, np.max(np.abs(ref)))


@pytest.mark.parametrize("blocks,b", [(2, 16), (7, 16), (12, 16), (5, 8)])
def test_top_eigenvalues_block_tridiagonal(hl, blocks, b):
    # the shape the probe builds: a symmetric block tridiagonal Lanczos matrix
    T = block_tridiagonal(np.random.default_rng(blocks * b), blocks, b)
    ref = np.sort(np.linalg.eigvalsh(T))[::-1][:26]
    got = top(hl, T, 26)
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


@pytest.mark.parametrize("blocks,b,count", [(41, 16, 64), (30, 8, 26), (70, 4, 40)])
def test_top_eigenvalues_band_path_at_the_probe_sizes(hl, blocks, b, count):
    # m >= 8 b: the band reduction (Givens rotations with bulge chasing) runs;
    # (41, 16) is the 64-eigenvalue probe's final Rayleigh-Ritz matrix
    T = block_tridiagonal(np.random.default_rng(blocks + b), blocks, b)
    ref = np.sort(np.linalg.eigvalsh(T))[::-1][:count]
    got = top(hl, T, count)
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


@pytest.mark.parametrize("w", [1, 2, 3, 7])
def test_top_eigenvalues_random_band_matrices(hl, w):
    # general band matrices (full bands, not triangular coupling blocks), zero
    # entries inside the band, a decoupled block and an indefinite spectrum
    rng = np.random.default_rng(w + 40)
    m = 120
    A = np.zeros((m, m))
    for dd in range(w + 1):
        v = rng.standard_normal(m - dd)
        v[rng.random(m - dd) < 0.2] = 0.0
        A += np.diag(v, -dd) + (np.diag(v, dd) if dd else 0)
    A[60:, :60] = 0.0
    A[:60, 60:] = 0.0
    ref = np.sort(np.linalg.eigvalsh(A))[::-1][:30]
    got = top(hl, A, 30)
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


@pytest.mark.parametrize("scale", [1e-200, 1e-150, 1e150, 1e200])
def test_top_eigenvalues_band_path_far_from_unit_scale(hl, scale):
    # rotations whose squared entries under- or overflow fall back to hypot
    T = block_tridiagonal(np.random.default_rng(9), 20, 4) * scale
    ref = np.sort(np.linalg.eigvalsh(T / scale))[::-1][:10] * scale
    got = top(hl, T, 10)
    assert np.all(np.isfinite(got))
    assert np.max(np.abs(got - ref)) <= 1e-11 * np.max(np.abs(ref))


def test_top_eigenvalues_repeated_negative_and_degenerate(hl):
    # repeated eigenvalues (a rotated diagonal), an indefinite spectrum, a zero
    # matrix and more requested values than rows
    rng = np.random.default_rng(7)
    lam = np.array([5.0, 5.0, 5.0, 2.0, 0.0, -1.0, -1.0, -7.0])
    Q, _ = np.linalg.qr(rng.standard_normal((8, 8)))
    A = (Q * lam) @ Q.T
    A = (A + A.T) / 2
    assert np.max(np.abs(top(hl, A, 8) - np.sort(lam)[::-1])) <= 1e-12 * 7.0
    assert np.array_equal(top(hl, np.zeros((5, 5)), 3), np.zeros(3))
    assert top(hl, np.eye(4) * 2.0, 9).shape == (4,)
    assert np.allclose(top(hl, np.array([[3.5]]), 1), [3.5], rtol=0, atol=1e-15)


@pytest.mark.parametrize("m", [1, 3, 16])
def test_jacobi_eigendecomposition(hl, m):
    rng = np.random.default_rng(m + 100)
    X = rng.standard_normal((m, m))
    A = np.ascontiguousarray((X + X.T) / 2)
    w, V = np.zeros(m), np.zeros((m, m))
    hl.hl_jacobi(m, _p(A), _p(w), _p(V))
    assert np.allclose(np.sort(w), np.linalg.eigvalsh(A), rtol=0, atol=1e-12)
    assert np.allclose(V.T @ V, np.eye(m), atol=1e-12)
    assert np.allclose(A @ V, V * w, atol=1e-11)


def test_cholesky_upper(hl):
    rng = np.random.default_rng(3)
    X = rng.standard_normal((16, 16))
    M = np.ascontiguousarray(X @ X.T + 16 * np.eye(16))
    R = np.zeros((16, 16))
    assert hl.hl_cholesky_upper(16, _p(M), _p(R)) == 1
    assert np.allclose(R, np.triu(R)) and np.all(np.diag(R) > 0)
    assert np.allclose(R.T @ R, M, rtol=1e-13, atol=1e-12)
    # not positive definite: refused
    N = np.ascontiguousarray(np.diag([1.0, -1.0, 2.0]))
    assert hl.hl_cholesky_upper(3, _p(N), _p(np.zeros((3, 3)))) == 0
