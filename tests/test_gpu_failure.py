"""Failure detection on the GPU without a fault: the bounded pipeline waits.

symnmf_test_stall_pipeline(1) makes the S-stream kernel's TMA producer issue
no loads.  Its consumers' waits run out after about 2 s; the kernel raises
its error word, lets nothing in flight behind, frees its tensor memory and
returns; the call reports SYMNMF_ERR_TIMEOUT.  With the hook cleared, the
same CUDA context computes correctly again.
"""
import numpy as np
import pytest

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


def _problem(n, k, seed):
    import torch
    rng = np.random.default_rng(seed)
    A = rng.random((n, n), dtype=np.float32)
    S = ((A + A.T) * np.float32(0.5)).astype(np.float32)
    X = (rng.random((n, k)) * 0.5).astype(np.float32)
    return S, torch.from_numpy(S).to(DEV), torch.from_numpy(X).to(DEV)


def _stalled(lib, call):
    from symmetric_nmf_clustering_b200 import _lib as L
    try:
        assert lib.symnmf_test_stall_pipeline(1) == 0
        with pytest.raises(L.SymNMFError) as e:
            call()
    finally:
        assert lib.symnmf_test_stall_pipeline(0) == 0
    assert e.value.status == L.SYMNMF_ERR_TIMEOUT
    assert "timed out" in str(e.value)


def test_sh_reports_the_timeout_and_the_context_recovers(m):
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    lib = L.load()
    S_host, S, X = _problem(1000, 8, 0)
    _stalled(lib, lambda: m.sh(S, X))
    Y = m.sh(S, X)
    torch.cuda.synchronize()
    ref = S_host.astype(np.float64) @ X.cpu().numpy().astype(np.float64)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) <= 1e-4 * np.linalg.norm(ref)


def test_fit_reports_the_timeout_and_the_context_recovers(m):
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    lib = L.load()
    _, S, _ = _problem(600, 6, 1)
    _stalled(lib, lambda: m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0))
    H1, st1 = m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0)
    H2, st2 = m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0)
    torch.cuda.synchronize()
    assert st1["iters"] == 20 and np.isfinite(st1["loss"])
    assert torch.equal(H1, H2) and st1["loss"] == st2["loss"]


def test_sh_upper_reports_the_timeout_and_the_context_recovers(m):
    # the upper-triangle stream's waits are bounded the same way
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    lib = L.load()
    S_host, S, X = _problem(1000, 8, 2)
    _stalled(lib, lambda: m.sh_upper(S, X))
    Y = m.sh_upper(S, X)
    torch.cuda.synchronize()
    ref = S_host.astype(np.float64) @ X.cpu().numpy().astype(np.float64)
    got = Y.cpu().numpy().astype(np.float64)
    assert np.linalg.norm(got - ref) <= 1e-4 * np.linalg.norm(ref)


def test_fit_on_the_fp16_stream_reports_the_timeout_and_the_context_recovers(m):
    # the fp16 S-stream (here forced at a small size) bounds its waits the same way
    import os
    import torch
    from symmetric_nmf_clustering_b200 import _lib as L
    lib = L.load()
    _, S, _ = _problem(600, 6, 3)
    old = os.environ.get("SYMNMF_H16_MIN_N")
    os.environ["SYMNMF_H16_MIN_N"] = "1"
    try:
        _stalled(lib, lambda: m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0))
        H1, st1 = m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0)
        H2, st2 = m.fit(S, 6, seed=3, max_iters=20, rel_tol=0.0)
        torch.cuda.synchronize()
    finally:
        if old is None:
            os.environ.pop("SYMNMF_H16_MIN_N", None)
        else:
            os.environ["SYMNMF_H16_MIN_N"] = old
    assert st1["stream_kernel"] == L.STREAM_FP16
    assert st1["iters"] == 20 and np.isfinite(st1["loss"])
    assert torch.equal(H1, H2) and st1["loss"] == st2["loss"]
