"""symnmf_sh_noalloc: the S-stream product for callers that cannot allocate.

Some callers cannot call cudaMalloc when they call into the library: a
runtime whose device memory is owned entirely by its own pool (or by another
framework's caching allocator), where an outside allocation would fragment it
or exceed its budget, or a latency-critical loop that cannot take cudaMalloc's
implicit synchronisation.  This entry point takes no workspace; its scratch is
a fixed device array inside the library.  The test calls it through the C ABI
twice in a row and compares it with symnmf_sh, which uses a workspace.

The file name makes pytest collect it last.
"""
import ctypes as C

import numpy as np
import pytest

DEV = "cuda:0"


def _rel(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    import torch
    from symmetric_nmf_clustering_b200 import build
    build.build()
    import symmetric_nmf_clustering_b200 as m
    from symmetric_nmf_clustering_b200 import _lib
    lib = _lib.load()

    n, k = 3001, 24                       # several 128-row tiles and a ragged tail
    lds = (n + 3) // 4 * 4
    rng = np.random.default_rng(21)
    A = rng.random((n, n), dtype=np.float32)
    S_host = (A + A.T) * np.float32(0.5)
    S = torch.zeros((n, lds), dtype=torch.float32, device=DEV)
    S[:, :n] = torch.from_numpy(S_host).to(DEV)
    S = S[:, :n]
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        X = torch.from_numpy((rng.random((n, k)) * 0.5).astype(np.float32)).to(DEV)
        Y = torch.empty_like(X)
        status = lib.symnmf_sh_noalloc(S.data_ptr(), n, lds, X.data_ptr(), k, Y.data_ptr(), stream)
        assert status == 0, lib.symnmf_last_error()
        Y_ws = m.sh(S, X)
        torch.cuda.synchronize()
        got, want = Y.cpu().numpy(), Y_ws.cpu().numpy()
        assert _rel(got, want) <= 2e-6, f"call {call}"
        ref = S_host.astype(np.float64) @ X.cpu().numpy().astype(np.float64)
        assert _rel(got, ref) <= 1e-4


def test_noalloc_rejects_sizes_beyond_its_scratch():
    # argument checks only (no device call): runs without a GPU as well
    from symmetric_nmf_clustering_b200 import build
    build.build()
    from symmetric_nmf_clustering_b200 import _lib
    lib = _lib.load()
    fake = 1 << 20   # never dereferenced: the size check comes first
    # k = 24: 2 * 24 * roundup(n, 32) + 64 <= 1,048,576 allows n <= 21,824
    assert lib.symnmf_sh_noalloc(fake, 21825, 21828, fake, 24, fake, None) == _lib.SYMNMF_ERR_INVALID_ARG
    assert b"static scratch" in lib.symnmf_last_error()
    # a size whose scratch product would wrap around 2^64 (2 * 8 * 2^60) is
    # rejected on n alone, before the product is formed
    big = 1 << 60
    assert lib.symnmf_sh_noalloc(fake, big, big, fake, 8, fake, None) == _lib.SYMNMF_ERR_INVALID_ARG
    # n * lds overflow, and misaligned X or Y, as for symnmf_sh
    assert lib.symnmf_sh_noalloc(fake, 1000, 1 << 62, fake, 8, fake, None) == _lib.SYMNMF_ERR_INVALID_ARG
    assert lib.symnmf_sh_noalloc(fake, 1000, 1000, fake + 2, 8, fake, None) == _lib.SYMNMF_ERR_INVALID_ARG
    assert lib.symnmf_sh_noalloc(fake, 1000, 1000, fake, 8, fake + 1, None) == _lib.SYMNMF_ERR_INVALID_ARG
