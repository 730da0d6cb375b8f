"""The row-sharded fit's exchange logic on CPU ranks (gloo, world size 2 and 3).

symmetric_nmf_clustering_b200.sharded.fit_sharded runs the loop and the
collectives; its four per-rank steps are passed in.  Here they are restated
with the oracle's functions on each rank's block of rows (fp64, H and G
rounded to float32 after every step as the library stores them), so the run
checks the sharding and the exchange -- which rows each rank owns, the
all-reduce of (Gram, trace), the all-gather of the new rows, the stopping rule
and the returned iterate -- against the oracle's single-process fit.
"""
import os
import socket
import tempfile
from datetime import timedelta

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
import synth


class OracleShardOps:
    """symnmf_shard_step and its helpers restated on one rank's rows."""

    def stats(self, S_rows, n):
        a, b, c = oracle.stats(S_rows.numpy())
        return torch.tensor([a, b, float(c)], dtype=torch.float64)

    def init(self, n, k, seed, s_sum):
        return torch.from_numpy(oracle.scale_matched_init(s_sum, n, k, seed))

    def gram(self, H_rows):
        h = H_rows.double().numpy()
        return torch.from_numpy(np.concatenate([(h.T @ h).ravel(), [0.0]]))

    def workspace(self, rows, n, k):
        return None

    def step(self, S_rows, row0, H, A, G_rows, lr, eps, H_next, G_next, ws):
        k = H.shape[1]
        rows = S_rows.shape[0]
        Hd = H.double().numpy()
        P = S_rows.double().numpy() @ Hd                 # this rank's rows of S H
        Hr = Hd[row0:row0 + rows]
        tr = float((Hr * P).sum())
        g = 4.0 * (Hr @ A.double().numpy().reshape(k, k) - P)
        Hn, Gn = oracle.adagrad_step(Hr, G_rows.double().numpy(), g, lr, eps)
        H_next.copy_(torch.from_numpy(Hn.astype(np.float32)))
        G_next.copy_(torch.from_numpy(Gn.astype(np.float32)))
        h = H_next.double().numpy()
        return torch.from_numpy(np.concatenate([(h.T @ h).ravel(), [tr]]))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, S, k, kw, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=120))
    try:
        from symmetric_nmf_clustering_b200.sharded import fit_sharded, shard_rows
        n = S.shape[0]
        r0, r1 = shard_rows(n, world, rank)
        H, st = fit_sharded(torch.from_numpy(np.ascontiguousarray(S[r0:r1])), r0, n, k,
                            ops=OracleShardOps(), **kw)
        torch.save({"H": H.numpy(), "st": st, "rows": (r0, r1)}, os.path.join(out, f"r{rank}.pt"))
    finally:
        dist.destroy_process_group()


def _run(world, S, k, **kw):
    with tempfile.TemporaryDirectory() as out:
        mp.spawn(_worker, args=(world, _free_port(), S, k, kw, out), nprocs=world, join=True)
        return [torch.load(os.path.join(out, f"r{r}.pt"), weights_only=False) for r in range(world)]


def _problem(n, k, seed):
    R, _, _ = synth.workload("corr_n2000_k8", seed=seed, n=n, T=60)
    return oracle.corr_abs(R).astype(np.float32)


@pytest.mark.parametrize("world,n", [(2, 300), (3, 520)])
def test_sharded_fit_equals_the_single_process_fit(world, n):
    k = 5
    S = _problem(n, k, world)
    res = _run(world, S, k, seed=11, max_iters=40, rel_tol=0.0)
    s_sum, sq, _ = oracle.stats(S)
    ref = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 11), max_iters=40,
                             S_sqnorm=sq)
    # every rank returns the same iterate, the oracle's
    for r in res:
        np.testing.assert_allclose(r["H"], ref.H, rtol=1e-9, atol=1e-12)
        np.testing.assert_allclose(r["st"]["history"], ref.history, rtol=1e-10)
        assert r["st"]["iters"] == 40 and r["st"]["world"] == world
    # the blocks are whole 128-row tiles in rank order covering [0, n)
    assert [r["rows"] for r in res][0][0] == 0 and res[-1]["rows"][1] == n
    assert all(res[p]["rows"][1] == res[p + 1]["rows"][0] for p in range(world - 1))
    assert all(r["rows"][0] % 128 == 0 for r in res)


def test_sharded_fit_stops_where_the_oracle_stops():
    n, k = 300, 4
    S = _problem(n, k, 7)
    res = _run(2, S, k, seed=3, max_iters=5000, rel_tol=1e-4)
    s_sum, sq, _ = oracle.stats(S)
    ref = oracle.fit_adagrad(S, k, oracle.scale_matched_init(s_sum, n, k, 3), max_iters=5000,
                             rel_tol=1e-4, S_sqnorm=sq)
    st = res[0]["st"]
    assert ref.converged and st["converged"] == 1
    assert st["iters"] == ref.iters and st["evaluations"] == len(ref.history)
    np.testing.assert_allclose(res[0]["H"], ref.H, rtol=1e-9, atol=1e-12)


def test_shard_rows_tiles_every_row_once():
    from symmetric_nmf_clustering_b200.sharded import shard_rows
    for n in (1, 127, 128, 129, 1000, 100000):
        for world in (1, 2, 3, 4, 8):
            b = [shard_rows(n, world, r) for r in range(world)]
            assert b[0][0] == 0 and b[-1][1] == n
            assert all(b[p][1] == b[p + 1][0] for p in range(world - 1))
            # a rank beyond the number of tiles gets an empty block at the end
            assert all(a % 128 == 0 or a == b2 == n for a, b2 in b)
            tiles = [(y - x + 127) // 128 for x, y in b]
            assert max(tiles) - min(tiles) <= 1
