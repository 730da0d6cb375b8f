"""Row-sharded full-batch fit across processes (one per GPU).

The pages scale the factorisation out by sharding S by rows while every GPU
keeps a replica of H: each forms its rows of S H locally, and the ranks
exchange O(n k) data per iteration ([CaS] "Factorization at scale",
"Scale-out").  Here rank p holds a contiguous block of rows of S (all n
columns) and the whole iterate H.  One iteration:

    every rank    symnmf_shard_step on its rows: S-stream, trace term, AdaGrad
                  step of its rows of H, Gram of its new rows (one kernel pass
                  with the fused epilogue)
    all-reduce    (Gram of the new rows, trace term): k^2 + 1 fp64 numbers,
                  giving H_{t+1}^T H_{t+1} and tr(H_t^T S H_t), hence the loss
                  f(H_t) = ||S||^2 - 2 tr + ||H_t^T H_t||^2 on every rank
    all-gather    the new rows of H (n k floats), giving H_{t+1} everywhere

The stopping rule and the returned iterate are those of symnmf_fit: evaluation
t computes f(H_t); the fit stops at the first t > 0 whose relative change is
below rel_tol, or at t = max_iters, and returns H_t.

This module is plumbing: it moves tensors and calls torch.distributed; every
step of the method runs in the library's kernels (``DeviceShardOps``).  The
per-rank operations are passed in as an object, so the exchange logic can be
exercised on CPU ranks with other implementations of the same four steps.
"""
from __future__ import annotations

import ctypes as C
import math

import torch
import torch.distributed as dist

from . import _lib as L

TILE = 128


def shard_rows(n: int, world: int, rank: int) -> tuple[int, int]:
    """Rows [r0, r1) of rank `rank`: whole 128-row tiles, split as evenly as
    possible, the first ranks taking one tile more."""
    tiles = (n + TILE - 1) // TILE
    base, extra = divmod(tiles, world)
    t0 = rank * base + min(rank, extra)
    t1 = t0 + base + (1 if rank < extra else 0)
    return min(n, t0 * TILE), min(n, t1 * TILE)


class DeviceShardOps:
    """The four per-rank steps through the C ABI, on the device that holds S."""

    def __init__(self, device):
        self.device = torch.device(device)
        self.lib = L.load()

    def _stream(self):
        return torch.cuda.current_stream(self.device).cuda_stream

    def stats(self, S_rows, n):
        rows, lds = S_rows.shape[0], S_rows.stride(0)
        out = torch.empty(3, dtype=torch.float64, device=self.device)
        size = C.c_size_t(0)
        L.check("symnmf_workspace_size", self.lib.symnmf_workspace_size(
            L.OP_STATS, n, 1, 0, None, C.byref(size)))
        ws = torch.empty(int(size.value), dtype=torch.uint8, device=self.device)
        L.check("symnmf_stats_rows", self.lib.symnmf_stats_rows(
            S_rows.data_ptr(), rows, n, lds, out.data_ptr(), ws.data_ptr(), ws.numel(),
            self._stream()))
        return out

    def init(self, n, k, seed, s_sum):
        H = torch.empty((n, k), dtype=torch.float32, device=self.device)
        L.check("symnmf_seeded_init", self.lib.symnmf_seeded_init(
            H.data_ptr(), n, k, int(seed) & (2 ** 64 - 1), float(s_sum), self._stream()))
        return H

    def gram(self, H_rows):
        rows, k = H_rows.shape
        A = torch.empty(k * k + 1, dtype=torch.float64, device=self.device)
        tiles = (rows + TILE - 1) // TILE
        ws = torch.empty((tiles * (k * k + 1) + 64) * 8 + 1024, dtype=torch.uint8, device=self.device)
        L.check("symnmf_gram", self.lib.symnmf_gram(H_rows.data_ptr(), rows, k, A.data_ptr(),
                                                    ws.data_ptr(), ws.numel(), self._stream()))
        A[k * k] = 0.0
        return A

    def workspace(self, rows, n, k):
        size = C.c_size_t(0)
        L.check("symnmf_shard_workspace_size",
                self.lib.symnmf_shard_workspace_size(rows, n, k, C.byref(size)))
        return torch.empty(int(size.value), dtype=torch.uint8, device=self.device)

    def step(self, S_rows, row0, H, A, G_rows, lr, eps, H_next, G_next, ws):
        rows, lds = S_rows.shape[0], S_rows.stride(0)
        n, k = H.shape
        part = torch.empty(k * k + 1, dtype=torch.float64, device=self.device)
        L.check("symnmf_shard_step", self.lib.symnmf_shard_step(
            S_rows.data_ptr(), rows, n, lds, row0, k, H.data_ptr(), A.data_ptr(),
            G_rows.data_ptr(), float(lr), float(eps), H_next.data_ptr(), G_next.data_ptr(),
            part.data_ptr(), ws.data_ptr(), ws.numel(), self._stream()))
        return part


def _all_reduce(t, group):
    if dist.is_available() and dist.is_initialized():
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
    return t


def _all_gather_rows(H, rows_local, r0s, r1s, rank, group):
    """H[r0s[p]:r1s[p]] = rows of rank p, for every p (blocks padded to one size)."""
    world = len(r0s)
    if world == 1:
        H[r0s[0]:r1s[0]].copy_(rows_local)
        return H
    mx = max(b - a for a, b in zip(r0s, r1s))
    k = H.shape[1]
    send = torch.zeros((mx, k), dtype=H.dtype, device=H.device)
    send[: rows_local.shape[0]].copy_(rows_local)
    recv = torch.empty((world * mx, k), dtype=H.dtype, device=H.device)
    dist.all_gather_into_tensor(recv, send, group=group)
    for p in range(world):
        H[r0s[p]:r1s[p]].copy_(recv[p * mx: p * mx + (r1s[p] - r0s[p])])
    return H


def fit_sharded(S_rows: torch.Tensor, row0: int, n: int, k: int, *, seed: int = 0,
                lr: float = 0.1, eps: float = 1e-10, max_iters: int = 2000,
                rel_tol: float = 1e-5, group=None, ops=None):
    """Full-batch projected AdaGrad on the row-sharded S (one call per rank).

    S_rows: this rank's rows [row0, row0 + rows) of S, rows x n (row pitch a
    multiple of 4).  Every rank must pass the same n, k and options, and the
    ranks' blocks must cover [0, n) in rank order.  Returns (H, stats): the
    returned iterate H (n x k, the same on every rank) and a dict with the
    loss history, iterations, convergence flag and final loss.
    """
    world = dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1
    rank = dist.get_rank(group) if world > 1 else 0
    rows = S_rows.shape[0]
    if rows < 1:
        raise ValueError("every rank needs at least one row of S (n > 128 (world - 1))")
    ops = DeviceShardOps(S_rows.device) if ops is None else ops
    # every rank's block, in rank order
    bounds = torch.tensor([row0, row0 + rows], dtype=torch.int64, device=S_rows.device)
    if world > 1:
        allb = [torch.empty_like(bounds) for _ in range(world)]
        dist.all_gather(allb, bounds, group=group)
        r0s = [int(b[0]) for b in allb]
        r1s = [int(b[1]) for b in allb]
    else:
        r0s, r1s = [row0], [row0 + rows]
    if r0s[0] != 0 or r1s[-1] != n or any(r1s[p] != r0s[p + 1] for p in range(world - 1)):
        raise ValueError(f"the ranks' row blocks {list(zip(r0s, r1s))} do not tile [0, {n})")

    st = _all_reduce(ops.stats(S_rows, n), group)
    s_sum, s_sq, bad = (float(x) for x in st.cpu())
    if bad > 0:
        raise ValueError(f"S holds {bad:.0f} non-finite entries")
    H = ops.init(n, k, seed, s_sum)                       # the same draw on every rank
    A = _all_reduce(ops.gram(H[row0:row0 + rows]), group)[: k * k].contiguous()
    Hn = torch.empty_like(H)
    G = torch.zeros((rows, k), dtype=torch.float32, device=S_rows.device)
    Gn = torch.empty_like(G)
    Hr_next = torch.empty((rows, k), dtype=torch.float32, device=S_rows.device)
    ws = ops.workspace(rows, n, k)
    history = []
    t, L_prev, rel, converged = 0, None, math.nan, False
    while True:
        part = ops.step(S_rows, row0, H, A, G, lr, eps, Hr_next, Gn, ws)
        part = _all_reduce(part, group)
        a2 = float((A.double() * A.double()).sum())
        tr = float(part[k * k])
        Lt = s_sq - 2.0 * tr + a2
        history.append(Lt)
        if not math.isfinite(Lt):
            raise FloatingPointError(f"the loss became non-finite at evaluation {t}")
        if L_prev is not None:
            rel = abs(Lt - L_prev) / abs(L_prev) if L_prev != 0.0 else (0.0 if Lt == L_prev else math.inf)
            if rel_tol > 0.0 and rel < rel_tol:
                converged = True
                break
        if t == max_iters:
            break
        # H_{t+1} on every rank, its Gram, the accumulator of this rank's rows
        _all_gather_rows(Hn, Hr_next, r0s, r1s, rank, group)
        H, Hn = Hn, H
        A = part[: k * k].contiguous()
        G, Gn = Gn, G
        L_prev = Lt
        t += 1
    return H, {"iters": t, "evaluations": len(history), "loss": history[-1], "rel_change": rel,
               "converged": int(converged), "history": history, "s_sqnorm": s_sq,
               "s_mean": s_sum / (float(n) * float(n)), "world": world}
