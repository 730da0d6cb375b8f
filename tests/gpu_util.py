"""Shared helpers of the GPU parity tests (inputs and comparisons only)."""
import numpy as np

import oracle
import synth


def rel_fro(a, b):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def corr_problem(n, T, seed, name="corr_n2000_k8"):
    """Returns window, planted labels and the oracle's |corr| S rounded to float32."""
    R, planted, _ = synth.workload(name, seed=seed, n=n, T=T)
    S = oracle.corr_abs(R).astype(np.float32)
    return R, planted, S


def tpdm_problem(n, T, seed, tail_frac=0.05):
    R, planted, _ = synth.workload("tpdm_n20000_k24", seed=seed, n=n, T=T)
    S = oracle.tpdm(R, tail_frac, 1).astype(np.float32)
    return R, planted, S


def to_dev(x, device, pad4=False):
    import torch
    x = np.ascontiguousarray(x)
    if pad4 and x.ndim == 2 and x.shape[1] % 4:
        lds = (x.shape[1] + 3) // 4 * 4
        buf = torch.full((x.shape[0], lds), float("nan"), dtype=torch.float32, device=device)
        buf[:, :x.shape[1]] = torch.from_numpy(x).to(device)
        return buf[:, :x.shape[1]]
    return torch.from_numpy(x).to(device)


def assert_labels_differ_only_on_near_ties(lab_gpu, lab_oracle, H_gpu, H_oracle, tol=1e-3):
    """Labels of two factors that agree to the fit's H tolerance.

    Every row whose labels differ must be a near-tie that the H difference
    explains: the oracle's top-two margin there is at most twice that row's
    largest deviation |H_gpu - H_oracle| (a smaller margin cannot flip the
    argmax), and at most tol * max|H| (the H tolerance).  Returns and prints
    the number of differing rows, so a run shows how many there were.
    """
    lab_gpu = np.asarray(lab_gpu)
    lab_oracle = np.asarray(lab_oracle)
    H_gpu = np.asarray(H_gpu, dtype=np.float64)
    H_oracle = np.asarray(H_oracle, dtype=np.float64)
    diff = lab_gpu != lab_oracle
    srt = np.sort(H_oracle, axis=1)
    margin = srt[:, -1] - srt[:, -2] if H_oracle.shape[1] > 1 else np.full(len(srt), np.inf)
    dev = np.abs(H_gpu - H_oracle).max(axis=1)
    bad = diff & ((margin > 2.0 * dev) | (margin > tol * np.abs(H_oracle).max()))
    print(f"labels: {int(diff.sum())} of {diff.size} rows differ, all on near-ties"
          if not bad.any() else f"labels: {int(bad.sum())} rows differ on clear margins")
    assert not bad.any(), np.flatnonzero(bad)[:10]
    return int(diff.sum())


class DeviceRowChunks:
    """A device n x n float32 matrix as the oracle's solvers see it when it is
    too large to widen at once: it supplies S @ X and S[:, cols] @ D in
    float64, copying row chunks (or their column slabs) from the device into
    pinned host memory, widening them exactly to float64 in a reused buffer
    and multiplying on the host.  Test plumbing only: copies and a library
    matrix product, none of the method's arithmetic."""

    exact_float64_products = True

    def __init__(self, S_dev, rows_per_chunk=2048):
        import torch
        self.S = S_dev
        self.n = S_dev.shape[0]
        self.shape = (self.n, S_dev.shape[1])
        self.c = rows_per_chunk
        self.cuda = S_dev.is_cuda
        pin = torch.empty(self.c * self.shape[1], dtype=torch.float32)
        self.pin = pin.pin_memory() if self.cuda else pin
        self.f64 = torch.empty(self.c * self.shape[1], dtype=torch.float64)

    def _chunks(self, c0=0, c1=None):
        import torch
        c1 = self.shape[1] if c1 is None else c1
        w = c1 - c0
        for r0 in range(0, self.n, self.c):
            r1 = min(self.n, r0 + self.c)
            hb = self.pin[: (r1 - r0) * w].view(r1 - r0, w)     # contiguous
            hb.copy_(self.S[r0:r1, c0:c1])
            if self.cuda:
                torch.cuda.synchronize()
            db = self.f64[: (r1 - r0) * w].view(r1 - r0, w)
            db.copy_(hb)
            yield r0, r1, db

    def __matmul__(self, X):
        import torch
        X = torch.from_numpy(np.ascontiguousarray(X, dtype=np.float64))
        out = np.empty((self.n, X.shape[1]))
        for r0, r1, db in self._chunks():
            out[r0:r1] = torch.mm(db, X).numpy()
        return out

    def __getitem__(self, key):
        rows, cols = key
        assert rows == slice(None, None, None) and isinstance(cols, slice) and cols.step is None
        return _ColumnSlab(self, cols.start, min(cols.stop, self.shape[1]))

    def stats(self):
        """(sum, squared norm, non-finite count) from the oracle's stats on each chunk."""
        t = [0.0, 0.0, 0]
        for _, _, db in self._chunks():
            a, b, c = oracle.stats(db.numpy())
            t[0] += a
            t[1] += b
            t[2] += c
        return tuple(t)


class _ColumnSlab:
    def __init__(self, parent, c0, c1):
        self.p, self.c0, self.c1 = parent, c0, c1

    def __matmul__(self, D):
        import torch
        D = torch.from_numpy(np.ascontiguousarray(D, dtype=np.float64))
        out = np.empty((self.p.n, D.shape[1]))
        for r0, r1, db in self.p._chunks(self.c0, self.c1):
            out[r0:r1] = torch.mm(db, D).numpy()
        return out
