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
