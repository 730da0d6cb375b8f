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
