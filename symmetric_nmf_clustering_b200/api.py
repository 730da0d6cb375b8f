"""Python binding of libsymnmf.so: argument marshalling only.

PyTorch provides device memory and the current CUDA stream; every step of the
SymNMF path runs in the library's kernels.  Function names follow the C ABI
(include/symnmf.h) without the ``symnmf_`` prefix.
"""
from __future__ import annotations

import ctypes as C

import numpy as np
import torch

from . import _lib as L

__all__ = ["alloc_S", "workspace", "build_corr", "build_tpdm", "stats", "sh",
           "spectral_probe", "fit", "labels", "fit_params", "FitParams", "FitStats"]

FitParams = L.FitParams
FitStats = L.FitStats
_SOLVERS = {"adagrad": L.SOLVER_ADAGRAD, "block_svrg": L.SOLVER_BLOCK_SVRG, "auto": L.SOLVER_AUTO}


def _lib():
    return L.load()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _check_cuda(t: torch.Tensor, name: str, dtype=torch.float32):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _dense(t: torch.Tensor, name: str):
    _check_cuda(t, name)
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous (row-major)")


def _matrix(t: torch.Tensor, name: str):
    """(rows, cols, leading dimension) of a row-major matrix with unit column stride."""
    _check_cuda(t, name)
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be a 2-D row-major matrix (unit column stride)")
    return t.shape[0], t.shape[1], t.stride(0)


def alloc_S(n: int, device=None) -> torch.Tensor:
    """An n x n float32 matrix whose rows are padded to a multiple of 4 floats."""
    lds = (n + 3) // 4 * 4
    return torch.empty((n, lds), dtype=torch.float32, device=device)[:, :n]


def workspace(op: int, n: int, k: int = 0, T: int = 0, params: FitParams | None = None,
              device=None) -> torch.Tensor:
    size = C.c_size_t(0)
    L.check("symnmf_workspace_size",
            _lib().symnmf_workspace_size(op, n, k, T, C.byref(params) if params is not None else None,
                                         C.byref(size)))
    return torch.empty(max(int(size.value), 256), dtype=torch.uint8, device=device)


def build_corr(R: torch.Tensor, out: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """S = |Pearson correlation| of the columns of the T x n window R."""
    T, n, ldr = _matrix(R, "R")
    S = alloc_S(n, R.device) if out is None else out
    nS, nS2, lds = _matrix(S, "out")
    if (nS, nS2) != (n, n):
        raise ValueError("out must be n x n")
    ws = workspace(L.OP_BUILD_CORR, n, 0, T, device=R.device) if ws is None else ws
    L.check("symnmf_build_corr", _lib().symnmf_build_corr(
        R.data_ptr(), T, n, ldr, S.data_ptr(), lds, ws.data_ptr(), ws.numel(), _stream(R.device)))
    return S


def build_tpdm(R: torch.Tensor, tail_frac: float = 0.05, tail_sign: int = 1,
               out: torch.Tensor | None = None, ws: torch.Tensor | None = None):
    """S = TPDM of the T x n window R (top tail_frac of days by radius, scaled by n)."""
    T, n, ldr = _matrix(R, "R")
    S = alloc_S(n, R.device) if out is None else out
    nS, nS2, lds = _matrix(S, "out")
    if (nS, nS2) != (n, n):
        raise ValueError("out must be n x n")
    ws = workspace(L.OP_BUILD_TPDM, n, 0, T, device=R.device) if ws is None else ws
    L.check("symnmf_build_tpdm", _lib().symnmf_build_tpdm(
        R.data_ptr(), T, n, ldr, float(tail_frac), int(tail_sign), S.data_ptr(), lds,
        ws.data_ptr(), ws.numel(), _stream(R.device)))
    return S


def stats(S: torch.Tensor, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Device tensor [sum S, ||S||_F^2, non-finite count] (float64)."""
    n, _, lds = _matrix(S, "S")
    out = torch.empty(3, dtype=torch.float64, device=S.device)
    ws = workspace(L.OP_STATS, n, device=S.device) if ws is None else ws
    L.check("symnmf_stats", _lib().symnmf_stats(S.data_ptr(), n, lds, out.data_ptr(),
                                                ws.data_ptr(), ws.numel(), _stream(S.device)))
    return out


def sh(S: torch.Tensor, X: torch.Tensor, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Y = S X for an n x k block X (one pass over S)."""
    n, _, lds = _matrix(S, "S")
    _dense(X, "X")
    k = X.shape[1]
    Y = torch.empty_like(X)
    ws = workspace(L.OP_SH, n, k, device=S.device) if ws is None else ws
    L.check("symnmf_sh", _lib().symnmf_sh(S.data_ptr(), n, lds, X.data_ptr(), k, Y.data_ptr(),
                                          ws.data_ptr(), ws.numel(), _stream(S.device)))
    return Y


def sh_upper(S: torch.Tensor, X: torch.Tensor, ws: torch.Tensor | None = None) -> torch.Tensor:
    """Y = S X reading only the tiles of S on or above the diagonal (k <= 24)."""
    n, _, lds = _matrix(S, "S")
    _dense(X, "X")
    k = X.shape[1]
    Y = torch.empty_like(X)
    ws = workspace(L.OP_SH_UPPER, n, k, device=S.device) if ws is None else ws
    L.check("symnmf_sh_upper", _lib().symnmf_sh_upper(S.data_ptr(), n, lds, X.data_ptr(), k,
                                                      Y.data_ptr(), ws.data_ptr(), ws.numel(),
                                                      _stream(S.device)))
    return Y


def spectral_probe(S: torch.Tensor, n_eig: int, block: int = 16, max_iter: int = 40,
                   tol: float = 1e-6, seed: int = 0, ws: torch.Tensor | None = None) -> np.ndarray:
    """The n_eig leading eigenvalues of S (descending) by block Lanczos."""
    n, _, lds = _matrix(S, "S")
    p = fit_params(probe_block=block, probe_max_iter=max_iter)
    ws = workspace(L.OP_SPECTRAL_PROBE, n, n_eig, params=p, device=S.device) if ws is None else ws
    out = (C.c_double * n_eig)()
    L.check("symnmf_spectral_probe", _lib().symnmf_spectral_probe(
        S.data_ptr(), n, lds, n_eig, block, max_iter, float(tol), int(seed) & (2**64 - 1), out,
        ws.data_ptr(), ws.numel(), _stream(S.device)))
    return np.array(out[:], dtype=np.float64)


def probe_last_info() -> dict:
    """S passes, block steps and kernel launches of the last spectral_probe
    call on this thread (the probe's bytes are s_passes * 4 n^2)."""
    info = L.ProbeInfo()
    L.check("symnmf_probe_last_info", _lib().symnmf_probe_last_info(C.byref(info)))
    return {"s_passes": info.s_passes, "block_steps": info.block_steps,
            "kernel_launches": info.kernel_launches}


def fit_params(**kw) -> FitParams:
    p = FitParams()
    _lib().symnmf_fit_params_default(C.byref(p))
    for key, val in kw.items():
        if key == "solver" and isinstance(val, str):
            val = _SOLVERS[val]
        setattr(p, key, val)
    return p


def fit(S: torch.Tensor, k: int, *, H0: torch.Tensor | None = None, G: torch.Tensor | None = None,
        solver: str = "adagrad", seed: int = 0, lr: float = 0.1, eps: float = 1e-10,
        max_iters: int = 2000, rel_tol: float = 1e-5, block_rows: int = 0, grow: bool = True,
        stall_tol: float = 1e-4, gap_threshold: float = 5.0, eigvals=None,
        probe_block: int = 16, probe_max_iter: int = 40, probe_tol: float = 1e-6,
        check_every: int = 16, timing: bool = False, history: bool = False, upper_only: bool = False,
        stream_times: bool = False, out: torch.Tensor | None = None,
        ws: torch.Tensor | None = None):
    """Factorise S ~ H H^T with H >= 0.  Returns (H, stats dict).

    H0 given: INIT_USER from a copy of H0 (or in place when ``out is H0``);
    otherwise the scale-matched seeded init.  G (n x k float32) is the AdaGrad
    accumulator, read and updated in place.  With ``history`` the per-
    evaluation losses are returned in stats["history"]; with ``stream_times``
    (implies ``timing``) the CUDA-event time of every S-stream launch, in
    order, in stats["stream_ms_each"].  stats["stream_kernel"] names the
    S-stream that ran the full-batch passes (``_lib.STREAM_KERNEL_NAMES``):
    the fp16 stream for the AdaGrad solver from n = 20,000 (k <= 24; the
    environment variable SYMNMF_H16_MIN_N moves the threshold, 0 turns it
    off), the TF32 stream otherwise.
    """
    n, _, lds = _matrix(S, "S")
    if H0 is not None:
        _dense(H0, "H0")
        H = H0 if out is H0 else H0.clone()
    else:
        H = torch.empty((n, k), dtype=torch.float32, device=S.device) if out is None else out
    _dense(H, "H")
    if tuple(H.shape) != (n, k):
        raise ValueError("H must be n x k")
    p = fit_params(solver=solver, init=L.INIT_USER if H0 is not None else L.INIT_SEEDED,
                   seed=int(seed) & (2**64 - 1), lr=lr, eps=eps, max_iters=max_iters,
                   rel_tol=rel_tol, block_rows=block_rows, grow=int(grow), stall_tol=stall_tol,
                   gap_threshold=gap_threshold, probe_block=probe_block,
                   probe_max_iter=probe_max_iter, probe_tol=probe_tol, check_every=check_every,
                   timing=int(timing or stream_times), upper_only=int(upper_only))
    if G is not None:
        _dense(G, "G")
        p.G_inout = G.data_ptr()
    hist = None
    if history:
        hist = (C.c_double * (max_iters + 1))()
        p.loss_history = C.cast(hist, C.POINTER(C.c_double))
        p.loss_history_len = max_iters + 1
    times = None
    if stream_times:
        times = (C.c_double * (max_iters + 8))()
        p.stream_ms_out = C.cast(times, C.POINTER(C.c_double))
        p.stream_ms_len = max_iters + 8
    ev = None
    if eigvals is not None:
        ev = (C.c_double * len(eigvals))(*[float(x) for x in eigvals])
        p.eigvals = C.cast(ev, C.POINTER(C.c_double))
        p.n_eigvals = len(eigvals)
    ws = workspace(L.OP_FIT, n, k, params=p, device=S.device) if ws is None else ws
    st = FitStats()
    L.check("symnmf_fit", _lib().symnmf_fit(S.data_ptr(), n, lds, k, C.byref(p), H.data_ptr(),
                                            C.byref(st), ws.data_ptr(), ws.numel(),
                                            _stream(S.device)))
    d = st.as_dict()
    if hist is not None:
        d["history"] = np.array(hist[:st.evaluations], dtype=np.float64)
    if times is not None:
        d["stream_ms_each"] = [float(x) for x in times[:min(st.stream_launches, max_iters + 8)]]
    return H, d


def labels(H: torch.Tensor) -> torch.Tensor:
    """Hard labels: row-wise argmax of H (lowest index on ties), int32."""
    _dense(H, "H")
    n, k = H.shape
    out = torch.empty(n, dtype=torch.int32, device=H.device)
    L.check("symnmf_labels", _lib().symnmf_labels(H.data_ptr(), n, k, out.data_ptr(),
                                                  _stream(H.device)))
    return out


def spherical_kmeans(S: torch.Tensor, k: int, *, seed: int = 0, max_iters: int = 100,
                     ws: torch.Tensor | None = None):
    """Spherical k-means on the L2-normalised rows of S (cosine similarity).

    Returns (labels int32 [n], centroids fp32 [n, k] with centroid c in column
    c, assignment steps, converged).  Two passes over S per step.
    """
    n, _, lds = _matrix(S, "S")
    labels_out = torch.empty(n, dtype=torch.int32, device=S.device)
    cent = torch.empty((n, k), dtype=torch.float32, device=S.device)
    ws = workspace(L.OP_SPHERICAL_KMEANS, n, k, device=S.device) if ws is None else ws
    steps, conv = C.c_int(0), C.c_int(0)
    L.check("symnmf_spherical_kmeans",
            _lib().symnmf_spherical_kmeans(S.data_ptr(), n, lds, k, seed, max_iters,
                                           labels_out.data_ptr(), cent.data_ptr(), C.byref(steps),
                                           C.byref(conv), ws.data_ptr(), ws.numel(),
                                           _stream(S.device)))
    return labels_out, cent, steps.value, bool(conv.value)


def ari(a: torch.Tensor, b: torch.Tensor, k: int, ws: torch.Tensor | None = None):
    """Adjusted Rand index of two int32 labelings in [0, k) (device tensors).

    Returns (ari, contingency table as a k x k int64 numpy array)."""
    _check_cuda(a, "a", torch.int32)
    _check_cuda(b, "b", torch.int32)
    if a.numel() != b.numel():
        raise ValueError("a and b must have the same length")
    ws = workspace(L.OP_ARI, a.numel(), k, device=a.device) if ws is None else ws
    out = C.c_double(0.0)
    table = np.zeros((k, k), dtype=np.int64)
    L.check("symnmf_ari", _lib().symnmf_ari(a.data_ptr(), b.data_ptr(), a.numel(), k, C.byref(out),
                                            table.ctypes.data_as(C.POINTER(C.c_int64)),
                                            ws.data_ptr(), ws.numel(), _stream(a.device)))
    return out.value, table


def rolling_params(**kw) -> "L.RollingParams":
    """Rolling-study parameters: the library defaults overridden by ``kw``;
    ``fit`` may be a dict of fit-parameter overrides."""
    p = L.RollingParams()
    _lib().symnmf_rolling_params_default(C.byref(p))
    fit_kw = kw.pop("fit", {})
    stressed = kw.pop("stressed", None)
    for key, v in kw.items():
        if not hasattr(p, key):
            raise TypeError(f"unknown rolling parameter {key!r}")
        setattr(p, key, v)
    if stressed is not None:
        stressed = [int(g) for g in stressed]
        if len(stressed) > 8:
            raise ValueError("at most 8 stressed groups")
        p.n_stressed = len(stressed)
        for i, g in enumerate(stressed):
            p.stressed[i] = g
    for key, v in fit_kw.items():
        if not hasattr(p.fit, key):
            raise TypeError(f"unknown fit parameter {key!r}")
        setattr(p.fit, key, v)
    return p


def rolling(R: torch.Tensor, *, groups: torch.Tensor | None = None, S: torch.Tensor | None = None,
            ws: torch.Tensor | None = None, **kw) -> dict:
    """The rolling-window study over a device-resident returns stream R (days x n).

    Keyword arguments are ``symnmf_rolling_params`` fields (window, stride,
    n_windows, k, kinds, tail_frac, tail_sign, delta, calib_begin, calib_end,
    stressed=[group ids], fit={...}).  Returns per kind ("corr", "tpdm") the
    labels (device, n_windows x n), ari_prev, ari_delta, cross, loss, flags
    (numpy), mean, std, limit, build_ms, fit_ms, plus total_ms and launches.
    """
    days, n, ldr = _matrix(R, "R")
    p = rolling_params(**kw)
    # output buffers; the library itself rejects windows that do not fit
    W = max(1, p.n_windows if p.n_windows > 0 else (days - p.window) // max(p.stride, 1) + 1)
    S = alloc_S(n, device=R.device) if S is None else S
    _, _, lds = _matrix(S, "S")
    if groups is not None:
        _check_cuda(groups, "groups", torch.int32)
    size = C.c_size_t(0)
    L.check("symnmf_workspace_size",
            _lib().symnmf_workspace_size(L.OP_ROLLING, n, p.k, p.window, C.byref(p.fit), C.byref(size)))
    if ws is None:
        ws = torch.empty(max(int(size.value), 256), dtype=torch.uint8, device=R.device)
    out = L.RollingOut()
    kinds = [("corr", L.KIND_CORR), ("tpdm", L.KIND_TPDM)]
    res = {}
    for c, (name, bit) in enumerate(kinds):
        if not p.kinds & bit:
            continue
        r = dict(labels=torch.empty((W, n), dtype=torch.int32, device=R.device),
                 ari_prev=np.zeros(W), ari_delta=np.zeros(W), cross=np.zeros(W), loss=np.zeros(W),
                 flags=np.zeros(W, dtype=np.uint8))
        out.labels[c] = r["labels"].data_ptr()
        out.ari_prev[c] = r["ari_prev"].ctypes.data_as(C.POINTER(C.c_double))
        out.ari_delta[c] = r["ari_delta"].ctypes.data_as(C.POINTER(C.c_double))
        out.cross[c] = r["cross"].ctypes.data_as(C.POINTER(C.c_double))
        out.loss[c] = r["loss"].ctypes.data_as(C.POINTER(C.c_double))
        out.flag[c] = r["flags"].ctypes.data_as(C.POINTER(C.c_uint8))
        res[name] = r
    L.check("symnmf_rolling",
            _lib().symnmf_rolling(R.data_ptr(), days, n, ldr,
                                  groups.data_ptr() if groups is not None else None,
                                  S.data_ptr(), lds, C.byref(p), C.byref(out), ws.data_ptr(),
                                  ws.numel(), _stream(R.device)))
    for c, (name, bit) in enumerate(kinds):
        if name in res:
            r = res[name]
            r["flags"] = r["flags"].astype(bool)
            r.update(mean=out.mean[c], std=out.std[c], limit=out.limit[c],
                     build_ms=out.build_ms[c], fit_ms=out.fit_ms[c])
    res["total_ms"] = out.total_ms
    res["launches"] = out.kernel_launches
    res["n_windows"] = out.n_windows
    return res

