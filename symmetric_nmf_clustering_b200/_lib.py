"""ctypes declarations of libsymnmf.so (include/symnmf.h).

Loading fails loudly: there is no fallback implementation anywhere in this
package.  Build the library with ``python -m symmetric_nmf_clustering_b200.build``.
"""
from __future__ import annotations

import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsymnmf.so")

SYMNMF_OK = 0
SYMNMF_ERR_INVALID_ARG = 1
SYMNMF_ERR_NONFINITE = 2
SYMNMF_ERR_WORKSPACE = 3
SYMNMF_ERR_CUDA = 4
SYMNMF_ERR_TIMEOUT = 5
SYMNMF_ERR_NOT_SUPPORTED = 6

SOLVER_ADAGRAD, SOLVER_BLOCK_SVRG, SOLVER_AUTO = 0, 1, 2
INIT_SEEDED, INIT_USER = 0, 1
(OP_BUILD_CORR, OP_BUILD_TPDM, OP_SPECTRAL_PROBE, OP_FIT, OP_SH, OP_STATS,
 OP_SPHERICAL_KMEANS, OP_ARI, OP_ROLLING, OP_SH_UPPER) = range(10)
KIND_CORR, KIND_TPDM = 1, 2


class FitParams(C.Structure):
    _fields_ = [
        ("solver", C.c_int),
        ("init", C.c_int),
        ("seed", C.c_uint64),
        ("lr", C.c_float),
        ("eps", C.c_float),
        ("max_iters", C.c_int),
        ("rel_tol", C.c_double),
        ("block_rows", C.c_int64),
        ("grow", C.c_int),
        ("stall_tol", C.c_double),
        ("gap_threshold", C.c_double),
        ("upper_only", C.c_int),
        ("G_inout", C.c_void_p),
        ("loss_history", C.POINTER(C.c_double)),
        ("loss_history_len", C.c_int),
        ("eigvals", C.POINTER(C.c_double)),
        ("n_eigvals", C.c_int),
        ("probe_block", C.c_int),
        ("probe_max_iter", C.c_int),
        ("probe_tol", C.c_double),
        ("check_every", C.c_int),
        ("timing", C.c_int),
        ("stream_ms_out", C.POINTER(C.c_double)),
        ("stream_ms_len", C.c_int),
    ]


# symnmf_fit_stats.stream_kernel
STREAM_TF32, STREAM_FP16, STREAM_UPPER, STREAM_CUDA_CORE = range(4)
STREAM_KERNEL_NAMES = {STREAM_TF32: "stream_tc_kernel", STREAM_FP16: "stream_h16_kernel",
                       STREAM_UPPER: "stream_tri_kernel", STREAM_CUDA_CORE: "stream_partial_kernel"}


class FitStats(C.Structure):
    _fields_ = [
        ("iters", C.c_int),
        ("epochs", C.c_int),
        ("converged", C.c_int),
        ("solver_used", C.c_int),
        ("block_final", C.c_int64),
        ("loss", C.c_double),
        ("rel_change", C.c_double),
        ("gamma", C.c_double),
        ("s_mean", C.c_double),
        ("s_sqnorm", C.c_double),
        ("evaluations", C.c_int),
        ("stream_launches", C.c_int),
        ("stream_ms", C.c_double),
        ("loop_ms", C.c_double),
        ("kernel_launches", C.c_int),
        ("stream_kernel", C.c_int),
    ]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


class RollingParams(C.Structure):
    _fields_ = [
        ("window", C.c_int64),
        ("stride", C.c_int64),
        ("n_windows", C.c_int64),
        ("k", C.c_int),
        ("kinds", C.c_int),
        ("tail_frac", C.c_double),
        ("tail_sign", C.c_int),
        ("delta", C.c_int),
        ("calib_begin", C.c_int64),
        ("calib_end", C.c_int64),
        ("n_stressed", C.c_int),
        ("stressed", C.c_int * 8),
        ("warm_start", C.c_int),
        ("fit", FitParams),
    ]


_P2 = lambda t: C.POINTER(t) * 2   # noqa: E731


class RollingOut(C.Structure):
    _fields_ = [
        ("labels", C.c_void_p * 2),
        ("ari_prev", _P2(C.c_double)),
        ("ari_delta", _P2(C.c_double)),
        ("cross", _P2(C.c_double)),
        ("loss", _P2(C.c_double)),
        ("flag", _P2(C.c_uint8)),
        ("mean", C.c_double * 2),
        ("std", C.c_double * 2),
        ("limit", C.c_double * 2),
        ("n_windows", C.c_int64),
        ("build_ms", C.c_double * 2),
        ("fit_ms", C.c_double * 2),
        ("total_ms", C.c_double),
        ("kernel_launches", C.c_int),
    ]


class ProbeInfo(C.Structure):
    _fields_ = [("s_passes", C.c_int), ("block_steps", C.c_int), ("kernel_launches", C.c_int)]


_vp, _i64, _int, _sz = C.c_void_p, C.c_int64, C.c_int, C.c_size_t

# name -> (restype, argtypes); every symbol include/symnmf.h declares
SIGNATURES = {
    "symnmf_fit_params_default": (None, [C.POINTER(FitParams)]),
    "symnmf_status_string": (C.c_char_p, [_int]),
    "symnmf_last_error": (C.c_char_p, []),
    "symnmf_version": (_int, []),
    "symnmf_workspace_size": (_int, [_int, _i64, _int, _i64, C.POINTER(FitParams), C.POINTER(_sz)]),
    "symnmf_build_corr": (_int, [_vp, _i64, _i64, _i64, _vp, _i64, _vp, _sz, _vp]),
    "symnmf_build_tpdm": (_int, [_vp, _i64, _i64, _i64, C.c_double, _int, _vp, _i64, _vp, _sz, _vp]),
    "symnmf_stats": (_int, [_vp, _i64, _i64, _vp, _vp, _sz, _vp]),
    "symnmf_sh": (_int, [_vp, _i64, _i64, _vp, _int, _vp, _vp, _sz, _vp]),
    "symnmf_sh_upper": (_int, [_vp, _i64, _i64, _vp, _int, _vp, _vp, _sz, _vp]),
    "symnmf_spectral_probe": (_int, [_vp, _i64, _i64, _int, _int, _int, C.c_double, C.c_uint64,
                                     C.POINTER(C.c_double), _vp, _sz, _vp]),
    "symnmf_probe_last_info": (_int, [C.POINTER(ProbeInfo)]),
    "symnmf_stats_rows": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _sz, _vp]),
    "symnmf_seeded_init": (_int, [_vp, _i64, _int, C.c_uint64, C.c_double, _vp]),
    "symnmf_gram": (_int, [_vp, _i64, _int, _vp, _vp, _sz, _vp]),
    "symnmf_shard_workspace_size": (_int, [_i64, _i64, _int, C.POINTER(_sz)]),
    "symnmf_shard_step": (_int, [_vp, _i64, _i64, _i64, _i64, _int, _vp, _vp, _vp, C.c_float,
                                 C.c_float, _vp, _vp, _vp, _vp, _sz, _vp]),
    "symnmf_fit": (_int, [_vp, _i64, _i64, _int, C.POINTER(FitParams), _vp, C.POINTER(FitStats),
                          _vp, _sz, _vp]),
    "symnmf_labels": (_int, [_vp, _i64, _int, _vp, _vp]),
    "symnmf_sh_noalloc": (_int, [_vp, _i64, _i64, _vp, _int, _vp, _vp]),
    "symnmf_spherical_kmeans": (_int, [_vp, _i64, _i64, _int, C.c_uint64, _int, _vp, _vp,
                                       C.POINTER(_int), C.POINTER(_int), _vp, _sz, _vp]),
    "symnmf_ari": (_int, [_vp, _vp, _i64, _int, C.POINTER(C.c_double), C.POINTER(C.c_int64), _vp,
                          _sz, _vp]),
    "symnmf_rolling_params_default": (None, [C.POINTER(RollingParams)]),
    "symnmf_test_stall_pipeline": (_int, [_int]),
    "symnmf_test_split16": (_int, [_vp, _i64, C.c_float, _vp, _vp, _vp]),
    "symnmf_rolling": (_int, [_vp, _i64, _i64, _i64, _vp, _vp, _i64, C.POINTER(RollingParams),
                              C.POINTER(RollingOut), _vp, _sz, _vp]),
}

_lib = None


def _open(path: str) -> C.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m symmetric_nmf_clustering_b200.build` "
            "(the SymNMF path has no CPU fallback)")
    lib = C.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


def load(path: str = LIB_PATH) -> C.CDLL:
    """Load libsymnmf.so and declare its signatures (raises if it is missing)."""
    global _lib
    if path != LIB_PATH:
        return _open(path)
    if _lib is None:
        _lib = _open(path)
    return _lib


class SymNMFError(RuntimeError):
    def __init__(self, fn: str, status: int, detail: str):
        self.status = status
        super().__init__(f"{fn} failed with status {status}: {detail}")


def check(fn: str, status: int):
    if status != SYMNMF_OK:
        lib = load()
        detail = (lib.symnmf_last_error() or b"").decode() or lib.symnmf_status_string(status).decode()
        raise SymNMFError(fn, status, detail)
