"""B200-native SymNMF clustering: dependence matrices, spectral probe,
AdaGrad / Block-SVRG factorisation and argmax labels behind a C ABI
(include/symnmf.h, libsymnmf.so) with a thin PyTorch binding."""
from . import _lib
from .api import (alloc_S, ari, build_corr, build_tpdm, fit, fit_params, labels,  # noqa: F401
                  probe_last_info, rolling, rolling_params, sh, sh_upper, spectral_probe, spherical_kmeans,
                  stats, workspace)

__version__ = "0.1.0"
