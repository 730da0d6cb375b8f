"""The C ABI on the CPU: the library loads, exports every declared symbol, and
the ctypes layouts match the C compiler's; argument validation answers
without touching a device."""
import ctypes as C
import os
import re
import subprocess
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "symnmf.h")


@pytest.fixture(scope="module")
def lib():
    from symmetric_nmf_clustering_b200 import build
    build.build()
    from symmetric_nmf_clustering_b200 import _lib
    return _lib.load()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"SYMNMF_API\s+[\w\s\*]+?\b(symnmf_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 12
    out = subprocess.run(["nm", "-D", "--defined-only", lib._name], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (symnmf_\w+)", out))
    assert set(names) <= exported, set(names) - exported
    from symmetric_nmf_clustering_b200 import _lib
    assert set(names) == set(_lib.SIGNATURES)


def test_struct_layout_matches_c(lib):
    from symmetric_nmf_clustering_b200 import _lib
    probes = []
    structs = (("symnmf_fit_params", _lib.FitParams), ("symnmf_fit_stats", _lib.FitStats),
               ("symnmf_probe_info", _lib.ProbeInfo))
    for cname, py in structs:
        probes.append(f'printf("{cname} %zu\\n", sizeof({cname}));')
        for f, _ in py._fields_:
            probes.append(f'printf("{cname}.{f} %zu\\n", offsetof({cname}, {f}));')
    src = "#include <stdio.h>\n#include <stddef.h>\n#include \"symnmf.h\"\nint main(void){\n" + \
          "\n".join(probes) + "\nreturn 0;}\n"
    with tempfile.TemporaryDirectory() as d:
        c = os.path.join(d, "p.c")
        exe = os.path.join(d, "p")
        open(c, "w").write(src)
        subprocess.run(["gcc", "-std=c11", "-I", os.path.dirname(HEADER), c, "-o", exe], check=True)
        lines = subprocess.run([exe], capture_output=True, text=True, check=True).stdout.split("\n")
    want = dict(l.split() for l in lines if l.strip())
    for cname, py in structs:
        assert int(want[cname]) == C.sizeof(py)
        for f, _ in py._fields_:
            assert int(want[f"{cname}.{f}"]) == getattr(py, f).offset, f


def test_defaults_and_strings(lib):
    from symmetric_nmf_clustering_b200 import _lib
    p = _lib.FitParams()
    lib.symnmf_fit_params_default(C.byref(p))
    assert (p.solver, p.init, p.seed) == (0, 0, 0)
    assert p.lr == pytest.approx(0.1) and p.eps == pytest.approx(1e-10)
    assert p.max_iters == 2000 and p.rel_tol == 1e-5 and p.grow == 1
    assert p.stall_tol == 1e-4 and p.gap_threshold == 5.0 and p.check_every == 16
    assert lib.symnmf_status_string(0) == b"ok"
    assert lib.symnmf_status_string(3) == b"workspace too small"
    assert lib.symnmf_version() >= 100


def test_workspace_sizes_without_device(lib):
    from symmetric_nmf_clustering_b200 import _lib
    size = C.c_size_t()
    p = _lib.FitParams()
    lib.symnmf_fit_params_default(C.byref(p))
    assert lib.symnmf_workspace_size(_lib.OP_FIT, 100000, 24, 0, C.byref(p), C.byref(size)) == 0
    n, k = 100000, 24
    assert size.value > 3 * n * k * 4            # second H buffer and two accumulators
    assert size.value < 200 * n * k * 4           # no n x n scratch
    assert lib.symnmf_workspace_size(_lib.OP_BUILD_CORR, 1000, 0, 250, None, C.byref(size)) == 0
    assert size.value >= 256 * 1024 * 4           # normalised window
    assert lib.symnmf_workspace_size(_lib.OP_FIT, 10, 65, 0, C.byref(p), C.byref(size)) == 1
    assert b"k = 65" in lib.symnmf_last_error()
    assert lib.symnmf_workspace_size(99, 10, 1, 0, None, C.byref(size)) == 1


def test_argument_validation_before_any_device_work(lib):
    from symmetric_nmf_clustering_b200 import _lib
    p = _lib.FitParams()
    lib.symnmf_fit_params_default(C.byref(p))
    fake = 1 << 20  # 16-byte aligned, never dereferenced: validation fails first
    # lds not a multiple of 4
    assert lib.symnmf_fit(fake, 10, 10, 3, C.byref(p), fake, None, fake, 0, None) == 1
    assert b"lds" in lib.symnmf_last_error()
    # k out of range
    assert lib.symnmf_fit(fake, 12, 12, 0, C.byref(p), fake, None, fake, 0, None) == 1
    # misaligned S
    assert lib.symnmf_sh(fake + 4, 12, 12, fake, 3, fake, fake, 0, None) == 1
    # bad tail parameters
    assert lib.symnmf_build_tpdm(fake, 20, 8, 8, 0.0, 1, fake, 8, fake, 0, None) == 1
    assert lib.symnmf_build_tpdm(fake, 20, 8, 8, 0.05, 2, fake, 8, fake, 0, None) == 1
    # T < 2 for correlation
    assert lib.symnmf_build_corr(fake, 1, 8, 8, fake, 8, fake, 0, None) == 1
    # upper_only: 0 or 1, and k <= 24 with the upper-triangle stream
    p.upper_only = 2
    assert lib.symnmf_fit(fake, 12, 12, 3, C.byref(p), fake, None, fake, 0, None) == 1
    assert b"upper_only" in lib.symnmf_last_error()
    p.upper_only = 1
    assert lib.symnmf_fit(fake, 40, 40, 25, C.byref(p), fake, None, fake, 0, None) == 1
    assert b"upper_only" in lib.symnmf_last_error()
    assert lib.symnmf_sh_upper(fake, 40, 40, fake, 25, fake, fake, 0, None) == 1
    assert lib.symnmf_sh_upper(fake + 4, 40, 40, fake, 8, fake, fake, 0, None) == 1


def test_python_binding_fails_loudly_without_library(tmp_path):
    from symmetric_nmf_clustering_b200 import _lib
    with pytest.raises(ImportError, match="no CPU fallback"):
        _lib.load(str(tmp_path / "missing.so"))
