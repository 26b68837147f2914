"""Host-side checks of the C-ABI library: it loads, exports every symbol that
include/fgmm.h declares, and rejects bad arguments before touching a device.
No kernel is launched here (these run on a CPU-only host)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADERS = [os.path.join(ROOT, "include", f) for f in os.listdir(os.path.join(ROOT, "include"))
           if f.endswith(".h")]


def declared_symbols():
    names = set()
    for h in HEADERS:
        txt = open(h).read()
        txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?\w+\s*\**\s*(fgmm_\w+)\s*\(", txt, re.M):
            names.add(m.group(1))
    return names


def test_header_declares_the_api():
    names = declared_symbols()
    for n in ["fgmm_create", "fgmm_destroy", "fgmm_em_step", "fgmm_fit", "fgmm_soft_assign",
              "fgmm_get_status", "fgmm_status_string", "fgmm_set_precision"]:
        assert n in names


def test_library_exports_every_declared_symbol():
    from ivf_quantizer_b200 import _lib
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in declared_symbols():
        assert hasattr(lib, n), n
    assert set(_lib.SIGNATURES) >= declared_symbols()


def test_status_strings():
    from ivf_quantizer_b200._lib import LIB
    for code in range(7):
        s = LIB.fgmm_status_string(code).decode()
        assert s and s != "unknown status"
    assert LIB.fgmm_status_string(99).decode() == "unknown status"


def test_create_rejects_bad_arguments_without_a_device():
    from ivf_quantizer_b200 import _lib
    LIB = _lib.LIB
    h = ctypes.c_void_p()
    assert LIB.fgmm_create(0, 4, 0, 1e-6, ctypes.byref(h)) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_create(4, 0, 0, 1e-6, ctypes.byref(h)) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_create(4, 4, 7, 1e-6, ctypes.byref(h)) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_create(4, 4, 0, -1.0, ctypes.byref(h)) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_create(4, 4, 0, float("nan"), ctypes.byref(h)) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_create(4, 4, 0, 1e-6, None) == _lib.ERR_INVALID_ARG
    assert not h.value


def test_calls_on_null_handle_are_invalid():
    from ivf_quantizer_b200 import _lib
    LIB = _lib.LIB
    z = ctypes.c_void_p(0)
    one = ctypes.c_void_p(16)
    assert LIB.fgmm_em_step(z, one, 0, 10, 4, one, one, one, z, z, z) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_soft_assign(z, one, 0, 10, 4, one, one, one, 1, 0.0, one, z, z) == \
        _lib.ERR_INVALID_ARG
    assert LIB.fgmm_set_precision(z, 0) == _lib.ERR_INVALID_ARG
    assert LIB.fgmm_set_block_skip(z, 1) == _lib.ERR_INVALID_ARG
    v = ctypes.c_int(7)
    assert LIB.fgmm_get_block_skip(z, ctypes.byref(v)) == _lib.ERR_INVALID_ARG
    assert v.value == 7
    assert LIB.fgmm_get_status(z, z) == _lib.ERR_INVALID_ARG
    # X from a file or a reader: a null handle, path or reader is an argument error
    assert LIB.fgmm_em_step_file(z, b"/nonexistent", 0, 0, 10, one, one, one, z, z, z) == \
        _lib.ERR_INVALID_ARG
    assert LIB.fgmm_em_partial_file(z, b"/nonexistent", 0, 0, 10, one, one, one, one, z, z) == \
        _lib.ERR_INVALID_ARG
    assert LIB.fgmm_em_step_reader(z, one, z, 0, 10, one, one, one, z, z, z) == \
        _lib.ERR_INVALID_ARG
    assert LIB.fgmm_em_partial_reader(z, one, z, 0, 10, one, one, one, one, z, z) == \
        _lib.ERR_INVALID_ARG
    assert LIB.fgmm_status_string(_lib.ERR_IO) == b"reading X failed"
    assert LIB.fgmm_destroy(z) == _lib.OK


def test_package_has_no_fallback(monkeypatch, tmp_path):
    """The loader raises when the library file is missing: no silent CPU path."""
    from ivf_quantizer_b200 import _lib
    with pytest.raises(ImportError):
        _lib.load(str(tmp_path / "missing.so"))


def test_profile_layout_and_kernel_names():
    """The ctypes mirror of fgmm_profile matches the header's array length, and every
    per-kernel slot has a distinct name; indices outside the table give NULL."""
    import re
    from ivf_quantizer_b200 import _lib
    hdr = open(os.path.join(ROOT, "include", "fgmm.h")).read()
    assert int(re.search(r"#define FGMM_PROF_KERNELS (\d+)", hdr).group(1)) == _lib.PROF_KERNELS
    assert re.search(r"#define FGMM_CHUNK_POINTS \(1 << (\d+)\)", hdr).group(1) == "20"
    assert _lib.CHUNK_POINTS == 1 << 20
    names = [_lib.LIB.fgmm_profile_kernel_name(i) for i in range(_lib.PROF_KERNELS)]
    assert all(n for n in names) and len(set(names)) == len(names)
    assert b"tc_lse" in names and b"tc_stats" in names and b"stats_simt" in names
    assert _lib.LIB.fgmm_profile_kernel_name(-1) is None
    assert _lib.LIB.fgmm_profile_kernel_name(_lib.PROF_KERNELS) is None


def test_step_info_rejects_null_arguments():
    from ivf_quantizer_b200 import _lib
    info = _lib.StepInfo()
    assert _lib.LIB.fgmm_last_step_info(None, ctypes.byref(info)) == _lib.ERR_INVALID_ARG
    assert _lib.LIB.fgmm_last_step_info(None, None) == _lib.ERR_INVALID_ARG
