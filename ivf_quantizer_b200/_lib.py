"""ctypes loader for the in-tree CUDA library ``_fgmm.so`` (C-ABI of include/fgmm.h).

There is no fallback: if the library is missing or fails to load, importing
this module raises, so that nothing silently runs elsewhere.
"""
from __future__ import annotations

import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "_fgmm.so")

# enum values mirrored from include/fgmm.h
COV_DIAG, COV_SPHERICAL = 0, 1
PREC_FP32, PREC_FP16X3, PREC_FP16, PREC_AUTO = 0, 1, 2, 3
F32, BF16 = 0, 1
# fgmm_read_fn: (ctx, row0, nrows, dst) -> 0 on success
READ_FN = ctypes.CFUNCTYPE(ctypes.c_int, ctypes.c_void_p, ctypes.c_int64, ctypes.c_int64,
                           ctypes.c_void_p)
OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_OOM, ERR_NUMERIC, ERR_TIMEOUT, ERR_IO = range(8)
MAX_TOP_M = 16
IVF_MAX_TOPK = 32
STATIC_MAX_KD = 1 << 18
STATIC_MAX_K = 1 << 14
EMPTY_NK = 1e-6
CHUNK_POINTS = 1 << 20

PROF_KERNELS = 25


class Profile(ctypes.Structure):
    _fields_ = [("launches", ctypes.c_int64), ("sweep1_launches", ctypes.c_int64),
                ("sweep1_ms", ctypes.c_double), ("sweep2_launches", ctypes.c_int64),
                ("sweep2_ms", ctypes.c_double), ("other_launches", ctypes.c_int64),
                ("other_ms", ctypes.c_double),
                ("kernel_launches", ctypes.c_int64 * PROF_KERNELS),
                ("kernel_ms", ctypes.c_double * PROF_KERNELS),
                ("kernel_active", ctypes.c_int64 * PROF_KERNELS),
                ("kernel_active_ms", ctypes.c_double * PROF_KERNELS)]


class StepInfo(ctypes.Structure):
    _fields_ = [("path", ctypes.c_int), ("n_stiff", ctypes.c_int), ("n_grey", ctypes.c_int),
                ("skip_pairs", ctypes.c_int64), ("skip_pairs_all", ctypes.c_int64)]


# every exported symbol of include/fgmm.h with (restype, argtypes)
_c = ctypes
_vp, _i64, _int, _dbl, _flt = _c.c_void_p, _c.c_int64, _c.c_int, _c.c_double, _c.c_float
SIGNATURES = {
    "fgmm_create": (_int, [_int, _int, _int, _dbl, _c.POINTER(_vp)]),
    "fgmm_destroy": (_int, [_vp]),
    "fgmm_set_precision": (_int, [_vp, _int]),
    "fgmm_get_precision": (_int, [_vp, _c.POINTER(_int)]),
    "fgmm_set_block_skip": (_int, [_vp, _int]),
    "fgmm_get_block_skip": (_int, [_vp, _c.POINTER(_int)]),
    "fgmm_workspace_bytes": (_int, [_vp, _c.POINTER(_c.c_size_t)]),
    "fgmm_last_step_path": (_int, [_vp, _c.POINTER(_int)]),
    "fgmm_last_step_info": (_int, [_vp, _c.POINTER(StepInfo)]),
    "fgmm_em_step": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_fit": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _int, _dbl,
                        _c.POINTER(_dbl), _c.POINTER(_int), _vp]),
    "fgmm_soft_assign": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _int, _flt,
                                _vp, _vp, _vp]),
    "fgmm_get_status": (_int, [_vp, _vp]),
    "fgmm_status_string": (_c.c_char_p, [_int]),
    "fgmm_profile_enable": (_int, [_vp, _int]),
    "fgmm_selftest_bounded_wait": (_int, [_int]),
    "fgmm_soft_assign_static": (_int, [_int, _int, _int, _vp, _int, _i64, _i64, _vp, _vp, _vp,
                                       _int, _flt, _vp, _vp, _vp]),
    "fgmm_profile_read": (_int, [_vp, _c.POINTER(Profile), _int]),
    "fgmm_profile_kernel_name": (_c.c_char_p, [_int]),
    "fgmm_em_partial": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_finish": (_int, [_vp, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_stats_sum": (_int, [_vp, _int, _i64, _vp, _vp]),
    "fgmm_score_samples": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_fisher_vector": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _int, _vp, _vp]),
    "fgmm_ivf_build_scratch_bytes": (_c.c_size_t, [_i64, _int]),
    "fgmm_ivf_build": (_int, [_int, _vp, _i64, _int, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_ivf_search": (_int, [_int, _int, _vp, _vp, _vp, _vp, _i64, _vp, _i64, _i64, _int, _int,
                               _vp, _vp, _vp, _vp]),
    "fgmm_kmeans_step": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_kmeans_seed": (_int, [_vp, _vp, _int, _i64, _i64, _i64, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_kmeans_seed_scratch_bytes": (_c.c_size_t, [_i64]),
    "fgmm_em_step_host": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_partial_host": (_int, [_vp, _vp, _int, _i64, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_step_reader": (_int, [_vp, _vp, _vp, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_partial_reader": (_int, [_vp, _vp, _vp, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_step_file": (_int, [_vp, _c.c_char_p, _i64, _int, _i64, _vp, _vp, _vp, _vp, _vp, _vp]),
    "fgmm_em_partial_file": (_int, [_vp, _c.c_char_p, _i64, _int, _i64, _vp, _vp, _vp, _vp, _vp,
                                    _vp]),
}


class FgmmError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {LIB.fgmm_status_string(code).decode()} (status {code})")


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run python ivf_quantizer_b200/build.py)")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


LIB = load()


def check(code: int, where: str) -> None:
    if code != OK:
        raise FgmmError(code, where)
