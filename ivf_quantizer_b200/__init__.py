"""Fused Gaussian-mixture EM on NVIDIA B200 (sm_100a).

Python binding of the C-ABI in ``include/fgmm.h`` ("Flash-GMM: A
Memory-Efficient Kernel for Scalable Soft Clustering": §2 EM, §3.1 fused
kernel, §4.2-4.3 assignment).  Argument marshalling only: every step of the
path runs in the CUDA library ``_fgmm.so``; PyTorch provides device memory and
streams.
"""
from ._lib import (BF16, CHUNK_POINTS, COV_DIAG, COV_SPHERICAL, EMPTY_NK, F32, MAX_TOP_M, PREC_AUTO,
                   PREC_FP16, PREC_FP16X3, PREC_FP32, FgmmError)
from .gmm import GMM, stats_sum

__all__ = ["GMM", "stats_sum", "CHUNK_POINTS", "FgmmError", "COV_DIAG", "COV_SPHERICAL", "PREC_FP32", "PREC_FP16X3",
           "PREC_FP16", "PREC_AUTO", "F32", "BF16", "MAX_TOP_M", "EMPTY_NK"]
