"""IVF index on the soft-assignment output ("Flash-GMM: A Memory-Efficient Kernel for
Scalable Soft Clustering", §4): posting lists with multi-assignment and nprobe search,
through fgmm_ivf_build / fgmm_ivf_search (include/fgmm.h).  CUDA tensors only;
argument marshalling only."""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import LIB, check
from .gmm import _ptr, _stream


class IVFIndex:
    """Posting lists of K clusters over the vectors X (kept by reference)."""

    def __init__(self, K: int, ids: torch.Tensor, X: torch.Tensor):
        if not (ids.is_cuda and ids.dtype == torch.int32 and ids.dim() == 2 and ids.is_contiguous()):
            raise ValueError("ids must be a contiguous [N, top_m] int32 CUDA tensor")
        if not (X.is_cuda and X.dtype == torch.float32 and X.dim() == 2 and X.stride(1) == 1
                and X.shape[0] == ids.shape[0]):
            raise ValueError("X must be a [N, D] float32 CUDA tensor with contiguous rows")
        N, m = ids.shape
        self.K, self.X = K, X
        self.offsets = torch.empty(K + 1, dtype=torch.int64, device=ids.device)
        self.entries = torch.empty(max(1, N * m), dtype=torch.int64, device=ids.device)
        n = torch.zeros(1, dtype=torch.int64, device=ids.device)
        scratch = torch.empty(int(LIB.fgmm_ivf_build_scratch_bytes(N, K)), dtype=torch.uint8,
                              device=ids.device)
        check(LIB.fgmm_ivf_build(K, _ptr(ids), N, m, _ptr(self.offsets), _ptr(self.entries),
                                 _ptr(n), _ptr(scratch), _stream()), "fgmm_ivf_build")
        self.n_entries = n

    def search(self, centroids: torch.Tensor, Q: torch.Tensor, nprobe: int, k: int):
        """Returns (ids int64 [nq, k], squared distances float32 [nq, k], DCO int64 [nq])."""
        if not (Q.is_cuda and Q.dtype == torch.float32 and Q.dim() == 2 and Q.stride(1) == 1):
            raise ValueError("Q must be a [nq, D] float32 CUDA tensor with contiguous rows")
        C = centroids.contiguous()
        nq, D = Q.shape
        out_i = torch.empty(nq, k, dtype=torch.int64, device=Q.device)
        out_d = torch.empty(nq, k, dtype=torch.float32, device=Q.device)
        dco = torch.empty(nq, dtype=torch.int64, device=Q.device)
        check(LIB.fgmm_ivf_search(self.K, D, _ptr(C), _ptr(self.offsets), _ptr(self.entries),
                                  _ptr(self.X), self.X.stride(0), _ptr(Q), nq, Q.stride(0),
                                  nprobe, k, _ptr(out_i), _ptr(out_d), _ptr(dco), _stream()),
              "fgmm_ivf_search")
        return out_i, out_d, dco
