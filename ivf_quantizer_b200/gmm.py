"""``GMM``: a thin object over one fgmm handle (include/fgmm.h).

All tensors are CUDA tensors on the handle's device; the current torch stream
is the stream of every call.  Parameters are float32: weights [K], means [K, D],
variances [K, D] (diagonal) or [K] (isotropic), updated in place by ``step``
and ``fit``.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np
import torch

from . import _lib
from ._lib import LIB, check


def _stream() -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else ctypes.c_void_p(0)


def _x_args(X: torch.Tensor, allow_host: bool = False):
    if X.dim() != 2 or not (X.is_cuda or (allow_host and X.device.type == "cpu")):
        raise ValueError("X must be a 2-D CUDA tensor" + (" or CPU tensor" if allow_host else ""))
    if X.dtype == torch.float32:
        dt = _lib.F32
    elif X.dtype == torch.bfloat16:
        dt = _lib.BF16
    else:
        raise TypeError("X must be float32 or bfloat16")
    if X.stride(1) != 1:
        raise ValueError("X rows must be contiguous")
    return _ptr(X), dt, X.shape[0], X.stride(0)


class GMM:
    def __init__(self, K: int, D: int, cov_type: int = _lib.COV_DIAG, reg_covar: float = 1e-6,
                 precision: int | None = None):
        self.K, self.D, self.cov_type, self.reg_covar = K, D, cov_type, reg_covar
        h = ctypes.c_void_p()
        check(LIB.fgmm_create(K, D, cov_type, reg_covar, ctypes.byref(h)), "fgmm_create")
        self._h = h
        if precision is not None:
            self.set_precision(precision)

    # ---------------------------------------------------------------- lifecycle
    def close(self):
        if getattr(self, "_h", None):
            LIB.fgmm_destroy(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

    def __enter__(self):
        return self

    def __exit__(self, *a):
        self.close()

    # ---------------------------------------------------------------- settings
    def set_precision(self, prec: int):
        check(LIB.fgmm_set_precision(self._h, prec), "fgmm_set_precision")

    @property
    def precision(self) -> int:
        v = ctypes.c_int()
        check(LIB.fgmm_get_precision(self._h, ctypes.byref(v)), "fgmm_get_precision")
        return v.value

    def set_block_skip(self, enable: bool):
        """Skip (tile, block) pairs of the tensor-core statistics sweep whose
        responsibilities are all zero at fp16 resolution (fgmm_set_block_skip)."""
        check(LIB.fgmm_set_block_skip(self._h, 1 if enable else 0), "fgmm_set_block_skip")

    @property
    def block_skip(self) -> bool:
        v = ctypes.c_int()
        check(LIB.fgmm_get_block_skip(self._h, ctypes.byref(v)), "fgmm_get_block_skip")
        return bool(v.value)

    def last_step_path(self) -> int:
        """PREC_FP32 or PREC_FP16X3: the path the last step ran (synchronises under AUTO)."""
        v = ctypes.c_int()
        check(LIB.fgmm_last_step_path(self._h, ctypes.byref(v)), "fgmm_last_step_path")
        return v.value

    def last_step_info(self) -> dict:
        """What the last step did (fgmm_last_step_info; synchronises): path, stiff and
        grey component counts (AUTO), and the statistics sweep's visited and dense
        (tile, block) pair counts on the last chunk (-1 when it ran dense)."""
        v = _lib.StepInfo()
        check(LIB.fgmm_last_step_info(self._h, ctypes.byref(v)), "fgmm_last_step_info")
        return {f: getattr(v, f) for f, _ in _lib.StepInfo._fields_}

    @property
    def workspace_bytes(self) -> int:
        v = ctypes.c_size_t()
        check(LIB.fgmm_workspace_bytes(self._h, ctypes.byref(v)), "fgmm_workspace_bytes")
        return v.value

    # ---------------------------------------------------------------- parameters
    def new_params(self, weights, means, variances, device="cuda"):
        """Copy (weights, means, variances) into contiguous float32 CUDA tensors."""
        w = torch.as_tensor(weights, dtype=torch.float32).to(device).contiguous()
        m = torch.as_tensor(means, dtype=torch.float32).to(device).contiguous()
        v = torch.as_tensor(variances, dtype=torch.float32).to(device).contiguous()
        self._check_params(w, m, v)
        return w, m, v

    def _check_params(self, w, m, v):
        K, D = self.K, self.D
        want_v = (K,) if self.cov_type == _lib.COV_SPHERICAL else (K, D)
        for t in (w, m, v):
            if not (t.is_cuda and t.dtype == torch.float32 and t.is_contiguous()):
                raise ValueError("parameters must be contiguous float32 CUDA tensors")
        if tuple(w.shape) != (K,) or tuple(m.shape) != (K, D) or tuple(v.shape) != want_v:
            raise ValueError("parameter shapes do not match (K, D, cov_type)")

    # ---------------------------------------------------------------- EM
    def step(self, X, weights, means, variances, loglik=None, logz=None):
        """One fused EM iteration; updates the parameters in place.

        X: CUDA tensor, or CPU tensor (ideally pinned), which is streamed to the device
        chunk by chunk with the copies overlapping the sweeps (fgmm_em_step_host).
        loglik: optional CUDA float64 tensor [1] receiving log p(X | Θ_in).
        logz:   optional CUDA float32 tensor [N] receiving per-point log p(x_i | Θ_in).
        """
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X, allow_host=True)
        if loglik is not None and not (loglik.is_cuda and loglik.dtype == torch.float64):
            raise ValueError("loglik must be a CUDA float64 tensor")
        if logz is not None and not (logz.is_cuda and logz.dtype == torch.float32
                                     and logz.numel() >= n):
            raise ValueError("logz must be a CUDA float32 tensor with N elements")
        fn = LIB.fgmm_em_step if X.is_cuda else LIB.fgmm_em_step_host
        check(fn(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means), _ptr(variances),
                 _ptr(loglik), _ptr(logz), _stream()), "fgmm_em_step")

    def _stream_args(self, weights, means, variances, dtype, loglik=None, logz=None, n=0):
        self._check_params(weights, means, variances)
        if dtype not in (torch.float32, torch.bfloat16):
            raise ValueError("dtype must be torch.float32 or torch.bfloat16")
        if loglik is not None and not (loglik.is_cuda and loglik.dtype == torch.float64):
            raise ValueError("loglik must be a CUDA float64 tensor")
        if logz is not None and not (logz.is_cuda and logz.dtype == torch.float32
                                     and logz.numel() >= n):
            raise ValueError("logz must be a CUDA float32 tensor with N elements")
        return _lib.F32 if dtype == torch.float32 else _lib.BF16

    def step_file(self, path, N, weights, means, variances, dtype=torch.float32, offset=0,
                  loglik=None, logz=None):
        """One EM iteration with X read from a file (fgmm_em_step_file): N rows of D
        elements of `dtype`, row-major, from byte `offset`; chunks are read into pinned
        buffers while the previous chunk is processed.  Bit-identical to step() on the
        same rows."""
        dt = self._stream_args(weights, means, variances, dtype, loglik, logz, N)
        check(LIB.fgmm_em_step_file(self._h, os.fsencode(path), int(offset), dt, int(N),
                                    _ptr(weights), _ptr(means), _ptr(variances),
                                    _ptr(loglik), _ptr(logz), _stream()), "fgmm_em_step_file")

    def partial_file(self, path, N, weights, means, variances, dtype=torch.float32, offset=0,
                     stats=None, logz=None):
        """partial() with this shard's rows read from a file (fgmm_em_partial_file)."""
        dt = self._stream_args(weights, means, variances, dtype, None, logz, N)
        if stats is None:
            stats = torch.empty(self.stats_len, dtype=torch.float64, device=weights.device)
        check(LIB.fgmm_em_partial_file(self._h, os.fsencode(path), int(offset), dt, int(N),
                                       _ptr(weights), _ptr(means), _ptr(variances),
                                       _ptr(stats), _ptr(logz), _stream()),
              "fgmm_em_partial_file")
        return stats

    def step_reader(self, read, N, weights, means, variances, dtype=torch.float32,
                    loglik=None, logz=None):
        """One EM iteration with X produced by `read(row0, out)`, which fills the numpy
        array `out` (nrows x D of `dtype`, bf16 as uint16) with rows row0 .. and returns
        True on success (fgmm_em_step_reader)."""
        dt = self._stream_args(weights, means, variances, dtype, loglik, logz, N)
        D = self.D
        npdt = np.float32 if dtype == torch.float32 else np.uint16

        def _cb(ctx, row0, nrows, dst):
            try:
                buf = (ctypes.c_char * (int(nrows) * D * np.dtype(npdt).itemsize)).from_address(dst)
                out = np.frombuffer(buf, dtype=npdt).reshape(int(nrows), D)
                return 0 if read(int(row0), out) else 1
            except Exception:  # a failing reader ends the step with ERR_IO
                return 1

        cb = _lib.READ_FN(_cb)
        check(LIB.fgmm_em_step_reader(self._h, ctypes.cast(cb, ctypes.c_void_p), None, dt,
                                      int(N), _ptr(weights), _ptr(means), _ptr(variances),
                                      _ptr(loglik), _ptr(logz), _stream()),
              "fgmm_em_step_reader")

    # ---------------------------------------------------------------- sharded EM
    @property
    def stats_len(self) -> int:
        """Length of the statistics vector exchanged between shards: K (1 + 2D) + 1."""
        return self.K * (1 + 2 * self.D) + 1

    def partial(self, X, weights, means, variances, stats=None, logz=None):
        """E-step and statistics of one EM iteration on this shard of the rows.

        Returns the statistics vector (CUDA float64 [stats_len]: per component N_k,
        Σ r (x − μ_k), Σ r (x − μ_k)², then Σ log Z); the parameters are not changed.
        Vectors of disjoint shards add up to the vector of their union.
        """
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X, allow_host=True)
        if stats is None:
            stats = torch.empty(self.stats_len, dtype=torch.float64, device=weights.device)
        elif not (stats.is_cuda and stats.dtype == torch.float64 and stats.is_contiguous()
                  and stats.numel() == self.stats_len):
            raise ValueError("stats must be a contiguous CUDA float64 tensor of stats_len")
        if logz is not None and not (logz.is_cuda and logz.dtype == torch.float32
                                     and logz.numel() >= n):
            raise ValueError("logz must be a CUDA float32 tensor with N elements")
        fn = LIB.fgmm_em_partial if X.is_cuda else LIB.fgmm_em_partial_host
        check(fn(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means), _ptr(variances),
                 _ptr(stats), _ptr(logz), _stream()), "fgmm_em_partial")
        return stats

    def finish(self, stats, weights, means, variances, loglik=None):
        """M-step from a statistics vector summed over every shard; updates the
        parameters (those the statistics were taken about) in place."""
        self._check_params(weights, means, variances)
        if not (stats.is_cuda and stats.dtype == torch.float64 and stats.is_contiguous()
                and stats.numel() == self.stats_len):
            raise ValueError("stats must be a contiguous CUDA float64 tensor of stats_len")
        if loglik is not None and not (loglik.is_cuda and loglik.dtype == torch.float64):
            raise ValueError("loglik must be a CUDA float64 tensor")
        check(LIB.fgmm_em_finish(self._h, _ptr(stats), _ptr(weights), _ptr(means),
                                 _ptr(variances), _ptr(loglik), _stream()), "fgmm_em_finish")

    def combine(self, parts):
        """Sum of gathered statistics vectors ([n, stats_len]) in row order."""
        return stats_sum(parts)


    # ---------------------------------------------------------------- scoring, encoding
    def score_samples(self, X, weights, means, variances, loglik=None):
        """Per-point log-density under the mixture (fgmm_score_samples); returns float32
        [N] on the GPU.  loglik: optional CUDA float64 [1] receiving the sum."""
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X)
        logz = torch.empty(n, dtype=torch.float32, device=X.device)
        check(LIB.fgmm_score_samples(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means),
                                     _ptr(variances), _ptr(logz), _ptr(loglik), _stream()),
              "fgmm_score_samples")
        return logz

    def fisher_vector(self, X, weights, means, variances, normalize=False):
        """Fisher-vector encoding of the point set X (fgmm_fisher_vector): float32
        [2 K D] = [G_mu, G_sigma] on the GPU."""
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X)
        fv = torch.empty(2 * self.K * self.D, dtype=torch.float32, device=X.device)
        check(LIB.fgmm_fisher_vector(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means),
                                     _ptr(variances), int(bool(normalize)), _ptr(fv), _stream()),
              "fgmm_fisher_vector")
        return fv

    # ---------------------------------------------------------------- k-means warm start
    def kmeans_step(self, X, centroids, assign=None, counts=None, inertia=None):
        """One Lloyd iteration (fgmm_kmeans_step); centroids [K, D] float32 CUDA, in/out.
        assign: optional int32 [N], counts: optional int64 [K], inertia: optional
        float64 [1] (all CUDA) receive the assignment to the input centroids."""
        xp, dt, n, ldx = _x_args(X)
        if not (centroids.is_cuda and centroids.dtype == torch.float32 and centroids.is_contiguous()
                and tuple(centroids.shape) == (self.K, self.D)):
            raise ValueError("centroids must be a contiguous [K, D] float32 CUDA tensor")
        check(LIB.fgmm_kmeans_step(self._h, xp, dt, n, ldx, _ptr(centroids), _ptr(assign),
                                   _ptr(counts), _ptr(inertia), _stream()), "fgmm_kmeans_step")

    def kmeans_seed(self, X, first, u):
        """k-means++ seeding (fgmm_kmeans_seed) from the first index and the K-1 uniforms
        u (float64, any device).  Returns (centroids [K, D] float32, indices int64 [K])."""
        xp, dt, n, ldx = _x_args(X)
        u = torch.as_tensor(u, dtype=torch.float64).to(X.device).contiguous()
        if u.numel() != max(self.K - 1, 0):
            raise ValueError("u must hold K - 1 uniforms")
        C = torch.empty(self.K, self.D, dtype=torch.float32, device=X.device)
        idx = torch.empty(self.K, dtype=torch.int64, device=X.device)
        scratch = torch.empty(int(LIB.fgmm_kmeans_seed_scratch_bytes(n)), dtype=torch.uint8,
                              device=X.device)
        check(LIB.fgmm_kmeans_seed(self._h, xp, dt, n, ldx, int(first), _ptr(u), _ptr(C),
                                   _ptr(idx), _ptr(scratch), _stream()), "fgmm_kmeans_seed")
        return C, idx

    def fit(self, X, weights, means, variances, max_iters=100, tol=0.0):
        """Repeat step up to max_iters times; returns (final_loglik, iters_done)."""
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X)
        ll = ctypes.c_double()
        it = ctypes.c_int()
        check(LIB.fgmm_fit(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means),
                           _ptr(variances), max_iters, tol, ctypes.byref(ll),
                           ctypes.byref(it), _stream()), "fgmm_fit")
        return ll.value, it.value

    def soft_assign(self, X, weights, means, variances, top_m=2, r_threshold=0.0,
                    ids=None, resp=None):
        """§4.3 multi-assignment; returns (ids int32 [N, top_m], resp float32 [N, top_m])."""
        self._check_params(weights, means, variances)
        xp, dt, n, ldx = _x_args(X)
        if ids is None:
            ids = torch.empty(n, top_m, dtype=torch.int32, device=X.device)
        if resp is None:
            resp = torch.empty(n, top_m, dtype=torch.float32, device=X.device)
        check(LIB.fgmm_soft_assign(self._h, xp, dt, n, ldx, _ptr(weights), _ptr(means),
                                   _ptr(variances), top_m, r_threshold, _ptr(ids), _ptr(resp),
                                   _stream()), "fgmm_soft_assign")
        return ids, resp

    def profile(self, enable: bool = True):
        check(LIB.fgmm_profile_enable(self._h, int(enable)), "fgmm_profile_enable")

    def profile_read(self, reset: bool = True) -> dict:
        """Event timings since the last reset: totals per kernel kind, and under
        ``"kernels"`` per kernel name {launches, ms, active, active_ms}, where the
        active launches are those that passed their path gate and did work."""
        p = _lib.Profile()
        check(LIB.fgmm_profile_read(self._h, ctypes.byref(p), int(reset)), "fgmm_profile_read")
        out = {f: getattr(p, f) for f, _ in _lib.Profile._fields_ if not f.startswith("kernel_")}
        out["kernels"] = {
            LIB.fgmm_profile_kernel_name(i).decode(): {
                "launches": p.kernel_launches[i], "ms": p.kernel_ms[i],
                "active": p.kernel_active[i], "active_ms": p.kernel_active_ms[i]}
            for i in range(_lib.PROF_KERNELS) if p.kernel_launches[i]}
        return out

    def status(self) -> int:
        """Synchronise and return (then clear) the device status word."""
        return LIB.fgmm_get_status(self._h, _stream())

    def check_status(self):
        check(self.status(), "device status")


def stats_sum(parts, out=None):
    """Sum of statistics vectors stacked as rows of ``parts`` ([n, len] CUDA float64),
    in row order (bit-reproducible whatever order they were gathered in)."""
    if not (parts.is_cuda and parts.dtype == torch.float64 and parts.dim() == 2
            and parts.is_contiguous()):
        raise ValueError("parts must be a contiguous [n, len] CUDA float64 tensor")
    n, length = parts.shape
    if out is None:
        out = torch.empty(length, dtype=torch.float64, device=parts.device)
    check(LIB.fgmm_stats_sum(_ptr(parts), n, length, _ptr(out), _stream()), "fgmm_stats_sum")
    return out
