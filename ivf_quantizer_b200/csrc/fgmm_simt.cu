// CUDA-core (fp32) kernels of the fused EM step and of the soft assignment.
//
// Paper: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering".
//   §2            log N(x | mu_k, Sigma_k), log-sum-exp over k, Eqs. (1)-(3)
//   §3.1, Alg. 1  two sweeps over the components per point tile: the first
//                 builds log Z_i with an online log-sum-exp, the second
//                 recomputes the log-densities, forms r_ik = exp(log z_ik - log Z_i)
//                 and folds them into per-component sufficient statistics.
//   §4.2-4.3      argmax / top-m thresholded assignment.
//
// This is the FGMM_PREC_FP32 mode: log-densities in the direct form
// sum_d -(x_d - mu_kd)^2 / (2 sigma_kd^2), statistics centred on each
// component's current mean (sum r (x - mu), sum r (x - mu)^2), which keeps the
// variance update free of cancellation.  The responsibilities only ever exist as
// one 64 x 32 tile in shared memory.  Two exceptions: for D > 128 the log-sum-exp sweep
// keeps the chunk's log-densities (2^20 x Kp) for the statistics sweep, whose
// feature-block CTAs would otherwise each recompute them.  With block skipping it
// writes each point's largest log-density per 64 components, and the statistics sweep
// visits the points in the resulting order (fgmm_order.cu).
//
// Data layout: prepared parameters are zero padded to [Kp, Dp] (Kp multiple of
// 64, Dp multiple of 32); padded / dead components carry cconst = -inf so that
// they contribute exp(-inf) = 0.  Statistics partials live in [slots][KpS][1+2Dp]
// fp64 slots, each written by exactly one CTA, summed in a fixed order by the
// M-step kernel: the result is bitwise reproducible.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fgmm_internal.h"

namespace fgmm {

__device__ __forceinline__ float ld_x(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ld_x(const __nv_bfloat16* p) { return __bfloat162float(*p); }

__device__ __forceinline__ void set_status(int* st, int code) { atomicCAS(st, FGMM_OK, code); }

// ------------------------------------------------------------------ parameter preparation
// One CTA per (padded) component.  cconst_k = log pi_k - 1/2 sum_d log(2 pi sigma_kd^2),
// the d-independent part of log z_ik (§2); the sum is taken in fp64.
__global__ void prep_simt_kernel(int K, int D, int Kp, int Dp, int cov, const float* __restrict__ w,
                                 const float* __restrict__ means, const float* __restrict__ vars,
                                 float* __restrict__ mu, float* __restrict__ prec,
                                 float* __restrict__ cconst, int* status) {
  __shared__ double red[kSimtThreads];
  const int k = blockIdx.x;
  double acc = 0.0;
  bool bad = false;
  for (int d = threadIdx.x; d < Dp; d += blockDim.x) {
    float m = 0.f, p = 0.f;
    if (k < K && d < D) {
      const float v = (cov == FGMM_COV_DIAG) ? vars[(size_t)k * D + d] : vars[k];
      m = means[(size_t)k * D + d];
      if (!(v > 0.f) || !isfinite(v) || !isfinite(m)) bad = true;
      p = -0.5f / v;
      acc += log(2.0 * CUDART_PI * (double)v);
    }
    mu[(size_t)k * Dp + d] = m;
    prec[(size_t)k * Dp + d] = p;
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] += red[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float c = -CUDART_INF_F;
    if (k < K) {
      const float wk = w[k];
      if (!(wk >= 0.f) || !isfinite(wk)) bad = true;
      if (wk > 0.f) c = (float)(log((double)wk) - 0.5 * red[0]);
    }
    cconst[k] = c;
  }
  if (bad) set_status(status, FGMM_ERR_INVALID_ARG);
}

// ------------------------------------------------------------------ shared logit tile
// Computes acc[j][q] = sum_d prec_kd (x_id - mu_kd)^2 for points r = ty + 16 j of the
// tile and components kb + tx + 16 q, looping over the features in chunks of kDC staged
// in shared memory.  NJ points x NQ components per thread.  Each chunk's 32 terms are
// summed in fp32 and the chunk sums in fp64, so that the rounding of the sum does not
// grow with D (at D = 960 a plain fp32 sum of log-densities near -2700 carries ~5e-3
// nats of error, enough to move the responsibilities of shared points by 0.5%).
// rows: nullptr, or the point behind each position i0 + r (block-skipping order).
// kidx: nullptr, or the components of the tile's columns (column r is component kidx[r];
// kb is then unused).
template <int NQ, typename T>
__device__ __forceinline__ void logit_tile(const T* __restrict__ X, int64_t n, int64_t ldx, int D,
                                           int Dp, int64_t i0, int kb,
                                           const float* __restrict__ mu,
                                           const float* __restrict__ prec,
                                           float (*xs)[kDC + 4], float (*ms)[kDC + 4],
                                           float (*ps)[kDC + 4], float (&acc)[4][NQ],
                                           const int* __restrict__ rows = nullptr,
                                           const int* __restrict__ kidx = nullptr) {
  constexpr int KBLK = 16 * NQ;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  double dacc[4][NQ];
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int q = 0; q < NQ; ++q) dacc[j][q] = 0.0;
  // the next feature chunk is fetched into registers while the current one is used
  constexpr int XPT = kTP * kDC / kSimtThreads, MPT = KBLK * kDC / kSimtThreads;
  float xr[XPT], mr[MPT], pr[MPT];
  auto fetch = [&](int d0) {
#pragma unroll
    for (int u = 0; u < XPT; ++u) {
      const int e = threadIdx.x + u * kSimtThreads;
      const int r = e / kDC, cx = e % kDC;
      const int64_t i = i0 + r;
      const int d = d0 + cx;
      xr[u] = (i < n && d < D) ? ld_x(X + (rows ? (int64_t)rows[i] : i) * ldx + d) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < MPT; ++u) {
      const int e = threadIdx.x + u * kSimtThreads;
      const int r = e / kDC, cx = e % kDC;
      const int kr = kidx ? kidx[r] : kb + r;
      mr[u] = mu[(size_t)kr * Dp + d0 + cx];
      pr[u] = prec[(size_t)kr * Dp + d0 + cx];
    }
  };
  fetch(0);
  for (int d0 = 0; d0 < Dp; d0 += kDC) {
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < NQ; ++q) acc[j][q] = 0.f;
#pragma unroll
    for (int u = 0; u < XPT; ++u) {
      const int e = threadIdx.x + u * kSimtThreads;
      xs[e / kDC][e % kDC] = xr[u];
    }
#pragma unroll
    for (int u = 0; u < MPT; ++u) {
      const int e = threadIdx.x + u * kSimtThreads;
      ms[e / kDC][e % kDC] = mr[u];
      ps[e / kDC][e % kDC] = pr[u];
    }
    __syncthreads();
    if (d0 + kDC < Dp) fetch(d0 + kDC);
#pragma unroll 2
    for (int d = 0; d < kDC; d += 4) {
      float4 xv[4], mv[NQ], pv[NQ];
#pragma unroll
      for (int j = 0; j < 4; ++j) xv[j] = *reinterpret_cast<const float4*>(&xs[ty + 16 * j][d]);
#pragma unroll
      for (int q = 0; q < NQ; ++q) {
        mv[q] = *reinterpret_cast<const float4*>(&ms[tx + 16 * q][d]);
        pv[q] = *reinterpret_cast<const float4*>(&ps[tx + 16 * q][d]);
      }
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int q = 0; q < NQ; ++q) {
          float t;
          t = xv[j].x - mv[q].x; acc[j][q] = fmaf(pv[q].x * t, t, acc[j][q]);
          t = xv[j].y - mv[q].y; acc[j][q] = fmaf(pv[q].y * t, t, acc[j][q]);
          t = xv[j].z - mv[q].z; acc[j][q] = fmaf(pv[q].z * t, t, acc[j][q]);
          t = xv[j].w - mv[q].w; acc[j][q] = fmaf(pv[q].w * t, t, acc[j][q]);
        }
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < NQ; ++q) dacc[j][q] += (double)acc[j][q];
  }
#pragma unroll
  for (int j = 0; j < 4; ++j)
#pragma unroll
    for (int q = 0; q < NQ; ++q) acc[j][q] = (float)dacc[j][q];
}

// ------------------------------------------------------------------ sweep 1: log Z_i
// One CTA per 64-point tile; online log-sum-exp over blocks of 64 components
// (Alg. 1, step 1).  Writes log Z_i for the chunk, optionally to the caller's
// per-point buffer, and one fp64 partial log-likelihood per tile.
template <typename T, bool KEEP, bool BMAX>
__global__ void __launch_bounds__(kSimtThreads, 2)
    lse_simt_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp, int Kp,
                    const float* __restrict__ mu, const float* __restrict__ prec,
                    const float* __restrict__ cconst, float* __restrict__ logz,
                    float* __restrict__ logz_out, double* __restrict__ ll_tiles,
                    float* __restrict__ lbuf, float* __restrict__ bmx, const int* mode) {
  if (mode && *mode != kModeSimt) return;
  __shared__ __align__(16) float xs[kTP][kDC + 4];
  __shared__ __align__(16) float ms[kKB][kDC + 4];
  __shared__ __align__(16) float ps[kKB][kDC + 4];
  __shared__ double lls[kTP];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t i0 = (int64_t)blockIdx.x * kTP;
  float run_m[4], run_s[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) { run_m[j] = -CUDART_INF_F; run_s[j] = 0.f; }

  for (int kb = 0; kb < Kp; kb += kKB) {
    float acc[4][4];
    logit_tile<4>(X, n, ldx, D, Dp, i0, kb, mu, prec, xs, ms, ps, acc);
    float cc[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) cc[q] = cconst[kb + tx + 16 * q];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float l[4];
      float bm = -CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < 4; ++q) { l[q] = acc[j][q] + cc[q]; bm = fmaxf(bm, l[q]); }
      if (KEEP && i0 + ty + 16 * j < n) {   // kept for the statistics sweep (D > kFC)
        float* lr = lbuf + (size_t)(i0 + ty + 16 * j) * Kp + kb + tx;
#pragma unroll
        for (int q = 0; q < 4; ++q) lr[16 * q] = l[q];
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) bm = fmaxf(bm, __shfl_xor_sync(0xffffffffu, bm, off));
      // block skipping: the point's largest log z in this block of kKB components
      if (BMAX && tx == 0 && i0 + ty + 16 * j < n)
        bmx[(size_t)(i0 + ty + 16 * j) * (Kp / kKB) + kb / kKB] = bm;
      const float nm = fmaxf(run_m[j], bm);
      const bool live = nm > -CUDART_INF_F;
      float s = 0.f;
#pragma unroll
      for (int q = 0; q < 4; ++q) s += live ? expf(l[q] - nm) : 0.f;
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
      run_s[j] = live ? run_s[j] * expf(run_m[j] - nm) + s : 0.f;
      run_m[j] = nm;
    }
  }
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int r = ty + 16 * j;
    const int64_t i = i0 + r;
    const float lz = run_m[j] + logf(run_s[j]);
    if (tx == 0) {
      if (i < n) {
        logz[i] = lz;
        if (logz_out) logz_out[i] = lz;
      }
      lls[r] = (i < n) ? (double)lz : 0.0;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    double s = 0.0;
    for (int r = 0; r < kTP; ++r) s += lls[r];
    ll_tiles[blockIdx.x] = s;
  }
}

// Adds the chunk's per-tile partial log-likelihoods, in tile order, to ll_total.
// Runs only when the step's path (device mode word, or fixed_mode when mode is null)
// equals `required`; the partial count depends on that path's tile size.
__global__ void ll_accumulate_kernel(const double* __restrict__ ll_tiles, int n_simt, int n_tc,
                                     const int* mode, int fixed_mode, int required,
                                     double* __restrict__ ll_total) {
  __shared__ double red[kSimtThreads];
  if ((mode ? *mode : fixed_mode) != required) return;
  const int ntiles = (required == kModeSimt) ? n_simt : n_tc;
  double s = 0.0;
  for (int t = threadIdx.x; t < ntiles; t += blockDim.x) s += ll_tiles[t];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *ll_total += red[0];
}

// ------------------------------------------------------------------ sweep 2: statistics
// Grid (Kp / 32 component blocks, kSlices point slices, ceil(Dp / 128) feature blocks).
// Each CTA recomputes the log-densities of its 32 components for every 64-point tile
// of its slice (Alg. 1, step 2), forms r = exp(l - log Z_i), and accumulates
//   N_k = sum_i r_ik,  S1_kd = sum_i r_ik (x_id - mu_kd),  S2_kd = sum_i r_ik (x_id - mu_kd)^2
// for its 128 features in fp32 registers, flushed to its fp64 slot every kFlushTiles tiles.
struct StatsSmem {
  float xs[kTP][kDC + 4];
  float ms[kKBs][kDC + 4];
  float ps[kKBs][kDC + 4];
  float rs[kTP][kKBs + 4];
  float xf[kTP][kFC];
  float lz[kTP];
};

template <typename T, bool LISTED>
__global__ void __launch_bounds__(kSimtThreads)
    stats_simt_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp, int Kp,
                      const float* __restrict__ mu, const float* __restrict__ prec,
                      const float* __restrict__ cconst, const float* __restrict__ logz,
                      double* __restrict__ stats, int kstride, int64_t slice_len,
                      const float* __restrict__ lbuf, const int* __restrict__ rows,
                      const int* __restrict__ tlist, const int* __restrict__ tcnt, int tl_stride,
                      const int* mode) {
  if (mode && *mode != kModeSimt) return;
  extern __shared__ __align__(16) unsigned char smem_raw[];
  StatsSmem& sm = *reinterpret_cast<StatsSmem*>(smem_raw);
  const int kb = blockIdx.x * kKBs;
  const int s = blockIdx.y;
  const int f0 = blockIdx.z * kFC;
  // Point tiles of the CTA: positions [p_begin, p_end) of the chunk in steps of kTP; or
  // (block skipping, tlist) an even share of the active tiles of the 128-component block
  // holding the CTA's components, over the chunk in sweep-2 order (position i is point
  // rows[i], its log Z at logz[i]).
  int64_t p_begin = 0, p_end = n;
  int ntl = 0;
  if (!LISTED) {   // compile-time: the plain path carries none of the reordering
    rows = nullptr;
    tlist = nullptr;
  }
  if (LISTED) {
    const int b = kb / 128;
    const int na = tcnt[b];
    const int per = (na + (int)gridDim.y - 1) / (int)gridDim.y;
    const int l0 = min(na, s * per);
    ntl = min(na, l0 + per) - l0;
    tlist += (size_t)b * tl_stride + l0;
    if (ntl == 0) return;  // uniform over the CTA
  } else {
    p_begin = (int64_t)s * slice_len;
    p_end = min(n, p_begin + slice_len);
    if (p_begin >= p_end) return;  // uniform over the CTA
  }

  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int fl = threadIdx.x % kFC;            // this thread's feature (local)
  const int h = threadIdx.x / kFC;             // component half: comps h*16 .. h*16+15
  const int f = f0 + fl;
  const bool f_ok = f < D;
  const size_t row = (size_t)(1 + 2 * Dp);
  double* slot = stats + (size_t)s * kstride * row;

  float mreg[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) mreg[jj] = f_ok ? mu[(size_t)(kb + h * 16 + jj) * Dp + f] : 0.f;
  float acc1[16], acc2[16], nka[16];
#pragma unroll
  for (int jj = 0; jj < 16; ++jj) { acc1[jj] = 0.f; acc2[jj] = 0.f; nka[jj] = 0.f; }
  const bool nk_owner = (blockIdx.z == 0) && (fl == 0);
  float cc[2];
  cc[0] = cconst[kb + tx];
  cc[1] = cconst[kb + tx + 16];

  auto flush = [&]() {
    if (f_ok) {
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        double* r = slot + (size_t)(kb + h * 16 + jj) * row;
        r[1 + f] += (double)acc1[jj];
        r[1 + Dp + f] += (double)acc2[jj];
        acc1[jj] = 0.f;
        acc2[jj] = 0.f;
      }
    }
    if (nk_owner) {
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        slot[(size_t)(kb + h * 16 + jj) * row] += (double)nka[jj];
        nka[jj] = 0.f;
      }
    }
  };

  int tiles = 0;
  for (int jt = 0;; ++jt) {
    const int64_t i0 = LISTED ? (jt < ntl ? (int64_t)__ldg(tlist + jt) * kTP : p_end)
                              : p_begin + (int64_t)jt * kTP;
    if (i0 >= p_end) break;   // uniform over the CTA
    if (threadIdx.x < kTP) {
      const int64_t i = i0 + threadIdx.x;
      sm.lz[threadIdx.x] = (i < p_end) ? logz[i] : -CUDART_INF_F;
    }
    float lg[4][2];   // log z of the tile's points for the CTA's 32 components
    if (lbuf) {       // kept by the log-sum-exp sweep: the same values, bit for bit
      __syncthreads();   // sm.lz of this tile (no logit_tile barrier in this branch)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int64_t i = i0 + ty + 16 * j;
#pragma unroll
        for (int q = 0; q < 2; ++q)
          lg[j][q] = i < p_end ? lbuf[(size_t)(rows ? rows[i] : i) * Kp + kb + tx + 16 * q]
                               : -CUDART_INF_F;
      }
    } else {
      float acc[4][2];
      logit_tile<2>(X, p_end, ldx, D, Dp, i0, kb, mu, prec, sm.xs, sm.ms, sm.ps, acc, rows);
#pragma unroll
      for (int j = 0; j < 4; ++j)
#pragma unroll
        for (int q = 0; q < 2; ++q) lg[j][q] = acc[j][q] + cc[q];
    }
    // responsibilities of this tile for the CTA's 32 components
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = ty + 16 * j;
      const float lz = sm.lz[r];
      const bool ok = lz > -CUDART_INF_F && lz < CUDART_INF_F;
#pragma unroll
      for (int q = 0; q < 2; ++q) sm.rs[r][tx + 16 * q] = ok ? expf(lg[j][q] - lz) : 0.f;
    }
    // the tile's features for the statistics
    for (int e = threadIdx.x; e < kTP * kFC; e += kSimtThreads) {
      const int r = e / kFC, cx = e % kFC;
      const int64_t i = i0 + r;
      const int d = f0 + cx;
      sm.xf[r][cx] = (i < p_end && d < D) ? ld_x(X + (rows ? (int64_t)rows[i] : i) * ldx + d) : 0.f;
    }
    __syncthreads();
#pragma unroll 2
    for (int r = 0; r < kTP; ++r) {
      const float x = sm.xf[r][fl];
      float rv[16];
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const float4 t = *reinterpret_cast<const float4*>(&sm.rs[r][h * 16 + 4 * v]);
        rv[4 * v] = t.x; rv[4 * v + 1] = t.y; rv[4 * v + 2] = t.z; rv[4 * v + 3] = t.w;
      }
#pragma unroll
      for (int jj = 0; jj < 16; ++jj) {
        const float dv = x - mreg[jj];
        const float rd = rv[jj] * dv;
        acc1[jj] += rd;
        acc2[jj] = fmaf(rd, dv, acc2[jj]);
        nka[jj] += rv[jj];
      }
    }
    __syncthreads();
    if (++tiles == kFlushTiles) { flush(); tiles = 0; }
  }
  flush();
}

// ------------------------------------------------------------------ reduction and M-step
// Fixed-order sum of the statistics slots and conversion to the exchange form: per
// component [N_k, sum r (x - mu_k), sum r (x - mu_k)^2] about the step's input means
// (data units), then sum log Z.  A CUDA-core step, or a stiff component of a
// tensor-core step (side path), accumulated about the input mean already; the tensor
// cores accumulated moments of x^ = (x - c) s about the centre c, which are unscaled
// and shifted here in fp64.  One CTA per component.
__global__ void reduce_stats_kernel(int K, int D, int Dp, int kstride,
                                    const double* __restrict__ stats, int s_simt, int s_tc,
                                    const int* mode, int fixed_mode, const int* __restrict__ stiff,
                                    const float* __restrict__ means,
                                    const float* __restrict__ center,
                                    const float* __restrict__ dscale,
                                    const double* __restrict__ ll_total, double* __restrict__ out) {
  const int k = blockIdx.x;
  const bool simt_step = ((mode ? *mode : fixed_mode) == kModeSimt);
  const int nslots = simt_step ? s_simt : s_tc;
  const bool simt = simt_step || (stiff && stiff[k]);
  const size_t row = (size_t)(1 + 2 * Dp);
  const size_t orow = (size_t)(1 + 2 * D);
  double nk = 0.0;
  for (int s = 0; s < nslots; ++s) nk += stats[stat_idx(!simt_step, s, k, 0, kstride, row)];
  double* o = out + (size_t)k * orow;
  if (threadIdx.x == 0) o[0] = nk;
  if (k == 0 && threadIdx.x == 0) out[(size_t)K * orow] = *ll_total;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double s1 = 0.0, s2 = 0.0;
    for (int s = 0; s < nslots; ++s) {
      s1 += stats[stat_idx(!simt_step, s, k, 1 + d, kstride, row)];
      s2 += stats[stat_idx(!simt_step, s, k, 1 + Dp + d, kstride, row)];
    }
    if (!simt) {
      // about c in scaled units -> about c in data units -> about mu_k
      const double sd = dscale[d];
      const double s1c = s1 / sd, s2c = s2 / (sd * sd);
      const double del = (double)means[(size_t)k * D + d] - (double)center[d];
      s1 = s1c - nk * del;
      s2 = s2c - 2.0 * del * s1c + nk * del * del;
    }
    o[1 + d] = s1;
    o[1 + D + d] = s2;
  }
}

// M-step Eqs. (1)-(3) from exchange-form statistics (summed over every shard of the
// rows): mu_new = mu + S1/N_k, sigma^2 = S2/N_k - (S1/N_k)^2 (+ floor; spherical: mean
// over d).  Empty components keep mu and sigma^2.  Parameters are updated in place; the
// means passed in must be those the statistics were taken about.  One CTA per component.
__global__ void finish_kernel(int K, int D, int cov, double reg, const double* __restrict__ st,
                              float* __restrict__ means, float* __restrict__ vars,
                              double* __restrict__ nk_out, int* status) {
  __shared__ double red[kSimtThreads];
  const int k = blockIdx.x;
  const size_t orow = (size_t)(1 + 2 * D);
  const double* o = st + (size_t)k * orow;
  const double nk = o[0];
  const bool ll_ok = isfinite(st[(size_t)K * orow]);
  if (threadIdx.x == 0) nk_out[k] = nk;
  const bool live = ll_ok && (nk >= FGMM_EMPTY_NK);
  double vsum = 0.0;
  if (live)
    for (int d = threadIdx.x; d < D; d += blockDim.x) {
      const double m1 = o[1 + d] / nk;
      const double v = fmax(o[1 + D + d] / nk - m1 * m1, 0.0);
      float* mp = means + (size_t)k * D + d;
      *mp = (float)((double)*mp + m1);
      if (cov == FGMM_COV_DIAG) vars[(size_t)k * D + d] = (float)(v + reg);
      vsum += v;
    }
  if (cov == FGMM_COV_SPHERICAL) {
    red[threadIdx.x] = vsum;
    __syncthreads();
    for (int w = blockDim.x / 2; w > 0; w >>= 1) {
      if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
      __syncthreads();
    }
    if (threadIdx.x == 0 && live) vars[k] = (float)(red[0] / D + reg);
  }
  if (threadIdx.x == 0 && !isfinite(nk)) set_status(status, FGMM_ERR_NUMERIC);
}

// Fisher vector of the set from exchange-form statistics about the input means:
//   G_mu_kd = S1_kd / (N sqrt(pi_k) sigma_kd),
//   G_sigma_kd = (S2_kd / sigma_kd^2 - N_k) / (N sqrt(2 pi_k)),
// written as [G_mu (K x D), G_sigma (K x D)]; with normalize, sign(z) sqrt(|z|) and the
// block's fp64 sum of squares for the L2 norm.  One CTA per component.
__global__ void fisher_kernel(int K, int D, int cov, double n_points, const float* __restrict__ w,
                              const float* __restrict__ vars, const double* __restrict__ st,
                              int normalize, float* __restrict__ fv, double* __restrict__ part) {
  __shared__ double red[kSimtThreads];
  const int k = blockIdx.x;
  const size_t orow = (size_t)(1 + 2 * D);
  const double* o = st + (size_t)k * orow;
  const double pk = w[k];
  double sq = 0.0;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double gm = 0.0, gs = 0.0;
    if (pk > 0.0) {
      const double v = (cov == FGMM_COV_DIAG) ? (double)vars[(size_t)k * D + d] : (double)vars[k];
      gm = o[1 + d] / (n_points * sqrt(pk) * sqrt(v));
      gs = (o[1 + D + d] / v - o[0]) / (n_points * sqrt(2.0 * pk));
    }
    if (normalize) {
      gm = copysign(sqrt(fabs(gm)), gm);
      gs = copysign(sqrt(fabs(gs)), gs);
      sq += gm * gm + gs * gs;
    }
    fv[(size_t)k * D + d] = (float)gm;
    fv[(size_t)K * D + (size_t)k * D + d] = (float)gs;
  }
  red[threadIdx.x] = sq;
  __syncthreads();
  for (int r = blockDim.x / 2; r > 0; r >>= 1) {
    if (threadIdx.x < r) red[threadIdx.x] += red[threadIdx.x + r];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[k] = red[0];
}

// L2 normalisation of the Fisher vector: fixed-order sum of the per-component squares.
__global__ void fisher_norm_kernel(int K, int64_t len, const double* __restrict__ part,
                                   float* __restrict__ fv) {
  __shared__ double red[kSimtThreads];
  double s = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) s += part[k];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int r = blockDim.x / 2; r > 0; r >>= 1) {
    if (threadIdx.x < r) red[threadIdx.x] += red[threadIdx.x + r];
    __syncthreads();
  }
  const double tot = red[0];
  if (!(tot > 0.0)) return;
  const float inv = (float)(1.0 / sqrt(tot));
  for (int64_t i = threadIdx.x; i < len; i += blockDim.x) fv[i] *= inv;
}

// Sum of n_parts exchange-form statistics vectors, in part order.
__global__ void stats_sum_kernel(const double* __restrict__ parts, int n_parts, int64_t len,
                                 double* __restrict__ out) {
  for (int64_t j = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; j < len;
       j += (int64_t)gridDim.x * blockDim.x) {
    double acc = 0.0;
    for (int p = 0; p < n_parts; ++p) acc += parts[(size_t)p * len + j];
    out[j] = acc;
  }
}

// Weights pi_k = N_k / sum_{live k'} N_k' (Alg. 1, final step), log-likelihood output,
// and the numeric checks.  One CTA, fixed-order sums.
__global__ void finalize_kernel(int K, const double* __restrict__ nk, const double* __restrict__ ll_total,
                                float* __restrict__ weights, double* __restrict__ loglik_out,
                                int* status) {
  __shared__ double red[kSimtThreads];
  const double ll = *ll_total;
  const bool ll_ok = isfinite(ll);
  double s = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) s += (nk[k] >= FGMM_EMPTY_NK) ? nk[k] : 0.0;
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  const double tot = red[0];
  if (ll_ok && tot > 0.0) {
    for (int k = threadIdx.x; k < K; k += blockDim.x)
      weights[k] = (nk[k] >= FGMM_EMPTY_NK) ? (float)(nk[k] / tot) : 0.f;
  }
  if (threadIdx.x == 0) {
    if (loglik_out) *loglik_out = ll;
    if (!ll_ok || !(tot > 0.0)) set_status(status, FGMM_ERR_NUMERIC);
  }
}

// ------------------------------------------------------------------ soft assignment
// One CTA per 64-point tile, one sweep over the components: log-densities, an online
// log-sum-exp and a running top-m of log z (ranking by log z equals ranking by r,
// exp being monotone), ties kept in component order.  Epilogue per §4.3.
template <typename T>
__global__ void __launch_bounds__(kSimtThreads, 2)
    soft_assign_simt_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp, int Kp,
                            int K, const float* __restrict__ mu, const float* __restrict__ prec,
                            const float* __restrict__ cconst, int top_m, float thr,
                            int32_t* __restrict__ ids, float* __restrict__ resp) {
  __shared__ __align__(16) float xs[kTP][kDC + 4];
  __shared__ __align__(16) float ms[kKB][kDC + 4];
  __shared__ __align__(16) float ps[kKB][kDC + 4];
  __shared__ float ls[kTP][kKB + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t i0 = (int64_t)blockIdx.x * kTP;
  float tv[FGMM_MAX_TOP_M];
  int ti[FGMM_MAX_TOP_M];
  int cnt = 0;
  float m = -CUDART_INF_F, ssum = 0.f;
  for (int kb = 0; kb < Kp; kb += kKB) {
    float acc[4][4];
    logit_tile<4>(X, n, ldx, D, Dp, i0, kb, mu, prec, xs, ms, ps, acc);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float cc = cconst[kb + tx + 16 * q];
#pragma unroll
      for (int j = 0; j < 4; ++j) ls[ty + 16 * j][tx + 16 * q] = acc[j][q] + cc;
    }
    __syncthreads();
    if (threadIdx.x < kTP) {
      const int r = threadIdx.x;
      const int kend = min(kKB, K - kb);
      for (int c = 0; c < kend; ++c) {
        const float l = ls[r][c];
        const float nm = fmaxf(m, l);
        if (nm > -CUDART_INF_F) {
          ssum = ssum * expf(m - nm) + expf(l - nm);
          m = nm;
        }
        if (cnt < top_m || l > tv[top_m - 1]) {
          int p = (cnt < top_m) ? cnt : top_m - 1;
          while (p > 0 && tv[p - 1] < l) { tv[p] = tv[p - 1]; ti[p] = ti[p - 1]; --p; }
          tv[p] = l;
          ti[p] = kb + c;
          if (cnt < top_m) ++cnt;
        }
      }
    }
    __syncthreads();
  }
  if (threadIdx.x < kTP) {
    const int64_t i = i0 + threadIdx.x;
    if (i < n) {
      const float lz = m + logf(ssum);
      for (int rnk = 0; rnk < top_m; ++rnk) {
        int id = -1;
        float rv = 0.f;
        if (rnk < cnt) {
          const float rr = expf(tv[rnk] - lz);
          if (rnk == 0 || rr > thr) { id = ti[rnk]; rv = rr; }
        }
        ids[i * top_m + rnk] = id;
        if (resp) resp[i * top_m + rnk] = rv;
      }
    }
  }
}

// Assignment over the points regrouped by block mask (tensor-core filtered): one CTA per
// 64-position tile of the sorted chunk, visiting in increasing order only the
// 128-component blocks in the tile's mask (the OR of its points' masks, each a superset
// of the blocks whose log-densities can matter to the point), then the listed
// components (those left out of the filter, flagged in `listed`; skipped in their
// blocks).  Same arithmetic as soft_assign_simt_kernel on those components; the results
// go to the original point index.  The ranking breaks exact ties between a listed and an
// unlisted component by evaluation order rather than component index.
template <typename T>
__global__ void __launch_bounds__(kSimtThreads, 2)
    soft_assign_skip_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp,
                            int Kp, int K, const float* __restrict__ mu,
                            const float* __restrict__ prec, const float* __restrict__ cconst,
                            const int* __restrict__ perm, const uint32_t* __restrict__ tmask,
                            const int* __restrict__ xlist, const int* __restrict__ nxlist,
                            const int* __restrict__ listed, int top_m, float thr,
                            int32_t* __restrict__ ids,
                            float* __restrict__ resp) {
  __shared__ __align__(16) float xs[kTP][kDC + 4];
  __shared__ __align__(16) float ms[kKB][kDC + 4];
  __shared__ __align__(16) float ps[kKB][kDC + 4];
  __shared__ float ls[kTP][kKB + 1];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t i0 = (int64_t)blockIdx.x * kTP;
  const uint32_t mask = tmask[blockIdx.x];
  float tv[FGMM_MAX_TOP_M];
  int ti[FGMM_MAX_TOP_M];
  int cnt = 0;
  float m = -CUDART_INF_F, ssum = 0.f;
  // the blocks of the mask in increasing order, then the listed components (those the
  // tensor-core filter leaves out) in 64-column groups
  const int nx = *nxlist;
  const int nmask = __popc(mask);
  const int ngroups = 2 * nmask + (nx + kKB - 1) / kKB;
  uint32_t rest = mask;
  int sub = 0;                               // 64-component half of the current block
  for (int gi = 0; gi < ngroups; ++gi) {
    int kb, kend;
    const int* kidx = nullptr;
    if (gi < 2 * nmask) {
      const int b = __ffs(rest) - 1;          // next block of the mask, increasing
      kb = 128 * b + kKB * sub;
      if (sub) rest &= rest - 1u;
      sub ^= 1;
      if (kb >= Kp) continue;                 // uniform: K ends in this block's first half
      kend = min(kKB, K - kb);
    } else {
      kb = kKB * (gi - 2 * nmask);
      kidx = xlist + kb;
      kend = min(kKB, nx - kb);
    }
    {
      float acc[4][4];
      logit_tile<4>(X, n, ldx, D, Dp, i0, kb, mu, prec, xs, ms, ps, acc, perm, kidx);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int cq = tx + 16 * q;
        // a listed component is evaluated with the list, not again with its block
        const float cc = kidx ? (cq < kend ? cconst[kidx[cq]] : -CUDART_INF_F)
                              : (listed[kb + cq] ? -CUDART_INF_F : cconst[kb + cq]);
#pragma unroll
        for (int j = 0; j < 4; ++j) ls[ty + 16 * j][cq] = acc[j][q] + cc;
      }
      __syncthreads();
      if (threadIdx.x < kTP) {
        const int r = threadIdx.x;
        for (int c = 0; c < kend; ++c) {
          const float l = ls[r][c];
          const float nm = fmaxf(m, l);
          if (nm > -CUDART_INF_F) {
            ssum = ssum * expf(m - nm) + expf(l - nm);
            m = nm;
          }
          if (cnt < top_m || l > tv[top_m - 1]) {
            int p = (cnt < top_m) ? cnt : top_m - 1;
            while (p > 0 && tv[p - 1] < l) { tv[p] = tv[p - 1]; ti[p] = ti[p - 1]; --p; }
            tv[p] = l;
            ti[p] = kidx ? kidx[c] : kb + c;
            if (cnt < top_m) ++cnt;
          }
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x < kTP) {
    const int64_t i = i0 + threadIdx.x;
    if (i < n) {
      const int64_t o = perm[i];
      const float lz = m + logf(ssum);
      for (int rnk = 0; rnk < top_m; ++rnk) {
        int id = -1;
        float rv = 0.f;
        if (rnk < cnt) {
          const float rr = expf(tv[rnk] - lz);
          if (rnk == 0 || rr > thr) { id = ti[rnk]; rv = rr; }
        }
        ids[o * top_m + rnk] = id;
        if (resp) resp[o * top_m + rnk] = rv;
      }
    }
  }
}

// ------------------------------------------------------------------ AUTO: variance check
// After the tensor-core sweeps, AUTO checks how much cancellation the variance update
// S2/N_k - (S1/N_k)^2 suffers.  The statistics are raw moments about the global centre,
// accumulated in fp32 in TMEM for short runs of tiles before each fp64 flush; the new
// variance carries a relative error proportional to A = (S2/N_k) / variance (the
// measured rates are with kMaxAmplification in fgmm_internal.h).  A component whose A
// exceeds kMaxAmplification (a tight cluster far from the centre, or one that collapsed
// onto a single point this step) becomes stiff and the pass is redone, or at stage 1 the
// step goes to the CUDA-core path, whose statistics are centred on each component's
// current mean.  One CTA per component.
constexpr double kCheckMinNk = 1.0;      // effective points below which nothing is checked

// Stage 0 (after the first tensor-core pass, gated on *gate == tensor): a failing
// component becomes stiff (it will be evaluated on the side path) and *redo is set to
// tensor, which enables a second, hybrid pass with the enlarged stiff set.  Stage 1
// (after that pass, gated on *gate = the redo word): any remaining failure sends the
// step to the CUDA-core path (*mode = CUDA cores).
__global__ void tc_variance_check_kernel(int K, int D, int Dp, int kstride,
                                         double* __restrict__ stats, int nslots,
                                         int* __restrict__ stiff, const int* gate, int* redo,
                                         int* mode, int stage, const int* __restrict__ grey_pos,
                                         const double* __restrict__ grey_stats) {
  if (*gate != kModeTensor || *mode != kModeTensor) return;
  const int k = blockIdx.x;
  if (stiff[k]) return;  // the side path's statistics are centred on the mean: exact
  const size_t row = (size_t)(1 + 2 * Dp);
  const int gp = grey_pos[k];
  if (gp >= 0) {
    // a grey component (few points last step): its side-path statistics, centred on the
    // mean and free of the fp16 rounding of small responsibilities, replace the
    // tensor-core ones in slot 0, the other slots are cleared; no pass is redone
    for (int c = threadIdx.x; c < (int)row; c += blockDim.x)
      for (int s = 0; s < nslots; ++s)
        stats[stat_idx(true, s, k, c, kstride, row)] = (s == 0) ? grey_stats[(size_t)gp * row + c] : 0.0;
    if (threadIdx.x == 0) stiff[k] = 1;
    return;
  }
  double nk = 0.0;  // tensor-core slot layout (this check runs after tensor-core passes only)
  for (int s = 0; s < nslots; ++s) nk += stats[stat_idx(true, s, k, 0, kstride, row)];
  // Below one effective point the new mean and variance rest on far-tail
  // responsibilities and are outside the accuracy contract; the variance is floored
  // (never negative) whatever the cancellation, so such a component is not checked.
  if (!(nk >= kCheckMinNk)) return;
  __shared__ int bad_any;
  if (threadIdx.x == 0) bad_any = 0;
  __syncthreads();
  bool bad = false;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    double s1 = 0.0, s2 = 0.0;
    for (int s = 0; s < nslots; ++s) {
      s1 += stats[stat_idx(true, s, k, 1 + d, kstride, row)];
      s2 += stats[stat_idx(true, s, k, 1 + Dp + d, kstride, row)];
    }
    const double m2 = s2 / nk, m1 = s1 / nk;
    const double v = m2 - m1 * m1;
    if (!(v > 0.0) || !(m2 <= (double)kMaxAmplification * v)) bad = true;
  }
  if (bad) atomicExch(&bad_any, 1);
  __syncthreads();
  if (!bad_any) return;
  if (threadIdx.x == 0) {
    if (stage == 0) {
      stiff[k] = 1;
      atomicExch(redo, kModeTensor);
    } else {
      atomicExch(mode, kModeSimt);
    }
  }
}

// Clears the statistics and the log-likelihood when *flag == value (a pass is about to be
// redone).  Grid-stride over the statistics slots.
__global__ void redo_reset_kernel(const int* flag, int value, double* __restrict__ stats,
                                  size_t n, double* __restrict__ ll_total) {
  if (*flag != value) return;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n;
       i += (size_t)gridDim.x * blockDim.x)
    stats[i] = 0.0;
  if (blockIdx.x == 0 && threadIdx.x == 0) *ll_total = 0.0;
}

// Before the hybrid redo pass: components made stiff by the stage-0 check leave the
// tensor-core sweeps (c_k = -inf there).
__global__ void remask_kernel(const int* redo, const int* __restrict__ stiff, int Kt,
                              float* __restrict__ tck) {
  if (*redo != kModeTensor) return;
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k < Kt && stiff[k]) tck[k] = -CUDART_INF_F;
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_prep_simt(const Ctx& c, const float* weights, const float* means,
                             const float* vars, cudaStream_t s) {
  prof_begin(c, KI_PREP_SIMT, s);
  prep_simt_kernel<<<c.ws.Kp, kSimtThreads, 0, s>>>(c.K, c.D, c.ws.Kp, c.ws.Dp, c.cov, weights,
                                                    means, vars, c.ws.mu, c.ws.prec,
                                                    c.ws.cconst, c.ws.status);
  prof_end(c, KI_PREP_SIMT, s);
  return cudaGetLastError();
}

cudaError_t launch_lse_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, bool keep_logits, const int* mode, cudaStream_t s) {
  const unsigned grid = (unsigned)ceil_div64(n, kTP);
  float* lb = keep_logits ? c.ws.lbuf : nullptr;
  float* bx = keep_logits && simt_skip(c) ? c.ws.bmx : nullptr;
  prof_begin(c, KI_LSE_SIMT, s, mode, kModeSimt);
#define LSE_SIMT(T_, K_, B_)                                                                    \
  lse_simt_kernel<T_, K_, B_><<<grid, kSimtThreads, 0, s>>>(                                    \
      (const T_*)X, n, ldx, c.D, c.ws.Dp, c.ws.Kp, c.ws.mu, c.ws.prec, c.ws.cconst, c.ws.logz,  \
      logz_out, c.ws.ll_tiles, lb, bx, mode)
  if (x_dtype == FGMM_BF16) {
    if (lb) {
      if (bx) LSE_SIMT(__nv_bfloat16, true, true); else LSE_SIMT(__nv_bfloat16, true, false);
    } else {
      if (bx) LSE_SIMT(__nv_bfloat16, false, true); else LSE_SIMT(__nv_bfloat16, false, false);
    }
  } else {
    if (lb) {
      if (bx) LSE_SIMT(float, true, true); else LSE_SIMT(float, true, false);
    } else {
      if (bx) LSE_SIMT(float, false, true); else LSE_SIMT(float, false, false);
    }
  }
#undef LSE_SIMT
  prof_end(c, KI_LSE_SIMT, s);
  return cudaGetLastError();
}

cudaError_t launch_ll_accumulate(const Ctx& c, int64_t n, const int* mode, int fixed_mode,
                                 int required, cudaStream_t s) {
  prof_begin(c, KI_LL_ACCUMULATE, s, mode, required);
  ll_accumulate_kernel<<<1, kSimtThreads, 0, s>>>(c.ws.ll_tiles, (int)ceil_div64(n, kTP),
                                                  (int)ceil_div64(n, 4096), mode, fixed_mode,
                                                  required, c.ws.ll_total);
  prof_end(c, KI_LL_ACCUMULATE, s);
  return cudaGetLastError();
}

cudaError_t launch_stats_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s) {
  const size_t smem = sizeof(StatsSmem);
  static bool attr_set = false;
  if (!attr_set) {
    cudaFuncSetAttribute(stats_simt_kernel<float, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(stats_simt_kernel<__nv_bfloat16, false>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(stats_simt_kernel<float, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    cudaFuncSetAttribute(stats_simt_kernel<__nv_bfloat16, true>,
                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    attr_set = true;
  }
  int64_t slice = ceil_div64(n, kSlices);
  slice = ceil_div64(slice, kTP) * kTP;
  dim3 grid(c.ws.Kp / kKBs, kSlices, (unsigned)ceil_div64(c.ws.Dp, kFC));
  // block skipping: the chunk in sweep-2 order (rows, log Z), tiles from the lists
  const bool skip = simt_skip(c);
  const int* rows = skip ? c.ws.perm : nullptr;
  const float* lz = skip ? c.ws.lzp : c.ws.logz;
  const int* tl = skip ? c.ws.tlist : nullptr;
  const int tl_stride = (int)(kChunk / kTP);
  prof_begin(c, KI_STATS_SIMT, s, mode, kModeSimt);
#define STATS_SIMT(T_, L_)                                                                      \
  stats_simt_kernel<T_, L_><<<grid, kSimtThreads, smem, s>>>(                                   \
      (const T_*)X, n, ldx, c.D, c.ws.Dp, c.ws.Kp, c.ws.mu, c.ws.prec, c.ws.cconst, lz,         \
      c.ws.stats, c.ws.KpS, slice, c.ws.lbuf, rows, tl, c.ws.tcnt, tl_stride, mode)
  if (x_dtype == FGMM_BF16) {
    if (skip) STATS_SIMT(__nv_bfloat16, true); else STATS_SIMT(__nv_bfloat16, false);
  } else {
    if (skip) STATS_SIMT(float, true); else STATS_SIMT(float, false);
  }
#undef STATS_SIMT
  prof_end(c, KI_STATS_SIMT, s);
  return cudaGetLastError();
}

cudaError_t launch_reduce_stats(const Ctx& c, const float* means, double* out, const int* mode,
                                int fixed_mode, cudaStream_t s) {
  prof_begin(c, KI_REDUCE_STATS, s);
  reduce_stats_kernel<<<c.K, kSimtThreads, 0, s>>>(
      c.K, c.D, c.ws.Dp, c.ws.KpS, c.ws.stats, kSlices, c.tc.ready ? tc_stat_slots(c) : 1, mode,
      fixed_mode, c.tc.ready ? c.ws.stiff : nullptr, means, c.ws.center, c.ws.dscale,
      c.ws.ll_total, out);
  prof_end(c, KI_REDUCE_STATS, s);
  return cudaGetLastError();
}

cudaError_t launch_finish(const Ctx& c, const double* st, float* weights, float* means,
                          float* vars, double* loglik_out, cudaStream_t s) {
  prof_begin(c, KI_MSTEP, s);
  finish_kernel<<<c.K, kSimtThreads, 0, s>>>(c.K, c.D, c.cov, c.reg, st, means, vars, c.ws.nk,
                                             c.ws.status);
  prof_end(c, KI_MSTEP, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prof_begin(c, KI_FINALIZE, s);
  finalize_kernel<<<1, kSimtThreads, 0, s>>>(c.K, c.ws.nk, st + (size_t)c.K * (1 + 2 * c.D),
                                             weights, loglik_out, c.ws.status);
  prof_end(c, KI_FINALIZE, s);
  return cudaGetLastError();
}

cudaError_t launch_fisher(const Ctx& c, const float* weights, const float* vars, double n_points,
                          const double* st, int normalize, float* fv, cudaStream_t s) {
  fisher_kernel<<<c.K, kSimtThreads, 0, s>>>(c.K, c.D, c.cov, n_points, weights, vars, st,
                                             normalize, fv, c.ws.ll_tiles);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || !normalize) return e;
  fisher_norm_kernel<<<1, kSimtThreads, 0, s>>>(c.K, (int64_t)2 * c.K * c.D, c.ws.ll_tiles, fv);
  return cudaGetLastError();
}

cudaError_t launch_stats_sum(const double* parts, int n_parts, int64_t len, double* out,
                             cudaStream_t s) {
  const int64_t blocks = (len + 255) / 256;
  stats_sum_kernel<<<(unsigned)(blocks < 1024 ? blocks : 1024), 256, 0, s>>>(parts, n_parts, len,
                                                                             out);
  return cudaGetLastError();
}

cudaError_t launch_soft_assign_skip(const Ctx& c, const void* X, int x_dtype, int64_t n,
                                    int64_t ldx, int top_m, float r_threshold, int32_t* ids,
                                    float* resp, cudaStream_t s) {
  const Workspace& w = c.ws;
  const unsigned grid = (unsigned)ceil_div64(n, kTP);
  prof_begin(c, KI_SOFT_ASSIGN, s);
  if (x_dtype == FGMM_BF16)
    soft_assign_skip_kernel<<<grid, kSimtThreads, 0, s>>>(
        (const __nv_bfloat16*)X, n, ldx, c.D, w.Dp, w.Kp, c.K, w.mu, w.prec, w.cconst, w.perm,
        w.tmask, w.alist, w.nalist, w.stiff, top_m, r_threshold, ids, resp);
  else
    soft_assign_skip_kernel<<<grid, kSimtThreads, 0, s>>>(
        (const float*)X, n, ldx, c.D, w.Dp, w.Kp, c.K, w.mu, w.prec, w.cconst, w.perm, w.tmask,
        w.alist, w.nalist, w.stiff, top_m, r_threshold, ids, resp);
  prof_end(c, KI_SOFT_ASSIGN, s);
  return cudaGetLastError();
}

cudaError_t launch_soft_assign_simt(const Ctx& c, const void* X, int x_dtype, int64_t n,
                                    int64_t ldx, int top_m, float r_threshold, int32_t* ids,
                                    float* resp, cudaStream_t s) {
  const unsigned grid = (unsigned)ceil_div64(n, kTP);
  prof_begin(c, KI_SOFT_ASSIGN, s);
  if (x_dtype == FGMM_BF16)
    soft_assign_simt_kernel<<<grid, kSimtThreads, 0, s>>>(
        (const __nv_bfloat16*)X, n, ldx, c.D, c.ws.Dp, c.ws.Kp, c.K, c.ws.mu, c.ws.prec,
        c.ws.cconst, top_m, r_threshold, ids, resp);
  else
    soft_assign_simt_kernel<<<grid, kSimtThreads, 0, s>>>(
        (const float*)X, n, ldx, c.D, c.ws.Dp, c.ws.Kp, c.K, c.ws.mu, c.ws.prec, c.ws.cconst,
        top_m, r_threshold, ids, resp);
  prof_end(c, KI_SOFT_ASSIGN, s);
  return cudaGetLastError();
}

}  // namespace fgmm

namespace fgmm {
cudaError_t launch_auto_check(const Ctx& c, int stage, cudaStream_t s) {
  const Workspace& w = c.ws;
  const size_t n = (size_t)w.slots * w.KpS * (1 + 2 * (size_t)w.Dp);
  prof_begin(c, KI_AUTO_CHECK, s);
  tc_variance_check_kernel<<<c.K, kSimtThreads, 0, s>>>(c.K, c.D, w.Dp, w.KpS, w.stats,
                                                        tc_stat_slots(c), w.stiff,
                                                        stage == 0 ? w.mode : w.mode2, w.mode2,
                                                        w.mode, stage, w.grey_pos,
                                                        w.grey_stats);
  prof_end(c, KI_AUTO_CHECK, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prof_begin(c, KI_REDO_RESET, s);
  if (stage == 0)
    redo_reset_kernel<<<2 * c.num_sms, 256, 0, s>>>(w.mode2, kModeTensor, w.stats, n, w.ll_total);
  else
    redo_reset_kernel<<<2 * c.num_sms, 256, 0, s>>>(w.mode, kModeSimt, w.stats, n, w.ll_total);
  prof_end(c, KI_REDO_RESET, s);
  e = cudaGetLastError();
  if (e != cudaSuccess || stage != 0) return e;
  prof_begin(c, KI_REMASK, s);
  remask_kernel<<<(w.Kt + 255) / 256, 256, 0, s>>>(w.mode2, w.stiff, w.Kt, w.tck);
  prof_end(c, KI_REMASK, s);
  return cudaGetLastError();
}
}  // namespace fgmm

namespace fgmm {
// Launchers on explicit buffers (no handle), for the allocation-free entry point.
cudaError_t launch_prep_simt_raw(int K, int D, int Kp, int Dp, int cov, const float* weights,
                                 const float* means, const float* vars, float* mu, float* prec,
                                 float* cconst, int* status, cudaStream_t s) {
  prep_simt_kernel<<<Kp, kSimtThreads, 0, s>>>(K, D, Kp, Dp, cov, weights, means, vars, mu, prec,
                                               cconst, status);
  return cudaGetLastError();
}

cudaError_t launch_soft_assign_simt_raw(const void* X, int x_dtype, int64_t n, int64_t ldx, int K,
                                        int D, int Kp, int Dp, const float* mu, const float* prec,
                                        const float* cconst, int top_m, float r_threshold,
                                        int32_t* ids, float* resp, cudaStream_t s) {
  const unsigned grid = (unsigned)ceil_div64(n, kTP);
  if (x_dtype == FGMM_BF16)
    soft_assign_simt_kernel<<<grid, kSimtThreads, 0, s>>>((const __nv_bfloat16*)X, n, ldx, D, Dp,
                                                          Kp, K, mu, prec, cconst, top_m,
                                                          r_threshold, ids, resp);
  else
    soft_assign_simt_kernel<<<grid, kSimtThreads, 0, s>>>((const float*)X, n, ldx, D, Dp, Kp, K,
                                                          mu, prec, cconst, top_m, r_threshold,
                                                          ids, resp);
  return cudaGetLastError();
}
}  // namespace fgmm
