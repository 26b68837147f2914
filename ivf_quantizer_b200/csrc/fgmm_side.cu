// Side path of the AUTO mode: the few components that the tensor-core expanded form
// cannot evaluate accurately ("stiff": collapsed onto a point, very few effective
// points, or tight and far from the coordinate centre) are taken out of the tensor-core
// sweeps (their c_k is -inf there) and handled here on CUDA cores in the direct form
// sum_d -(x_d - mu_kd)^2 / (2 sigma_kd^2), with statistics centred on their current mean
// ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", §2 for the
// density and Eqs. (1)-(3); the same quantities as the tensor-core sweeps, exactly).
//
//   stiff_compact      ordered list of the stiff (then grey) components (deterministic)
//   side_flag_count,   the points that sweep 1 flagged (a side component may come within
//   side_flagged       the cut), as a list in index order
//   side_lse           per flagged point: log Z <- logsumexp(log Z_tensor, log z_ik for
//                      stiff k); keeps the (component, log z) pairs within the cut
//   ll_partials        per-block fp64 sums of the chunk's log Z (fixed order)
//   side_stats         per side component, over the flagged list: N_k, sum r (x - mu),
//                      sum r (x - mu)^2 from the kept pairs
//
// A stiff component's log-density is evaluated dimension by dimension and abandoned
// as soon as its upper bound (the constant plus the partial sum, every remaining term
// being <= 0) falls more than kCut nats below the point's log Z: its responsibility
// would be below exp(-kCut) (see kSideCut).  A collapsed component costs one or two
// dimensions per point.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fgmm_internal.h"

namespace fgmm {
namespace {

constexpr float kCut = kSideCut;
constexpr double kErrRel = 2e-5;      // tensor-core logit error per unit of sum |W' phi|
constexpr float kLzMargin = 5000.f;   // nats below the lowest component peak

__device__ __forceinline__ float ldx_f(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ldx_f(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// Direct-form log z for one point and one component, abandoned (returns -inf) once the
// bound drops below `floor`.
template <typename T>
__device__ __forceinline__ float stiff_logit(const T* __restrict__ x, int D,
                                             const float* __restrict__ mu,
                                             const float* __restrict__ prec, float c,
                                             float floor) {
  if (!(c > floor)) return -CUDART_INF_F;
  float acc = 0.f;  // sum of prec (x - mu)^2, prec = -1/(2 sigma^2) <= 0
  int d = 0;
  for (; d < D; ++d) {
    const float t = ldx_f(x + d) - mu[d];
    acc = fmaf(prec[d] * t, t, acc);
    if ((d & 3) == 3 && c + acc < floor) return -CUDART_INF_F;
  }
  return c + acc;
}

}  // namespace

constexpr int kMaxStiff = kSideMaxStiff;   // stiff + grey components of one pass

// Block-wide, order-preserving append of the components k < K with sel(k) != 0 to
// list[*base ..], by warp ballots; entries at or beyond cap are dropped (pos = -1).
// pos (optional) receives the index relative to `start`.  Returns through *base the
// uncapped count.  Every thread of the CTA must call it.
template <typename Sel>
__device__ void append_list(Sel sel, int K, int* __restrict__ list, int* base, int start, int cap,
                            int* __restrict__ pos) {
  __shared__ int wsum[32];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  for (int k0 = 0; k0 < K; k0 += blockDim.x) {
    const int k = k0 + threadIdx.x;
    const int f = (k < K) ? sel(k) : 0;
    const unsigned m = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[w] = __popc(m);
    __syncthreads();
    int off = *base;
    for (int i = 0; i < w; ++i) off += wsum[i];
    const int at = off + __popc(m & ((1u << lane) - 1u));
    if (f && at < cap) list[at] = k;
    if (pos && k < K) pos[k] = (f && at < cap) ? at - start : -1;
    __syncthreads();
    if (threadIdx.x == 0) {
      int t = 0;
      for (int i = 0; i < (int)(blockDim.x >> 5); ++i) t += wsum[i];
      *base += t;
    }
    __syncthreads();
  }
}

// One CTA: the stiff components (list[0 .. n_stiff)), then the grey ones that fit
// (list[n_stiff .. n_stiff + n_grey), at most kMaxStiff in all), the filter constants.
// More than kMaxStiff stiff components: the side path would cost as much as the
// CUDA-core path, so the whole step goes there (*mode), and the gated pass is switched
// off (*gate).  Runs when *gate is tensor (or gate is null).
__global__ void stiff_compact_kernel(const int* __restrict__ stiff, const int* __restrict__ grey,
                                     int K, int Kt, int* __restrict__ list,
                                     int* __restrict__ n_out, int* __restrict__ grey_pos,
                                     const float* __restrict__ craw, const float* __restrict__ mq,
                                     const float* __restrict__ peak, float* __restrict__ ckf,
                                     float* __restrict__ lzlow, int* gate, int* mode) {
  if (gate && *gate != kModeTensor) return;
  __shared__ int base, nst;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  append_list([&](int k) { return stiff[k]; }, K, list, &base, 0, Kt, nullptr);
  if (threadIdx.x == 0) nst = base;
  __syncthreads();
  const int n_st = nst;
  append_list([&](int k) { return grey[k] && !stiff[k]; }, K, list, &base, n_st,
              max(n_st, kMaxStiff), grey_pos);
  for (int k = K + threadIdx.x; k < Kt; k += blockDim.x) grey_pos[k] = -1;
  if (threadIdx.x == 0) {
    n_out[0] = n_st;
    n_out[1] = (n_st < kMaxStiff) ? min(base, kMaxStiff) - n_st : 0;
    if (gate && n_st > kMaxStiff) {
      *mode = kModeSimt;
      *gate = kModeSimt;
    }
  }
  __syncthreads();
  // Filter constants.  The tensor-core logit of component k at x is exact up to
  // |err| <= kErrRel * sum_j |W'_kj phi_j(x)| (three-product split: 3 * 2^-22 per product;
  // fp32 accumulation over at most 64 steps: 64 * 2^-23; kErrRel carries a factor 2.4 of
  // margin).  With M_k = sum_d p_d mu~_d^2 (p = 1/sigma^2, mu~ = mu - c) and
  // s = sum_d p_d (x_d - mu_d)^2, that sum is at most 1.5 M + 2 sqrt(M s) + s / 2.  A point
  // with log Z >= L for which k matters (log z_k >= log Z - kCut) has
  // s = 2 (P_k - log z_k) <= Q_k = 2 (P_k - L + kCut), so its estimate exceeds
  // log Z - kCut - E_k, E_k = kErrRel (1.5 M + 2 sqrt(M Q) + Q / 2) + 1.  L = the lowest
  // peak minus kLzMargin; points below L are always flagged.
  __shared__ float red[256];
  float pm = CUDART_INF_F;
  for (int k = threadIdx.x; k < K; k += blockDim.x)
    if (peak[k] > -CUDART_INF_F) pm = fminf(pm, peak[k]);
  red[threadIdx.x] = pm;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) red[threadIdx.x] = fminf(red[threadIdx.x], red[threadIdx.x + s]);
    __syncthreads();
  }
  const float low = red[0] - kLzMargin;
  if (threadIdx.x == 0) *lzlow = low;
  for (int k = threadIdx.x; k < Kt; k += blockDim.x) {
    float f = -CUDART_INF_F;
    if (k < K && (stiff[k] || grey_pos[k] >= 0) && craw[k] > -CUDART_INF_F) {
      const double M = mq[k];
      const double Q = fmax(2.0 * ((double)peak[k] - (double)low + (double)kCut), 0.0);
      const double E = kErrRel * (1.5 * M + 2.0 * sqrt(M * Q) + 0.5 * Q) + 1.0;
      f = (float)((double)craw[k] + E);
    }
    ckf[k] = f;
  }
}

// The flagged points of the chunk as a list in increasing index order, so that side_lse
// runs on full warps and side_stats visits only them, deterministically: per 4096-point
// CTA a count (side_flag_count), then each CTA writes its points after those of the CTAs
// before it (side_flagged).  Unflagged points get pair count 0.
__global__ void side_flag_count_kernel(const uint8_t* __restrict__ flag, int64_t n,
                                       const int* __restrict__ n_stiff, int* __restrict__ cnts,
                                       uint8_t* __restrict__ pair_cnt, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  if (n_stiff[0] + n_stiff[1] == 0) return;
  __shared__ int wsum[8];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int64_t i0 = (int64_t)blockIdx.x * 4096;
  int c = 0;
  for (int r0 = 0; r0 < 4096; r0 += 256) {
    const int64_t i = i0 + r0 + threadIdx.x;
    const bool f = i < n && flag[i];
    if (i < n && !f) pair_cnt[i] = 0;
    c += __popc(__ballot_sync(0xffffffffu, f));
  }
  if (lane == 0) wsum[warp] = c;
  __syncthreads();
  if (threadIdx.x == 0) {
    int t = 0;
    for (int w2 = 0; w2 < 8; ++w2) t += wsum[w2];
    cnts[blockIdx.x] = t;
  }
}

__global__ void side_flagged_kernel(const uint8_t* __restrict__ flag, int64_t n,
                                    const int* __restrict__ n_stiff, const int* __restrict__ cnts,
                                    int* __restrict__ list, int* __restrict__ count,
                                    const int* mode) {
  if (mode && *mode != kModeTensor) return;
  if (n_stiff[0] + n_stiff[1] == 0) return;
  __shared__ int wsum[8], base;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    int t = 0;
    for (int b = 0; b < (int)blockIdx.x; ++b) t += cnts[b];
    base = t;
    if (blockIdx.x == gridDim.x - 1) *count = t + cnts[blockIdx.x];
  }
  const int64_t i0 = (int64_t)blockIdx.x * 4096;
  for (int r0 = 0; r0 < 4096; r0 += 256) {
    const int64_t i = i0 + r0 + threadIdx.x;
    const bool f = i < n && flag[i];
    const unsigned m = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[warp] = __popc(m);
    __syncthreads();
    int off = base, tot = 0;
    for (int w2 = 0; w2 < 8; ++w2) {
      off += w2 < warp ? wsum[w2] : 0;
      tot += wsum[w2];
    }
    if (f) list[off + __popc(m & ((1u << lane) - 1u))] = (int)i;
    __syncthreads();
    if (threadIdx.x == 0) base += tot;
  }
}

// Thread per flagged point: merge the stiff components' log-densities into log Z.  Every stiff
// or grey component that comes within kCut of the point's log Z is remembered (index in
// the side-path list and log z, up to kSidePairs of them) for the statistics, which then
// need no second evaluation; the grey ones are evaluated for that alone (their
// log-densities are in the tensor-core log Z already).
template <typename T>
__global__ void side_lse_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp,
                                const float* __restrict__ mu, const float* __restrict__ prec,
                                const float* __restrict__ cconst, const int* __restrict__ list,
                                const int* __restrict__ n_stiff,
                                float* __restrict__ logz, float* __restrict__ logz_out,
                                uint8_t* __restrict__ pair_cnt, uint8_t* __restrict__ pair_j,
                                float* __restrict__ pair_l, const int* __restrict__ flagged,
                                const int* __restrict__ n_flagged, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  const int ns = n_stiff[0], nall = n_stiff[0] + n_stiff[1];
  if (nall == 0) return;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= *n_flagged) return;
  const int64_t i = flagged[e];
  const T* x = X + i * ldx;
  float lz = logz[i];
  int cnt = 0;
  for (int j = 0; j < nall; ++j) {
    const int k = list[j];
    const float l = stiff_logit(x, D, mu + (size_t)k * Dp, prec + (size_t)k * Dp, cconst[k],
                                lz - kCut);
    if (l > -CUDART_INF_F) {
      if (cnt < kSidePairs) {
        pair_j[i * kSidePairs + cnt] = (uint8_t)j;
        pair_l[i * kSidePairs + cnt] = l;
      }
      ++cnt;
      if (j < ns) {
        const float m = fmaxf(lz, l);
        lz = (lz > -CUDART_INF_F) ? m + log1pf(expf(fminf(lz, l) - m)) : l;
      }
    }
  }
  pair_cnt[i] = (uint8_t)min(cnt, 255);
  if (ns > 0) {
    logz[i] = lz;
    if (logz_out) logz_out[i] = lz;
  }
}

// Fixed-order per-block fp64 sums of log Z over [b * 4096, (b + 1) * 4096).
__global__ void ll_partials_kernel(const float* __restrict__ logz, int64_t n,
                                   double* __restrict__ part, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  __shared__ double red[256];
  const int64_t b0 = (int64_t)blockIdx.x * 4096;
  double s = 0.0;
  for (int e = threadIdx.x; e < 4096; e += 256) {
    const int64_t i = b0 + e;
    if (i < n) s += (double)logz[i];
  }
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) part[blockIdx.x] = red[0];
}

// Grid (kSideMaxStiff, kSideParts): CTA (j, p) folds stiff component list[j] over the
// p-th of kSideParts equal point ranges of the chunk.  Each warp takes a contiguous part
// of the range; for a batch of 32 points the lanes evaluate r = exp(log z - log Z), and
// the points with r > 0 are folded into the warp's shared-memory sums by the whole warp
// (lanes over dimensions, points in index order).  The 8 warp sums are combined in warp
// order and written as this CTA's partial row; side_reduce adds the partial rows, in p
// order, to the component's statistics.  Everything is deterministic.
struct SideAcc {
  float s1[128];   // the tensor-core path (and so this side path) has D <= 128
  float s2[128];
  float nk;
};

template <typename T>
__global__ void __launch_bounds__(256)
    side_stats_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp,
                      const float* __restrict__ mu, const float* __restrict__ prec,
                      const float* __restrict__ cconst, const int* __restrict__ list,
                      const int* __restrict__ n_stiff, const uint8_t* __restrict__ pair_cnt,
                      const uint8_t* __restrict__ pair_j, const float* __restrict__ pair_l,
                      const float* __restrict__ logz, const int* __restrict__ flagged,
                      const int* __restrict__ n_flagged, double* __restrict__ part,
                      const int* mode) {
  if (mode && *mode != kModeTensor) return;
  const int j = blockIdx.x;
  if (j >= n_stiff[0] + n_stiff[1]) return;   // stiff, then grey components
  __shared__ SideAcc acc[8];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k = list[j];
  const float* muk = mu + (size_t)k * Dp;
  const float* pk = prec + (size_t)k * Dp;
  const float ck = cconst[k];
  // the p-th of kSideParts equal ranges of the flagged list (points in index order)
  const int64_t nf = *n_flagged;
  const int64_t range = (nf + kSideParts - 1) / kSideParts;
  const int64_t p0 = (int64_t)blockIdx.y * range, p1 = min(nf, p0 + range);
  const int64_t wlen = (range + 7) / 8;
  const int64_t w0 = p0 + warp * wlen, w1 = min(p1, w0 + wlen);
  SideAcc& a = acc[warp];
  for (int d = lane; d < 128; d += 32) { a.s1[d] = 0.f; a.s2[d] = 0.f; }
  float nk = 0.f;
  __syncwarp();
  for (int64_t b = w0; b < w1; b += 32) {
    const int64_t i = b + lane < w1 ? (int64_t)flagged[b + lane] : 0;
    float r = 0.f;
    const int cnt = b + lane < w1 ? pair_cnt[i] : 0;
    if (cnt > 0) {
      const float lz = logz[i];
      float l = -CUDART_INF_F;
      if (cnt <= kSidePairs) {   // the log z that side_lse found, if j was within the cut
        for (int s = 0; s < cnt; ++s)
          if (pair_j[i * kSidePairs + s] == j) l = pair_l[i * kSidePairs + s];
      } else {                   // more components than slots: evaluate again
        l = stiff_logit(X + i * ldx, D, muk, pk, ck, lz - kCut);
      }
      if (l > -CUDART_INF_F && lz > -CUDART_INF_F) r = fminf(expf(l - lz), 1.f);
    }
    unsigned live = __ballot_sync(0xffffffffu, r > 0.f);
    while (live) {
      const int src = __ffs(live) - 1;
      live &= live - 1;
      const float rr = __shfl_sync(0xffffffffu, r, src);
      const T* x = X + __shfl_sync(0xffffffffu, i, src) * ldx;
      for (int d = lane; d < D; d += 32) {
        const float t = ldx_f(x + d) - muk[d];
        const float rt = rr * t;
        a.s1[d] += rt;
        a.s2[d] = fmaf(rt, t, a.s2[d]);
      }
      nk += rr;   // the same running sum in every lane
    }
  }
  if (lane == 0) a.nk = nk;
  __syncthreads();
  const size_t row = (size_t)(1 + 2 * Dp);
  double* dst = part + ((size_t)blockIdx.y * kSideMaxStiff + j) * row;
  for (int d = threadIdx.x; d < D; d += blockDim.x) {
    float s1 = 0.f, s2 = 0.f;
    for (int w = 0; w < 8; ++w) { s1 += acc[w].s1[d]; s2 += acc[w].s2[d]; }
    dst[1 + d] = (double)s1;
    dst[1 + Dp + d] = (double)s2;
  }
  if (threadIdx.x == 0) {
    float t = 0.f;
    for (int w = 0; w < 8; ++w) t += acc[w].nk;
    dst[0] = (double)t;
  }
}

// One CTA per stiff slot j: the kSideParts partial rows, summed in p order, are added to
// the statistics of component list[j] (slot 0 of the point slices, in the tensor-core
// layout; the tensor-core sweep added zeros there, the component being masked out of it).
// A grey component's row goes to grey_stats (its statistics in waiting) instead.
__global__ void side_reduce_kernel(const double* __restrict__ part, const int* __restrict__ list,
                                   const int* __restrict__ n_stiff, int D, int Dp, int kstride,
                                   double* __restrict__ stats, double* __restrict__ grey_stats,
                                   const int* mode) {
  if (mode && *mode != kModeTensor) return;
  const int j = blockIdx.x;
  const int ns = n_stiff[0];
  if (j >= ns + n_stiff[1]) return;
  const size_t row = (size_t)(1 + 2 * Dp);
  const int k = list[j];
  for (int c = threadIdx.x; c < (int)row; c += blockDim.x) {
    const int d = (c == 0) ? 0 : (c <= Dp ? c - 1 : c - 1 - Dp);
    if (c != 0 && d >= D) continue;
    double s = 0.0;
    for (int p = 0; p < kSideParts; ++p) s += part[((size_t)p * kSideMaxStiff + j) * row + c];
    if (j < ns)
      stats[stat_idx(true, 0, k, c, kstride, row)] += s;
    else
      grey_stats[(size_t)(j - ns) * row + c] += s;
  }
}

// ------------------------------------------------------------------ launchers
cudaError_t launch_stiff_compact(const Ctx& c, int* gate, int* mode, cudaStream_t s) {
  prof_begin(c, KI_STIFF_COMPACT, s);
  const Workspace& w = c.ws;
  stiff_compact_kernel<<<1, 256, 0, s>>>(w.stiff, w.grey, c.K, w.Kt, w.stiff_list, w.n_stiff,
                                         w.grey_pos, w.tcraw, w.tcm, w.tcpk, w.tckf, w.lzlow,
                                         gate, mode);
  prof_end(c, KI_STIFF_COMPACT, s);
  return cudaGetLastError();
}

cudaError_t launch_side_lse(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, const int* mode, cudaStream_t s) {
  const unsigned grid = (unsigned)ceil_div64(n, 128);
  const Workspace& w = c.ws;
  const unsigned nfc = (unsigned)ceil_div64(n, 4096);
  cudaError_t e = cudaMemsetAsync(w.n_flagged, 0, sizeof(int), s);
  if (e != cudaSuccess) return e;
  prof_begin(c, KI_SIDE_LSE, s, mode, kModeTensor);
  side_flag_count_kernel<<<nfc, 256, 0, s>>>(w.side_flag, n, w.n_stiff, w.flag_cnt, w.pair_cnt,
                                             mode);
  prof_end(c, KI_SIDE_LSE, s);
  prof_begin(c, KI_SIDE_LSE, s, mode, kModeTensor);
  side_flagged_kernel<<<nfc, 256, 0, s>>>(w.side_flag, n, w.n_stiff, w.flag_cnt, w.flagged,
                                          w.n_flagged, mode);
  prof_end(c, KI_SIDE_LSE, s);
  prof_begin(c, KI_SIDE_LSE, s, mode, kModeTensor);
  if (x_dtype == FGMM_BF16)
    side_lse_kernel<<<grid, 128, 0, s>>>((const __nv_bfloat16*)X, n, ldx, c.D, w.Dp, w.mu, w.prec,
                                         w.cconst, w.stiff_list, w.n_stiff, w.logz,
                                         logz_out, w.pair_cnt, w.pair_j, w.pair_l, w.flagged,
                                         w.n_flagged, mode);
  else
    side_lse_kernel<<<grid, 128, 0, s>>>((const float*)X, n, ldx, c.D, w.Dp, w.mu, w.prec,
                                         w.cconst, w.stiff_list, w.n_stiff, w.logz,
                                         logz_out, w.pair_cnt, w.pair_j, w.pair_l, w.flagged,
                                         w.n_flagged, mode);
  prof_end(c, KI_SIDE_LSE, s);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prof_begin(c, KI_LL_PARTIALS, s, mode, kModeTensor);
  ll_partials_kernel<<<(unsigned)ceil_div64(n, 4096), 256, 0, s>>>(w.logz, n, w.ll_tiles, mode);
  prof_end(c, KI_LL_PARTIALS, s);
  return cudaGetLastError();
}

cudaError_t launch_side_stats(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s) {
  const Workspace& w = c.ws;
  dim3 grid(kSideMaxStiff, kSideParts);
  prof_begin(c, KI_SIDE_STATS, s, mode, kModeTensor);
  if (x_dtype == FGMM_BF16)
    side_stats_kernel<<<grid, 256, 0, s>>>((const __nv_bfloat16*)X, n, ldx, c.D, w.Dp, w.mu,
                                           w.prec, w.cconst, w.stiff_list, w.n_stiff, w.pair_cnt,
                                           w.pair_j, w.pair_l, w.logz, w.flagged, w.n_flagged,
                                           w.side_part, mode);
  else
    side_stats_kernel<<<grid, 256, 0, s>>>((const float*)X, n, ldx, c.D, w.Dp, w.mu, w.prec,
                                           w.cconst, w.stiff_list, w.n_stiff, w.pair_cnt,
                                           w.pair_j, w.pair_l, w.logz, w.flagged, w.n_flagged,
                                           w.side_part, mode);
  prof_end(c, KI_SIDE_STATS, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  prof_begin(c, KI_SIDE_REDUCE, s, mode, kModeTensor);
  side_reduce_kernel<<<kSideMaxStiff, 256, 0, s>>>(w.side_part, w.stiff_list, w.n_stiff, c.D,
                                                   w.Dp, w.KpS, w.stats, w.grey_stats, mode);
  prof_end(c, KI_SIDE_REDUCE, s);
  return cudaGetLastError();
}

}  // namespace fgmm
