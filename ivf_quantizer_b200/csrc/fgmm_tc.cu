// Tensor-core (tcgen05 / TMEM / TMA) kernels of the fused EM step, sm_100a.
//
// Paper: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering",
// §3.1 and Algorithm 1: per point tile, sweep 1 builds log Z_i with an online
// log-sum-exp over component blocks; sweep 2 recomputes the log-densities, forms
// r_ik = exp(log z_ik - log Z_i) and folds them into the sufficient statistics.
// The N x K responsibilities exist only as one 128 x 128 tile in TMEM / shared memory.
//
// Expanded form.  With a per-dimension centre c_d and power-of-two scale s_d,
// x^_d = (x_d - c_d) s_d and phi(x) = [x^_0 .. x^_{Dq-1}, x^_0^2 .. x^_{Dq-1}^2]:
//   log z_ik = 2^t_k * sum_j W'_kj phi_j(x_i) + c_k,
//   W_k = [ (mu_kd - c_d) / (sigma_kd^2 s_d) , -1 / (2 sigma_kd^2 s_d^2) ],  W' = W 2^-t_k,
//   c_k = log pi_k - 1/2 sum_d log(2 pi sigma_kd^2) - 1/2 sum_d (mu_kd - c_d)^2 / sigma_kd^2,
// which is §2's log pi_k + log N(x | mu_k, diag sigma_k^2) rewritten as one dot product:
// a dense contraction of K1 = 2 Dq terms per (point, component), i.e. a GEMM.
//
// Precision (FGMM_PREC_FP16X3).  Every operand a is split a = a_hi + a_lo with
// a_hi = fp16(a), a_lo = fp16(a - a_hi); the product uses three tcgen05 kind::f16
// MMAs (hi*hi + hi*lo + lo*hi) with fp32 accumulation in TMEM, about 22 significant
// bits per term.  One fp16 product (~11 bits) misses the 1e-4 log-likelihood
// tolerance on the Table-1 generator; bf16 splits (16 bits) pass with little margin.
// Statistics: r is scaled by 2^15 and rounded once to fp16 (the same rounded values
// feed N_k and the GEMM, so the weights stay consistent); phi is split hi/lo, two MMAs.
// The moments are raw (about the global centre): the variance of a component whose
// spread is small next to its distance from the centre loses accuracy to cancellation,
// which AUTO detects after the sweeps (see the M-step kernels).
//
// Kernels (one chunk of <= 2^20 points at a time):
//   tc_center     per-dimension centre and scale from the parameters
//   tc_prep       W' hi/lo, c_k, 2^t_k; conditioning check for AUTO mode
//   tc_convert    X chunk -> phi hi/lo (fp16, row-major, TMA-ready); with a
//                 permutation, the chunk in sweep-2 order (block skipping)
//   tc_lse        sweep 1: persistent, one pair of 128-point tiles per CTA at a time
//                 (each W' box feeds the products of both tiles); phi hi resident in
//                 smem, phi lo in TMEM, W' streamed through a TMA ring; S = phi W'^T in
//                 TMEM (one buffer per tile), online log-sum-exp by 16 epilogue warps
//                 (four column quarters, one row of each tile), block masks for skipping.
//   tc_stats      sweep 2: CTA owns a 128-component block (W' hi resident in smem, lo
//                 in TMEM) and a slice of points, or with block skipping a share of the
//                 block's active tiles; S^T = W' phi^T in TMEM, responsibilities
//                 written as the A operand of the second GEMM acc += R^T phi (TMEM,
//                 128 x 2Dq), flushed to the CTA's fp64 slot.
//
// Warp roles in both sweeps: warp 0 TMA producer, warp 1 MMA issuer (one thread,
// also owns the TMEM allocation), warps 4.. epilogue (warp w reads TMEM lane quarter
// w % 4): 16 epilogue warps in sweep 1, 8 in sweep 2.
// Every wait is bounded (ptx::mbar_wait); on expiry the kernel latches
// FGMM_ERR_TIMEOUT, the other roles see the abort flag, and the CTA drains and frees
// its TMEM before returning.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fgmm_internal.h"
#include "sm100_ptx.cuh"

namespace fgmm {

namespace {

constexpr int BM = 128;          // points per tile
constexpr int BKc = 128;         // components per block
constexpr int KC = 64;           // K elements per swizzle row / TMA box
constexpr int BOX = 128 * 64 * 2;  // bytes of one [128 rows][64 fp16] box
constexpr int SX = 8;            // X ring stages (sweep 2)
constexpr float kRScale = 32768.f;  // r is stored as fp16(r * 2^15)
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ void set_status(int* st, int code) { atomicCAS(st, FGMM_OK, code); }

// fp16 split of a float: hi = fp16(a) (saturating), lo = fp16(a - hi).
__device__ __forceinline__ void split16(float a, __half& hi, __half& lo) {
  hi = __float2half_rn(fminf(fmaxf(a, -65504.f), 65504.f));
  lo = __float2half_rn(a - __half2float(hi));
}

// Order in which the NKC 64-element chunks of phi enter the log-density contraction:
// the squares' chunks first, then the linear ones.  The sum ends near
// 1/2 sum_d mu~_d^2 / sigma_d^2 (the part of log z the dot product carries); taking the
// negative square terms first keeps the running fp32 accumulator about 2.5x smaller over
// the K-steps than letting the linear terms overshoot first, and each MMA step's
// rounding of the accumulator is proportional to its magnitude.
template <int NKC>
__device__ __forceinline__ int lg_chunk(int i) { return (i + NKC / 2) % NKC; }

}  // namespace

// ------------------------------------------------------------------ centre and scale
// One CTA per dimension d: c_d = sum_k pi_k mu_kd / sum_k pi_k, spread_d^2 =
// sum_k pi_k (sigma_kd^2 + (mu_kd - c_d)^2) / sum pi, s_d = 2^-round(log2 spread_d).
__global__ void tc_center_kernel(int K, int D, int cov, const float* __restrict__ w,
                                 const float* __restrict__ means, const float* __restrict__ vars,
                                 float* __restrict__ center, float* __restrict__ scale) {
  __shared__ double r0[kSimtThreads], r1[kSimtThreads];
  const int d = blockIdx.x;
  double sw = 0.0, sm = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double wk = fmax((double)w[k], 0.0);
    sw += wk;
    sm += wk * (double)means[(size_t)k * D + d];
  }
  r0[threadIdx.x] = sw;
  r1[threadIdx.x] = sm;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) { r0[threadIdx.x] += r0[threadIdx.x + s]; r1[threadIdx.x] += r1[threadIdx.x + s]; }
    __syncthreads();
  }
  const double W = r0[0];
  const double c = (W > 0.0) ? r1[0] / W : 0.0;
  __syncthreads();
  double sv = 0.0;
  for (int k = threadIdx.x; k < K; k += blockDim.x) {
    const double wk = fmax((double)w[k], 0.0);
    const double v = (cov == FGMM_COV_DIAG) ? vars[(size_t)k * D + d] : vars[k];
    const double dm = (double)means[(size_t)k * D + d] - c;
    sv += wk * (v + dm * dm);
  }
  r0[threadIdx.x] = sv;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) r0[threadIdx.x] += r0[threadIdx.x + s];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const double spread = (W > 0.0) ? sqrt(r0[0] / W) : 1.0;
    double sc = 1.0;
    if (spread > 0.0 && isfinite(spread)) sc = exp2(-rint(log2(spread)));
    center[d] = isfinite(c) ? (float)c : 0.f;
    scale[d] = (float)sc;
  }
}

// ------------------------------------------------------------------ parameter preparation
// One CTA per padded component k (grid Kt).  Writes W' = W 2^-t_k as fp16 hi/lo into
// wop[part][k][j] (part 0 hi, 1 lo; j < Dq the linear terms, Dq + d the squares),
// c_k (fp64 sums, -inf for an absent or zero-weight component) and 2^t_k.
// Stiff components (AUTO only, when `stiff` is non-null) are left to the CUDA-core
// side path: their c_k here is -inf, so the tensor-core sweeps ignore them.  A live
// component is stiff when
//   * its expanded-form logit error, ~2^-20 sqrt(sum_d t_d^2) with
//     t_d = 1.5 (|mu~| + sigma)^2 / sigma^2 (the size of the cancelling terms near
//     its mean), exceeds 1e-3 nats (a collapsed or very tight component);
//   * its variance update would cancel: A_d = 1 + mu~_d^2 / sigma_d^2 > kMaxAmplification
//     for some d;
//   * it had fewer than 4 effective points in the previous step (about to collapse).
__global__ void tc_prep_kernel(int K, int D, int Dq, int Kt, int cov,
                               const float* __restrict__ w, const float* __restrict__ means,
                               const float* __restrict__ vars, const float* __restrict__ center,
                               const float* __restrict__ scale, const double* __restrict__ nk_prev,
                               __half* __restrict__ wop, float* __restrict__ ck,
                               float* __restrict__ kscale, int* __restrict__ stiff,
                               float* __restrict__ craw, float* __restrict__ mq,
                               float* __restrict__ peak, int* __restrict__ grey,
                               float* __restrict__ ek, float assign_e, int* status) {
  __shared__ double rs[kSimtThreads], rq[kSimtThreads], rt[kSimtThreads];
  __shared__ float rmax[kSimtThreads], amax[kSimtThreads];
  __shared__ float s_pow;
  const int k = blockIdx.x;
  const int K1 = 2 * Dq;
  __half* hi = wop + (size_t)k * K1;
  __half* lo = wop + ((size_t)Kt + k) * K1;
  double slog = 0.0, squad = 0.0, stf = 0.0;
  float wmax = 0.f, amp = 0.f;
  bool bad = false;
  const bool live_k = k < K;
  // pass 1: constants, max |W|, conditioning
  for (int d = threadIdx.x; d < Dq; d += blockDim.x) {
    if (live_k && d < D) {
      const double v = (cov == FGMM_COV_DIAG) ? vars[(size_t)k * D + d] : vars[k];
      const double m = means[(size_t)k * D + d];
      if (!(v > 0.0) || !isfinite(v) || !isfinite(m)) bad = true;
      const double mt = m - (double)center[d];
      const double p = 1.0 / v;
      const double sd = scale[d];
      slog += log(2.0 * CUDART_PI * v);
      squad += mt * mt * p;
      const double a = mt * p / sd, b = -0.5 * p / (sd * sd);
      wmax = fmaxf(wmax, (float)fmax(fabs(a), fabs(b)));
      const double t = 1.5 * (fabs(mt) + sqrt(v)) * (fabs(mt) + sqrt(v)) * p;
      stf += t * t;
      amp = fmaxf(amp, (float)(1.0 + mt * mt * p));
    }
  }
  rs[threadIdx.x] = slog;
  rq[threadIdx.x] = squad;
  rt[threadIdx.x] = stf;
  rmax[threadIdx.x] = wmax;
  amax[threadIdx.x] = amp;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (threadIdx.x < s) {
      rs[threadIdx.x] += rs[threadIdx.x + s];
      rq[threadIdx.x] += rq[threadIdx.x + s];
      rt[threadIdx.x] += rt[threadIdx.x + s];
      rmax[threadIdx.x] = fmaxf(rmax[threadIdx.x], rmax[threadIdx.x + s]);
      amax[threadIdx.x] = fmaxf(amax[threadIdx.x], amax[threadIdx.x + s]);
    }
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    float c = -CUDART_INF_F;
    float pw = 1.f;
    int is_stiff = 0, is_grey = 0;
    if (live_k) {
      const float wk = w[k];
      if (!(wk >= 0.f) || !isfinite(wk)) bad = true;
      if (wk > 0.f) c = (float)(log((double)wk) - 0.5 * rs[0] - 0.5 * rq[0]);
      const float mx = rmax[0];
      if (mx > 0.f && isfinite(mx)) pw = exp2f(ceilf(log2f(mx)) - 14.f);
      const float E = (float)ldexp(sqrt(rt[0]), -20);   // bound on the logit error
      if (stiff && wk > 0.f)
        is_stiff = assign_e > 0.f
                       ? !(E <= assign_e)   // the assignment: the bound alone decides
                       : !(E <= 1e-3f) || !(amax[0] <= kMaxAmplification) ||
                             (nk_prev[k] < 4.0);
      // few points last step: the variance check may fail, so its side-path statistics
      // are taken as well (AUTO; swapped in instead of redoing the pass)
      if (stiff && wk > 0.f && !is_stiff && !(assign_e > 0.f)) is_grey = nk_prev[k] < kGreyNk;
    }
    craw[k] = c;
    // the logit-error bound of the components left on the tensor cores (assignment cut)
    ek[k] = (live_k && w[k] > 0.f && !is_stiff) ? (float)ldexp(sqrt(rt[0]), -20) : 0.f;
    mq[k] = live_k ? (float)rq[0] : 0.f;
    peak[k] = (live_k && w[k] > 0.f) ? (float)(log((double)w[k]) - 0.5 * rs[0]) : -CUDART_INF_F;
    if (stiff) {
      stiff[k] = is_stiff;
      grey[k] = is_grey;
      if (is_stiff) c = -CUDART_INF_F;
    }
    ck[k] = c;
    kscale[k] = pw;
    s_pow = pw;
  }
  __syncthreads();
  const float inv = 1.f / s_pow;
  // pass 2: write the split operand rows
  for (int j = threadIdx.x; j < K1; j += blockDim.x) {
    const int d = (j < Dq) ? j : j - Dq;
    float val = 0.f;
    if (live_k && d < D) {
      const double v = (cov == FGMM_COV_DIAG) ? vars[(size_t)k * D + d] : vars[k];
      const double m = means[(size_t)k * D + d];
      const double p = 1.0 / v;
      const double sd = scale[d];
      const double wv = (j < Dq) ? (m - (double)center[d]) * p / sd : -0.5 * p / (sd * sd);
      val = (float)wv * inv;
      if (!isfinite(val)) val = 0.f;
    }
    __half h, l;
    split16(val, h, l);
    hi[j] = h;
    lo[j] = l;
  }
  if (bad) set_status(status, FGMM_ERR_INVALID_ARG);
}

// ------------------------------------------------------------------ X -> phi (fp16 hi / lo)
// Thread per (point, group of 8 dims).  xop[part][i][j]: part 0 hi, 1 lo; j < Dq the
// scaled centred coordinate, Dq + d its square.  With perm, row i holds point perm[i].
// VEC (fp32 X, 16-byte aligned rows, D a multiple of 8): each group of 8 features is
// read as two 16-byte loads.
template <typename T, bool VEC>
__global__ void tc_convert_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dq,
                                  int64_t ncmax, const float* __restrict__ center,
                                  const float* __restrict__ scale, __half* __restrict__ xop,
                                  const int* __restrict__ perm, const int* mode) {
  if (mode && *mode != 0) return;
  const int groups = Dq / 8;
  const int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= n * groups) return;
  const int64_t i = e / groups;
  const int g = (int)(e % groups);
  const int64_t src = perm ? (int64_t)__ldg(perm + i) : i;
  const int K1 = 2 * Dq;
  __align__(16) __half xh[8], xl[8], qh[8], ql[8];
  float xr[8];
  if constexpr (VEC) {
    if (8 * g < D) {
      const float4* p = reinterpret_cast<const float4*>(reinterpret_cast<const float*>(X) +
                                                        src * ldx + 8 * g);
      const float4 a = __ldg(p), b = __ldg(p + 1);
      xr[0] = a.x; xr[1] = a.y; xr[2] = a.z; xr[3] = a.w;
      xr[4] = b.x; xr[5] = b.y; xr[6] = b.z; xr[7] = b.w;
    }
  }
#pragma unroll
  for (int u = 0; u < 8; ++u) {
    const int d = 8 * g + u;
    float xv = 0.f;
    if (d < D) {
      float x;
      if constexpr (VEC) x = xr[u];
      else if constexpr (sizeof(T) == 4) x = __ldg(reinterpret_cast<const float*>(X) + src * ldx + d);
      else x = __bfloat162float(X[src * ldx + d]);
      xv = (x - center[d]) * scale[d];
    }
    split16(xv, xh[u], xl[u]);
    split16(xv * xv, qh[u], ql[u]);
  }
  __half* hi = xop + (size_t)i * K1;
  __half* lo = xop + ((size_t)ncmax + i) * K1;
  *reinterpret_cast<uint4*>(hi + 8 * g) = *reinterpret_cast<uint4*>(xh);
  *reinterpret_cast<uint4*>(lo + 8 * g) = *reinterpret_cast<uint4*>(xl);
  *reinterpret_cast<uint4*>(hi + Dq + 8 * g) = *reinterpret_cast<uint4*>(qh);
  *reinterpret_cast<uint4*>(lo + Dq + 8 * g) = *reinterpret_cast<uint4*>(ql);
}

// ------------------------------------------------------------------ sweep 1 (log Z)
// Grid (component block b, point slice).  CTA (b, slice) keeps the W' rows of its 128
// components resident in shared memory (the hi box of every K-chunk and, with the split,
// the lo boxes) and streams the phi boxes of its slice's 128-point tiles through a TMA
// ring; S = phi W'^T of tile j goes to TMEM buffer j mod 3, so the epilogue of a tile
// overlaps the products of the next two and no tile waits for another's epilogue.  The
// nkb CTAs of one slice read the same tiles in the same order: after the first, the phi
// boxes come from L2.  With the split, three products per K-step (phi hi W' hi + phi hi
// W' lo + phi lo W' hi), each with both operands in shared memory.
// 640 threads: warp 0 TMA producer, warp 1 MMA issuer, warps 4..19 epilogue.  Epilogue
// warpgroup g reads columns 32g .. 32g+31 of a tile, one row (point) per thread, and
// reduces them to (max, sum of 2^(l - max)) in log2 units, plus the maximum of the stiff
// components' estimate + error bound; warpgroups 1..3 hand theirs to warpgroup 0 through
// tensor memory (the warps of one lane quarter share its lanes; shared memory is left to
// the phi ring), and warpgroup 0 writes the block's partial of each point.  lse_merge_kernel then
// combines the nkb partials of a point into log Z, the side-path flag and the block mask
// (exactly the blocks whose largest log-density lies within the cut of log Z).
constexpr int kEpiWarps = 8;                        // statistics sweep
constexpr int kTcThreads = 128 + 32 * kEpiWarps;
constexpr int kLseEpiWarps = 16;                    // log-sum-exp sweep
constexpr int kLseThreads = 128 + 32 * kLseEpiWarps;
constexpr int kLseSBuf = 3;                         // S buffers in TMEM (3 x 128 columns)
constexpr int kLseXcCol = 128 * kLseSBuf;           // TMEM columns of the quarters' hand-over
constexpr int kLseRingMax = 16;
constexpr int kLsePrefetch = 4;                     // tiles of L2 prefetch ahead (block 0)
constexpr int kSmemMax = 232448;                    // 227 KB of dynamic shared memory
constexpr float kCut2 = kSkipCut * kLog2e;          // the block-skipping cut in log2 units

struct LseBars {
  uint64_t w_full;
  uint64_t x_full[kLseRingMax], x_empty[kLseRingMax];
  uint64_t s_full[kLseSBuf], s_empty[kLseSBuf];
  uint64_t xc_full[2], xc_empty[2];
  uint64_t drain;
  uint32_t tmem;
  int abort;
  alignas(16) float ckl[BKc];   // the block's c_k log2(e)
  float ksl[BKc];               //             2^t_k log2(e)
  float cfl[BKc];               //             (c_k + E_k) log2(e) if stiff, else -inf
};
static_assert(offsetof(LseBars, ckl) % 16 == 0, "the staged parameters are read as float4");

// phi boxes in the ring: what shared memory the resident W' block leaves
__host__ __device__ constexpr int lse_ring(int nkc, bool split) {
  return ((kSmemMax - 1024 - (int)sizeof(LseBars)) / BOX - (split ? 2 : 1) * nkc) < kLseRingMax
             ? ((kSmemMax - 1024 - (int)sizeof(LseBars)) / BOX - (split ? 2 : 1) * nkc)
             : kLseRingMax;
}

// SPLIT: the three-product fp16 hi/lo split (FGMM_PREC_FP16X3 and AUTO); false: one fp16
// product per term (FGMM_PREC_FP16: no W' lo, no phi lo)
template <int NKC, bool SPLIT>
__global__ void __launch_bounds__(kLseThreads, 1)
    tc_lse_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                  int nc, int ncmax, int Kt, int slice_len, const float* __restrict__ ck,
                  const float* __restrict__ kscale, const float* __restrict__ ckf,
                  const __half* __restrict__ xop, float2* __restrict__ part,
                  float* __restrict__ partf, const int* mode, int* status) {
  if (mode && *mode != kModeTensor) return;
  constexpr int NP = SPLIT ? 2 : 1;                   // boxes per K-chunk (hi, lo)
  constexpr int RING = lse_ring(NKC, SPLIT);
  static_assert(RING >= 2 * NP, "the phi ring must hold two K-chunks");
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* wbuf = base;                         // [NP][NKC][BOX]: W' hi boxes, lo boxes
  unsigned char* xring = base + NP * NKC * BOX;       // [RING][BOX]
  LseBars* bars = reinterpret_cast<LseBars*>(xring + RING * BOX);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int kb = blockIdx.x;
  const int p0 = blockIdx.y * slice_len;
  const int p1 = min(nc, p0 + slice_len);
  const int ntl = p1 > p0 ? (p1 - p0 + BM - 1) / BM : 0;
  if (ntl == 0) return;  // uniform over the CTA, before any barrier or TMEM use

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->w_full, 1);
    for (int s = 0; s < RING; ++s) { ptx::mbar_init(&bars->x_full[s], 1); ptx::mbar_init(&bars->x_empty[s], 1); }
    for (int b = 0; b < kLseSBuf; ++b) {
      ptx::mbar_init(&bars->s_full[b], 1);
      ptx::mbar_init(&bars->s_empty[b], kLseEpiWarps);
    }
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bars->xc_full[b], 3 * kLseEpiWarps / 4);
      ptx::mbar_init(&bars->xc_empty[b], kLseEpiWarps / 4);
    }
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  int any_f = 0;
  for (int k = threadIdx.x; k < BKc; k += blockDim.x) {
    const int kk = kb * BKc + k;
    bars->ckl[k] = ck[kk] * kLog2e;
    bars->ksl[k] = kscale[kk] * kLog2e;
    const float f = ckf ? ckf[kk] * kLog2e : -CUDART_INF_F;
    bars->cfl[k] = f;
    any_f |= f > -CUDART_INF_F;
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  // a block without stiff components needs no filter maximum (uniform over the CTA)
  const bool has_f = __syncthreads_or(any_f) != 0;
  ptx::tc_fence_after();
  const uint32_t tmem = bars->tmem;                   // S buffer b: columns 128 b .. 128 b + 127

  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmx);
      ptx::prefetch_tmap(&tmw);
      ptx::mbar_arrive_expect_tx(&bars->w_full, NP * NKC * BOX);
      for (int part_ = 0; part_ < NP; ++part_)
        for (int c = 0; c < NKC; ++c)
          ptx::tma_load_2d(wbuf + (part_ * NKC + c) * BOX, &tmw, &bars->w_full, c * KC,
                           part_ * Kt + kb * BKc);
      uint32_t itx = 0;
      for (int j = 0; j < ntl && !*abort; ++j) {
        const int row0 = p0 + j * BM;
        // the block-0 CTA of the slice moves the phi rows of tile j + kLsePrefetch from
        // DRAM into L2, so that the slice's nkb CTAs find them there
        if (kb == 0 && j + kLsePrefetch < ntl) {
          const size_t r = (size_t)(row0 + kLsePrefetch * BM);
          for (int part_ = 0; part_ < NP; ++part_)
            ptx::bulk_prefetch_l2(xop + ((size_t)part_ * ncmax + r) * (NKC * 64),
                                  (uint32_t)BM * NKC * 128);
        }
        for (int ci = 0; ci < NKC; ++ci)
          for (int part_ = 0; part_ < NP; ++part_, ++itx) {
            const int s = itx % RING;
            if (itx >= RING && !ptx::mbar_wait(&bars->x_empty[s], ((itx / RING) - 1) & 1, abort))
              goto fail_p;
            ptx::mbar_arrive_expect_tx(&bars->x_full[s], BOX);
            ptx::tma_load_2d(xring + s * BOX, &tmx, &bars->x_full[s], lg_chunk<NKC>(ci) * KC,
                             part_ * ncmax + row0);
          }
      }
      goto done_p;
    fail_p:
      set_status(status, FGMM_ERR_TIMEOUT);
      bars->abort = 1;
    done_p:
      if (*abort) {  // let every copy this thread started land before the CTA exits
        ptx::mbar_drain(&bars->w_full, 0);
        for (uint32_t k = (itx > RING ? itx - RING : 0); k < itx; ++k)
          ptx::mbar_drain(&bars->x_full[k % RING], (k / RING) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = ptx::idesc_f16(128, 128, false, false);
      constexpr uint64_t kHiK = ptx::sw128_hi(16, 1024);
      uint32_t itx = 0;
      if (!ptx::mbar_wait(&bars->w_full, 0, abort)) goto fail_m;
      for (int j = 0; j < ntl && !*abort; ++j) {
        const int b = j % kLseSBuf;
        const uint32_t use = (uint32_t)(j / kLseSBuf);
        // S_b free: the epilogue arrives only after tcgen05.wait::ld returned, i.e. once
        // its reads of S_b are complete, and these products are issued after the arrival
        // is observed.  No tcgen05 fence here: in the issuing thread an after_thread_sync
        // fence idles the tensor pipe for several hundred cycles (the queue of issued
        // products is short), measured on B200
        if (use >= 1 && !ptx::mbar_wait(&bars->s_empty[b], (use - 1) & 1, abort)) goto fail_m;
        const uint32_t d_tmem = tmem + b * 128;
        for (int ci = 0; ci < NKC; ++ci) {
          const int c = lg_chunk<NKC>(ci);
          const int sh = itx % RING;
          if (!ptx::mbar_wait(&bars->x_full[sh], (itx / RING) & 1, abort)) goto fail_m;
          ++itx;
          int sl = sh;
          if constexpr (SPLIT) {
            sl = itx % RING;
            if (!ptx::mbar_wait(&bars->x_full[sl], (itx / RING) & 1, abort)) goto fail_m;
            ++itx;
          }
          // K-major 128 B-swizzled boxes: one descriptor per box, + 2 (32 bytes) per K-step
          const uint64_t ah0 = ptx::sw128_desc(ptx::smem_u32(xring + sh * BOX), kHiK);
          const uint64_t al0 = ptx::sw128_desc(ptx::smem_u32(xring + sl * BOX), kHiK);
          const uint64_t bh0 = ptx::sw128_desc(ptx::smem_u32(wbuf + c * BOX), kHiK);
          const uint64_t bl0 = ptx::sw128_desc(ptx::smem_u32(wbuf + (NKC + c) * BOX), kHiK);
#pragma unroll
          for (int ks = 0; ks < KC / 16; ++ks) {
            const uint64_t dk = (uint64_t)(2 * ks);
            ptx::mma_f16_ss(d_tmem, ah0 + dk, bh0 + dk, idesc, (ci > 0 || ks > 0) ? 1u : 0u);
            if constexpr (SPLIT) {
              ptx::mma_f16_ss(d_tmem, ah0 + dk, bl0 + dk, idesc, 1u);
              ptx::mma_f16_ss(d_tmem, al0 + dk, bh0 + dk, idesc, 1u);
            }
          }
          ptx::mma_commit(&bars->x_empty[sh]);
          if constexpr (SPLIT) ptx::mma_commit(&bars->x_empty[sl]);
        }
        ptx::mma_commit(&bars->s_full[b]);
      }
      goto done_m;
    fail_m:
      set_status(status, FGMM_ERR_TIMEOUT);
      bars->abort = 1;
    done_m:
      if (*abort) {  // wait for the MMAs already issued before TMEM is freed
        ptx::mma_commit(&bars->drain);
        ptx::mbar_drain(&bars->drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;         // column quarter of the S tile
    const int q = warp & 3;                // TMEM lane quarter
    const int r = q * 32 + lane;           // row of the tile = TMEM lane
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const float* ckg = bars->ckl + 32 * g;
    const float* ksg = bars->ksl + 32 * g;
    const float* cfg = bars->cfl + 32 * g;
    for (int j = 0; j < ntl && !*abort; ++j) {
      const int b = j % kLseSBuf;
      const uint32_t use = (uint32_t)(j / kLseSBuf);
      if (!ptx::mbar_wait_warp(&bars->s_full[b], use & 1, abort)) {
        set_status(status, FGMM_ERR_TIMEOUT);
        bars->abort = 1;
        break;
      }
      ptx::tc_fence_after();
      uint32_t u[32];
      ptx::tmem_ld32(tmem + lane_base + b * 128 + 32 * g, u);
      ptx::tmem_wait_ld();
      // the values are in registers: hand S_b back to the MMA warp now
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->s_empty[b]);
      // log2-scaled log-densities of the 32 columns, two per packed fp32x2 operation;
      // the maxima and sums run as four independent partial chains
      uint64_t v2[16];
      float mx[4], fx[4];
#pragma unroll
      for (int z = 0; z < 4; ++z) mx[z] = fx[z] = -CUDART_INF_F;
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const float4 cc = *reinterpret_cast<const float4*>(ckg + 4 * e4);
        const float4 kk = *reinterpret_cast<const float4*>(ksg + 4 * e4);
        const uint64_t f01 = ptx::f2_pack(__uint_as_float(u[4 * e4 + 0]), __uint_as_float(u[4 * e4 + 1]));
        const uint64_t f23 = ptx::f2_pack(__uint_as_float(u[4 * e4 + 2]), __uint_as_float(u[4 * e4 + 3]));
        const uint64_t k01 = ptx::f2_pack(kk.x, kk.y), k23 = ptx::f2_pack(kk.z, kk.w);
        v2[2 * e4 + 0] = ptx::f2_fma(f01, k01, ptx::f2_pack(cc.x, cc.y));
        v2[2 * e4 + 1] = ptx::f2_fma(f23, k23, ptx::f2_pack(cc.z, cc.w));
        float v[4];
        ptx::f2_unpack(v2[2 * e4 + 0], v[0], v[1]);
        ptx::f2_unpack(v2[2 * e4 + 1], v[2], v[3]);
        mx[e4 & 3] = fmaxf(mx[e4 & 3], fmaxf(fmaxf(v[0], v[1]), fmaxf(v[2], v[3])));
        if (has_f) {
          // stiff components (c_k = -inf above): estimate + error bound, for the filter
          const float4 cf = *reinterpret_cast<const float4*>(cfg + 4 * e4);
          float h[4];
          ptx::f2_unpack(ptx::f2_fma(f01, k01, ptx::f2_pack(cf.x, cf.y)), h[0], h[1]);
          ptx::f2_unpack(ptx::f2_fma(f23, k23, ptx::f2_pack(cf.z, cf.w)), h[2], h[3]);
          fx[e4 & 3] = fmaxf(fx[e4 & 3], fmaxf(fmaxf(h[0], h[1]), fmaxf(h[2], h[3])));
        }
      }
      const float m = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float fm = fmaxf(fmaxf(fx[0], fx[1]), fmaxf(fx[2], fx[3]));
      float s = 0.f;
      if (m > -CUDART_INF_F) {
        // every argument is <= 0 after the shift, so 2^x in (0, 1]; the SFU's exp2
        // (flushing results below 2^-126, far under fp32 resolution of the sum)
        const uint64_t shift = ptx::f2_pack(-m, -m);
        uint64_t acc[4];
#pragma unroll
        for (int z = 0; z < 4; ++z) acc[z] = ptx::f2_pack(0.f, 0.f);
#pragma unroll
        for (int e2 = 0; e2 < 16; ++e2) {
          float t0, t1;
          ptx::f2_unpack(ptx::f2_add(v2[e2], shift), t0, t1);
          acc[e2 & 3] = ptx::f2_add(acc[e2 & 3], ptx::f2_pack(ptx::ex2(t0), ptx::ex2(t1)));
        }
        float a0, a1;
        ptx::f2_unpack(ptx::f2_add(ptx::f2_add(acc[0], acc[1]), ptx::f2_add(acc[2], acc[3])), a0, a1);
        s = a0 + a1;
      }
      // the four column quarters of the row: quarters 1..3 hand theirs to quarter 0, in
      // TMEM columns kLseXcCol + 16 xb + 4 (g - 1) .. +2 of the row's lane
      const int xb = j & 1;
      const uint32_t xc_tmem = tmem + lane_base + kLseXcCol + 16 * xb;
      if (g != 0) {
        if (j >= 2 && !ptx::mbar_wait_warp(&bars->xc_empty[xb], ((j >> 1) - 1) & 1, abort)) {
          set_status(status, FGMM_ERR_TIMEOUT);
          bars->abort = 1;
          break;
        }
        ptx::tc_fence_after();
        const uint32_t w4[4] = {__float_as_uint(m), __float_as_uint(s), __float_as_uint(fm), 0u};
        ptx::tmem_st4(xc_tmem + 4 * (g - 1), w4);
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->xc_full[xb]);
      } else {
        if (!ptx::mbar_wait_warp(&bars->xc_full[xb], (j >> 1) & 1, abort)) {
          set_status(status, FGMM_ERR_TIMEOUT);
          bars->abort = 1;
          break;
        }
        ptx::tc_fence_after();
        uint32_t x16[16];
        ptx::tmem_ld16(xc_tmem, x16);
        ptx::tmem_wait_ld();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->xc_empty[xb]);
        const float mq[4] = {m, __uint_as_float(x16[0]), __uint_as_float(x16[4]), __uint_as_float(x16[8])};
        const float sq[4] = {s, __uint_as_float(x16[1]), __uint_as_float(x16[5]), __uint_as_float(x16[9])};
        const float F = fmaxf(fmaxf(fm, __uint_as_float(x16[2])),
                              fmaxf(__uint_as_float(x16[6]), __uint_as_float(x16[10])));
        const float M = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
        float S = 0.f;
        if (M > -CUDART_INF_F) {
#pragma unroll
          for (int z = 0; z < 4; ++z) S += sq[z] * ptx::ex2(mq[z] - M);
        }
        const int i = p0 + j * BM + r;
        if (i < p1) {
          part[(size_t)kb * ncmax + i] = make_float2(M, S);
          partf[(size_t)kb * ncmax + i] = F;
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// One thread per point: log Z from the nkb partials (m_b, s_b) of sweep 1 (log2 units),
// log2 Z = M + log2 sum_b s_b 2^(m_b - M) with M = max_b m_b; the side-path flag (a stiff
// component's estimate plus error bound within kSideCut nats of log Z, or log Z below
// the bound the side path relies on); and the block mask: the blocks whose largest
// log-density lies within the cut of log Z (every block when log Z is -inf).
__global__ void __launch_bounds__(256)
    lse_merge_kernel(const float2* __restrict__ part, const float* __restrict__ partf, int nc,
                     int ncmax, int nkb, float* __restrict__ logz, float* __restrict__ logz_out,
                     const float* __restrict__ lzlow, uint8_t* __restrict__ side_flag,
                     uint32_t* __restrict__ bmask, const float* __restrict__ cutp, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= nc) return;
  float M = -CUDART_INF_F, F = -CUDART_INF_F;
  for (int b = 0; b < nkb; ++b) {
    M = fmaxf(M, part[(size_t)b * ncmax + i].x);
    F = fmaxf(F, partf[(size_t)b * ncmax + i]);
  }
  float S = 0.f;
  if (M > -CUDART_INF_F)
    for (int b = 0; b < nkb; ++b) {
      const float2 v = part[(size_t)b * ncmax + i];
      if (v.x > -CUDART_INF_F) S += v.y * exp2f(v.x - M);
    }
  const float lz2 = M + log2f(S);
  const float lz = lz2 / kLog2e;
  logz[i] = lz;
  if (logz_out) logz_out[i] = lz;
  side_flag[i] = (F > lz2 - kSideCut * kLog2e) || !(lz >= *lzlow);
  if (bmask) {
    const float lim = lz2 - (cutp ? *cutp : kCut2);
    uint32_t mk = 0;
    for (int b = 0; b < nkb; ++b)
      if (part[(size_t)b * ncmax + i].x > lim) mk |= 1u << b;
    const uint32_t all = nkb >= 32 ? 0xFFFFFFFFu : (1u << nkb) - 1u;
    bmask[i] = !(lz2 > -CUDART_INF_F) ? all : mk;
  }
}

// ------------------------------------------------------------------ sweep 2 (statistics)
// 384 threads: warp 0 TMA producer (W block once, phi boxes, log Z tiles by bulk copy),
// warp 1 MMA issuer, warps 4..11 epilogue.  Epilogue warpgroup g handles points
// 64g .. 64g+63 of each tile (and, when flushing, accumulator columns g*Dq .. g*Dq+Dq-1:
// g = 0 the linear moments, g = 1 the squares).  Each statistic of the CTA's fp64 slot
// has exactly one writing thread, whose fire-and-forget reductions land in program
// order: the sums stay bitwise reproducible.
struct StatBars {
  uint64_t w_full, wlo_ready;
  uint64_t x_full[SX], x_empty[SX];
  uint64_t s_full, s_empty;
  uint64_t r_full, r_empty;
  uint64_t acc_full, acc_empty;
  uint64_t lz_full[2], lz_empty[2];
  uint64_t nk_full;
  uint64_t drain;
  uint32_t tmem;
  int abort;
  alignas(16) float lz[2][BM];   // bulk-copy destination, read as float4: 16-byte aligned
  float nkx[BKc];
};
static_assert(offsetof(StatBars, lz) % 16 == 0, "log Z tiles must be 16-byte aligned");

template <int NKC, bool SPLIT>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_stats_kernel(const __grid_constant__ CUtensorMap tmx, const __grid_constant__ CUtensorMap tmw,
                    int nc, int ncmax, int Kt, int slice_len, int flush_tiles,
                    const float* __restrict__ ck, const float* __restrict__ kscale,
                    const float* __restrict__ logz, double* __restrict__ stats, int kstride,
                    int Dp, const __half* __restrict__ wop, const int* __restrict__ tlist,
                    const int* __restrict__ tcnt, int tl_stride, int max_cta, const int* mode,
                    int* status) {
  if (mode && *mode != kModeTensor) return;
  constexpr int Dq = NKC * 32;            // features: phi has 2 Dq = NKC * 64 entries
  constexpr int NP = SPLIT ? 2 : 1;       // phi boxes per chunk (hi, lo)
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  unsigned char* base = (unsigned char*)(((uintptr_t)smem_raw + 1023) & ~(uintptr_t)1023);
  unsigned char* wbuf = base;                          // [NKC][BOX]: W' hi of the block
  unsigned char* xring = base + NKC * BOX;             // [SX][BOX]
  unsigned char* rbuf = xring + SX * BOX;              // [2][BOX]: R^T, 64 points per box
  StatBars* bars = reinterpret_cast<StatBars*>(rbuf + 2 * BOX);
  volatile int* abort = &bars->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // The CTA's component block kb, statistics slot, and point tiles: grid (block, slice)
  // with a contiguous slice of the chunk each; or (block skipping, 1-D grid of G CTAs)
  // the G CTAs shared among the blocks in proportion to their active tiles, block b
  // taking c_b = 1 + floor(n_b (G - nkb) / sum n) CTAs (none if n_b = 0, at most
  // max_cta), each an even share of b's list; tiles are 128 rows of the reordered phi.
  // The shares depend on the counts alone: every CTA derives the same ones.
  int kb = blockIdx.x, sl = blockIdx.y;
  int p0, p1, ntl, l0 = 0;
  if (tlist) {
    const int nkb = Kt / BKc;
    const int G = (int)gridDim.x;
    long long tot = 0;
    for (int b = 0; b < nkb; ++b) tot += tcnt[b];
    int before = 0, na = 0, cb = 0;
    kb = -1;
    for (int b = 0; b < nkb; ++b) {
      const int nb = tcnt[b];
      const int c = nb > 0 ? min(max_cta, 1 + (int)((long long)nb * (G - nkb) / tot)) : 0;
      if (kb < 0 && (int)blockIdx.x < before + c) { kb = b; sl = blockIdx.x - before; na = nb; cb = c; }
      before += c;
    }
    if (kb < 0) return;  // a spare CTA: uniform over the CTA, before any barrier
    const int per = (na + cb - 1) / cb;
    l0 = min(na, sl * per);
    ntl = min(na, l0 + per) - l0;
    p0 = 0;
    p1 = nc;
    tlist += (size_t)kb * tl_stride + l0;
  } else {
    p0 = blockIdx.y * slice_len;
    p1 = min(nc, p0 + slice_len);
    ntl = (p1 > p0) ? (p1 - p0 + BM - 1) / BM : 0;
  }
  if (ntl == 0) return;  // uniform over the CTA, before any barrier or TMEM use
  // first row of the CTA's tile j
  auto tile_row = [&](int j) -> int { return tlist ? __ldg(tlist + j) * BM : p0 + j * BM; };

  if (threadIdx.x == 0) {
    ptx::mbar_init(&bars->w_full, 1);
    ptx::mbar_init(&bars->wlo_ready, kEpiWarps);
    for (int s = 0; s < SX; ++s) { ptx::mbar_init(&bars->x_full[s], 1); ptx::mbar_init(&bars->x_empty[s], 1); }
    ptx::mbar_init(&bars->s_full, 1);
    ptx::mbar_init(&bars->s_empty, kEpiWarps);
    for (int b = 0; b < 2; ++b) {
      ptx::mbar_init(&bars->lz_full[b], 1);
      ptx::mbar_init(&bars->lz_empty[b], kEpiWarps);
    }
    ptx::mbar_init(&bars->r_full, kEpiWarps);
    ptx::mbar_init(&bars->r_empty, 1);
    ptx::mbar_init(&bars->acc_full, 1);
    ptx::mbar_init(&bars->acc_empty, kEpiWarps);
    ptx::mbar_init(&bars->nk_full, kEpiWarps / 2);
    ptx::mbar_init(&bars->drain, 1);
    bars->abort = 0;
    ptx::fence_mbar_init();
  }
  if (warp == 1) {
    ptx::tmem_alloc(&bars->tmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // TMEM columns: [0,128) S^T, [128, 128 + Dq) W' lo of the block (A operand of the
  // third product, two fp16 per column), [256, 256 + 2 Dq) the statistics accumulator
  const uint32_t tmem = bars->tmem;
  const uint32_t wlo_tmem = tmem + 128;
  const uint32_t acc_tmem = tmem + 256;

  // The schedule of MMA groups (and of the producer's loads) is
  //   G1(0), G1(1), G2(0), G1(2), G2(1), ..., G1(n-1), G2(n-2), G2(n-1)
  // so the epilogue's softmax of tile j overlaps G1(j+1).
  if (warp == 0) {
    if (lane == 0) {
      ptx::prefetch_tmap(&tmx);
      ptx::prefetch_tmap(&tmw);
      ptx::mbar_arrive_expect_tx(&bars->w_full, NKC * BOX);
      for (int c = 0; c < NKC; ++c)
        ptx::tma_load_2d(wbuf + c * BOX, &tmw, &bars->w_full, c * KC, kb * BKc);
      uint32_t itx = 0;
      int lz_issued = 0;
      for (int g = 0; g <= ntl && !*abort; ++g) {
        for (int which = 0; which < 2; ++which) {
          int tile;
          if (which == 0) { if (g >= ntl) continue; tile = g; }
          else { if (g == 0) continue; tile = g - 1; }
          const int row0 = tile_row(tile);
          if (which == 0) {  // log Z of the tile's points, for the epilogue
            const int lb = tile & 1;
            if (tile >= 2 &&
                !ptx::mbar_wait(&bars->lz_empty[lb], ((tile >> 1) - 1) & 1, abort)) {
              set_status(status, FGMM_ERR_TIMEOUT);
              bars->abort = 1;
              goto done_p;
            }
            ptx::mbar_arrive_expect_tx(&bars->lz_full[lb], BM * sizeof(float));
            ptx::bulk_load(bars->lz[lb], logz + row0, BM * sizeof(float), &bars->lz_full[lb]);
            lz_issued = tile + 1;
          }
          for (int ci = 0; ci < NKC; ++ci)
            for (int part = 0; part < NP; ++part, ++itx) {
              // G1 takes the chunks in the log-density order, G2 in feature order
              const int c = which == 0 ? lg_chunk<NKC>(ci) : ci;
              const int s = itx % SX;
              if (itx >= SX && !ptx::mbar_wait(&bars->x_empty[s], ((itx / SX) - 1) & 1, abort)) {
                set_status(status, FGMM_ERR_TIMEOUT);
                bars->abort = 1;
                goto done_p;
              }
              ptx::mbar_arrive_expect_tx(&bars->x_full[s], BOX);
              ptx::tma_load_2d(xring + s * BOX, &tmx, &bars->x_full[s], c * KC,
                               part * ncmax + row0);
            }
        }
      }
    done_p:
      if (*abort) {  // let every copy this thread started land before the CTA exits
        ptx::mbar_drain(&bars->w_full, 0);
        for (uint32_t k = (itx > SX ? itx - SX : 0); k < itx; ++k)
          ptx::mbar_drain(&bars->x_full[k % SX], (k / SX) & 1);
        for (int t = (lz_issued > 2 ? lz_issued - 2 : 0); t < lz_issued; ++t)
          ptx::mbar_drain(&bars->lz_full[t & 1], (t >> 1) & 1);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc1 = ptx::idesc_f16(128, 128, false, false);  // S^T = W phi^T
      uint32_t itx = 0;
      int tiles_since_flush = 0;
      bool fresh = true;   // next G2 starts a new accumulation period
      int flushes = 0;
      if (!ptx::mbar_wait(&bars->w_full, 0, abort)) goto fail_m;
      if (SPLIT && !ptx::mbar_wait(&bars->wlo_ready, 0, abort)) goto fail_m;
      for (int g = 0; g <= ntl && !*abort; ++g) {
        if (g < ntl) {  // ---- G1(g): S^T is single-buffered, released once loaded
          if (g >= 1 && !ptx::mbar_wait(&bars->s_empty, (g - 1) & 1, abort)) goto fail_m;
          ptx::tc_fence_after();
          const uint32_t d_tmem = tmem;
          for (int ci = 0; ci < NKC; ++ci) {
            const int c = lg_chunk<NKC>(ci);
            const int sh = itx % SX;
            if (!ptx::mbar_wait(&bars->x_full[sh], (itx / SX) & 1, abort)) goto fail_m;
            ++itx;
            int sl = sh;
            if constexpr (SPLIT) {
              sl = itx % SX;
              if (!ptx::mbar_wait(&bars->x_full[sl], (itx / SX) & 1, abort)) goto fail_m;
              ++itx;
            }
            // (TMA arrivals: no tcgen05 fence needed; the one after s_empty orders the
            // epilogue's reads of S^T ahead of these products)
            // K-major boxes: one descriptor per box, + 2 (32 bytes) per K-step
            constexpr uint64_t kHiK = ptx::sw128_hi(16, 1024);
            const uint64_t ah0 = ptx::sw128_desc(ptx::smem_u32(wbuf + c * BOX), kHiK);
            const uint64_t bh0 = ptx::sw128_desc(ptx::smem_u32(xring + sh * BOX), kHiK);
            const uint64_t bl0 = ptx::sw128_desc(ptx::smem_u32(xring + sl * BOX), kHiK);
            // W' lo from TMEM: K elements c*64 + ks*16 .. +15 = columns c*32 + ks*8 .. +7
            const uint32_t wl_tmem = wlo_tmem + c * 32;
#pragma unroll
            for (int ks = 0; ks < KC / 16; ++ks) {
              const uint64_t dk = (uint64_t)(2 * ks);
              ptx::mma_f16_ss(d_tmem, ah0 + dk, bh0 + dk, idesc1, (ci > 0 || ks > 0) ? 1u : 0u);
              if constexpr (SPLIT) {
                ptx::mma_f16_ss(d_tmem, ah0 + dk, bl0 + dk, idesc1, 1u);
                ptx::mma_f16_ts(d_tmem, wl_tmem + ks * 8, bh0 + dk, idesc1, 1u);
              }
            }
            ptx::mma_commit(&bars->x_empty[sh]);
            if constexpr (SPLIT) ptx::mma_commit(&bars->x_empty[sl]);
          }
          ptx::mma_commit(&bars->s_full);
        }
        if (g >= 1) {  // ---- G2(g-1)
          const int tile = g - 1;
          if (!ptx::mbar_wait(&bars->r_full, tile & 1, abort)) goto fail_m;
          if (fresh && flushes > 0 && !ptx::mbar_wait(&bars->acc_empty, (flushes - 1) & 1, abort))
            goto fail_m;
          ptx::tc_fence_after();
          const uint32_t r0 = ptx::smem_u32(rbuf);
          // A phase's phi boxes sit in ring slots hi(0), lo(0), hi(1), lo(1), ... (hi(0),
          // hi(1), ... with one product); when the ring holds a whole number of phases,
          // every phase starts at a multiple of its size, its hi boxes are NP slots apart
          // without wrapping, and one MMA with N = 64 NKC features (leading byte offset
          // NP BOX between the 64-feature atoms) covers all chunks.
          constexpr int CP = (SX % (NP * NKC) == 0) ? NKC : 1;
          constexpr uint32_t idesc2 = ptx::idesc_f16(128, 64 * CP, false, true);
          for (int c = 0; c < NKC; c += CP) {
            const uint32_t it0 = itx;
            for (int i = 0; i < NP * CP; ++i, ++itx)
              if (!ptx::mbar_wait(&bars->x_full[itx % SX], (itx / SX) & 1, abort)) goto fail_m;
            const uint32_t d_tmem = acc_tmem + c * 64;
            constexpr uint64_t kHiA = ptx::sw128_hi(16, 1024);
            constexpr uint64_t kHiB = ptx::sw128_hi(NP * BOX, 1024);
            const uint64_t a0 = ptx::sw128_desc(r0, kHiA);
            const uint64_t bh0 = ptx::sw128_desc(ptx::smem_u32(xring + (it0 % SX) * BOX), kHiB);
            const uint64_t bl0 = ptx::sw128_desc(ptx::smem_u32(xring + ((it0 + 1) % SX) * BOX), kHiB);
#pragma unroll
            for (int ks = 0; ks < BM / 16; ++ks) {
              // A = R^T (K-major, K = points): box ks/4, 32 B per 16 points inside it
              const uint64_t a = a0 + (uint64_t)((((ks >> 2) * BOX) + (ks & 3) * 32) >> 4);
              // B = phi (MN-major, K = points = rows): 16 rows = 2 atoms of 1024 B
              const uint64_t db = (uint64_t)(ks * (2048 >> 4));
              ptx::mma_f16_ss(d_tmem, a, bh0 + db, idesc2, (fresh && ks == 0) ? 0u : 1u);
              if constexpr (SPLIT) ptx::mma_f16_ss(d_tmem, a, bl0 + db, idesc2, 1u);
            }
            for (uint32_t i = it0; i < itx; ++i) ptx::mma_commit(&bars->x_empty[i % SX]);
          }
          ptx::mma_commit(&bars->r_empty);
          fresh = false;
          if (++tiles_since_flush == flush_tiles || tile == ntl - 1) {
            ptx::mma_commit(&bars->acc_full);
            tiles_since_flush = 0;
            fresh = true;
            ++flushes;
          }
        }
      }
      goto done_m;
    fail_m:
      set_status(status, FGMM_ERR_TIMEOUT);
      bars->abort = 1;
    done_m:
      if (*abort) {  // wait for the MMAs already issued before TMEM is freed
        ptx::mma_commit(&bars->drain);
        ptx::mbar_drain(&bars->drain, 0);
      }
    }
  } else if (warp >= 4) {
    const int g = (warp - 4) >> 2;            // point half of each tile / moment half of acc
    const int q = warp & 3;
    const int kl = q * 32 + lane;             // component within the block = TMEM lane
    const int k = kb * BKc + kl;
    // log2(e)-scaled epilogue constants; fp16(r 2^15) = exp2(v ksl + ckl - log Z log2(e))
    const float ksl = kscale[k] * kLog2e;
    const float ckl = ck[k] * kLog2e + 15.f;
    const uint32_t lane_base = (uint32_t)(q * 32) << 16;
    const size_t row = (size_t)(1 + 2 * Dp);
    // this CTA's slot, [row][kstride] layout: statistic c of component k at c * kstride + k
    double* slot = stats + stat_idx(true, sl, k, 0, kstride, row);
    float nk = 0.f;
    int tiles_since_flush = 0, flushes = 0;
    // R^T row kl, points 64g .. 64g+63 = box g: 8-row atoms of 1024 B, 128 B per row,
    // 16-byte units XOR-swizzled by (row & 7).
    unsigned char* rrow = rbuf + g * BOX + (kl >> 3) * 1024 + (kl & 7) * 128;
    // W' lo of this component into TMEM (the third product's A operand): this
    // warpgroup writes K elements g*Dq .. g*Dq+Dq-1 = columns g*Dq/2 .. +Dq/2-1
    if constexpr (SPLIT) {
      const uint4* src = reinterpret_cast<const uint4*>(wop + ((size_t)Kt + k) * (2 * Dq) + g * Dq);
#pragma unroll 1
      for (int c8 = 0; c8 < Dq / 16; ++c8) {   // 8 columns = 16 fp16 per store
        const uint4 v0 = __ldg(src + 2 * c8), v1 = __ldg(src + 2 * c8 + 1);
        const uint32_t r8[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
        ptx::tmem_st8(wlo_tmem + lane_base + g * (Dq / 2) + c8 * 8, r8);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->wlo_ready);
    }
    for (int tile = 0; tile < ntl && !*abort; ++tile) {
      const int row0 = tile_row(tile);
      const int b = tile & 1;
      const int nvalid = p1 - row0;            // points of this tile inside the slice
      if (!ptx::mbar_wait_warp(&bars->s_full, tile & 1, abort))
        goto fail_e;
      if (!ptx::mbar_wait_warp(&bars->lz_full[b], (tile >> 1) & 1, abort))
        goto fail_e;
      ptx::tc_fence_after();
      // load this warpgroup's 64 columns of S^T, then free the buffer for G1(tile + 1)
      uint32_t u[2][32];
      ptx::tmem_ld32(tmem + lane_base + 64 * g, u[0]);
      ptx::tmem_ld32(tmem + lane_base + 64 * g + 32, u[1]);
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(&bars->s_empty);
      const float* lzt = bars->lz[b];
      uint32_t pk[2][16];
      // t = log2(r 2^15) = S ksl + (ckl - log Z log2(e)), two points per packed operation;
      // r <= 1 up to rounding, and the clamp keeps fp16(r 2^15) finite even where the two
      // sweeps' roundings disagree.  Rows past the tile's points get r = 0.
      const uint64_t ksl2 = ptx::f2_pack(ksl, ksl), ckl2 = ptx::f2_pack(ckl, ckl);
      const uint64_t nl2e = ptx::f2_pack(-kLog2e, -kLog2e);
      const bool full = nvalid >= BM;
      uint64_t nk2 = ptx::f2_pack(0.f, 0.f);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const int pb = 64 * g + 32 * h;        // first point of this 32-column group
#pragma unroll
        for (int e = 0; e < 32; e += 4) {
          const float4 lz4 = *reinterpret_cast<const float4*>(lzt + pb + e);
          float t[4];
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(u[h][e]), __uint_as_float(u[h][e + 1])),
                                     ksl2, ptx::f2_fma(ptx::f2_pack(lz4.x, lz4.y), nl2e, ckl2)),
                         t[0], t[1]);
          ptx::f2_unpack(ptx::f2_fma(ptx::f2_pack(__uint_as_float(u[h][e + 2]), __uint_as_float(u[h][e + 3])),
                                     ksl2, ptx::f2_fma(ptx::f2_pack(lz4.z, lz4.w), nl2e, ckl2)),
                         t[2], t[3]);
          float rr[4];
#pragma unroll
          for (int z = 0; z < 4; ++z)
            rr[z] = ptx::ex2((full || pb + e + z < nvalid) ? fminf(t[z], 15.f) : -CUDART_INF_F);
          const __half2 h01 = __floats2half2_rn(rr[0], rr[1]);
          const __half2 h23 = __floats2half2_rn(rr[2], rr[3]);
          const float2 f01 = __half22float2(h01), f23 = __half22float2(h23);
          nk2 = ptx::f2_add(nk2, ptx::f2_add(ptx::f2_pack(f01.x, f01.y), ptx::f2_pack(f23.x, f23.y)));
          pk[h][e >> 1] = *reinterpret_cast<const uint32_t*>(&h01);
          pk[h][(e >> 1) + 1] = *reinterpret_cast<const uint32_t*>(&h23);
        }
      }
      {
        float n0, n1;
        ptx::f2_unpack(nk2, n0, n1);
        nk += n0 + n1;
      }
      // R^T of the previous tile must have been consumed by G2 before it is overwritten
      if (tile >= 1 &&
          !ptx::mbar_wait_warp(&bars->r_empty, (tile - 1) & 1, abort))
        goto fail_e;
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          const int unit = (h * 4 + uu) ^ (kl & 7);
          *reinterpret_cast<uint4*>(rrow + unit * 16) =
              make_uint4(pk[h][uu * 4], pk[h][uu * 4 + 1], pk[h][uu * 4 + 2], pk[h][uu * 4 + 3]);
        }
      ptx::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        ptx::mbar_arrive(&bars->lz_empty[b]);
        ptx::mbar_arrive(&bars->r_full);
      }
      if (++tiles_since_flush == flush_tiles || tile == ntl - 1) {
        if (!ptx::mbar_wait_warp(&bars->acc_full, flushes & 1, abort))
          goto fail_e;
        ptx::tc_fence_after();
        const double inv = 1.0 / (double)kRScale;
        // g 0: linear moments, g 1: squares; the warp's 32 lanes (components) add into
        // 32 consecutive doubles per statistic
        double* dst = slot + (size_t)(1 + (g == 0 ? 0 : Dp)) * kstride;
#pragma unroll 1
        for (int h = 0; h < NKC; ++h) {
          uint32_t u[32];
          ptx::tmem_ld32(acc_tmem + lane_base + g * Dq + h * 32, u);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e)
            atomicAdd(dst + (size_t)(h * 32 + e) * kstride, (double)__uint_as_float(u[e]) * inv);
        }
        // N_k: the upper half hands its partial sum to the lower half
        if (g == 1) {
          bars->nkx[kl] = nk;
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(&bars->nk_full);
        } else {
          if (!ptx::mbar_wait_warp(&bars->nk_full, flushes & 1, abort))
            goto fail_e;
          atomicAdd(slot, ((double)nk + (double)bars->nkx[kl]) * inv);
        }
        nk = 0.f;
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(&bars->acc_empty);
        tiles_since_flush = 0;
        ++flushes;
      }
    }
    goto done_e;
  fail_e:
    set_status(status, FGMM_ERR_TIMEOUT);
    bars->abort = 1;
  done_e:;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    ptx::tc_fence_after();
    ptx::tmem_dealloc(tmem, 512);
  }
}

// ------------------------------------------------------------------ bounded-wait self-test
// One thread initialises an mbarrier expecting one arrival that never comes and
// waits on it through the same bounded wait as the sweeps.
__global__ void bounded_wait_probe_kernel(uint64_t limit_ns, int* status) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    ptx::mbar_init(&bar, 1);
    abort_flag = 0;
    ptx::fence_mbar_init();
    const bool ok = ptx::mbar_wait(&bar, 0, &abort_flag, limit_ns);
    *status = ok ? FGMM_OK : FGMM_ERR_TIMEOUT;
  }
}

cudaError_t run_bounded_wait_probe(int64_t limit_ns, int* status_host) {
  int* d = nullptr;
  cudaError_t e = cudaMalloc(&d, sizeof(int));
  if (e != cudaSuccess) return e;
  bounded_wait_probe_kernel<<<1, 32>>>((uint64_t)limit_ns, d);
  e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(status_host, d, sizeof(int), cudaMemcpyDeviceToHost);
  cudaFree(d);
  return e;
}

// ------------------------------------------------------------------ host side
namespace {

// The driver's tensor-map encoder, fetched through the runtime so that the library
// does not link libcuda (it must load on hosts without a driver).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

bool make_tmap(CUtensorMap* m, const void* ptr, uint64_t inner, uint64_t rows) {
  EncodeTiledFn enc = encode_tiled();
  if (!enc) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
                                      const_cast<void*>(ptr), dims, strides, box, estr,
                                      CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                                      CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                                      CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

size_t lse_smem(int nkc, bool split) {
  return 1024 + (size_t)((split ? 2 : 1) * nkc + lse_ring(nkc, split)) * BOX + sizeof(LseBars);
}
size_t stats_smem(int nkc) { return 1024 + (size_t)(nkc + SX + 2) * BOX + sizeof(StatBars); }

template <int NKC, bool SPLIT>
cudaError_t set_attrs_split() {
  static_assert(1024 + ((SPLIT ? 2 : 1) * NKC + lse_ring(NKC, SPLIT)) * BOX + sizeof(LseBars) <=
                    (size_t)kSmemMax, "sweep 1 exceeds the shared memory of a block");
  cudaError_t e = cudaFuncSetAttribute(tc_lse_kernel<NKC, SPLIT>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)lse_smem(NKC, SPLIT));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(tc_stats_kernel<NKC, SPLIT>,
                              cudaFuncAttributeMaxDynamicSharedMemorySize, (int)stats_smem(NKC));
}
template <int NKC>
cudaError_t set_attrs() {
  cudaError_t e = set_attrs_split<NKC, true>();
  return e != cudaSuccess ? e : set_attrs_split<NKC, false>();
}

}  // namespace

bool tc_supported(const Ctx& c) { return round_up(c.D, 32) <= 128; }

cudaError_t tc_init(Ctx& c) {
  if (!tc_supported(c)) return cudaSuccess;
  const int nkc = round_up(c.D, 32) / 32;
  cudaError_t e = cudaSuccess;
  switch (nkc) {
    case 1: e = set_attrs<1>(); break;
    case 2: e = set_attrs<2>(); break;
    case 3: e = set_attrs<3>(); break;
    default: e = set_attrs<4>(); break;
  }
  if (e != cudaSuccess) return e;
  const Workspace& w = c.ws;
  c.tc.ready = false;
  if (!make_tmap(&c.tc.tmap_x, w.xop, (uint64_t)w.K1, (uint64_t)2 * kChunk) ||
      !make_tmap(&c.tc.tmap_w, w.wop, (uint64_t)w.K1, (uint64_t)2 * w.Kt))
    return cudaErrorInvalidValue;
  c.tc.ready = true;
  return cudaSuccess;
}

// One CTA: the marked components in increasing order, padded with component 0 to a
// multiple of 64 (the exact assignment reads 64 list entries at a time).
__global__ void assign_list_kernel(const int* __restrict__ stiff, int K, int* __restrict__ list,
                                   int* __restrict__ nlist) {
  __shared__ int wsum[32];
  __shared__ int base;
  if (threadIdx.x == 0) base = 0;
  __syncthreads();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  for (int k0 = 0; k0 < K; k0 += blockDim.x) {
    const int k = k0 + (int)threadIdx.x;
    const bool f = k < K && stiff[k];
    const unsigned ball = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[warp] = __popc(ball);
    __syncthreads();
    int before = 0, tot = 0;
    for (int w2 = 0; w2 < nw; ++w2) {
      before += w2 < warp ? wsum[w2] : 0;
      tot += wsum[w2];
    }
    if (f) list[base + before + __popc(ball & ((1u << lane) - 1u))] = k;
    __syncthreads();
    if (threadIdx.x == 0) base += tot;
    __syncthreads();
  }
  const int n = base;
  for (int j = n + (int)threadIdx.x; j < (n + 63) / 64 * 64; j += blockDim.x) list[j] = 0;
  if (threadIdx.x == 0) *nlist = n;
}

cudaError_t launch_tc_prep(const Ctx& c, const float* weights, const float* means,
                           const float* vars, bool auto_mode, cudaStream_t s, bool assign) {
  const Workspace& w = c.ws;
  prof_begin(c, KI_TC_CENTER, s);
  tc_center_kernel<<<c.D, kSimtThreads, 0, s>>>(c.K, c.D, c.cov, weights, means, vars, w.center,
                                                w.dscale);
  prof_end(c, KI_TC_CENTER, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (w.Dq > c.D) cudaMemsetAsync(w.center + c.D, 0, (w.Dq - c.D) * sizeof(float), s);
  const bool mark = auto_mode || assign;
  if (!mark) {
    cudaMemsetAsync(w.stiff, 0, w.Kt * sizeof(int), s);
    cudaMemsetAsync(w.grey, 0, w.Kt * sizeof(int), s);
  }
  prof_begin(c, KI_TC_PREP, s);
  tc_prep_kernel<<<w.Kt, kSimtThreads, 0, s>>>(c.K, c.D, w.Dq, w.Kt, c.cov, weights, means, vars,
                                               w.center, w.dscale, w.nk, w.wop, w.tck, w.tks,
                                               mark ? w.stiff : nullptr, w.tcraw, w.tcm,
                                               w.tcpk, w.grey, w.tce,
                                               assign ? kAssignMaxE : -1.f, w.status);
  prof_end(c, KI_TC_PREP, s);
  if (assign) {
    assign_list_kernel<<<1, 1024, 0, s>>>(w.stiff, c.K, w.alist, w.nalist);
  }
  return cudaGetLastError();
}

cudaError_t launch_tc_convert(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* perm, const int* mode, cudaStream_t s) {
  const Workspace& w = c.ws;
  const int64_t total = n * (w.Dq / 8);
  const unsigned grid = (unsigned)ceil_div64(total, 256);
  const KernelId id = perm ? KI_TC_GATHER : KI_TC_CONVERT;
  prof_begin(c, id, s, mode, kModeTensor);
  const bool vec = x_dtype == FGMM_F32 && (uintptr_t)X % 16 == 0 && ldx % 4 == 0 && c.D % 8 == 0;
  if (x_dtype == FGMM_BF16)
    tc_convert_kernel<__nv_bfloat16, false><<<grid, 256, 0, s>>>(
        (const __nv_bfloat16*)X, n, ldx, c.D, w.Dq, kChunk, w.center, w.dscale, w.xop, perm, mode);
  else if (vec)
    tc_convert_kernel<float, true><<<grid, 256, 0, s>>>((const float*)X, n, ldx, c.D, w.Dq, kChunk,
                                                        w.center, w.dscale, w.xop, perm, mode);
  else
    tc_convert_kernel<float, false><<<grid, 256, 0, s>>>((const float*)X, n, ldx, c.D, w.Dq,
                                                         kChunk, w.center, w.dscale, w.xop, perm,
                                                         mode);
  prof_end(c, id, s);
  return cudaGetLastError();
}

// One CTA: cut2 = (base + 8 max_k E_k + 0.5) log2(e); a non-finite bound gives an
// unbounded cut (every block marked: the exact evaluation then visits all of them).
__global__ void assign_cut_kernel(const float* __restrict__ ek, int Kt, float base,
                                  float* __restrict__ cut2) {
  __shared__ float red[kSimtThreads];
  float m = 0.f;
  for (int k = threadIdx.x; k < Kt; k += blockDim.x) m = fmaxf(m, isfinite(ek[k]) ? ek[k] : CUDART_INF_F);
  red[threadIdx.x] = m;
  __syncthreads();
  for (int w = blockDim.x / 2; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const float c = (base + 8.f * red[0] + 0.5f) * kLog2e;
    *cut2 = isfinite(c) ? c : 1e30f;
  }
}

cudaError_t launch_assign_cut(const Ctx& c, float base_nats, cudaStream_t s) {
  assign_cut_kernel<<<1, kSimtThreads, 0, s>>>(c.ws.tce, c.ws.Kt, base_nats, c.ws.acut);
  return cudaGetLastError();
}

bool tc_skip(const Ctx& c) {
  const int nkb = c.ws.Kt / BKc;
  return c.skip && c.tc.ready && c.ws.bmask && nkb >= 2 && nkb <= kSkipMaxBlocks;
}

cudaError_t launch_tc_lse(const Ctx& c, int64_t n, float* logz_out, const int* mode,
                          cudaStream_t s, bool assign) {
  const Workspace& w = c.ws;
  const int nkc = w.K1 / 64;
  const int nkb = w.Kt / BKc;
  // grid (component block, point slice), as many slices as fill the SMs once
  int S = c.num_sms / nkb;
  if (S < 1) S = 1;
  const int slice = (int)ceil_div64(ceil_div64(n, S), BM) * BM;
  const dim3 grid(nkb, S);
  const CUtensorMap& tx = c.tc.tmap_x;
  const CUtensorMap& tw = c.tc.tmap_w;
  const bool split = c.prec != FGMM_PREC_FP16;
  const size_t smem = lse_smem(nkc, split);
  uint32_t* bm = (assign || tc_skip(c)) ? w.bmask : nullptr;
  const float* cutp = assign ? w.acut : nullptr;
  const float* ckf = assign ? nullptr : w.tckf;   // the assignment has no side path
  prof_begin(c, KI_TC_LSE, s, mode, kModeTensor);
#define LSE_CASE(N_)                                                                          \
  case N_:                                                                                    \
    if (split)                                                                                \
      tc_lse_kernel<N_, true><<<grid, kLseThreads, smem, s>>>(                                \
          tx, tw, (int)n, (int)kChunk, w.Kt, slice, w.tck, w.tks, ckf, w.xop, w.lpart,       \
          w.lpartf, mode, w.status);                                                          \
    else                                                                                      \
      tc_lse_kernel<N_, false><<<grid, kLseThreads, smem, s>>>(                               \
          tx, tw, (int)n, (int)kChunk, w.Kt, slice, w.tck, w.tks, ckf, w.xop, w.lpart,       \
          w.lpartf, mode, w.status);                                                          \
    break;
  switch (nkc) {
    LSE_CASE(1)
    LSE_CASE(2)
    LSE_CASE(3)
    LSE_CASE(4)
  }
#undef LSE_CASE
  // the merge of the blocks' partials: a second launch inside the same profiled region
  prof_extra_launch(c);
  lse_merge_kernel<<<(unsigned)ceil_div64(n, 256), 256, 0, s>>>(
      w.lpart, w.lpartf, (int)n, (int)kChunk, nkb, w.logz, logz_out, w.lzlow, w.side_flag, bm,
      cutp, mode);
  prof_end(c, KI_TC_LSE, s);
  return cudaGetLastError();
}

int tc_stat_slots(const Ctx& c) {
  const int S2 = 2 * tc_slices(c);
  return S2 < c.ws.slots ? S2 : c.ws.slots;
}

int tc_slices(const Ctx& c) {
  const int nkb = c.ws.Kt / BKc;
  int S = c.num_sms / nkb;
  if (S < 1) S = 1;
  if (S > c.ws.slots) S = c.ws.slots;
  return S;
}

cudaError_t launch_tc_stats(const Ctx& c, int64_t n, const int* mode, cudaStream_t s) {
  const Workspace& w = c.ws;
  const int nkc = w.K1 / 64;
  const int S = tc_slices(c);
  int slice = (int)ceil_div64(ceil_div64(n, S), BM) * BM;
  const bool skip = tc_skip(c);
  // block skipping: a 1-D grid of the same size, shared among the blocks by their work
  const dim3 grid = skip ? dim3((w.Kt / BKc) * S, 1) : dim3(w.Kt / BKc, S);
  const CUtensorMap& tx = c.tc.tmap_x;
  const CUtensorMap& tw = c.tc.tmap_w;
  // fp32 runs (in tiles of 128 points) between fp64 flushes of the statistics
  const int flush_tiles = skip ? kFlushTilesSkip : kFlushTilesDense;
  // block skipping: phi and log Z were rewritten in sweep-2 order, tiles come from lists
  const float* lz = skip ? w.lzp : w.logz;
  const int* tl = skip ? w.tlist : nullptr;
  const int tl_stride = (int)(kChunk / BM);
  const bool split = c.prec != FGMM_PREC_FP16;
  prof_begin(c, KI_TC_STATS, s, mode, kModeTensor);
#define STATS_CASE(N_)                                                                         \
  case N_:                                                                                     \
    if (split)                                                                                 \
      tc_stats_kernel<N_, true><<<grid, kTcThreads, stats_smem(N_), s>>>(                      \
          tx, tw, (int)n, (int)kChunk, w.Kt, slice, flush_tiles, w.tck, w.tks, lz, w.stats,    \
          w.KpS, w.Dp, w.wop, tl, w.tcnt, tl_stride, tc_stat_slots(c), mode, w.status);        \
    else                                                                                       \
      tc_stats_kernel<N_, false><<<grid, kTcThreads, stats_smem(N_), s>>>(                     \
          tx, tw, (int)n, (int)kChunk, w.Kt, slice, flush_tiles, w.tck, w.tks, lz, w.stats,    \
          w.KpS, w.Dp, w.wop, tl, w.tcnt, tl_stride, tc_stat_slots(c), mode, w.status);        \
    break;
  switch (nkc) {
    STATS_CASE(1)
    STATS_CASE(2)
    STATS_CASE(3)
    STATS_CASE(4)
  }
#undef STATS_CASE
  prof_end(c, KI_TC_STATS, s);
  return cudaGetLastError();
}

}  // namespace fgmm
