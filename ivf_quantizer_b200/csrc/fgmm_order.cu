// Block skipping in the statistics sweep: the point order of sweep 2 (both paths).
//
// Paper: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", §3.1 and
// Algorithm 1.  Sweep 2 forms r_ik = exp(log z_ik - log Z_i) for every point and every
// component and folds them into N_k, sum r x, sum r x^2.  The tensor-core version keeps
// r as fp16(r 2^15), exactly 0 for a log-density more than 27.7 nats below log Z, so a
// (128-point tile, 128-component block) pair in which that holds for every pair adds
// exactly nothing.  Sweep 1 records, per point, the blocks that come within kSkipCut of
// log Z (a bit mask).  The kernels here
//   order_count / order_scan / order_scatter
//                 a stable LSD radix sort of the chunk's points by their 32-bit block
//                 mask, 8 bits per pass (one pass up to 8 blocks, four for 32), so that
//                 points with the same set of blocks become neighbours;
//   tile_mask     per tile of the sorted order, the OR of its points' masks, and log Z
//                 in the sorted order;
//   block_list    per component block, the tiles whose mask holds it, in increasing order.
// Between scatter and tile_mask, tc_convert rewrites phi(x) in the sorted order.  Sweep 2
// then runs each block over its own list.  Every step is deterministic (counts, prefix
// sums, ordered scatter), so the sums stay bitwise reproducible from run to run; they
// differ from the natural order only by the order of fp32 additions.
//
// The CUDA-core path uses the same sort and lists with 64-point tiles: simt_mask builds
// the masks from sweep 1's per-64-component maxima against log Z - kSimtSkipCut (its fp32
// statistics keep r down to e^-104, so there the cut is set for r < 2e-22 instead), and
// its statistics sweep reads X through the permutation instead of a converted copy.
#include <math_constants.h>

#include "fgmm_internal.h"

namespace fgmm {

namespace {

constexpr int kOrdThreads = 256;
static_assert(kOrdThreads == kOrdBuckets, "one thread per digit value");
static_assert(FGMM_CHUNK_POINTS / kOrdPts <= kOrdThreads, "one scan thread per counting CTA");
constexpr int kTileRows = 128;
constexpr int kListThreads = 1024;

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t r;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(r));
  return r;
}

// Counts of each digit value among the kOrdPts points of this CTA (positions
// [c kOrdPts, (c + 1) kOrdPts) of the current order: point in[j], or j without `in`).
__global__ void order_count_kernel(const uint32_t* __restrict__ bmask, const int* __restrict__ in,
                                   int n, int shift, int* __restrict__ hist, const int* mode,
                                   int required) {
  if (mode && *mode != required) return;
  __shared__ int cnt[kOrdBuckets];
  for (int b = threadIdx.x; b < kOrdBuckets; b += blockDim.x) cnt[b] = 0;
  __syncthreads();
  const int j0 = blockIdx.x * kOrdPts;
  for (int j = threadIdx.x; j < kOrdPts; j += blockDim.x) {
    const int jj = j0 + j;
    if (jj < n) atomicAdd(&cnt[(bmask[in ? in[jj] : jj] >> shift) & (kOrdBuckets - 1)], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < kOrdBuckets; b += blockDim.x)
    hist[(size_t)b * gridDim.x + blockIdx.x] = cnt[b];   // digit-major: the scan order
}

// Exclusive prefix sum over the 256 threads of a CTA (kOrdThreads == kOrdBuckets);
// `tot` receives the sum.  `ws` holds 8 ints of shared memory.
__device__ __forceinline__ int block_exclusive_scan(int v, int* ws, int* tot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += u;
  }
  if (lane == 31) ws[warp] = x;
  __syncthreads();
  int before = 0, all = 0;
#pragma unroll
  for (int w2 = 0; w2 < kOrdThreads / 32; ++w2) {
    const int t = ws[w2];
    before += w2 < warp ? t : 0;
    all += t;
  }
  __syncthreads();   // ws may be reused by the caller
  *tot = all;
  return before + x - v;
}

// CTA per digit value b: hist[b][c] (counts of CTA c, digit-major) -> exclusive prefix
// over c, and the digit's total in dtot[b].
__global__ void __launch_bounds__(kOrdThreads)
    order_scan_kernel(int* __restrict__ hist, int ncta, int* __restrict__ dtot, const int* mode,
                      int required) {
  if (mode && *mode != required) return;
  __shared__ int ws[kOrdThreads / 32];
  const int b = blockIdx.x, c = threadIdx.x;   // ncta <= kOrdThreads
  int* row = hist + (size_t)b * ncta;
  const int v = c < ncta ? row[c] : 0;
  int tot;
  const int ex = block_exclusive_scan(v, ws, &tot);
  if (c < ncta) row[c] = ex;
  if (c == 0) dtot[b] = tot;
}

// Stable scatter of one radix pass: CTA c walks its positions in order, 256 at a time;
// an element's new position is its digit's running offset + the elements with the same
// digit in earlier warps of the round + those in earlier lanes of its warp.
__global__ void __launch_bounds__(kOrdThreads)
    order_scatter_kernel(const uint32_t* __restrict__ bmask, const int* __restrict__ in, int n,
                         int shift, const int* __restrict__ offs, const int* __restrict__ dtot,
                         int* __restrict__ out, const int* mode, int required) {
  if (mode && *mode != required) return;
  constexpr int kWarps = kOrdThreads / 32;
  __shared__ int run[kOrdBuckets];
  __shared__ int wc[kWarps][kOrdBuckets];
  __shared__ int ws[kWarps];
  const int warp = threadIdx.x >> 5;
  {  // first position of digit b: the totals of the smaller digits + earlier CTAs' counts
    const int b = threadIdx.x;   // kOrdThreads == kOrdBuckets
    int tot;
    const int base = block_exclusive_scan(dtot[b], ws, &tot);
    run[b] = base + offs[(size_t)b * gridDim.x + blockIdx.x];
  }
  const int j0 = blockIdx.x * kOrdPts;
  for (int r0 = 0; r0 < kOrdPts; r0 += kOrdThreads) {
    for (int e = threadIdx.x; e < kWarps * kOrdBuckets; e += blockDim.x) (&wc[0][0])[e] = 0;
    __syncthreads();
    const int jj = j0 + r0 + (int)threadIdx.x;
    const int p = jj < n ? (in ? in[jj] : jj) : -1;
    const int k = p >= 0 ? (int)((bmask[p] >> shift) & (kOrdBuckets - 1)) : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, k);
    const int rank = __popc(peers & lanemask_lt());
    if (k >= 0 && rank == 0) wc[warp][k] = __popc(peers);
    __syncthreads();
    if (k >= 0) {
      int pos = run[k] + rank;
      for (int w2 = 0; w2 < warp; ++w2) pos += wc[w2][k];
      out[pos] = p;
    }
    __syncthreads();
    for (int b = threadIdx.x; b < kOrdBuckets; b += blockDim.x) {
      int add = 0;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; ++w2) add += wc[w2][b];
      run[b] += add;
    }
    __syncthreads();
  }
}

// One warp per tile (`trows` rows, a multiple of 32) of the sorted order: OR of the
// block masks, log Z gathered.
__global__ void tile_mask_kernel(const int* __restrict__ perm, const uint32_t* __restrict__ bmask,
                                 const float* __restrict__ logz, int n, int trows,
                                 float* __restrict__ lzp, uint32_t* __restrict__ tmask,
                                 const int* mode, int required) {
  if (mode && *mode != required) return;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t * trows >= n) return;
  uint32_t m = 0;
  for (int j = 0; j < trows / 32; ++j) {
    const int i = t * trows + j * 32 + lane;
    if (i < n) {
      const int p = perm[i];
      lzp[i] = logz[p];
      m |= bmask[p];
    }
  }
  m = __reduce_or_sync(0xffffffffu, m);
  if (lane == 0) tmask[t] = m;
}

// CTA per component block b: the tiles whose mask holds b, in increasing order.
__global__ void __launch_bounds__(kListThreads)
    block_list_kernel(const uint32_t* __restrict__ tmask, int ntiles, int* __restrict__ tlist,
                      int stride, int* __restrict__ tcnt, const int* mode, int required) {
  if (mode && *mode != required) return;
  __shared__ int wsum[kListThreads / 32];
  const int b = blockIdx.x;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int base = 0;   // identical in every thread
  for (int t0 = 0; t0 < ntiles; t0 += kListThreads) {
    const int t = t0 + (int)threadIdx.x;
    const bool f = t < ntiles && ((tmask[t] >> b) & 1u);
    const uint32_t ball = __ballot_sync(0xffffffffu, f);
    if (lane == 0) wsum[warp] = __popc(ball);
    __syncthreads();
    int before = 0, total = 0;
    for (int w2 = 0; w2 < kListThreads / 32; ++w2) {
      const int cw = wsum[w2];
      before += w2 < warp ? cw : 0;
      total += cw;
    }
    if (f) tlist[(size_t)b * stride + base + before + __popc(ball & lanemask_lt())] = t;
    base += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) tcnt[b] = base;
}

// CUDA-core path: per point, the 128-component blocks whose largest log z (from the
// per-64-component maxima of the log-sum-exp sweep) lies within kSimtSkipCut of log Z.
__global__ void simt_mask_kernel(const float* __restrict__ bmx, const float* __restrict__ logz,
                                 int n, int nb64, int nkb, uint32_t* __restrict__ bmask,
                                 const int* mode) {
  if (mode && *mode != kModeSimt) return;
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const float lz = logz[i];
  const float lim = lz - kSimtSkipCut;
  uint32_t m = 0;
  const float* b = bmx + (size_t)i * nb64;
  for (int q = 0; q < nb64; ++q)
    if (b[q] > lim) m |= 1u << (q >> 1);
  const uint32_t full = nkb >= 32 ? 0xFFFFFFFFu : (1u << nkb) - 1u;
  bmask[i] = (lz > -CUDART_INF_F && lz < CUDART_INF_F && m) ? m : full;
}

// Radix passes over the block masks: the last one leaves the order in perm.
cudaError_t order_sort(const Ctx& c, int nkb, int ni, const int* mode, int required,
                       cudaStream_t s) {
  const Workspace& w = c.ws;
  const int ncta = (int)ceil_div64(ni, kOrdPts);
  const int passes = (nkb + 7) / 8;
  const int* in = nullptr;
  int* out = (passes & 1) ? w.perm : w.perm2;
  for (int ps = 0; ps < passes; ++ps) {
    const int shift = 8 * ps;
    prof_begin(c, KI_TC_ORDER, s, mode, required);
    order_count_kernel<<<ncta, kOrdThreads, 0, s>>>(w.bmask, in, ni, shift, w.ord_hist, mode,
                                                    required);
    prof_end(c, KI_TC_ORDER, s);
    prof_begin(c, KI_TC_ORDER, s, mode, required);
    order_scan_kernel<<<kOrdBuckets, kOrdThreads, 0, s>>>(w.ord_hist, ncta, w.ord_tot, mode,
                                                          required);
    prof_end(c, KI_TC_ORDER, s);
    prof_begin(c, KI_TC_ORDER, s, mode, required);
    order_scatter_kernel<<<ncta, kOrdThreads, 0, s>>>(w.bmask, in, ni, shift, w.ord_hist,
                                                       w.ord_tot, out, mode, required);
    prof_end(c, KI_TC_ORDER, s);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    in = out;
    out = (out == w.perm) ? w.perm2 : w.perm;
  }
  return cudaSuccess;
}

// Tile masks (tiles of trows positions), log Z in sorted order, lists of active tiles.
cudaError_t order_lists(const Ctx& c, int nkb, int ni, int trows, const int* mode, int required,
                        cudaStream_t s) {
  const Workspace& w = c.ws;
  const int ntiles = (int)ceil_div64(ni, trows);
  prof_begin(c, KI_TC_ORDER, s, mode, required);
  tile_mask_kernel<<<(unsigned)ceil_div64(ntiles, 8), 256, 0, s>>>(w.perm, w.bmask, w.logz, ni,
                                                                   trows, w.lzp, w.tmask, mode,
                                                                   required);
  prof_end(c, KI_TC_ORDER, s);
  prof_begin(c, KI_TC_ORDER, s, mode, required);
  block_list_kernel<<<nkb, kListThreads, 0, s>>>(w.tmask, ntiles, w.tlist, (int)(kChunk / trows),
                                                 w.tcnt, mode, required);
  prof_end(c, KI_TC_ORDER, s);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_tc_order(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            const int* mode, cudaStream_t s) {
  const int nkb = c.ws.Kt / 128;
  cudaError_t e;
  if ((e = order_sort(c, nkb, (int)n, mode, kModeTensor, s)) != cudaSuccess) return e;
  if ((e = launch_tc_convert(c, X, x_dtype, n, ldx, c.ws.perm, mode, s)) != cudaSuccess) return e;
  return order_lists(c, nkb, (int)n, kTileRows, mode, kModeTensor, s);
}

cudaError_t launch_assign_order(const Ctx& c, int64_t n, cudaStream_t s) {
  const int nkb = c.ws.Kt / 128;
  cudaError_t e;
  if ((e = order_sort(c, nkb, (int)n, nullptr, 0, s)) != cudaSuccess) return e;
  return order_lists(c, nkb, (int)n, kTP, nullptr, 0, s);
}

bool simt_skip(const Ctx& c) {
  // with fewer blocks there is too little to leave out (measured: 2 blocks at D = 960
  // lose 13% to the ordering and the indirect loads)
  const int nkb = (c.ws.Kp + 127) / 128;
  return c.skip && c.ws.bmx && nkb >= 4 && nkb <= kSkipMaxBlocks;
}

cudaError_t launch_simt_order(const Ctx& c, int64_t n, const int* mode, cudaStream_t s) {
  const Workspace& w = c.ws;
  const int nkb = (w.Kp + 127) / 128;
  prof_begin(c, KI_TC_ORDER, s, mode, kModeSimt);
  simt_mask_kernel<<<(unsigned)ceil_div64(n, 256), 256, 0, s>>>(w.bmx, w.logz, (int)n, w.Kp / kKB,
                                                                nkb, w.bmask, mode);
  prof_end(c, KI_TC_ORDER, s);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if ((e = order_sort(c, nkb, (int)n, mode, kModeSimt, s)) != cudaSuccess) return e;
  return order_lists(c, nkb, (int)n, kTP, mode, kModeSimt, s);
}

}  // namespace fgmm
