// Block skipping in the tensor-core statistics sweep: the point order of sweep 2.
//
// Paper: "Flash-GMM: A Memory-Efficient Kernel for Scalable Soft Clustering", §3.1 and
// Algorithm 1.  Sweep 2 forms r_ik = exp(log z_ik - log Z_i) for every point and every
// component and folds them into N_k, sum r x, sum r x^2.  The tensor-core version keeps
// r as fp16(r 2^15), exactly 0 for a log-density more than 27.7 nats below log Z, so a
// (128-point tile, 128-component block) pair in which that holds for every pair adds
// exactly nothing.  Sweep 1 records, per point, the blocks that come within kSkipCut of
// log Z (a bit mask).  The kernels here
//   order_count / order_scan / order_scatter
//                 a stable counting sort of the chunk's points by bucket: the single
//                 block of a one-block point, or a last bucket for every other point;
//   tile_mask     per tile of the sorted order, the OR of its points' masks, and log Z
//                 in the sorted order;
//   block_list    per component block, the tiles whose mask holds it, in increasing order.
// Between scatter and tile_mask, tc_convert rewrites phi(x) in the sorted order.  Sweep 2
// then runs each block over its own list.  Every step is deterministic (counts, prefix
// sums, ordered scatter), so the sums stay bitwise reproducible from run to run; they
// differ from the natural order only by the order of fp32 additions.
#include "fgmm_internal.h"

namespace fgmm {

namespace {

constexpr int kOrdThreads = 256;
constexpr int kOrdBuckets = kSkipMaxBlocks + 1;
constexpr int kTileRows = 128;
constexpr int kListThreads = 1024;

__device__ __forceinline__ int order_key(uint32_t m, int nkb) {
  return __popc(m) == 1 ? __ffs(m) - 1 : nkb;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
  uint32_t r;
  asm("mov.u32 %0, %%lanemask_lt;" : "=r"(r));
  return r;
}

// Counts of each bucket among the kOrdPts points of this CTA.
__global__ void order_count_kernel(const uint32_t* __restrict__ bmask, int n, int nkb,
                                   int* __restrict__ hist, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  __shared__ int cnt[kOrdBuckets];
  const int nb = nkb + 1;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) cnt[b] = 0;
  __syncthreads();
  const int i0 = blockIdx.x * kOrdPts;
  for (int j = threadIdx.x; j < kOrdPts; j += blockDim.x) {
    const int i = i0 + j;
    if (i < n) atomicAdd(&cnt[order_key(bmask[i], nkb)], 1);
  }
  __syncthreads();
  for (int b = threadIdx.x; b < nb; b += blockDim.x) hist[blockIdx.x * nb + b] = cnt[b];
}

// hist[c][b] (counts) -> exclusive prefix sums in (bucket, CTA) order: the first sorted
// position of CTA c's points of bucket b.  One CTA of kListThreads threads.
__global__ void order_scan_kernel(int* __restrict__ hist, int ncta, int nb, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  __shared__ int wsum[32];
  const int E = ncta * nb;
  const int per = (E + blockDim.x - 1) / blockDim.x;
  const int e0 = threadIdx.x * per;
  // scan position e = b * ncta + c is stored at hist[c * nb + b]
  auto at = [&](int e) -> int& { return hist[(e % ncta) * nb + e / ncta]; };
  int local = 0;
  for (int e = e0; e < e0 + per && e < E; ++e) local += at(e);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int v = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  if (lane == 31) wsum[warp] = v;
  __syncthreads();
  if (warp == 0) {
    int t = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, t, o);
      if (lane >= o) t += u;
    }
    wsum[lane] = t;   // inclusive over warps
  }
  __syncthreads();
  int run = v - local + (warp > 0 ? wsum[warp - 1] : 0);
  for (int e = e0; e < e0 + per && e < E; ++e) {
    const int cnt = at(e);
    at(e) = run;
    run += cnt;
  }
}

// Stable scatter: CTA c walks its points in index order, 256 at a time; a point's
// position is its bucket's running offset + the points of the same bucket in earlier
// warps of the round + those in earlier lanes of its warp.
__global__ void __launch_bounds__(kOrdThreads)
    order_scatter_kernel(const uint32_t* __restrict__ bmask, int n, int nkb,
                         const int* __restrict__ offs, int* __restrict__ perm, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  constexpr int kWarps = kOrdThreads / 32;
  __shared__ int run[kOrdBuckets];
  __shared__ int wc[kWarps][kOrdBuckets];
  const int nb = nkb + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  for (int b = threadIdx.x; b < nb; b += blockDim.x) run[b] = offs[blockIdx.x * nb + b];
  const int i0 = blockIdx.x * kOrdPts;
  for (int r0 = 0; r0 < kOrdPts; r0 += kOrdThreads) {
    for (int e = threadIdx.x; e < kWarps * kOrdBuckets; e += blockDim.x) (&wc[0][0])[e] = 0;
    __syncthreads();
    const int i = i0 + r0 + (int)threadIdx.x;
    const int k = i < n ? order_key(bmask[i], nkb) : -1;
    const uint32_t peers = __match_any_sync(0xffffffffu, k);
    const int rank = __popc(peers & lanemask_lt());
    if (k >= 0 && rank == 0) wc[warp][k] = __popc(peers);
    __syncthreads();
    if (k >= 0) {
      int pos = run[k] + rank;
      for (int w2 = 0; w2 < warp; ++w2) pos += wc[w2][k];
      perm[pos] = i;
    }
    __syncthreads();
    if ((int)threadIdx.x < nb) {
      int add = 0;
#pragma unroll
      for (int w2 = 0; w2 < kWarps; ++w2) add += wc[w2][threadIdx.x];
      run[threadIdx.x] += add;
    }
    __syncthreads();
  }
}

// One warp per tile of the sorted order: OR of the block masks, log Z gathered.
__global__ void tile_mask_kernel(const int* __restrict__ perm, const uint32_t* __restrict__ bmask,
                                 const float* __restrict__ logz, int n, float* __restrict__ lzp,
                                 uint32_t* __restrict__ tmask, const int* mode) {
  if (mode && *mode != kModeTensor) return;
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (t * kTileRows >= n) return;
  uint32_t m = 0;
#pragma unroll
  for (int j = 0; j < kTileRows / 32; ++j) {
    const int i = t * kTileRows + j * 32 + lane;
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
                      int stride, int* __restrict__ tcnt, const int* mode) {
  if (mode && *mode != kModeTensor) return;
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

}  // namespace

cudaError_t launch_tc_order(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            const int* mode, cudaStream_t s) {
  const Workspace& w = c.ws;
  const int nkb = w.Kt / 128;
  const int nb = nkb + 1;
  const int ni = (int)n;
  const int ncta = (int)ceil_div64(n, kOrdPts);
  const int ntiles = (int)ceil_div64(n, kTileRows);
  cudaError_t e;
  prof_begin(c, KI_TC_ORDER, s, mode, kModeTensor);
  order_count_kernel<<<ncta, kOrdThreads, 0, s>>>(w.bmask, ni, nkb, w.ord_hist, mode);
  prof_end(c, KI_TC_ORDER, s);
  prof_begin(c, KI_TC_ORDER, s, mode, kModeTensor);
  order_scan_kernel<<<1, kListThreads, 0, s>>>(w.ord_hist, ncta, nb, mode);
  prof_end(c, KI_TC_ORDER, s);
  prof_begin(c, KI_TC_ORDER, s, mode, kModeTensor);
  order_scatter_kernel<<<ncta, kOrdThreads, 0, s>>>(w.bmask, ni, nkb, w.ord_hist, w.perm, mode);
  prof_end(c, KI_TC_ORDER, s);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_tc_convert(c, X, x_dtype, n, ldx, w.perm, mode, s)) != cudaSuccess) return e;
  prof_begin(c, KI_TC_ORDER, s, mode, kModeTensor);
  tile_mask_kernel<<<(unsigned)ceil_div64(ntiles, 8), 256, 0, s>>>(w.perm, w.bmask, w.logz, ni,
                                                                   w.lzp, w.tmask, mode);
  prof_end(c, KI_TC_ORDER, s);
  prof_begin(c, KI_TC_ORDER, s, mode, kModeTensor);
  block_list_kernel<<<nkb, kListThreads, 0, s>>>(w.tmask, ntiles, w.tlist, (int)(kChunk / kTileRows),
                                                 w.tcnt, mode);
  prof_end(c, KI_TC_ORDER, s);
  return cudaGetLastError();
}

}  // namespace fgmm
