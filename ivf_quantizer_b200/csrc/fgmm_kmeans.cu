// k-means warm start before EM ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
// Clustering", §4.4: k-means, then soft EM from its centroids; the initialisation
// appendix: k-means++ seeding).
//
//   Lloyd iteration   a_i = argmin_k ||x_i - c_k||^2 (lowest k on ties),
//                     c_k = mean of the points assigned to k (empty: c_k kept),
//                     inertia = sum_i ||x_i - c_{a_i}||^2
//   k-means++ seeding c_0 = x_first; c_t = x_i drawn with probability D(x_i) / sum D,
//                     D(x) = min_{j<t} ||x - c_j||^2, one uniform u_t per draw (input)
//
// Decisions that floating point turns into indices are taken in a precision fixed
// here, so that they are reproducible and checkable: squared distances are fp32,
// accumulated over dimensions in increasing order with every subtraction, product and
// sum rounded separately (no fused multiply-add).  The seeding weights are integers,
// floor(D * 2^s) with 2^s bringing the largest D to [2^29, 2^30), and the draw picks the
// smallest i whose running integer sum exceeds floor(u_t * total).  Cluster sums are
// accumulated as 64-bit fixed-point integers (scale 2^F from the data's largest |x| and
// N), whose atomic additions are exact and order-independent: every result is bitwise
// reproducible.
#include <cuda_bf16.h>
#include <math_constants.h>

#include "fgmm_internal.h"

namespace fgmm {
namespace {

constexpr int kKmTP = 64;        // points per assignment tile
constexpr int kKmKB = 64;        // centroids per block
constexpr int kSeedBlk = 4096;   // points per seeding block (partial max / weight sums)

__device__ __forceinline__ float ldv(const float* p) { return __ldg(p); }
__device__ __forceinline__ float ldv(const __nv_bfloat16* p) { return __bfloat162float(*p); }

// ||x - c||^2 term by term: subtract, square, add, each rounded to fp32.
__device__ __forceinline__ float sq_step(float acc, float x, float c) {
  const float t = __fsub_rn(x, c);
  return __fadd_rn(acc, __fmul_rn(t, t));
}

__device__ void set_status_km(int* st, int code) { atomicCAS(st, FGMM_OK, code); }

}  // namespace

// ------------------------------------------------------------------ Lloyd: preparation
// Centroids [K][D] -> padded [Kp][Dp] (zeros beyond D: they add exact zeros).
__global__ void km_pad_kernel(int K, int D, int Kp, int Dp, const float* __restrict__ c,
                              float* __restrict__ cp, int* status) {
  const int k = blockIdx.x;
  for (int d = threadIdx.x; d < Dp; d += blockDim.x) {
    const float v = (k < K && d < D) ? c[(size_t)k * D + d] : 0.f;
    if (k < K && d < D && !isfinite(v)) set_status_km(status, FGMM_ERR_INVALID_ARG);
    cp[(size_t)k * Dp + d] = v;
  }
}

// Largest |x| over a chunk, as the bit pattern of a non-negative float (integer order
// equals float order there), combined by atomicMax: exact and order-independent.
template <typename T>
__global__ void km_maxabs_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D,
                                 unsigned int* __restrict__ out) {
  unsigned int m = 0;
  for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < n * D;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t i = e / D;
    const int d = (int)(e - i * D);
    const float v = fabsf(ldv(X + i * ldx + d));
    m = max(m, isfinite(v) ? __float_as_uint(v) : 0x7f7fffffu);
  }
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) m = max(m, __shfl_xor_sync(0xffffffffu, m, off));
  if ((threadIdx.x & 31) == 0) atomicMax(out, m);
}

// ------------------------------------------------------------------ Lloyd: assignment
// One CTA per 64-point tile, 256 threads: thread (ty, tx) owns points ty + 16 j and, per
// centroid block, centroids kb + tx + 16 q (j, q < 4).  Features in chunks of kDC staged
// in shared memory, in increasing order, so every distance is the fixed fp32 sequence.
// After the assignment the tile adds its points to the cluster sums (64-bit fixed point,
// scale 2^F) and counts, and writes its inertia partial (fp64, points in order).
template <typename T>
__global__ void __launch_bounds__(256)
    km_assign_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D, int Dp, int Kp,
                     int K, const float* __restrict__ cp, const unsigned int* __restrict__ fbits,
                     long long* __restrict__ sums, long long* __restrict__ counts,
                     int32_t* __restrict__ assign_out, double* __restrict__ part) {
  __shared__ float xs[kKmTP][kDC + 1];
  __shared__ float cs[kKmKB][kDC + 1];
  __shared__ int as[kKmTP];
  __shared__ float ds[kKmTP];
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int64_t i0 = (int64_t)blockIdx.x * kKmTP;
  float best_d[4];
  int best_k[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) { best_d[j] = CUDART_INF_F; best_k[j] = 0; }
  for (int kb = 0; kb < Kp; kb += kKmKB) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
#pragma unroll
      for (int q = 0; q < 4; ++q) acc[j][q] = 0.f;
    for (int d0 = 0; d0 < Dp; d0 += kDC) {
      for (int e = threadIdx.x; e < kKmTP * kDC; e += blockDim.x) {
        const int r = e / kDC, cx = e % kDC;
        const int64_t i = i0 + r;
        const int d = d0 + cx;
        xs[r][cx] = (i < n && d < D) ? ldv(X + i * ldx + d) : 0.f;
        cs[r][cx] = cp[(size_t)(kb + r) * Dp + d];
      }
      __syncthreads();
#pragma unroll 4
      for (int d = 0; d < kDC; ++d) {
        float xv[4], cv[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) xv[j] = xs[ty + 16 * j][d];
#pragma unroll
        for (int q = 0; q < 4; ++q) cv[q] = cs[tx + 16 * q][d];
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[j][q] = sq_step(acc[j][q], xv[j], cv[q]);
      }
      __syncthreads();
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      // this thread's best of its 4 centroids (increasing k), then the 16 threads of the
      // point row: lexicographic minimum of (distance, index)
      float bd = CUDART_INF_F;
      int bk = 0x7fffffff;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int k = kb + tx + 16 * q;
        if (k < K && acc[j][q] < bd) { bd = acc[j][q]; bk = k; }
      }
#pragma unroll
      for (int off = 8; off > 0; off >>= 1) {
        const float od = __shfl_xor_sync(0xffffffffu, bd, off);
        const int ok = __shfl_xor_sync(0xffffffffu, bk, off);
        if (od < bd || (od == bd && ok < bk)) { bd = od; bk = ok; }
      }
      // earlier blocks hold lower indices: only a strictly smaller distance replaces
      if (bd < best_d[j]) { best_d[j] = bd; best_k[j] = bk; }
    }
  }
  if (tx == 0)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      as[ty + 16 * j] = best_k[j];
      ds[ty + 16 * j] = best_d[j];
    }
  __syncthreads();
  const int nt = (int)min((int64_t)kKmTP, n - i0);
  if (threadIdx.x < nt) {
    if (assign_out) assign_out[i0 + threadIdx.x] = as[threadIdx.x];
    atomicAdd(reinterpret_cast<unsigned long long*>(counts + as[threadIdx.x]), 1ull);
  }
  if (threadIdx.x == 0) {
    double p = 0.0;
    for (int r = 0; r < nt; ++r) p += (double)ds[r];
    part[blockIdx.x] = p;
  }
  const double scale = ldexp(1.0, (int)*fbits);
  for (int e = threadIdx.x; e < nt * D; e += blockDim.x) {
    const int r = e / D, d = e - r * D;
    const long long v = llrint((double)ldv(X + (i0 + r) * ldx + d) * scale);
    atomicAdd(reinterpret_cast<unsigned long long*>(sums + (size_t)as[r] * Dp + d),
              (unsigned long long)v);
  }
}

// Fixed-order sum of a chunk's tile partials into the running inertia.
__global__ void km_partial_sum_kernel(const double* __restrict__ part, int ntiles,
                                      double* __restrict__ total) {
  __shared__ double red[256];
  double s = 0.0;
  for (int t = threadIdx.x; t < ntiles; t += blockDim.x) s += part[t];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) *total += red[0];
}

// Fixed-point scale from the largest |x| and N: 2^F * max|x| * N < 2^62.
__global__ void km_scale_kernel(const unsigned int* __restrict__ maxbits, int64_t n,
                                unsigned int* __restrict__ fbits) {
  const float m = __uint_as_float(*maxbits);
  int e = 0;
  if (m > 0.f) frexpf(m, &e);            // m < 2^e
  int ln = 0;
  while ((1ll << ln) < n && ln < 62) ++ln;  // n <= 2^ln
  int F = 61 - e - ln;
  if (F > 60) F = 60;
  if (F < -60) F = -60;
  *fbits = (unsigned int)F;
}

// New centroids: mean of the assigned points (fixed-point sums / count); empty
// clusters keep theirs.  One CTA per cluster.
__global__ void km_finish_kernel(int K, int D, int Dp, const long long* __restrict__ sums,
                                 const long long* __restrict__ counts,
                                 const unsigned int* __restrict__ fbits, float* __restrict__ c,
                                 int64_t* __restrict__ counts_out,
                                 const double* __restrict__ inertia,
                                 double* __restrict__ inertia_out) {
  const int k = blockIdx.x;
  const long long cnt = counts[k];
  const double inv_scale = ldexp(1.0, -(int)*fbits);
  if (cnt > 0)
    for (int d = threadIdx.x; d < D; d += blockDim.x)
      c[(size_t)k * D + d] = (float)(((double)sums[(size_t)k * Dp + d] * inv_scale) / (double)cnt);
  if (threadIdx.x == 0) {
    if (counts_out) counts_out[k] = cnt;
    if (k == 0 && inertia_out) *inertia_out = *inertia;
  }
}

// ------------------------------------------------------------------ k-means++ seeding
// Per draw t: (1) dist_i = min(dist_i, ||x_i - c_{t-1}||^2) (t = 1: the distance to c_0)
// and the largest dist of each block of kSeedBlk points; (2) the scale 2^s from the
// global largest; (3) each block's sum of the integer weights floor(dist * 2^s);
// (4) one CTA finds the drawn point and copies it into centroid row t.
template <typename T>
__global__ void seed_update_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D,
                                   const float* __restrict__ c, int init,
                                   float* __restrict__ dist, float* __restrict__ bmax) {
  __shared__ float red[256];
  float m = 0.f;
  const int64_t b0 = (int64_t)blockIdx.x * kSeedBlk;
  for (int e = threadIdx.x; e < kSeedBlk; e += blockDim.x) {
    const int64_t i = b0 + e;
    if (i >= n) break;
    const T* x = X + i * ldx;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = sq_step(acc, ldv(x + d), c[d]);
    const float v = init ? acc : fminf(dist[i], acc);
    dist[i] = v;
    m = fmaxf(m, v);
  }
  red[threadIdx.x] = m;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x == 0) bmax[blockIdx.x] = red[0];
}

// Exponent s: the largest distance times 2^s lies in [2^29, 2^30) (s = 0 when all are 0).
__global__ void seed_scale_kernel(const float* __restrict__ bmax, int nblk, int* __restrict__ sexp) {
  __shared__ float red[256];
  float m = 0.f;
  for (int b = threadIdx.x; b < nblk; b += blockDim.x) m = fmaxf(m, bmax[b]);
  red[threadIdx.x] = m;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] = fmaxf(red[threadIdx.x], red[threadIdx.x + w]);
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    int e = 0;
    if (red[0] > 0.f) frexpf(red[0], &e);
    *sexp = 30 - e;
  }
}

template <typename T>
__global__ void seed_first_kernel(const T* __restrict__ X, int64_t ldx, int D, int64_t first,
                                  int64_t* __restrict__ idx, float* __restrict__ c) {
  if (threadIdx.x == 0) idx[0] = first;
  for (int d = threadIdx.x; d < D; d += blockDim.x) c[d] = ldv(X + first * ldx + d);
}

__device__ __forceinline__ long long seed_weight(float dist, int sexp) {
  return (long long)floor((double)dist * ldexp(1.0, sexp));
}

__global__ void seed_wsum_kernel(const float* __restrict__ dist, int64_t n,
                                 const int* __restrict__ sexp, long long* __restrict__ bsum) {
  __shared__ long long red[256];
  const int s = *sexp;
  long long acc = 0;
  const int64_t b0 = (int64_t)blockIdx.x * kSeedBlk;
  for (int e = threadIdx.x; e < kSeedBlk; e += blockDim.x) {
    const int64_t i = b0 + e;
    if (i < n) acc += seed_weight(dist[i], s);
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) bsum[blockIdx.x] = red[0];
}

// One CTA of 1024 threads: total weight, target floor(u * total), the block holding the
// target by a prefix over the block sums, then the point by a prefix over that block's
// weights: the smallest i whose running sum exceeds the target.  All integer, exact.
template <typename T>
__global__ void __launch_bounds__(1024)
    seed_select_kernel(const T* __restrict__ X, int64_t n, int64_t ldx, int D,
                       const float* __restrict__ dist, const long long* __restrict__ bsum,
                       int nblk, const int* __restrict__ sexp, const double* __restrict__ u,
                       int t, int64_t* __restrict__ idx, float* __restrict__ c) {
  __shared__ long long part[1024];
  __shared__ long long sh_target, sh_base;
  __shared__ int sh_blk;
  __shared__ int64_t sh_i;
  const int tid = threadIdx.x;
  // (a) per-thread sums over contiguous ranges of blocks, then an inclusive prefix
  const int per = (nblk + 1023) / 1024;
  long long acc = 0;
  for (int b = tid * per; b < min(nblk, (tid + 1) * per); ++b) acc += bsum[b];
  part[tid] = acc;
  __syncthreads();
  for (int off = 1; off < 1024; off <<= 1) {
    const long long v = (tid >= off) ? part[tid - off] : 0;
    __syncthreads();
    part[tid] += v;
    __syncthreads();
  }
  if (tid == 0) {
    const long long total = part[1023];
    sh_i = -1;
    if (total > 0) {
      sh_target = (long long)floor(u[t - 1] * (double)total);
      // first thread range whose inclusive sum exceeds the target, then the block
      int r = 0;
      while (r < 1023 && part[r] <= sh_target) ++r;
      long long base = (r > 0) ? part[r - 1] : 0;
      int b = r * per;
      while (b < nblk - 1 && base + bsum[b] <= sh_target) { base += bsum[b]; ++b; }
      sh_blk = b;
      sh_base = base;
    } else {
      sh_blk = -1;
      sh_i = idx[t - 1];            // every point sits on a chosen centre
    }
  }
  __syncthreads();
  if (sh_blk >= 0) {
    // (b) inside block sh_blk: prefix of the point weights in 1024-point rounds
    const int s = *sexp;
    const int64_t b0 = (int64_t)sh_blk * kSeedBlk;
    long long run = sh_base;
    for (int r0 = 0; r0 < kSeedBlk; r0 += 1024) {
      const int64_t i = b0 + r0 + tid;
      part[tid] = (i < n) ? seed_weight(dist[i], s) : 0;
      __syncthreads();
      for (int off = 1; off < 1024; off <<= 1) {
        const long long v = (tid >= off) ? part[tid - off] : 0;
        __syncthreads();
        part[tid] += v;
        __syncthreads();
      }
      const long long incl = run + part[tid];
      const long long excl = run + (tid > 0 ? part[tid - 1] : 0);
      if (excl <= sh_target && incl > sh_target && i < n) sh_i = i;   // exactly one thread
      run += part[1023];
      __syncthreads();
      if (sh_i >= 0) break;
    }
    if (tid == 0 && sh_i < 0) sh_i = min(n - 1, b0 + kSeedBlk - 1);
    __syncthreads();
  }
  const int64_t i = sh_i;
  if (tid == 0) idx[t] = i;
  for (int d = tid; d < D; d += blockDim.x) c[(size_t)t * D + d] = ldv(X + i * ldx + d);
}

// ------------------------------------------------------------------ launchers
size_t kmeans_seed_scratch_bytes(int64_t n) {
  const int64_t nblk = (n + kSeedBlk - 1) / kSeedBlk;
  return (size_t)(((n * 4 + 255) / 256) * 256 + nblk * 8 + ((nblk * 4 + 255) / 256) * 256 + 256);
}

cudaError_t launch_kmeans_step(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                               float* centroids, int32_t* assign_out, int64_t* counts_out,
                               double* inertia_out, cudaStream_t s) {
  const Workspace& w = c.ws;
  long long* sums = reinterpret_cast<long long*>(w.stats);              // [K][Dp]
  long long* counts = sums + (size_t)c.K * w.Dp;                        // [K]
  unsigned int* maxbits = w.km_word;
  unsigned int* fbits = w.km_word + 1;
  const size_t eb = x_dtype == FGMM_BF16 ? 2 : 4;
  cudaError_t e;
  if ((e = cudaMemsetAsync(sums, 0, ((size_t)c.K * w.Dp + c.K) * sizeof(long long), s)) != cudaSuccess ||
      (e = cudaMemsetAsync(w.km_word, 0, 2 * sizeof(unsigned int), s)) != cudaSuccess ||
      (e = cudaMemsetAsync(w.ll_total, 0, sizeof(double), s)) != cudaSuccess)
    return e;
  km_pad_kernel<<<w.Kp, 128, 0, s>>>(c.K, c.D, w.Kp, w.Dp, centroids, w.mu, w.status);
  for (int64_t c0 = 0; c0 < n; c0 += kChunk) {
    const int64_t nc = (n - c0 < kChunk) ? n - c0 : kChunk;
    const void* Xc = (const char*)X + (size_t)c0 * ldx * eb;
    if (x_dtype == FGMM_BF16)
      km_maxabs_kernel<<<4 * c.num_sms, 256, 0, s>>>((const __nv_bfloat16*)Xc, nc, ldx, c.D, maxbits);
    else
      km_maxabs_kernel<<<4 * c.num_sms, 256, 0, s>>>((const float*)Xc, nc, ldx, c.D, maxbits);
  }
  km_scale_kernel<<<1, 1, 0, s>>>(maxbits, n, fbits);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int64_t c0 = 0; c0 < n; c0 += kChunk) {
    const int64_t nc = (n - c0 < kChunk) ? n - c0 : kChunk;
    const void* Xc = (const char*)X + (size_t)c0 * ldx * eb;
    const unsigned grid = (unsigned)((nc + kKmTP - 1) / kKmTP);
    int32_t* ao = assign_out ? assign_out + c0 : nullptr;
    prof_begin(c, KI_KM_ASSIGN, s);
    if (x_dtype == FGMM_BF16)
      km_assign_kernel<<<grid, 256, 0, s>>>((const __nv_bfloat16*)Xc, nc, ldx, c.D, w.Dp, w.Kp,
                                            c.K, w.mu, fbits, sums, counts, ao, w.ll_tiles);
    else
      km_assign_kernel<<<grid, 256, 0, s>>>((const float*)Xc, nc, ldx, c.D, w.Dp, w.Kp, c.K,
                                            w.mu, fbits, sums, counts, ao, w.ll_tiles);
    prof_end(c, KI_KM_ASSIGN, s);
    km_partial_sum_kernel<<<1, 256, 0, s>>>(w.ll_tiles, (int)grid, w.ll_total);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  km_finish_kernel<<<c.K, 128, 0, s>>>(c.K, c.D, w.Dp, sums, counts, fbits, centroids,
                                       counts_out, w.ll_total, inertia_out);
  return cudaGetLastError();
}

cudaError_t launch_kmeans_seed(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                               int64_t first, const double* u, float* centroids,
                               int64_t* idx_out, void* scratch, cudaStream_t s) {
  const int64_t nblk64 = (n + kSeedBlk - 1) / kSeedBlk;
  const int nblk = (int)nblk64;
  char* p = static_cast<char*>(scratch);
  float* dist = reinterpret_cast<float*>(p);
  p += ((n * 4 + 255) / 256) * 256;
  long long* bsum = reinterpret_cast<long long*>(p);
  p += nblk64 * 8;
  float* bmax = reinterpret_cast<float*>(p);
  p += ((nblk64 * 4 + 255) / 256) * 256;
  int* sexp = reinterpret_cast<int*>(p);
  int64_t* idx = idx_out;
  cudaError_t e;
  // c_0 = x_first
  if (x_dtype == FGMM_BF16)
    seed_first_kernel<<<1, 128, 0, s>>>((const __nv_bfloat16*)X, ldx, c.D, first, idx, centroids);
  else
    seed_first_kernel<<<1, 128, 0, s>>>((const float*)X, ldx, c.D, first, idx, centroids);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  for (int t = 1; t < c.K; ++t) {
    const float* cprev = centroids + (size_t)(t - 1) * c.D;
    prof_begin(c, KI_KM_SEED, s);
    if (x_dtype == FGMM_BF16)
      seed_update_kernel<<<nblk, 256, 0, s>>>((const __nv_bfloat16*)X, n, ldx, c.D, cprev,
                                              t == 1, dist, bmax);
    else
      seed_update_kernel<<<nblk, 256, 0, s>>>((const float*)X, n, ldx, c.D, cprev, t == 1, dist,
                                              bmax);
    prof_end(c, KI_KM_SEED, s);
    seed_scale_kernel<<<1, 256, 0, s>>>(bmax, nblk, sexp);
    seed_wsum_kernel<<<nblk, 256, 0, s>>>(dist, n, sexp, bsum);
    if (x_dtype == FGMM_BF16)
      seed_select_kernel<<<1, 1024, 0, s>>>((const __nv_bfloat16*)X, n, ldx, c.D, dist, bsum,
                                            nblk, sexp, u, t, idx, centroids);
    else
      seed_select_kernel<<<1, 1024, 0, s>>>((const float*)X, n, ldx, c.D, dist, bsum, nblk, sexp,
                                            u, t, idx, centroids);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  return cudaSuccess;
}

}  // namespace fgmm
