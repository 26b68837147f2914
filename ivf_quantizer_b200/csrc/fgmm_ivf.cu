// IVF application of the soft assignment ("Flash-GMM: A Memory-Efficient Kernel for
// Scalable Soft Clustering", §4): posting lists built from the top-m assignment ids
// (a vector sits in the list of every cluster it is assigned to, §4.3) and nprobe
// search with exact re-ranking.
//
//   build   counts per (block of 4096 vectors, cluster) -> per-cluster exclusive prefix
//           over the blocks -> cluster offsets -> each block's thread writes its vectors
//           in index order: lists come out in increasing vector index, deterministically
//   search  one CTA per query: fp32 distances to every centroid, the nprobe nearest
//           (ties: lower index), exact distances to every entry of their lists, the k
//           nearest distinct vectors (ties: lower index), and the number of entries
//           scanned (distance computations).
//
// Distances are fp32 squared L2 with dimensions in increasing order and every
// subtraction, product and sum rounded separately (no fused multiply-add), the same
// fixed sequence as the k-means warm start, so rankings are reproducible and exact
// against a reference that follows the same sequence.
#include <math_constants.h>

#include "fgmm_internal.h"

namespace fgmm {
namespace {

constexpr int kIvfBlk = 4096;   // vectors per counting block
constexpr int kIvfThreads = 256;

__device__ __forceinline__ float sq_step_ivf(float acc, float x, float c) {
  const float t = __fsub_rn(x, c);
  return __fadd_rn(acc, __fmul_rn(t, t));
}

__global__ void ivf_count_kernel(const int32_t* __restrict__ ids, int64_t n, int m, int K,
                                 int* __restrict__ counts) {
  extern __shared__ int hist[];
  for (int k = threadIdx.x; k < K; k += blockDim.x) hist[k] = 0;
  __syncthreads();
  const int64_t i0 = (int64_t)blockIdx.x * kIvfBlk;
  for (int e = threadIdx.x; e < kIvfBlk * m; e += blockDim.x) {
    const int64_t i = i0 + e / m;
    if (i >= n) break;
    const int c = ids[i * m + e % m];
    if (c >= 0 && c < K) atomicAdd(&hist[c], 1);
  }
  __syncthreads();
  for (int k = threadIdx.x; k < K; k += blockDim.x) counts[(size_t)blockIdx.x * K + k] = hist[k];
}

// Per cluster: exclusive prefix over the blocks (in place) and the cluster's total.
__global__ void ivf_colscan_kernel(int* __restrict__ counts, int nblk, int K,
                                   int64_t* __restrict__ totals) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  int64_t run = 0;
  for (int b = 0; b < nblk; ++b) {
    const int c = counts[(size_t)b * K + k];
    counts[(size_t)b * K + k] = (int)run;
    run += c;
  }
  totals[k] = run;
}

// Offsets [K + 1] from the totals: one CTA, chunked inclusive scan.
__global__ void ivf_offsets_kernel(const int64_t* __restrict__ totals, int K,
                                   int64_t* __restrict__ offsets, int64_t* __restrict__ n_out) {
  __shared__ int64_t part[1024];
  __shared__ int64_t carry;
  if (threadIdx.x == 0) carry = 0;
  __syncthreads();
  for (int k0 = 0; k0 < K; k0 += 1024) {
    const int k = k0 + threadIdx.x;
    part[threadIdx.x] = (k < K) ? totals[k] : 0;
    __syncthreads();
    for (int off = 1; off < 1024; off <<= 1) {
      const int64_t v = (threadIdx.x >= off) ? part[threadIdx.x - off] : 0;
      __syncthreads();
      part[threadIdx.x] += v;
      __syncthreads();
    }
    if (k < K) offsets[k + 1] = carry + part[threadIdx.x];
    __syncthreads();
    if (threadIdx.x == 0) carry += part[1023];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    offsets[0] = 0;
    if (n_out) *n_out = carry;
  }
}

// One thread per counting block: its vectors in index order, each entry at
// offsets[c] + cursor[b][c]++ (the cursor row is owned by this thread alone).
__global__ void ivf_fill_kernel(const int32_t* __restrict__ ids, int64_t n, int m, int K,
                                int nblk, int* __restrict__ cursor,
                                const int64_t* __restrict__ offsets, int64_t* __restrict__ entries) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= nblk) return;
  int* cur = cursor + (size_t)b * K;
  const int64_t i0 = (int64_t)b * kIvfBlk;
  const int64_t i1 = min(n, i0 + kIvfBlk);
  for (int64_t i = i0; i < i1; ++i)
    for (int r = 0; r < m; ++r) {
      const int c = ids[i * m + r];
      if (c >= 0 && c < K) entries[offsets[c] + cur[c]++] = i;
    }
}

// (d, i) lexicographic order; NaN never precedes anything.
__device__ __forceinline__ bool lex_less(float da, int64_t ia, float db, int64_t ib) {
  return da < db || (da == db && ia < ib);
}

}  // namespace

namespace {

// Block-wide lexicographic minimum of (d, i) with the proposing thread in t; every
// thread receives the winner.  rd / ri / rt: shared scratch of blockDim.x entries.
__device__ void block_argmin(float d, int64_t i, float* rd, int64_t* ri, int* rt, float* od,
                             int64_t* oi, int* ot) {
  const int tid = threadIdx.x;
  rd[tid] = d;
  ri[tid] = i;
  rt[tid] = tid;
  __syncthreads();
  for (int s = blockDim.x / 2; s > 0; s >>= 1) {
    if (tid < s && lex_less(rd[tid + s], ri[tid + s], rd[tid], ri[tid])) {
      rd[tid] = rd[tid + s];
      ri[tid] = ri[tid + s];
      rt[tid] = rt[tid + s];
    }
    __syncthreads();
  }
  *od = rd[0];
  *oi = ri[0];
  *ot = rt[0];
  __syncthreads();
}

// One CTA per query.  Dynamic shared memory: query [D], centroid distances [K], probes
// [nprobe], per-thread top-k (distance, id) [blockDim][topk], reduction scratch.
__global__ void __launch_bounds__(kIvfThreads)
    ivf_search_kernel(int K, int D, const float* __restrict__ C, const int64_t* __restrict__ off,
                      const int64_t* __restrict__ entries, const float* __restrict__ X,
                      int64_t ldx, const float* __restrict__ Q, int64_t ldq, int nprobe, int topk,
                      int64_t* __restrict__ out_i, float* __restrict__ out_d,
                      int64_t* __restrict__ dco) {
  extern __shared__ __align__(16) unsigned char sm[];
  int64_t* tki = reinterpret_cast<int64_t*>(sm);                       // [T][topk]
  int64_t* ri = tki + (size_t)blockDim.x * topk;                        // [T]
  float* qv = reinterpret_cast<float*>(ri + blockDim.x);               // [D]
  float* dc = qv + D;                                                  // [K]
  float* tkd = dc + K;                                                 // [T][topk]
  float* rd = tkd + (size_t)blockDim.x * topk;                         // [T]
  int* rt = reinterpret_cast<int*>(rd + blockDim.x);                   // [T]
  int* probe = rt + blockDim.x;                                        // [nprobe]
  const int tid = threadIdx.x;
  const int64_t q = blockIdx.x;
  for (int d = tid; d < D; d += blockDim.x) qv[d] = Q[q * ldq + d];
  __syncthreads();
  // (a) distances to the centroids
  for (int k = tid; k < K; k += blockDim.x) {
    const float* c = C + (size_t)k * D;
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = sq_step_ivf(acc, qv[d], c[d]);
    dc[k] = acc;
  }
  __syncthreads();
  // (b) the nprobe nearest, ties to the lower index; a taken centroid becomes NaN
  for (int j = 0; j < nprobe; ++j) {
    float bd = CUDART_NAN_F;
    int64_t bi = INT64_MAX;
    for (int k = tid; k < K; k += blockDim.x)
      if (!isnan(dc[k]) && (isnan(bd) || lex_less(dc[k], k, bd, bi))) { bd = dc[k]; bi = k; }
    if (isnan(bd)) bd = CUDART_INF_F;            // no candidate on this thread
    float wd;
    int64_t wi;
    int wt;
    block_argmin(bd, bi, rd, ri, rt, &wd, &wi, &wt);
    if (tid == 0) {   // no candidate left (non-finite distances): the probe is empty
      probe[j] = (wi == INT64_MAX) ? -1 : (int)wi;
      if (wi != INT64_MAX) dc[wi] = CUDART_NAN_F;
    }
    __syncthreads();
  }
  // (c) exact distances to the entries of the probed lists; per-thread sorted top-k
  float* myd = tkd + (size_t)tid * topk;
  int64_t* myi = tki + (size_t)tid * topk;
  int cnt = 0;
  int64_t scanned = 0;
  for (int j = 0; j < nprobe; ++j) {
    const int c = probe[j];
    if (c < 0) continue;
    const int64_t e0 = off[c], e1 = off[c + 1];
    scanned += e1 - e0;
    for (int64_t e = e0 + tid; e < e1; e += blockDim.x) {
      const int64_t i = entries[e];
      const float* x = X + i * ldx;
      float acc = 0.f;
      for (int d = 0; d < D; ++d) acc = sq_step_ivf(acc, qv[d], x[d]);
      if (cnt == topk && !lex_less(acc, i, myd[topk - 1], myi[topk - 1])) continue;
      bool dup = false;
      for (int r = 0; r < cnt; ++r) dup |= (myi[r] == i);
      if (dup) continue;
      int r = (cnt < topk) ? cnt++ : topk - 1;
      while (r > 0 && lex_less(acc, i, myd[r - 1], myi[r - 1])) {
        myd[r] = myd[r - 1];
        myi[r] = myi[r - 1];
        --r;
      }
      myd[r] = acc;
      myi[r] = i;
    }
  }
  // (d) merge: repeatedly take the smallest head; a vector met twice is emitted once
  int head = 0, emitted = 0;
  int64_t last = -1;
  for (int round = 0; round < (int)blockDim.x * topk + 1 && emitted < topk; ++round) {
    const bool has = head < cnt;
    float wd;
    int64_t wi;
    int wt;
    block_argmin(has ? myd[head] : CUDART_INF_F, has ? myi[head] : INT64_MAX, rd, ri, rt, &wd,
                 &wi, &wt);
    if (wi == INT64_MAX) break;
    if (wi != last) {
      if (tid == 0) {
        out_i[q * topk + emitted] = wi;
        out_d[q * topk + emitted] = wd;
      }
      ++emitted;
      last = wi;
    }
    if (tid == wt) ++head;
  }
  for (int r = emitted + tid; r < topk; r += blockDim.x) {
    out_i[q * topk + r] = -1;
    out_d[q * topk + r] = CUDART_INF_F;
  }
  if (tid == 0 && dco) dco[q] = scanned;
}

}  // namespace

// ------------------------------------------------------------------ launchers
size_t ivf_build_scratch_bytes(int64_t n, int K) {
  const int64_t nblk = (n + kIvfBlk - 1) / kIvfBlk;
  return (size_t)(nblk * K * 4 + 256) / 256 * 256 + (size_t)K * 8 + 256;
}

cudaError_t launch_ivf_build(int K, const int32_t* ids, int64_t n, int m, int64_t* offsets,
                             int64_t* entries, int64_t* n_entries, void* scratch,
                             cudaStream_t s) {
  const int nblk = (int)((n + kIvfBlk - 1) / kIvfBlk);
  int* counts = static_cast<int*>(scratch);
  int64_t* totals = reinterpret_cast<int64_t*>(static_cast<char*>(scratch) +
                                               ((size_t)nblk * K * 4 + 256) / 256 * 256);
  const size_t hist_bytes = (size_t)K * sizeof(int);
  cudaError_t e = cudaFuncSetAttribute(ivf_count_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)hist_bytes);
  if (e != cudaSuccess) return e;
  ivf_count_kernel<<<nblk, kIvfThreads, hist_bytes, s>>>(ids, n, m, K, counts);
  ivf_colscan_kernel<<<(K + 255) / 256, 256, 0, s>>>(counts, nblk, K, totals);
  ivf_offsets_kernel<<<1, 1024, 0, s>>>(totals, K, offsets, n_entries);
  ivf_fill_kernel<<<(nblk + 127) / 128, 128, 0, s>>>(ids, n, m, K, nblk, counts, offsets, entries);
  return cudaGetLastError();
}

size_t ivf_search_smem(int K, int D, int nprobe, int topk) {
  return (size_t)kIvfThreads * topk * (8 + 4) + (size_t)kIvfThreads * (8 + 4 + 4) +
         (size_t)(D + K) * 4 + (size_t)nprobe * 4 + 64;
}

cudaError_t launch_ivf_search(int K, int D, const float* C, const int64_t* offsets,
                              const int64_t* entries, const float* X, int64_t ldx, const float* Q,
                              int64_t nq, int64_t ldq, int nprobe, int topk, int64_t* out_i,
                              float* out_d, int64_t* dco, cudaStream_t s) {
  const size_t smem = ivf_search_smem(K, D, nprobe, topk);
  cudaError_t e = cudaFuncSetAttribute(ivf_search_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  ivf_search_kernel<<<(unsigned)nq, kIvfThreads, smem, s>>>(K, D, C, offsets, entries, X, ldx, Q,
                                                              ldq, nprobe, topk, out_i, out_d, dco);
  return cudaGetLastError();
}

}  // namespace fgmm
