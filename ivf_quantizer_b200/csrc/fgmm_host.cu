// Host side of the C-ABI declared in include/fgmm.h: argument checks, workspace
// ownership, the chunk loop over N and the kernel sequence of one EM step.
//
// One EM step ("Flash-GMM: A Memory-Efficient Kernel for Scalable Soft
// Clustering", §3.1, Algorithm 1) is enqueued as
//   prep                       parameters -> padded means / precisions / constants
//   for each chunk of <= kChunk points:
//     sweep 1 (log-sum-exp)    log Z_i for the chunk, partial log-likelihood
//     ll_accumulate            adds the chunk's partials in a fixed order
//     sweep 2 (statistics)     recompute, responsibilities, sufficient statistics
//   M-step + finalize          Eqs. (1)-(3), weights, log-likelihood, status
// Every buffer the step touches is O(K D) or O(kChunk): device memory beyond X
// does not grow with N.
#include <math.h>
#include <stdio.h>
#include <string.h>
#include <errno.h>
#include <fcntl.h>
#include <unistd.h>

#include <new>

#include "fgmm_internal.h"

#include <vector>

using namespace fgmm;

// Streaming of X from host memory (fgmm_em_step_host): two device staging buffers of
// one chunk each, filled on a copy stream while the compute stream works on the other.
// Streaming from a reader (fgmm_em_step_reader, _file) adds two pinned host buffers
// that the reader fills, each refilled only after its previous copy has completed.
struct HostStaging {
  void* buf[2] = {nullptr, nullptr};
  void* pin[2] = {nullptr, nullptr};
  cudaStream_t cs = nullptr;
  cudaEvent_t copied[2] = {nullptr, nullptr};
  cudaEvent_t consumed[2] = {nullptr, nullptr};
  uint64_t seq = 0;
  void release() {
    for (int b = 0; b < 2; ++b) {
      if (buf[b]) cudaFree(buf[b]);
      if (pin[b]) cudaFreeHost(pin[b]);
      if (copied[b]) cudaEventDestroy(copied[b]);
      if (consumed[b]) cudaEventDestroy(consumed[b]);
      buf[b] = pin[b] = nullptr;
      copied[b] = consumed[b] = nullptr;
    }
    if (cs) cudaStreamDestroy(cs);
    cs = nullptr;
  }
};

// A reader of X (fgmm_read_fn and its context), for the streamed steps.
struct ReaderSrc {
  fgmm_read_fn fn;
  void* ctx;
};

struct fgmm_ctx {
  fgmm::Ctx c;
  HostStaging hs;
};

// Optional per-launch event timing (fgmm_profile_*).  Events are pooled and
// reused after each read; gate snapshots go to pinned host blocks.
struct fgmm::Profiler {
  static constexpr int kSnapBlock = 4096;
  bool enabled = false;
  int64_t launches = 0;
  struct Rec {
    cudaEvent_t a, b;
    int kernel;
    int64_t snap;  // index of the gate snapshot, -1 for an ungated launch
    int required;
  };
  std::vector<Rec> recs;
  std::vector<cudaEvent_t> pool;
  std::vector<int*> snaps;  // pinned blocks of kSnapBlock words
  int64_t nsnap = 0;
  cudaEvent_t pending = nullptr;
  int64_t pending_snap = -1;
  int pending_required = 0;
  // The gate words change only between passes over the data, so within one pass every
  // launch behind the same gate shares one snapshot (one small copy per gate and pass
  // instead of one per launch); prof_gates_changed() starts a new epoch.
  std::vector<std::pair<const int*, int64_t>> gate_snap;
  cudaEvent_t get() {
    if (!pool.empty()) {
      cudaEvent_t e = pool.back();
      pool.pop_back();
      return e;
    }
    cudaEvent_t e = nullptr;
    cudaEventCreate(&e);
    return e;
  }
  int* snap_slot(int64_t i) { return snaps[i / kSnapBlock] + i % kSnapBlock; }
  int64_t new_snap() {
    if (nsnap == (int64_t)snaps.size() * kSnapBlock) {
      int* blk = nullptr;
      if (cudaHostAlloc((void**)&blk, kSnapBlock * sizeof(int), cudaHostAllocDefault) !=
          cudaSuccess)
        return -1;
      snaps.push_back(blk);
    }
    return nsnap++;
  }
  ~Profiler() {
    for (auto& r : recs) {
      cudaEventDestroy(r.a);
      cudaEventDestroy(r.b);
    }
    for (auto e : pool) cudaEventDestroy(e);
    if (pending) cudaEventDestroy(pending);
    for (int* blk : snaps) cudaFreeHost(blk);
  }
};

namespace {
const char* const kKernelNames[fgmm::KI_COUNT] = {
    "tc_center",   "tc_prep",   "tc_convert",  "tc_lse",         "tc_stats",
    "prep_simt",   "lse_simt",  "ll_accumulate", "stats_simt",   "reduce_stats", "mstep",
    "finalize",    "soft_assign", "auto_check", "redo_reset",    "remask",
    "stiff_compact", "side_lse", "ll_partials", "side_stats",    "side_reduce",
    "km_assign",   "km_seed_update", "tc_order", "tc_gather"};
static_assert(fgmm::KI_COUNT == FGMM_PROF_KERNELS, "kernel table and public arrays differ");
}  // namespace

namespace fgmm {
void prof_begin(const Ctx& c, KernelId, cudaStream_t s, const int* gate, int required) {
  Profiler* p = c.prof;
  if (!p) return;
  ++p->launches;
  if (!p->enabled) return;
  p->pending_snap = -1;
  if (gate) {
    int64_t i = -1;
    for (auto& gs : p->gate_snap)
      if (gs.first == gate) i = gs.second;
    if (i < 0) {
      i = p->new_snap();
      if (i >= 0 &&
          cudaMemcpyAsync(p->snap_slot(i), gate, sizeof(int), cudaMemcpyDeviceToHost, s) !=
              cudaSuccess)
        i = -1;
      if (i >= 0) p->gate_snap.push_back({gate, i});
    }
    if (i >= 0) {
      p->pending_snap = i;
      p->pending_required = required;
    }
  }
  p->pending = p->get();
  cudaEventRecord(p->pending, s);
}
void prof_gates_changed(const Ctx& c) {
  if (c.prof) c.prof->gate_snap.clear();
}
void prof_extra_launch(const Ctx& c) {
  if (c.prof) ++c.prof->launches;
}

void prof_end(const Ctx& c, KernelId k, cudaStream_t s) {
  Profiler* p = c.prof;
  if (!p || !p->enabled || !p->pending) return;
  cudaEvent_t b = p->get();
  cudaEventRecord(b, s);
  p->recs.push_back({p->pending, b, (int)k, p->pending_snap, p->pending_required});
  p->pending = nullptr;
}
}  // namespace fgmm

namespace {

bool valid_dtype(int t) { return t == FGMM_F32 || t == FGMM_BF16; }
size_t dtype_bytes(int t) { return t == FGMM_BF16 ? 2 : 4; }

int map_cuda(cudaError_t e) {
  if (e == cudaSuccess) return FGMM_OK;
  if (e == cudaErrorMemoryAllocation) return FGMM_ERR_OOM;
  return FGMM_ERR_CUDA;
}

void free_ws(Workspace& w) {
  void* ptrs[] = {w.mu,     w.prec,   w.cconst, w.logz, w.ll_tiles, w.ll_total,
                  w.stats,  w.nk,     w.status, w.center, w.dscale, w.wop,
                  w.tck,    w.tks,    w.xop,    w.mode, w.stiff,    w.stiff_list, w.n_stiff,
                  w.tce,    w.acut,   w.alist,  w.nalist,
                  w.side_part, w.mode2, w.canon, w.tcraw, w.tcm, w.tcpk, w.tckf, w.lzlow, w.lpart, w.lpartf,
                  w.side_flag, w.pair_cnt, w.pair_j, w.pair_l, w.flagged, w.n_flagged, w.flag_cnt, w.km_word,
                  w.grey, w.grey_pos,
                  w.grey_stats,
                  w.lbuf, w.bmx, w.bmask, w.perm, w.perm2, w.lzp, w.ord_hist, w.ord_tot, w.tmask, w.tlist, w.tcnt};
  for (void* p : ptrs)
    if (p) cudaFree(p);
  w = Workspace{};
}

template <typename T>
cudaError_t alloc(T** p, size_t count, size_t* total) {
  *total += count * sizeof(T);
  return cudaMalloc((void**)p, count * sizeof(T));
}

size_t stats_bytes(const Workspace& w) {
  return (size_t)w.slots * w.KpS * (1 + 2 * (size_t)w.Dp) * sizeof(double);
}

cudaError_t alloc_ws(Ctx& c) {
  Workspace& w = c.ws;
  w.Kp = round_up(c.K, kKB);
  w.Dp = round_up(c.D, kDC);
  w.KpS = round_up(c.K, 128);
  w.Kt = w.KpS;
  w.Dq = w.Dp;
  w.K1 = 2 * w.Dq;
  const bool tc = tc_supported(c);
  int s_tc = c.num_sms / (w.Kt / 128);
  if (s_tc < 1) s_tc = 1;
  // the tensor-core statistics sweep writes up to 2 s_tc slots (block skipping)
  w.slots = tc && 2 * s_tc > kSlices ? 2 * s_tc : kSlices;
  size_t t = 0;
  cudaError_t e;
  const size_t kd = (size_t)w.Kp * w.Dp;
  if ((e = alloc(&w.mu, kd, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.prec, kd, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.cconst, (size_t)w.Kp, &t)) != cudaSuccess) return e;
  if (w.Dp > kFC && w.Kp <= kLbufMaxKp &&
      (e = alloc(&w.lbuf, (size_t)kChunk * w.Kp, &t)) != cudaSuccess)
    return e;
  if ((e = alloc(&w.logz, (size_t)kChunk, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.ll_tiles, (size_t)(kChunk / 32), &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.ll_total, (size_t)1, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.canon, (size_t)c.K * (1 + 2 * (size_t)c.D) + 1, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.stats, stats_bytes(w) / sizeof(double), &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.nk, (size_t)w.KpS, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.status, (size_t)1, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.km_word, (size_t)2, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.mode, (size_t)1, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.mode2, (size_t)1, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.center, (size_t)w.Dq, &t)) != cudaSuccess) return e;
  if ((e = alloc(&w.dscale, (size_t)w.Dq, &t)) != cudaSuccess) return e;
  if ((e = cudaMemset(w.status, 0, sizeof(int))) != cudaSuccess) return e;
  if ((e = cudaMemset(w.center, 0, w.Dq * sizeof(float))) != cudaSuccess) return e;
  if ((e = cudaMemset(w.dscale, 0, w.Dq * sizeof(float))) != cudaSuccess) return e;
  // the previous step's N_k feeds AUTO's "about to collapse" test: start far above it
  if ((e = cudaMemset(w.nk, 0x7F, (size_t)w.KpS * sizeof(double))) != cudaSuccess) return e;
  if (tc) {
    if ((e = alloc(&w.stiff, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.stiff_list, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.n_stiff, (size_t)2, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.grey, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.grey_pos, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.grey_stats, (size_t)kSideMaxStiff * (1 + 2 * (size_t)w.Dp), &t)) !=
        cudaSuccess)
      return e;
    if ((e = cudaMemset(w.grey, 0, (size_t)w.Kt * sizeof(int))) != cudaSuccess) return e;
    if ((e = alloc(&w.side_part, (size_t)kSideParts * kSideMaxStiff * (1 + 2 * (size_t)w.Dp), &t)) !=
        cudaSuccess)
      return e;
    if ((e = cudaMemset(w.stiff, 0, (size_t)w.Kt * sizeof(int))) != cudaSuccess) return e;
    if ((e = cudaMemset(w.n_stiff, 0, 2 * sizeof(int))) != cudaSuccess) return e;
    if ((e = alloc(&w.wop, (size_t)2 * w.Kt * w.K1, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tck, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tks, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tcraw, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tcm, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tcpk, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tckf, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.lzlow, (size_t)1, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.lpart, (size_t)(w.Kt / 128) * kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.lpartf, (size_t)(w.Kt / 128) * kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tce, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.acut, (size_t)1, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.alist, (size_t)w.Kt, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.nalist, (size_t)1, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.side_flag, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = cudaMemset(w.side_flag, 0, (size_t)kChunk)) != cudaSuccess) return e;
    if ((e = alloc(&w.pair_cnt, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.pair_j, (size_t)kChunk * kSidePairs, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.pair_l, (size_t)kChunk * kSidePairs, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.flagged, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.n_flagged, (size_t)1, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.flag_cnt, (size_t)(kChunk / 4096), &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.xop, (size_t)2 * kChunk * w.K1, &t)) != cudaSuccess) return e;
    // rows past the end of a short chunk are read by the tensor cores (and multiplied
    // by r = 0): keep them finite from the start
    if ((e = cudaMemset(w.xop, 0, (size_t)2 * kChunk * w.K1 * sizeof(__half))) != cudaSuccess)
      return e;
  }
  // block skipping (tensor-core statistics sweep, or the CUDA-core one for 4 to 32
  // blocks of 128 components)
  const int nkb_simt = (w.Kp + 127) / 128;
  const bool simt_blocks = nkb_simt >= 4 && nkb_simt <= kSkipMaxBlocks;
  if (tc || simt_blocks) {
    if ((e = alloc(&w.bmask, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.perm, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.perm2, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.lzp, (size_t)kChunk, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.ord_tot, (size_t)kOrdBuckets, &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.ord_hist, (size_t)(kChunk / kOrdPts) * kOrdBuckets, &t)) != cudaSuccess)
      return e;
    if ((e = alloc(&w.tmask, (size_t)(kChunk / kTP), &t)) != cudaSuccess) return e;
    if ((e = alloc(&w.tlist, (size_t)kSkipMaxBlocks * (kChunk / kTP), &t)) != cudaSuccess)
      return e;
    if ((e = alloc(&w.tcnt, (size_t)kSkipMaxBlocks, &t)) != cudaSuccess) return e;
  }
  if (simt_blocks && (e = alloc(&w.bmx, (size_t)kChunk * (w.Kp / kKB), &t)) != cudaSuccess)
    return e;
  w.bytes = t;
  if (tc && (e = tc_init(c)) != cudaSuccess) return e;
  return cudaSuccess;
}

int check_x(const fgmm_ctx* h, const void* X, int x_dtype, int64_t N, int64_t ldx) {
  if (!h || !X) return FGMM_ERR_INVALID_ARG;
  if (!valid_dtype(x_dtype)) return FGMM_ERR_INVALID_ARG;
  if (N < 1 || ldx < h->c.D) return FGMM_ERR_INVALID_ARG;
  return FGMM_OK;
}

int set_device(const Ctx& c) {
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return FGMM_ERR_CUDA;
  if (cur != c.device && cudaSetDevice(c.device) != cudaSuccess) return FGMM_ERR_CUDA;
  return FGMM_OK;
}

}  // namespace

extern "C" {

int fgmm_create(int K, int D, int cov_type, double reg_covar, fgmm_handle* out) {
  if (!out) return FGMM_ERR_INVALID_ARG;
  *out = nullptr;
  if (K < 1 || D < 1 || (cov_type != FGMM_COV_DIAG && cov_type != FGMM_COV_SPHERICAL))
    return FGMM_ERR_INVALID_ARG;
  if (!(reg_covar >= 0.0) || !isfinite(reg_covar)) return FGMM_ERR_INVALID_ARG;
  // 32-bit index arithmetic inside the kernels: bound the parameter block.
  if ((int64_t)K * D > (int64_t)1 << 28 || K > (1 << 24) || D > (1 << 16))
    return FGMM_ERR_UNSUPPORTED;
  fgmm_ctx* h = new (std::nothrow) fgmm_ctx();
  if (!h) return FGMM_ERR_OOM;
  h->c.K = K;
  h->c.D = D;
  h->c.cov = cov_type;
  h->c.reg = reg_covar;
  h->c.prec = FGMM_PREC_AUTO;
  if (cudaGetDevice(&h->c.device) != cudaSuccess ||
      cudaDeviceGetAttribute(&h->c.num_sms, cudaDevAttrMultiProcessorCount, h->c.device) !=
          cudaSuccess) {
    delete h;
    return FGMM_ERR_CUDA;
  }
  h->c.prof = new (std::nothrow) Profiler();
  cudaError_t e = alloc_ws(h->c);
  if (e != cudaSuccess) {
    free_ws(h->c.ws);
    delete h->c.prof;
    delete h;
    cudaGetLastError();
    return map_cuda(e);
  }
  *out = h;
  return FGMM_OK;
}

int fgmm_destroy(fgmm_handle h) {
  if (!h) return FGMM_OK;
  int rc = set_device(h->c);
  cudaDeviceSynchronize();
  free_ws(h->c.ws);
  h->hs.release();
  delete h->c.prof;
  delete h;
  return rc;
}

int fgmm_set_precision(fgmm_handle h, int prec) {
  if (!h) return FGMM_ERR_INVALID_ARG;
  if (prec != FGMM_PREC_FP32 && prec != FGMM_PREC_FP16X3 && prec != FGMM_PREC_FP16 &&
      prec != FGMM_PREC_AUTO)
    return FGMM_ERR_INVALID_ARG;
  if ((prec == FGMM_PREC_FP16X3 || prec == FGMM_PREC_FP16) && !h->c.tc.ready)
    return FGMM_ERR_UNSUPPORTED;
  h->c.prec = prec;
  return FGMM_OK;
}

int fgmm_get_precision(fgmm_handle h, int* prec_out) {
  if (!h || !prec_out) return FGMM_ERR_INVALID_ARG;
  *prec_out = h->c.prec;
  return FGMM_OK;
}

int fgmm_set_block_skip(fgmm_handle h, int enable) {
  if (!h) return FGMM_ERR_INVALID_ARG;
  h->c.skip = enable != 0;
  return FGMM_OK;
}

int fgmm_get_block_skip(fgmm_handle h, int* enable_out) {
  if (!h || !enable_out) return FGMM_ERR_INVALID_ARG;
  *enable_out = h->c.skip ? 1 : 0;
  return FGMM_OK;
}

int fgmm_workspace_bytes(fgmm_handle h, size_t* bytes_out) {
  if (!h || !bytes_out) return FGMM_ERR_INVALID_ARG;
  *bytes_out = h->c.ws.bytes;
  return FGMM_OK;
}

namespace {
// Everything of one EM iteration up to the exchange-form statistics (written to `st`):
// preparation, both sweeps over all chunks on the selected path(s), slot reduction.
// Device staging for host-resident X: buffers, copy stream and events, made on first use.
cudaError_t ensure_staging(fgmm_ctx* h) {
  HostStaging& hs = h->hs;
  if (hs.cs) return cudaSuccess;
  const size_t bytes = (size_t)kChunk * h->c.D * sizeof(float);
  cudaError_t e;
  for (int b = 0; b < 2; ++b) {
    if ((e = cudaMalloc(&hs.buf[b], bytes)) != cudaSuccess) break;
    if ((e = cudaEventCreateWithFlags(&hs.copied[b], cudaEventDisableTiming)) != cudaSuccess) break;
    if ((e = cudaEventCreateWithFlags(&hs.consumed[b], cudaEventDisableTiming)) != cudaSuccess) break;
  }
  if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&hs.cs, cudaStreamNonBlocking);
  if (e != cudaSuccess) hs.release();
  return e;
}

// Pinned host buffers for a reader, made on first use (after ensure_staging).
cudaError_t ensure_pinned(fgmm_ctx* h) {
  HostStaging& hs = h->hs;
  const size_t bytes = (size_t)kChunk * h->c.D * sizeof(float);
  cudaError_t e = cudaSuccess;
  for (int b = 0; b < 2 && e == cudaSuccess; ++b)
    if (!hs.pin[b]) e = cudaHostAlloc(&hs.pin[b], bytes, cudaHostAllocDefault);
  return e;
}

int read_word(const int* dev, int* out, cudaStream_t s) {
  cudaError_t e = cudaMemcpyAsync(out, dev, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  return map_cuda(e);
}

int run_partial(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                const float* weights, const float* means, const float* vars, double* st,
                float* logz_out, fgmm_stream_t stream, bool host_x = false,
                bool want_stats = true, const ReaderSrc* rd = nullptr) {
  // a reader stands in for X: the checks see a dummy non-null pointer, rows of D
  int rc = check_x(h, rd ? (const void*)rd : X, x_dtype, N, rd ? (h ? h->c.D : 0) : ldx);
  if (rc) return rc;
  if (rd) {
    host_x = true;
    ldx = h->c.D;
  }
  if (!weights || !means || !vars) return FGMM_ERR_INVALID_ARG;
  Ctx& c = h->c;
  if ((rc = set_device(c))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  const Workspace& w = c.ws;
  if (host_x && (e = ensure_staging(h)) != cudaSuccess) return map_cuda(e);
  if (rd && (e = ensure_pinned(h)) != cudaSuccess) return map_cuda(e);
  prof_gates_changed(c);
  // which path(s) to enqueue: FP32 -> CUDA cores; FP16X3 -> tensor cores; AUTO ->
  // both, each kernel returning at once unless the device-side mode word (set by the
  // tensor-core preparation's conditioning check) selects its path
  const bool auto_mode = c.prec == FGMM_PREC_AUTO && c.tc.ready;
  const bool run_tc =
      (c.prec == FGMM_PREC_FP16X3 || c.prec == FGMM_PREC_FP16 || auto_mode) && c.tc.ready;
  const bool run_simt = c.prec == FGMM_PREC_FP32 || !c.tc.ready || auto_mode;
  const int fixed_mode = run_tc && !run_simt ? kModeTensor : kModeSimt;
  const int* mode = auto_mode ? w.mode : nullptr;
  if (run_tc && !host_x && x_dtype == FGMM_F32 && ((uintptr_t)X % 4 != 0))
    return FGMM_ERR_INVALID_ARG;
  if ((e = cudaMemsetAsync(w.ll_total, 0, sizeof(double), s)) != cudaSuccess) return map_cuda(e);
  if ((e = cudaMemsetAsync(w.stats, 0, stats_bytes(w), s)) != cudaSuccess) return map_cuda(e);
  if (auto_mode && (e = cudaMemsetAsync(w.mode, 0, sizeof(int), s)) != cudaSuccess)
    return map_cuda(e);
  if (run_simt && (e = launch_prep_simt(c, weights, means, vars, s)) != cudaSuccess)
    return map_cuda(e);
  if (run_tc) {
    if ((e = launch_tc_prep(c, weights, means, vars, auto_mode, s)) != cudaSuccess)
      return map_cuda(e);
    if ((e = launch_stiff_compact(c, auto_mode ? w.mode : nullptr, w.mode, s)) != cudaSuccess)
      return map_cuda(e);
  }
  const size_t eb = dtype_bytes(x_dtype);
  // The rows of chunk [c0, c0 + nc) on the device: X itself, or (host X) a staging
  // buffer filled on the copy stream once the kernels that last read it are done; the
  // copy of the next chunk overlaps the kernels of this one.
  HostStaging& hs = h->hs;
  cudaError_t copy_err = cudaSuccess;
  bool read_failed = false;
  auto acquire = [&](int64_t c0, int64_t nc, const void** Xc, int64_t* ldc) -> int {
    if (!host_x) {
      *Xc = (const char*)X + (size_t)c0 * ldx * eb;
      *ldc = ldx;
      return -1;
    }
    const int b = (int)(hs.seq++ & 1);
    const void* src = rd ? nullptr : (const void*)((const char*)X + (size_t)c0 * ldx * eb);
    cudaError_t r = cudaSuccess;
    if (rd) {
      // the pinned buffer's previous copy to the device (recorded as copied[b]) must be
      // complete before the reader overwrites it
      r = cudaEventSynchronize(hs.copied[b]);
      if (r == cudaSuccess && !read_failed && rd->fn(rd->ctx, c0, nc, hs.pin[b]) != 0)
        read_failed = true;
      if (read_failed) {   // no copy: the caller enqueues nothing for this chunk
        *Xc = hs.buf[b];
        *ldc = c.D;
        if (r != cudaSuccess && copy_err == cudaSuccess) copy_err = r;
        return b;
      }
      src = hs.pin[b];
    }
    if (r == cudaSuccess) r = cudaStreamWaitEvent(hs.cs, hs.consumed[b], 0);
    if (r == cudaSuccess)
      r = cudaMemcpy2DAsync(hs.buf[b], (size_t)c.D * eb, src, (size_t)ldx * eb,
                            (size_t)c.D * eb, (size_t)nc, cudaMemcpyHostToDevice, hs.cs);
    if (r == cudaSuccess) r = cudaEventRecord(hs.copied[b], hs.cs);
    if (r == cudaSuccess) r = cudaStreamWaitEvent(s, hs.copied[b], 0);
    if (r != cudaSuccess && copy_err == cudaSuccess) copy_err = r;
    *Xc = hs.buf[b];
    *ldc = c.D;
    return b;
  };
  auto release = [&](int b) {
    if (b >= 0) cudaEventRecord(hs.consumed[b], s);
  };
  // one tensor-core pass over all chunks, its kernels gated on the word `gate`
  prof_gates_changed(c);
  auto tc_pass = [&](const int* gate) -> cudaError_t {
    prof_gates_changed(c);   // the gate words were last written before this pass
    // the grey components' side-path statistics of this pass accumulate from zero
    cudaError_t r = cudaMemsetAsync(w.grey_stats, 0,
                                    (size_t)kSideMaxStiff * (1 + 2 * (size_t)w.Dp) * sizeof(double), s);
    for (int64_t c0 = 0; c0 < N && r == cudaSuccess; c0 += kChunk) {
      const int64_t nc = (N - c0 < kChunk) ? N - c0 : kChunk;
      const void* Xc;
      int64_t ldc;
      const int b = acquire(c0, nc, &Xc, &ldc);
      if (read_failed) {   // nothing more of this pass is enqueued
        release(b);
        break;
      }
      float* lzo = logz_out ? logz_out + c0 : nullptr;
      if ((r = launch_tc_convert(c, Xc, x_dtype, nc, ldc, nullptr, gate, s)) == cudaSuccess &&
          (r = launch_tc_lse(c, nc, lzo, gate, s)) == cudaSuccess &&
          // stiff components (AUTO) join log Z here; then the chunk's log-likelihood
          (r = launch_side_lse(c, Xc, x_dtype, nc, ldc, lzo, gate, s)) == cudaSuccess &&
          (r = launch_ll_accumulate(c, nc, gate, fixed_mode, kModeTensor, s)) == cudaSuccess &&
          want_stats &&
          // block skipping: sweep 2 runs on phi rewritten in the order of the block masks
          (!tc_skip(c) || (r = launch_tc_order(c, Xc, x_dtype, nc, ldc, gate, s)) == cudaSuccess) &&
          (r = launch_tc_stats(c, nc, gate, s)) == cudaSuccess)
        r = launch_side_stats(c, Xc, x_dtype, nc, ldc, gate, s);
      release(b);
      if (r == cudaSuccess) r = copy_err;
    }
    return r;
  };
  if (run_tc) {
    if (auto_mode && (e = cudaMemsetAsync(w.mode2, 0xFF, sizeof(int), s)) != cudaSuccess)
      return map_cuda(e);
    // With host X a pass whose gate is off would still copy every chunk, so under AUTO
    // the gate words are read back (one synchronisation each) before such a pass.
    int word = kModeTensor;
    if (host_x && auto_mode && (rc = read_word(w.mode, &word, s))) return rc;
    if (word == kModeTensor && (e = tc_pass(mode)) != cudaSuccess) return map_cuda(e);
    if (read_failed) return FGMM_ERR_IO;
    if (auto_mode && want_stats) {
      // AUTO: components whose new variance would lose accuracy to cancellation move to
      // the side path and the pass is redone (gated on mode2); a failure after that sends
      // the step to the CUDA-core kernels below (gated on mode)
      if ((e = launch_auto_check(c, 0, s)) != cudaSuccess) return map_cuda(e);
      prof_gates_changed(c);
      if ((e = launch_stiff_compact(c, w.mode2, w.mode, s)) != cudaSuccess) return map_cuda(e);
      word = kModeTensor;
      if (host_x && (rc = read_word(w.mode2, &word, s))) return rc;
      if (word == kModeTensor && (e = tc_pass(w.mode2)) != cudaSuccess) return map_cuda(e);
      if ((e = launch_auto_check(c, 1, s)) != cudaSuccess) return map_cuda(e);
    }
  }
  prof_gates_changed(c);
  int simt_word = kModeSimt;
  if (run_simt && host_x && auto_mode && (rc = read_word(w.mode, &simt_word, s))) return rc;
  if (run_simt && simt_word == kModeSimt) {
    for (int64_t c0 = 0; c0 < N; c0 += kChunk) {
      const int64_t nc = (N - c0 < kChunk) ? N - c0 : kChunk;
      const void* Xc;
      int64_t ldc;
      const int b = acquire(c0, nc, &Xc, &ldc);
      if (read_failed) {
        release(b);
        break;
      }
      float* lzo = logz_out ? logz_out + c0 : nullptr;
      if ((e = launch_lse_simt(c, Xc, x_dtype, nc, ldc, lzo, want_stats, mode, s)) == cudaSuccess &&
          (e = launch_ll_accumulate(c, nc, mode, fixed_mode, kModeSimt, s)) == cudaSuccess &&
          want_stats &&
          (!simt_skip(c) || (e = launch_simt_order(c, nc, mode, s)) == cudaSuccess))
        e = launch_stats_simt(c, Xc, x_dtype, nc, ldc, mode, s);
      release(b);
      if (e == cudaSuccess) e = copy_err;
      if (e != cudaSuccess) return map_cuda(e);
    }
  }
  if (read_failed) return FGMM_ERR_IO;
  if (want_stats && (e = launch_reduce_stats(c, means, st, mode, fixed_mode, s)) != cudaSuccess)
    return map_cuda(e);
  h->c.last_auto = auto_mode;
  h->c.last_path = fixed_mode != kModeTensor ? FGMM_PREC_FP32
                   : c.prec == FGMM_PREC_FP16   ? FGMM_PREC_FP16
                                                : FGMM_PREC_FP16X3;
  h->c.last_nc = N - (N - 1) / kChunk * kChunk;
  h->c.last_stats = want_stats;
  return FGMM_OK;
}
}  // namespace

int fgmm_em_step(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                 float* weights, float* means, float* vars, double* loglik_out, float* logz_out,
                 fgmm_stream_t stream) {
  int rc = run_partial(h, X, x_dtype, N, ldx, weights, means, vars,
                       h ? h->c.ws.canon : nullptr, logz_out, stream);
  if (rc) return rc;
  return map_cuda(launch_finish(h->c, h->c.ws.canon, weights, means, vars, loglik_out,
                                (cudaStream_t)stream));
}

int fgmm_em_partial(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                    const float* weights, const float* means, const float* vars,
                    double* stats_out, float* logz_out, fgmm_stream_t stream) {
  if (!stats_out) return FGMM_ERR_INVALID_ARG;
  return run_partial(h, X, x_dtype, N, ldx, weights, means, vars, stats_out, logz_out, stream);
}

int fgmm_em_step_host(fgmm_handle h, const void* X_host, int x_dtype, int64_t N, int64_t ldx,
                      float* weights, float* means, float* vars, double* loglik_out,
                      float* logz_out, fgmm_stream_t stream) {
  int rc = run_partial(h, X_host, x_dtype, N, ldx, weights, means, vars,
                       h ? h->c.ws.canon : nullptr, logz_out, stream, true);
  if (rc) return rc;
  return map_cuda(launch_finish(h->c, h->c.ws.canon, weights, means, vars, loglik_out,
                                (cudaStream_t)stream));
}

int fgmm_em_partial_host(fgmm_handle h, const void* X_host, int x_dtype, int64_t N,
                         int64_t ldx, const float* weights, const float* means,
                         const float* vars, double* stats_out, float* logz_out,
                         fgmm_stream_t stream) {
  if (!stats_out) return FGMM_ERR_INVALID_ARG;
  return run_partial(h, X_host, x_dtype, N, ldx, weights, means, vars, stats_out, logz_out,
                     stream, true);
}

}  // extern "C"

namespace {
// X in a file: rows of row_bytes bytes from byte `offset`, read with pread.
struct FileSrc {
  int fd;
  int64_t offset;
  int64_t row_bytes;
};

int file_read(void* ctx, int64_t row0, int64_t nrows, void* dst) {
  const FileSrc* f = static_cast<const FileSrc*>(ctx);
  char* p = static_cast<char*>(dst);
  int64_t left = nrows * f->row_bytes;
  off_t at = (off_t)(f->offset + row0 * f->row_bytes);
  while (left > 0) {
    const ssize_t got = pread(f->fd, p, (size_t)left, at);
    if (got < 0 && errno == EINTR) continue;
    if (got <= 0) return 1;   // an error, or the file ends before the rows do
    p += got;
    at += got;
    left -= got;
  }
  return 0;
}

// Open the file and run `body` with a reader of it; FGMM_ERR_IO if it cannot be opened.
template <typename Body>
int with_file(fgmm_handle h, const char* path, int64_t offset, int x_dtype, Body body) {
  if (!h || !path || offset < 0 || !valid_dtype(x_dtype)) return FGMM_ERR_INVALID_ARG;
  const int fd = open(path, O_RDONLY);
  if (fd < 0) return FGMM_ERR_IO;
  FileSrc f{fd, offset, (int64_t)h->c.D * (int64_t)dtype_bytes(x_dtype)};
  const ReaderSrc rd{file_read, &f};
  const int rc = body(&rd);
  close(fd);
  return rc;
}
}  // namespace

extern "C" {

int fgmm_em_step_reader(fgmm_handle h, fgmm_read_fn read, void* ctx, int x_dtype, int64_t N,
                        float* weights, float* means, float* vars, double* loglik_out,
                        float* logz_out, fgmm_stream_t stream) {
  if (!h || !read) return FGMM_ERR_INVALID_ARG;
  const ReaderSrc rd{read, ctx};
  int rc = run_partial(h, nullptr, x_dtype, N, 0, weights, means, vars, h->c.ws.canon, logz_out,
                       stream, true, true, &rd);
  if (rc) return rc;
  return map_cuda(launch_finish(h->c, h->c.ws.canon, weights, means, vars, loglik_out,
                                (cudaStream_t)stream));
}

int fgmm_em_partial_reader(fgmm_handle h, fgmm_read_fn read, void* ctx, int x_dtype,
                           int64_t N, const float* weights, const float* means,
                           const float* vars, double* stats_out, float* logz_out,
                           fgmm_stream_t stream) {
  if (!h || !read || !stats_out) return FGMM_ERR_INVALID_ARG;
  const ReaderSrc rd{read, ctx};
  return run_partial(h, nullptr, x_dtype, N, 0, weights, means, vars, stats_out, logz_out,
                     stream, true, true, &rd);
}

int fgmm_em_step_file(fgmm_handle h, const char* path, int64_t offset, int x_dtype, int64_t N,
                      float* weights, float* means, float* vars, double* loglik_out,
                      float* logz_out, fgmm_stream_t stream) {
  return with_file(h, path, offset, x_dtype, [&](const ReaderSrc* rd) {
    return fgmm_em_step_reader(h, rd->fn, rd->ctx, x_dtype, N, weights, means, vars,
                               loglik_out, logz_out, stream);
  });
}

int fgmm_em_partial_file(fgmm_handle h, const char* path, int64_t offset, int x_dtype,
                         int64_t N, const float* weights, const float* means,
                         const float* vars, double* stats_out, float* logz_out,
                         fgmm_stream_t stream) {
  return with_file(h, path, offset, x_dtype, [&](const ReaderSrc* rd) {
    return fgmm_em_partial_reader(h, rd->fn, rd->ctx, x_dtype, N, weights, means, vars,
                                  stats_out, logz_out, stream);
  });
}

int fgmm_em_finish(fgmm_handle h, const double* stats, float* weights, float* means,
                   float* vars, double* loglik_out, fgmm_stream_t stream) {
  if (!h || !stats || !weights || !means || !vars) return FGMM_ERR_INVALID_ARG;
  int rc = set_device(h->c);
  if (rc) return rc;
  return map_cuda(launch_finish(h->c, stats, weights, means, vars, loglik_out,
                                (cudaStream_t)stream));
}

int fgmm_stats_sum(const double* parts, int n_parts, int64_t len, double* out,
                   fgmm_stream_t stream) {
  if (!parts || !out || n_parts < 1 || len < 1) return FGMM_ERR_INVALID_ARG;
  return map_cuda(launch_stats_sum(parts, n_parts, len, out, (cudaStream_t)stream));
}

int fgmm_last_step_path(fgmm_handle h, int* path_out) {
  if (!h || !path_out) return FGMM_ERR_INVALID_ARG;
  if (!h->c.last_auto) {
    *path_out = h->c.last_path;
    return FGMM_OK;
  }
  int rc = set_device(h->c);
  if (rc) return rc;
  int m = 0;
  cudaError_t e = cudaDeviceSynchronize();
  if (e == cudaSuccess) e = cudaMemcpy(&m, h->c.ws.mode, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return map_cuda(e);
  *path_out = m == kModeTensor ? FGMM_PREC_FP16X3 : FGMM_PREC_FP32;
  return FGMM_OK;
}

int fgmm_last_step_info(fgmm_handle h, fgmm_step_info* out) {
  if (!h || !out) return FGMM_ERR_INVALID_ARG;
  int rc = fgmm_last_step_path(h, &out->path);
  if (rc) return rc;
  out->n_stiff = out->n_grey = 0;
  out->skip_pairs = out->skip_pairs_all = -1;
  if (out->path < 0) return FGMM_OK;
  const Ctx& c = h->c;
  const Workspace& w = c.ws;
  if ((rc = set_device(c))) return rc;
  cudaError_t e = cudaDeviceSynchronize();
  int ns[2] = {0, 0};
  if (e == cudaSuccess && c.last_auto && w.n_stiff)
    e = cudaMemcpy(ns, w.n_stiff, sizeof(ns), cudaMemcpyDeviceToHost);
  out->n_stiff = ns[0];
  out->n_grey = ns[1];
  // block lists of the last chunk: 128-point tiles on the tensor cores, 64 on CUDA cores
  const bool tc = out->path == FGMM_PREC_FP16X3 || out->path == FGMM_PREC_FP16;
  const bool skipped = c.last_stats && (tc ? tc_skip(c) : simt_skip(c));
  if (e == cudaSuccess && skipped) {
    const int nkb = tc ? w.Kt / 128 : (w.Kp + 127) / 128;
    const int rows = tc ? 128 : kTP;
    std::vector<int> cnt(nkb);
    e = cudaMemcpy(cnt.data(), w.tcnt, nkb * sizeof(int), cudaMemcpyDeviceToHost);
    int64_t tot = 0;
    for (int v : cnt) tot += v;
    out->skip_pairs = tot;
    out->skip_pairs_all = (int64_t)nkb * ((c.last_nc + rows - 1) / rows);
  }
  return map_cuda(e);
}

int fgmm_fit(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx, float* weights,
             float* means, float* vars, int max_iters, double tol, double* final_loglik_host,
             int* iters_done_host, fgmm_stream_t stream) {
  int rc = check_x(h, X, x_dtype, N, ldx);
  if (rc) return rc;
  if (max_iters < 0 || !(tol >= 0.0)) return FGMM_ERR_INVALID_ARG;
  if (!weights || !means || !vars) return FGMM_ERR_INVALID_ARG;
  if ((rc = set_device(h->c))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  double* d_ll = nullptr;
  cudaError_t e = cudaMalloc(&d_ll, 2 * sizeof(double));
  if (e != cudaSuccess) return map_cuda(e);
  double prev = 0.0, cur = NAN;
  int it = 0;
  for (it = 0; it < max_iters; ++it) {
    rc = fgmm_em_step(h, X, x_dtype, N, ldx, weights, means, vars, d_ll, nullptr, stream);
    if (rc) break;
    if (tol > 0.0) {
      if ((e = cudaMemcpyAsync(&cur, d_ll, sizeof(double), cudaMemcpyDeviceToHost, s)) !=
              cudaSuccess ||
          (e = cudaStreamSynchronize(s)) != cudaSuccess) {
        rc = map_cuda(e);
        break;
      }
      if (it > 0 && fabs(cur - prev) / (double)N < tol) {
        ++it;
        break;
      }
      prev = cur;
    }
  }
  if (!rc) {
    if ((e = cudaMemcpyAsync(&cur, d_ll, sizeof(double), cudaMemcpyDeviceToHost, s)) !=
        cudaSuccess)
      rc = map_cuda(e);
    else if ((e = cudaStreamSynchronize(s)) != cudaSuccess)
      rc = map_cuda(e);
  }
  cudaFree(d_ll);
  if (!rc) rc = fgmm_get_status(h, stream);
  if (final_loglik_host) *final_loglik_host = (max_iters > 0) ? cur : NAN;
  if (iters_done_host) *iters_done_host = it;
  return rc;
}

int fgmm_soft_assign(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     const float* weights, const float* means, const float* vars, int top_m,
                     float r_threshold, int32_t* ids, float* resp, fgmm_stream_t stream) {
  int rc = check_x(h, X, x_dtype, N, ldx);
  if (rc) return rc;
  if (!weights || !means || !vars || !ids) return FGMM_ERR_INVALID_ARG;
  if (top_m < 1 || top_m > FGMM_MAX_TOP_M || top_m > h->c.K) return FGMM_ERR_INVALID_ARG;
  if (!(r_threshold >= 0.f) || !(r_threshold < 1.f)) return FGMM_ERR_INVALID_ARG;
  const Ctx& c = h->c;
  if ((rc = set_device(c))) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  cudaError_t e;
  if ((e = launch_prep_simt(c, weights, means, vars, s)) != cudaSuccess) return map_cuda(e);
  const size_t eb = dtype_bytes(x_dtype);
  // Tensor-core filtered path (split-product modes, 2 to 32 component blocks): sweep 1 on
  // the tensor cores with every component marks, per point, the 128-component blocks
  // whose log-densities come within the cut of log Z; the cut is what the exact result
  // needs (30 nats for log Z and the ranks; -ln(tau) when the threshold reaches further;
  // fp32's exp underflow, 104 nats, when tau = 0) widened by the expanded form's error
  // bounds.  The CUDA-core kernel then evaluates exactly, in the direct form, only those
  // blocks, over the points regrouped by mask.
  const int nkb = c.ws.Kt / 128;
  const bool tc = c.tc.ready && c.ws.bmask && nkb >= 2 && nkb <= kSkipMaxBlocks &&
                  (c.prec == FGMM_PREC_FP16X3 || c.prec == FGMM_PREC_AUTO);
  if (tc) {
    const float base = r_threshold > 0.f ? fmaxf(kSkipCut, -logf(r_threshold) + 1.f) : 104.f;
    if ((e = launch_tc_prep(c, weights, means, vars, false, s, true)) != cudaSuccess ||
        (e = launch_assign_cut(c, base, s)) != cudaSuccess)
      return map_cuda(e);
  }
  for (int64_t c0 = 0; c0 < N; c0 += kChunk) {
    const int64_t nc = (N - c0 < kChunk) ? N - c0 : kChunk;
    const void* Xc = (const char*)X + (size_t)c0 * ldx * eb;
    int32_t* idc = ids + c0 * top_m;
    float* rc_ = resp ? resp + c0 * top_m : nullptr;
    if (tc) {
      if ((e = launch_tc_convert(c, Xc, x_dtype, nc, ldx, nullptr, nullptr, s)) != cudaSuccess ||
          (e = launch_tc_lse(c, nc, nullptr, nullptr, s, true)) != cudaSuccess ||
          (e = launch_assign_order(c, nc, s)) != cudaSuccess ||
          (e = launch_soft_assign_skip(c, Xc, x_dtype, nc, ldx, top_m, r_threshold, idc, rc_, s)) !=
              cudaSuccess)
        return map_cuda(e);
    } else if ((e = launch_soft_assign_simt(c, Xc, x_dtype, nc, ldx, top_m, r_threshold, idc, rc_,
                                            s)) != cudaSuccess) {
      return map_cuda(e);
    }
  }
  return FGMM_OK;
}

int fgmm_get_status(fgmm_handle h, fgmm_stream_t stream) {
  if (!h) return FGMM_ERR_INVALID_ARG;
  int rc = set_device(h->c);
  if (rc) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  int st = 0;
  cudaError_t e;
  if ((e = cudaMemcpyAsync(&st, h->c.ws.status, sizeof(int), cudaMemcpyDeviceToHost, s)) !=
      cudaSuccess)
    return map_cuda(e);
  if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return map_cuda(e);
  if (st != FGMM_OK) {
    if ((e = cudaMemsetAsync(h->c.ws.status, 0, sizeof(int), s)) != cudaSuccess)
      return map_cuda(e);
    if ((e = cudaStreamSynchronize(s)) != cudaSuccess) return map_cuda(e);
  }
  return st;
}

int fgmm_profile_enable(fgmm_handle h, int enable) {
  if (!h || !h->c.prof) return FGMM_ERR_INVALID_ARG;
  h->c.prof->enabled = enable != 0;
  return FGMM_OK;
}

int fgmm_profile_read(fgmm_handle h, fgmm_profile* out, int reset) {
  if (!h || !h->c.prof || !out) return FGMM_ERR_INVALID_ARG;
  int rc = set_device(h->c);
  if (rc) return rc;
  Profiler* p = h->c.prof;
  cudaError_t e = cudaDeviceSynchronize();
  if (e != cudaSuccess) return map_cuda(e);
  fgmm_profile r{};
  r.launches = p->launches;
  for (auto& rec : p->recs) {
    float ms = 0.f;
    if ((e = cudaEventElapsedTime(&ms, rec.a, rec.b)) != cudaSuccess) return map_cuda(e);
    const bool active = rec.snap < 0 || *p->snap_slot(rec.snap) == rec.required;
    r.kernel_launches[rec.kernel]++;
    r.kernel_ms[rec.kernel] += ms;
    if (active) {
      r.kernel_active[rec.kernel]++;
      r.kernel_active_ms[rec.kernel] += ms;
    }
    if (rec.kernel == KI_TC_LSE || rec.kernel == KI_LSE_SIMT) { r.sweep1_launches++; r.sweep1_ms += ms; }
    else if (rec.kernel == KI_TC_STATS || rec.kernel == KI_STATS_SIMT) { r.sweep2_launches++; r.sweep2_ms += ms; }
    else { r.other_launches++; r.other_ms += ms; }
  }
  *out = r;
  if (reset) {
    for (auto& rec : p->recs) {
      p->pool.push_back(rec.a);
      p->pool.push_back(rec.b);
    }
    p->recs.clear();
    p->launches = 0;
    p->nsnap = 0;
    p->gate_snap.clear();
  }
  return FGMM_OK;
}

int fgmm_score_samples(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                       const float* weights, const float* means, const float* vars,
                       float* logz_out, double* loglik_out, fgmm_stream_t stream) {
  if (!logz_out && !loglik_out) return FGMM_ERR_INVALID_ARG;
  int rc = run_partial(h, X, x_dtype, N, ldx, weights, means, vars, nullptr, logz_out, stream,
                       false, false);
  if (rc || !loglik_out) return rc;
  return map_cuda(cudaMemcpyAsync(loglik_out, h->c.ws.ll_total, sizeof(double),
                                  cudaMemcpyDeviceToDevice, (cudaStream_t)stream));
}

int fgmm_fisher_vector(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                       const float* weights, const float* means, const float* vars,
                       int normalize, float* fv_out, fgmm_stream_t stream) {
  if (!fv_out) return FGMM_ERR_INVALID_ARG;
  if (h && h->c.K > (int)(kChunk / 32)) return FGMM_ERR_UNSUPPORTED;
  int rc = run_partial(h, X, x_dtype, N, ldx, weights, means, vars, h ? h->c.ws.canon : nullptr,
                       nullptr, stream);
  if (rc) return rc;
  return map_cuda(launch_fisher(h->c, weights, vars, (double)N, h->c.ws.canon, normalize,
                                fv_out, (cudaStream_t)stream));
}

int fgmm_kmeans_step(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     float* centroids, int32_t* assign_out, int64_t* counts_out,
                     double* inertia_out, fgmm_stream_t stream) {
  int rc = check_x(h, X, x_dtype, N, ldx);
  if (rc) return rc;
  if (!centroids) return FGMM_ERR_INVALID_ARG;
  if ((rc = set_device(h->c))) return rc;
  return map_cuda(launch_kmeans_step(h->c, X, x_dtype, N, ldx, centroids, assign_out,
                                     counts_out, inertia_out, (cudaStream_t)stream));
}

int fgmm_kmeans_seed(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     int64_t first, const double* u, float* centroids, int64_t* idx_out,
                     void* scratch, fgmm_stream_t stream) {
  int rc = check_x(h, X, x_dtype, N, ldx);
  if (rc) return rc;
  if (!centroids || !idx_out || !scratch || first < 0 || first >= N ||
      (h->c.K > 1 && !u))
    return FGMM_ERR_INVALID_ARG;
  if ((rc = set_device(h->c))) return rc;
  return map_cuda(launch_kmeans_seed(h->c, X, x_dtype, N, ldx, first, u, centroids, idx_out,
                                     scratch, (cudaStream_t)stream));
}

size_t fgmm_kmeans_seed_scratch_bytes(int64_t N) {
  return N > 0 ? kmeans_seed_scratch_bytes(N) : 0;
}

size_t fgmm_ivf_build_scratch_bytes(int64_t N, int K) {
  return (N > 0 && K > 0) ? ivf_build_scratch_bytes(N, K) : 0;
}

int fgmm_ivf_build(int K, const int32_t* ids, int64_t N, int top_m, int64_t* offsets,
                   int64_t* entries, int64_t* n_entries, void* scratch, fgmm_stream_t stream) {
  if (K < 1 || N < 1 || top_m < 1 || !ids || !offsets || !entries || !scratch)
    return FGMM_ERR_INVALID_ARG;
  if ((size_t)K * sizeof(int) > 227 * 1024) return FGMM_ERR_UNSUPPORTED;
  return map_cuda(launch_ivf_build(K, ids, N, top_m, offsets, entries, n_entries, scratch,
                                   (cudaStream_t)stream));
}

int fgmm_ivf_search(int K, int D, const float* centroids, const int64_t* offsets,
                    const int64_t* entries, const float* X, int64_t ldx, const float* Q,
                    int64_t nq, int64_t ldq, int nprobe, int topk, int64_t* out_ids,
                    float* out_dist, int64_t* dco_out, fgmm_stream_t stream) {
  if (K < 1 || D < 1 || nq < 0 || ldx < D || ldq < D || nprobe < 1 || nprobe > K ||
      topk < 1 || topk > FGMM_IVF_MAX_TOPK || !centroids || !offsets || !entries || !X || !Q ||
      !out_ids || !out_dist)
    return FGMM_ERR_INVALID_ARG;
  if (ivf_search_smem(K, D, nprobe, topk) > 227 * 1024) return FGMM_ERR_UNSUPPORTED;
  if (nq == 0) return FGMM_OK;
  return map_cuda(launch_ivf_search(K, D, centroids, offsets, entries, X, ldx, Q, nq, ldq, nprobe,
                                    topk, out_ids, out_dist, dco_out, (cudaStream_t)stream));
}

const char* fgmm_profile_kernel_name(int index) {
  return (index >= 0 && index < FGMM_PROF_KERNELS) ? kKernelNames[index] : nullptr;
}

int fgmm_selftest_bounded_wait(int limit_ms) {
  if (limit_ms < 1 || limit_ms > 10000) return FGMM_ERR_INVALID_ARG;
  int st = FGMM_OK;
  cudaError_t e = run_bounded_wait_probe((int64_t)limit_ms * 1000000, &st);
  if (e != cudaSuccess) return map_cuda(e);
  return st;
}

const char* fgmm_status_string(int status) {
  switch (status) {
    case FGMM_OK: return "ok";
    case FGMM_ERR_INVALID_ARG: return "invalid argument";
    case FGMM_ERR_UNSUPPORTED: return "unsupported";
    case FGMM_ERR_CUDA: return "CUDA runtime error";
    case FGMM_ERR_OOM: return "out of device memory";
    case FGMM_ERR_NUMERIC: return "non-finite log-likelihood or every component empty";
    case FGMM_ERR_TIMEOUT: return "bounded device wait expired";
    case FGMM_ERR_IO: return "reading X failed";
    default: return "unknown status";
  }
}

}  // extern "C"
