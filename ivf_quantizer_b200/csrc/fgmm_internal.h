// Internal declarations shared by the host library and the kernels.
// Not part of the public ABI (include/fgmm.h is).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cuda_fp16.h>

#include "../../include/fgmm.h"

namespace fgmm {

// ---------------------------------------------------------------- tiling constants
constexpr int kSimtThreads = 256;
constexpr int kTP = 64;        // points per tile (CUDA-core kernels)
constexpr int kKB = 64;        // components per block in the log-sum-exp sweep
constexpr int kKBs = 32;       // components per CTA in the statistics sweep
constexpr int kDC = 32;        // feature chunk staged in shared memory
constexpr int kFC = 128;       // features per CTA in the statistics sweep
constexpr int kSlices = 16;    // point slices of a chunk in the statistics sweep
constexpr int kFlushTiles = 64;  // fp32 run length (tiles) before an fp64 flush
constexpr int kLbufMaxKp = 1024; // largest Kp whose chunk of log-densities is kept (4 GB)
constexpr int64_t kChunk = FGMM_CHUNK_POINTS;  // points per chunk: bounds every N-sized buffer
constexpr int kSideMaxStiff = 256;   // AUTO side path: most stiff components per step
constexpr int kSideParts = 64;       // AUTO side path: point ranges per chunk
constexpr int kSidePairs = 4;        // AUTO side path: (component, log z) pairs kept per point
// AUTO side path: a stiff or grey component whose log-density is more than this many
// nats below a point's log Z is skipped there: its responsibility is below
// exp(-40) = 4e-18, far under fp32 resolution of log Z and under what the tensor-core
// statistics keep (they store r as fp16(r 2^15), which drops r below ~1e-12)
constexpr float kSideCut = 40.f;
// AUTO: a component with fewer effective points than this in the previous step is grey
constexpr double kGreyNk = 8.0;
// Block skipping in the tensor-core statistics sweep.  That sweep stores r as
// fp16(r 2^15), which is exactly 0 for r <= 2^-40, i.e. for a log-density 27.7 nats or
// more below log Z.  A (point tile, 128-component block) pair in which every point has
// every log-density of the block more than kSkipCut nats below its log Z therefore adds
// exactly nothing to N_k, S1, S2, and is left out.  The 2.3-nat margin covers the two
// sweeps' rounding differences (about 1e-4 nats) many times over.
constexpr float kSkipCut = 30.f;
constexpr int kSkipMaxBlocks = 32;   // block masks are 32-bit words: K <= 4096
// The same on the CUDA-core path, whose fp32 statistics keep every responsibility down to
// the underflow of expf (about e^-104): there a pair is left out when every log-density
// is more than kSimtSkipCut nats below log Z, i.e. each dropped r is below e^-50 = 2e-22,
// and all that a component can lose over 10^9 points is below 2e-13 effective points.
constexpr float kSimtSkipCut = 50.f;
// Tensor-core statistics: the products accumulate in fp32 in TMEM for a run of tiles
// before each fp64 flush, and each MMA step loses up to about half an fp32 unit of the
// running sum (measured on B200: the error of the raw moments grows linearly with the
// run length, i.e. it is biased, not a random walk).  The variance update
// S2/N_k - (S1/N_k)^2 multiplies that relative error by A = (S2/N_k) / variance =
// 1 + (mu - c)^2 / sigma^2.  Measured at K = 1024, D = 128 in the steady state with
// block skipping (whose sorted tiles put a component's points into fewer, denser runs):
// largest relative variance error over 1.3e5 (component, dimension) pairs = 2.3e-3 with
// 8-tile runs, 6.9e-4 with 2-tile runs, 3.1e-4 with 1-tile runs, at A up to ~510; the
// dense sweep's runs hold few non-zero responsibilities per component and stay below
// 2e-4 with 8-tile runs.  Hence 2-tile runs with block skipping, 8 without, and
// components whose A exceeds kMaxAmplification go to the direct-form CUDA-core side path:
// with 2-tile runs the error is ~1.35e-6 A, at most 6e-4 below the bound.
constexpr int kFlushTilesDense = 8;
constexpr int kFlushTilesSkip = 2;
constexpr float kMaxAmplification = 450.f;
// Tensor-core filtered assignment: a component whose expanded-form logit-error bound
// exceeds this many nats (a collapsed or very tight component far from the centre)
// leaves the filter and is evaluated exactly for every point instead, so that one such
// component cannot widen the block-mask cut for all the others.
constexpr float kAssignMaxE = 0.5f;
constexpr int kOrdPts = 4096;        // points per CTA of the radix sort
constexpr int kOrdBuckets = 256;     // values of one 8-bit radix digit

static inline int round_up(int a, int b) { return (a + b - 1) / b * b; }

// Index of statistic c (0: N_k, 1 + d: first moment, 1 + Dp + d: second moment) of
// component k in slot s.  The CUDA-core kernels use [slot][component][row] (a component's
// row contiguous); the tensor-core kernels use [slot][row][component] (consecutive
// components contiguous, so that the 32 lanes of a flushing warp, 32 components, reduce
// into 32 consecutive doubles).  kstride = components per slot, row = 1 + 2 Dp.
__host__ __device__ __forceinline__ size_t stat_idx(bool tc_layout, int s, int k, int c,
                                                    int kstride, size_t row) {
  return tc_layout ? ((size_t)s * row + (size_t)c) * (size_t)kstride + (size_t)k
                   : ((size_t)s * (size_t)kstride + (size_t)k) * row + (size_t)c;
}
static inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Device-side status word values are the public fgmm_status codes.
// The first error wins (atomicCAS from FGMM_OK).

struct Workspace {
  // padded sizes
  int Kp = 0;   // K rounded up to kKB (CUDA-core path)
  int Dp = 0;   // D rounded up to kDC
  int KpS = 0;  // component stride of the statistics slots: K rounded up to 128
  int slots = 0;  // statistics slots (point slices) allocated
  // tensor-core path
  int Kt = 0;   // K rounded up to 128
  int Dq = 0;   // D rounded up to 32 (= Dp)
  int K1 = 0;   // 2 * Dq: length of phi(x) = [x^, x^2]
  float* center = nullptr;  // [Dq] per-dimension centre c_d
  float* dscale = nullptr;  // [Dq] per-dimension power-of-two scale s_d
  __half* wop = nullptr;    // [2][Kt][K1] W' hi / lo
  float* tck = nullptr;     // [Kt] c_k
  float* tks = nullptr;     // [Kt] 2^t_k
  // AUTO side-path filter: a stiff component's tensor-core logit is only an estimate, but
  // with a per-component error bound E_k it tells which points can need the side path
  float* tcraw = nullptr;   // [Kt] c_k before masking
  float* tcm = nullptr;     // [Kt] M_k = sum_d (mu_kd - c_d)^2 / sigma_kd^2
  float* tcpk = nullptr;    // [Kt] P_k = log pi_k + log N(mu_k | mu_k, Sigma_k), the peak
  float* tckf = nullptr;    // [Kt] c_k + E_k for stiff components, -inf otherwise
  float* lzlow = nullptr;   // [1] log Z below which a point is always flagged
  // sweep 1: per (component block, point) the block's (max, sum of 2^(l - max)) of the
  // log2-scaled log-densities and the stiff filter's maximum, merged into log Z after it
  float2* lpart = nullptr;  // [Kt / 128][kChunk]
  float* lpartf = nullptr;  // [Kt / 128][kChunk]
  // tensor-core assignment: per-component bound on the expanded-form logit error, and the
  // block-mask cut it widens (log2 units)
  float* tce = nullptr;     // [Kt] E_k
  float* acut = nullptr;    // [1]
  // components whose bound exceeds kAssignMaxE: left out of the tensor-core filter and
  // evaluated exactly for every point (ordered, padded to a multiple of 64 with 0)
  int* alist = nullptr;     // [Kt]
  int* nalist = nullptr;    // [1]
  uint8_t* side_flag = nullptr;  // [kChunk] 1: the point may have a stiff component within kCut
  // side-path components within kCut of a flagged point, found while merging log Z and
  // reused by the statistics (a count above kSidePairs: the statistics re-evaluate)
  uint8_t* pair_cnt = nullptr;   // [kChunk] number of such components
  uint8_t* pair_j = nullptr;     // [kChunk][kSidePairs] their index in the side-path list
  float* pair_l = nullptr;       // [kChunk][kSidePairs] their log z
  int* flagged = nullptr;        // [kChunk] the flagged points of the chunk, as a list
  int* n_flagged = nullptr;      // [1] their number
  int* flag_cnt = nullptr;       // [kChunk / 4096] flagged points per 4096-point block
  __half* xop = nullptr;    // [2][kChunk][K1] phi(x) hi / lo of the current chunk
  // block skipping (sweep 2 visits only the (tile, block) pairs that can contribute)
  uint32_t* bmask = nullptr;  // [kChunk] per point: blocks within kSkipCut of log Z
  int* perm = nullptr;        // [kChunk] sweep-2 order: row j of phi is point perm[j]
  int* perm2 = nullptr;       // [kChunk] the other buffer of the radix passes
  float* lzp = nullptr;       // [kChunk] log Z in sweep-2 order
  int* ord_hist = nullptr;    // [kOrdBuckets][kChunk / kOrdPts] counts, then offsets
  int* ord_tot = nullptr;     // [kOrdBuckets] points per digit value
  uint32_t* tmask = nullptr;  // [kChunk / kTP] per sweep-2 tile: OR of its points' masks
  int* tlist = nullptr;       // [kSkipMaxBlocks][kChunk / tile rows] active tiles of each block
  float* bmx = nullptr;       // CUDA-core path: [kChunk][Kp / kKB] largest log z per 64 components
  int* tcnt = nullptr;        // [kSkipMaxBlocks] their number
  int* mode = nullptr;      // [1] path of the current step: 0 tensor cores, 1 CUDA cores
  int* mode2 = nullptr;     // [1] AUTO: tensor when the hybrid redo pass must run
  int* stiff = nullptr;     // [Kt] AUTO: 1 = component handled by the CUDA-core side path
  int* stiff_list = nullptr;  // [Kt] stiff components in index order
  int* n_stiff = nullptr;   // [2] stiff count, grey count (the grey follow the stiff in the list)
  // AUTO grey components: kept on the tensor cores, but their statistics are also taken
  // on the side path, to be swapped in should the variance check fail
  int* grey = nullptr;      // [Kt] 1: grey
  int* grey_pos = nullptr;  // [Kt] index among the grey of this pass, -1 if none
  double* grey_stats = nullptr;  // [kSideMaxStiff][1 + 2 Dp] side-path statistics of the grey
  double* side_part = nullptr;  // [kSideParts][kSideMaxStiff][1 + 2 Dp] side-path partial rows
  // prepared parameters (CUDA-core path)
  float* mu = nullptr;     // [Kp, Dp] means, zero padded
  float* prec = nullptr;   // [Kp, Dp] -1/(2 sigma^2), zero padded
  float* cconst = nullptr; // [Kp] log pi_k - 1/2 sum_d log(2 pi sigma_kd^2); -inf if absent
  // D > kFC: the statistics sweep covers the features in several CTAs per component
  // block, each of which would recompute the log-densities; the log-sum-exp sweep keeps
  // them here instead (allocated for Kp <= kLbufMaxKp only)
  float* lbuf = nullptr;   // [kChunk][Kp] log z_ik of the chunk
  // per chunk
  float* logz = nullptr;   // [kChunk] log Z_i of the chunk being processed
  double* ll_tiles = nullptr;  // [kChunk / 32] partial log-likelihoods of the chunk
  double* ll_total = nullptr;  // [1]
  double* canon = nullptr;  // [K (1 + 2D) + 1] exchange-form statistics of the step
  // statistics partials, one slot per point slice: [slots][KpS][1 + 2 Dp]
  double* stats = nullptr;
  double* nk = nullptr;    // [Kp] reduced N_k of the last step
  int* status = nullptr;   // [1]
  unsigned int* km_word = nullptr;  // [2] k-means: largest |x| (float bits), fixed-point exponent
  size_t bytes = 0;
};

// Kernels, for the optional event timing (fgmm_profile_*); the order is the index into
// fgmm_profile's per-kernel arrays and must match the names in fgmm_host.cu.
enum KernelId {
  KI_TC_CENTER = 0, KI_TC_PREP, KI_TC_CONVERT, KI_TC_LSE, KI_TC_STATS,
  KI_PREP_SIMT, KI_LSE_SIMT, KI_LL_ACCUMULATE, KI_STATS_SIMT, KI_REDUCE_STATS, KI_MSTEP,
  KI_FINALIZE,
  KI_SOFT_ASSIGN, KI_AUTO_CHECK, KI_REDO_RESET, KI_REMASK,
  KI_STIFF_COMPACT, KI_SIDE_LSE, KI_LL_PARTIALS, KI_SIDE_STATS, KI_SIDE_REDUCE,
  KI_KM_ASSIGN, KI_KM_SEED, KI_TC_ORDER, KI_TC_GATHER,
  KI_COUNT
};

struct Profiler;  // defined in fgmm_host.cu

struct TcState {
  alignas(64) CUtensorMap tmap_x;  // phi(x) hi/lo of the chunk, [2 kChunk][K1] fp16
  alignas(64) CUtensorMap tmap_w;  // W' hi/lo, [2 Kt][K1] fp16
  bool ready = false;
};

struct Ctx {
  int K = 0, D = 0, cov = FGMM_COV_DIAG, prec = FGMM_PREC_AUTO;
  double reg = 1e-6;
  int device = 0, num_sms = 0;
  Workspace ws;
  TcState tc;
  Profiler* prof = nullptr;
  int last_path = -1;      // FGMM_PREC_FP32 / FGMM_PREC_FP16X3, or -1
  bool last_auto = false;  // last step decided its path on the device
  bool skip = true;        // block skipping in the tensor-core statistics sweep
  int64_t last_nc = 0;     // points of the last chunk of the last step (fgmm_last_step_info)
  bool last_stats = false; // the last step ran a statistics sweep
};

// Path codes stored in Workspace::mode.
constexpr int kModeTensor = 0;
constexpr int kModeSimt = 1;

// Brackets one launch with events when profiling is enabled.  A launch whose kernel
// returns at once unless *gate == required passes gate (else nullptr): the profiler then
// snapshots the word in stream order, so that it can tell launches that did work from
// launches that returned at their gate.
void prof_begin(const Ctx& c, KernelId k, cudaStream_t s, const int* gate = nullptr,
                int required = 0);
void prof_end(const Ctx& c, KernelId k, cudaStream_t s);
// A further kernel launched inside the current profiled region (counted, timed with it).
void prof_extra_launch(const Ctx& c);
// A kernel that may write a gate word has been enqueued: launches after it take new
// snapshots of their gate (until then, launches behind one gate share a snapshot).
void prof_gates_changed(const Ctx& c);

// ---------------------------------------------------------------- launchers
// `mode` arguments: nullptr runs the kernel unconditionally; otherwise the kernel
// returns at once unless *mode selects its path (AUTO decides on the device).
cudaError_t launch_prep_simt(const Ctx& c, const float* weights, const float* means,
                             const float* vars, cudaStream_t s);
// keep_logits: also write every log z_ik of the chunk to ws.lbuf (when it exists), for the
// statistics sweep to read instead of recomputing them once per feature block
cudaError_t launch_lse_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, bool keep_logits, const int* mode, cudaStream_t s);
cudaError_t launch_ll_accumulate(const Ctx& c, int64_t n, const int* mode, int fixed_mode,
                                 int required, cudaStream_t s);
// AUTO only: variance-cancellation check after a tensor-core pass.  Stage 0: failing
// components become stiff and a hybrid redo pass is enabled (mode2 word); stage 1: a
// failure after the redo sends the step to the CUDA-core path.  Each stage clears the
// partial results it invalidates.
cudaError_t launch_auto_check(const Ctx& c, int stage, cudaStream_t s);
cudaError_t launch_stats_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s);
// Slot sums -> exchange-form statistics (out: [K (1 + 2D) + 1], about `means`).
cudaError_t launch_reduce_stats(const Ctx& c, const float* means, double* out, const int* mode,
                                int fixed_mode, cudaStream_t s);
// M-step and weights from exchange-form statistics; parameters updated in place.
cudaError_t launch_finish(const Ctx& c, const double* st, float* weights, float* means,
                          float* vars, double* loglik_out, cudaStream_t s);
// Fisher vector from exchange-form statistics (fv: [2 K D]); uses ll_tiles (K <= kChunk/32).
cudaError_t launch_fisher(const Ctx& c, const float* weights, const float* vars, double n_points,
                          const double* st, int normalize, float* fv, cudaStream_t s);
cudaError_t launch_stats_sum(const double* parts, int n_parts, int64_t len, double* out,
                             cudaStream_t s);
// IVF application (fgmm_ivf.cu)
size_t ivf_build_scratch_bytes(int64_t n, int K);
cudaError_t launch_ivf_build(int K, const int32_t* ids, int64_t n, int m, int64_t* offsets,
                             int64_t* entries, int64_t* n_entries, void* scratch, cudaStream_t s);
size_t ivf_search_smem(int K, int D, int nprobe, int topk);
cudaError_t launch_ivf_search(int K, int D, const float* C, const int64_t* offsets,
                              const int64_t* entries, const float* X, int64_t ldx, const float* Q,
                              int64_t nq, int64_t ldq, int nprobe, int topk, int64_t* out_i,
                              float* out_d, int64_t* dco, cudaStream_t s);
// k-means warm start (fgmm_kmeans.cu)
size_t kmeans_seed_scratch_bytes(int64_t n);
cudaError_t launch_kmeans_step(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                               float* centroids, int32_t* assign_out, int64_t* counts_out,
                               double* inertia_out, cudaStream_t s);
cudaError_t launch_kmeans_seed(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                               int64_t first, const double* u, float* centroids,
                               int64_t* idx_out, void* scratch, cudaStream_t s);
// tensor-core path (fgmm_tc.cu)
bool tc_supported(const Ctx& c);
cudaError_t tc_init(Ctx& c);
int tc_slices(const Ctx& c);
// statistics slots the tensor-core statistics sweep may write (block skipping can give a
// busy block more CTAs than tc_slices); the reduction sums this many
int tc_stat_slots(const Ctx& c);
// assign: the assignment's preparation (components whose logit-error bound exceeds
// kAssignMaxE are marked and listed in ws.alist instead of AUTO's stiffness rules)
cudaError_t launch_tc_prep(const Ctx& c, const float* weights, const float* means,
                           const float* vars, bool auto_mode, cudaStream_t s,
                           bool assign = false);
// AUTO side path for stiff components (fgmm_side.cu)
cudaError_t launch_stiff_compact(const Ctx& c, int* gate, int* mode, cudaStream_t s);
cudaError_t launch_side_lse(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, const int* mode, cudaStream_t s);
cudaError_t launch_side_stats(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s);
// perm: nullptr for the natural order, else row j of phi is point perm[j] of the chunk
cudaError_t launch_tc_convert(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* perm, const int* mode, cudaStream_t s);
// block skipping applies to this handle's tensor-core sweeps
bool tc_skip(const Ctx& c);
// assign: block masks for the assignment (always kept, with the cut in ws.acut)
cudaError_t launch_tc_lse(const Ctx& c, int64_t n, float* logz_out, const int* mode,
                          cudaStream_t s, bool assign = false);
// the assignment's block-mask cut from the components' logit-error bounds: base_nats
// (what the exact evaluation needs within the cut) + 8 max_k E_k + 0.5 nats
cudaError_t launch_assign_cut(const Ctx& c, float base_nats, cudaStream_t s);
// block order and 64-row tile masks from ws.bmask (assignment)
cudaError_t launch_assign_order(const Ctx& c, int64_t n, cudaStream_t s);
// CUDA-core assignment over the sorted 64-point tiles, visiting only the 128-component
// blocks of each tile's mask; results written for the original point indices
cudaError_t launch_soft_assign_skip(const Ctx& c, const void* X, int x_dtype, int64_t n,
                                    int64_t ldx, int top_m, float r_threshold, int32_t* ids,
                                    float* resp, cudaStream_t s);
// block skipping (fgmm_order.cu): sweep-2 order from sweep 1's block masks, phi and
// log Z rewritten in that order, and the active tiles of every component block
cudaError_t launch_tc_order(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            const int* mode, cudaStream_t s);
cudaError_t launch_tc_stats(const Ctx& c, int64_t n, const int* mode, cudaStream_t s);
// block skipping on the CUDA-core path: masks from sweep 1's block maxima (ws.bmx), the
// sweep-2 order (ws.perm, ws.lzp) and the active 64-point tiles of each 128-component block
bool simt_skip(const Ctx& c);
cudaError_t launch_simt_order(const Ctx& c, int64_t n, const int* mode, cudaStream_t s);
cudaError_t run_bounded_wait_probe(int64_t limit_ns, int* status_host);
// soft assignment on caller-provided scratch (allocation-free entry point)
cudaError_t launch_prep_simt_raw(int K, int D, int Kp, int Dp, int cov, const float* weights,
                                 const float* means, const float* vars, float* mu, float* prec,
                                 float* cconst, int* status, cudaStream_t s);
cudaError_t launch_soft_assign_simt_raw(const void* X, int x_dtype, int64_t n, int64_t ldx, int K,
                                        int D, int Kp, int Dp, const float* mu, const float* prec,
                                        const float* cconst, int top_m, float r_threshold,
                                        int32_t* ids, float* resp, cudaStream_t s);
cudaError_t launch_soft_assign_simt(const Ctx& c, const void* X, int x_dtype, int64_t n,
                                    int64_t ldx, int top_m, float r_threshold, int32_t* ids,
                                    float* resp, cudaStream_t s);

}  // namespace fgmm
