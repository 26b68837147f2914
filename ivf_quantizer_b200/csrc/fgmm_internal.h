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
constexpr int64_t kChunk = 1 << 20;  // points per chunk: bounds every N-sized buffer
constexpr int kSideMaxStiff = 256;   // AUTO side path: most stiff components per step
constexpr int kSideParts = 64;       // AUTO side path: point ranges per chunk

static inline int round_up(int a, int b) { return (a + b - 1) / b * b; }
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
  __half* xop = nullptr;    // [2][kChunk][K1] phi(x) hi / lo of the current chunk
  int* mode = nullptr;      // [1] path of the current step: 0 tensor cores, 1 CUDA cores
  int* mode2 = nullptr;     // [1] AUTO: tensor when the hybrid redo pass must run
  int* stiff = nullptr;     // [Kt] AUTO: 1 = component handled by the CUDA-core side path
  int* stiff_list = nullptr;  // [Kt] stiff components in index order
  int* n_stiff = nullptr;   // [1]
  double* side_part = nullptr;  // [kSideParts][kSideMaxStiff][1 + 2 Dp] side-path partial rows
  // prepared parameters (CUDA-core path)
  float* mu = nullptr;     // [Kp, Dp] means, zero padded
  float* prec = nullptr;   // [Kp, Dp] -1/(2 sigma^2), zero padded
  float* cconst = nullptr; // [Kp] log pi_k - 1/2 sum_d log(2 pi sigma_kd^2); -inf if absent
  // per chunk
  float* logz = nullptr;   // [kChunk] log Z_i of the chunk being processed
  double* ll_tiles = nullptr;  // [kChunk / 32] partial log-likelihoods of the chunk
  double* ll_total = nullptr;  // [1]
  // statistics partials, one slot per point slice: [slots][KpS][1 + 2 Dp]
  double* stats = nullptr;
  double* nk = nullptr;    // [Kp] reduced N_k of the last step
  int* status = nullptr;   // [1]
  size_t bytes = 0;
};

// Kernel kinds for the optional event timing (fgmm_profile_*).
enum KernelKind { KK_SWEEP1 = 0, KK_SWEEP2 = 1, KK_OTHER = 2 };

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
};

// Path codes stored in Workspace::mode.
constexpr int kModeTensor = 0;
constexpr int kModeSimt = 1;

// Brackets one kernel launch with profiling events when profiling is enabled.
void prof_begin(const Ctx& c, KernelKind k, cudaStream_t s);
void prof_end(const Ctx& c, KernelKind k, cudaStream_t s);

// ---------------------------------------------------------------- launchers
// `mode` arguments: nullptr runs the kernel unconditionally; otherwise the kernel
// returns at once unless *mode selects its path (AUTO decides on the device).
cudaError_t launch_prep_simt(const Ctx& c, const float* weights, const float* means,
                             const float* vars, cudaStream_t s);
cudaError_t launch_lse_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, const int* mode, cudaStream_t s);
cudaError_t launch_ll_accumulate(const Ctx& c, int64_t n, const int* mode, int fixed_mode,
                                 int required, cudaStream_t s);
// AUTO only: variance-cancellation check after a tensor-core pass.  Stage 0: failing
// components become stiff and a hybrid redo pass is enabled (mode2 word); stage 1: a
// failure after the redo sends the step to the CUDA-core path.  Each stage clears the
// partial results it invalidates.
cudaError_t launch_auto_check(const Ctx& c, int stage, cudaStream_t s);
cudaError_t launch_stats_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s);
cudaError_t launch_mstep(const Ctx& c, float* weights, float* means, float* vars,
                         double* loglik_out, const int* mode, int fixed_mode, cudaStream_t s);
// tensor-core path (fgmm_tc.cu)
bool tc_supported(const Ctx& c);
cudaError_t tc_init(Ctx& c);
int tc_slices(const Ctx& c);
cudaError_t launch_tc_prep(const Ctx& c, const float* weights, const float* means,
                           const float* vars, bool auto_mode, cudaStream_t s);
// AUTO side path for stiff components (fgmm_side.cu)
cudaError_t launch_stiff_compact(const Ctx& c, int* gate, int* mode, cudaStream_t s);
cudaError_t launch_side_lse(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, const int* mode, cudaStream_t s);
cudaError_t launch_side_stats(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s);
cudaError_t launch_tc_convert(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              const int* mode, cudaStream_t s);
cudaError_t launch_tc_lse(const Ctx& c, int64_t n, float* logz_out, const int* mode,
                          cudaStream_t s);
cudaError_t launch_tc_stats(const Ctx& c, int64_t n, const int* mode, cudaStream_t s);
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
