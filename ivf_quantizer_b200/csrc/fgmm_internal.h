// Internal declarations shared by the host library and the kernels.
// Not part of the public ABI (include/fgmm.h is).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

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

static inline int round_up(int a, int b) { return (a + b - 1) / b * b; }
static inline int64_t ceil_div64(int64_t a, int64_t b) { return (a + b - 1) / b; }

// Device-side status word values are the public fgmm_status codes.
// The first error wins (atomicCAS from FGMM_OK).

struct Workspace {
  // padded sizes
  int Kp = 0;   // K rounded up to kKB
  int Dp = 0;   // D rounded up to kDC
  // prepared parameters (CUDA-core path)
  float* mu = nullptr;     // [Kp, Dp] means, zero padded
  float* prec = nullptr;   // [Kp, Dp] -1/(2 sigma^2), zero padded
  float* cconst = nullptr; // [Kp] log pi_k - 1/2 sum_d log(2 pi sigma_kd^2); -inf if absent
  // per chunk
  float* logz = nullptr;   // [kChunk] log Z_i of the chunk being processed
  double* ll_tiles = nullptr;  // [kChunk / kTP] per-tile partial log-likelihood
  double* ll_total = nullptr;  // [1]
  // statistics partials, one slot per slice: [kSlices][Kp][1 + 2 Dp]
  double* stats = nullptr;
  double* nk = nullptr;    // [Kp] reduced N_k of the last step
  int* status = nullptr;   // [1]
  size_t bytes = 0;
};

// Kernel kinds for the optional event timing (fgmm_profile_*).
enum KernelKind { KK_SWEEP1 = 0, KK_SWEEP2 = 1, KK_OTHER = 2 };

struct Profiler;  // defined in fgmm_host.cu

struct Ctx {
  int K = 0, D = 0, cov = FGMM_COV_DIAG, prec = FGMM_PREC_FP32;
  double reg = 1e-6;
  int device = 0, num_sms = 0;
  Workspace ws;
  Profiler* prof = nullptr;
};

// Brackets one kernel launch with profiling events when profiling is enabled.
void prof_begin(const Ctx& c, KernelKind k, cudaStream_t s);
void prof_end(const Ctx& c, KernelKind k, cudaStream_t s);

// ---------------------------------------------------------------- launchers (CUDA-core path)
cudaError_t launch_prep_simt(const Ctx& c, const float* weights, const float* means,
                             const float* vars, cudaStream_t s);
cudaError_t launch_lse_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                            float* logz_out, cudaStream_t s);
cudaError_t launch_ll_accumulate(const Ctx& c, int64_t n, cudaStream_t s);
cudaError_t launch_stats_simt(const Ctx& c, const void* X, int x_dtype, int64_t n, int64_t ldx,
                              cudaStream_t s);
cudaError_t launch_mstep(const Ctx& c, float* weights, float* means, float* vars,
                         double* loglik_out, cudaStream_t s);
cudaError_t launch_soft_assign_simt(const Ctx& c, const void* X, int x_dtype, int64_t n,
                                    int64_t ldx, int top_m, float r_threshold, int32_t* ids,
                                    float* resp, cudaStream_t s);

}  // namespace fgmm
