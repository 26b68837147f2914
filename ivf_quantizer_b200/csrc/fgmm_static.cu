// fgmm_soft_assign_static: the soft assignment for callers that cannot allocate device
// memory (see include/fgmm.h).  Its scratch is one fixed-size array in this library's
// device memory instead of a handle's workspace.
#include <mutex>

#include "fgmm_internal.h"

namespace fgmm {
namespace {

// Layout of the scratch: padded means | padded precisions | constants | status word.
constexpr size_t kOffMu = 0;
constexpr size_t kOffPrec = kOffMu + (size_t)FGMM_STATIC_MAX_KD * sizeof(float);
constexpr size_t kOffConst = kOffPrec + (size_t)FGMM_STATIC_MAX_KD * sizeof(float);
constexpr size_t kOffStatus = kOffConst + (size_t)FGMM_STATIC_MAX_K * sizeof(float);
constexpr size_t kScratchBytes = kOffStatus + 256;

// Device-side scratch.  In host code this name is only a stand-in for the symbol: a
// kernel must be given the address cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_static_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
unsigned char* g_base[kMaxDevices] = {};
std::mutex g_lock;

// Device address of the scratch on `dev` (the current device), looked up once per device.
int scratch_address(int dev, unsigned char** out) {
  if (dev < 0 || dev >= kMaxDevices) return FGMM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> guard(g_lock);
  if (!g_base[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e != cudaSuccess || !p) {
      cudaGetLastError();
      return FGMM_ERR_CUDA;
    }
    g_base[dev] = static_cast<unsigned char*>(p);
  }
  *out = g_base[dev];
  return FGMM_OK;
}

}  // namespace
}  // namespace fgmm

using namespace fgmm;

extern "C" int fgmm_soft_assign_static(int K, int D, int cov_type, const void* X, int x_dtype,
                                       int64_t N, int64_t ldx, const float* weights,
                                       const float* means, const float* vars, int top_m,
                                       float r_threshold, int32_t* ids, float* resp,
                                       fgmm_stream_t stream) {
  if (K < 1 || D < 1 || (cov_type != FGMM_COV_DIAG && cov_type != FGMM_COV_SPHERICAL))
    return FGMM_ERR_INVALID_ARG;
  if (!X || !weights || !means || !vars || !ids) return FGMM_ERR_INVALID_ARG;
  if (x_dtype != FGMM_F32 && x_dtype != FGMM_BF16) return FGMM_ERR_INVALID_ARG;
  if (N < 1 || ldx < D) return FGMM_ERR_INVALID_ARG;
  if (top_m < 1 || top_m > FGMM_MAX_TOP_M || top_m > K) return FGMM_ERR_INVALID_ARG;
  if (!(r_threshold >= 0.f) || !(r_threshold < 1.f)) return FGMM_ERR_INVALID_ARG;
  if (K > FGMM_STATIC_MAX_K || D > FGMM_STATIC_MAX_KD) return FGMM_ERR_UNSUPPORTED;
  const int Kp = round_up(K, kKB), Dp = round_up(D, kDC);
  if ((int64_t)Kp * Dp > FGMM_STATIC_MAX_KD || Kp > FGMM_STATIC_MAX_K) return FGMM_ERR_UNSUPPORTED;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return FGMM_ERR_CUDA;
  unsigned char* base = nullptr;
  int rc = scratch_address(dev, &base);
  if (rc) return rc;
  float* mu = reinterpret_cast<float*>(base + kOffMu);
  float* prec = reinterpret_cast<float*>(base + kOffPrec);
  float* cconst = reinterpret_cast<float*>(base + kOffConst);
  int* status = reinterpret_cast<int*>(base + kOffStatus);

  cudaStream_t s = (cudaStream_t)stream;
  // the status word still holds the previous call's value; the other regions are
  // fully rewritten by the preparation kernel
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(int), s);
  if (e == cudaSuccess)
    e = launch_prep_simt_raw(K, D, Kp, Dp, cov_type, weights, means, vars, mu, prec, cconst,
                             status, s);
  const size_t eb = x_dtype == FGMM_BF16 ? 2 : 4;
  for (int64_t c0 = 0; e == cudaSuccess && c0 < N; c0 += kChunk) {
    const int64_t nc = (N - c0 < kChunk) ? N - c0 : kChunk;
    e = launch_soft_assign_simt_raw((const char*)X + (size_t)c0 * ldx * eb, x_dtype, nc, ldx, K,
                                    D, Kp, Dp, mu, prec, cconst, top_m, r_threshold,
                                    ids + c0 * top_m, resp ? resp + c0 * top_m : nullptr, s);
  }
  int st = FGMM_OK;
  if (e == cudaSuccess) e = cudaMemcpyAsync(&st, status, sizeof(int), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) {
    cudaGetLastError();
    return FGMM_ERR_CUDA;
  }
  return st;
}
