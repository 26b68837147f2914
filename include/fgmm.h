/*
 * fgmm.h — C-ABI of the fused Gaussian-mixture EM library for NVIDIA B200 (sm_100a).
 *
 * The operations are those of "Flash-GMM: A Memory-Efficient Kernel for
 * Scalable Soft Clustering" (Bloch et al., arXiv 2606.10896):
 *   - §2: mixture density, log-likelihood, E-step responsibilities computed in
 *     log space, M-step Eqs. (1)-(3), stopping rule;
 *   - §3.1, Algorithm 1: one EM iteration as a fused two-sweep pass over point
 *     tiles that never stores the N x K responsibility matrix;
 *   - §4.2-4.3: argmax and top-2 thresholded multi-assignment for IVF lists.
 *
 * Conventions for every call:
 *   - Device pointers unless a name ends in _host.  All device work is
 *     enqueued on the caller's stream and is asynchronous, unless a call says
 *     it synchronises.
 *   - X is row-major [N, D] with row stride ldx elements (ldx >= D).  x_dtype is
 *     FGMM_F32 or FGMM_BF16.  The tensor-core precision modes require
 *     ldx * sizeof(element) to be a multiple of 16 bytes and X 16-byte aligned.
 *   - Parameters: weights float[K]; means float[K*D] row-major; vars float[K*D]
 *     (diagonal model) or float[K] (isotropic model).  They are read at the
 *     start of a step and overwritten in place with the M-step result.
 *   - The caller owns X, the parameters and every output buffer.  The handle
 *     owns only its workspace (allocated by fgmm_create, O(K*D), independent of
 *     N) and its device status word.
 *   - Errors are returned as fgmm_status codes; nothing throws across the ABI.
 *     Errors found on the device (non-finite log-likelihood, invalid
 *     parameters, every component empty) are latched in the handle's status
 *     word and read with fgmm_get_status.
 *   - A handle must not be used from two streams concurrently.
 */
#ifndef FGMM_H
#define FGMM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct fgmm_ctx* fgmm_handle;
/* Same object as cudaStream_t / CUstream; 0 is the legacy default stream. */
typedef struct CUstream_st* fgmm_stream_t;

/* Covariance model.  SPHERICAL is the paper's isotropic sigma_k^2 I (§2,
 * footnote 1; Appendix A); DIAG has one variance per component and dimension. */
enum fgmm_cov { FGMM_COV_DIAG = 0, FGMM_COV_SPHERICAL = 1 };

/* Arithmetic of the log-density evaluation and of the sufficient statistics.
 *   FP32   : CUDA cores, fp32, log-densities in the direct (x - mu)^2 form and
 *            statistics centred on each component's current mean.
 *   FP16X3 : tensor cores (tcgen05), expanded form [x, x^2] . W with every
 *            operand split into two fp16 halves and three products, fp32
 *            accumulation (about 22 significant bits per product).
 *   FP16   : tensor cores, one fp16 product per term in both sweeps (about 11
 *            significant bits per term; no W' lo or phi lo operands).  A speed mode for
 *            callers that can accept its error: it does not hold the 1e-4 per-point
 *            log-likelihood accuracy of the other modes where the expanded-form terms
 *            are large next to the log-density (high D, tight components far from
 *            the data's centre); AUTO never selects it.
 *   AUTO   : the default; FP16X3 for the components that are well conditioned for
 *            the expanded form, the others ("stiff") on a CUDA-core side path in the
 *            direct form, decided per component and per step on the device; the whole
 *            step goes to FP32 when more than 256 components are stiff or a variance
 *            check still fails after one redo pass. */
enum fgmm_prec { FGMM_PREC_FP32 = 0, FGMM_PREC_FP16X3 = 1, FGMM_PREC_FP16 = 2, FGMM_PREC_AUTO = 3 };

/* Element type of X. */
enum fgmm_dtype { FGMM_F32 = 0, FGMM_BF16 = 1 };

enum fgmm_status {
  FGMM_OK = 0,
  FGMM_ERR_INVALID_ARG = 1, /* bad size, null pointer, bad enum, or invalid parameters */
  FGMM_ERR_UNSUPPORTED = 2, /* valid request this build or device cannot run */
  FGMM_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  FGMM_ERR_OOM = 4,         /* workspace allocation failed */
  FGMM_ERR_NUMERIC = 5,     /* non-finite log-likelihood, or every component empty */
  FGMM_ERR_TIMEOUT = 6,     /* a bounded device-side wait expired */
  FGMM_ERR_IO = 7           /* a reader of X (file or callback) failed */
};

/* Largest top_m accepted by fgmm_soft_assign. */
#define FGMM_MAX_TOP_M 16
/* A component with responsibility mass N_k below this is treated as empty:
 * its mean and variance are kept and its weight becomes 0. */
#define FGMM_EMPTY_NK 1e-6
/* A step walks X in chunks of this many points (the last one ragged); each sweep
 * kernel is launched once per chunk, and every buffer the handle holds that grows
 * with the point count is sized for one chunk. */
#define FGMM_CHUNK_POINTS (1 << 20)

/* Create a handle for K components in D dimensions.
 * reg_covar >= 0 is added to every variance after each M-step (variance floor).
 * Allocates the workspace on the current CUDA device; the handle is bound to
 * that device.  Returns FGMM_ERR_INVALID_ARG for K < 1, D < 1, a bad cov_type or
 * a negative / non-finite reg_covar, FGMM_ERR_OOM if allocation fails. */
int fgmm_create(int K, int D, int cov_type, double reg_covar, fgmm_handle* out);

/* Free the workspace (synchronises the device first).  NULL is accepted. */
int fgmm_destroy(fgmm_handle h);

/* Select the precision mode (enum fgmm_prec).  FGMM_ERR_INVALID_ARG for an
 * unknown value; FGMM_ERR_UNSUPPORTED for a tensor-core mode (FP16X3, FP16) when the
 * handle's D has no tensor-core path (D > 128). */
int fgmm_set_precision(fgmm_handle h, int prec);
int fgmm_get_precision(fgmm_handle h, int* prec_out);

/* Block skipping in the tensor-core statistics sweep (on by default).
 * Paper: "Flash-GMM", §3.1 and Algorithm 1.  Sweep 2 forms r_ik = exp(log z_ik - log Z_i)
 * for all i, k and adds them into the statistics.  The tensor-core path keeps r as
 * fp16(r 2^15), which is exactly 0 once log z_ik < log Z_i - 27.7.  With skipping on,
 * sweep 1 marks for each point the 128-component blocks that come within 30 nats of
 * log Z_i.  Sweep 2 then visits the points grouped by those marks, and only the
 * (128-point tile, block) pairs that hold a mark; every pair it leaves out adds
 * exactly 0.  Results match the dense sweep up to the order of fp32 additions and stay
 * bitwise reproducible from run to run.  Tensor-core path: K of 129 ... 4096 (2 to 32
 * blocks).  The CUDA-core path (FGMM_PREC_FP32, or an AUTO step sent there) skips the
 * same way for K of 385 ... 4096 (4 to 32 blocks, counted as K rounded up to 64, then
 * to 128).  Its fp32 statistics keep responsibilities down to about e^-104, so there a
 * pair is left out only when every log-density is 50 nats or more below log Z_i: each
 * dropped r is below 2e-22.
 * enable: 0 off, nonzero on.  FGMM_ERR_INVALID_ARG for a NULL handle. */
int fgmm_set_block_skip(fgmm_handle h, int enable);
int fgmm_get_block_skip(fgmm_handle h, int* enable_out);

/* Path the last fgmm_em_step of this handle ran: FGMM_PREC_FP32 (CUDA cores),
 * FGMM_PREC_FP16X3 (tensor cores, split products) or FGMM_PREC_FP16 (tensor cores, one
 * product, when selected explicitly).  Under FGMM_PREC_AUTO the choice is made on the
 * device per step, so this call synchronises the device.  -1 before any step. */
int fgmm_last_step_path(fgmm_handle h, int* path_out);

/* What the last fgmm_em_step / fgmm_em_partial of this handle did, for tests and
 * benchmarks that must show which regime they covered.  Synchronises the device.
 *   path           : as fgmm_last_step_path (-1 before any step)
 *   n_stiff        : FGMM_PREC_AUTO: components the last pass evaluated on the CUDA-core
 *                    side path (ill-conditioned for the expanded form); 0 otherwise
 *   n_grey         : FGMM_PREC_AUTO: components kept on the tensor cores whose statistics
 *                    the side path also took (fewer than 8 effective points before)
 *   skip_pairs     : block skipping, last chunk of the last tensor-core pass: the
 *                    (point tile, component block) pairs the statistics sweep visited;
 *                    -1 when that sweep ran dense or did not run
 *   skip_pairs_all : the pairs a dense sweep of that chunk visits (tiles x blocks)
 * FGMM_ERR_INVALID_ARG for a NULL handle or output. */
typedef struct fgmm_step_info {
  int path;
  int n_stiff;
  int n_grey;
  int64_t skip_pairs;
  int64_t skip_pairs_all;
} fgmm_step_info;
int fgmm_last_step_info(fgmm_handle h, fgmm_step_info* out);

/* Bytes of device memory the handle holds (independent of N). */
int fgmm_workspace_bytes(fgmm_handle h, size_t* bytes_out);

/* One EM iteration (§2; §3.1 Algorithm 1) on device data.
 *   E-step with a log-sum-exp over the K components, responsibilities folded
 *   straight into the sufficient statistics N_k, sum r (x - c), sum r (x - c)^2
 *   (never stored as an N x K matrix), then the M-step Eqs. (1)-(3) with the
 *   updated mean in the variance, pi_k = N_k / sum_k' N_k', the variance floor,
 *   and the empty-component rule (FGMM_EMPTY_NK).
 *   weights, means, vars : in/out, the parameters Theta_in are replaced by Theta_out.
 *   loglik_out           : device double, receives log p(X | Theta_in) (may be NULL).
 *   logz_out             : optional device float[N], per-point log p(x_i | Theta_in)
 *                          (NULL to skip; the library itself never stores it).
 * N must be >= 1.  Asynchronous; device-side errors go to the status word. */
int fgmm_em_step(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                 float* weights, float* means, float* vars,
                 double* loglik_out, float* logz_out, fgmm_stream_t stream);

/* fgmm_em_step with X in host memory: rows are copied to the device one chunk
 * (FGMM_CHUNK_POINTS points) at a time into two device staging buffers, the copy of
 * the next chunk overlapping the sweeps of the current one on an internal copy stream,
 * so N is not limited by device memory (the paper's path to N beyond HBM, §6).  X_host
 * should be pinned (page-locked) for the copies to overlap; pageable memory works but
 * serialises them.  The staging buffers (2 x FGMM_CHUNK_POINTS x D x 4 bytes) are
 * allocated by the first call and kept by the handle.  Under FGMM_PREC_AUTO the
 * device's path decision is read back (one synchronisation per decision) so that only
 * the passes that run copy X.  Other arguments as fgmm_em_step (weights, means, vars,
 * loglik_out and logz_out are device memory).  The call returns when the last copy has
 * been enqueued; X_host must stay valid until the stream reaches the step's end. */
int fgmm_em_step_host(fgmm_handle h, const void* X_host, int x_dtype, int64_t N, int64_t ldx,
                      float* weights, float* means, float* vars, double* loglik_out,
                      float* logz_out, fgmm_stream_t stream);

/* Reader of X for the streamed steps below: fill dst (pinned host memory owned by the
 * handle) with rows row0 .. row0 + nrows - 1 of X, row-major and contiguous (D
 * elements of the step's x_dtype per row; nrows <= FGMM_CHUNK_POINTS).  Return 0 on
 * success, anything else on failure.  Called on the calling thread, one chunk at a
 * time, in increasing row order within each pass over X (a step makes one pass per
 * sweep pair that runs: two or three under FGMM_PREC_AUTO when its device-side
 * decision asks for the redo or the CUDA-core pass). */
typedef int (*fgmm_read_fn)(void* ctx, int64_t row0, int64_t nrows, void* dst);

/* fgmm_em_step with X produced chunk by chunk by a reader: for X on storage, the
 * paper's path for N beyond host memory (§6, streaming from SSD into the same
 * O(K D) buffers).  Each chunk is read into one of two pinned host buffers
 * (2 x FGMM_CHUNK_POINTS x D x 4 bytes, allocated by the first call and kept by the
 * handle; a buffer is refilled only after its previous copy to the device completed),
 * copied to a device staging buffer on the copy stream of fgmm_em_step_host, and
 * processed there, so that reading chunk i + 1 overlaps the sweeps of chunk i.
 * Results are bit-identical to fgmm_em_step on the same rows.  Returns FGMM_ERR_IO
 * (with the step's outputs undefined and the parameters unchanged) when the reader
 * fails; other arguments and errors as fgmm_em_step_host.  The call returns when the
 * last chunk has been read and its copy enqueued. */
int fgmm_em_step_reader(fgmm_handle h, fgmm_read_fn read, void* ctx, int x_dtype, int64_t N,
                        float* weights, float* means, float* vars, double* loglik_out,
                        float* logz_out, fgmm_stream_t stream);

/* fgmm_em_step_reader for X stored in a file: N rows of D elements of x_dtype,
 * row-major and contiguous, starting at byte `offset` of the file at `path` (read with
 * pread; a short read or an unopenable file gives FGMM_ERR_IO). */
int fgmm_em_step_file(fgmm_handle h, const char* path, int64_t offset, int x_dtype, int64_t N,
                      float* weights, float* means, float* vars, double* loglik_out,
                      float* logz_out, fgmm_stream_t stream);

/* Data-parallel EM over row shards of X (one exchange per iteration).  Each entry
 * of the M-step's input is a sum over rows (§2, Eqs. (1)-(3)), so an iteration over
 * shards held by several handles, devices or processes is: fgmm_em_partial on every
 * shard with the same parameters, an elementwise sum of the statistics vectors (a
 * collective such as an all-reduce, or an all-gather and fgmm_stats_sum), then
 * fgmm_em_finish with the sum on every shard.  fgmm_em_step is exactly
 * fgmm_em_partial followed by fgmm_em_finish on one shard.
 *
 * Statistics vector: device double[FGMM_STATS_LEN(K, D)], for component k at offset
 * k (1 + 2D):  N_k = sum_i r_ik,  then D entries sum_i r_ik (x_id - mu_kd),  then D
 * entries sum_i r_ik (x_id - mu_kd)^2, about the means passed to fgmm_em_partial; last
 * entry sum_i log Z_i (this shard's log-likelihood).  The same layout serves both
 * covariance types. */
#define FGMM_STATS_LEN(K, D) ((int64_t)(K) * (1 + 2 * (int64_t)(D)) + 1)

/* E-step and statistics sweep of one EM iteration on this shard.  weights, means,
 * vars are read, not changed; stats_out receives the statistics vector (device,
 * caller-owned, FGMM_STATS_LEN(K, D) doubles); logz_out as in fgmm_em_step.  Same
 * precision modes, paths and status handling as fgmm_em_step.  Asynchronous. */
int fgmm_em_partial(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                    const float* weights, const float* means, const float* vars,
                    double* stats_out, float* logz_out, fgmm_stream_t stream);

/* fgmm_em_partial with X in host memory, streamed as in fgmm_em_step_host. */
int fgmm_em_partial_host(fgmm_handle h, const void* X_host, int x_dtype, int64_t N,
                         int64_t ldx, const float* weights, const float* means,
                         const float* vars, double* stats_out, float* logz_out,
                         fgmm_stream_t stream);

/* fgmm_em_partial with X produced by a reader, as in fgmm_em_step_reader (a shard on
 * storage: each rank reads its own rows). */
int fgmm_em_partial_reader(fgmm_handle h, fgmm_read_fn read, void* ctx, int x_dtype,
                           int64_t N, const float* weights, const float* means,
                           const float* vars, double* stats_out, float* logz_out,
                           fgmm_stream_t stream);

/* fgmm_em_partial_reader for a shard stored in a file, as in fgmm_em_step_file. */
int fgmm_em_partial_file(fgmm_handle h, const char* path, int64_t offset, int x_dtype,
                         int64_t N, const float* weights, const float* means,
                         const float* vars, double* stats_out, float* logz_out,
                         fgmm_stream_t stream);

/* M-step (Eqs. (1)-(3), the variance floor and the empty-component rule) from a
 * statistics vector summed over every shard.  weights, means, vars: in/out, the
 * parameters the statistics were taken about, replaced by Theta_out.  loglik_out:
 * optional device double, receives the summed log-likelihood.  A non-finite
 * log-likelihood or an all-empty mixture leaves the parameters unchanged and sets
 * FGMM_ERR_NUMERIC in the status word.  Asynchronous. */
int fgmm_em_finish(fgmm_handle h, const double* stats, float* weights, float* means,
                   float* vars, double* loglik_out, fgmm_stream_t stream);

/* out[j] = sum_{p = 0 .. n_parts-1} parts[p * len + j], summed in part order, so the
 * result does not depend on how the parts arrived (device buffers; out may not
 * overlap parts).  For combining gathered statistics vectors bit-reproducibly.
 * FGMM_ERR_INVALID_ARG for NULL pointers, n_parts < 1 or len < 1.  Asynchronous on
 * `stream` of the current device. */
int fgmm_stats_sum(const double* parts, int n_parts, int64_t len, double* out,
                   fgmm_stream_t stream);

/* Repeat fgmm_em_step up to max_iters times (§2, stopping rule).  With tol > 0
 * it stops early once |L_t - L_{t-1}| / N < tol, which needs one 8-byte
 * device-to-host read per iteration; with tol == 0 it only enqueues work.
 * Synchronises the stream before returning.
 *   final_loglik_host : log-likelihood of the last step's input parameters (may be NULL)
 *   iters_done_host   : iterations run (may be NULL)
 * Returns the first error of any step, including the device status word. */
int fgmm_fit(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
             float* weights, float* means, float* vars, int max_iters, double tol,
             double* final_loglik_host, int* iters_done_host, fgmm_stream_t stream);

/* Multi-assignment from responsibilities under the given parameters (§4.2 argmax,
 * §4.3 top-2 with r_ik > tau).  Per point the components are ranked by their
 * log joint (ties to the lower index); rank 1 is always kept; ranks 2..top_m are
 * kept only where r_ik > r_threshold (strict); the rest is padded with id -1 and
 * responsibility 0.
 *   ids  : device int32[N * top_m], row-major
 *   resp : device float[N * top_m], row-major (may be NULL)
 * 1 <= top_m <= min(K, FGMM_MAX_TOP_M), 0 <= r_threshold < 1. */
int fgmm_soft_assign(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     const float* weights, const float* means, const float* vars,
                     int top_m, float r_threshold, int32_t* ids, float* resp,
                     fgmm_stream_t stream);

/* Soft assignment for callers that cannot allocate device memory.
 *
 * The paper has no counterpart to this call; it exists for the host programs that
 * may not call cudaMalloc or cudaFree at all: applications whose device memory is
 * owned by one arena reserved up front (servers, engines, embedded runtimes that
 * account for every byte), and latency-critical loops where the allocator's implicit
 * device synchronisation is not acceptable.  fgmm_create allocates a workspace, so
 * those callers cannot use a handle.
 *
 * Same result as fgmm_soft_assign with the same arguments, but without a handle: K, D
 * and cov_type are passed directly.  Its scratch (padded means,
 * precisions and per-component constants) lives in one fixed array inside the
 * library's own device memory, which every GPU that loads the library holds until
 * the process exits (about 2.1 MB).  Limits: padded K x padded D <= FGMM_STATIC_MAX_KD
 * and padded K <= FGMM_STATIC_MAX_K (K rounded up to 64, D to 32); larger problems
 * return FGMM_ERR_UNSUPPORTED and enqueue nothing.
 *
 * The first call on a device looks up that array's device address (once per device,
 * with that device current), and the CUDA runtime may allocate the array then if it
 * loads modules lazily.  The address
 * is kept for the life of the process: after cudaDeviceReset (or anything else that
 * destroys and re-creates the device's primary context) it is stale, and this call
 * must not be used on that device again.  Every
 * call shares the array and overwrites what the previous call left there; calls that
 * overlap on the GPU (two streams, two host threads) race on it and must be
 * serialised by the caller.  The call synchronises the stream and returns the device
 * status (FGMM_ERR_INVALID_ARG for invalid parameters), or the argument error. */
#define FGMM_STATIC_MAX_KD (1 << 18)
#define FGMM_STATIC_MAX_K (1 << 14)
int fgmm_soft_assign_static(int K, int D, int cov_type, const void* X, int x_dtype, int64_t N,
                            int64_t ldx, const float* weights, const float* means,
                            const float* vars, int top_m, float r_threshold, int32_t* ids,
                            float* resp, fgmm_stream_t stream);

/* Per-point log-density log p(x_i | Theta) = log sum_k pi_k N(x_i | mu_k, Sigma_k) (the
 * first sweep of fgmm_em_step alone: no statistics, parameters unchanged).  With equal
 * weights, the points of a sample as means and a shared isotropic bandwidth this is a
 * Gaussian kernel density estimate (the paper, §6, names KDE as a use of the same
 * kernel).  logz_out: device float[N] (may be NULL if loglik_out is given); loglik_out:
 * optional device double, the sum.  Precision modes as fgmm_em_step.  Asynchronous. */
int fgmm_score_samples(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                       const float* weights, const float* means, const float* vars,
                       float* logz_out, double* loglik_out, fgmm_stream_t stream);

/* Fisher-vector encoding of the point set X (N points) under the mixture: the
 * gradients of the average log-likelihood with respect to the means and the standard
 * deviations, whitened by the diagonal Fisher information (Perronnin & Dance 2007;
 * the paper, §6, names the encoding as a use of the same E-step and weighted
 * statistics):  G_mu_kd = sum_i r_ik (x_id - mu_kd) / sigma_kd / (N sqrt(pi_k)),
 * G_sigma_kd = sum_i r_ik ((x_id - mu_kd)^2 / sigma_kd^2 - 1) / (N sqrt(2 pi_k)).
 * fv_out: device float[2 K D] = [G_mu (K x D, row-major), G_sigma (K x D)]; components
 * with pi_k = 0 give zeros.  normalize != 0: power (sign(z) sqrt|z|) and L2
 * normalisation.  Runs the E-step and statistics sweep of fgmm_em_step (same precision
 * modes); K <= 32768 (FGMM_ERR_UNSUPPORTED otherwise).  Asynchronous. */
int fgmm_fisher_vector(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                       const float* weights, const float* means, const float* vars,
                       int normalize, float* fv_out, fgmm_stream_t stream);

/* k-means warm start ("Flash-GMM", §4.4: k-means, then soft EM from its centroids;
 * the initialisation appendix: k-means++ seeding).  Both use the handle's K and D (and
 * its workspace; they may not run concurrently with another call on the same handle).
 * Decisions that floating point turns into indices are taken in a fixed precision so
 * that they are reproducible: squared distances are fp32, summed over dimensions in
 * increasing order with every subtraction, product and sum rounded separately (no
 * fused multiply-add); ties go to the lower centroid index.  Results are bitwise
 * reproducible run to run.
 *
 * fgmm_kmeans_step: one Lloyd iteration on device X.  centroids: device float [K][D],
 * in/out (an empty cluster keeps its centroid).  assign_out: optional device int32[N],
 * the argmin per point for the INPUT centroids.  counts_out: optional device int64[K].
 * inertia_out: optional device double, sum of the points' squared distances to their
 * assigned input centroid (fp64 sum of the fp32 distances).  Cluster sums are exact
 * 64-bit fixed-point sums (scale from the data's largest |x| and N).  Asynchronous. */
int fgmm_kmeans_step(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     float* centroids, int32_t* assign_out, int64_t* counts_out,
                     double* inertia_out, fgmm_stream_t stream);

/* k-means++ seeding on device X (N >= 1).  first: index of the first centre (0 <= first
 * < N).  u: device double[K-1], the uniforms in [0, 1) of draws 1 .. K-1 (the caller
 * draws them; the method's randomness is an input).  Draw t weighs point i by
 * w_i = floor(D_i * 2^s), D_i its fp32 squared distance to the nearest chosen centre and
 * 2^s the power of two bringing the largest D to [2^29, 2^30), and picks the smallest i
 * whose running sum of w exceeds floor(u_t * sum w) (fp64 product); when every w is 0
 * it repeats the previous centre.  centroids: device float [K][D] out; idx_out: device
 * int64[K] out (required).  scratch: device memory of fgmm_kmeans_seed_scratch_bytes(N)
 * bytes, caller-owned.  K sequential draws, each a pass over X.  Asynchronous. */
int fgmm_kmeans_seed(fgmm_handle h, const void* X, int x_dtype, int64_t N, int64_t ldx,
                     int64_t first, const double* u, float* centroids, int64_t* idx_out,
                     void* scratch, fgmm_stream_t stream);
size_t fgmm_kmeans_seed_scratch_bytes(int64_t N);

/* IVF application (the paper, §4): posting lists from the soft-assignment ids and nprobe
 * search.  Stateless (no handle); device pointers; asynchronous on `stream`.
 *
 * fgmm_ivf_build: ids = device int32 [N][top_m] from fgmm_soft_assign (-1 = none); a
 * vector goes to the list of every cluster it is assigned to (§4.3).  offsets: device
 * int64[K + 1]; entries: device int64 with room for N * top_m (the list of cluster k is
 * entries[offsets[k] .. offsets[k+1]), vector indices in increasing order); n_entries:
 * optional device int64, the total.  scratch: device memory of
 * fgmm_ivf_build_scratch_bytes(N, K) bytes.  Deterministic.  K * 4 bytes must fit in
 * shared memory (FGMM_ERR_UNSUPPORTED otherwise).
 *
 * fgmm_ivf_search: for each of the nq queries (device float [nq][ldq]) the nprobe
 * centroids (device float [K][D]) nearest by squared L2, then exact squared L2 to every
 * entry of their lists (X: device float [N][ldx], the indexed vectors), the topk nearest
 * distinct vectors (ids into out_ids int64 [nq][topk], -1 padded; distances into out_dist
 * float [nq][topk], +inf padded), and the entries scanned per query (distance
 * computations, "DCO") into dco_out (optional int64 [nq]).  Distances are fp32 with
 * dimensions in increasing order, each subtraction, product and sum rounded
 * separately; ties go to the lower index (centroid or vector).  1 <= nprobe <= K,
 * 1 <= topk <= FGMM_IVF_MAX_TOPK. */
#define FGMM_IVF_MAX_TOPK 32
size_t fgmm_ivf_build_scratch_bytes(int64_t N, int K);
int fgmm_ivf_build(int K, const int32_t* ids, int64_t N, int top_m, int64_t* offsets,
                   int64_t* entries, int64_t* n_entries, void* scratch, fgmm_stream_t stream);
int fgmm_ivf_search(int K, int D, const float* centroids, const int64_t* offsets,
                    const int64_t* entries, const float* X, int64_t ldx, const float* Q,
                    int64_t nq, int64_t ldq, int nprobe, int topk, int64_t* out_ids,
                    float* out_dist, int64_t* dco_out, fgmm_stream_t stream);

/* Kernel timing, for benchmarks.  When enabled, the library records a CUDA
 * event pair on the call's stream around every kernel it launches and keeps a
 * launch counter; fgmm_profile_read synchronises the device, sums the elapsed
 * times per kernel and per kernel kind and (if reset != 0) clears the record.
 * Under FGMM_PREC_AUTO a step enqueues the kernels of both paths and those of the
 * path it does not take return at once; for each launch the library also copies
 * the device word that decides this (stream-ordered, 4 bytes into pinned host
 * memory), so that launches which did work are counted apart ("active").
 * Disabled by default; costs two event records per launch, and one 4-byte copy
 * per gated launch, when enabled. */
#define FGMM_PROF_KERNELS 25
typedef struct fgmm_profile {
  int64_t launches;          /* kernels launched while enabled (all kinds) */
  int64_t sweep1_launches;   /* log-sum-exp sweep (first pass over the components) */
  double sweep1_ms;
  int64_t sweep2_launches;   /* statistics sweep (recompute + responsibilities + stats) */
  double sweep2_ms;
  int64_t other_launches;    /* preparation, reductions, M-step, soft assignment */
  double other_ms;
  /* per kernel, indexed as fgmm_profile_kernel_name: every launch, and the launches
   * that passed their path gate and did work */
  int64_t kernel_launches[FGMM_PROF_KERNELS];
  double kernel_ms[FGMM_PROF_KERNELS];
  int64_t kernel_active[FGMM_PROF_KERNELS];
  double kernel_active_ms[FGMM_PROF_KERNELS];
} fgmm_profile;
/* Name of kernel `index` of fgmm_profile's arrays; NULL outside [0, FGMM_PROF_KERNELS). */
const char* fgmm_profile_kernel_name(int index);
int fgmm_profile_enable(fgmm_handle h, int enable);
int fgmm_profile_read(fgmm_handle h, fgmm_profile* out, int reset);

/* Synchronise the stream and return the device status word (first error
 * latched since the last call), then clear it. */
int fgmm_get_status(fgmm_handle h, fgmm_stream_t stream);

/* Self-test of the bounded device-side wait every tensor-core kernel uses: one thread
 * waits on an mbarrier that nothing completes, with a limit of limit_ms (1..10000)
 * milliseconds, and records FGMM_ERR_TIMEOUT when the limit expires.  Synchronises.
 * Returns the recorded status (FGMM_ERR_TIMEOUT when the wait gave up as it must),
 * FGMM_ERR_INVALID_ARG for a limit out of range.  It faults, traps and hangs nothing. */
int fgmm_selftest_bounded_wait(int limit_ms);

/* Static text for a status code. */
const char* fgmm_status_string(int status);

#ifdef __cplusplus
}
#endif

#endif /* FGMM_H */
