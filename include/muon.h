/* muon.h -- C ABI of libmuon: the Muon optimizer step with Newton-Schulz
 * orthogonalisation (standard, Gram and stabilised Gram forms) on NVIDIA B200.
 *
 * Sources of the operations (web pages, cited by title and section):
 *   [Moonlight] "Moonlight 16B Guide: Scalable MoE & Muon Optimizer":
 *       box "Scalable Muon Optimizer Step" (steps 1-4); section "The
 *       Newton-Schulz Iteration for Matrix Orthogonalization"; "Innovation 1:
 *       Decoupled Weight Decay in Muon"; "Innovation 2: Per-Parameter Update
 *       Scale Alignment"; listing "End-to-End PyTorch Implementation".
 *   [GramNS] "Gram Newton-Schulz" news write-up (Machine Heart, m.web578.cn):
 *       standard iteration and its three products; Gram rewrite; stabilised
 *       variant (float16 Gram iteration, restart after step 2).
 *
 * Conventions shared by every entry point
 *   - Every matrix is dense row-major in device memory (leading dimension =
 *     cols) and 16-byte aligned.  The caller owns all memory, including the
 *     workspace; the library allocates nothing and carries no data from one
 *     call to the next (it only caches per-device launch settings on first
 *     use: the SM count, shared-memory opt-ins, how many CTA pairs fit).
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = legacy
 *     default stream).  They take no lock on the launch path; the opt-in
 *     profiler and the allocation-free entry point's scratch lookup
 *     take a mutex.  The return value reports argument
 *     and launch errors only (MUON_OK, MUON_ERR_*).  Conditions found on the
 *     device are OR-ed into the optional per-matrix status words (device int
 *     array, one per matrix, zeroed by the call): MUON_STATUS_NONFINITE when
 *     an orthogonalised matrix holds Inf/NaN, MUON_STATUS_TIMEOUT when a
 *     device-side wait gave up (the kernel then returned without finishing).
 *   - A matrix of storage shape rows x cols is orthogonalised in its
 *     short-side-first orientation n x m (n = min, m = max): tall matrices
 *     are transposed on the way in and back on the way out [Moonlight
 *     listing, "ensure m <= n"; GramNS, X in R^{n x m}].
 *   - Calls that overlap on the GPU must not share a workspace.
 */
#ifndef MUON_H_
#define MUON_H_

#include <stddef.h>

#if defined(__GNUC__)
#define MUON_API __attribute__((visibility("default")))
#else
#define MUON_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum { MUON_BF16 = 0, MUON_FP16 = 1, MUON_FP32 = 2 } muon_dtype;

/* Which form of the Newton-Schulz iteration runs [GramNS]:
 *   STANDARD         X <- a X + (b A + c A^2) X, A = X X^T, per iteration
 *   GRAM             naive Gram form: R = X0 X0^T; Q_k = a I + b R + c R^2;
 *                    Q_acc <- Q_k Q_acc; R <- Q_k R Q_k; X = Q_acc X0
 *   GRAM_STABILIZED  Gram form restarted after iteration restart_after (and,
 *                    if restart_every > 0, every restart_every iterations
 *                    after it): X0 <- Q_acc X0, R <- X0 X0^T, Q_acc <- I */
typedef enum { MUON_NS_STANDARD = 0, MUON_NS_GRAM = 1, MUON_NS_GRAM_STABILIZED = 2 } muon_ns_mode;

enum {
  MUON_OK = 0,
  MUON_ERR_INVALID = -1,     /* null pointer, bad size/shape/count, misaligned pointer, bad enum */
  MUON_ERR_UNSUPPORTED = -2, /* dtype combination the kernels do not implement */
  MUON_ERR_WORKSPACE = -3,   /* ws_bytes below muon_*_workspace_size's minimum for one matrix */
  MUON_ERR_CUDA = -4         /* a CUDA launch or tensor-map encode failed */
};
#define MUON_STATUS_NONFINITE 1
#define MUON_STATUS_TIMEOUT 2

/* Newton-Schulz parameters.
 *   iters          K >= 1 iterations
 *   coeffs         host array of 3*iters floats, (a_k, b_k, c_k) per iteration;
 *                  the quintic (3.4445, -4.7750, 2.0315) or the cubic
 *                  (1.5, -0.5, 0) of [Moonlight, NS section]
 *   mode           muon_ns_mode
 *   restart_after  GRAM_STABILIZED only: iteration after which the Gram
 *                  matrix is rebuilt (1 <= restart_after < iters; 2 in [GramNS])
 *   restart_every  GRAM_STABILIZED only: 0 = rebuild once; e > 0 = also after
 *                  iterations restart_after + e, + 2e, ... before the last
 *                  (the periodic reading of [GramNS]'s "re-initialise")
 *   eps            X0 = U / (||U||_F + eps)  [Moonlight, NS section; listing eps]
 *   compute_dtype  MUON_BF16 or MUON_FP16: tcgen05 tensor cores, fp32
 *                  accumulate, 16-bit storage of X, A, B between the products
 *                  of the standard form; MUON_FP32: fp32 storage throughout
 *                  (any mode), products as 3xTF32 on the tensor cores (operands
 *                  split into TF32 hi + lo, fp32 sums per 32-deep k-block) when
 *                  min(rows, cols) >= 256, else fp32 FFMA (a matrix whose whole
 *                  chain fits in one block's shared memory runs it in one launch)
 *   gram_dtype     Gram modes on tensor cores: the 16-bit type of every matrix
 *                  the Gram chain stores (R, Q, Q_acc, X0 and the restart X),
 *                  MUON_FP16 (the stabilised variant's float16) or MUON_BF16 */
typedef struct {
  int iters;
  const float* coeffs;
  int mode;
  int restart_after;
  float eps;
  int compute_dtype;
  int gram_dtype;
  int restart_every;
} muon_ns_params;

/* One group of `count` parameters that share storage shape rows x cols.
 *   W  host array of `count` device pointers, rows x cols of w_dtype; updated
 *   G  host array of device pointers, rows x cols of g_dtype; read only
 *   M  host array of device pointers, rows x cols fp32 momentum; updated */
typedef struct {
  int rows, cols, count;
  int w_dtype, g_dtype;
  void* const* W;
  const void* const* G;
  float* const* M;
} muon_group;

/* Optimizer hyper-parameters of one step.
 *   lr, weight_decay  W <- (1 - lr wd) W - lr s(W) O   [Moonlight, Innovation 1, box step 4]
 *   momentum, nesterov  M <- mu M + (1 - mu) G [Moonlight, box step 1];
 *                     U = nesterov ? (1 - mu) G + mu M : M
 *   scale_coef        s(W) = scale_coef sqrt(max(rows, cols)) [Moonlight, Innovation 2]
 *   ns                the orthogonalisation */
typedef struct {
  float lr, momentum, weight_decay, scale_coef;
  int nesterov;
  muon_ns_params ns;
} muon_hparams;

/* Workspace bytes that let muon_step process every group in a single chunk
 * (the fastest setting).  A smaller workspace is accepted down to
 * muon_workspace_min; groups are then processed in chunks.  Returns 0 on
 * invalid arguments. */
MUON_API size_t muon_workspace_size(const muon_group* groups, int n_groups, const muon_hparams* hp);
MUON_API size_t muon_workspace_min(const muon_group* groups, int n_groups, const muon_hparams* hp);

/* One Muon step over n_groups groups  [Moonlight, box steps 1-4]:
 *   M <- mu M + (1 - mu) G;  U = nesterov ? (1 - mu) G + mu M : M
 *   O = NS(U / (||U||_F + eps))   (oriented n x m, see muon_ns_params)
 *   W <- (1 - lr wd) W - lr scale_coef sqrt(max(rows, cols)) O
 * Groups whose matrices orient to the same n x m (e.g. 2048 x 1408 and
 * 1408 x 2048) are orthogonalised together.
 *   ws, ws_bytes       device workspace (256-byte aligned)
 *   status_per_matrix  optional device int array, one word per matrix in
 *                      group order; zeroed, then OR-ed with MUON_STATUS_* */
MUON_API int muon_step(const muon_group* groups, int n_groups, const muon_hparams* hp, void* ws, size_t ws_bytes,
              int* status_per_matrix, void* stream);

/* In-place orthogonalisation of `count` matrices of storage shape rows x cols
 * and dtype `dtype` (X[i] is a device pointer; O replaces X in the same
 * orientation).  This is the listing's newton_schulz_orthogonalize without
 * the optimizer around it. */
MUON_API size_t muon_ns_workspace_size(int count, int rows, int cols, const muon_ns_params* ns);
MUON_API int muon_ns_batched(void* const* X, int count, int rows, int cols, int dtype, const muon_ns_params* ns, void* ws,
                    size_t ws_bytes, int* status_per_matrix, void* stream);

/* muon_ns_batched without a caller workspace, for callers that cannot
 * allocate device memory when they orthogonalise: a host whose caching
 * allocator already owns the GPU's memory (a raw cudaMalloc would fail or
 * fragment its pool), a loop that forbids allocation after start-up, or a
 * plugin that receives only input/output pointers.  The pages have no
 * counterpart of this entry point; it is a library convenience.
 *
 * The workspace is a fixed array of MUON_NOALLOC_SCRATCH_BYTES inside the
 * library, present on every GPU that loads the library until the process
 * exits.  The call allocates and frees nothing.  A shape whose one-matrix
 * workspace (muon_ns_workspace_size(1, rows, cols, ns)) exceeds the array is
 * rejected with MUON_ERR_WORKSPACE; larger counts of fitting matrices are
 * processed in chunks.  Results equal muon_ns_batched's.
 *
 * A call outside a stream capture looks up the array's device address on
 * the current device (cudaGetSymbolAddress) and remembers it; a call on a
 * capturing stream uses the address remembered by the last uncaptured call on
 * that device (none: MUON_ERR_CUDA), so make one uncaptured call before
 * capturing, and again after a cudaDeviceReset.  Every call uses the same
 * array, which keeps the previous call's contents (the call resets what must
 * start at zero): calls that can overlap on the GPU (other streams, other
 * host threads) race on it and must be serialised by the caller, e.g. on one
 * stream. */
#define MUON_NOALLOC_SCRATCH_BYTES (64u << 20)
MUON_API int muon_ns_batched_noalloc(void* const* X, int count, int rows, int cols, int dtype,
                                     const muon_ns_params* ns, int* status_per_matrix, void* stream);

/* Algorithmic FLOPs of one orthogonalisation of a rows x cols matrix, every
 * product counted as 2 * rows * cols * inner [GramNS cost list]. */
MUON_API double muon_ns_flops(int rows, int cols, const muon_ns_params* ns);

/* Opt-in launch profiler (tracing aid).  Between muon_profile_begin() and
 * muon_profile_end(), every kernel the library launches is bracketed by a pair
 * of CUDA events recorded on the launch stream; this is the only state the
 * library keeps between calls, and only while profiling is on.
 * muon_profile_end synchronises on those events and fills up to max_entries
 * rows, one per kernel kind that ran: its name, launch count, summed device
 * time, and for those launches
 *   flops       algorithmic FLOPs: every product 2 * M * N * K, the full
 *               product even where only a triangle is computed [GramNS cost list]
 *   exec_flops  FLOPs the kernels execute: tensor-core MMAs over whole tiles
 *               (zero padding included), only the tiles of a symmetric
 *               product's upper triangle, three TF32 MMAs per 3xTF32 product;
 *               equal to flops for the other kernels
 *   bytes       algorithmic bytes (each operand read once, result written once)
 * Returns the number of rows written, or a MUON_ERR_* code. */
typedef struct {
  const char* kernel;
  int launches;
  double ms;
  double flops;
  double exec_flops;
  double bytes;
} muon_profile_entry;
MUON_API int muon_profile_begin(void);
MUON_API int muon_profile_end(muon_profile_entry* out, int max_entries);

/* Static text for a MUON_* return code or status bit set. */
MUON_API const char* muon_status_string(int code);

#ifdef __cplusplus
}
#endif
#endif /* MUON_H_ */
