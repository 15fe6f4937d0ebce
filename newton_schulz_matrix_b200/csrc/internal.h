// Internal launchers shared between the translation units of libmuon.
// Nothing here is part of the C ABI (see include/muon.h).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

namespace muon {

// ---------------------------------------------------------------- elementwise
// One "segment" = `count` matrices of one storage shape rows x cols that land
// in consecutive slots [slot0, slot0 + count) of an oriented n x m workspace
// batch (n = min, m = max; a tall matrix is transposed on the way in and out).
struct SegmentPtrs {
  static constexpr int kMax = 256;  // matrices per launch (kernel-parameter space)
  const void* src[kMax];  // G (momentum mode) or X (copy mode)
  float* mom[kMax];       // M (momentum mode only)
  void* dst[kMax];        // W (update mode) or X (copy mode)
};

struct PackArgs {
  int rows, cols, count;
  int src_dtype;        // G or X storage dtype
  int x_dtype;          // workspace dtype (bf16/fp16 tensor path, fp32 SIMT path)
  int momentum_mode;    // 1: M <- mu M + (1-mu) G, U = nesterov ? lerp : M;  0: U = src
  float mu;
  int nesterov;
  void* x;              // workspace X batch, slot0 already applied
  int ld_x;             // leading dimension of X (>= m)
  long long x_batch_stride;
  float* partials;      // [count][tiles] sums of squares, slot0 applied
  int partial_stride;   // partial entries per matrix
  // pass 0: store M and raw U, write partials (one pass; the chain applies the norm)
  // pass 1: write partials only (no stores): the first half of a normalised pack
  // pass 2: store M and U * scale[b] (scale = 1/(||U||+eps) from pass 1), no partials
  int pass;
  const float* scale;   // pass 2: per-matrix factor, slot0 applied
};
int pack_tiles(int rows, int cols);
void launch_pack(const PackArgs& a, const SegmentPtrs& p, cudaStream_t s);

// inv[b] = 1 / (sqrt(sum partials[b][:]) + eps), deterministic order.
void launch_norm(const float* partials, int partial_stride, int n_partials, int count,
                 float eps, float* inv, cudaStream_t s);

struct UnpackArgs {
  int rows, cols, count;
  int dst_dtype;        // W or X storage dtype
  int x_dtype;
  int update_mode;      // 1: W <- decay W - step O;  0: X <- O
  float decay, step;    // decay = 1 - lr wd, step = lr * scale_coef * sqrt(max(r,c))
  const void* x;        // oriented result batch, slot0 applied
  int ld_x;
  long long x_batch_stride;
  int* status;          // per-matrix status words for these matrices (may be null)
  const int* chunk_err; // device word with errors raised by the chunk's GEMMs (may be null)
};
void launch_unpack(const UnpackArgs& a, const SegmentPtrs& p, cudaStream_t s);

void launch_convert(const void* src, int src_dtype, void* dst, int dst_dtype, long long n,
                    cudaStream_t s);

// status[i] |= *chunk_err for i < count (the chunk's device-side error bits,
// e.g. a wait timeout, reported to every matrix of the chunk).
void launch_status_or(int* status, int count, const int* chunk_err, cudaStream_t s);

// ---------------------------------------------------------------- products
// The last product of a Muon step's chain can write the update itself: its
// epilogue rounds O to the chain's type (as the stored X would be) and writes
// W <- decay W - step O for every matrix of the launch, in W's storage
// orientation, instead of storing O (the paired-CTA kernel; see run_batches).
struct UpdateSlots {
  static constexpr int kMax = 512;  // matrices per launch (kernel-parameter space)
  float decay, step;                // decay = 1 - lr wd, step = lr scale_coef sqrt(max(r, c))
  int* status;                      // per-matrix status words (may be null)
  void* w[kMax];                    // W of batch index b
  int status_idx[kMax];             // its index into status
  unsigned char kind[kMax];         // bit 0: stored transposed (m x n); bits 1-2: W dtype
};

// D[b] = epilogue(A[b] * op(B[b])) for b < batch, all row-major.
//   A is M x K (K contiguous).  op(B) is K x N given either as rows of
//   length K (b_kmajor = 1: B stored N x K, i.e. D = A B^T) or as rows of
//   length N (b_kmajor = 0: B stored K x N, D = A B).
//   epilogue: out = f*(c_acc*acc + c_in*Cin) + (row == col ? c_eye : 0),
//   f = scale[b]^scale_pow.  symmetric = 1 asks for the upper-triangle tiles
//   only (M == N, result known symmetric), mirrored on store.
struct GemmDesc {
  int M, N, K, batch;
  const void* A; int lda; long long a_bs;
  const void* B; int ldb; long long b_bs; int b_kmajor;
  int in_dtype;           // operand dtype (A and B share it)
  void* D; int ldd; long long d_bs; int d_dtype;
  const void* C; int ldc; long long c_bs; int c_dtype;  // optional Cin
  float c_acc, c_in, c_eye;
  const float* scale; int scale_pow;
  int symmetric;
  int* err;               // device word: timeout bits land here (may be null)
  int* tile_counter;      // device word, 0 before the launch: the paired-CTA kernel's tile scheduler
  const UpdateSlots* update;  // host struct: write the Muon update instead of D (non-symmetric, M >= 256)
};
// Tensor-core (tcgen05) path: bf16/fp16 operands.  Returns 0 or a CUDA error.
int gemm_tc(const GemmDesc& g, cudaStream_t s);
// Whether gemm_tc runs an M-row product on the paired-CTA kernel (the one
// that can write the fused update).
bool gemm_tc_paired(int M);
// A chain of n <= 24 products (16-bit, M >= 256, one batch size, one operand
// type) as one persistent launch; product i waits, per matrix, for product
// i - 1 (see gemm_chain.cu).  tile_counter: one zeroed word; done: n * batch
// zeroed words.  Only the last product may carry `update`.
int gemm_chain(const GemmDesc* prods, int n, int* tile_counter, int* done, int* err, cudaStream_t s);
constexpr int kChainMaxProducts = 24;
// FLOPs the tensor cores execute for one gemm_tc / gemm_tf32x3 launch of `g`:
// every MMA over whole tiles (zero padding of ragged tiles and k-blocks
// included), only the tiles a symmetric product computes, and for 3xTF32 the
// three MMAs per product term.  The algorithmic count is 2 M N K per matrix.
double gemm_tc_exec_flops(const GemmDesc& g);
double gemm_tf32x3_exec_flops(const GemmDesc& g);
// Tensor-core path for fp32 operands (3xTF32, paired CTAs): fp32 C and D; A
// and B are read as their TF32 splits, hi = x rounded to TF32 and lo = x - hi,
// stored as fp32 planes with the operand's own strides (split_tf32 writes
// them).  g.A / g.B are not read.
struct Tf32Planes {
  const float* a_hi; const float* a_lo;
  const float* b_hi; const float* b_lo;
};
int gemm_tf32x3(const GemmDesc& g, const Tf32Planes& planes, cudaStream_t s);
// hi / lo planes of `elems` fp32 values (a multiple of 4, 16-byte aligned).
int split_tf32(const float* src, float* hi, float* lo, long long elems, cudaStream_t s);
// SIMT path (any dtype, fp32 math): fp32 products with fewer than 256 rows.
int gemm_simt(const GemmDesc& g, cudaStream_t s);

// Whole fp32 Newton-Schulz chain of small matrices, one CTA per matrix, in
// shared memory (single launch).  x: workspace batch (count x n x ld_x fp32),
// overwritten with the result; raw: scale by inv[b] on load.
struct FusedSmallArgs {
  static constexpr int kMaxIters = 64;
  int n, m, count;
  float* x; int ld_x; long long x_bs;
  const float* inv; int raw;
  int mode;            // 0 standard, 1 Gram (restart_after 0 = naive)
  int restart_after;
  int restart_every;   // 0: restart once; e > 0: also every e iterations after it
  int iters;
  float coeffs[3 * kMaxIters];
};
constexpr size_t kFusedSmallMaxSmem = 200 * 1024;
size_t fused_small_smem(int n, int m, int mode);
int launch_fused_small(const FusedSmallArgs& a, cudaStream_t s);

// Per-device caches cover device ordinals below kMaxDevices.
constexpr int kMaxDevices = 64;
int current_device();   // -1 on error or an ordinal beyond kMaxDevices
int num_sms();          // of the current device (cached per device)
long long wait_timeout_ns();

}  // namespace muon
