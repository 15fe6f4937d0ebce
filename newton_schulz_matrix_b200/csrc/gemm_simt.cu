// CUDA-core (FFMA) batched product with the same epilogue as the tensor-core
// kernel.  It carries the fp32 compute mode: tcgen05 offers only TF32 for
// 32-bit operands, whose 10-bit mantissa cannot hold a 1e-4 relative error
// through five Newton-Schulz iterations.
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace muon {

constexpr int kSB = 64;   // output tile edge
constexpr int kSK = 16;   // k step

template <typename T>
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const GemmDesc g) {
  __shared__ __align__(16) float As[kSK][kSB + 4];
  __shared__ __align__(16) float Bs[kSK][kSB + 4];
  const int b = blockIdx.z;
  const int i0 = blockIdx.y * kSB, j0 = blockIdx.x * kSB;
  // symmetric results: blocks below the diagonal are mirrors of blocks above it
  if (g.symmetric && blockIdx.x < blockIdx.y) return;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const T* A = reinterpret_cast<const T*>(g.A) + (long long)b * g.a_bs;
  const T* B = reinterpret_cast<const T*>(g.B) + (long long)b * g.b_bs;

  float acc[4][4] = {};
  for (int k0 = 0; k0 < g.K; k0 += kSK) {
    // A tile: 64 rows x 16 k -> As[k][row]
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = threadIdx.x + 256 * q;
      const int row = e >> 4, kk = e & 15;
      const int gi = i0 + row, gk = k0 + kk;
      As[kk][row] = (gi < g.M && gk < g.K) ? to_f32(A[(long long)gi * g.lda + gk]) : 0.f;
    }
    // B tile: 16 k x 64 cols -> Bs[k][col]
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = threadIdx.x + 256 * q;
      int kk, col;
      if (g.b_kmajor) { col = e >> 4; kk = e & 15; }
      else { kk = e >> 6; col = e & 63; }
      const int gj = j0 + col, gk = k0 + kk;
      float v = 0.f;
      if (gj < g.N && gk < g.K)
        v = to_f32(g.b_kmajor ? B[(long long)gj * g.ldb + gk] : B[(long long)gk * g.ldb + gj]);
      Bs[kk][col] = v;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < kSK; ++kk) {
      const float4 a4 = *reinterpret_cast<const float4*>(&As[kk][ty * 4]);
      const float4 b4 = *reinterpret_cast<const float4*>(&Bs[kk][tx * 4]);
      const float av[4] = {a4.x, a4.y, a4.z, a4.w};
      const float bv[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
    }
    __syncthreads();
  }

  const float f = matrix_scale(g.scale, g.scale_pow, b);
  char* D = reinterpret_cast<char*>(g.D) + (long long)b * g.d_bs * dtype_size(g.d_dtype);
  const char* C = g.C ? reinterpret_cast<const char*>(g.C) + (long long)b * g.c_bs * dtype_size(g.c_dtype) : nullptr;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int gi = i0 + ty * 4 + i;
    if (gi >= g.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int gj = j0 + tx * 4 + j;
      if (gj >= g.N) continue;
      float v = g.c_acc * acc[i][j];
      if (C) v += g.c_in * load_any(C, (long long)gi * g.ldc + gj, g.c_dtype);
      v *= f;
      if (gi == gj) v += g.c_eye;
      if (g.symmetric) {
        // upper triangle stored twice (direct and mirrored): exactly symmetric
        if (gj < gi) continue;
        store_any(D, (long long)gi * g.ldd + gj, g.d_dtype, v);
        if (gj != gi) store_any(D, (long long)gj * g.ldd + gi, g.d_dtype, v);
        continue;
      }
      store_any(D, (long long)gi * g.ldd + gj, g.d_dtype, v);
    }
  }
}

int gemm_simt(const GemmDesc& g, cudaStream_t s) {
  dim3 grid((g.N + kSB - 1) / kSB, (g.M + kSB - 1) / kSB, g.batch);
  switch (g.in_dtype) {
    case kBF16: gemm_simt_kernel<__nv_bfloat16><<<grid, 256, 0, s>>>(g); break;
    case kFP16: gemm_simt_kernel<__half><<<grid, 256, 0, s>>>(g); break;
    default: gemm_simt_kernel<float><<<grid, 256, 0, s>>>(g); break;
  }
  return (int)cudaGetLastError();
}

// ----------------------------------------------------------------------------
// Fused fp32 chain for small matrices: one CTA per matrix runs every product of
// the iteration in shared memory, so the whole Newton-Schulz chain is a single
// launch.  The products are the same as the chained kernels' (standard form:
// A = X X^T, B = b A + c A A, X <- a X + B X; Gram form: R = X X^T,
// Q = a I + b R + c R R, Q_acc <- Q Q_acc, R <- (Q R) Q, restart, X = Q_acc X0),
// here every product is formed in full (R R, not the R R^T of the chained
// path, so R needs no exact symmetry).  The norm f = 1/(||U|| + eps) scales X0
// as it is loaded.
// ----------------------------------------------------------------------------
namespace {

constexpr int kFusedThreads = 512;  // two groups of 256
constexpr int kRedFloats = 16 * 256;  // split-K partial sums of the second group

// C = alpha * A op(B) + beta * Cin + eye * I, all in shared memory.
// A: M x K (lda).  NT: B stored N x K (C = A B^T), else K x N (C = A B).
// The block is two groups of 16 x 16 threads; a thread holds a 4 x 4 block of
// a 64 x 64 output tile: rows i0 + ty + 16 r; columns j0 + tx + 16 c (NT) or
// j0 + 4 tx + c (NN, so that a thread's four B values are one 16-byte load).
// A product of two or more tiles gives the groups alternate tiles; a one-tile
// product splits K between them and adds the second group's partial sums
// through `red` (16 x 256 floats).  k advances by 4 with 16-byte loads (a
// warp's A rows are two broadcast addresses; its B reads are 256 contiguous or
// row-strided bytes), then a scalar tail.  Every leading dimension is a
// multiple of 4 whose quarter is odd, which keeps 16-byte loads aligned and
// row-strided ones free of bank conflicts.  Rows and columns past M / N read a
// clamped (valid) index and are not stored, so the k loop carries no
// predicates.
template <bool NT>
__device__ __forceinline__ void tile_acc(const float* A, int lda, const float* B, int ldb, int M, int N, int i0,
                                         int j0, int kbeg, int kend, int tx, int ty, float (&acc)[4][4]) {
  const float* ap[4];
  const float* bp[4];
#pragma unroll
  for (int r = 0; r < 4; ++r) ap[r] = A + min(i0 + ty + 16 * r, M - 1) * lda;
  if (NT) {
#pragma unroll
    for (int c = 0; c < 4; ++c) bp[c] = B + min(j0 + tx + 16 * c, N - 1) * ldb;
  } else {
    bp[0] = B + min(j0 + 4 * tx, (N - 1) & ~3);  // 4 aligned columns inside the row
  }
  const int kend4 = kbeg + ((kend - kbeg) & ~3);  // kbeg is a multiple of 4
#pragma unroll 2
  for (int k = kbeg; k < kend4; k += 4) {
    float4 av[4], bv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) av[r] = *reinterpret_cast<const float4*>(ap[r] + k);
    if (NT) {
#pragma unroll
      for (int c = 0; c < 4; ++c) bv[c] = *reinterpret_cast<const float4*>(bp[c] + k);
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[r][c] = fmaf(av[r].x, bv[c].x, acc[r][c]);
          acc[r][c] = fmaf(av[r].y, bv[c].y, acc[r][c]);
          acc[r][c] = fmaf(av[r].z, bv[c].z, acc[r][c]);
          acc[r][c] = fmaf(av[r].w, bv[c].w, acc[r][c]);
        }
    } else {
#pragma unroll
      for (int q = 0; q < 4; ++q) bv[q] = *reinterpret_cast<const float4*>(bp[0] + (k + q) * ldb);
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float a4[4] = {av[r].x, av[r].y, av[r].z, av[r].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          acc[r][0] = fmaf(a4[q], bv[q].x, acc[r][0]);
          acc[r][1] = fmaf(a4[q], bv[q].y, acc[r][1]);
          acc[r][2] = fmaf(a4[q], bv[q].z, acc[r][2]);
          acc[r][3] = fmaf(a4[q], bv[q].w, acc[r][3]);
        }
      }
    }
  }
  for (int k = kend4; k < kend; ++k) {
    float av[4], bv[4];
#pragma unroll
    for (int r = 0; r < 4; ++r) av[r] = ap[r][k];
#pragma unroll
    for (int c = 0; c < 4; ++c) bv[c] = NT ? bp[c][k] : bp[0][k * ldb + c];
#pragma unroll
    for (int r = 0; r < 4; ++r)
#pragma unroll
      for (int c = 0; c < 4; ++c) acc[r][c] = fmaf(av[r], bv[c], acc[r][c]);
  }
}

template <bool NT>
__device__ __forceinline__ void tile_store(float* C, int ldc, int M, int N, int i0, int j0, int tx, int ty,
                                           const float (&acc)[4][4], float alpha, const float* Cin, int ldcin,
                                           float beta, float eye) {
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int i = i0 + ty + 16 * r;
    if (i >= M) continue;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = NT ? j0 + tx + 16 * c : j0 + 4 * tx + c;
      if (j >= N) continue;
      float v = alpha * acc[r][c];
      if (Cin) v += beta * Cin[i * ldcin + j];
      if (i == j) v += eye;
      C[i * ldc + j] = v;
    }
  }
}

template <bool NT>
__device__ void smem_mm(const float* A, int lda, const float* B, int ldb, float* C, int ldc, int M, int N, int K,
                        float alpha, const float* Cin, int ldcin, float beta, float eye, float* red) {
  const int g = threadIdx.x >> 8, t = threadIdx.x & 255;
  const int tx = t & 15, ty = t >> 4;
  const int tn = (N + 63) / 64, tiles = ((M + 63) / 64) * tn;
  if (tiles == 1) {
    const int Kh = (K / 2) & ~3;
    float acc[4][4] = {};
    tile_acc<NT>(A, lda, B, ldb, M, N, 0, 0, g == 0 ? 0 : Kh, g == 0 ? Kh : K, tx, ty, acc);
    if (g == 1) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) red[(r * 4 + c) * 256 + t] = acc[r][c];
    }
    __syncthreads();
    if (g == 0) {
#pragma unroll
      for (int r = 0; r < 4; ++r)
#pragma unroll
        for (int c = 0; c < 4; ++c) acc[r][c] += red[(r * 4 + c) * 256 + t];
      tile_store<NT>(C, ldc, M, N, 0, 0, tx, ty, acc, alpha, Cin, ldcin, beta, eye);
    }
  } else {
    for (int tile = g; tile < tiles; tile += 2) {
      const int i0 = (tile / tn) * 64, j0 = (tile % tn) * 64;
      float acc[4][4] = {};
      tile_acc<NT>(A, lda, B, ldb, M, N, i0, j0, 0, K, tx, ty, acc);
      tile_store<NT>(C, ldc, M, N, i0, j0, tx, ty, acc, alpha, Cin, ldcin, beta, eye);
    }
  }
  __syncthreads();
}

// Leading dimension for a row of `cols` floats: a multiple of 4 with an odd quarter.
__host__ __device__ inline int fused_ld(int cols) {
  const int q = (cols + 3) / 4;
  return 4 * (q | 1);
}

__device__ void smem_identity(float* Q, int ld, int n) {
  for (int e = threadIdx.x; e < n * n; e += blockDim.x) {
    const int i = e / n, j = e % n;
    Q[i * ld + j] = i == j ? 1.f : 0.f;
  }
  __syncthreads();
}

}  // namespace

__global__ void __launch_bounds__(kFusedThreads)
ns_fused_small_kernel(const FusedSmallArgs a) {
  extern __shared__ float sm[];
  const int n = a.n, m = a.m, ldx = fused_ld(m), ldn = fused_ld(n);
  float* X = sm;
  float* Y = X + n * ldx;
  float* S = Y + n * ldx;  // Gram-sized matrices, ldn each
  float* red = S + (a.mode == 0 ? 2 : 5) * n * ldn;
  float* xg = a.x + (long long)blockIdx.x * a.x_bs;
  const float f = a.raw ? a.inv[blockIdx.x] : 1.f;
  for (int e = threadIdx.x; e < n * m; e += blockDim.x) {
    const int i = e / m, j = e % m;
    X[i * ldx + j] = f * xg[(long long)i * a.ld_x + j];
  }
  __syncthreads();
  if (a.mode == 0) {
    float* Am = S;
    float* Bm = S + n * ldn;
    for (int k = 0; k < a.iters; ++k) {
      const float ca = a.coeffs[3 * k], cb = a.coeffs[3 * k + 1], cc = a.coeffs[3 * k + 2];
      smem_mm<true>(X, ldx, X, ldx, Am, ldn, n, n, m, 1.f, nullptr, 0, 0.f, 0.f, red);       // A = X X^T
      const float* P = Am;
      float coef = cb;
      if (cc != 0.f) {
        smem_mm<false>(Am, ldn, Am, ldn, Bm, ldn, n, n, n, cc, Am, ldn, cb, 0.f, red);       // B = c A A + b A
        P = Bm;
        coef = 1.f;
      }
      smem_mm<false>(P, ldn, X, ldx, Y, ldx, n, m, n, coef, X, ldx, ca, 0.f, red);           // X' = a X + B X
      float* t = X; X = Y; Y = t;
    }
  } else {
    float* R = S;
    float* Q = R + n * ldn;
    float* T = Q + n * ldn;
    float* Qa = T + n * ldn;
    float* Qb = Qa + n * ldn;
    smem_mm<true>(X, ldx, X, ldx, R, ldn, n, n, m, 1.f, nullptr, 0, 0.f, 0.f, red);         // R = X0 X0^T
    smem_identity(Qa, ldn, n);
    for (int k = 1; k <= a.iters; ++k) {
      const float ca = a.coeffs[3 * (k - 1)], cb = a.coeffs[3 * (k - 1) + 1], cc = a.coeffs[3 * (k - 1) + 2];
      smem_mm<false>(R, ldn, R, ldn, Q, ldn, n, n, n, cc, R, ldn, cb, ca, red);              // Q = a I + b R + c R R
      smem_mm<false>(Q, ldn, Qa, ldn, Qb, ldn, n, n, n, 1.f, nullptr, 0, 0.f, 0.f, red);      // Q_acc <- Q Q_acc
      float* t = Qa; Qa = Qb; Qb = t;
      if (k == a.iters) break;
      if (a.restart_after > 0 && k >= a.restart_after &&
          (k == a.restart_after || (a.restart_every > 0 && (k - a.restart_after) % a.restart_every == 0))) {
        smem_mm<false>(Qa, ldn, X, ldx, Y, ldx, n, m, n, 1.f, nullptr, 0, 0.f, 0.f, red);     // X <- Q_acc X0
        float* u = X; X = Y; Y = u;
        smem_mm<true>(X, ldx, X, ldx, R, ldn, n, n, m, 1.f, nullptr, 0, 0.f, 0.f, red);       // R <- X X^T
        smem_identity(Qa, ldn, n);
      } else {
        smem_mm<false>(Q, ldn, R, ldn, T, ldn, n, n, n, 1.f, nullptr, 0, 0.f, 0.f, red);      // T = Q R
        smem_mm<false>(T, ldn, Q, ldn, R, ldn, n, n, n, 1.f, nullptr, 0, 0.f, 0.f, red);      // R <- T Q
      }
    }
    smem_mm<false>(Qa, ldn, X, ldx, Y, ldx, n, m, n, 1.f, nullptr, 0, 0.f, 0.f, red);         // X = Q_acc X0
    X = Y;
  }
  for (int e = threadIdx.x; e < n * m; e += blockDim.x) {
    const int i = e / m, j = e % m;
    xg[(long long)i * a.ld_x + j] = X[i * ldx + j];
  }
}

size_t fused_small_smem(int n, int m, int mode) {
  const size_t sq = mode == 0 ? 2 : 5;
  return sizeof(float) * (2 * (size_t)n * fused_ld(m) + sq * (size_t)n * fused_ld(n) + kRedFloats);
}

int launch_fused_small(const FusedSmallArgs& a, cudaStream_t s) {
  const size_t bytes = fused_small_smem(a.n, a.m, a.mode);
  if (bytes > kFusedSmallMaxSmem || a.iters > FusedSmallArgs::kMaxIters) return (int)cudaErrorInvalidValue;
  static std::atomic<int> attr_done[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return (int)cudaErrorInvalidDevice;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(ns_fused_small_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kFusedSmallMaxSmem);
    if (e != cudaSuccess) return (int)e;
    attr_done[dev].store(1, std::memory_order_release);
  }
  ns_fused_small_kernel<<<a.count, kFusedThreads, bytes, s>>>(a);
  return (int)cudaGetLastError();
}

}  // namespace muon
