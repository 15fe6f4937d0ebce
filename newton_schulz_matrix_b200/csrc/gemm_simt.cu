// CUDA-core (FFMA) batched product with the same epilogue as the tensor-core
// kernel.  It carries the fp32 compute mode: tcgen05 offers only TF32 for
// 32-bit operands, whose 10-bit mantissa cannot hold a 1e-4 relative error
// through five Newton-Schulz iterations.
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

}  // namespace muon
