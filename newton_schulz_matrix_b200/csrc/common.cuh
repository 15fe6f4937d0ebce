// Shared device/host helpers for the Muon step kernels (sm_100a).
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace muon {

// Storage types the kernels read and write.  The numbering matches muon_dtype.
enum DType : int { kBF16 = 0, kFP16 = 1, kFP32 = 2 };

__host__ __device__ inline int dtype_size(int dt) { return dt == kFP32 ? 4 : 2; }

template <typename T> struct TypeOf;
template <> struct TypeOf<__nv_bfloat16> { static constexpr int value = kBF16; };
template <> struct TypeOf<__half> { static constexpr int value = kFP16; };
template <> struct TypeOf<float> { static constexpr int value = kFP32; };

__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }
__device__ __forceinline__ float to_f32(__half v) { return __half2float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) { return __float2bfloat16_rn(v); }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }

// Read a float from a pointer whose element type is only known at run time.
__device__ __forceinline__ float load_any(const void* p, long long i, int dt) {
  if (dt == kBF16) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
  if (dt == kFP16) return __half2float(reinterpret_cast<const __half*>(p)[i]);
  return reinterpret_cast<const float*>(p)[i];
}
__device__ __forceinline__ void store_any(void* p, long long i, int dt, float v) {
  if (dt == kBF16) reinterpret_cast<__nv_bfloat16*>(p)[i] = __float2bfloat16_rn(v);
  else if (dt == kFP16) reinterpret_cast<__half*>(p)[i] = __float2half_rn(v);
  else reinterpret_cast<float*>(p)[i] = v;
}

// Per-matrix scale factor f = scale[b]^pow (pow 0 or a null pointer -> 1).
__device__ __forceinline__ float matrix_scale(const float* scale, int pow, int b) {
  if (scale == nullptr || pow == 0) return 1.f;
  float s = scale[b];
  return pow == 2 ? s * s : s;
}

// The decoupled-weight-decay update of one element, W <- (1 - lr wd) W - step O
// ("Moonlight 16B Guide", Innovation 1 and box step 4), with its rounding fixed:
// decay * w rounded once, then one fused multiply-add.  Every kernel that
// writes W uses this, so the results do not depend on which one ran.
__device__ __forceinline__ float weight_update(float w, float o, float decay, float step) {
  return __fmaf_rn(-step, o, __fmul_rn(decay, w));
}

// Device-side error bits (also the bits of the per-matrix status words).
constexpr int kStatusNonFinite = 1;
constexpr int kStatusTimeout = 2;

}  // namespace muon
