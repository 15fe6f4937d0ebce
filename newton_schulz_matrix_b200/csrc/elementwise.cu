// HBM-bound kernels of the Muon step: momentum + Nesterov + orientation pack
// with per-tile sums of squares, the Frobenius-norm finalisation, and the
// update (decoupled weight decay + scaled orthogonalised step) with the
// transpose back to storage orientation.
//
// Steps follow "Moonlight 16B Guide: Scalable MoE & Muon Optimizer":
//   box "Scalable Muon Optimizer Step" step 1 (M = beta M + (1 - beta) G),
//   step 3 (s(W) = sqrt(max(d_out, d_in))), step 4 and "Innovation 1"
//   (W = (1 - eta lambda) W - eta U), and the listing's orientation (m <= n).
//
// Layout: a 64 x 64 storage tile per 256-thread block.  The pack gives each
// thread 4 consecutive elements of 4 tile rows (16 threads per 64-element row
// segment); the update pass gives each thread 16 consecutive elements of one
// tile row (it measured faster that way).  Tall matrices go through a padded
// shared-memory tile so that both the storage read and the oriented write
// stay row-contiguous.
#include "common.cuh"
#include "internal.h"

namespace muon {

constexpr int kTile = 64;
constexpr int kPackThreads = 256;

int pack_tiles(int rows, int cols) {
  return ((rows + kTile - 1) / kTile) * ((cols + kTile - 1) / kTile);
}

template <typename T>
__device__ __forceinline__ void load4(const T* p, float* v) {
  // 4 elements: p is 8-byte aligned for 16-bit types, 16-byte aligned for fp32
  if constexpr (sizeof(T) == 2) {
    const uint2 q = *reinterpret_cast<const uint2*>(p);
    const T* e = reinterpret_cast<const T*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = to_f32(e[i]);
  } else {
    const float4 f = *reinterpret_cast<const float4*>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
  }
}
template <typename T>
__device__ __forceinline__ void store4(T* p, const float* v) {
  if constexpr (sizeof(T) == 2) {
    uint2 q;
    T* e = reinterpret_cast<T*>(&q);
#pragma unroll
    for (int i = 0; i < 4; ++i) e[i] = from_f32<T>(v[i]);
    *reinterpret_cast<uint2*>(p) = q;
  } else {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
}

template <typename T>
__device__ __forceinline__ void load16(const T* p, float* v) {
  // p is 16-byte aligned; 16 elements.
  if constexpr (sizeof(T) == 2) {
    uint4 q0 = reinterpret_cast<const uint4*>(p)[0];
    uint4 q1 = reinterpret_cast<const uint4*>(p)[1];
    const T* e0 = reinterpret_cast<const T*>(&q0);
    const T* e1 = reinterpret_cast<const T*>(&q1);
#pragma unroll
    for (int i = 0; i < 8; ++i) { v[i] = to_f32(e0[i]); v[8 + i] = to_f32(e1[i]); }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      float4 f = reinterpret_cast<const float4*>(p)[q];
      v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
    }
  }
}

template <typename T>
__device__ __forceinline__ void store16(T* p, const float* v) {
  if constexpr (sizeof(T) == 2) {
    uint4 q0, q1;
    T* e0 = reinterpret_cast<T*>(&q0);
    T* e1 = reinterpret_cast<T*>(&q1);
#pragma unroll
    for (int i = 0; i < 8; ++i) { e0[i] = from_f32<T>(v[i]); e1[i] = from_f32<T>(v[8 + i]); }
    reinterpret_cast<uint4*>(p)[0] = q0;
    reinterpret_cast<uint4*>(p)[1] = q1;
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      reinterpret_cast<float4*>(p)[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
}

__device__ __forceinline__ float block_sum_fixed(float v, float* red) {
  // Deterministic: fixed shuffle tree, then warp 0 adds the 8 warp sums in order.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_down_sync(0xffffffffu, v, o);
  const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
  if (l == 0) red[w] = v;
  __syncthreads();
  float s = 0.f;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kPackThreads / 32; ++i) s += red[i];
  }
  return s;
}

// ----------------------------------------------------------------------------
// pack: U -> oriented workspace X (+ momentum update), sums of squares per tile
// ----------------------------------------------------------------------------
// Thread mapping: 16 threads per 64-element row segment, 4 elements each, four
// row passes of 16 rows.  Every load and store instruction of a warp then
// covers two whole row segments (2 x 128 bytes of a 16-bit type, 2 x 256 bytes
// of fp32), so no L1 sector is requested twice.  (With 4 threads per segment
// and 16 elements each, consecutive 16-byte accesses of a thread each touched
// half of a sector: half the L1 requests were repeats, and the pack slowed with
// the SM clock under the power cap.)
template <typename TS, typename TX, bool MOMENTUM, bool TRANS>
__global__ void __launch_bounds__(kPackThreads)
pack_kernel(const PackArgs a, const __grid_constant__ SegmentPtrs p) {
  __shared__ float tile[TRANS ? kTile : 1][kTile + 1];
  __shared__ float red[kPackThreads / 32];
  const int b = blockIdx.y;
  const int tcols = (a.cols + kTile - 1) / kTile;
  const int r0 = (blockIdx.x / tcols) * kTile, c0 = (blockIdx.x % tcols) * kTile;
  const int lr = threadIdx.x >> 4, lc = (threadIdx.x & 15) * 4;
  const TS* src = reinterpret_cast<const TS*>(p.src[b]);
  float* mom = MOMENTUM ? p.mom[b] : nullptr;
  TX* x = reinterpret_cast<TX*>(a.x) + (long long)b * a.x_batch_stride;

  const bool full = (r0 + kTile <= a.rows) && (c0 + kTile <= a.cols) && (a.cols % 8 == 0);
  const bool store = a.pass != 1;
  float u[4][4];  // [row pass][element]
  if (full) {
    // every load of the four passes first: one memory round trip per thread
    float g[4][4], m[4][4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const long long off = (long long)(r0 + q * 16 + lr) * a.cols + c0 + lc;
      load4(src + off, g[q]);
      if (MOMENTUM) load4(mom + off, m[q]);
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (MOMENTUM) {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          m[q][i] = a.mu * m[q][i] + (1.f - a.mu) * g[q][i];
          u[q][i] = a.nesterov ? (1.f - a.mu) * g[q][i] + a.mu * m[q][i] : m[q][i];
        }
        if (store) store4(mom + (long long)(r0 + q * 16 + lr) * a.cols + c0 + lc, m[q]);
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) u[q][i] = g[q][i];
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + q * 16 + lr;
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int c = c0 + lc + i;
        u[q][i] = 0.f;
        if (r < a.rows && c < a.cols) {
          const long long off = (long long)r * a.cols + c;
          const float gv = to_f32(src[off]);
          if (MOMENTUM) {
            const float mv = a.mu * mom[off] + (1.f - a.mu) * gv;
            if (store) mom[off] = mv;
            u[q][i] = a.nesterov ? (1.f - a.mu) * gv + a.mu * mv : mv;
          } else {
            u[q][i] = gv;
          }
        }
      }
    }
  }
  float ssq = 0.f;
  if (a.pass != 2) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) ssq += u[q][i] * u[q][i];
  }
  if (a.pass == 1) {
    const float s = block_sum_fixed(ssq, red);
    if (threadIdx.x == 0) a.partials[(long long)b * a.partial_stride + blockIdx.x] = s;
    return;
  }
  if (a.pass == 2) {
    const float f = a.scale[b];
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) u[q][i] *= f;
  }

  if (!TRANS) {
    // oriented == storage: row r, columns c0 + lc ...
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int r = r0 + q * 16 + lr;
      if (full) {
        store4(x + (long long)r * a.ld_x + c0 + lc, u[q]);
      } else if (r < a.rows) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (c0 + lc + i < a.cols) x[(long long)r * a.ld_x + c0 + lc + i] = from_f32<TX>(u[q][i]);
      }
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q)
#pragma unroll
      for (int i = 0; i < 4; ++i) tile[q * 16 + lr][lc + i] = u[q][i];
    __syncthreads();
    // oriented row j = storage column c0 + q * 16 + lr; oriented columns = storage rows r0 + lc + i
    const bool fullT = (c0 + kTile <= a.cols) && (r0 + kTile <= a.rows);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int j = c0 + q * 16 + lr;
      float v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = tile[lc + i][q * 16 + lr];
      if (fullT) {
        store4(x + (long long)j * a.ld_x + r0 + lc, v);
      } else if (j < a.cols) {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          if (r0 + lc + i < a.rows) x[(long long)j * a.ld_x + r0 + lc + i] = from_f32<TX>(v[i]);
      }
    }
  }
  if (a.pass == 0) {
    const float s = block_sum_fixed(ssq, red);
    if (threadIdx.x == 0) a.partials[(long long)b * a.partial_stride + blockIdx.x] = s;
  }
}

// ----------------------------------------------------------------------------
// norm: inv[b] = 1 / (sqrt(sum_i partials[b][i]) + eps)
// ----------------------------------------------------------------------------
__global__ void __launch_bounds__(256)
norm_kernel(const float* __restrict__ partials, int stride, int n, float eps, float* __restrict__ inv) {
  __shared__ double red[256];
  const int b = blockIdx.x;
  double s = 0.0;
  for (int i = threadIdx.x; i < n; i += 256) s += (double)partials[(long long)b * stride + i];
  red[threadIdx.x] = s;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) inv[b] = (float)(1.0 / (sqrt(red[0]) + (double)eps));
}

// ----------------------------------------------------------------------------
// unpack: oriented O -> storage (update W, or overwrite X), non-finite flags
// ----------------------------------------------------------------------------
template <typename TD, typename TX, bool UPDATE, bool TRANS>
__global__ void __launch_bounds__(kPackThreads)
unpack_kernel(const UnpackArgs a, const __grid_constant__ SegmentPtrs p) {
  __shared__ float tile[TRANS ? kTile : 1][kTile + 1];
  const int b = blockIdx.y;
  const int tcols = (a.cols + kTile - 1) / kTile;
  const int r0 = (blockIdx.x / tcols) * kTile, c0 = (blockIdx.x % tcols) * kTile;
  const int lr = threadIdx.x >> 2, lc = (threadIdx.x & 3) * 16;
  const TX* __restrict__ x = reinterpret_cast<const TX*>(a.x) + (long long)b * a.x_batch_stride;
  TD* __restrict__ dst = reinterpret_cast<TD*>(p.dst[b]);
  const bool full = (r0 + kTile <= a.rows) && (c0 + kTile <= a.cols) && (a.cols % 8 == 0);
  const int r = r0 + lr;
  const long long off = (long long)r * a.cols + c0 + lc;

  // Both global loads (W and the orientated O) are issued before either is used,
  // so each thread waits for one memory round trip, not two.
  float w[16];
  if (UPDATE && full) load16(dst + off, w);
  float o[16];
  if (!TRANS) {
    if (full) {
      load16(x + (long long)r * a.ld_x + c0 + lc, o);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        o[i] = (r < a.rows && c0 + lc + i < a.cols) ? to_f32(x[(long long)r * a.ld_x + c0 + lc + i]) : 0.f;
    }
  } else {
    // read oriented rows j = c0 + lr (storage columns), oriented cols = storage rows
    const int j = c0 + lr;
    float v[16];
    if (full) {
      load16(x + (long long)j * a.ld_x + r0 + lc, v);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i)
        v[i] = (j < a.cols && r0 + lc + i < a.rows) ? to_f32(x[(long long)j * a.ld_x + r0 + lc + i]) : 0.f;
    }
#pragma unroll
    for (int i = 0; i < 16; ++i) tile[lr][lc + i] = v[i];
    __syncthreads();
#pragma unroll
    for (int i = 0; i < 16; ++i) o[i] = tile[lc + i][lr];
  }

  if (full) {
    if (UPDATE) {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = weight_update(w[i], o[i], a.decay, a.step);
    } else {
#pragma unroll
      for (int i = 0; i < 16; ++i) w[i] = o[i];
    }
    store16(dst + off, w);
  } else if (r < a.rows) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      const int c = c0 + lc + i;
      if (c < a.cols) {
        const long long o2 = (long long)r * a.cols + c;
        float v = UPDATE ? weight_update(to_f32(dst[o2]), o[i], a.decay, a.step) : o[i];
        dst[o2] = from_f32<TD>(v);
      }
    }
  }

  if (a.status != nullptr) {
    int bad = 0;
#pragma unroll
    for (int i = 0; i < 16; ++i) bad |= !isfinite(o[i]);
    bad = __any_sync(0xffffffffu, bad);
    if ((threadIdx.x & 31) == 0) {
      int st = bad ? kStatusNonFinite : 0;
      if (blockIdx.x == 0 && threadIdx.x == 0 && a.chunk_err != nullptr) st |= *a.chunk_err;
      if (st) atomicOr(a.status + b, st);
    }
  }
}

// ----------------------------------------------------------------------------
// dtype conversion of a flat array (rare Gram-mode corner cases)
// ----------------------------------------------------------------------------
__global__ void convert_kernel(const void* src, int sdt, void* dst, int ddt, long long n) {
  for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    store_any(dst, i, ddt, load_any(src, i, sdt));
}

// ----------------------------------------------------------------------------
// launchers
// ----------------------------------------------------------------------------
template <typename TS, typename TX>
static void pack_dispatch2(const PackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  const bool trans = a.rows > a.cols;
  dim3 grid(pack_tiles(a.rows, a.cols), a.count);
  if (a.momentum_mode) {
    if (trans) pack_kernel<TS, TX, true, true><<<grid, kPackThreads, 0, s>>>(a, p);
    else pack_kernel<TS, TX, true, false><<<grid, kPackThreads, 0, s>>>(a, p);
  } else {
    if (trans) pack_kernel<TS, TX, false, true><<<grid, kPackThreads, 0, s>>>(a, p);
    else pack_kernel<TS, TX, false, false><<<grid, kPackThreads, 0, s>>>(a, p);
  }
}

template <typename TS>
static void pack_dispatch1(const PackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  switch (a.x_dtype) {
    case kBF16: pack_dispatch2<TS, __nv_bfloat16>(a, p, s); break;
    case kFP16: pack_dispatch2<TS, __half>(a, p, s); break;
    default: pack_dispatch2<TS, float>(a, p, s); break;
  }
}

void launch_pack(const PackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  if (a.count <= 0) return;
  switch (a.src_dtype) {
    case kBF16: pack_dispatch1<__nv_bfloat16>(a, p, s); break;
    case kFP16: pack_dispatch1<__half>(a, p, s); break;
    default: pack_dispatch1<float>(a, p, s); break;
  }
}

void launch_norm(const float* partials, int stride, int n, int count, float eps, float* inv, cudaStream_t s) {
  if (count <= 0) return;
  norm_kernel<<<count, 256, 0, s>>>(partials, stride, n, eps, inv);
}

template <typename TD, typename TX>
static void unpack_dispatch2(const UnpackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  dim3 grid(pack_tiles(a.rows, a.cols), a.count);
  const bool trans = a.rows > a.cols;
  if (a.update_mode) {
    if (trans) unpack_kernel<TD, TX, true, true><<<grid, kPackThreads, 0, s>>>(a, p);
    else unpack_kernel<TD, TX, true, false><<<grid, kPackThreads, 0, s>>>(a, p);
  } else {
    if (trans) unpack_kernel<TD, TX, false, true><<<grid, kPackThreads, 0, s>>>(a, p);
    else unpack_kernel<TD, TX, false, false><<<grid, kPackThreads, 0, s>>>(a, p);
  }
}

template <typename TD>
static void unpack_dispatch1(const UnpackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  switch (a.x_dtype) {
    case kBF16: unpack_dispatch2<TD, __nv_bfloat16>(a, p, s); break;
    case kFP16: unpack_dispatch2<TD, __half>(a, p, s); break;
    default: unpack_dispatch2<TD, float>(a, p, s); break;
  }
}

void launch_unpack(const UnpackArgs& a, const SegmentPtrs& p, cudaStream_t s) {
  if (a.count <= 0) return;
  switch (a.dst_dtype) {
    case kBF16: unpack_dispatch1<__nv_bfloat16>(a, p, s); break;
    case kFP16: unpack_dispatch1<__half>(a, p, s); break;
    default: unpack_dispatch1<float>(a, p, s); break;
  }
}

__global__ void status_or_kernel(int* status, int count, const int* chunk_err) {
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  const int e = *chunk_err;
  if (i < count && e != 0) status[i] |= e;
}

void launch_status_or(int* status, int count, const int* chunk_err, cudaStream_t s) {
  if (count <= 0 || status == nullptr) return;
  status_or_kernel<<<(count + 255) / 256, 256, 0, s>>>(status, count, chunk_err);
}

void launch_convert(const void* src, int sdt, void* dst, int ddt, long long n, cudaStream_t s) {
  if (n <= 0) return;
  int blocks = (int)((n + 255) / 256);
  if (blocks > 148 * 16) blocks = 148 * 16;
  convert_kernel<<<blocks, 256, 0, s>>>(src, sdt, dst, ddt, n);
}

}  // namespace muon
