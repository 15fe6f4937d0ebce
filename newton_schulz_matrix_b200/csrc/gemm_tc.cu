// Tensor-core product for the Newton-Schulz chain on sm_100a (tcgen05 + TMEM + TMA).
//
// Every product of the iteration ("Gram Newton-Schulz" write-up: X X^T, A^2,
// B X; and the Gram form's R^2, Q Q_acc, Q R Q, Q_acc X_0) is one launch of
// this kernel over a batch of same-shape matrices:
//
//   D[b] = f_b * (c_acc * A[b] op(B[b]) + c_in * C[b]) + c_eye * I
//
// with f_b = scale[b]^p carrying the Frobenius normalisation into the first
// products (so the packed X_0 never has to be rescaled in memory), C the
// polynomial's linear term (b A, b R) or the a X term, and c_eye the a I of
// Q = a I + b R + c R^2.  Symmetric results (X X^T, A A, R R) are computed on
// the upper-triangle 128 x 128 blocks only and mirrored on store.
//
// Structure (one CTA per SM, persistent over the batch's tiles):
//   warp 0        TMA producer: 128x64 A tile + 256x64 B tile per stage,
//                 128-byte swizzle, STAGES-deep ring of shared-memory slots
//   warp 1        TMEM allocator + single-thread tcgen05.mma issuer
//                 (M=128, N=256, K=16 per instruction, fp32 accumulate)
//   warps 2..5    epilogue: tcgen05.ld of the accumulator (one TMEM lane =
//                 one output row per thread), polynomial epilogue, stores
//   TMEM holds two 128x256 fp32 accumulators so the epilogue of tile i
//   overlaps the main loop of tile i+1.
// Every mbarrier wait is bounded (global-timer deadline plus a CTA-wide abort
// flag); on expiry the CTA drains its in-flight copies and MMAs, frees TMEM,
// raises the timeout bit in the caller's error word and returns.
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "tc_common.cuh"

namespace muon {
namespace tc {

// ------------------------------------------------------------------ kernel
template <bool B_MN, int IN_FMT, bool SYM>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
            const __grid_constant__ CUtensorMap tmap_d,
            const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * STAGE_BYTES;  // per epilogue warp: two 1024-aligned 2 KB boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + STAGING_BYTES);
  uint64_t* full_bar = bars;                    // [STAGES]
  uint64_t* empty_bar = bars + STAGES;          // [STAGES]
  uint64_t* tfull_bar = bars + 2 * STAGES;      // [2]
  uint64_t* tempty_bar = bars + 2 * STAGES + 2; // [2]
  uint64_t* drain_bar = bars + 2 * STAGES + 4;  // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 5);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), 32 * NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_a)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_b)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_d)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.K + BK - 1) / BK;

  if (warp == 0) {
    // ---------------------------------------------------------------- producer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      uint32_t issued[STAGES];
      for (int s = 0; s < STAGES; ++s) issued[s] = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x) {
        const Tile tl = decode_tile(p, t);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          const uint32_t fb = smem_u32(&full_bar[stage]);
          mbar_expect_tx(fb, STAGE_BYTES);
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          tma_load_3d(sa, &tmap_a, fb, kb * BK, tl.tm * BM, tl.b);
          if (B_MN) {
#pragma unroll
            for (int q = 0; q < BN / 64; ++q) tma_load_3d(sb + q * (BK * 128), &tmap_b, fb, tl.tn * BN + q * 64, kb * BK, tl.b);
          } else {
            tma_load_3d(sb, &tmap_b, fb, kb * BK, tl.tn * BN, tl.b);
          }
          issued[stage]++;
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
      if (!ok) {
        // drain: every stage's most recent load must land before the CTA exits
        for (int s = 0; s < STAGES; ++s)
          if (issued[s]) {
            volatile int never = 0;
            mbar_wait(smem_u32(&full_bar[s]), (issued[s] - 1) & 1u, &never, p.timeout_ns);
          }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = make_idesc(IN_FMT, B_MN ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < p.total_tiles && ok; t += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), aph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = smem_desc(sa + k * (UMMA_K * 2), 16, 1024);
            const uint64_t bd = B_MN ? smem_desc(sb + k * (UMMA_K * 128), BK * 128, 1024)
                                     : smem_desc(sb + k * (UMMA_K * 2), 16, 1024);
            tc_mma(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          tc_commit(smem_u32(&empty_bar[stage]));  // slot free once these MMAs retire
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        tc_commit(smem_u32(&tfull_bar[acc]));      // accumulator ready for the epilogue
      }
      // all issued MMAs retire before TMEM is released
      tc_commit(smem_u32(drain_bar));
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, &never, p.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------------- epilogue
    const int q = warp & 3;                      // TMEM lane quarter this warp may access
    const int half = (warp - 2) >> 2;            // which 4 of the 8 column chunks
    uint8_t* S = staging + (warp - 2) * 2 * STAGE_TILE_BYTES;
    uint8_t* T = S + STAGE_TILE_BYTES;
    int it = 0;
    for (int t = blockIdx.x; t < p.total_tiles; t += gridDim.x, ++it) {
      const Tile tl = decode_tile(p, t);
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&tfull_bar[acc]), aph, abort_flag, p.timeout_ns);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const float f = matrix_scale(p.scale, p.scale_pow, tl.b);
      const uint32_t tbase = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      const int gi = tl.tm * BM + q * 32 + lane;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        const int c = half * 4 + cc;
        const int gj0 = tl.tn * BN + c * 32;
        // C row segment first, so its latency overlaps the TMEM read
        uint4 creg[4];
        bool c_ready = false;
        if (p.C != nullptr && gi < p.M && gj0 + 32 <= p.N) {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.C) +
                                                            ((long long)tl.b * p.c_bs + (long long)gi * p.ldc + gj0) * 2);
#pragma unroll
          for (int i = 0; i < 4; ++i) creg[i] = src[i];
          c_ready = true;
        }
        uint32_t r[32];
        tmem_ld32(tbase + (uint32_t)(c * 32), r);
        if (cc == 3) {
          tc_fence_before();
          mbar_arrive(smem_u32(&tempty_bar[acc]));
        }
        epilogue_chunk<SYM>(p, &tmap_d, tl, q, lane, c, r, creg, c_ready, f, S, T);
      }
    }
    if (lane == 0) bulk_wait_all0();  // this warp's output stores have completed
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS)
                 : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag && p.err != nullptr) atomicOr(p.err, kStatusTimeout);
}

// ------------------------------------------------------------------ host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  // thread-safe one-time lookup (the entry point does not depend on the device)
  static const EncodeTiledFn fn = [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      return reinterpret_cast<EncodeTiledFn>(ptr);
    return static_cast<EncodeTiledFn>(nullptr);
  }();
  return fn;
}

// 3-D tiled map over a batch of row-major matrices: dims (inner, outer, batch).
bool encode_map(CUtensorMap* map, int dtype, const void* base, long long inner, long long outer, long long batch,
                long long ld_elems, long long bs_elems, int box_inner, int box_outer, TmaSwizzle swizzle) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return false;
  const CUtensorMapDataType dt = dtype == kBF16   ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16
                                 : dtype == kFP16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16
                                                  : CU_TENSOR_MAP_DATA_TYPE_FLOAT32;
  const long long es = dtype_size(dtype);
  cuuint64_t dims[3] = {(cuuint64_t)inner, (cuuint64_t)outer, (cuuint64_t)batch};
  cuuint64_t strides[2] = {(cuuint64_t)(ld_elems * es), (cuuint64_t)((bs_elems > 0 ? bs_elems : ld_elems * outer) * es)};
  cuuint32_t box[3] = {(cuuint32_t)box_inner, (cuuint32_t)box_outer, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  const CUtensorMapSwizzle sw = swizzle == kTmaSw64          ? CU_TENSOR_MAP_SWIZZLE_64B
                                : swizzle == kTmaSw128Atom32 ? CU_TENSOR_MAP_SWIZZLE_128B_ATOM_32B
                                                             : CU_TENSOR_MAP_SWIZZLE_128B;
  CUresult r = enc(map, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool encode_out_map(CUtensorMap* map, const GemmDesc& g) {
  return encode_map(map, g.d_dtype, g.D, g.N, g.M, g.batch, g.ldd, g.d_bs, 32, 32, kTmaSw64);
}

template <bool B_MN, int IN_FMT, bool SYM>
static int launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md, const Params& p,
                  cudaStream_t s) {
  // the shared-memory opt-in is a per-device function attribute: set once per device
  static std::atomic<int> attr_done[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return (int)cudaErrorInvalidDevice;
  if (!attr_done[dev].load(std::memory_order_acquire)) {
    cudaError_t e = cudaFuncSetAttribute(gemm_kernel<B_MN, IN_FMT, SYM>, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return (int)e;
    attr_done[dev].store(1, std::memory_order_release);
  }
  const int grid = p.total_tiles < num_sms() ? p.total_tiles : num_sms();
  gemm_kernel<B_MN, IN_FMT, SYM><<<grid, NUM_THREADS, SMEM_BYTES, s>>>(ma, mb, md, p);
  return (int)cudaGetLastError();
}

}  // namespace tc

namespace {
// 256-row products go to the paired-CTA kernel (a third less operand
// traffic per MMA); MUON_GEMM_PAIR=0 keeps every product on the 1-CTA one.
bool use_pair_kernel(const GemmDesc& g) {
  static const int use_pair = [] {
    const char* e = getenv("MUON_GEMM_PAIR");
    return (e && e[0] == '0') ? 0 : 1;
  }();
  return use_pair && g.M >= 256;
}
}  // namespace

bool gemm_tc_paired(int M) {
  GemmDesc g{};
  g.M = M;
  return use_pair_kernel(g);
}

double gemm_tc_exec_flops(const GemmDesc& g) {
  using namespace tc;
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return 0.0;
  const double k_pad = (double)((g.K + BK - 1) / BK) * BK;
  double per_batch = 0.0;  // sum over launched tiles of tile_rows * tile_cols
  if (use_pair_kernel(g)) {
    const int tm = (g.M + 255) / 256, tn = (g.N + 255) / 256;
    const bool narrow = g.N - (tn - 1) * 256 <= 128;  // last column tile runs N = 128 MMAs
    for (int r = 0; r < tm; ++r)
      for (int c = g.symmetric ? r : 0; c < tn; ++c) per_batch += 256.0 * ((c == tn - 1 && narrow) ? 128 : 256);
  } else {
    const int tm = (g.M + BM - 1) / BM, tn = (g.N + BN - 1) / BN;
    for (int r = 0; r < tm; ++r) per_batch += (double)(tn - (g.symmetric ? r / 2 : 0)) * BM * BN;
  }
  return 2.0 * per_batch * k_pad * g.batch;
}

int gemm_tc(const GemmDesc& g, cudaStream_t s) {
  using namespace tc;
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return 0;
  if (g.in_dtype != kBF16 && g.in_dtype != kFP16) return (int)cudaErrorInvalidValue;
  if (g.d_dtype == kFP32 || (g.C && g.c_dtype == kFP32)) return (int)cudaErrorInvalidValue;
  if (g.symmetric && g.M != g.N) return (int)cudaErrorInvalidValue;
  Params p{};
  p.M = g.M; p.N = g.N; p.K = g.K; p.batch = g.batch;
  p.tiles_m = (g.M + BM - 1) / BM;
  p.tiles_n = (g.N + BN - 1) / BN;
  if (g.symmetric) {
    int cnt = 0;
    for (int tm = 0; tm < p.tiles_m; ++tm) cnt += p.tiles_n - tm / 2;
    p.tiles_per_batch = cnt;
  } else {
    p.tiles_per_batch = p.tiles_m * p.tiles_n;
  }
  long long total = (long long)p.tiles_per_batch * g.batch;
  if (total > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  p.total_tiles = (int)total;
  p.symmetric = g.symmetric;
  p.D = g.D; p.ldd = g.ldd; p.d_bs = g.d_bs; p.d_dtype = g.d_dtype;
  p.C = g.C; p.ldc = g.ldc; p.c_bs = g.c_bs; p.c_dtype = g.c_dtype;
  p.c_acc = g.c_acc; p.c_in = g.c_in; p.c_eye = g.c_eye;
  p.scale = g.scale; p.scale_pow = g.scale_pow;
  p.err = g.err;
  p.timeout_ns = wait_timeout_ns();
  p.tile_counter = g.tile_counter;
  p.static_order = static_tile_order() ? 1 : 0;

  if (use_pair_kernel(g)) return gemm_tc_pair(g, p, s);
  if (g.update != nullptr) return (int)cudaErrorInvalidValue;  // the fused update is a paired-kernel epilogue

  CUtensorMap ma, mb;
  if (!encode_map(&ma, g.in_dtype, g.A, g.K, g.M, g.batch, g.lda, g.a_bs, BK, BM)) return (int)cudaErrorInvalidValue;
  const bool bmn = !g.b_kmajor;
  if (bmn) {
    if (!encode_map(&mb, g.in_dtype, g.B, g.N, g.K, g.batch, g.ldb, g.b_bs, 64, BK)) return (int)cudaErrorInvalidValue;
  } else {
    if (!encode_map(&mb, g.in_dtype, g.B, g.K, g.N, g.batch, g.ldb, g.b_bs, BK, BN)) return (int)cudaErrorInvalidValue;
  }
  CUtensorMap md;
  if (!encode_out_map(&md, g)) return (int)cudaErrorInvalidValue;
  const int fmt = g.in_dtype == kBF16 ? 1 : 0;
  if (g.symmetric) {
    if (bmn) return fmt ? launch<true, 1, true>(ma, mb, md, p, s) : launch<true, 0, true>(ma, mb, md, p, s);
    return fmt ? launch<false, 1, true>(ma, mb, md, p, s) : launch<false, 0, true>(ma, mb, md, p, s);
  }
  if (bmn) return fmt ? launch<true, 1, false>(ma, mb, md, p, s) : launch<true, 0, false>(ma, mb, md, p, s);
  return fmt ? launch<false, 1, false>(ma, mb, md, p, s) : launch<false, 0, false>(ma, mb, md, p, s);
}

bool tc::static_tile_order() {
  static const bool on = [] {
    const char* e = getenv("MUON_TILE_ORDER");
    return e && strcmp(e, "static") == 0;
  }();
  return on;
}

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int num_sms() {
  static std::atomic<int> cached[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return 148;
  int n = cached[dev].load(std::memory_order_acquire);
  if (n <= 0) {
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cached[dev].store(n, std::memory_order_release);
  }
  return n;
}

long long wait_timeout_ns() {
  static const long long ns = [] {
    const char* e = getenv("MUON_WAIT_TIMEOUT_MS");
    long long ms = e ? atoll(e) : 4000;
    if (ms <= 0) ms = 4000;
    return ms * 1000000LL;
  }();
  return ns;
}

}  // namespace muon
