// Device-side building blocks shared by the tcgen05 product kernels (1-CTA
// and 2-CTA): constants, launch parameters, PTX wrappers for mbarriers, TMA,
// tcgen05 MMA / TMEM, shared-memory descriptors, the tile order and the
// fused polynomial epilogue.
#pragma once

#include <cuda.h>

#include "common.cuh"
#include "internal.h"

namespace muon {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;                   // 64 x 2 B = one 128-byte swizzle row
constexpr int UMMA_K = 16;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;     // 16 KB
constexpr int B_BYTES = BN * BK * 2;     // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int NUM_EPI_WARPS = 8;         // two per TMEM lane quarter, 4 chunks of 32 columns each
constexpr int NUM_THREADS = 64 + 32 * NUM_EPI_WARPS;
constexpr int TMEM_COLS = 2 * BN;        // two fp32 accumulators
constexpr int STAGE_TILE_BYTES = 32 * 32 * 2;                     // one 32 x 32 16-bit output box
constexpr int STAGING_BYTES = NUM_EPI_WARPS * 2 * STAGE_TILE_BYTES;  // per epilogue warp: direct + transposed box
constexpr int SMEM_BYTES = STAGES * STAGE_BYTES + STAGING_BYTES + 1024 /*align*/ + 256 /*barriers*/;
constexpr int GROUP_M = 8;               // tile raster grouping for L2 reuse

struct Params {
  int M, N, K, batch;
  int tiles_m, tiles_n, tiles_per_batch, total_tiles;
  int symmetric;
  void* D; int ldd; long long d_bs; int d_dtype;
  const void* C; int ldc; long long c_bs; int c_dtype;
  float c_acc, c_in, c_eye;
  const float* scale; int scale_pow;
  int* err;
  long long timeout_ns;
  int* tile_counter;      // paired-CTA kernel: device word, 0 at launch; tiles are taken from it in order
  int static_order;       // 1: tiles round-robin over the pairs instead (comparison runs)
};

// ------------------------------------------------------------------ PTX helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ uint64_t global_timer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: false when the deadline passed or another role aborted.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          long long timeout_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if ((long long)(global_timer() - t0) > timeout_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
  *abort_flag = 1;
  return false;
}

__device__ __forceinline__ void tma_load_3d(uint32_t dst, const CUtensorMap* map, uint32_t bar, int x, int y,
                                            int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(x), "r"(y), "r"(z)
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
        "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
        "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
        "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, sm_100 version field.  Layout 2 is the
// 128-byte swizzle with 16-byte granules (every K-major operand, and 16-bit
// MN-major ones); layout 1 is the 128-byte swizzle with 32-byte granules,
// which 32-bit (TF32) MN-major operands take.
constexpr uint32_t kLayoutSw128 = 2;
constexpr uint32_t kLayoutSw128Atom32 = 1;
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo,
                                              uint32_t layout = kLayoutSw128) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;  // descriptor version for tcgen05
  d |= (uint64_t)layout << 61;
  return d;
}

// Instruction descriptor for kind::f16: fp32 D, A/B of one 16-bit type,
// A K-major, B K-major or MN-major, M x N (default 128 x 256).
__host__ __device__ constexpr uint32_t make_idesc(int in_fmt /*0 f16, 1 bf16*/, int b_mn, int m = BM, int n = BN) {
  return (1u << 4) | ((uint32_t)in_fmt << 7) | ((uint32_t)in_fmt << 10) | ((uint32_t)b_mn << 16) |
         ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// ------------------------------------------------------------------ tile order
struct Tile { int b, tm, tn; };

__device__ __forceinline__ Tile decode_tile(const Params& p, int t) {
  Tile r;
  r.b = t / p.tiles_per_batch;
  int q = t - r.b * p.tiles_per_batch;
  if (p.symmetric) {
    // upper-triangle tiles in 128-block units: row tm keeps tn >= tm / 2
    int tm = 0;
    for (; tm < p.tiles_m; ++tm) {
      const int cnt = p.tiles_n - tm / 2;
      if (q < cnt) break;
      q -= cnt;
    }
    r.tm = tm;
    r.tn = tm / 2 + q;
  } else {
    const int per_group = GROUP_M * p.tiles_n;
    const int g = q / per_group;
    const int first = g * GROUP_M;
    const int gsz = min(p.tiles_m - first, GROUP_M);
    const int w = q - g * per_group;
    r.tm = first + w % gsz;
    r.tn = w / gsz;
  }
  return r;
}

// ------------------------------------------------------------------ epilogue
__device__ __forceinline__ void cvt_row32(const uint4 (&q)[4], int dt, float* v) {
  if (dt == kBF16) {
    const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(q);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __bfloat162float(e[i]);
  } else {
    const __half* e = reinterpret_cast<const __half*>(q);
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __half2float(e[i]);
  }
}

__device__ __forceinline__ uint16_t to_bits(float v, int dt) {
  if (dt == kBF16) return __bfloat16_as_ushort(__float2bfloat16_rn(v));
  return __half_as_ushort(__float2half_rn(v));
}

// ------------------------------------------------------------------ epilogue stores via TMA
// A warp writes one 32 x 32 output box into shared memory in the layout of a
// 64-byte-swizzled tensor map (row r, 16-byte chunk k at r*64 + ((k ^ (r>>1 & 3)) << 4),
// conflict-free for both row-wise and column-wise writes), and one lane hands it to
// the TMA unit with a bulk tensor store, which also clips rows and columns past
// the matrix edge.
__device__ __forceinline__ uint32_t sw64(int row, int chunk16) {
  return (uint32_t)(row * 64 + ((chunk16 ^ ((row >> 1) & 3)) << 4));
}
// T = S^T for a warp's 32 x 32 box of 16-bit values, both in the sw64 layout.
// Round g moves column block g of the four 8 x 8 row blocks of S: ldmatrix
// .trans reads them (lane l addresses row l of S) transposed into the
// fragment layout, and stmatrix writes each as row block g of T (lane l
// addresses row 8 g + l % 8 of block l / 8): 8 instructions per lane.
__device__ __forceinline__ void transpose_box16(const uint8_t* S, uint8_t* T, int lane) {
  const uint32_t s0 = smem_u32(S), t0 = smem_u32(T);
#pragma unroll
  for (int g = 0; g < 4; ++g) {
    uint32_t r0, r1, r2, r3;
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(s0 + sw64(lane, g))
                 : "memory");
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(
                     t0 + sw64(g * 8 + (lane & 7), lane >> 3)),
                 "r"(r0), "r"(r1), "r"(r2), "r"(r3)
                 : "memory");
  }
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* map, uint32_t src, int x, int y, int z) {
  asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%2, %3, %4}], [%1];" ::"l"(
                   reinterpret_cast<uint64_t>(map)),
               "r"(src), "r"(x), "r"(y), "r"(z)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all0() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void pack_row32(const float* v, int dt, uint4 (&q)[4]) {
  if (dt == kBF16) {
    __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(q);
#pragma unroll
    for (int i = 0; i < 32; ++i) e[i] = __float2bfloat16_rn(v[i]);
  } else {
    __half* e = reinterpret_cast<__half*>(q);
#pragma unroll
    for (int i = 0; i < 32; ++i) e[i] = __float2half_rn(v[i]);
  }
}

// v = f (c_acc acc + c_in C) + c_eye I for one 32-column chunk of row gi;
// the C term is added by the caller.  Multiplications by 1 and a zero
// identity term are skipped (warp-uniform tests): the default chains have
// f = 1, most products c_acc = 1, and only the Gram form's Q has c_eye != 0,
// whose diagonal lies in the boxes with gj0 == gi_base only.
__device__ __forceinline__ void scale_acc32(const Params& p, const uint32_t (&acc)[32], float* v) {
  if (p.c_acc != 1.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = p.c_acc * __uint_as_float(acc[j]);
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(acc[j]);
  }
}
__device__ __forceinline__ void finish32(const Params& p, float f, int gi_base, int gj0, int lane, float* v) {
  if (f != 1.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= f;
  }
  if (p.c_eye != 0.f && gj0 == gi_base) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == lane) v[j] += p.c_eye;
  }
}

// One 32 x 32 chunk of the output: this warp's 32 tile rows (one per lane,
// TMEM lane quarter q) times columns [gj0, gj0 + 32).  `creg` holds the C row
// segment when `c_ready` (loaded before the TMEM read to hide its latency).
// Symmetric products: off-diagonal 128-blocks are stored directly and
// transposed; inside a diagonal 128-block, boxes above the diagonal are stored
// both ways, boxes below are skipped (their transposes cover them) and the box
// on the diagonal is made exactly symmetric in shared memory first.
// S and T are this warp's two staging boxes (1024-byte aligned).
template <bool SYM>
__device__ __forceinline__ void epilogue_chunk(const Params& p, const CUtensorMap* tmap_d, const Tile& t, int q,
                                               int lane, int chunk, const uint32_t (&acc)[32],
                                               const uint4 (&creg)[4], bool c_ready, float f, uint8_t* S,
                                               uint8_t* T) {
  const int gi_base = t.tm * BM + q * 32;
  const int gi = gi_base + lane;
  const int gj0 = t.tn * BN + chunk * 32;
  bool mirror = false, diag_box = false;
  if (SYM) {
    const int bj = t.tn * 2 + (chunk >> 2);  // 128-column block of this chunk
    if (bj < t.tm) return;                   // lower block: stored as the transpose of its mirror
    if (bj > t.tm) {
      mirror = true;
    } else {                                 // diagonal 128-block
      if (gj0 < gi_base) return;             // box below the diagonal
      diag_box = gj0 == gi_base;
      mirror = !diag_box;
    }
  }
  if (gj0 >= p.N || gi_base >= p.M) return;  // warp-uniform
  float v[32];
  scale_acc32(p, acc, v);
  if (p.C != nullptr && gi < p.M) {
    if (c_ready) {
      float c[32];
      cvt_row32(creg, p.c_dtype, c);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += p.c_in * c[j];
    } else {
      const char* cb = reinterpret_cast<const char*>(p.C) + (long long)t.b * p.c_bs * 2;
      const long long off = (long long)gi * p.ldc + gj0;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (gj0 + j < p.N) v[j] += p.c_in * load_any(cb, off + j, p.c_dtype);
    }
  }
  finish32(p, f, gi_base, gj0, lane, v);

  // the staging boxes are free once the previous chunk's stores have read them
  if (lane == 0) bulk_wait_read0();
  __syncwarp();
  uint4 dq[4];
  pack_row32(v, p.d_dtype, dq);
#pragma unroll
  for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(S + sw64(lane, k)) = dq[k];
  if (SYM && (mirror || diag_box)) {
    // transposed box T = S^T
    __syncwarp();
    transpose_box16(S, T, lane);
    if (diag_box) {
      __syncwarp();
      // below the diagonal take the transposed value, so the box is exactly symmetric
      uint4 tq[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) tq[k] = *reinterpret_cast<const uint4*>(T + sw64(lane, k));
      const uint16_t* te = reinterpret_cast<const uint16_t*>(tq);
      uint16_t* de = reinterpret_cast<uint16_t*>(dq);
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (j < lane) de[j] = te[j];
#pragma unroll
      for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(S + sw64(lane, k)) = dq[k];
    }
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(tmap_d, smem_u32(S), gj0, gi_base, t.b);
    if (SYM && mirror) tma_store_3d(tmap_d, smem_u32(T), gi_base, gj0, t.b);
    bulk_commit();
  }
}

// ------------------------------------------------------------------ fused Muon update
// The last product of a Muon step's chain can write W <- decay W - step O
// itself.  A warp's 32 x 32 box of O is staged in its shared-memory box in W's
// own orientation (row r of the staging box = row r of the W block the box
// covers), and the lanes then update W in four passes of 8 rows x 64 bytes:
// lane L takes row 8 it + L / 4 and its 16-byte segment L % 4, so every access
// instruction of the warp covers 8 contiguous 64-byte row pieces.

// Where the box of (t, q, chunk) lies in W: its first element, the row pitch,
// and how many rows and columns of it exist.
struct WBox {
  char* base;
  long long ld;
  int rows, cols, wdt, es;
};
template <typename Slots>
__device__ __forceinline__ WBox w_box(const Params& p, const Slots& u, const Tile& t, int q, int chunk) {
  const int gi_base = t.tm * BM + q * 32;
  const int gj0 = t.tn * BN + chunk * 32;
  const unsigned kind = u.kind[t.b];
  WBox w;
  w.wdt = (int)(kind >> 1);
  w.es = w.wdt == kFP32 ? 4 : 2;
  char* W = reinterpret_cast<char*>(u.w[t.b]);
  if (!(kind & 1u)) {  // W is M x N like O
    w.ld = p.N;
    w.base = W + ((long long)gi_base * p.N + gj0) * w.es;
    w.rows = min(32, p.M - gi_base);
    w.cols = min(32, p.N - gj0);
  } else {             // W is N x M: the box's rows are O's columns
    w.ld = p.M;
    w.base = W + ((long long)gj0 * p.M + gi_base) * w.es;
    w.rows = min(32, p.N - gj0);
    w.cols = min(32, p.M - gi_base);
  }
  return w;
}

// The 16-bit W segments a lane updates (one per pass), loaded ahead of the
// accumulator read so that their latency overlaps it.
struct WPrefetch {
  uint4 q[4];
  bool ok;
};
template <typename Slots>
__device__ __forceinline__ WPrefetch prefetch_w(const Params& p, const Slots& u, const Tile& t, int q, int lane,
                                                int chunk) {
  WPrefetch pf;
  pf.ok = false;
  const int gi_base = t.tm * BM + q * 32;
  const int gj0 = t.tn * BN + chunk * 32;
  if (gj0 + 32 > p.N || gi_base + 32 > p.M) return pf;  // ragged boxes load W as they go
  const WBox w = w_box(p, u, t, q, chunk);
  if (w.wdt == kFP32 || (w.ld * 2) % 16 != 0) return pf;
#pragma unroll
  for (int it = 0; it < 4; ++it)
    pf.q[it] = *reinterpret_cast<const uint4*>(w.base + ((long long)(it * 8 + (lane >> 2)) * w.ld + (lane & 3) * 8) * 2);
  pf.ok = true;
  return pf;
}

// W[0..valid) <- weight_update(W, o) for 8 consecutive elements at `w`
// (16-byte aligned when `vec`, then `pre` may hold them already for 16-bit W).
__device__ __forceinline__ void update8(char* w, int wdt, const float* o, int valid, bool vec, float decay, float step,
                                        bool have_pre, uint4 pre) {
  if (vec && wdt == kFP32) {
    float4* q = reinterpret_cast<float4*>(w);
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      float4 x = q[k];
      x.x = weight_update(x.x, o[4 * k], decay, step);
      x.y = weight_update(x.y, o[4 * k + 1], decay, step);
      x.z = weight_update(x.z, o[4 * k + 2], decay, step);
      x.w = weight_update(x.w, o[4 * k + 3], decay, step);
      q[k] = x;
    }
  } else if (vec) {
    uint4 x = have_pre ? pre : *reinterpret_cast<const uint4*>(w);
    if (wdt == kBF16) {
      __nv_bfloat16* e = reinterpret_cast<__nv_bfloat16*>(&x);
#pragma unroll
      for (int k = 0; k < 8; ++k) e[k] = __float2bfloat16_rn(weight_update(__bfloat162float(e[k]), o[k], decay, step));
    } else {
      __half* e = reinterpret_cast<__half*>(&x);
#pragma unroll
      for (int k = 0; k < 8; ++k) e[k] = __float2half_rn(weight_update(__half2float(e[k]), o[k], decay, step));
    }
    *reinterpret_cast<uint4*>(w) = x;
  } else {
#pragma unroll
    for (int k = 0; k < 8; ++k)
      if (k < valid) store_any(w, k, wdt, weight_update(load_any(w, k, wdt), o[k], decay, step));
  }
}

// The fused-update counterpart of epilogue_chunk (non-symmetric products):
// O = f (c_acc acc + c_in C) for this warp's 32 rows x 32 columns, rounded to
// the chain's type as the stored X would be, then W <- decay W - step O for
// matrix t.b through the staging box S (see above).  Non-finite O raises
// MUON_STATUS_NONFINITE in the matrix's status word.
template <typename Slots>
__device__ __forceinline__ void update_chunk(const Params& p, const Slots& u, const Tile& t, int q, int lane,
                                             int chunk, const uint32_t (&acc)[32], const uint4 (&creg)[4],
                                             bool c_ready, float f, uint8_t* S, const WPrefetch& pf) {
  const int gi_base = t.tm * BM + q * 32;
  const int gi = gi_base + lane;
  const int gj0 = t.tn * BN + chunk * 32;
  if (gj0 >= p.N || gi_base >= p.M) return;  // warp-uniform
  float v[32];
  scale_acc32(p, acc, v);
  if (p.C != nullptr && gi < p.M) {
    if (c_ready) {
      float c[32];
      cvt_row32(creg, p.c_dtype, c);
#pragma unroll
      for (int j = 0; j < 32; ++j) v[j] += p.c_in * c[j];
    } else {
      const char* cb = reinterpret_cast<const char*>(p.C) + (long long)t.b * p.c_bs * 2;
      const long long off = (long long)gi * p.ldc + gj0;
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (gj0 + j < p.N) v[j] += p.c_in * load_any(cb, off + j, p.c_dtype);
    }
  }
  finish32(p, f, gi_base, gj0, lane, v);
  uint4 oq[4];
  pack_row32(v, p.d_dtype, oq);   // O in the chain's storage type
  cvt_row32(oq, p.d_dtype, v);
  int bad = 0;
  if (gi < p.M) {
#pragma unroll
    for (int j = 0; j < 32; ++j) bad |= (gj0 + j < p.N) && !isfinite(v[j]);
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad && lane == 0 && u.status != nullptr) atomicOr(u.status + u.status_idx[t.b], kStatusNonFinite);

  const bool trans = (u.kind[t.b] & 1u) != 0;
  __syncwarp();  // every lane is done with S's previous contents
  if (!trans) {
#pragma unroll
    for (int k = 0; k < 4; ++k) *reinterpret_cast<uint4*>(S + sw64(lane, k)) = oq[k];
  } else {
    const uint16_t* ob = reinterpret_cast<const uint16_t*>(oq);
#pragma unroll
    for (int j = 0; j < 32; ++j)
      *reinterpret_cast<uint16_t*>(S + sw64(j, lane >> 3) + (lane & 7) * 2) = ob[j];
  }
  __syncwarp();
  const WBox w = w_box(p, u, t, q, chunk);
  const bool rows_vec = (w.ld * w.es) % 16 == 0;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int r = it * 8 + (lane >> 2);
    const int c0 = (lane & 3) * 8;
    if (r >= w.rows || c0 >= w.cols) continue;
    const int valid = min(8, w.cols - c0);
    // this lane's 8 values of O: row r of the staging box, 16-byte chunk lane % 4
    const uint4 oseg = *reinterpret_cast<const uint4*>(S + sw64(r, lane & 3));
    float o[8];
    if (p.d_dtype == kBF16) {
      const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&oseg);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = __bfloat162float(e[k]);
    } else {
      const __half* e = reinterpret_cast<const __half*>(&oseg);
#pragma unroll
      for (int k = 0; k < 8; ++k) o[k] = __half2float(e[k]);
    }
    update8(w.base + ((long long)r * w.ld + c0) * w.es, w.wdt, o, valid, valid == 8 && rows_vec, u.decay, u.step,
            pf.ok, pf.q[it]);
  }
}

// ------------------------------------------------------------------ clusters of two CTAs
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t mapa(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrive (once MMAs issued so far retire) on the barrier at this offset in
// every CTA of `mask`.
__device__ __forceinline__ void commit_pair(uint32_t bar, uint16_t mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(bar),
      "h"(mask)
      : "memory");
}
__device__ __forceinline__ void remote_arrive(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// Arrive on a barrier of a CTA of the cluster with release at CTA scope only:
// for signals that hand over no memory contents, such as "this TMEM buffer
// has been read out" (after tcgen05.wait::ld and a tcgen05 fence), where the
// cluster-scope release of remote_arrive would add a memory barrier to every
// arrival.
__device__ __forceinline__ void remote_arrive_cta(uint32_t bar_cluster) {
  asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(bar_cluster) : "memory");
}
// Store to the same shared-memory object in another CTA of the cluster (address from mapa).
__device__ __forceinline__ void st_cluster_s32(uint32_t addr_cluster, int v) {
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(addr_cluster), "r"(v) : "memory");
}
// Wait on a barrier of this CTA whose arrivals (and the data they publish)
// come from other CTAs of the cluster: acquire at cluster scope.
__device__ __forceinline__ bool mbar_try_wait_cluster(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded as mbar_wait: false when the deadline passed or another role aborted.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                                  long long timeout_ns) {
  if (mbar_try_wait_cluster(bar, parity)) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (mbar_try_wait_cluster(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*abort_flag) return false;
      if ((long long)(global_timer() - t0) > timeout_ns) {
        *abort_flag = 1;
        return false;
      }
    }
  }
  *abort_flag = 1;
  return false;
}

// Tile order of the paired-CTA kernels: 256 x 256 tiles (upper triangle only
// for symmetric products), grouped rasterisation otherwise.
struct PairTile { int b, TM, TN; };

__device__ __forceinline__ PairTile decode_pair(const Params& p, int t) {
  PairTile r;
  r.b = t / p.tiles_per_batch;
  int q = t - r.b * p.tiles_per_batch;
  if (p.symmetric) {
    int tm = 0;
    for (; tm < p.tiles_m; ++tm) {
      const int cnt = p.tiles_n - tm;
      if (q < cnt) break;
      q -= cnt;
    }
    r.TM = tm;
    r.TN = tm + q;
  } else {
    const int per_group = GROUP_M * p.tiles_n;
    const int g = q / per_group;
    const int first = g * GROUP_M;
    const int gsz = min(p.tiles_m - first, GROUP_M);
    const int w = q - g * per_group;
    r.TM = first + w % gsz;
    r.TN = w / gsz;
  }
  return r;
}

// ------------------------------------------------------------------ whole chains in one launch (gemm_chain.cu)
// One product of a chain launch: its operand and output maps, shape, tile
// range in the launch's tile space, epilogue and the product it depends on.
struct alignas(64) ChainProduct {
  CUtensorMap ma, mb, md;
  int M, N, K, batch;
  int tiles_m, tiles_n, tiles_per_batch, first_tile;
  int symmetric, b_mn, dep;
  void* D; int ldd; long long d_bs; int d_dtype;
  const void* C; int ldc; long long c_bs; int c_dtype;
  float c_acc, c_in, c_eye;
  const float* scale; int scale_pow;
};
struct ChainParams {
  static constexpr int kMaxProducts = 24;
  int n_products, batch, total_tiles, static_order;
  int* tile_counter;      // device word, 0 at launch
  int* done;              // [n_products][batch] arrival counters, 0 at launch
  int* err;
  long long timeout_ns;
  ChainProduct prod[kMaxProducts];
};

// Tiles from the counter (default) or round-robin (MUON_TILE_ORDER=static):
// the same tiles and arithmetic either way, only the hand-out order differs.
bool static_tile_order();

// ------------------------------------------------------------------ host side (gemm_tc.cu)
// 3-D tiled tensor map over a batch of row-major matrices.  Shared-memory
// layouts: 128-byte swizzle (16-byte granules), 64-byte swizzle, or 128-byte
// swizzle with 32-byte granules (TF32 MN-major operands).
enum TmaSwizzle { kTmaSw128, kTmaSw64, kTmaSw128Atom32 };
bool encode_map(CUtensorMap* map, int dtype, const void* base, long long inner, long long outer, long long batch,
                long long ld_elems, long long bs_elems, int box_inner, int box_outer, TmaSwizzle swizzle = kTmaSw128);
// Output map of a product: 32 x 32 boxes, 64-byte swizzle (the epilogue's staging layout).
bool encode_out_map(CUtensorMap* map, const GemmDesc& g);
// 2-CTA (cta_group::2) variant for 256-row tiles (gemm_tc2.cu).
int gemm_tc_pair(const GemmDesc& g, Params p, cudaStream_t s);

}  // namespace tc
}  // namespace muon
