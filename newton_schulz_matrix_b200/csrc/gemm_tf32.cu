// fp32 products on the tensor cores: 3xTF32 on paired CTAs (tcgen05 kind::tf32).
//
// TF32 keeps 10 explicit mantissa bits, too few for fp32 chains on their own.
// Each fp32 operand value is split as a = hi + lo, hi = a rounded to TF32 and
// lo = a - hi (exact in fp32), and a product accumulates lo*hi + hi*lo + hi*hi;
// the dropped lo*lo term is below 2^-22 of |a b| and the TF32 reading of lo
// below 2^-21.
//
// Accumulation: the tensor core's own fp32 accumulation rounds with a bias
// (its error grows linearly with K: measured ~1.8e-6 relative at K = 256 and
// ~9e-6 at K = 1024 when one accumulator takes the whole sum), which the Gram
// recurrences amplify past the fp32 bar.  So every 32-deep k-block is
// accumulated afresh in one of three TMEM buffers, and the epilogue warps fold
// it into an fp32 register sum (round to nearest): the biased part then spans
// only the 12 MMAs of one k-block, whatever K is.
//
// Layout: persistent CTA pairs on 256 x 128 output tiles (each CTA 128 rows;
// the leader issues M=256, N=128, K=8 MMAs reading both CTAs' shared memory).
//   - the split is done before the product, by an HBM-bound pass that writes
//     hi and lo as two fp32 planes of each operand (same strides as the
//     operand; X X^T and A^2 read one pair for both operands).  The product
//     kernel loads the four planes by TMA, each CTA's loads completing on the
//     leader's barrier: the plain TMA -> MMA pipeline of the 16-bit kernels.
//     Splitting in the kernel instead measured slower: in shared memory, each
//     split needs a proxy fence before the tensor core may read it; into
//     tensor memory (A only), the A tile becomes a third stream of loads and
//     the converter hand-off adds latency;
//   - the fold's per-k-block "buffer read out" arrivals use a CTA-scope
//     release (they hand over no data): with a cluster-scope release each of
//     them carried a memory barrier, and those paced the kernel;
//   - MN-major B tiles use the 128-byte swizzle with 32-byte granules (the
//     only shared-memory layout the tensor core takes for 32-bit MN-major
//     operands), in the tensor map and in the descriptor alike;
//   - eight epilogue warps per CTA (two per TMEM lane quarter, 64 columns
//     each) fold the k-blocks and store the tile through 32-row x 16-column
//     fp32 boxes;
//   - symmetric products store the boxes on and above the diagonal only, and
//     a mirror kernel then copies the strict upper triangle onto the lower one,
//     so the result is exactly symmetric.
// Every wait is bounded, as in the 16-bit kernels.
#include <algorithm>
#include <atomic>
#include <cmath>

#include "tc_common.cuh"

namespace muon {
namespace tc {
namespace tf32k {

constexpr int BK32 = 32;                       // 32 x 4 B = one 128-byte swizzle row
constexpr int UMMA_K32 = 8;                    // K of one kind::tf32 MMA
constexpr int TILE_N = 128;                    // pair tile: 256 rows x 128 columns
constexpr int STAGES3 = 4;
constexpr int A_OP = 128 * BK32 * 4;           // this CTA's 128 rows of one A plane: 16 KB
constexpr int B_OP = (TILE_N / 2) * BK32 * 4;  // this CTA's 64 columns of one B plane: 8 KB
constexpr int RAW_BYTES = A_OP + B_OP;         // the hi planes of A and B; the lo planes follow
constexpr int STAGE_BYTES3 = 2 * RAW_BYTES;
constexpr int NUM_PBUF = 4;                    // k-block accumulators in TMEM
constexpr int TMEM_COLS3 = NUM_PBUF * TILE_N;
constexpr int NUM_THREADS3 = 64 + 32 * NUM_EPI_WARPS;
constexpr int NUM_BARS3 = 2 * STAGES3 + 2 * NUM_PBUF + 1;
constexpr int SMEM_BYTES3 = STAGES3 * STAGE_BYTES3 + STAGING_BYTES + 1024 + 256;
static_assert(SMEM_BYTES3 <= 232448, "exceeds the per-block shared-memory limit");
static_assert(NUM_BARS3 * 8 + 8 <= 256, "barrier area");
static_assert(TMEM_COLS3 == 512, "TMEM allocation is a power of two");

// fp32 D, TF32 A and B, A K-major, B K- or MN-major, M = 256, N = 128.
__host__ __device__ constexpr uint32_t make_idesc_tf32(int b_mn) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)b_mn << 16) | ((uint32_t)(TILE_N >> 3) << 17) |
         ((uint32_t)(256 >> 4) << 24);
}

__device__ __forceinline__ void mma_tf32_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 64 consecutive 32-bit TMEM columns of this warp's lane quarter, one wait.
__device__ __forceinline__ void tmem_ld64(uint32_t taddr, uint32_t (&r)[64]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x64.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32,%33,%34,%35,%36,%37,%38,%39,%40,%41,%42,%43,%44,%45,%46,%47,%48,%49,%50,%51,%52,%53,%54,%55,%56,%57,%58,%59,%60,%61,%62,%63}, [%64];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31]), "=r"(r[32]), "=r"(r[33]), "=r"(r[34]), "=r"(r[35]), "=r"(r[36]), "=r"(r[37]), "=r"(r[38]), "=r"(r[39]), "=r"(r[40]), "=r"(r[41]), "=r"(r[42]), "=r"(r[43]), "=r"(r[44]), "=r"(r[45]), "=r"(r[46]), "=r"(r[47]), "=r"(r[48]), "=r"(r[49]), "=r"(r[50]), "=r"(r[51]), "=r"(r[52]), "=r"(r[53]), "=r"(r[54]), "=r"(r[55]), "=r"(r[56]), "=r"(r[57]), "=r"(r[58]), "=r"(r[59]), "=r"(r[60]), "=r"(r[61]), "=r"(r[62]), "=r"(r[63])
      : "r"(taddr));
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// TMA load into this CTA's shared memory whose completion is reported on a
// barrier of the pair (the leader's full barrier, a cluster address).
__device__ __forceinline__ void tma_load_3d_to_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                    int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}

// Wait on a local barrier that other CTAs of the cluster arrive on.
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

// a rounded to TF32 (nearest, ties away from zero), low 13 bits zero.
__device__ __forceinline__ float tf32_hi(float a) {
  uint32_t r;
  asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(a));
  return __uint_as_float(r);
}

// Tile order: 256-row x 128-column tiles, grouped rasterisation; symmetric
// products keep the tiles that reach the diagonal or lie above it (TN >= 2 TM).
struct Tile32 { int b, TM, TN; };

__device__ __forceinline__ Tile32 decode_t32(const Params& p, int t) {
  Tile32 r;
  r.b = t / p.tiles_per_batch;
  int q = t - r.b * p.tiles_per_batch;
  if (p.symmetric) {
    int tm = 0;
    for (; tm < p.tiles_m; ++tm) {
      const int cnt = p.tiles_n - 2 * tm;
      if (q < cnt) break;
      q -= cnt;
    }
    r.TM = tm;
    r.TN = 2 * tm + q;
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

// One 32 x 32 fp32 output chunk from the folded sums s[0..31] (row gi_base +
// lane, columns [gj0, gj0 + 32)): epilogue out = f (c_acc acc + c_in C) + c_eye I,
// written as two 32 x 16 boxes (S: columns 0-15, T: 16-31), 64-byte rows in
// the 64-byte-swizzled layout of the output map.
__device__ __forceinline__ void store_chunk_f32(const Params& p, const CUtensorMap* tmap_d, int b, int gi_base,
                                                int gj0, int lane, const float* s, float f, uint8_t* S, uint8_t* T) {
  const int gi = gi_base + lane;
  // multiplications by 1 and a zero identity term are skipped (warp-uniform
  // tests); the identity's diagonal lies in the boxes with gj0 == gi_base only
  float v[32];
  if (p.c_acc != 1.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = p.c_acc * s[j];
  } else {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = s[j];
  }
  if (p.C != nullptr && gi < p.M) {
    const float* crow = reinterpret_cast<const float*>(p.C) + (long long)b * p.c_bs + (long long)gi * p.ldc + gj0;
    if (gj0 + 32 <= p.N) {
      const float4* c4 = reinterpret_cast<const float4*>(crow);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 c = c4[i];
        v[4 * i + 0] += p.c_in * c.x;
        v[4 * i + 1] += p.c_in * c.y;
        v[4 * i + 2] += p.c_in * c.z;
        v[4 * i + 3] += p.c_in * c.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < 32; ++j)
        if (gj0 + j < p.N) v[j] += p.c_in * crow[j];
    }
  }
  if (f != 1.f) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] *= f;
  }
  if (p.c_eye != 0.f && gj0 == gi_base) {
#pragma unroll
    for (int j = 0; j < 32; ++j)
      if (j == lane) v[j] += p.c_eye;
  }
  if (lane == 0) bulk_wait_read0();  // the boxes are free once earlier stores have read them
  __syncwarp();
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    *reinterpret_cast<float4*>(S + sw64(lane, k)) = make_float4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]);
    *reinterpret_cast<float4*>(T + sw64(lane, k)) =
        make_float4(v[16 + 4 * k], v[16 + 4 * k + 1], v[16 + 4 * k + 2], v[16 + 4 * k + 3]);
  }
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
    tma_store_3d(tmap_d, smem_u32(S), gj0, gi_base, b);
    if (gj0 + 16 < p.N) tma_store_3d(tmap_d, smem_u32(T), gj0 + 16, gi_base, b);
    bulk_commit();
  }
}

template <bool B_MN, bool SYM>
__global__ void __launch_bounds__(NUM_THREADS3, 1)
gemm_tf32x3_kernel(const __grid_constant__ CUtensorMap tmap_ah, const __grid_constant__ CUtensorMap tmap_al,
                   const __grid_constant__ CUtensorMap tmap_bh, const __grid_constant__ CUtensorMap tmap_bl,
                   const __grid_constant__ CUtensorMap tmap_d, const __grid_constant__ Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES3 * STAGE_BYTES3;  // per epilogue warp: two 2 KB boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(staging + STAGING_BYTES);
  uint64_t* full_bar = bars;                                   // [STAGES3] both CTAs' loads landed (leader)
  uint64_t* empty_bar = bars + STAGES3;                        // [STAGES3] MMAs done with the stage (both CTAs)
  uint64_t* pfull_bar = bars + 2 * STAGES3;                    // [NUM_PBUF] k-block sum ready (both CTAs)
  uint64_t* pempty_bar = bars + 2 * STAGES3 + NUM_PBUF;        // [NUM_PBUF] k-block sum folded (leader)
  uint64_t* drain_bar = bars + 2 * STAGES3 + 2 * NUM_PBUF;     // [1]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + NUM_BARS3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader, 1 = peer
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES3; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < NUM_PBUF; ++a) {
      mbar_init(smem_u32(&pfull_bar[a]), 1);
      mbar_init(smem_u32(&pempty_bar[a]), 2 * NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_ah)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_al)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_bh)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_bl)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmap_d)) : "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS3)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.K + BK32 - 1) / BK32;
  const uint32_t leader_full = mapa(smem_u32(full_bar), 0);
  const uint32_t leader_pempty = mapa(smem_u32(pempty_bar), 0);

  if (warp == 0) {
    // ---------------------------------------------------------------- producers (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = pair; t < p.total_tiles && ok; t += npairs) {
        const Tile32 tl = decode_t32(p, t);
        const int row0 = tl.TM * 256 + (int)rank * 128;            // this CTA's rows of A
        const int col0 = tl.TN * TILE_N + (int)rank * (TILE_N / 2);  // this CTA's columns of B
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          if (leader) mbar_expect_tx(smem_u32(&full_bar[stage]), 2 * STAGE_BYTES3);
          const uint32_t fb = leader_full + stage * 8;
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES3);  // A hi, B hi, A lo, B lo
          const uint32_t sb = sa + A_OP;
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t off = h * RAW_BYTES;
            tma_load_3d_to_pair(sa + off, h ? &tmap_al : &tmap_ah, fb, kb * BK32, row0, tl.b);
            const CUtensorMap* mb = h ? &tmap_bl : &tmap_bh;
            if (B_MN) {
#pragma unroll
              for (int q = 0; q < TILE_N / 64; ++q)
                tma_load_3d_to_pair(sb + off + q * (BK32 * 128), mb, fb, col0 + q * 32, kb * BK32, tl.b);
            } else {
              tma_load_3d_to_pair(sb + off, mb, fb, kb * BK32, col0, tl.b);
            }
          }
          if (++stage == STAGES3) { stage = 0; phase ^= 1u; }
        }
      }
      // no drain needed here: the leader's MMAs consume every issued stage,
      // and the final cluster barrier keeps this CTA resident until then
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = make_idesc_tf32(B_MN ? 1 : 0);
      int stage = 0;
      uint32_t phase = 0;
      uint32_t jb = 0;  // k-blocks issued so far (selects the TMEM buffer)
      bool ok = true;
      for (int t = pair; t < p.total_tiles && ok; t += npairs) {
        for (int kb = 0; kb < num_kb; ++kb, ++jb) {
          const uint32_t pb = jb % NUM_PBUF;
          const uint32_t pph = (jb / NUM_PBUF) & 1u;
          if (!mbar_wait_cluster(smem_u32(&pempty_bar[pb]), pph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + pb * TILE_N;
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES3);
          const uint32_t sb = sa + A_OP;
          const uint32_t la = sa + RAW_BYTES;
          const uint32_t lb = la + A_OP;
#pragma unroll
          for (int k = 0; k < BK32 / UMMA_K32; ++k) {
            const uint64_t a_hi = smem_desc(sa + k * (UMMA_K32 * 4), 16, 1024);
            const uint64_t a_lo = smem_desc(la + k * (UMMA_K32 * 4), 16, 1024);
            // MN-major B: 32-column x 4-row swizzle atoms (128-byte rows, 32-byte
            // granules); LBO steps 32 columns (one 32-row chunk), SBO 4 rows
            const uint64_t b_hi = B_MN ? smem_desc(sb + k * (UMMA_K32 * 128), BK32 * 128, 512, kLayoutSw128Atom32)
                                       : smem_desc(sb + k * (UMMA_K32 * 4), 16, 1024);
            const uint64_t b_lo = B_MN ? smem_desc(lb + k * (UMMA_K32 * 128), BK32 * 128, 512, kLayoutSw128Atom32)
                                       : smem_desc(lb + k * (UMMA_K32 * 4), 16, 1024);
            mma_tf32_pair(d_tmem, a_lo, b_hi, idesc, k != 0);  // a fresh sum per k-block
            mma_tf32_pair(d_tmem, a_hi, b_lo, idesc, 1);
            mma_tf32_pair(d_tmem, a_hi, b_hi, idesc, 1);
          }
          commit_pair(smem_u32(&empty_bar[stage]), 0x3);  // stage free in both CTAs
          commit_pair(smem_u32(&pfull_bar[pb]), 0x3);     // k-block sum ready in both CTAs
          if (++stage == STAGES3) { stage = 0; phase ^= 1u; }
        }
      }
      commit_pair(smem_u32(drain_bar), 0x1);
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, &never, p.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------------- fold + epilogue (both CTAs)
    const int q = warp & 3;             // TMEM lane quarter: rows q*32 .. q*32+31 of this CTA
    const int half = (warp - 2) >> 2;   // columns half*64 .. half*64+63 of the tile
    uint8_t* S = staging + (warp - 2) * 2 * STAGE_TILE_BYTES;
    uint8_t* T = S + STAGE_TILE_BYTES;
    uint32_t jb = 0;
    bool ok = true;
    for (int t = pair; t < p.total_tiles && ok; t += npairs) {
      const Tile32 tl = decode_t32(p, t);
      float acc[64];
#pragma unroll
      for (int j = 0; j < 64; ++j) acc[j] = 0.f;
      for (int kb = 0; kb < num_kb; ++kb, ++jb) {
        const uint32_t pb = jb % NUM_PBUF;
        const uint32_t pph = (jb / NUM_PBUF) & 1u;
        int w = 1;
        if (lane == 0) w = mbar_wait(smem_u32(&pfull_bar[pb]), pph, abort_flag, p.timeout_ns);
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) { ok = false; break; }
        tc_fence_after();
        const uint32_t taddr = tmem_base + pb * TILE_N + (uint32_t)(half * 64) + ((uint32_t)(q * 32) << 16);
        uint32_t r[64];
        tmem_ld64(taddr, r);
        // the buffer is free once read out: release it before folding, which
        // keeps the fold's adds off the MMA issuer's path
        tc_fence_before();
        __syncwarp();
        if (lane == 0) remote_arrive_cta(leader_pempty + pb * 8);  // no data handed over
#pragma unroll
        for (int j = 0; j < 64; ++j) acc[j] += __uint_as_float(r[j]);
      }
      if (!ok) break;
      const float f = matrix_scale(p.scale, p.scale_pow, tl.b);
      const int gi_base = tl.TM * 256 + (int)rank * 128 + q * 32;
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        const int gj0 = tl.TN * TILE_N + half * 64 + c * 32;
        if (gj0 >= p.N || gi_base >= p.M) continue;  // warp-uniform
        if (SYM && gj0 < gi_base) continue;          // below the diagonal: mirrored afterwards
        store_chunk_f32(p, &tmap_d, tl.b, gi_base, gj0, lane, acc + 32 * c, f, S, T);
      }
    }
    if (lane == 0) bulk_wait_all0();  // this warp's output stores have completed
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the leader's MMAs into this CTA's TMEM are drained
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS3) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag && p.err != nullptr) atomicOr(p.err, kStatusTimeout);
}

// D[i][j] = D[j][i] for i > j: the strict upper triangle of each n x n matrix
// copied onto the lower one through 32 x 32 shared-memory tiles.  Work item w
// is (matrix, lower-triangle tile (bi, bj), bi >= bj), t = bi (bi + 1) / 2 + bj.
__global__ void __launch_bounds__(256) mirror_upper_kernel(float* D, int n, int ld, long long bs, int batch,
                                                           int ntri) {
  __shared__ float tile[32][33];
  const int tx = threadIdx.x & 31, ty = threadIdx.x >> 5;
  const long long total = (long long)ntri * batch;
  for (long long w = blockIdx.x; w < total; w += gridDim.x) {
    const int b = (int)(w / ntri);
    const int t = (int)(w - (long long)b * ntri);
    int bi = (int)((sqrt(8.0 * t + 1.0) - 1.0) * 0.5);
    while ((bi + 1) * (bi + 2) / 2 <= t) ++bi;
    while (bi * (bi + 1) / 2 > t) --bi;
    const int bj = t - bi * (bi + 1) / 2;
    float* Db = D + (long long)b * bs;
    for (int r = ty; r < 32; r += 8) {  // source: rows of block bj, columns of block bi
      const int i = bj * 32 + r, j = bi * 32 + tx;
      if (i < n && j < n) tile[r][tx] = Db[(long long)i * ld + j];
    }
    __syncthreads();
    for (int r = ty; r < 32; r += 8) {  // destination: rows of block bi, columns of block bj
      const int i = bi * 32 + r, j = bj * 32 + tx;
      if (i < n && j < n && i > j) Db[(long long)i * ld + j] = tile[tx][r];
    }
    __syncthreads();
  }
}

// hi = src rounded to TF32, lo = src - hi (exact in fp32), over n4 float4s.
__global__ void __launch_bounds__(256) split_tf32_kernel(const float4* __restrict__ src, float4* __restrict__ hi,
                                                         float4* __restrict__ lo, long long n4) {
  for (long long i = blockIdx.x * 256LL + threadIdx.x; i < n4; i += (long long)gridDim.x * 256) {
    const float4 x = src[i];
    const float4 h = make_float4(tf32_hi(x.x), tf32_hi(x.y), tf32_hi(x.z), tf32_hi(x.w));
    hi[i] = h;
    lo[i] = make_float4(x.x - h.x, x.y - h.y, x.z - h.z, x.w - h.w);
  }
}

template <bool B_MN, bool SYM>
static int launch(const CUtensorMap (&m)[5], const Params& p, cudaStream_t s) {
  static std::atomic<int> max_pairs_of[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return (int)cudaErrorInvalidDevice;
  auto kern = gemm_tf32x3_kernel<B_MN, SYM>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(NUM_THREADS3);
  cfg.dynamicSmemBytes = SMEM_BYTES3;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_pairs = max_pairs_of[dev].load(std::memory_order_acquire);
  if (max_pairs <= 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES3);
    if (e != cudaSuccess) return (int)e;
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n <= 0) n = num_sms() / 2;
    max_pairs = n;
    max_pairs_of[dev].store(n, std::memory_order_release);
  }
  const int pairs = p.total_tiles < max_pairs ? p.total_tiles : max_pairs;
  cfg.gridDim = dim3(2 * pairs);
  return (int)cudaLaunchKernelEx(&cfg, kern, m[0], m[1], m[2], m[3], m[4], p);
}

}  // namespace tf32k
}  // namespace tc

double gemm_tf32x3_exec_flops(const GemmDesc& g) {
  using namespace tc::tf32k;
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return 0.0;
  const int tm = (g.M + 255) / 256, tn = (g.N + TILE_N - 1) / TILE_N;
  double tiles = 0.0;
  for (int r = 0; r < tm; ++r) tiles += g.symmetric ? tn - 2 * r : tn;
  const double k_pad = (double)((g.K + BK32 - 1) / BK32) * BK32;
  return 3.0 * 2.0 * tiles * 256.0 * TILE_N * k_pad * g.batch;  // hi*hi + hi*lo + lo*hi
}

int split_tf32(const float* src, float* hi, float* lo, long long elems, cudaStream_t s) {
  using namespace tc::tf32k;
  if (elems <= 0) return 0;
  if ((elems & 3) || (reinterpret_cast<uintptr_t>(src) & 15) || (reinterpret_cast<uintptr_t>(hi) & 15) ||
      (reinterpret_cast<uintptr_t>(lo) & 15))
    return (int)cudaErrorInvalidValue;
  const long long n4 = elems / 4;
  const long long want = (n4 + 255) / 256;
  const int blocks = (int)std::min<long long>(want, 8LL * num_sms());
  split_tf32_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<const float4*>(src), reinterpret_cast<float4*>(hi),
                                           reinterpret_cast<float4*>(lo), n4);
  return (int)cudaGetLastError();
}

int gemm_tf32x3(const GemmDesc& g, const Tf32Planes& pl, cudaStream_t s) {
  using namespace tc;
  using namespace tc::tf32k;
  if (g.M <= 0 || g.N <= 0 || g.batch <= 0) return 0;
  if (g.in_dtype != kFP32 || g.d_dtype != kFP32 || (g.C && g.c_dtype != kFP32)) return (int)cudaErrorInvalidValue;
  if (g.symmetric && g.M != g.N) return (int)cudaErrorInvalidValue;
  Params p{};
  p.M = g.M; p.N = g.N; p.K = g.K; p.batch = g.batch;
  p.tiles_m = (g.M + 255) / 256;
  p.tiles_n = (g.N + TILE_N - 1) / TILE_N;
  if (g.symmetric) {
    int cnt = 0;  // tiles reaching the diagonal or above it: TN >= 2 TM
    for (int tm = 0; tm < p.tiles_m; ++tm) cnt += p.tiles_n - 2 * tm;
    p.tiles_per_batch = cnt;
  } else {
    p.tiles_per_batch = p.tiles_m * p.tiles_n;
  }
  const long long total = (long long)p.tiles_per_batch * g.batch;
  if (total > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  p.total_tiles = (int)total;
  p.symmetric = g.symmetric;
  p.D = g.D; p.ldd = g.ldd; p.d_bs = g.d_bs; p.d_dtype = g.d_dtype;
  p.C = g.C; p.ldc = g.ldc; p.c_bs = g.c_bs; p.c_dtype = g.c_dtype;
  p.c_acc = g.c_acc; p.c_in = g.c_in; p.c_eye = g.c_eye;
  p.scale = g.scale; p.scale_pow = g.scale_pow;
  p.err = g.err;
  p.timeout_ns = wait_timeout_ns();

  // m: A hi, A lo, B hi, B lo (planes with the operands' strides), D
  CUtensorMap m[5];
  if (!pl.a_hi || !pl.a_lo || !pl.b_hi || !pl.b_lo) return (int)cudaErrorInvalidValue;
  const float* ap[2] = {pl.a_hi, pl.a_lo};
  const float* bp[2] = {pl.b_hi, pl.b_lo};
  const bool bmn = !g.b_kmajor;
  for (int h = 0; h < 2; ++h) {
    if (!encode_map(&m[h], kFP32, ap[h], g.K, g.M, g.batch, g.lda, g.a_bs, BK32, 128)) return (int)cudaErrorInvalidValue;
    if (bmn) {
      if (!encode_map(&m[2 + h], kFP32, bp[h], g.N, g.K, g.batch, g.ldb, g.b_bs, 32, BK32, kTmaSw128Atom32))
        return (int)cudaErrorInvalidValue;
    } else {
      if (!encode_map(&m[2 + h], kFP32, bp[h], g.K, g.N, g.batch, g.ldb, g.b_bs, BK32, TILE_N / 2))
        return (int)cudaErrorInvalidValue;
    }
  }
  if (!encode_map(&m[4], kFP32, g.D, g.N, g.M, g.batch, g.ldd, g.d_bs, 16, 32, kTmaSw64)) return (int)cudaErrorInvalidValue;
  int rc;
  if (g.symmetric) rc = bmn ? launch<true, true>(m, p, s) : launch<false, true>(m, p, s);
  else rc = bmn ? launch<true, false>(m, p, s) : launch<false, false>(m, p, s);
  if (rc != 0 || !g.symmetric) return rc;
  const int T = (g.M + 31) / 32;
  const int ntri = T * (T + 1) / 2;
  const long long work = (long long)ntri * g.batch;
  const int blocks = (int)(work < 8LL * num_sms() ? work : 8LL * num_sms());
  mirror_upper_kernel<<<blocks, 256, 0, s>>>(reinterpret_cast<float*>(g.D), g.M, g.ldd, g.d_bs, g.batch, ntri);
  return (int)cudaGetLastError();
}

}  // namespace muon
