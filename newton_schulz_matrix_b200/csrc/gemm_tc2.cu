// Paired-CTA (cta_group::2) variant of the tensor-core product kernel.
//
// Same computation and epilogue as the 1-CTA kernel (gemm_tc.cu), on 256 x 256
// output tiles owned by a cluster of two CTAs on two SMs:
//   - each CTA loads its own 128 rows of A and its own 128 of the tile's 256
//     columns of B (plain TMA loads in the cta_group::2 form, which report
//     completion to the leader CTA's barrier; no multicast), so a CTA moves
//     32 KB per 64-deep k-step for 128 x 256 x 64 MACs instead of 48 KB;
//   - the leader CTA issues one M=256, N=256, K=16 tcgen05.mma per k16 that
//     reads both CTAs' shared memory and writes both CTAs' TMEM (128 lanes
//     each), and releases each stage in both CTAs with a multicast commit;
//   - each CTA drains its own 128 x 256 accumulator (two TMEM buffers) with
//     the shared epilogue; both CTAs' epilogue warps hand the buffer back to
//     the leader's MMA issuer through a remote mbarrier arrive;
//   - a ragged last column tile with at most 128 valid columns (e.g. 1408 =
//     5.5 x 256) runs N = 128 MMAs, each CTA supplying 64 columns, which halves
//     its tensor work; its accumulator's upper 128 columns are never stored;
//   - tiles are handed out dynamically: the leader's producer takes the next
//     tile index from a device counter (one atomic per tile) and publishes it
//     in a small ring in both CTAs' shared memory, which the MMA issuer, the
//     peer's producer and every epilogue warp follow.  All pairs therefore
//     work on a window of consecutive tiles at any time, so tiles that share an
//     operand panel run together and read it from L2.  (A fixed round-robin
//     assignment lets pairs drift apart over a long launch, and with 341
//     matrices per launch that tripled the DRAM reads of the products.)
// Waits are bounded as in the 1-CTA kernel.
#include <stdio.h>
#include <stdlib.h>

#include <atomic>
#include <type_traits>

#include "tc_common.cuh"

namespace muon {
namespace tc {
namespace pairk {

constexpr int STAGES2 = 6;
constexpr int A_BYTES2 = BM * BK * 2;   // this CTA's 128 rows of A: 16 KB
constexpr int B_BYTES2 = 128 * BK * 2;  // this CTA's 128 columns of B: 16 KB
constexpr int STAGE_BYTES2 = A_BYTES2 + B_BYTES2;
constexpr int RING = 8;                 // tile indices in flight from the scheduler to the roles following it
// arrivals that free a ring slot: the MMA issuer, the peer's producer, and
// the epilogue warps of both CTAs
constexpr int RING_CONSUMERS = 1 + 1 + 2 * NUM_EPI_WARPS;
constexpr int BAR_BYTES2 = 512;         // barriers, the ring, the TMEM address, the abort flag
constexpr int SMEM_BYTES2 = STAGES2 * STAGE_BYTES2 + STAGING_BYTES + 1024 + BAR_BYTES2;
static_assert((2 * STAGES2 + 5 + 2 * RING) * 8 + RING * 4 + 8 <= BAR_BYTES2, "barrier area");

__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x,
                                                 int y, int z) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster), "r"(x), "r"(y), "r"(z)
      : "memory");
}
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Kernel parameter of launches without the fused update (keeps their
// parameter block small; UpdateSlots is ~7 KB).
struct NoUpdate {
  int unused;
};

template <bool B_MN, int IN_FMT, bool SYM, bool UPD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                 const __grid_constant__ CUtensorMap tmap_d, const __grid_constant__ Params p,
                 const __grid_constant__ std::conditional_t<UPD, UpdateSlots, NoUpdate> u) {
  static_assert(!(UPD && SYM), "the fused update follows a non-symmetric product");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES2 * STAGE_BYTES2;  // per epilogue warp: two 1024-aligned 2 KB boxes
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES2 * STAGE_BYTES2 + STAGING_BYTES);
  uint64_t* full_bar = bars;                      // [STAGES2]   (used in the leader)
  uint64_t* empty_bar = bars + STAGES2;           // [STAGES2]   (both CTAs)
  uint64_t* tfull_bar = bars + 2 * STAGES2;       // [2]         (both CTAs)
  uint64_t* tempty_bar = bars + 2 * STAGES2 + 2;  // [2]         (used in the leader)
  uint64_t* drain_bar = bars + 2 * STAGES2 + 4;   // [1]
  uint64_t* ring_full = bars + 2 * STAGES2 + 5;   // [RING]      (both CTAs)
  uint64_t* ring_empty = ring_full + RING;        // [RING]      (used in the leader)
  int* tile_ring = reinterpret_cast<int*>(ring_empty + RING);  // [RING] (both CTAs)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_ring + RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();  // 0 = leader, 1 = peer
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES2; ++s) {
      mbar_init(smem_u32(&full_bar[s]), 1);
      mbar_init(smem_u32(&empty_bar[s]), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(smem_u32(&tfull_bar[a]), 1);
      mbar_init(smem_u32(&tempty_bar[a]), 2 * NUM_EPI_WARPS);
    }
    mbar_init(smem_u32(drain_bar), 1);
    for (int r = 0; r < RING; ++r) {
      mbar_init(smem_u32(&ring_full[r]), 1);
      mbar_init(smem_u32(&ring_empty[r]), RING_CONSUMERS);
    }
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
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // both CTAs' barriers exist before any cross-CTA signal
  tc_fence_after();
  // Programmatic dependent launch: the set-up above may overlap the previous
  // kernel's last tiles; nothing below reads global memory before that kernel
  // has finished and its writes are visible.  The next kernel may be scheduled
  // now (its CTAs need a whole SM's shared memory, so they start on the SMs
  // this grid leaves).  Both are no-ops when the launch does not use it.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;
  const int num_kb = (p.K + BK - 1) / BK;
  const uint32_t leader_full = mapa(smem_u32(full_bar), 0);
  const uint32_t leader_tempty = mapa(smem_u32(tempty_bar), 0);
  const uint32_t leader_ring_empty = mapa(smem_u32(ring_empty), 0);
  // Tile index number i of this pair (in order; -1 once the launch's tiles are
  // exhausted).  The leader's producer takes it from the counter and
  // publishes it in both CTAs; every other role reads it from its own CTA's
  // ring and frees the slot in the leader.  false on timeout or abort.
  auto next_tile = [&](int i, int& t) -> bool {
    const int slot = i % RING;
    const uint32_t rph = (uint32_t)(i / RING) & 1u;
    if (leader) {
      // the ring and its barriers are this CTA's own: CTA-scope wait and arrive
      if (!mbar_wait(smem_u32(&ring_full[slot]), rph, abort_flag, p.timeout_ns)) return false;
      t = tile_ring[slot];
      mbar_arrive(smem_u32(&ring_empty[slot]));
    } else {
      // published from the leader CTA: cluster-scope acquire, remote release
      if (!mbar_wait_cluster(smem_u32(&ring_full[slot]), rph, abort_flag, p.timeout_ns)) return false;
      t = tile_ring[slot];
      remote_arrive(leader_ring_empty + slot * 8);
    }
    return true;
  };

  if (warp == 0) {
    // ---------------------------------------------------------------- producers (both CTAs)
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      // the scheduler (leader) takes tile indices one ahead: the next index is
      // requested while this tile's loads go out, so the atomic's latency stays
      // off the pipeline; MUON_TILE_ORDER=static hands them out round-robin
      const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);
      auto take = [&](int i) -> int {
        const int t = p.static_order ? pair + i * npairs : atomicAdd(p.tile_counter, 1);
        return t < p.total_tiles ? t : -1;
      };
      int held = leader ? take(0) : -1;
      for (int i = 0; ok; ++i) {
        int t;
        if (leader) {
          // scheduler: wait until every role has taken index i - RING from this slot
          const int slot = i % RING;
          if (!mbar_wait_cluster(smem_u32(&ring_empty[slot]), ((uint32_t)(i / RING) & 1u) ^ 1u, abort_flag,
                                 p.timeout_ns))
            break;
          t = held;
          if (t >= 0) held = take(i + 1);
          tile_ring[slot] = t;
          st_cluster_s32(mapa(smem_u32(&tile_ring[slot]), 1), t);
          mbar_arrive(smem_u32(&ring_full[slot]));            // this CTA's roles
          remote_arrive(mapa(smem_u32(&ring_full[slot]), 1));  // the peer's
        } else if (!next_tile(i, t)) {
          break;
        }
        if (t < 0) break;
        const PairTile tl = decode_pair(p, t);
        // a ragged last column tile with at most 128 valid columns runs N = 128
        // MMAs: each CTA then supplies 64 columns (the first 64 it loads)
        const bool narrow = p.N - tl.TN * 256 <= 128;
        const int row0 = tl.TM * 256 + (int)rank * 128;                   // this CTA's rows of A
        const int col0 = tl.TN * 256 + (int)rank * (narrow ? 64 : 128);  // this CTA's columns of B
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
          if (leader) mbar_expect_tx(smem_u32(&full_bar[stage]), 2 * STAGE_BYTES2);
          const uint32_t fb = leader_full + stage * 8;
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES2);
          const uint32_t sb = sa + A_BYTES2;
          tma_load_3d_pair(sa, &tmap_a, fb, kb * BK, row0, tl.b);
          if (B_MN) {
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_3d_pair(sb + q * (BK * 128), &tmap_b, fb, col0 + q * 64, kb * BK, tl.b);
          } else {
            tma_load_3d_pair(sb, &tmap_b, fb, kb * BK, col0, tl.b);
          }
          if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
        }
      }
      // no drain needed here: the leader's MMAs consume every issued stage,
      // and the final cluster barrier keeps this CTA resident until then
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && leader) {
      constexpr uint32_t idesc_full = make_idesc(IN_FMT, B_MN ? 1 : 0, 256, 256);
      constexpr uint32_t idesc_narrow = make_idesc(IN_FMT, B_MN ? 1 : 0, 256, 128);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int i = 0; ok; ++i, ++it) {
        int t;
        if (!next_tile(i, t) || t < 0) break;
        const uint32_t idesc = p.N - decode_pair(p, t).TN * 256 <= 128 ? idesc_narrow : idesc_full;
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), aph ^ 1u, abort_flag, p.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, p.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES2);
          const uint32_t sb = sa + A_BYTES2;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = smem_desc(sa + k * (UMMA_K * 2), 16, 1024);
            const uint64_t bd = B_MN ? smem_desc(sb + k * (UMMA_K * 128), BK * 128, 1024)
                                     : smem_desc(sb + k * (UMMA_K * 2), 16, 1024);
            mma_pair(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          commit_pair(smem_u32(&empty_bar[stage]), 0x3);  // stage free in both CTAs
          if (++stage == STAGES2) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        commit_pair(smem_u32(&tfull_bar[acc]), 0x3);      // accumulator ready in both CTAs
      }
      commit_pair(smem_u32(drain_bar), 0x1);
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, &never, p.timeout_ns);
    }
  } else {
    // ---------------------------------------------------------------- epilogue (both CTAs)
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    uint8_t* S = staging + (warp - 2) * 2 * STAGE_TILE_BYTES;
    uint8_t* T = S + STAGE_TILE_BYTES;
    int it = 0;
    for (int ti = 0;; ++ti, ++it) {
      int t = -1, got = 1;
      if (lane == 0) got = next_tile(ti, t);
      got = __shfl_sync(0xffffffffu, got, 0);
      t = __shfl_sync(0xffffffffu, t, 0);
      if (!got || t < 0) break;
      const PairTile pt = decode_pair(p, t);
      const Tile tl{pt.b, pt.TM * 2 + (int)rank, pt.TN};
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
        uint4 creg[4];
        bool c_ready = false;
        if (p.C != nullptr && gi < p.M && gj0 + 32 <= p.N) {
          const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const char*>(p.C) +
                                                            ((long long)tl.b * p.c_bs + (long long)gi * p.ldc + gj0) * 2);
#pragma unroll
          for (int i = 0; i < 4; ++i) creg[i] = src[i];
          c_ready = true;
        }
        WPrefetch wpf;
        wpf.ok = false;
        if constexpr (UPD) {
          wpf = prefetch_w(p, u, tl, q, lane, c);
        }
        uint32_t r[32];
        tmem_ld32(tbase + (uint32_t)(c * 32), r);
        if (cc == 3) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) {
            if (leader) mbar_arrive(smem_u32(&tempty_bar[acc]));
            else remote_arrive_cta(leader_tempty + acc * 8);  // accumulator read out: no data handed over
          }
        }
        if constexpr (UPD) {
          update_chunk(p, u, tl, q, lane, c, r, creg, c_ready, f, S, wpf);
        } else {
          epilogue_chunk<SYM>(p, &tmap_d, tl, q, lane, c, r, creg, c_ready, f, S, T);
        }
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
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag && p.err != nullptr) atomicOr(p.err, kStatusTimeout);
}

// Product launches may start while the previous kernel on the stream drains
// (programmatic dependent launch); MUON_PDL=0 launches them fully serialised.
static bool programmatic_launch() {
  static const bool on = [] {
    const char* e = getenv("MUON_PDL");
    return !(e && e[0] == '0');
  }();
  return on;
}

template <bool B_MN, int IN_FMT, bool SYM, bool UPD = false, typename Slots = NoUpdate>
static int launch(const CUtensorMap& ma, const CUtensorMap& mb, const CUtensorMap& md, const Params& p,
                  cudaStream_t s, const Slots& u = Slots{}) {
  // per device: shared-memory opt-in done and how many CTA pairs fit at once
  static std::atomic<int> max_pairs_of[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return (int)cudaErrorInvalidDevice;
  auto kern = gemm_pair_kernel<B_MN, IN_FMT, SYM, UPD>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES2;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_pairs = max_pairs_of[dev].load(std::memory_order_acquire);
  if (max_pairs <= 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES2);
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
  cfg.numAttrs = programmatic_launch() ? 2 : 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, kern, ma, mb, md, p, u);
  return (int)e;
}

}  // namespace pairk

int gemm_tc_pair(const GemmDesc& g, Params p, cudaStream_t s) {
  using namespace pairk;
  if (p.tile_counter == nullptr) return (int)cudaErrorInvalidValue;
  // pair tiles: 256 rows x 256 columns
  p.tiles_m = (g.M + 255) / 256;
  p.tiles_n = (g.N + BN - 1) / BN;
  if (g.symmetric) {
    p.tiles_per_batch = p.tiles_m * (p.tiles_m + 1) / 2;  // M == N: tiles_m == tiles_n
  } else {
    p.tiles_per_batch = p.tiles_m * p.tiles_n;
  }
  const long long total = (long long)p.tiles_per_batch * g.batch;
  if (total > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
  p.total_tiles = (int)total;
  CUtensorMap ma, mb;
  if (!encode_map(&ma, g.in_dtype, g.A, g.K, g.M, g.batch, g.lda, g.a_bs, BK, BM)) return (int)cudaErrorInvalidValue;
  const bool bmn = !g.b_kmajor;
  if (bmn) {
    if (!encode_map(&mb, g.in_dtype, g.B, g.N, g.K, g.batch, g.ldb, g.b_bs, 64, BK)) return (int)cudaErrorInvalidValue;
  } else {
    if (!encode_map(&mb, g.in_dtype, g.B, g.K, g.N, g.batch, g.ldb, g.b_bs, BK, 128)) return (int)cudaErrorInvalidValue;
  }
  CUtensorMap md;
  if (!encode_out_map(&md, g)) return (int)cudaErrorInvalidValue;
  const int fmt = g.in_dtype == kBF16 ? 1 : 0;
  if (g.update != nullptr) {
    // the fused update follows the chain's last product: X' = a X + B X (B MN-major)
    if (g.symmetric || !bmn || g.batch > UpdateSlots::kMax) return (int)cudaErrorInvalidValue;
    return fmt ? launch<true, 1, false, true>(ma, mb, md, p, s, *g.update)
               : launch<true, 0, false, true>(ma, mb, md, p, s, *g.update);
  }
  if (g.symmetric) {
    if (bmn) return fmt ? launch<true, 1, true>(ma, mb, md, p, s) : launch<true, 0, true>(ma, mb, md, p, s);
    return fmt ? launch<false, 1, true>(ma, mb, md, p, s) : launch<false, 0, true>(ma, mb, md, p, s);
  }
  if (bmn) return fmt ? launch<true, 1, false>(ma, mb, md, p, s) : launch<true, 0, false>(ma, mb, md, p, s);
  return fmt ? launch<false, 1, false>(ma, mb, md, p, s) : launch<false, 0, false>(ma, mb, md, p, s);
}

}  // namespace tc
}  // namespace muon
