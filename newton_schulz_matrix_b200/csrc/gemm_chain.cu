// One persistent launch for a whole Newton-Schulz chain (16-bit operands,
// products with 256 or more rows).
//
// Every product of the chain ("Gram Newton-Schulz" write-up: X X^T, A^2, B X
// per standard iteration; R0, R^2, Q Q_acc, Q R, (Q R) Q, the restart pair and
// the final Q_acc X0 in the Gram forms) becomes a range of tiles in one index
// space, in chain order.  CTA pairs take tiles from that space in order, as in
// the paired-CTA product kernel (gemm_tc2.cu: 256 x 256 tiles, cta_group::2
// MMAs, TMA loads and stores, the same fused epilogue), so the tail of one
// product overlaps the head of the next and there is no launch boundary
// between products.
//
// Dependencies are tracked per product and matrix: every epilogue warp of a
// tile, once its stores have landed in memory, adds one to done[p][b] (release,
// GPU scope).  The scheduler publishes a tile of product p for matrix b only
// when done[p-1][b] has reached all arrivals of product p-1 for that matrix
// (acquire); the roles that follow it read the tile through the cluster-scope
// ring, which carries that ordering to them.  Product p-1 itself waited for p-2, so every earlier product of
// the chain is complete for matrix b, which covers every read-after-write and
// write-after-read hazard of the chain's buffers.  Tiles are handed out in
// chain order and the grid is co-resident, so a waiting tile only waits for
// tiles that were handed out earlier and are being processed: the waits end.
// They are bounded all the same (MUON_STATUS_TIMEOUT on expiry).
#include <stdio.h>
#include <stdlib.h>

#include <atomic>
#include <type_traits>

#include "tc_common.cuh"

namespace muon {
namespace tc {
namespace chaink {

constexpr int STAGES = 6;
constexpr int A_BYTES = BM * BK * 2;   // this CTA's 128 rows of A: 16 KB
constexpr int B_BYTES = 128 * BK * 2;  // this CTA's 128 columns of B: 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int RING = 8;
constexpr int RING_CONSUMERS = 1 + 1 + 2 * NUM_EPI_WARPS;
constexpr int BAR_BYTES = 512;
constexpr int SMEM_BYTES_CHAIN = STAGES * STAGE_BYTES + STAGING_BYTES + 1024 + BAR_BYTES;
constexpr int ARRIVALS_PER_TILE = 2 * NUM_EPI_WARPS;  // epilogue warps of both CTAs
static_assert((2 * STAGES + 5 + 2 * RING) * 8 + RING * 4 + 8 <= BAR_BYTES, "barrier area");

__device__ __forceinline__ void tma_load_pair(uint32_t dst, const CUtensorMap* map, uint32_t bar_cluster, int x, int y,
                                              int z) {
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
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void red_release_gpu_add(int* p, int v) {
  asm volatile("red.release.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait until *cnt >= target (acquire); false on timeout or abort.
__device__ __forceinline__ bool wait_count(const int* cnt, int target, volatile int* abort_flag, long long timeout_ns) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = global_timer();
  for (uint32_t it = 1; it < (1u << 30); ++it) {
    if (ld_acquire_gpu(cnt) >= target) return true;
    if ((it & 15u) == 0) {
      if (*abort_flag) return false;
      if ((long long)(global_timer() - t0) > timeout_ns) {
        *abort_flag = 1;
        return false;
      }
    }
    __nanosleep(64);
  }
  *abort_flag = 1;
  return false;
}

// A chain tile: product index, and the product's own Params view and tile.
struct ChainTile {
  int prod;
  PairTile t;
};

__device__ __forceinline__ Params product_params(const ChainProduct& c) {
  Params p{};
  p.M = c.M; p.N = c.N; p.K = c.K; p.batch = c.batch;
  p.tiles_m = c.tiles_m; p.tiles_n = c.tiles_n; p.tiles_per_batch = c.tiles_per_batch;
  p.total_tiles = c.tiles_per_batch * c.batch;
  p.symmetric = c.symmetric;
  p.D = c.D; p.ldd = c.ldd; p.d_bs = c.d_bs; p.d_dtype = c.d_dtype;
  p.C = c.C; p.ldc = c.ldc; p.c_bs = c.c_bs; p.c_dtype = c.c_dtype;
  p.c_acc = c.c_acc; p.c_in = c.c_in; p.c_eye = c.c_eye;
  p.scale = c.scale; p.scale_pow = c.scale_pow;
  return p;
}

template <typename CP>
__device__ __forceinline__ ChainTile decode_chain(const CP& cp, int t) {
  int pi = 0;
  while (pi + 1 < cp.n_products && t >= cp.prod[pi + 1].first_tile) ++pi;
  ChainTile r;
  r.prod = pi;
  r.t = decode_pair(product_params(cp.prod[pi]), t - cp.prod[pi].first_tile);
  return r;
}

struct NoUpdate {
  int unused;
};

template <int IN_FMT, bool UPD>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_chain_kernel(const __grid_constant__ ChainParams cp,
                  const __grid_constant__ std::conditional_t<UPD, UpdateSlots, NoUpdate> u) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* staging = smem + STAGES * STAGE_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + STAGES * STAGE_BYTES + STAGING_BYTES);
  uint64_t* full_bar = bars;
  uint64_t* empty_bar = bars + STAGES;
  uint64_t* tfull_bar = bars + 2 * STAGES;
  uint64_t* tempty_bar = bars + 2 * STAGES + 2;
  uint64_t* drain_bar = bars + 2 * STAGES + 4;
  uint64_t* ring_full = bars + 2 * STAGES + 5;
  uint64_t* ring_empty = ring_full + RING;
  int* tile_ring = reinterpret_cast<int*>(ring_empty + RING);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tile_ring + RING);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
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
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const uint32_t tmem_base = *tmem_slot;
  const uint32_t leader_full = mapa(smem_u32(full_bar), 0);
  const uint32_t leader_tempty = mapa(smem_u32(tempty_bar), 0);
  const uint32_t leader_ring_empty = mapa(smem_u32(ring_empty), 0);
  auto next_tile = [&](int i, int& t) -> bool {
    const int slot = i % RING;
    const uint32_t rph = (uint32_t)(i / RING) & 1u;
    if (leader) {
      // the ring and its barriers are this CTA's own: CTA-scope wait and arrive
      if (!mbar_wait(smem_u32(&ring_full[slot]), rph, abort_flag, cp.timeout_ns)) return false;
      t = tile_ring[slot];
      mbar_arrive(smem_u32(&ring_empty[slot]));
    } else {
      // published from the leader CTA: cluster-scope acquire, remote release
      if (!mbar_wait_cluster(smem_u32(&ring_full[slot]), rph, abort_flag, cp.timeout_ns)) return false;
      t = tile_ring[slot];
      remote_arrive(leader_ring_empty + slot * 8);
    }
    return true;
  };
  // The arrivals that mark product p's tiles of matrix b complete.
  auto dep_ready = [&](int p, int b) -> bool {
    const ChainProduct& d = cp.prod[p];
    if (d.dep < 0) return true;
    const int target = cp.prod[d.dep].tiles_per_batch * ARRIVALS_PER_TILE;
    return wait_count(cp.done + (long long)d.dep * cp.batch + b, target, abort_flag, cp.timeout_ns);
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
        const int t = cp.static_order ? pair + i * npairs : atomicAdd(cp.tile_counter, 1);
        return t < cp.total_tiles ? t : -1;
      };
      int held = leader ? take(0) : -1;
      for (int i = 0; ok; ++i) {
        int t;
        if (leader) {
          const int slot = i % RING;
          if (!mbar_wait_cluster(smem_u32(&ring_empty[slot]), ((uint32_t)(i / RING) & 1u) ^ 1u, abort_flag,
                                 cp.timeout_ns))
            break;
          t = held;
          if (t >= 0) {
            held = take(i + 1);
            // the tile's operands were written by earlier products of the chain:
            // acquire them here, once for the whole pair, before publishing it
            const ChainTile dt = decode_chain(cp, t);
            if (!dep_ready(dt.prod, dt.t.b)) break;
          }
          tile_ring[slot] = t;
          st_cluster_s32(mapa(smem_u32(&tile_ring[slot]), 1), t);
          mbar_arrive(smem_u32(&ring_full[slot]));            // this CTA's roles
          remote_arrive(mapa(smem_u32(&ring_full[slot]), 1));  // the peer's
        } else if (!next_tile(i, t)) {
          break;
        }
        if (t < 0) break;
        const ChainTile ct = decode_chain(cp, t);
        const ChainProduct& pr = cp.prod[ct.prod];
        // the leader acquired this tile's inputs before publishing it (below);
        // the peer synchronised with the leader through the ring, and both
        // order the acquire before their TMA (async proxy) reads
        fence_proxy_async_global();
        const bool narrow = pr.N - ct.t.TN * 256 <= 128;
        const int row0 = ct.t.TM * 256 + (int)rank * 128;
        const int col0 = ct.t.TN * 256 + (int)rank * (narrow ? 64 : 128);
        const int num_kb = (pr.K + BK - 1) / BK;
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&empty_bar[stage]), phase ^ 1u, abort_flag, cp.timeout_ns)) { ok = false; break; }
          if (leader) mbar_expect_tx(smem_u32(&full_bar[stage]), 2 * STAGE_BYTES);
          const uint32_t fb = leader_full + stage * 8;
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
          tma_load_pair(sa, &pr.ma, fb, kb * BK, row0, ct.t.b);
          if (pr.b_mn) {
#pragma unroll
            for (int q = 0; q < 2; ++q) tma_load_pair(sb + q * (BK * 128), &pr.mb, fb, col0 + q * 64, kb * BK, ct.t.b);
          } else {
            tma_load_pair(sb, &pr.mb, fb, kb * BK, col0, ct.t.b);
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer (leader only)
    if (lane == 0 && leader) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int i = 0; ok; ++i, ++it) {
        int t;
        if (!next_tile(i, t) || t < 0) break;
        const ChainTile ct = decode_chain(cp, t);
        const ChainProduct& pr = cp.prod[ct.prod];
        const bool narrow = pr.N - ct.t.TN * 256 <= 128;
        const uint32_t idesc = make_idesc(IN_FMT, pr.b_mn, 256, narrow ? 128 : 256);
        const int num_kb = (pr.K + BK - 1) / BK;
        const int acc = it & 1;
        const uint32_t aph = (uint32_t)(it >> 1) & 1u;
        if (!mbar_wait(smem_u32(&tempty_bar[acc]), aph ^ 1u, abort_flag, cp.timeout_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (uint32_t)(acc * BN);
        for (int kb = 0; kb < num_kb; ++kb) {
          if (!mbar_wait(smem_u32(&full_bar[stage]), phase, abort_flag, cp.timeout_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + stage * STAGE_BYTES);
          const uint32_t sb = sa + A_BYTES;
#pragma unroll
          for (int k = 0; k < BK / UMMA_K; ++k) {
            const uint64_t ad = smem_desc(sa + k * (UMMA_K * 2), 16, 1024);
            const uint64_t bd = pr.b_mn ? smem_desc(sb + k * (UMMA_K * 128), BK * 128, 1024)
                                        : smem_desc(sb + k * (UMMA_K * 2), 16, 1024);
            mma_pair(d_tmem, ad, bd, idesc, (kb | k) != 0);
          }
          commit_pair(smem_u32(&empty_bar[stage]), 0x3);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        commit_pair(smem_u32(&tfull_bar[acc]), 0x3);
      }
      commit_pair(smem_u32(drain_bar), 0x1);
      volatile int never = 0;
      mbar_wait(smem_u32(drain_bar), 0, &never, cp.timeout_ns);
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
      const ChainTile ct = decode_chain(cp, t);
      const ChainProduct& pr = cp.prod[ct.prod];
      const Params p = product_params(pr);
      const Tile tl{ct.t.b, ct.t.TM * 2 + (int)rank, ct.t.TN};
      const int acc = it & 1;
      const uint32_t aph = (uint32_t)(it >> 1) & 1u;
      // C was written by an earlier product: the leader acquired it before
      // publishing this tile, and lane 0 read the tile from the ring with
      // acquire semantics; the warp barrier orders that before every lane's loads
      int ok = 1;
      if (lane == 0) ok = mbar_wait(smem_u32(&tfull_bar[acc]), aph, abort_flag, cp.timeout_ns);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) break;
      tc_fence_after();
      const float f = matrix_scale(p.scale, p.scale_pow, tl.b);
      const uint32_t tbase = tmem_base + (uint32_t)(acc * BN) + ((uint32_t)(q * 32) << 16);
      const int gi = tl.tm * BM + q * 32 + lane;
      const bool upd = UPD && ct.prod == cp.n_products - 1;
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
          for (int k = 0; k < 4; ++k) creg[k] = src[k];
          c_ready = true;
        }
        WPrefetch wpf;
        wpf.ok = false;
        if constexpr (UPD) {
          if (upd) wpf = prefetch_w(p, u, tl, q, lane, c);
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
          if (upd) {
            update_chunk(p, u, tl, q, lane, c, r, creg, c_ready, f, S, wpf);
            continue;
          }
        }
        if (p.symmetric) epilogue_chunk<true>(p, &pr.md, tl, q, lane, c, r, creg, c_ready, f, S, T);
        else epilogue_chunk<false>(p, &pr.md, tl, q, lane, c, r, creg, c_ready, f, S, T);
      }
      // this warp's part of the tile is in memory: count it for the products that read it
      if (lane == 0) {
        bulk_wait_all0();
        fence_proxy_async_global();
        red_release_gpu_add(cp.done + (long long)ct.prod * cp.batch + tl.b, 1);
      }
      __syncwarp();
    }
    if (lane == 0) bulk_wait_all0();
    __syncwarp();
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem_base), "r"(TMEM_COLS) : "memory");
  }
  if (threadIdx.x == 0 && *abort_flag && cp.err != nullptr) atomicOr(cp.err, kStatusTimeout);
}

template <int IN_FMT, bool UPD, typename Slots>
static int launch(const ChainParams& cp, const Slots& u, cudaStream_t s) {
  static std::atomic<int> max_pairs_of[kMaxDevices];
  const int dev = current_device();
  if (dev < 0) return (int)cudaErrorInvalidDevice;
  auto kern = gemm_chain_kernel<IN_FMT, UPD>;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = SMEM_BYTES_CHAIN;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int max_pairs = max_pairs_of[dev].load(std::memory_order_acquire);
  if (max_pairs <= 0) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES_CHAIN);
    if (e != cudaSuccess) return (int)e;
    cfg.gridDim = dim3(2 * (num_sms() / 2));
    int n = 0;
    e = cudaOccupancyMaxActiveClusters(&n, kern, &cfg);
    if (e != cudaSuccess || n <= 0) n = num_sms() / 2;
    max_pairs = n;
    max_pairs_of[dev].store(n, std::memory_order_release);
  }
  // every pair must be resident at once: a tile may wait for tiles other pairs hold
  const int pairs = cp.total_tiles < max_pairs ? cp.total_tiles : max_pairs;
  cfg.gridDim = dim3(2 * pairs);
  cfg.numAttrs = 2;
  return (int)cudaLaunchKernelEx(&cfg, kern, cp, u);
}

}  // namespace chaink
}  // namespace tc

int gemm_chain(const GemmDesc* prods, int n, int* tile_counter, int* done, int* err, cudaStream_t s) {
  using namespace tc;
  using namespace tc::chaink;
  if (n <= 0 || n > ChainParams::kMaxProducts || !tile_counter || !done) return (int)cudaErrorInvalidValue;
  ChainParams cp{};
  cp.n_products = n;
  cp.batch = prods[0].batch;
  cp.tile_counter = tile_counter;
  cp.done = done;
  cp.err = err;
  cp.timeout_ns = wait_timeout_ns();
  cp.static_order = static_tile_order() ? 1 : 0;
  long long first = 0;
  const UpdateSlots* upd = nullptr;
  int fmt = -1;
  for (int i = 0; i < n; ++i) {
    const GemmDesc& g = prods[i];
    ChainProduct& c = cp.prod[i];
    if (g.batch != cp.batch || g.M < 256 || g.M <= 0 || g.N <= 0) return (int)cudaErrorInvalidValue;
    if (g.in_dtype != kBF16 && g.in_dtype != kFP16) return (int)cudaErrorInvalidValue;
    if (g.d_dtype == kFP32 || (g.C && g.c_dtype == kFP32)) return (int)cudaErrorInvalidValue;
    if (g.symmetric && g.M != g.N) return (int)cudaErrorInvalidValue;
    const int f = g.in_dtype == kBF16 ? 1 : 0;
    if (fmt >= 0 && f != fmt) return (int)cudaErrorInvalidValue;  // one operand type per chain
    fmt = f;
    if (g.update != nullptr) {
      if (i != n - 1 || g.symmetric || g.b_kmajor || g.batch > UpdateSlots::kMax) return (int)cudaErrorInvalidValue;
      upd = g.update;
    }
    c.M = g.M; c.N = g.N; c.K = g.K; c.batch = g.batch;
    c.tiles_m = (g.M + 255) / 256;
    c.tiles_n = (g.N + 255) / 256;
    c.tiles_per_batch = g.symmetric ? c.tiles_m * (c.tiles_m + 1) / 2 : c.tiles_m * c.tiles_n;
    c.first_tile = (int)first;
    first += (long long)c.tiles_per_batch * g.batch;
    if (first > 0x7fffffffLL) return (int)cudaErrorInvalidValue;
    c.symmetric = g.symmetric;
    c.b_mn = !g.b_kmajor;
    c.dep = i - 1;
    c.D = g.D; c.ldd = g.ldd; c.d_bs = g.d_bs; c.d_dtype = g.d_dtype;
    c.C = g.C; c.ldc = g.ldc; c.c_bs = g.c_bs; c.c_dtype = g.c_dtype;
    c.c_acc = g.c_acc; c.c_in = g.c_in; c.c_eye = g.c_eye;
    c.scale = g.scale; c.scale_pow = g.scale_pow;
    if (!encode_map(&c.ma, g.in_dtype, g.A, g.K, g.M, g.batch, g.lda, g.a_bs, BK, BM)) return (int)cudaErrorInvalidValue;
    if (c.b_mn) {
      if (!encode_map(&c.mb, g.in_dtype, g.B, g.N, g.K, g.batch, g.ldb, g.b_bs, 64, BK)) return (int)cudaErrorInvalidValue;
    } else {
      if (!encode_map(&c.mb, g.in_dtype, g.B, g.K, g.N, g.batch, g.ldb, g.b_bs, BK, 128)) return (int)cudaErrorInvalidValue;
    }
    if (!encode_out_map(&c.md, g)) return (int)cudaErrorInvalidValue;
  }
  cp.total_tiles = (int)first;
  if (upd) return fmt ? launch<1, true>(cp, *upd, s) : launch<0, true>(cp, *upd, s);
  return fmt ? launch<1, false>(cp, NoUpdate{}, s) : launch<0, false>(cp, NoUpdate{}, s);
}

}  // namespace muon
