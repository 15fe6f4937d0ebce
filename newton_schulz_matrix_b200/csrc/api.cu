// C ABI of libmuon (include/muon.h): argument checks, the shape planner that
// merges groups by oriented shape and cuts them into workspace-sized chunks,
// the workspace layout, and the launch sequence of one Muon step:
//
//   pack (momentum, Nesterov, orientation, sums of squares)  -> norm
//   -> Newton-Schulz chain                                    -> unpack (update)
//
// The chain's products run on the tensor cores: tcgen05 kind::f16 for bf16 and
// fp16 storage, 3xTF32 (kind::tf32) for fp32 storage with n >= 256.  An fp32
// chain of matrices small enough for one CTA's shared memory runs as a single
// fused launch, and the remaining fp32 products run on a CUDA-core kernel.
//
// The iteration order follows the "Gram Newton-Schulz" write-up (standard
// form: A = X X^T, B = b A + c A^2, X = a X + B X; Gram form: iterate on
// R = X X^T, accumulate Q_acc = Q_k ... Q_1, restart in the stabilised
// variant) and the optimizer step of "Moonlight 16B Guide" (box steps 1-4).
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <algorithm>
#include <cmath>
#include <mutex>
#include <vector>

#include "../../include/muon.h"
#include "common.cuh"
#include "internal.h"

using namespace muon;

namespace {

constexpr size_t kAlign = 256;
inline size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }
inline int round8(int v) { return (v + 7) / 8 * 8; }

// ------------------------------------------------------------------ profiler
enum ProfKind {
  kProfPack, kProfNorm, kProfSyrkTc, kProfGemmTc, kProfGemmSimt, kProfUnpack, kProfFusedSmall, kProfTf32, kProfChain,
  kProfStatus, kProfSplit, kProfKinds
};
// product kinds cover both tensor-core kernels (gemm_pair_kernel for M >= 256, gemm_kernel below);
// tc_chain is a whole chain in one launch (gemm_chain_kernel)
const char* const kProfNames[kProfKinds] = {"pack_kernel", "norm_kernel", "tc_product[symmetric]", "tc_product",
                                            "gemm_simt_kernel", "unpack_kernel", "ns_fused_small_kernel",
                                            "tc_product[3xtf32]", "tc_chain", "status_or_kernel",
                                            "split_tf32_kernel"};
struct ProfRec {
  int kind;
  cudaEvent_t a, b;
  double flops, exec_flops, bytes;
};
struct Profiler {
  bool on = false;
  std::vector<ProfRec> recs;
  std::mutex mu;
};
Profiler& profiler() {
  static Profiler p;
  return p;
}
// Brackets one launch with events on its stream while profiling is on.
struct ProfScope {
  ProfRec rec{};
  bool active = false;
  cudaStream_t s;
  ProfScope(int kind, double flops, double bytes, cudaStream_t st, double exec_flops = -1.0) : s(st) {
    Profiler& P = profiler();
    if (!P.on) return;
    rec.kind = kind; rec.flops = flops; rec.bytes = bytes;
    rec.exec_flops = exec_flops < 0.0 ? flops : exec_flops;
    if (cudaEventCreate(&rec.a) != cudaSuccess) return;
    if (cudaEventCreate(&rec.b) != cudaSuccess) { cudaEventDestroy(rec.a); return; }
    cudaEventRecord(rec.a, s);
    active = true;
  }
  ~ProfScope() {
    if (!active) return;
    cudaEventRecord(rec.b, s);
    Profiler& P = profiler();
    std::lock_guard<std::mutex> g(P.mu);
    P.recs.push_back(rec);
  }
};

struct Seg {          // `count` matrices of one caller group, starting at index `first`
  int group, first, count;
};

struct Batch {        // matrices that orient to the same n x m
  int n, m;
  std::vector<Seg> segs;
  int total = 0;
};

struct Layout {       // per-chunk workspace layout for a batch
  int n, m, ld_m, ld_n;
  int x_es, g_es;     // element sizes of X and Gram buffers
  int n_sq;           // number of n x n buffers
  int tiles;          // pack tiles per matrix (sums-of-squares partials)
  int n_counters;     // tile-scheduler words: one per product launch of the chain
  size_t head;        // error word + counters, zeroed at the start of each chunk
                      // (followed by the chain launches' done counters: n_counters per matrix)
  bool tf32;          // fp32 chain on the tensor cores: TF32 hi/lo planes of the operands
  size_t per_matrix;  // bytes per matrix (all buffers)
  size_t fixed;       // bytes independent of the chunk size
};

bool fp32_tensor_cores();

bool ns_params_ok(const muon_ns_params* ns) {
  if (!ns || ns->iters < 1 || ns->iters > 1000 || !ns->coeffs) return false;
  if (ns->mode < MUON_NS_STANDARD || ns->mode > MUON_NS_GRAM_STABILIZED) return false;
  if (ns->mode == MUON_NS_GRAM_STABILIZED && (ns->restart_after < 1 || ns->restart_after >= ns->iters)) return false;
  if (ns->restart_every < 0) return false;
  if (!(ns->eps >= 0.f) || !std::isfinite(ns->eps)) return false;
  if (ns->compute_dtype < MUON_BF16 || ns->compute_dtype > MUON_FP32) return false;
  if (ns->mode != MUON_NS_STANDARD && ns->compute_dtype != MUON_FP32 && ns->gram_dtype != MUON_BF16 &&
      ns->gram_dtype != MUON_FP16)
    return false;
  for (int i = 0; i < 3 * ns->iters; ++i)
    if (!std::isfinite(ns->coeffs[i])) return false;
  return true;
}

bool dtype_ok(int d) { return d == MUON_BF16 || d == MUON_FP16 || d == MUON_FP32; }

Layout make_layout(int n, int m, const muon_ns_params* ns) {
  Layout L{};
  L.n = n; L.m = m;
  L.ld_m = round8(m);
  L.ld_n = round8(n);
  L.x_es = ns->compute_dtype == MUON_FP32 ? 4 : 2;
  L.g_es = ns->compute_dtype == MUON_FP32 ? 4 : 2;
  L.n_sq = ns->mode == MUON_NS_STANDARD ? 2 : 5;
  L.tiles = pack_tiles(n, m);
  // at most 6 product launches per iteration (Gram form: R^2, Q Q_acc, T, R or a
  // restart pair) plus R0 and the final apply
  L.n_counters = 6 * ns->iters + 8;
  L.head = align_up(kAlign + (size_t)L.n_counters * 4, kAlign);
  // buffers: 2 X, n_sq Gram-sized, partials, inv (each 256-byte aligned per chunk)
  L.per_matrix = 2 * (size_t)n * L.ld_m * L.x_es + (size_t)L.n_sq * n * L.ld_n * L.g_es + (size_t)L.tiles * 4 + 4 +
                 (size_t)L.n_counters * 4;
  L.fixed = kAlign * (2 + L.n_sq + 3) + kAlign + L.head;  // alignment slack + error word and counters
  // every product of an fp32 chain with n >= 256 runs as 3xTF32 and reads its
  // operands as hi / lo planes: one X-sized pair and two n x n pairs (a
  // product has at most two distinct operands, and at most one is X-sized)
  L.tf32 = ns->compute_dtype == MUON_FP32 && n >= 256 && fp32_tensor_cores();
  if (L.tf32) {
    L.per_matrix += 2 * ((size_t)n * L.ld_m + 2 * (size_t)n * L.ld_n) * 4;
    L.fixed += kAlign * 6;
  }
  return L;
}

size_t chunk_bytes(const Layout& L, int chunk) { return L.fixed + L.per_matrix * (size_t)chunk; }

struct Bufs {
  void* X[2];
  void* S[5];
  float* planes[3][2];  // fp32 tensor-core chains: [X-sized, n x n, n x n][hi, lo]
  size_t plane_elems[3];
  float* partials;
  float* inv;
  int* err;
  int* counters;      // L.n_counters words after the error word's 256-byte slot
  int* done;          // chunk * L.n_counters words: per product and matrix, for chain launches
  size_t zero_bytes;  // from err through done: zeroed at the start of the chunk
  long long x_bs, s_bs;
};

Bufs carve(const Layout& L, int chunk, void* ws) {
  Bufs B{};
  char* p = reinterpret_cast<char*>(align_up(reinterpret_cast<uintptr_t>(ws), kAlign));
  B.err = reinterpret_cast<int*>(p);
  B.counters = reinterpret_cast<int*>(p + kAlign);
  p += L.head;
  B.done = reinterpret_cast<int*>(p);
  p += align_up((size_t)chunk * L.n_counters * 4, kAlign);
  B.zero_bytes = L.head + align_up((size_t)chunk * L.n_counters * 4, kAlign);
  B.x_bs = (long long)L.n * L.ld_m;
  B.s_bs = (long long)L.n * L.ld_n;
  for (int i = 0; i < 2; ++i) {
    B.X[i] = p;
    p += align_up((size_t)chunk * B.x_bs * L.x_es, kAlign);
  }
  for (int i = 0; i < L.n_sq; ++i) {
    B.S[i] = p;
    p += align_up((size_t)chunk * B.s_bs * L.g_es, kAlign);
  }
  B.partials = reinterpret_cast<float*>(p);
  p += align_up((size_t)chunk * L.tiles * 4, kAlign);
  B.inv = reinterpret_cast<float*>(p);
  p += align_up((size_t)chunk * 4, kAlign);
  if (L.tf32) {
    for (int i = 0; i < 3; ++i) {
      B.plane_elems[i] = (size_t)chunk * (i == 0 ? B.x_bs : B.s_bs);
      for (int h = 0; h < 2; ++h) {
        B.planes[i][h] = reinterpret_cast<float*>(p);
        p += align_up(B.plane_elems[i] * 4, kAlign);
      }
    }
  }
  return B;
}

std::vector<Batch> plan_groups(const muon_group* groups, int n_groups) {
  std::vector<Batch> out;
  for (int g = 0; g < n_groups; ++g) {
    const int n = std::min(groups[g].rows, groups[g].cols), m = std::max(groups[g].rows, groups[g].cols);
    if (groups[g].count == 0) continue;
    Batch* b = nullptr;
    for (auto& x : out)
      if (x.n == n && x.m == m) b = &x;
    if (!b) {
      out.push_back(Batch{n, m, {}, 0});
      b = &out.back();
    }
    b->segs.push_back(Seg{g, 0, groups[g].count});
    b->total += groups[g].count;
  }
  return out;
}

// ------------------------------------------------------------------ products
// The TF32 hi / lo planes of the chunk's fp32 operands, and which buffer's
// split each pair holds now: a split is reused until a product overwrites its
// source (X's split serves both X X^T and the update X <- aX + BX).
struct PlaneCache {
  float* hi[3] = {};
  float* lo[3] = {};
  size_t cap[3] = {};            // elements
  const void* held[3] = {};      // source buffer of the split the pair holds, or null
  int n = 0;
};

struct Ctx {
  int compute;   // MUON_BF16 / MUON_FP16 / MUON_FP32
  cudaStream_t s;
  int* err;
  int* counters;       // zeroed tile-scheduler words, one per product launch
  int n_counters;
  int* used;           // how many of them the chain has taken so far
  std::vector<GemmDesc>* record = nullptr;  // chain mode: collect the products instead of launching them
  PlaneCache* planes = nullptr;             // fp32 tensor-core chains
};

// The plane pair that holds (or is to receive) the split of `src`, `elems`
// values, not pair `avoid` (-1: none).  *fresh: the pair must be (re)written.
int plane_pair(PlaneCache& pc, const void* src, size_t elems, int avoid, bool* fresh) {
  for (int i = 0; i < pc.n; ++i)
    if (i != avoid && pc.held[i] == src && pc.cap[i] >= elems) {
      *fresh = false;
      return i;
    }
  int best = -1;
  for (int i = 0; i < pc.n; ++i) {
    if (i == avoid || pc.cap[i] < elems) continue;
    // the smallest pair that fits (an n x n operand never takes the X-sized
    // pair that the update product's X needs), an empty one among equals
    if (best < 0 || pc.cap[i] < pc.cap[best] ||
        (pc.cap[i] == pc.cap[best] && pc.held[i] == nullptr && pc.held[best] != nullptr))
      best = i;
  }
  *fresh = true;
  return best;
}

// fp32 products with 256 or more rows run as 3xTF32 on the tensor cores;
// MUON_FP32_TC=0 keeps every fp32 product on the SIMT kernel.
bool fp32_tensor_cores() {
  static const bool on = [] {
    const char* e = getenv("MUON_FP32_TC");
    return !(e && e[0] == '0');
  }();
  return on;
}

int gemm(const Ctx& c, GemmDesc g) {
  g.err = c.err;
  if (c.record != nullptr) {
    c.record->push_back(g);
    return 0;
  }
  if (*c.used >= c.n_counters) return (int)cudaErrorInvalidValue;
  g.tile_counter = c.counters + (*c.used)++;
  const double flops = 2.0 * g.M * g.N * (double)g.K * g.batch;
  const int es = dtype_size(g.in_dtype);
  const double bytes = ((double)g.M * g.K * es + (double)g.N * g.K * es + (double)g.M * g.N * dtype_size(g.d_dtype) +
                        (g.C ? (double)g.M * g.N * dtype_size(g.c_dtype) : 0.0)) * g.batch;
  const bool prof = profiler().on;
  if (c.compute == MUON_FP32) {
    if (g.M >= 256 && fp32_tensor_cores()) {
      if (c.planes == nullptr) return (int)cudaErrorInvalidValue;
      PlaneCache& pc = *c.planes;
      const size_t a_elems = (size_t)g.a_bs * g.batch, b_elems = (size_t)g.b_bs * g.batch;
      bool fresh_a = false, fresh_b = false;
      const int ia = plane_pair(pc, g.A, a_elems, -1, &fresh_a);
      if (ia < 0) return (int)cudaErrorInvalidValue;
      if (fresh_a) pc.held[ia] = nullptr;  // being rewritten
      int ib = ia;
      if (g.B != g.A) {
        ib = plane_pair(pc, g.B, b_elems, ia, &fresh_b);
        if (ib < 0) return (int)cudaErrorInvalidValue;
        if (fresh_b) pc.held[ib] = nullptr;
      }
      int rc;
      if (fresh_a) {
        ProfScope ps(kProfSplit, 0.0, a_elems * 12.0, c.s);
        if ((rc = split_tf32(reinterpret_cast<const float*>(g.A), pc.hi[ia], pc.lo[ia], (long long)a_elems, c.s)))
          return rc;
        pc.held[ia] = g.A;
      }
      if (fresh_b) {
        ProfScope ps(kProfSplit, 0.0, b_elems * 12.0, c.s);
        if ((rc = split_tf32(reinterpret_cast<const float*>(g.B), pc.hi[ib], pc.lo[ib], (long long)b_elems, c.s)))
          return rc;
        pc.held[ib] = g.B;
      }
      const Tf32Planes tp{pc.hi[ia], pc.lo[ia], pc.hi[ib], pc.lo[ib]};
      {
        ProfScope ps(kProfTf32, flops, bytes, c.s, prof ? gemm_tf32x3_exec_flops(g) : 0.0);
        rc = gemm_tf32x3(g, tp, c.s);
      }
      for (int i = 0; i < pc.n; ++i)
        if (pc.held[i] == g.D) pc.held[i] = nullptr;  // its source has been overwritten
      return rc;
    }
    ProfScope ps(kProfGemmSimt, flops, bytes, c.s);
    return gemm_simt(g, c.s);
  }
  ProfScope ps(g.symmetric ? kProfSyrkTc : kProfGemmTc, flops, bytes, c.s, prof ? gemm_tc_exec_flops(g) : 0.0);
  return gemm_tc(g, c.s);
}

GemmDesc desc(int M, int N, int K, int batch) {
  GemmDesc g{};
  g.M = M; g.N = N; g.K = K; g.batch = batch;
  g.c_acc = 1.f;
  g.b_kmajor = 1;
  return g;
}

// Runs the Newton-Schulz chain on `chunk` packed matrices in X[0] and returns
// the index of the X buffer that holds the result and the result's dtype.
//
// 16-bit chains: the standard form stores X, A, B in compute_dtype; the Gram
// forms store every matrix of the chain (R, Q, Q_acc, X0, restart X) in
// gram_dtype, so that no product mixes operand types.  A bf16 chain receives
// the raw U (bf16's range holds any gradient) and applies f = 1/(||U||+eps)
// inside the first products' epilogues; an fp16 chain receives X0 = f U
// already normalised (`prescaled`), rounded once from fp32 to fp16.
// Whether the stabilised Gram chain restarts after iteration k (1-based).
bool restart_at(const muon_ns_params* ns, int k) {
  if (ns->mode != MUON_NS_GRAM_STABILIZED || k >= ns->iters || k < ns->restart_after) return false;
  if (k == ns->restart_after) return true;
  return ns->restart_every > 0 && (k - ns->restart_after) % ns->restart_every == 0;
}

int chain_dtype(const muon_ns_params* ns) {
  if (ns->compute_dtype == MUON_FP32) return MUON_FP32;
  return ns->mode == MUON_NS_STANDARD ? ns->compute_dtype : ns->gram_dtype;
}

double flops_of(int rows, int cols, const muon_ns_params* ns);  // algorithmic FLOPs of one matrix's chain

// 16-bit chains of a Muon step whose last product runs on the paired-CTA
// kernel write the update from that product's epilogue (no unpack pass, no X
// round trip through memory); MUON_FUSED_UPDATE=0 keeps the separate pass.
bool fused_update_enabled() {
  static const bool on = [] {
    const char* e = getenv("MUON_FUSED_UPDATE");
    return !(e && e[0] == '0');
  }();
  return on;
}

// fp32 chains whose matrices fit in one CTA's shared memory run as a single
// fused launch (one CTA per matrix); MUON_FUSED_SMALL=0 keeps the chained
// products instead.
bool fused_small_enabled() {
  static const bool on = [] {
    const char* e = getenv("MUON_FUSED_SMALL");
    return !(e && e[0] == '0');
  }();
  return on;
}

bool use_fused_small(const Layout& L, const muon_ns_params* ns) {
  if (ns->compute_dtype != MUON_FP32 || ns->iters > FusedSmallArgs::kMaxIters || !fused_small_enabled()) return false;
  return fused_small_smem(L.n, L.m, ns->mode == MUON_NS_STANDARD ? 0 : 1) <= kFusedSmallMaxSmem;
}

int run_fused_small(const Ctx& c, const Layout& L, const Bufs& B, int chunk, const muon_ns_params* ns, bool prescaled) {
  FusedSmallArgs a{};
  a.n = L.n; a.m = L.m; a.count = chunk;
  a.x = reinterpret_cast<float*>(B.X[0]); a.ld_x = L.ld_m; a.x_bs = B.x_bs;
  a.inv = B.inv; a.raw = prescaled ? 0 : 1;
  a.mode = ns->mode == MUON_NS_STANDARD ? 0 : 1;
  a.restart_after = ns->mode == MUON_NS_GRAM_STABILIZED ? ns->restart_after : 0;
  a.restart_every = ns->mode == MUON_NS_GRAM_STABILIZED ? ns->restart_every : 0;
  a.iters = ns->iters;
  for (int i = 0; i < 3 * ns->iters; ++i) a.coeffs[i] = ns->coeffs[i];
  ProfScope ps(kProfFusedSmall, flops_of(L.n, L.m, ns) * chunk, 2.0 * chunk * L.n * L.m * 4, c.s);
  return launch_fused_small(a, c.s);
}

// `update` (may be null): the chain's last product writes the Muon update
// into W through these slots instead of storing O (the result X is then not
// written; see run_batches).
int run_chain(const Ctx& c, const Layout& L, const Bufs& B, int chunk, const muon_ns_params* ns, bool prescaled,
              int* out_x, int* out_dtype, const UpdateSlots* update = nullptr) {
  if (use_fused_small(L, ns)) {
    *out_x = 0;
    *out_dtype = MUON_FP32;
    return run_fused_small(c, L, B, chunk, ns, prescaled);
  }
  const int n = L.n, m = L.m, K = ns->iters;
  const int cdt = chain_dtype(ns);
  const int xdt = cdt;  // X storage
  const int gdt = cdt;  // Gram-sized storage
  int rc;
  const int start = 0;
  const bool raw = !prescaled;
  *out_dtype = xdt;
  if (ns->mode == MUON_NS_STANDARD) {
    int cur = start;
    for (int k = 0; k < K; ++k) {
      const float a = ns->coeffs[3 * k], bb = ns->coeffs[3 * k + 1], cc = ns->coeffs[3 * k + 2];
      const bool first = k == 0 && raw;
      // A = f^2 X X^T  (f = 1/(||U||+eps) on the first iteration)
      GemmDesc g = desc(n, n, m, chunk);
      g.A = B.X[cur]; g.lda = L.ld_m; g.a_bs = B.x_bs;
      g.B = B.X[cur]; g.ldb = L.ld_m; g.b_bs = B.x_bs; g.b_kmajor = 1;
      g.in_dtype = xdt;
      g.D = B.S[0]; g.ldd = L.ld_n; g.d_bs = B.s_bs; g.d_dtype = xdt;
      g.scale = B.inv; g.scale_pow = first ? 2 : 0;
      g.symmetric = 1;
      if ((rc = gemm(c, g))) return rc;
      const void* Bm = B.S[0];
      float coefB = bb;
      if (cc != 0.f) {
        // B = c A A + b A   (A symmetric: A A = A A^T)
        g = desc(n, n, n, chunk);
        g.A = B.S[0]; g.lda = L.ld_n; g.a_bs = B.s_bs;
        g.B = B.S[0]; g.ldb = L.ld_n; g.b_bs = B.s_bs; g.b_kmajor = 1;
        g.in_dtype = xdt;
        g.D = B.S[1]; g.ldd = L.ld_n; g.d_bs = B.s_bs; g.d_dtype = xdt;
        g.C = B.S[0]; g.ldc = L.ld_n; g.c_bs = B.s_bs; g.c_dtype = xdt;
        g.c_acc = cc; g.c_in = bb;
        g.symmetric = 1;
        if ((rc = gemm(c, g))) return rc;
        Bm = B.S[1];
        coefB = 1.f;
      }
      // X' = f (a X + coefB Bm X)
      g = desc(n, m, n, chunk);
      g.A = Bm; g.lda = L.ld_n; g.a_bs = B.s_bs;
      g.B = B.X[cur]; g.ldb = L.ld_m; g.b_bs = B.x_bs; g.b_kmajor = 0;
      g.in_dtype = xdt;
      g.D = B.X[1 - cur]; g.ldd = L.ld_m; g.d_bs = B.x_bs; g.d_dtype = xdt;
      g.C = B.X[cur]; g.ldc = L.ld_m; g.c_bs = B.x_bs; g.c_dtype = xdt;
      g.c_acc = coefB; g.c_in = a;
      g.scale = B.inv; g.scale_pow = first ? 1 : 0;
      if (k == K - 1) g.update = update;
      if ((rc = gemm(c, g))) return rc;
      cur = 1 - cur;
    }
    *out_x = cur;
    return 0;
  }

  // ---------------------------------------------------------------- Gram forms
  int x0 = start;          // X buffer holding the matrix the Gram iteration applies to
  bool x0_raw = raw;       // still the unnormalised packed U (scale by inv on use)
  void* R = B.S[0];
  void* T = B.S[1];
  void* Qbuf[3] = {B.S[2], B.S[3], B.S[4]};
  int q_acc = -1;          // index into Qbuf, -1 = identity

  auto gram_of_x = [&](bool raw) -> int {
    GemmDesc g = desc(n, n, m, chunk);
    g.A = B.X[x0]; g.lda = L.ld_m; g.a_bs = B.x_bs;
    g.B = B.X[x0]; g.ldb = L.ld_m; g.b_bs = B.x_bs; g.b_kmajor = 1;
    g.in_dtype = xdt;
    g.D = R; g.ldd = L.ld_n; g.d_bs = B.s_bs; g.d_dtype = gdt;
    g.scale = B.inv; g.scale_pow = raw ? 2 : 0;
    g.symmetric = 1;
    return gemm(c, g);
  };
  auto sq = [&](GemmDesc& g, const void* A, const void* Bop, int b_kmajor, void* D, int ddt) {
    g = desc(n, n, n, chunk);
    g.A = A; g.lda = L.ld_n; g.a_bs = B.s_bs;
    g.B = Bop; g.ldb = L.ld_n; g.b_bs = B.s_bs; g.b_kmajor = b_kmajor;
    g.in_dtype = gdt;
    g.D = D; g.ldd = L.ld_n; g.d_bs = B.s_bs; g.d_dtype = ddt;
  };
  auto apply = [&](int x_out, const UpdateSlots* upd) -> int {  // X[x_out] = f Q_acc X0
    GemmDesc g = desc(n, m, n, chunk);
    g.update = upd;
    g.A = Qbuf[q_acc]; g.lda = L.ld_n; g.a_bs = B.s_bs;
    g.B = B.X[x0]; g.ldb = L.ld_m; g.b_bs = B.x_bs; g.b_kmajor = 0;
    g.in_dtype = xdt;
    g.D = B.X[x_out]; g.ldd = L.ld_m; g.d_bs = B.x_bs; g.d_dtype = xdt;
    g.scale = B.inv; g.scale_pow = x0_raw ? 1 : 0;
    return gemm(c, g);
  };

  if ((rc = gram_of_x(x0_raw))) return rc;
  for (int k = 1; k <= K; ++k) {
    const float a = ns->coeffs[3 * (k - 1)], bb = ns->coeffs[3 * (k - 1) + 1], cc = ns->coeffs[3 * (k - 1) + 2];
    const bool last = k == K;
    const bool restart = restart_at(ns, k);
    const bool to_apply = last || restart;
    // Q = a I + b R + c R R, into a slot that is not Q_acc
    int qi = 0;
    while (qi == q_acc) ++qi;
    const int q_dt = (q_acc < 0 && to_apply) ? xdt : gdt;
    GemmDesc g;
    sq(g, R, R, 1, Qbuf[qi], q_dt);
    g.C = R; g.ldc = L.ld_n; g.c_bs = B.s_bs; g.c_dtype = gdt;
    g.c_acc = cc; g.c_in = bb; g.c_eye = a;
    g.symmetric = 1;
    if ((rc = gemm(c, g))) return rc;
    if (q_acc < 0) {
      q_acc = qi;
    } else {
      // Q_acc <- Q Q_acc, a full product.  It is symmetric in exact arithmetic
      // (every Q_k is a polynomial in R_0), but mirroring its upper triangle
      // makes its rounding error wholly symmetric, and that part moves the
      // result: in an fp16 emulation of the stabilised form on log-uniform
      // spectra the mirrored product raised the error by ~19 %.
      int ni = 0;
      while (ni == q_acc || ni == qi) ++ni;
      const int n_dt = to_apply ? xdt : gdt;
      sq(g, Qbuf[qi], Qbuf[q_acc], 0, Qbuf[ni], n_dt);
      if ((rc = gemm(c, g))) return rc;
      q_acc = ni;
    }
    if (last) break;
    if (restart) {
      const int x_new = 1 - x0;
      if ((rc = apply(x_new, nullptr))) return rc;
      x0 = x_new;
      x0_raw = false;
      if ((rc = gram_of_x(false))) return rc;
      q_acc = -1;
    } else {
      // R <- Q R Q  as T = Q R, R = T Q.  Both are symmetric in exact
      // arithmetic (Q is a polynomial in R).  R is formed on the upper triangle
      // and mirrored, which is required: the next Q takes R R^T (SYRK form),
      // which equals R R only for an exactly symmetric R; a rounding-level
      // antisymmetric part of R would otherwise enter Q through R R^T - R R and
      // grow with every iteration.  T stays a full product: mirroring it, like
      // mirroring Q Q_acc, raised the emulated fp16 error by ~20 %.
      sq(g, Qbuf[qi], R, 0, T, gdt);
      if ((rc = gemm(c, g))) return rc;
      sq(g, T, Qbuf[qi], 0, R, gdt);
      g.symmetric = 1;
      if ((rc = gemm(c, g))) return rc;
    }
  }
  const int x_out = 1 - x0;
  if ((rc = apply(x_out, update))) return rc;
  *out_x = x_out;
  return 0;
}

// Host-side slot table of the fused update (about 7 KB): one per host thread,
// reused for every chunk; its contents are copied into the kernel parameters
// at launch, so reuse after the launch call is safe.
UpdateSlots& slots_storage() {
  thread_local UpdateSlots slots;
  return slots;
}

// MUON_CHAIN=1: 16-bit chains whose products all run on the paired-CTA kernel
// go out as one persistent launch per (up to 24) products, with per-matrix
// dependency counters in place of launch boundaries.  Off by default: on one
// B200 it measured 4-5 % slower than the separate launches, which overlap
// through programmatic dependent launch (Kimi-K2 step 426 against 408 ms, MoE
// 21.2 against 20.1 ms, dense 6.2 against 5.9 ms, same box).
bool chain_enabled() {
  static const bool on = [] {
    const char* e = getenv("MUON_CHAIN");
    return e && e[0] == '1';
  }();
  return on;
}

// run_chain in one of two ways: product by product, or (chain mode) the same
// products recorded and then launched as whole-chain segments.
int run_chain_launch(const Ctx& c, const Layout& L, const Bufs& B, int chunk, const muon_ns_params* ns,
                     bool prescaled, int* out_x, int* out_dtype, const UpdateSlots* update) {
  const bool chain = chain_enabled() && ns->compute_dtype != MUON_FP32 && gemm_tc_paired(L.n);
  if (!chain) return run_chain(c, L, B, chunk, ns, prescaled, out_x, out_dtype, update);
  std::vector<GemmDesc> prods;
  Ctx rc = c;
  rc.record = &prods;
  int rv = run_chain(rc, L, B, chunk, ns, prescaled, out_x, out_dtype, update);
  if (rv) return rv;
  const bool prof = profiler().on;
  for (size_t first = 0; first < prods.size(); first += kChainMaxProducts) {
    const int n = (int)std::min<size_t>(kChainMaxProducts, prods.size() - first);
    if (*c.used >= c.n_counters) return (int)cudaErrorInvalidValue;
    int* counter = c.counters + (*c.used)++;
    double flops = 0.0, exec = 0.0, bytes = 0.0;
    if (prof) {
      for (int i = 0; i < n; ++i) {
        const GemmDesc& g = prods[first + i];
        flops += 2.0 * g.M * g.N * (double)g.K * g.batch;
        exec += gemm_tc_exec_flops(g);
        bytes += ((double)g.M * g.K * 2 + (double)g.N * g.K * 2 + (double)g.M * g.N * 2 +
                  (g.C ? (double)g.M * g.N * 2 : 0.0)) * g.batch;
      }
    }
    ProfScope ps(kProfChain, flops, bytes, c.s, exec);
    rv = gemm_chain(prods.data() + first, n, counter, B.done + first * (size_t)chunk, c.err, c.s);
    if (rv) return rv;
  }
  return 0;
}

// ------------------------------------------------------------------ driver
struct SrcView {      // what the pack / unpack kernels need for one caller group
  int rows, cols;
  int src_dtype, dst_dtype;
  const void* const* src;
  float* const* mom;
  void* const* dst;
};

int run_batches(const std::vector<Batch>& batches, const std::vector<SrcView>& views, const std::vector<long long>& first_index,
                const muon_ns_params* ns, bool update, float mu, int nesterov, float lr, float wd, float scale_coef,
                void* ws, size_t ws_bytes, int* status, cudaStream_t s) {
  for (const Batch& bt : batches) {
    const Layout L = make_layout(bt.n, bt.m, ns);
    if (ws_bytes < chunk_bytes(L, 1)) return MUON_ERR_WORKSPACE;
    const bool fuse = update && ns->compute_dtype != MUON_FP32 && fused_update_enabled() && gemm_tc_paired(L.n);
    int chunk_cap = (int)std::min<size_t>((size_t)bt.total, (ws_bytes - L.fixed) / L.per_matrix);
    if (fuse) chunk_cap = std::min(chunk_cap, UpdateSlots::kMax);
    // slots are assigned in segment order; walk them chunk by chunk
    int seg_i = 0, seg_off = 0;
    int done = 0;
    while (done < bt.total) {
      const int chunk = std::min(chunk_cap, bt.total - done);
      const Bufs B = carve(L, chunk, ws);
      if (cudaMemsetAsync(B.err, 0, B.zero_bytes, s) != cudaSuccess) return MUON_ERR_CUDA;
      // pieces of segments covering slots [done, done + chunk)
      struct Piece { int group, first, count, slot; };
      std::vector<Piece> pieces;
      {
        int slot = 0, si = seg_i, so = seg_off;
        while (slot < chunk) {
          const Seg& sg = bt.segs[si];
          int take = std::min(sg.count - so, chunk - slot);
          int left = take, f = sg.first + so, sl = slot;
          while (left > 0) {
            const int t = std::min(left, SegmentPtrs::kMax);
            pieces.push_back(Piece{sg.group, f, t, sl});
            f += t; sl += t; left -= t;
          }
          slot += take;
          so += take;
          if (so == sg.count) { ++si; so = 0; }
        }
        seg_i = si;
        seg_off = so;
      }
      // fp16 chains take X0 normalised and rounded once to fp16: a sums-of-squares
      // pass, the norm, then the storing pass with the scale.  Otherwise one pass
      // stores the raw U (bf16 or fp32) and the chain applies the norm.
      const int cdt = chain_dtype(ns);
      const bool prescale = cdt == MUON_FP16;
      const int pack_dt = ns->compute_dtype == MUON_FP32 ? MUON_FP32 : (prescale ? MUON_FP16 : MUON_BF16);
      auto launch_pieces = [&](int pass) {
        for (const Piece& pc : pieces) {
          const SrcView& v = views[pc.group];
          SegmentPtrs ptrs;
          for (int i = 0; i < pc.count; ++i) {
            ptrs.src[i] = v.src[pc.first + i];
            ptrs.mom[i] = v.mom ? v.mom[pc.first + i] : nullptr;
            ptrs.dst[i] = nullptr;
          }
          PackArgs a{};
          a.rows = v.rows; a.cols = v.cols; a.count = pc.count;
          a.src_dtype = v.src_dtype; a.x_dtype = pack_dt;
          a.momentum_mode = update ? 1 : 0; a.mu = mu; a.nesterov = nesterov;
          a.x = reinterpret_cast<char*>(B.X[0]) + (size_t)pc.slot * B.x_bs * L.x_es;
          a.ld_x = L.ld_m; a.x_batch_stride = B.x_bs;
          a.partials = B.partials + (size_t)pc.slot * L.tiles;
          a.partial_stride = L.tiles;
          a.pass = pass;
          a.scale = B.inv + pc.slot;
          const double elems = (double)v.rows * v.cols * pc.count;
          const double in_b = dtype_size(v.src_dtype) + (update ? 4 : 0);
          const double out_b = pass == 1 ? 0.0 : L.x_es + (update ? 4 : 0);
          ProfScope ps(kProfPack, 0.0, elems * (in_b + out_b), s);
          launch_pack(a, ptrs, s);
        }
      };
      launch_pieces(prescale ? 1 : 0);
      {
        ProfScope ps(kProfNorm, 0.0, (double)chunk * L.tiles * 4 + chunk * 4.0, s);
        launch_norm(B.partials, L.tiles, L.tiles, chunk, ns->eps, B.inv, s);
      }
      if (prescale) launch_pieces(2);
      if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
      int used = 0;
      PlaneCache planes;
      if (L.tf32) {
        planes.n = 3;
        for (int i = 0; i < 3; ++i) {
          planes.hi[i] = B.planes[i][0];
          planes.lo[i] = B.planes[i][1];
          planes.cap[i] = B.plane_elems[i];
        }
      }
      Ctx ctx{ns->compute_dtype, s, B.err, B.counters, L.n_counters, &used};
      ctx.planes = &planes;
      int xi = 0, out_dt = pack_dt;
      if (fuse) {
        UpdateSlots& us = slots_storage();
        us.decay = 1.f - lr * wd;
        us.step = lr * scale_coef * std::sqrt((float)bt.m);  // max(rows, cols) = m for every matrix of the batch
        us.status = status;
        for (const Piece& pc : pieces) {
          const SrcView& v = views[pc.group];
          for (int i = 0; i < pc.count; ++i) {
            us.w[pc.slot + i] = v.dst[pc.first + i];
            us.status_idx[pc.slot + i] = (int)(first_index[pc.group] + pc.first + i);
            us.kind[pc.slot + i] = (unsigned char)((v.rows > v.cols ? 1 : 0) | (v.dst_dtype << 1));
          }
        }
        if (run_chain_launch(ctx, L, B, chunk, ns, prescale, &xi, &out_dt, &us) != 0) return MUON_ERR_CUDA;
        if (status)
          for (const Piece& pc : pieces) {
            ProfScope ps(kProfStatus, 0.0, pc.count * 8.0, s);
            launch_status_or(status + first_index[pc.group] + pc.first, pc.count, B.err, s);
          }
        if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
        done += chunk;
        continue;
      }
      if (run_chain_launch(ctx, L, B, chunk, ns, prescale, &xi, &out_dt, nullptr) != 0) return MUON_ERR_CUDA;
      for (const Piece& pc : pieces) {
        const SrcView& v = views[pc.group];
        SegmentPtrs ptrs;
        for (int i = 0; i < pc.count; ++i) {
          ptrs.src[i] = nullptr;
          ptrs.mom[i] = nullptr;
          ptrs.dst[i] = v.dst[pc.first + i];
        }
        UnpackArgs u{};
        u.rows = v.rows; u.cols = v.cols; u.count = pc.count;
        u.dst_dtype = v.dst_dtype; u.x_dtype = out_dt;
        u.update_mode = update ? 1 : 0;
        u.decay = 1.f - lr * wd;
        u.step = lr * scale_coef * std::sqrt((float)std::max(v.rows, v.cols));
        u.x = reinterpret_cast<const char*>(B.X[xi]) + (size_t)pc.slot * B.x_bs * L.x_es;
        u.ld_x = L.ld_m; u.x_batch_stride = B.x_bs;
        u.status = status ? status + first_index[pc.group] + pc.first : nullptr;
        u.chunk_err = B.err;
        const double elems = (double)v.rows * v.cols * pc.count;
        ProfScope ps(kProfUnpack, 0.0, elems * (L.x_es + dtype_size(v.dst_dtype) * (update ? 2 : 1)), s);
        launch_unpack(u, ptrs, s);
      }
      if (cudaGetLastError() != cudaSuccess) return MUON_ERR_CUDA;
      done += chunk;
    }
  }
  return MUON_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15) == 0; }

int check_groups(const muon_group* groups, int n_groups, const muon_hparams* hp, long long* total) {
  if (!groups || n_groups <= 0 || !hp) return MUON_ERR_INVALID;
  if (!ns_params_ok(&hp->ns)) return MUON_ERR_INVALID;
  if (!std::isfinite(hp->lr) || !std::isfinite(hp->momentum) || !std::isfinite(hp->weight_decay) ||
      !std::isfinite(hp->scale_coef))
    return MUON_ERR_INVALID;
  long long t = 0;
  for (int g = 0; g < n_groups; ++g) {
    const muon_group& G = groups[g];
    if (G.rows <= 0 || G.cols <= 0 || G.count < 0) return MUON_ERR_INVALID;
    if ((long long)G.rows * G.cols > (1LL << 34)) return MUON_ERR_INVALID;
    if (!dtype_ok(G.w_dtype) || !dtype_ok(G.g_dtype)) return MUON_ERR_UNSUPPORTED;
    if (G.count > 0 && (!G.W || !G.G || !G.M)) return MUON_ERR_INVALID;
    for (int i = 0; i < G.count; ++i) {
      if (!G.W[i] || !G.G[i] || !G.M[i]) return MUON_ERR_INVALID;
      if (!aligned16(G.W[i]) || !aligned16(G.G[i]) || !aligned16(G.M[i])) return MUON_ERR_INVALID;
    }
    t += G.count;
  }
  *total = t;
  return MUON_OK;
}

size_t ws_for(const std::vector<Batch>& batches, const muon_ns_params* ns, bool full) {
  size_t best = 0;
  for (const Batch& b : batches) {
    const Layout L = make_layout(b.n, b.m, ns);
    best = std::max(best, chunk_bytes(L, full ? b.total : 1));
  }
  return best;
}

double flops_of(int rows, int cols, const muon_ns_params* ns) {
  const double n = std::min(rows, cols), m = std::max(rows, cols);
  const double sq = 2.0 * m * n * n, cube = 2.0 * n * n * n;
  const int K = ns->iters;
  if (ns->mode == MUON_NS_STANDARD) {
    double per = sq + sq;  // X X^T and B X
    double total = 0;
    for (int k = 0; k < K; ++k) total += per + (ns->coeffs[3 * k + 2] != 0.f ? cube : 0.0);
    return total;
  }
  // Gram forms: R0, per iteration R^2 (+ Q Q_acc unless Q_acc = I), R update
  // (2 products) or the restart pair, final apply
  double total = sq;
  bool fresh = true;
  for (int k = 1; k <= K; ++k) {
    total += cube;
    if (!fresh) total += cube;
    fresh = false;
    if (k == K) break;
    if (restart_at(ns, k)) {
      total += 2 * sq;
      fresh = true;
    } else {
      total += 2 * cube;
    }
  }
  return total + sq;
}

}  // namespace

extern "C" {

size_t muon_workspace_size(const muon_group* groups, int n_groups, const muon_hparams* hp) {
  long long total = 0;
  if (check_groups(groups, n_groups, hp, &total) != MUON_OK) return 0;
  return ws_for(plan_groups(groups, n_groups), &hp->ns, true);
}

size_t muon_workspace_min(const muon_group* groups, int n_groups, const muon_hparams* hp) {
  long long total = 0;
  if (check_groups(groups, n_groups, hp, &total) != MUON_OK) return 0;
  return ws_for(plan_groups(groups, n_groups), &hp->ns, false);
}

int muon_step(const muon_group* groups, int n_groups, const muon_hparams* hp, void* ws, size_t ws_bytes,
              int* status_per_matrix, void* stream) {
  long long total = 0;
  int rc = check_groups(groups, n_groups, hp, &total);
  if (rc != MUON_OK) return rc;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return MUON_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  std::vector<Batch> batches = plan_groups(groups, n_groups);
  if (ws_bytes < ws_for(batches, &hp->ns, false)) return MUON_ERR_WORKSPACE;
  std::vector<SrcView> views(n_groups);
  std::vector<long long> first(n_groups);
  long long acc = 0;
  for (int g = 0; g < n_groups; ++g) {
    views[g] = SrcView{groups[g].rows, groups[g].cols, groups[g].g_dtype, groups[g].w_dtype,
                       groups[g].G, groups[g].M, groups[g].W};
    first[g] = acc;
    acc += groups[g].count;
  }
  if (status_per_matrix && total > 0 && cudaMemsetAsync(status_per_matrix, 0, (size_t)total * sizeof(int), s) != cudaSuccess)
    return MUON_ERR_CUDA;
  return run_batches(batches, views, first, &hp->ns, true, hp->momentum, hp->nesterov, hp->lr, hp->weight_decay,
                     hp->scale_coef, ws, ws_bytes, status_per_matrix, s);
}

size_t muon_ns_workspace_size(int count, int rows, int cols, const muon_ns_params* ns) {
  if (count <= 0 || rows <= 0 || cols <= 0 || !ns_params_ok(ns)) return 0;
  const Layout L = make_layout(std::min(rows, cols), std::max(rows, cols), ns);
  return chunk_bytes(L, count);
}

int muon_ns_batched(void* const* X, int count, int rows, int cols, int dtype, const muon_ns_params* ns, void* ws,
                    size_t ws_bytes, int* status_per_matrix, void* stream) {
  if (!X || count < 0 || rows <= 0 || cols <= 0 || !ns_params_ok(ns)) return MUON_ERR_INVALID;
  if ((long long)rows * cols > (1LL << 34)) return MUON_ERR_INVALID;
  if (!dtype_ok(dtype)) return MUON_ERR_UNSUPPORTED;
  if (count == 0) return MUON_OK;
  for (int i = 0; i < count; ++i)
    if (!X[i] || !aligned16(X[i])) return MUON_ERR_INVALID;
  if (!ws || (reinterpret_cast<uintptr_t>(ws) & (kAlign - 1))) return MUON_ERR_INVALID;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  Batch b{std::min(rows, cols), std::max(rows, cols), {Seg{0, 0, count}}, count};
  std::vector<Batch> batches{b};
  if (ws_bytes < ws_for(batches, ns, false)) return MUON_ERR_WORKSPACE;
  std::vector<SrcView> views{SrcView{rows, cols, dtype, dtype, const_cast<const void* const*>(X), nullptr, X}};
  std::vector<long long> first{0};
  if (status_per_matrix && cudaMemsetAsync(status_per_matrix, 0, (size_t)count * sizeof(int), s) != cudaSuccess)
    return MUON_ERR_CUDA;
  return run_batches(batches, views, first, ns, false, 0.f, 0, 0.f, 0.f, 0.f, ws, ws_bytes, status_per_matrix, s);
}

double muon_ns_flops(int rows, int cols, const muon_ns_params* ns) {
  if (rows <= 0 || cols <= 0 || !ns_params_ok(ns)) return 0.0;
  return flops_of(rows, cols, ns);
}

int muon_profile_begin(void) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  for (auto& r : P.recs) { cudaEventDestroy(r.a); cudaEventDestroy(r.b); }
  P.recs.clear();
  P.on = true;
  return MUON_OK;
}

int muon_profile_end(muon_profile_entry* out, int max_entries) {
  Profiler& P = profiler();
  std::lock_guard<std::mutex> g(P.mu);
  P.on = false;
  muon_profile_entry acc[kProfKinds];
  for (int k = 0; k < kProfKinds; ++k) acc[k] = muon_profile_entry{kProfNames[k], 0, 0.0, 0.0, 0.0, 0.0};
  int rc = MUON_OK;
  for (auto& r : P.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) rc = MUON_ERR_CUDA;
    acc[r.kind].launches += 1;
    acc[r.kind].ms += ms;
    acc[r.kind].flops += r.flops;
    acc[r.kind].exec_flops += r.exec_flops;
    acc[r.kind].bytes += r.bytes;
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  P.recs.clear();
  if (rc != MUON_OK) return rc;
  if (!out && max_entries > 0) return MUON_ERR_INVALID;
  int n = 0;
  for (int k = 0; k < kProfKinds && n < max_entries; ++k)
    if (acc[k].launches) out[n++] = acc[k];
  return n;
}

const char* muon_status_string(int code) {
  switch (code) {
    case MUON_OK: return "ok";
    case MUON_ERR_INVALID: return "invalid argument (null or misaligned pointer, bad shape, count or parameter)";
    case MUON_ERR_UNSUPPORTED: return "unsupported dtype";
    case MUON_ERR_WORKSPACE: return "workspace too small";
    case MUON_ERR_CUDA: return "CUDA launch or tensor-map encode failed";
    case MUON_STATUS_NONFINITE: return "non-finite values in the orthogonalised matrix";
    case MUON_STATUS_TIMEOUT: return "a device-side wait timed out; the matrix was not finished";
    case MUON_STATUS_NONFINITE | MUON_STATUS_TIMEOUT: return "non-finite values and a device-side wait timeout";
    default: return "unknown code";
  }
}

}  // extern "C"
