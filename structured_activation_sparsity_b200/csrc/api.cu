// Host side of the C ABI declared in include/sparsesam.h: argument validation, workspace carving,
// TMA descriptor encoding, launch tracing and the status word. Every GPU step runs in this
// library's kernels; nothing here computes on the host except the static pattern's integers.
#include <math.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "kernels.h"

namespace ss {

// Device status word written by bounded device waits that give up (see sparsesam_device_status).
__device__ int g_status = 0;
// A counter nothing increments unless the self-test asks for it (sparsesam_wait_selftest).
__device__ int g_selftest_counter = 0;

// One CTA of 32 threads; thread 0 runs one bounded wait that (which 0, 1) nobody satisfies or
// (which 2, 3) is satisfied before it starts: an mbarrier phase (0, 2) or a global counter (1, 3).
// No copy or MMA is in flight, so giving up leaves nothing behind.
__global__ void k_wait_selftest(int which, int* counter, int* status) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0;
    fence_barrier_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (which == 0 || which == 2) {
      if (which == 2) mbar_arrive(&bar);
      mbar_wait(&bar, 0, &abort_flag, status);
    } else {
      *counter = which == 3 ? 1 : 0;
      __threadfence();
      wait_counter_geq(counter, 1, &abort_flag, status);
      *counter = 0;
    }
  }
  __syncthreads();
}

namespace {

std::mutex g_mu;
std::atomic<uint64_t> g_launches{0};

// ---- per-device address of the status word ----------------------------------------------------
int* status_word() {
  static int* addr[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!addr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_status) != cudaSuccess) return nullptr;
    addr[dev] = static_cast<int*>(p);
  }
  return addr[dev];
}

// ---- launch tracing -----------------------------------------------------------------------------
struct TraceRec {
  const char* name;
  cudaEvent_t e0, e1;
  float ms;
};
std::vector<TraceRec> g_trace;
int g_trace_used = 0;
bool g_tracing = false;

template <class F>
cudaError_t traced(const char* name, cudaStream_t st, F&& f) {
  TraceRec* rec = nullptr;
  if (g_tracing && g_trace_used < (int)g_trace.size()) {
    rec = &g_trace[g_trace_used++];
    rec->name = name;
    cudaEventRecord(rec->e0, st);
  }
  cudaError_t e = f();
  if (rec) cudaEventRecord(rec->e1, st);
  g_launches.fetch_add(1, std::memory_order_relaxed);
  return e;
}

// ---- tensor maps --------------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// bf16 tensor of `mats` matrices [rows, inner] with rows `row_bytes` apart; box [box_rows, box_inner].
// `rank` must match the dimensionality of the kernel's TMA instruction (2: one matrix, 3: a stack).
bool encode_bf16(CUtensorMap* m, cuuint32_t rank, const void* base, uint64_t inner, uint64_t rows,
                 uint64_t mats, uint64_t row_bytes, uint32_t box_inner, uint32_t box_rows,
                 CUtensorMapSwizzle sw) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {inner, rows, mats};
  cuuint64_t strides[2] = {row_bytes, row_bytes * rows};
  cuuint32_t box[3] = {box_inner, box_rows, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  if (rank != 2 && rank != 3) return false;
  if (rank == 2 && mats != 1) return false;
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// ---- geometry -----------------------------------------------------------------------------------
struct Geo {
  int B, Hg, Wg, T;      // images, grid, tokens per image
  int window_mode, ws, wpr, windows;
  int U, N;              // attention units, tokens per unit
};

int geometry(const ss_cfg* c, Geo* g) {
  if (!c) return SS_EINVAL;
  if (c->batch < 1 || c->grid_h < 1 || c->grid_w < 1) return SS_EINVAL;
  if (c->mode != SS_GLOBAL && c->mode != SS_WINDOW) return SS_EINVAL;
  if (c->mode == SS_WINDOW && c->window < 1) return SS_EINVAL;
  if (!(c->density > 0.0 && c->density <= 1.0)) return SS_EINVAL;   // also rejects NaN
  if ((int64_t)c->grid_h * c->grid_w > (1 << 24) || c->batch > (1 << 20)) return SS_EUNSUPPORTED;
  g->B = c->batch;
  g->Hg = c->grid_h;
  g->Wg = c->grid_w;
  g->T = c->grid_h * c->grid_w;
  g->window_mode = c->mode == SS_WINDOW;
  if (g->window_mode) {
    g->ws = c->window;
    g->wpr = (c->grid_w + c->window - 1) / c->window;
    g->windows = g->wpr * ((c->grid_h + c->window - 1) / c->window);
    g->N = c->window * c->window;
  } else {
    g->ws = 0;
    g->wpr = 1;
    g->windows = 1;
    g->N = g->T;
  }
  if ((int64_t)g->B * g->windows > (1 << 24)) return SS_EUNSUPPORTED;
  g->U = g->B * g->windows;
  return SS_OK;
}

int pattern_of(const ss_cfg* c, const Geo& g, ss_pattern* p) {
  if (g.N % kStripes != 0) return SS_EUNSUPPORTED;
  const int L = g.N / kStripes;
  const int b = block_size_for(L);
  if (b == 0) return SS_EUNSUPPORTED;
  const int nb = L / b;
  const int W = choose_band(nb, kGlobalBlocks, c->density);
  p->units = g.U;
  p->unit_tokens = g.N;
  p->stripes = kStripes;
  p->L = L;
  p->b = b;
  p->nb = nb;
  p->W = W;
  p->g = kGlobalBlocks;
  p->nnz = pattern_nnz(W, nb, kGlobalBlocks);
  p->keep = keep_count(c->density, g.T);
  p->rho = (double)p->nnz / (double)(nb * nb);
  return SS_OK;
}

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }
inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int cuda_err(cudaError_t e) { return e == cudaSuccess ? SS_OK : SS_ECUDA; }

// The GEMM and attention work splits are planned for the B200's 148 SMs, so workspace sizes do
// not depend on the device a call runs on; launches use min(units, the device's SMs) CTAs.
constexpr int kPlanSMs = 148;

// The attention workspace: the gathered Q, K and V ([U*heads, N, dh] bf16 each); for the pair
// kernel its permuted output Op (the same layout), and, when it splits pairs into pieces, its
// per-piece partials.
struct AttnLayout {
  AttnParams ap;     // geometry and plan fields filled; perm, out, sms by the launch
  AttnPlan plan;
  size_t one;        // bytes of one gathered array (256-byte multiple)
  size_t operm, partial, total;   // byte offsets, total size
};

int attn_layout(const ss_cfg* c, const Geo& g, AttnLayout* L, bool force_pair = false) {
  ss_pattern p;
  int rc = pattern_of(c, g, &p);
  if (rc) return rc;
  AttnParams& ap = L->ap;
  ap = AttnParams{};
  ap.U = g.U;
  ap.N = g.N;
  ap.heads = c->heads;
  ap.L = p.L;
  ap.b = p.b;
  ap.nb = p.nb;
  ap.W = p.W;
  ap.g = p.g;
  ap.scale_log2 = (float)(1.4426950408889634 / sqrt((double)c->head_dim));
  L->plan = attn_plan(ap, c->head_dim, kPlanSMs, force_pair);
  ap.whole = L->plan.whole;
  ap.tail_split = L->plan.tail_split;
  L->one = align256((size_t)g.U * c->heads * g.N * c->head_dim * 2);
  L->operm = 3 * L->one;
  L->partial = L->operm + (L->plan.pair_kernel ? L->one : 0);
  L->total = L->partial + align256(L->plan.partial_bytes);
  return SS_OK;
}

struct MlpPlan {
  GemmPlan fc1, fc2;
  size_t xk, h, partial, counters, total;   // byte offsets/sizes inside the workspace
};

MlpPlan mlp_plan(const Geo& g, int K, int C, int hidden) {
  MlpPlan p;
  const int M = g.B * K;
  p.fc1 = gemm_plan(M, hidden, C, kPlanSMs);
  p.fc2 = gemm_plan(M, C, hidden, kPlanSMs);
  const size_t xk_bytes = align256((size_t)M * C * 2);
  const size_t h_bytes = align256((size_t)M * hidden * 2);
  const size_t part = align256(gemm_partial_bytes(p.fc1) > gemm_partial_bytes(p.fc2)
                                   ? gemm_partial_bytes(p.fc1)
                                   : gemm_partial_bytes(p.fc2));
  const int tiles = (p.fc1.m_tiles * p.fc1.n_tiles > p.fc2.m_tiles * p.fc2.n_tiles)
                        ? p.fc1.m_tiles * p.fc1.n_tiles
                        : p.fc2.m_tiles * p.fc2.n_tiles;
  const size_t cnt = part ? align256((size_t)tiles * 2 * 4) : 0;   // two counters per tile
  p.xk = 0;
  p.h = xk_bytes;
  p.partial = xk_bytes + h_bytes;
  p.counters = p.partial + part;
  p.total = p.counters + cnt;
  return p;
}

size_t rcmlp_ws_bytes(const Geo& g, int K, int C, int hidden) {
  return mlp_plan(g, K, C, hidden).total;
}

int sm_count() {
  static int cached[128] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 128) return kPlanSMs;
  if (!cached[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n < 1)
      n = kPlanSMs;
    cached[dev] = n;
  }
  return cached[dev];
}

}  // namespace
}  // namespace ss

using namespace ss;

extern "C" {

int sparsesam_pattern(const ss_cfg* cfg, ss_pattern* out) {
  if (!out) return SS_EINVAL;
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  return pattern_of(cfg, g, out);
}

int sparsesam_blocklist(const ss_cfg* cfg, int32_t* row_ptr, int32_t* col_idx, int32_t cap) {
  if (!row_ptr || !col_idx) return SS_EINVAL;
  ss_pattern p;
  int rc = sparsesam_pattern(cfg, &p);
  if (rc) return rc;
  if (cap < p.nnz) return SS_EINVAL;
  int n = 0;
  row_ptr[0] = 0;
  for (int a = 0; a < p.nb; ++a) {
    for (int ka = 0; ka < p.nb; ++ka)
      if (block_kept(a, ka, p.W, p.nb, p.g)) col_idx[n++] = ka;
    row_ptr[a + 1] = n;
  }
  return SS_OK;
}

int sparsesam_score(const ss_cfg* cfg, const float* lum, double* score, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (!lum || !score) return SS_EINVAL;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_err(traced("sobel_score", st, [&] {
    return launch_sobel_score(lum, score, g.B, g.Hg, g.Wg, st);
  }));
}

// S2 from given scores (score non-null, lum null) or S1 + S2 in one pass (lum non-null; the scores
// are computed from lum and written to score when it is non-null).
static int rank_path(const ss_cfg* cfg, const float* lum, const double* score, double* score_out,
                     int32_t* perm, int32_t* inv, int32_t* keep, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (!perm && !inv && !keep) return SS_EINVAL;
  ss_pattern p;
  if ((perm || inv) && (rc = pattern_of(cfg, g, &p))) return rc;
  if (g.N > kMaxRankTokens || g.T > kMaxRankTokens) return SS_EUNSUPPORTED;
  if (g.U > 65535) return SS_EUNSUPPORTED;
  const int K = keep_count(cfg->density, g.T);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (!g.window_mode) {
    return cuda_err(traced(lum ? "score_rank" : "stripe_rank", st, [&] {
      return launch_stripe_rank(score, lum, score_out, 0, g.B, g.Hg, g.Wg, 0, g.B, g.T, K, perm,
                                inv, keep, st);
    }));
  }
  if (perm || inv) {
    rc = cuda_err(traced(lum ? "score_rank_window" : "stripe_rank_window", st, [&] {
      return launch_stripe_rank(score, lum, score_out, 1, g.B, g.Hg, g.Wg, g.ws, g.U, g.N, 0, perm,
                                inv, nullptr, st);
    }));
    if (rc) return rc;
  }
  if (keep) {
    // The per-image keep ranking reads the scores: those the window pass just wrote, or the
    // caller's.
    const double* sc = lum ? score_out : score;
    rc = cuda_err(traced("keep_rank", st, [&] {
      return launch_stripe_rank(sc, nullptr, nullptr, 0, g.B, g.Hg, g.Wg, 0, g.B, g.T, K, nullptr,
                                nullptr, keep, st);
    }));
  }
  return rc;
}

int sparsesam_perm(const ss_cfg* cfg, const double* score, int32_t* perm, int32_t* inv,
                   int32_t* keep, void* stream) {
  if (!score) return SS_EINVAL;
  return rank_path(cfg, nullptr, score, nullptr, perm, inv, keep, stream);
}

int sparsesam_score_perm(const ss_cfg* cfg, const float* lum, double* score, int32_t* perm,
                         int32_t* inv, int32_t* keep, void* stream) {
  if (!lum || !score) return SS_EINVAL;
  return rank_path(cfg, lum, nullptr, score, perm, inv, keep, stream);
}

int sparsesam_random_perm(const ss_cfg* cfg, uint64_t seed, double* score, int32_t* perm,
                          int32_t* inv, int32_t* keep, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (!score || (!perm && !inv && !keep)) return SS_EINVAL;
  if (perm || inv) {
    ss_pattern p;
    if ((rc = pattern_of(cfg, g, &p))) return rc;
  }
  if (g.N > kMaxRankTokens || g.T > kMaxRankTokens || g.U > 65535) return SS_EUNSUPPORTED;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = cuda_err(traced("random_score", st, [&] {
    return launch_random_score(score, (long long)g.B * g.T, seed, st);
  }));
  if (rc) return rc;
  return rank_path(cfg, nullptr, score, nullptr, perm, inv, keep, stream);
}

int sparsesam_keep_by_update(const ss_cfg* cfg, const uint16_t* delta, int32_t C, int32_t K,
                             double* mag, int32_t* keep, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (!delta || !mag || !keep || C < 1 || K < 0 || K > g.T) return SS_EINVAL;
  if (C % 8 != 0) return SS_EUNSUPPORTED;
  if (!aligned(delta, 16)) return SS_EINVAL;
  if (g.T > kMaxRankTokens) return SS_EUNSUPPORTED;
  if (K == 0) return SS_OK;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  rc = cuda_err(traced("update_magnitude", st, [&] {
    return launch_update_magnitude(delta, mag, (long long)g.B * g.T, C, st);
  }));
  if (rc) return rc;
  return cuda_err(traced("keep_rank", st, [&] {
    return launch_stripe_rank(mag, nullptr, nullptr, 0, g.B, g.Hg, g.Wg, 0, g.B, g.T, K, nullptr,
                              nullptr, keep, st);
  }));
}

size_t sparsesam_attn_workspace(const ss_cfg* cfg) {
  Geo g;
  AttnLayout L;
  if (geometry(cfg, &g) || cfg->heads < 1 || cfg->head_dim < 1 || attn_layout(cfg, g, &L))
    return 0;
  return L.total;
}

// Argument checks of the attention step (also for the whole-block path); fills the pattern.
static int attn_check(const ss_cfg* cfg, const Geo& g, const uint16_t* q, const uint16_t* k,
                      const uint16_t* v, const int32_t* perm, const uint16_t* out, ss_pattern* p) {
  if (cfg->heads < 1 || cfg->head_dim < 1) return SS_EINVAL;
  if (!q || !k || !v || !perm || !out) return SS_EINVAL;
  if (cfg->head_dim != 64 && cfg->head_dim != 80) return SS_EUNSUPPORTED;
  int rc = pattern_of(cfg, g, p);
  if (rc) return rc;
  const int heads = cfg->heads, dh = cfg->head_dim;
  if ((int64_t)g.U * heads > 65535) return SS_EUNSUPPORTED;
  if ((int64_t)g.U * g.N * heads * (dh / 8) >= (int64_t)1 << 31) return SS_EUNSUPPORTED;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(out, 16))
    return SS_EINVAL;
  return SS_OK;
}

// The Q/K/V gather into ws (laid out as attn_layout describes).
static int gather_launch(const Geo& g, int heads, int dh, const AttnLayout& L, const uint16_t* q,
                         const uint16_t* k, const uint16_t* v, const int32_t* perm, uint8_t* ws,
                         int* status, cudaStream_t st) {
  return cuda_err(traced("gather_qkv", st, [&] {
    return launch_gather_qkv(q, k, v, perm, reinterpret_cast<uint16_t*>(ws),
                             reinterpret_cast<uint16_t*>(ws + L.one),
                             reinterpret_cast<uint16_t*>(ws + 2 * L.one), g.U, g.N, heads, dh,
                             L.ap.b, status, st);
  }));
}

// The attention over the gathered Q, K, V in ws (laid out as attn_layout describes).
// rel: the relative-position fields of AttnParams (null: none).
static int attn_launch(const ss_cfg* cfg, const Geo& g, const AttnLayout& L, uint8_t* ws,
                       const int32_t* perm, uint16_t* out, int* status, cudaStream_t st,
                       float2* ml = nullptr, const AttnParams* rel = nullptr,
                       const CUtensorMap* te = nullptr) {
  const int heads = cfg->heads, dh = cfg->head_dim;
  const uint16_t* bufs[3] = {reinterpret_cast<uint16_t*>(ws),
                             reinterpret_cast<uint16_t*>(ws + L.one),
                             reinterpret_cast<uint16_t*>(ws + 2 * L.one)};
  uint16_t* operm = reinterpret_cast<uint16_t*>(ws + L.operm);
  CUtensorMap tm[7];   // Q, K, V; Q and K tails; Op and its tail (pair kernel)
  const uint64_t mats = (uint64_t)g.U * heads;
  for (int i = 0; i < 3; ++i)
    if (!encode_bf16(&tm[i], 3, bufs[i], dh, g.N, mats, (uint64_t)dh * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return SS_ECUDA;
  for (int i = 0; i < 2; ++i)   // columns 64..79 of Q and K at head dim 80
    if (dh == 80 && !encode_bf16(&tm[3 + i], 3, bufs[i], dh, g.N, mats, (uint64_t)dh * 2, 16, 128,
                                 CU_TENSOR_MAP_SWIZZLE_32B))
      return SS_ECUDA;
  if (L.plan.pair_kernel) {
    if (!encode_bf16(&tm[5], 3, operm, dh, g.N, mats, (uint64_t)dh * 2, 64, 128,
                     CU_TENSOR_MAP_SWIZZLE_128B))
      return SS_ECUDA;
    if (dh == 80 && !encode_bf16(&tm[6], 3, operm, dh, g.N, mats, (uint64_t)dh * 2, 16, 128,
                                 CU_TENSOR_MAP_SWIZZLE_32B))
      return SS_ECUDA;
  }
  AttnParams ap = L.ap;
  ap.perm = perm;
  ap.out = out;
  ap.sms = sm_count();
  ap.partial = reinterpret_cast<float*>(ws + L.partial);
  ap.operm = operm;
  ap.ml = ml;
  if (rel) {
    ap.rel_tab = rel->rel_tab;
    ap.rel_ld = rel->rel_ld;
    ap.rel_h = rel->rel_h;
    ap.rel_w = rel->rel_w;
    ap.rel_ksteps = rel->rel_ksteps;
  }
  int rc = cuda_err(traced("attn", st, [&] {
    return launch_attn(&tm[0], &tm[1], &tm[2], &tm[3], &tm[4], &tm[5], &tm[6], ap, dh, status,
                       st, te);
  }));
  if (rc || !L.plan.pair_kernel) return rc;
  if (L.plan.tail_split > 1 &&
      (rc = cuda_err(traced("merge_pieces", st, [&] { return launch_merge_pieces(ap, dh, st); }))))
    return rc;
  return cuda_err(traced("unpermute_out", st, [&] {
    return launch_unpermute_out(operm, perm, out, g.U, g.N, heads, dh, ap.b, status, st);
  }));
}

int sparsesam_attn(const ss_cfg* cfg, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const int32_t* perm, uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  ss_pattern p;
  if ((rc = attn_check(cfg, g, q, k, v, perm, out, &p))) return rc;
  AttnLayout L;
  if ((rc = attn_layout(cfg, g, &L))) return rc;
  if (!ws || !aligned(ws, 256) || ws_bytes < L.total) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = gather_launch(g, cfg->heads, cfg->head_dim, L, q, k, v, perm, wsb, status, st)))
    return rc;
  return attn_launch(cfg, g, L, wsb, perm, out, status, st);
}

int sparsesam_attn_gathered(const ss_cfg* cfg, const void* ws, size_t ws_bytes,
                            const int32_t* perm, uint16_t* out, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  ss_pattern p;
  // The checks of sparsesam_attn, with the workspace standing in for q, k and v.
  if ((rc = attn_check(cfg, g, static_cast<const uint16_t*>(ws), static_cast<const uint16_t*>(ws),
                       static_cast<const uint16_t*>(ws), perm, out, &p)))
    return rc == SS_EINVAL && !ws ? SS_EWORKSPACE : rc;
  AttnLayout L;
  if ((rc = attn_layout(cfg, g, &L))) return rc;
  if (!aligned(ws, 256) || ws_bytes < L.total) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  return attn_launch(cfg, g, L, static_cast<uint8_t*>(const_cast<void*>(ws)), perm, out, status,
                     static_cast<cudaStream_t>(stream));
}

size_t sparsesam_rcmlp_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden, int32_t K) {
  Geo g;
  if (geometry(cfg, &g) || C < 1 || hidden < 1 || K < 0 || K > g.T) return 0;
  return rcmlp_ws_bytes(g, K, C, hidden);
}

// Argument checks of the RC-MLP step (also for the whole-block path).
static int rcmlp_check(const Geo& g, const uint16_t* x, int32_t C, int32_t hidden,
                       const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                       const uint16_t* b2, const int32_t* keep, int32_t K) {
  if (!x || !w1 || !w2 || !keep || C < 1 || hidden < 1 || K < 0 || K > g.T) return SS_EINVAL;
  if (C % 64 != 0 || hidden % 64 != 0) return SS_EUNSUPPORTED;
  if (!aligned(x, 16) || !aligned(w1, 16) || !aligned(w2, 16) || !aligned(b1, 16) ||
      !aligned(b2, 16))
    return SS_EINVAL;
  const int64_t M = (int64_t)g.B * K;
  if (M * (hidden > C ? hidden : C) >= ((int64_t)1 << 31) || (M + 127) / 128 > 65535)
    return SS_EUNSUPPORTED;
  return SS_OK;
}

// fc1 and fc2 over the gathered rows in ws (laid out as mlp_plan describes).
static int rcmlp_launch(const Geo& g, int K, uint16_t* x, int32_t C, int32_t hidden,
                        const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                        const uint16_t* b2, const int32_t* keep, uint8_t* wsb, int* status,
                        cudaStream_t st) {
  const MlpPlan plan = mlp_plan(g, K, C, hidden);
  const int64_t M = (int64_t)g.B * K;
  uint16_t* xk = reinterpret_cast<uint16_t*>(wsb + plan.xk);
  uint16_t* hbuf = reinterpret_cast<uint16_t*>(wsb + plan.h);
  float* partial = reinterpret_cast<float*>(wsb + plan.partial);
  int* counters = reinterpret_cast<int*>(wsb + plan.counters);
  const int sms = sm_count();
  CUtensorMap ta1, tb1, ta2, tb2;
  if (!encode_bf16(&ta1, 2, xk, C, M, 1, (uint64_t)C * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tb1, 2, w1, C, hidden, 1, (uint64_t)C * 2, 64, plan.fc1.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&ta2, 2, hbuf, hidden, M, 1, (uint64_t)hidden * 2, 64, 128,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tb2, 2, w2, hidden, C, 1, (uint64_t)hidden * 2, 64, plan.fc2.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return SS_ECUDA;
  GemmEpilogue e1 = {};
  e1.kind = 0;
  e1.bias = b1;
  e1.out = hbuf;
  int rc = cuda_err(traced("rcmlp_fc1", st, [&] {
    return launch_gemm(&ta1, &tb1, plan.fc1, (int)M, hidden, C, e1, partial, counters, sms, status,
                       st);
  }));
  if (rc) return rc;
  GemmEpilogue e2 = {};
  e2.kind = 1;
  e2.bias = b2;
  e2.x = x;
  e2.keep = keep;
  e2.K_per_image = K;
  e2.T = g.T;
  return cuda_err(traced("rcmlp_fc2", st, [&] {
    return launch_gemm(&ta2, &tb2, plan.fc2, (int)M, C, hidden, e2, partial, counters, sms, status,
                       st);
  }));
}

int sparsesam_rcmlp(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden, const uint16_t* w1,
                    const uint16_t* b1, const uint16_t* w2, const uint16_t* b2,
                    const int32_t* keep, int32_t K, void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if ((rc = rcmlp_check(g, x, C, hidden, w1, b1, w2, b2, keep, K))) return rc;
  if (K == 0) return SS_OK;   // an empty keep-set: every row is residual, nothing to launch
  const size_t need = rcmlp_ws_bytes(g, K, C, hidden);
  if (!ws || !aligned(ws, 256) || ws_bytes < need) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  const MlpPlan plan = mlp_plan(g, K, C, hidden);
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // The gather also zeroes the GEMMs' k-split counters (a memset here would stand between two
  // kernels and end their launch overlap).
  const int n_counters = (int)((plan.total - plan.counters) / sizeof(int));
  rc = cuda_err(traced("gather_rows", st, [&] {
    return launch_gather_rows(x, keep, reinterpret_cast<uint16_t*>(wsb + plan.xk), g.B, g.T, K, C,
                              reinterpret_cast<int*>(wsb + plan.counters), n_counters, status,
                              st);
  }));
  if (rc) return rc;
  return rcmlp_launch(g, K, x, C, hidden, w1, b1, w2, b2, keep, wsb, status, st);
}

size_t sparsesam_block_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden) {
  Geo g;
  AttnLayout L;
  if (geometry(cfg, &g) || cfg->heads < 1 || cfg->head_dim < 1 || C < 1 || hidden < 1 ||
      attn_layout(cfg, g, &L))
    return 0;
  return align256(L.total) + rcmlp_ws_bytes(g, keep_count(cfg->density, g.T), C, hidden);
}

int sparsesam_block(const ss_cfg* cfg, const float* lum, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, uint16_t* x, int32_t C, int32_t hidden, const uint16_t* w1,
                    const uint16_t* b1, const uint16_t* w2, const uint16_t* b2, double* score,
                    int32_t* perm, int32_t* inv, int32_t* keep, uint16_t* out, void* ws,
                    size_t ws_bytes, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (!lum || !score) return SS_EINVAL;
  ss_pattern p;
  if ((rc = attn_check(cfg, g, q, k, v, perm, out, &p))) return rc;
  const int K = keep_count(cfg->density, g.T);
  if ((rc = rcmlp_check(g, x, C, hidden, w1, b1, w2, b2, keep, K))) return rc;
  if (g.N > kMaxRankTokens || g.T > kMaxRankTokens) return SS_EUNSUPPORTED;
  const int heads = cfg->heads, dh = cfg->head_dim;
  AttnLayout L;
  if ((rc = attn_layout(cfg, g, &L))) return rc;
  const size_t attn_part = align256(L.total);
  if (!ws || !aligned(ws, 256) || ws_bytes < attn_part + rcmlp_ws_bytes(g, K, C, hidden))
    return SS_EWORKSPACE;
  // out may not overlap x: S4's row gather starts before S3 has finished writing out.
  {
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(out);
    const uintptr_t o1 = o0 + (size_t)g.U * g.N * heads * dh * 2;
    const uintptr_t x0 = reinterpret_cast<uintptr_t>(x);
    const uintptr_t x1 = x0 + (size_t)g.B * g.T * C * 2;
    if (o0 < x1 && x0 < o1) return SS_EINVAL;
  }
  int* status = status_word();
  if (!status) return SS_ECUDA;
  uint8_t* wsa = static_cast<uint8_t*>(ws);
  uint8_t* wsm = wsa + attn_part;
  const MlpPlan plan = mlp_plan(g, K, C, hidden);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  // S1 + S2 in one pass, the attention's gather and the attention, the MLP's gather (which also
  // zeroes the GEMMs' k-split counters) and fc1, fc2: the launches of the per-step calls. (Fusing
  // the two gathers into the ranking launch was measured slower: its 128 ranking CTAs copy the
  // rows less efficiently than the gathers spread over every SM.)
  if ((rc = rank_path(cfg, lum, nullptr, score, perm, inv, keep, stream))) return rc;
  if ((rc = gather_launch(g, heads, dh, L, q, k, v, perm, wsa, status, st))) return rc;
  if ((rc = attn_launch(cfg, g, L, wsa, perm, out, status, st))) return rc;
  // The row gather's inputs are final: keep came from the ranking launch, which the Q/K/V gather
  // and the attention waited for before this launch can start, and x is not written before fc2.
  // Its copy runs in the attention's tail; its dependency wait comes last (late_wait).
  const int n_counters = (int)((plan.total - plan.counters) / sizeof(int));
  rc = cuda_err(traced("gather_rows", st, [&] {
    return launch_gather_rows(x, keep, reinterpret_cast<uint16_t*>(wsm + plan.xk), g.B, g.T, K, C,
                              reinterpret_cast<int*>(wsm + plan.counters), n_counters, status, st,
                              /*late_wait=*/true);
  }));
  if (rc) return rc;
  return rcmlp_launch(g, K, x, C, hidden, w1, b1, w2, b2, keep, wsm, status, st);
}

// ---- the relative-position variant ------------------------------------------------------------

// Workspace: the attention's (pair kernel), then the stacked tables rpack [nr, dh], the bias
// products [U*heads*N, nr] fp16 and the one-hot rows [U, npad, 128] fp16.
struct RelLayout {
  AttnLayout L;
  GemmPlan gp;
  int Hu, Wu, nr, npad;
  size_t rpack, tab, onehot, total;
};

static int rel_layout(const ss_cfg* cfg, const Geo& g, RelLayout* R) {
  int rc = attn_layout(cfg, g, &R->L, /*force_pair=*/true);
  if (rc) return rc;
  R->Hu = g.window_mode ? g.ws : g.Hg;
  R->Wu = g.window_mode ? g.ws : g.Wg;
  R->nr = (2 * R->Hu - 1 + 2 * R->Wu - 1 + 63) / 64 * 64;
  R->npad = (g.N + 127) / 128 * 128;
  const long long M = (long long)g.U * cfg->heads * g.N;
  R->gp = gemm_plan((int)M, R->nr, cfg->head_dim, kPlanSMs);
  R->rpack = align256(R->L.total);
  R->tab = R->rpack + align256((size_t)R->nr * cfg->head_dim * 2);
  R->onehot = R->tab + align256((size_t)M * R->nr * 2);
  R->total = R->onehot + align256((size_t)g.U * R->npad * kRelPosOneHotCols * 2);
  return SS_OK;
}

size_t sparsesam_attn_relpos_workspace(const ss_cfg* cfg) {
  Geo g;
  RelLayout R;
  if (geometry(cfg, &g) || cfg->heads < 1 || cfg->head_dim < 1 || rel_layout(cfg, g, &R))
    return 0;
  return R.total;
}

int sparsesam_attn_relpos(const ss_cfg* cfg, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* perm, const uint16_t* rel_h,
                          const uint16_t* rel_w, uint16_t* out, void* ws, size_t ws_bytes,
                          void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  ss_pattern p;
  if ((rc = attn_check(cfg, g, q, k, v, perm, out, &p))) return rc;
  if (!rel_h || !rel_w || !aligned(rel_h, 16) || !aligned(rel_w, 16)) return SS_EINVAL;
  if (cfg->head_dim != 64) return SS_EUNSUPPORTED;
  RelLayout R;
  if ((rc = rel_layout(cfg, g, &R))) return rc;
  // A query row's bias slices (Hu + Wu fp16 values) fill at most the 64 TMEM columns of its group.
  if (R.Hu + R.Wu > kRelPosOneHotCols) return SS_EUNSUPPORTED;
  if ((long long)g.U * cfg->heads * g.N * R.nr >= (1ll << 31) ||
      ((long long)g.U * cfg->heads * g.N + 127) / 128 > 65535)
    return SS_EUNSUPPORTED;
  if (!ws || !aligned(ws, 256) || ws_bytes < R.total) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  const int heads = cfg->heads, dh = cfg->head_dim;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint16_t* rpack = reinterpret_cast<uint16_t*>(wsb + R.rpack);
  uint16_t* tab = reinterpret_cast<uint16_t*>(wsb + R.tab);
  uint16_t* onehot = reinterpret_cast<uint16_t*>(wsb + R.onehot);
  // The packed tables are the bias GEMM's B operand, whose first tiles it requests before its
  // dependency wait: they come from the launch before the gather (which completes before the
  // gather lets the GEMM start).
  rc = cuda_err(traced("relpos_prep", st, [&] {
    return launch_relpos_prep(rel_h, rel_w, rpack, dh, R.nr, perm, onehot, g.U, g.N, R.npad, R.Hu,
                              R.Wu, R.L.ap.b, status, st);
  }));
  if (rc) return rc;
  if ((rc = gather_launch(g, heads, dh, R.L, q, k, v, perm, wsb, status, st))) return rc;
  const long long M = (long long)g.U * heads * g.N;
  CUtensorMap ta, tb, te;
  if (!encode_bf16(&ta, 2, wsb, dh, M, 1, (uint64_t)dh * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tb, 2, rpack, dh, R.nr, 1, (uint64_t)dh * 2, 64, R.gp.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      // the one-hot rows as [U][npad][128] 16-bit values: 64-column boxes of 128 rows (the
      // layout of a K tile); TMA moves bytes, so the bf16 encoding serves the fp16 data
      !encode_bf16(&te, 3, onehot, kRelPosOneHotCols, R.npad, g.U,
                   (uint64_t)kRelPosOneHotCols * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
    return SS_ECUDA;
  GemmEpilogue e = {};
  e.kind = 4;
  e.out = tab;
  // sqrt(dh): the attention scales S = q.k + bias * sqrt(dh) by 1/sqrt(dh) (and log2 e) as a whole
  e.scale = (float)sqrt((double)dh);
  rc = cuda_err(traced("relpos_gemm", st, [&] {
    return launch_gemm(&ta, &tb, R.gp, (int)M, R.nr, dh, e, nullptr, nullptr, sm_count(), status,
                       st);
  }));
  if (rc) return rc;
  AttnParams rel = {};
  rel.rel_tab = tab;
  rel.rel_ld = R.nr;
  rel.rel_h = R.Hu;
  rel.rel_w = R.Wu;
  rel.rel_ksteps = (R.Hu + R.Wu + 15) / 16;
  return attn_launch(cfg, g, R.L, wsb, perm, out, status, st, nullptr, &rel, &te);
}

// ---- the partial-token-count variant (prefix tokens, RoPE) -------------------------------------

// Workspace: the attention's (gathered and rotated Q, K, V; ...), then the patch rows' attention
// output in token order [U, N, heads, dh] and their (m, l) [U*heads, N].
struct PartialLayout {
  AttnLayout L;
  size_t po, ml, total;
};

static int partial_layout(const ss_cfg* cfg, const Geo& g, PartialLayout* P) {
  int rc = attn_layout(cfg, g, &P->L);
  if (rc) return rc;
  const size_t rows = (size_t)g.U * cfg->heads * g.N;
  P->po = align256(P->L.total);
  P->ml = P->po + align256(rows * cfg->head_dim * 2);
  P->total = P->ml + align256(rows * 8);
  return SS_OK;
}

size_t sparsesam_attn_partial_workspace(const ss_cfg* cfg, int32_t prefix) {
  Geo g;
  PartialLayout P;
  if (geometry(cfg, &g) || cfg->heads < 1 || cfg->head_dim < 1 || prefix < 0 ||
      prefix > kMaxPrefix || partial_layout(cfg, g, &P))
    return 0;
  return P.total;
}

int sparsesam_attn_partial(const ss_cfg* cfg, int32_t prefix, float rope_base, const uint16_t* q,
                           const uint16_t* k, const uint16_t* v, const int32_t* perm,
                           uint16_t* out, void* ws, size_t ws_bytes, void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if (g.window_mode) return SS_EUNSUPPORTED;
  if (prefix < 0 || prefix > kMaxPrefix) return SS_EINVAL;
  if (!(rope_base == 0.f || (rope_base > 1.f && rope_base < INFINITY))) return SS_EINVAL;
  ss_pattern p;
  if ((rc = attn_check(cfg, g, q, k, v, perm, out, &p))) return rc;
  if (cfg->heads > kMaxPrefixHeads) return SS_EUNSUPPORTED;
  if ((size_t)(prefix + g.N) * sizeof(float) > kMaxPrefixRowsSmem) return SS_EUNSUPPORTED;
  if ((int64_t)g.U * (g.N + prefix) * cfg->heads * (cfg->head_dim / 8) >= (int64_t)1 << 31)
    return SS_EUNSUPPORTED;
  PartialLayout P;
  if ((rc = partial_layout(cfg, g, &P))) return rc;
  if (!ws || !aligned(ws, 256) || ws_bytes < P.total) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  const int heads = cfg->heads, dh = cfg->head_dim;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  uint16_t* qp = reinterpret_cast<uint16_t*>(wsb);
  uint16_t* kp = reinterpret_cast<uint16_t*>(wsb + P.L.one);
  uint16_t* vp = reinterpret_cast<uint16_t*>(wsb + 2 * P.L.one);
  uint16_t* po = reinterpret_cast<uint16_t*>(wsb + P.po);
  float2* ml = reinterpret_cast<float2*>(wsb + P.ml);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const float log2_base = rope_base == 0.f ? 0.f : (float)log2((double)rope_base);
  rc = cuda_err(traced("gather_rope", st, [&] {
    return launch_gather_rope(q, k, v, perm, qp, kp, vp, g.U, g.N, heads, dh, p.b, prefix, g.Wg,
                              log2_base, status, st);
  }));
  if (rc) return rc;
  // Without prefix tokens the patch rows are the output itself.
  if ((rc = attn_launch(cfg, g, P.L, wsb, perm, prefix ? po : out, status, st, ml))) return rc;
  if (prefix == 0) return SS_OK;
  rc = cuda_err(traced("prefix_merge", st, [&] {
    return launch_prefix_merge(po, ml, qp, k, v, perm, out, g.U, g.N, heads, dh, p.b, prefix,
                               P.L.ap.scale_log2, status, st);
  }));
  if (rc) return rc;
  return cuda_err(traced("prefix_rows", st, [&] {
    return launch_prefix_rows(q, k, v, kp, vp, out, g.U, g.N, heads, dh, prefix,
                              P.L.ap.scale_log2, st);
  }));
}

// ---- the full encoder block -----------------------------------------------------------------

static UnitRows unit_rows_of(const Geo& g) {
  UnitRows r;
  r.N = g.N;
  r.T = g.T;
  r.grid_w = g.Wg;
  r.grid_h = g.Hg;
  r.window = g.window_mode ? g.ws : 0;
  r.win_per_row = g.wpr;
  r.windows = g.windows;
  return r;
}

// The encoder block's workspace: LN1's output over the units [U*N, C] (later the attention's
// output, which the projection reads), the attention's workspace (the qkv GEMM writes the gathered
// Q, K, V into it), the qkv and proj GEMMs' k-split scratch, then the RC-MLP's workspace.
struct EncLayout {
  AttnLayout L;
  GemmPlan qkv, proj;
  MlpPlan mlp;
  size_t attn, gemm_partial, gemm_counters, mlp_base, total;   // byte offsets, total size
};

static int enc_layout(const ss_cfg* cfg, const Geo& g, int C, int hidden, int K, EncLayout* E) {
  int rc = attn_layout(cfg, g, &E->L);
  if (rc) return rc;
  const long long M = (long long)g.U * g.N;
  E->qkv = gemm_plan((int)M, 3 * C, C, kPlanSMs);
  E->proj = gemm_plan((int)M, C, C, kPlanSMs);
  const size_t p1 = gemm_partial_bytes(E->qkv), p2 = gemm_partial_bytes(E->proj);
  const size_t part = align256(p1 > p2 ? p1 : p2);
  const int t1 = E->qkv.m_tiles * E->qkv.n_tiles, t2 = E->proj.m_tiles * E->proj.n_tiles;
  const size_t cnt = part ? align256((size_t)(t1 > t2 ? t1 : t2) * 2 * 4) : 0;
  E->mlp = mlp_plan(g, K, C, hidden);
  E->attn = align256((size_t)M * C * 2);
  E->gemm_partial = E->attn + align256(E->L.total);
  E->gemm_counters = E->gemm_partial + part;
  E->mlp_base = E->gemm_counters + cnt;
  E->total = E->mlp_base + (K > 0 ? E->mlp.total : 0);
  return SS_OK;
}

static int enc_check(const ss_cfg* cfg, const Geo& g, const uint16_t* x, int32_t C,
                     int32_t hidden, const ss_block_weights* w, const int32_t* perm,
                     const int32_t* inv, const int32_t* keep, int32_t K) {
  if (cfg->heads < 1 || cfg->head_dim < 1 || C < 1 || hidden < 1) return SS_EINVAL;
  if (cfg->head_dim != 64 && cfg->head_dim != 80) return SS_EUNSUPPORTED;
  if ((int64_t)cfg->heads * cfg->head_dim != C) return SS_EINVAL;
  if (C % 64 != 0 || hidden % 64 != 0) return SS_EUNSUPPORTED;
  if (!x || !w || !perm || !inv || K < 0 || K > g.T || (K > 0 && !keep)) return SS_EINVAL;
  if (!w->ln1_w || !w->ln1_b || !w->w_qkv || !w->w_proj || !w->ln2_w || !w->ln2_b || !w->w1 ||
      !w->w2)
    return SS_EINVAL;
  const void* al[] = {x, w->ln1_w, w->ln1_b, w->w_qkv, w->b_qkv, w->w_proj, w->b_proj,
                      w->ln2_w, w->ln2_b, w->w1, w->b1, w->w2, w->b2};
  for (const void* a : al)
    if (!aligned(a, 16)) return SS_EINVAL;
  ss_pattern p;
  int rc = pattern_of(cfg, g, &p);
  if (rc) return rc;
  const int64_t M = (int64_t)g.U * g.N, Mk = (int64_t)g.B * K;
  if ((int64_t)g.U * cfg->heads > 65535) return SS_EUNSUPPORTED;
  if (M * 3 * C >= ((int64_t)1 << 31) || (M + 127) / 128 > 65535) return SS_EUNSUPPORTED;
  if (Mk * (hidden > C ? hidden : C) >= ((int64_t)1 << 31) || (Mk + 127) / 128 > 65535)
    return SS_EUNSUPPORTED;
  if ((int64_t)g.B * g.T * C >= ((int64_t)1 << 31)) return SS_EUNSUPPORTED;
  return SS_OK;
}

// LN1 -> qkv GEMM (straight into the gathered layout) -> attention -> proj GEMM (+ residual, pads
// dropped) -> LN2 over the kept rows -> fc1 -> fc2 (+ residual). ws laid out as enc_layout says.
static int enc_launch(const ss_cfg* cfg, const Geo& g, const EncLayout& E, uint16_t* x, int C,
                      int hidden, const ss_block_weights* w, const int32_t* perm,
                      const int32_t* inv, const int32_t* keep, int K, uint8_t* ws, int* status,
                      cudaStream_t st) {
  const long long M = (long long)g.U * g.N;
  const UnitRows ur = unit_rows_of(g);
  uint16_t* xn = reinterpret_cast<uint16_t*>(ws);
  uint8_t* wsa = ws + E.attn;
  float* partial = reinterpret_cast<float*>(ws + E.gemm_partial);
  int* counters = reinterpret_cast<int*>(ws + E.gemm_counters);
  const int n_counters = (int)((E.mlp_base - E.gemm_counters) / sizeof(int));
  const int sms = sm_count();
  int rc = cuda_err(traced("ln1", st, [&] {
    return launch_ln_rows(x, w->ln1_w, w->ln1_b, xn, M, C, ur, nullptr, 0, counters, n_counters,
                          status, st);
  }));
  if (rc) return rc;
  CUtensorMap ta, tb, tp;
  if (!encode_bf16(&ta, 2, xn, C, M, 1, (uint64_t)C * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tb, 2, w->w_qkv, C, 3 * C, 1, (uint64_t)C * 2, 64, E.qkv.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_bf16(&tp, 2, w->w_proj, C, C, 1, (uint64_t)C * 2, 64, E.proj.bn,
                   CU_TENSOR_MAP_SWIZZLE_128B))
    return SS_ECUDA;
  GemmEpilogue eq = {};
  eq.kind = 2;
  eq.bias = w->b_qkv;
  eq.out = reinterpret_cast<uint16_t*>(wsa);
  eq.inv = inv;
  eq.which_stride = (long long)(E.L.one / 2);
  eq.heads = cfg->heads;
  eq.dh = cfg->head_dim;
  eq.C = C;
  eq.b = E.L.ap.b;
  eq.L = E.L.ap.L;
  eq.ur = ur;
  rc = cuda_err(traced("qkv", st, [&] {
    return launch_gemm(&ta, &tb, E.qkv, (int)M, 3 * C, C, eq, partial, counters, sms, status, st);
  }));
  if (rc) return rc;
  // The attention writes its [U, N, heads, dh] output over LN1's rows, which the qkv GEMM has
  // finished reading: each launch of the chain starts its work only after the previous one has
  // completed.
  if ((rc = attn_launch(cfg, g, E.L, wsa, perm, xn, status, st))) return rc;
  GemmEpilogue ep = {};
  ep.kind = 3;
  ep.bias = w->b_proj;
  ep.x = x;
  ep.ur = ur;
  rc = cuda_err(traced("proj", st, [&] {
    return launch_gemm(&ta, &tp, E.proj, (int)M, C, C, ep, partial, counters, sms, status, st);
  }));
  if (rc || K == 0) return rc;
  uint8_t* wsm = ws + E.mlp_base;
  const int n_mlp_counters = (int)((E.mlp.total - E.mlp.counters) / sizeof(int));
  rc = cuda_err(traced("ln2_rows", st, [&] {
    return launch_ln_rows(x, w->ln2_w, w->ln2_b, reinterpret_cast<uint16_t*>(wsm + E.mlp.xk),
                          (long long)g.B * K, C, ur, keep, K,
                          reinterpret_cast<int*>(wsm + E.mlp.counters), n_mlp_counters, status,
                          st);
  }));
  if (rc) return rc;
  return rcmlp_launch(g, K, x, C, hidden, w->w1, w->b1, w->w2, w->b2, keep, wsm, status, st);
}

size_t sparsesam_encoder_block_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden, int32_t K) {
  Geo g;
  EncLayout E;
  if (geometry(cfg, &g) || cfg->heads < 1 || cfg->head_dim < 1 || C < 1 || hidden < 1 || K < 0 ||
      K > g.T || enc_layout(cfg, g, C, hidden, K, &E))
    return 0;
  return E.total;
}

int sparsesam_encoder_block(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden,
                            const ss_block_weights* w, const int32_t* perm, const int32_t* inv,
                            const int32_t* keep, int32_t K, void* ws, size_t ws_bytes,
                            void* stream) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if ((rc = enc_check(cfg, g, x, C, hidden, w, perm, inv, keep, K))) return rc;
  EncLayout E;
  if ((rc = enc_layout(cfg, g, C, hidden, K, &E))) return rc;
  if (!ws || !aligned(ws, 256) || ws_bytes < E.total) return SS_EWORKSPACE;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  return enc_launch(cfg, g, E, x, C, hidden, w, perm, inv, keep, K, static_cast<uint8_t*>(ws),
                    status, static_cast<cudaStream_t>(stream));
}

// ---- the encoder stack ------------------------------------------------------------------------

// The stack's workspace: scores, both permutations with their inverses, the keep list, then one
// encoder block's workspace (the larger of the two geometries'), reused by every block.
struct StackLayout {
  ss_cfg cg, cw;       // the global and the windowed blocks' cfg
  Geo gg, gw;
  EncLayout eg, ew;
  int K;
  size_t score, perm_g, inv_g, perm_w, inv_w, keep, block, total;
};

static int stack_layout(const ss_cfg* cfg, int C, int hidden, StackLayout* S) {
  if (!cfg) return SS_EINVAL;
  S->cg = *cfg;
  S->cg.mode = SS_GLOBAL;
  S->cw = *cfg;
  S->cw.mode = SS_WINDOW;
  int rc = geometry(&S->cg, &S->gg);
  if (rc || (rc = geometry(&S->cw, &S->gw))) return rc;
  if (cfg->heads < 1 || cfg->head_dim < 1 || C < 1 || hidden < 1) return SS_EINVAL;
  S->K = keep_count(cfg->density, S->gg.T);
  if ((rc = enc_layout(&S->cg, S->gg, C, hidden, S->K, &S->eg)) ||
      (rc = enc_layout(&S->cw, S->gw, C, hidden, S->K, &S->ew)))
    return rc;
  const size_t BT = (size_t)S->gg.B * S->gg.T, UNw = (size_t)S->gw.U * S->gw.N;
  S->score = 0;
  S->perm_g = align256(BT * 8);
  S->inv_g = S->perm_g + align256(BT * 4);
  S->perm_w = S->inv_g + align256(BT * 4);
  S->inv_w = S->perm_w + align256(UNw * 4);
  S->keep = S->inv_w + align256(UNw * 4);
  S->block = S->keep + align256((size_t)S->gg.B * (S->K > 0 ? S->K : 1) * 4);
  S->total = S->block + (S->eg.total > S->ew.total ? S->eg.total : S->ew.total);
  return SS_OK;
}

size_t sparsesam_encoder_stack_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden) {
  StackLayout S;
  return stack_layout(cfg, C, hidden, &S) ? 0 : S.total;
}

int sparsesam_encoder_stack(const ss_cfg* cfg, const float* lum, uint16_t* x, int32_t C,
                            int32_t hidden, int32_t n_blocks, const ss_block_weights* w,
                            const uint8_t* is_global, void* ws, size_t ws_bytes, void* stream) {
  StackLayout S;
  int rc = stack_layout(cfg, C, hidden, &S);
  if (rc) return rc;
  if (!lum || n_blocks < 0 || (n_blocks > 0 && (!w || !is_global))) return SS_EINVAL;
  if (S.gg.T > kMaxRankTokens || S.gw.N > kMaxRankTokens || S.gw.U > 65535 || S.gg.U > 65535)
    return SS_EUNSUPPORTED;
  if (!ws || !aligned(ws, 256) || ws_bytes < S.total) return SS_EWORKSPACE;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  double* score = reinterpret_cast<double*>(wsb + S.score);
  int32_t* perm_g = reinterpret_cast<int32_t*>(wsb + S.perm_g);
  int32_t* inv_g = reinterpret_cast<int32_t*>(wsb + S.inv_g);
  int32_t* perm_w = reinterpret_cast<int32_t*>(wsb + S.perm_w);
  int32_t* inv_w = reinterpret_cast<int32_t*>(wsb + S.inv_w);
  int32_t* keep = reinterpret_cast<int32_t*>(wsb + S.keep);
  // Every block's arguments are checked before the first launch.
  for (int i = 0; i < n_blocks; ++i) {
    const bool glob = is_global[i] != 0;
    rc = enc_check(glob ? &S.cg : &S.cw, glob ? S.gg : S.gw, x, C, hidden, &w[i],
                   glob ? perm_g : perm_w, glob ? inv_g : inv_w, keep, S.K);
    if (rc) return rc;
  }
  int* status = status_word();
  if (!status) return SS_ECUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if ((rc = rank_path(&S.cg, lum, nullptr, score, perm_g, inv_g, S.K > 0 ? keep : nullptr,
                      stream)))
    return rc;
  if ((rc = rank_path(&S.cw, nullptr, score, nullptr, perm_w, inv_w, nullptr, stream))) return rc;
  for (int i = 0; i < n_blocks; ++i) {
    const bool glob = is_global[i] != 0;
    rc = enc_launch(glob ? &S.cg : &S.cw, glob ? S.gg : S.gw, glob ? S.eg : S.ew, x, C, hidden,
                    &w[i], glob ? perm_g : perm_w, glob ? inv_g : inv_w, keep, S.K,
                    wsb + S.block, status, st);
    if (rc) return rc;
  }
  return SS_OK;
}

int sparsesam_device_status(int32_t* out, void* stream) {
  if (!out) return SS_EINVAL;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int v = 0;
  if (cudaMemcpyAsync(&v, status, sizeof(int), cudaMemcpyDeviceToHost, st) != cudaSuccess ||
      cudaMemsetAsync(status, 0, sizeof(int), st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess)
    return SS_ECUDA;
  *out = v;
  return SS_OK;
}

uint64_t sparsesam_launch_count(void) { return g_launches.load(); }

int sparsesam_set_wait_limit_ns(uint64_t ns) {
  const uint64_t v = ns ? ns : kWaitLimitNs;
  if (set_wait_limit_here(v) != cudaSuccess || set_wait_limit_attn(v) != cudaSuccess ||
      set_wait_limit_mlp(v) != cudaSuccess)
    return SS_ECUDA;
  return SS_OK;
}

int sparsesam_wait_selftest(int32_t which, void* stream) {
  if (which < 0 || which > 3) return SS_EINVAL;
  int* status = status_word();
  if (!status) return SS_ECUDA;
  int* counter = nullptr;
  if (cudaGetSymbolAddress(reinterpret_cast<void**>(&counter), g_selftest_counter) != cudaSuccess)
    return SS_ECUDA;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  return cuda_err(traced("wait_selftest", st, [&] {
    k_wait_selftest<<<1, 32, 0, st>>>(which, counter, status);
    return cudaGetLastError();
  }));
}

int sparsesam_trace_start(int32_t capacity) {
  if (capacity < 1) return SS_EINVAL;
  std::lock_guard<std::mutex> lk(g_mu);
  for (auto& r : g_trace) {
    cudaEventDestroy(r.e0);
    cudaEventDestroy(r.e1);
  }
  g_trace.assign(capacity, TraceRec{nullptr, nullptr, nullptr, 0.f});
  for (auto& r : g_trace)
    if (cudaEventCreate(&r.e0) != cudaSuccess || cudaEventCreate(&r.e1) != cudaSuccess)
      return SS_ECUDA;
  g_trace_used = 0;
  g_tracing = true;
  return SS_OK;
}

int sparsesam_trace_stop(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_tracing = false;
  for (int i = 0; i < g_trace_used; ++i) {
    TraceRec& r = g_trace[i];
    if (cudaEventSynchronize(r.e1) != cudaSuccess ||
        cudaEventElapsedTime(&r.ms, r.e0, r.e1) != cudaSuccess)
      return SS_ECUDA;
  }
  return g_trace_used;
}

int sparsesam_trace_get(int32_t i, const char** name, float* ms) {
  if (i < 0 || i >= g_trace_used || !name || !ms) return SS_EINVAL;
  *name = g_trace[i].name;
  *ms = g_trace[i].ms;
  return SS_OK;
}

const char* sparsesam_strerror(int code) {
  switch (code) {
    case SS_OK: return "ok";
    case SS_EINVAL: return "invalid argument";
    case SS_EUNSUPPORTED: return "unsupported shape";
    case SS_EWORKSPACE: return "workspace missing, misaligned or too small";
    case SS_ECUDA: return "CUDA call failed";
    case SS_ETIMEOUT: return "device wait timed out";
    case SS_EINDEX: return "perm or keep index outside its unit or image (access skipped)";
  }
  return "unknown error";
}

}  // extern "C"

// The argument checks of sparsesam_rcmlp, in its order, and its workspace size (for the entry point
// without a workspace, which must answer as sparsesam_rcmlp does).
int ss::rcmlp_validate(const ss_cfg* cfg, const uint16_t* x, int32_t C, int32_t hidden,
                       const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                       const uint16_t* b2, const int32_t* keep, int32_t K, size_t* need) {
  Geo g;
  int rc = geometry(cfg, &g);
  if (rc) return rc;
  if ((rc = rcmlp_check(g, x, C, hidden, w1, b1, w2, b2, keep, K))) return rc;
  *need = K == 0 ? 0 : rcmlp_ws_bytes(g, K, C, hidden);
  return SS_OK;
}
