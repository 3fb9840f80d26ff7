// S3: Stripe-Sort block-sparse attention on tcgen05 / TMEM.
//
// SparseSAM Dutch technical summary, "Statisch Sparsiteitspatroon": after the stripe permutation
// the N x N attention matrix is a 4 x 4 mosaic of sub-maps sharing one banded-diagonal pattern plus
// a global keep-set, executed by a FlashAttention-2-style kernel with no runtime mask building.
//
// Layout. The gather kernel writes Q, K, V of every (unit, head) in block-major permuted order:
// position q = a*(4b) + j*b + r holds canonical permuted position p = j*L + a*b + r (offset block
// a of stripe j). All four stripes of an offset block are then contiguous, and since all 16
// sub-maps share one pattern, a 128-row query tile of one offset block has a single key set: the
// offset blocks [0, g) and [s(a), s(a)+W), i.e. at most two contiguous runs of 128-row key tiles.
// The kernel derives that tile list from (b, nb, W, g) itself: no block list is read.
//
// One CTA = one (unit, head, 128-row query tile). Warp roles:
//   warp 0     TMA producer (Q once, then K/V tiles into a 2-stage ring)
//   warp 1     TMEM allocator and tcgen05.mma issuer (S = Q K^T, then O_tile = P V)
//   warps 2-5  softmax: one thread per query row (TMEM lane), online softmax in fp32,
//              P written to shared memory as bf16 (128B-swizzled, K-major A operand),
//              O accumulated in registers; epilogue scatters rows to out[perm[p]].
// TMEM columns: [0,128) S (fp32), [128, 128+dh) P*V of the current tile (fp32).
#include "common.cuh"
#include "kernels.h"

namespace ss {

// ---------------------------------------------------------------------------------------------
// Gather: Xp[(u*heads + h), q, :] = X[u, perm[u, p(q)], h, :]
// ---------------------------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_gather_qkv(const uint16_t* __restrict__ q,
                                                    const uint16_t* __restrict__ k,
                                                    const uint16_t* __restrict__ v,
                                                    const int32_t* __restrict__ perm,
                                                    uint16_t* __restrict__ qp,
                                                    uint16_t* __restrict__ kp,
                                                    uint16_t* __restrict__ vp, int U, int N,
                                                    int heads, int dh, int b, int L) {
  const uint16_t* src = blockIdx.y == 0 ? q : (blockIdx.y == 1 ? k : v);
  uint16_t* dst = blockIdx.y == 0 ? qp : (blockIdx.y == 1 ? kp : vp);
  const int cpr = dh / 8;            // 16-byte chunks per head row
  const int per_tok = heads * cpr;   // 16-byte chunks per token (all heads)
  const int total = U * N * per_tok;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int c = i % per_tok;
    const int uq = i / per_tok;
    const int qpos = uq % N;
    const int u = uq / N;
    const int h = c / cpr, cc = c - (c / cpr) * cpr;
    const int p = blockmajor_to_canonical(qpos, b, L);
    const int t = min(max(__ldg(perm + (size_t)u * N + p), 0), N - 1);   // never leave the unit
    const uint4* s = reinterpret_cast<const uint4*>(src + (size_t)(u * N + t) * heads * dh) + c;
    uint4* d = reinterpret_cast<uint4*>(dst + ((size_t)(u * heads + h) * N + qpos) * dh) + cc;
    *d = __ldg(s);
  }
}

cudaError_t launch_gather_qkv(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int32_t* perm, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                              int U, int N, int heads, int dh, int b, cudaStream_t st) {
  const int total = U * N * heads * (dh / 8);
  int blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_gather_qkv<<<dim3(blocks, 3), 256, 0, st>>>(q, k, v, perm, qp, kp, vp, U, N, heads, dh, b,
                                                N / kStripes);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------------------------
constexpr int kBM = 128;          // query rows per CTA
constexpr int kBN = 128;          // keys per tile
constexpr int kStages = 3;        // K/V ring depth
constexpr int kAttnThreads = 320; // 10 warps
constexpr float kLazyRescale = 8.f;   // log2 headroom before O and l are rescaled

template <int DH>
struct AttnSmem {
  static constexpr int kTail = DH - 64;                // 0 or 16 columns past the 128B atom
  static constexpr int kMain = kBM * 128;              // 128 rows x 128 B
  static constexpr int kTailBytes = kTail ? kBM * kTail * 2 : 0;
  static constexpr int kQ = 0;
  static constexpr int kQTail = kQ + kMain;
  static constexpr int kK = ((kQTail + kTailBytes + 1023) / 1024) * 1024;
  static constexpr int kStageBytes = ((kMain + kTailBytes + 1023) / 1024) * 1024;
  static constexpr int kV = kK + kStages * kStageBytes;
  static constexpr int kP = kV + kStages * kStageBytes;  // two P buffers, one per softmax group
  static constexpr int kPBytes = kBM * kBN * 2;        // two 128B-swizzled atoms of 64 keys
  static constexpr int kML = kP + 2 * kPBytes;         // float m[2][128], l[2][128]
  static constexpr int kBar = kML + 4 * kBM * 4;
  static constexpr int kBytes = kBar + 256;
  static constexpr int kAlloc = kBytes + 1024;         // slack to align the base to 1024
};

struct KeyTiles {
  int lo0, hi0, lo1, hi1;
  __device__ int count() const { return (hi0 - lo0) + (hi1 - lo1); }
  __device__ int tile(int n) const { return n < hi0 - lo0 ? lo0 + n : lo1 + (n - (hi0 - lo0)); }
};

// Key tiles a query tile [q0, q_last] needs: the global rows [0, g*4b) and the band rows
// [s(a_lo)*4b, (s(a_hi)+W)*4b), both clipped to N, as two (possibly merged) runs of tiles.
__device__ __forceinline__ KeyTiles key_tiles(int q0, int q_last, const AttnParams& P) {
  const int b4 = P.b * kStripes;
  const int a_lo = q0 / b4, a_hi = q_last / b4;
  const int s_lo = band_start(a_lo, P.W, P.nb), s_hi = band_start(a_hi, P.W, P.nb);
  const int g_end = min(P.N, P.g * b4);
  KeyTiles t;
  t.lo0 = 0;
  t.hi0 = (g_end + kBN - 1) / kBN;
  t.lo1 = (s_lo * b4) / kBN;
  t.hi1 = (min(P.N, (s_hi + P.W) * b4) + kBN - 1) / kBN;
  if (t.lo1 <= t.hi0) {
    t.hi0 = max(t.hi0, t.hi1);
    t.lo1 = t.hi1 = t.hi0;
  }
  return t;
}

// True if every (query row, key) pair of the tile is kept (no element mask needed).
__device__ __forceinline__ bool tile_full(int q0, int q_last, int c0, const AttnParams& P) {
  const int c_last = c0 + kBN - 1;
  if (c_last >= P.N) return false;
  const int b4 = P.b * kStripes;
  for (int a = q0 / b4; a <= q_last / b4; ++a)
    for (int ka = c0 / b4; ka <= c_last / b4; ++ka)
      if (!block_kept(a, ka, P.W, P.nb, P.g)) return false;
  return true;
}

// One CTA = one (unit, head, 128-row query tile). The key tiles are split between two softmax
// warpgroups (tile n goes to group n % 2), so the MMA warp alternates between them: while one
// group turns its S tile into probabilities, the tensor core runs the other group's P*V and the
// next Q*K^T. Each group keeps its own running max m, sum l and accumulator O (in TMEM); at the
// end the two partial results of every row are merged.
//   warp 0      TMA producer (Q once, then K/V tiles into a 3-stage ring)
//   warp 1      TMEM allocator and tcgen05.mma issuer
//   warps 2-5   softmax group 0 (one thread per query row = TMEM lane)
//   warps 6-9   softmax group 1
// TMEM columns: S0 [0,128), S1 [128,256), O0 [256, 256+dh), O1 [384, 384+dh).
template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tq_tail,
           const __grid_constant__ CUtensorMap tk_tail, const __grid_constant__ CUtensorMap tv_tail,
           const AttnParams P, int* status) {
  using S = AttnSmem<DH>;
  constexpr bool kHasTail = S::kTail > 0;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* s_m = reinterpret_cast<float*>(smem + S::kML);   // [2][128]
  float* s_l = s_m + 2 * kBM;                              // [2][128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* q_full = bars + 0;
  uint64_t* k_full = bars + 1;                 // [kStages]
  uint64_t* v_full = k_full + kStages;         // [kStages]
  uint64_t* kv_empty = v_full + kStages;       // [kStages]
  uint64_t* s_full = kv_empty + kStages;       // [2]
  uint64_t* p_full = s_full + 2;               // [2]
  uint64_t* o_done = p_full + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int uh = blockIdx.y;
  const int q0 = blockIdx.x * kBM;
  const int q_last = min(q0 + kBM, P.N) - 1;
  const KeyTiles tiles = key_tiles(q0, q_last, P);
  const int ntiles = tiles.count();

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(k_full + i, 1);
      mbar_init(v_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    for (int w = 0; w < 2; ++w) {
      mbar_init(s_full + w, 1);
      mbar_init(p_full + w, 128);
    }
    mbar_init(o_done, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ------------------------------ TMA producer ------------------------------
    if (lane == 0) {
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      mbar_expect_tx(q_full, S::kMain + S::kTailBytes);
      tma_load_3d(smem + S::kQ, &tq, q_full, 0, q0, uh);
      if (kHasTail) tma_load_3d(smem + S::kQTail, &tq_tail, q_full, 64, q0, uh);
      for (int n = 0; n < ntiles; ++n) {
        const int st = n % kStages;
        if (n >= kStages && !mbar_wait(kv_empty + st, ((n / kStages) - 1) & 1, abort, status))
          break;
        const int c0 = tiles.tile(n) * kBN;
        uint8_t* kb = smem + S::kK + st * S::kStageBytes;
        uint8_t* vb = smem + S::kV + st * S::kStageBytes;
        mbar_expect_tx(k_full + st, S::kMain + S::kTailBytes);
        tma_load_3d(kb, &tk, k_full + st, 0, c0, uh);
        if (kHasTail) tma_load_3d(kb + S::kMain, &tk_tail, k_full + st, 64, c0, uh);
        mbar_expect_tx(v_full + st, S::kMain + S::kTailBytes);
        tma_load_3d(vb, &tv, v_full + st, 0, c0, uh);
        if (kHasTail) tma_load_3d(vb + S::kMain, &tv_tail, v_full + st, 64, c0, uh);
      }
    }
  } else if (warp == 1) {
    // ------------------------------ MMA issuer --------------------------------
    if (lane == 0) {
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, 64, false, true);
      constexpr uint32_t idesc_pv_tail = idesc_bf16_f32(kBM, 16, false, true);
      const uint32_t q_addr = smem_u32(smem + S::kQ);
      bool ok = mbar_wait(q_full, 0, abort, status);
      // S_w = Q K_n^T for tile n (w = n % 2).
      auto issue_qk = [&](int n) -> bool {
        const int st = n % kStages;
        if (!mbar_wait(k_full + st, (n / kStages) & 1, abort, status)) return false;
        tc_fence_after();
        const uint32_t k_addr = smem_u32(smem + S::kK + st * S::kStageBytes);
        const uint32_t d = tmem + (n & 1) * kBN;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss(d, smem_desc(q_addr + kk * 32, 16, 1024, kSwizzle128B),
                       smem_desc(k_addr + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, kk > 0);
        if (kHasTail)
          umma_bf16_ss(d, smem_desc(q_addr + S::kMain, 16, 256, kSwizzle32B),
                       smem_desc(k_addr + S::kMain, 16, 256, kSwizzle32B), idesc_qk, 1);
        umma_commit(s_full + (n & 1));
        return true;
      };
      // O_w (+)= P_w V_n once group w has written P_w for tile n.
      auto issue_pv = [&](int n) -> bool {
        const int st = n % kStages, w = n & 1;
        if (!mbar_wait(p_full + w, (n >> 1) & 1, abort, status)) return false;
        if (!mbar_wait(v_full + st, (n / kStages) & 1, abort, status)) return false;
        tc_fence_after();
        const uint32_t v_addr = smem_u32(smem + S::kV + st * S::kStageBytes);
        const uint32_t p_addr = smem_u32(smem + S::kP + w * S::kPBytes);
        const uint32_t d = tmem + 256 + w * 128;
        const uint32_t acc = n >= 2;
#pragma unroll
        for (int kk = 0; kk < kBN / 16; ++kk) {
          const uint64_t a = smem_desc(p_addr + (kk >> 2) * (kBM * 128) + (kk & 3) * 32, 16, 1024,
                                       kSwizzle128B);
          umma_bf16_ss(d, a, smem_desc(v_addr + kk * 2048, kBN * 128, 1024, kSwizzle128B),
                       idesc_pv, acc | (kk > 0));
          if (kHasTail)
            umma_bf16_ss(d + 64, a,
                         smem_desc(v_addr + S::kMain + kk * 512, kBN * 32, 256, kSwizzle32B),
                         idesc_pv_tail, acc | (kk > 0));
        }
        umma_commit(kv_empty + st);
        return true;
      };
      if (ok) tc_fence_after();
      if (ok && ntiles > 0) ok = issue_qk(0);
      if (ok && ntiles > 1) ok = issue_qk(1);
      for (int n = 0; ok && n < ntiles; ++n) {
        ok = issue_pv(n);
        if (ok && n + 2 < ntiles) ok = issue_qk(n + 2);
      }
      if (ok) umma_commit(o_done);
    }
  } else {
    // ------------------------------ softmax groups ----------------------------
    const int grp = (warp - 2) >> 2;                    // 0 or 1
    const int row = 32 * (warp & 3) + lane;             // TMEM lane == query row
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t t_s = tmem + grp * kBN + lane_off;
    const uint32_t t_o = tmem + 256 + grp * 128 + lane_off;
    const int qrow = q0 + row;
    const int b4 = P.b * kStripes;
    const int a_q = min(qrow, P.N - 1) / b4;
    const int s_q = band_start(a_q, P.W, P.nb);
    const int band_lo = s_q * b4, band_hi = (s_q + P.W) * b4, glob_hi = P.g * b4;
    const uint32_t p_base = smem_u32(smem + S::kP + grp * S::kPBytes);
    const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
    float m_ref = -INFINITY, l_run = 0.f;
    bool ok = true;
    int j = 0;
    for (int n = grp; n < ntiles; n += 2, ++j) {
      // Warp-collective wait: either every lane goes on to the .sync.aligned TMEM ops or none.
      ok = __all_sync(0xffffffffu, mbar_wait(s_full + grp, j & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      float sv[kBN];
      {
        uint32_t r[128];
        tmem_ld128(t_s, r);
#pragma unroll
        for (int i = 0; i < kBN; ++i) sv[i] = __uint_as_float(r[i]);
      }
      const int c0 = tiles.tile(n) * kBN;
      if (!tile_full(q0, q_last, c0, P)) {
#pragma unroll
        for (int i = 0; i < kBN; ++i) {
          const int c = c0 + i;
          const bool kept = c < P.N && (c < glob_hi || (c >= band_lo && c < band_hi));
          if (!kept) sv[i] = -INFINITY;
        }
      }
      // Row max: eight independent chains of 3-input max over elements k, k+8, k+16, ...
      float mx[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmax3(sv[k], sv[k + 8], sv[k + 16]);
#pragma unroll
      for (int t = 3; t + 1 < 16; t += 2)
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv[k + 8 * t], sv[k + 8 * t + 8]);
#pragma unroll
      for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], sv[k + 8 * 15]);
      const float x_max =
          fmaxf(fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5])), fmaxf(mx[6], mx[7])) *
          P.scale_log2;
      // Lazy rescale: the reference max moves only when the row max passes it by 2^8, so O in
      // TMEM is rescaled on few tiles. The decision is warp-wide (TMEM ops are warp-collective);
      // the rescale itself runs after P is written, when the S registers are free.
      const bool grow = x_max > m_ref + kLazyRescale;
      const bool rescale = __any_sync(0xffffffffu, grow);
      float alpha = 1.f;
      if (rescale) {
        const float m_new = grow ? x_max : m_ref;
        alpha = (m_ref == -INFINITY) ? 0.f : ex2_mufu(m_ref - m_new);
        l_run *= alpha;
        m_ref = m_new;
      }
      const float ref = (m_ref == -INFINITY) ? 0.f : m_ref;
      const uint64_t nref2 = f2_pack(-ref, -ref);
      uint64_t sum2a = 0, sum2b = 0;   // two packed partial sums (bit pattern 0 = +0.0f pair)
#pragma unroll
      for (int at = 0; at < 2; ++at) {
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t w[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int i = at * 64 + cc * 8 + 2 * e;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(sv[i], sv[i + 1]), scale2, nref2), x0, x1);
            const float p0 = ex2_mufu(x0), p1 = ex2_mufu(x1);
            if (e & 1)
              sum2b = f2_add(sum2b, f2_pack(p0, p1));
            else
              sum2a = f2_add(sum2a, f2_pack(p0, p1));
            w[e] = pack_bf16(p0, p1);
          }
          st_shared_v4(p_base + at * (kBM * 128) + sw128_offset(row, cc), w[0], w[1], w[2], w[3]);
        }
      }
      float sa0, sa1;
      f2_unpack(f2_add(sum2a, sum2b), sa0, sa1);
      l_run += sa0 + sa1;
      if (rescale && j > 0) {
        // O_w holds the group's earlier tiles: their P*V completed before this S was committed,
        // and this tile's P*V is issued only after the arrive below.
#pragma unroll 1
        for (int c = 0; c < (DH + 31) / 32; ++c) {
          uint32_t o[32];
          tmem_ld32(t_o + c * 32, o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st32(t_o + c * 32, o);
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      mbar_arrive(p_full + grp);
    }
    // ---- merge the two groups' partial rows and scatter them to out[u, perm[p], h, :] ----
    s_m[grp * kBM + row] = m_ref;
    s_l[grp * kBM + row] = l_run;
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, 0, abort, status));
    tc_fence_after();
    named_barrier(1, 256);
    if (ok) {
      const float m0 = s_m[row], m1 = s_m[kBM + row];
      const float l0 = s_l[row], l1 = s_l[kBM + row];
      const float mm = fmaxf(m0, m1);
      const float a0 = (m0 == -INFINITY) ? 0.f : ex2_mufu(m0 - mm);
      const float a1 = (m1 == -INFINITY) ? 0.f : ex2_mufu(m1 - mm);
      const float L = l0 * a0 + l1 * a1;
      const float inv = L > 0.f ? 1.f / L : 0.f;
      const float f0 = a0 * inv, f1 = a1 * inv;
      const bool has0 = ntiles > 0, has1 = ntiles > 1;   // a group with no tile has no O
      const bool store = qrow < P.N;
      uint16_t* dst = nullptr;
      if (store) {
        const int u = uh / P.heads, h = uh - (uh / P.heads) * P.heads;
        const int p = blockmajor_to_canonical(qrow, P.b, P.L);
        const int t = min(max(__ldg(P.perm + (size_t)u * P.N + p), 0), P.N - 1);
        dst = P.out + ((size_t)(u * P.N + t) * P.heads + h) * DH;
      }
      const uint32_t o0 = tmem + 256 + lane_off, o1 = tmem + 384 + lane_off;
      constexpr int kChunks = DH / 8;            // 8 or 10 chunks of 8 columns
      for (int c = grp; c < kChunks; c += 2) {    // the two groups split the columns
        uint32_t x0[8], x1[8];
        tmem_ld8(o0 + c * 8, x0);                 // every lane loads (warp-collective) ...
        tmem_ld8(o1 + c * 8, x1);
        float v[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          v[i] = (has0 ? __uint_as_float(x0[i]) * f0 : 0.f) +
                 (has1 ? __uint_as_float(x1[i]) * f1 : 0.f);
        uint4 wv;
        wv.x = pack_bf16(v[0], v[1]);
        wv.y = pack_bf16(v[2], v[3]);
        wv.z = pack_bf16(v[4], v[5]);
        wv.w = pack_bf16(v[6], v[7]);
        if (store) reinterpret_cast<uint4*>(dst)[c] = wv;   // ... only rows < N store
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

template <int DH>
static cudaError_t launch_attn_dh(const CUtensorMap* tq, const CUtensorMap* tk,
                                  const CUtensorMap* tv, const CUtensorMap* tq_tail,
                                  const CUtensorMap* tk_tail, const CUtensorMap* tv_tail,
                                  const AttnParams& p, int* status, cudaStream_t st) {
  using S = AttnSmem<DH>;
  cudaError_t e = cudaFuncSetAttribute(k_attn<DH>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       S::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid((p.N + kBM - 1) / kBM, p.U * p.heads);
  k_attn<DH><<<grid, kAttnThreads, S::kAlloc, st>>>(*tq, *tk, *tv, *tq_tail, *tk_tail, *tv_tail, p,
                                                    status);
  return cudaGetLastError();
}

cudaError_t launch_attn(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* tq_tail, const CUtensorMap* tk_tail,
                        const CUtensorMap* tv_tail, const AttnParams& p, int dh, int* status,
                        cudaStream_t st) {
  if (dh == 64) return launch_attn_dh<64>(tq, tk, tv, tq, tk, tv, p, status, st);
  if (dh == 80) return launch_attn_dh<80>(tq, tk, tv, tq_tail, tk_tail, tv_tail, p, status, st);
  return cudaErrorInvalidValue;
}

}  // namespace ss
