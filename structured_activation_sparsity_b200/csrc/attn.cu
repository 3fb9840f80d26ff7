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
// Persistent: one CTA per SM walks the (unit, head, 128-row query tile) items. Per item a TMA
// producer streams Q and the item's key tiles (K and V) into shared memory, two single-thread
// issuers run S = Q K^T and O += P V on the tensor core with S, P and O in TMEM, and two softmax
// warpgroups (one thread per query row) take alternate key tiles with an online softmax in fp32;
// the epilogue merges the two groups' partial rows and scatters them to out[perm[p]].
#include <algorithm>
#include <type_traits>

#include "common.cuh"
#include "kernels.h"

namespace ss {

// ---------------------------------------------------------------------------------------------
// Gather: Xp[(u*heads + h), q, :] = X[u, perm[u, p(q)], h, :]
// ---------------------------------------------------------------------------------------------
// One CTA per (unit, 8 consecutive block-major positions), a warp per position: the warp resolves
// its source token, then copies the token's heads*dh row (contiguous in the source) as 16-byte
// chunks into the per-head rows of the gathered buffers. CPR = 16-byte chunks per head; KPL =
// chunks of one tensor per lane (heads*CPR <= 32*KPL), all 3*KPL loads of a lane in flight before
// its stores. MINB: CTAs per SM the registers are sized for.
template <int CPR, int KPL, int MINB>
__global__ void __launch_bounds__(256, MINB) k_gather_qkv(const uint16_t* __restrict__ q,
                                                       const uint16_t* __restrict__ k,
                                                       const uint16_t* __restrict__ v,
                                                       const int32_t* __restrict__ perm,
                                                       uint16_t* __restrict__ qp,
                                                       uint16_t* __restrict__ kp,
                                                       uint16_t* __restrict__ vp, int N,
                                                       int heads, int b, int L, int* status) {
  griddep_wait();
  griddep_launch();
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qpos = blockIdx.x * 8 + warp;
  if (qpos >= N) return;
  const int p = blockmajor_to_canonical(qpos, b, L);
  const int tok = __ldg(perm + (size_t)u * N + p);
  if ((unsigned)tok >= (unsigned)N) {   // not a token of this unit: skip the row, report it
    if (lane == 0) record_bad_index(status);
    return;
  }
  const int per_tok = heads * CPR;
  const size_t plane = (size_t)N * CPR;       // 16-byte chunks per (unit, head) matrix
  const size_t src_row = ((size_t)u * N + tok) * per_tok;
  const size_t dst_row = (size_t)u * heads * plane + (size_t)qpos * CPR;
  const uint4* src[3] = {reinterpret_cast<const uint4*>(q) + src_row,
                         reinterpret_cast<const uint4*>(k) + src_row,
                         reinterpret_cast<const uint4*>(v) + src_row};
  uint4* dst[3] = {reinterpret_cast<uint4*>(qp) + dst_row, reinterpret_cast<uint4*>(kp) + dst_row,
                   reinterpret_cast<uint4*>(vp) + dst_row};
  uint4 buf[3][KPL];
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int c = e * 32 + lane;
      if (c < per_tok) buf[t][e] = __ldg(src[t] + c);
    }
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int c = e * 32 + lane;
      if (c < per_tok) {
        const int h = c / CPR, cc = c - h * CPR;   // CPR is a compile-time constant
        dst[t][h * plane + cc] = buf[t][e];
      }
    }
}

cudaError_t launch_gather_qkv(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int32_t* perm, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                              int U, int N, int heads, int dh, int b, int* status,
                              cudaStream_t st) {
  dim3 grid((N + 7) / 8, U);
  const int L = N / kStripes;
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, grid, dim3(256), 0, st, q, k, v, perm, qp, kp, vp, N, heads, b, L,
                      status);
  };
  const int per_tok = heads * (dh / 8);
  if (dh != 64 && dh != 80) return cudaErrorInvalidValue;
  if (per_tok > 32 * 8) return cudaErrorInvalidValue;   // heads * dh > 2048
  const int kpl = (per_tok + 31) / 32;
  // Measured on one B200 (block step): head dim 80 with five chunks per lane sized for three CTAs
  // per SM, ViT-H 441.5 -> 435.2 us against the four-chunk form; at head dim 64 sizing for four
  // CTAs per SM (one wave at ViT-B) measured slower (108.8 -> 110.2 us), so it keeps its shape.
  if (dh == 64) return kpl <= 4 ? go(k_gather_qkv<8, 4, 1>) : go(k_gather_qkv<8, 8, 1>);
  return kpl <= 5 ? go(k_gather_qkv<10, 5, 3>) : go(k_gather_qkv<10, 8, 2>);
}

// ---------------------------------------------------------------------------------------------
// Attention kernel
// ---------------------------------------------------------------------------------------------
constexpr int kBM = 128;              // query rows per CTA
constexpr int kBN = 128;              // keys per tile
constexpr int kAttnThreads = 384;     // 12 warps = 3 warpgroups
constexpr float kLazyRescale = 8.f;   // log2 headroom before O and l are rescaled
constexpr int kPairTiles = 4;         // items of at most this many key tiles: k_attn_pairs
constexpr bool kPairInterleave = true;   // k_attn_pairs ring order A_0, B_0, A_1, B_1, ...
constexpr int kPolyPairs = 0;         // of every 16 exp pairs on full tiles, those on the FMA pipe
// Register split (launch: 384 threads x 168): producer warpgroup 56, softmax warpgroups 224.
constexpr uint32_t kRegsProducer = 56, kRegsSoftmax = 224;
static_assert(128 * kRegsProducer + 256 * kRegsSoftmax <= 384 * 168, "register split too large");

template <int DH>
struct AttnTmem {
  static constexpr bool kSeparateP = DH <= 64;
  static constexpr uint32_t kS = 0, kSStride = 128;
  static constexpr uint32_t kO = 256, kOStride = DH <= 64 ? 64 : 128;
  static constexpr uint32_t kP = kSeparateP ? 384 : 0, kPStride = kSeparateP ? 64 : 128;
};

template <int DH>
struct AttnSmem {
  static constexpr int kTail = DH - 64;                // 0 or 16 columns past the 128B atom
  static constexpr int kMain = kBM * 128;              // 128 rows x 128 B
  static constexpr int kTailBytes = kTail ? kBM * kTail * 2 : 0;
  static constexpr int kTileBytes = ((kMain + kTailBytes + 1023) / 1024) * 1024;
  static constexpr int kStages = DH == 64 ? 5 : 4;     // depth of the K/V ring
  static constexpr int kQ = 0;                         // two Q buffers (consecutive items)
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  // group 0's float m[2 items][128], l[2 items][128]: one item's rows stay intact while the
  // next item's are written
  static constexpr int kML = kV + kStages * kTileBytes;
  // Output staging: 128 rows of DH bf16, padded by 16 bytes so that the 32 rows a warp writes
  // at once spread over all banks; then the rows' destination tokens.
  static constexpr int kStageStride = DH * 2 + 16;
  static constexpr int kStage = kML + 4 * kBM * 4;
  static constexpr int kDst = kStage + kBM * kStageStride;
  static constexpr int kBar = kDst + kBM * 4;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;         // slack to align the base to 1024
  static_assert(kAlloc <= 227 * 1024, "attention shared memory above the per-CTA limit");
};

// The key tiles of one query tile, visited from an item-dependent starting point: CTAs that share
// key tiles (every query tile keeps the global block) then read different tiles at a time instead
// of all hitting the same L2 lines. The softmax is order-independent up to rounding.
struct KeyTiles {
  int lo0, hi0, lo1, hi1, rot;
  __host__ __device__ int count() const { return (hi0 - lo0) + (hi1 - lo1); }
  __device__ int tile(int n) const {
    const int c = count();
    n = n + rot < c ? n + rot : n + rot - c;
    return n < hi0 - lo0 ? lo0 + n : lo1 + (n - (hi0 - lo0));
  }
};

// Key tiles a query tile [q0, q_last] needs: the global rows [0, g*4b) and the band rows
// [s(a_lo)*4b, (s(a_hi)+W)*4b), both clipped to N, as two (possibly merged) runs of tiles.
__host__ __device__ __forceinline__ KeyTiles key_tiles(int q0, int q_last, int qt, int uh,
                                                       const AttnParams& P) {
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
  t.rot = (int)((qt * 5u + uh * 3u) % (unsigned)max(1, t.count()));
  return t;
}

// Every (query row, key) pair of a key tile is kept when offset blocks are whole multiples of the
// 128-row tile (4b % 128 == 0, e.g. b = 64): a query tile then lies in one offset block, and each
// key tile of its list lies in one kept offset block. Otherwise (b = 16, 7, ...) tiles straddle
// blocks and take the element mask; so does the ragged last key tile.
__device__ __forceinline__ bool tile_full(int c0, const AttnParams& P) {
  return (P.b * kStripes) % kBN == 0 && c0 + kBN <= P.N;
}

// Bits of the columns [lo, hi) that fall in [base, base + 32), as a 32-bit mask.
__device__ __forceinline__ uint32_t run_bits(int lo, int hi, int base) {
  const int l = min(max(lo - base, 0), 32), h = min(max(hi - base, 0), 32);
  const uint32_t mh = h >= 32 ? 0xffffffffu : (1u << h) - 1u;
  const uint32_t ml = l >= 32 ? 0xffffffffu : (1u << l) - 1u;
  return h > l ? (mh & ~ml) : 0u;
}

// 2^x on the FMA pipe for x in [-125, 8] (Cody-Waite style reduction 2^x = 2^n 2^f, n = round(x),
// f in [-1/2, 1/2]; 2^f by the cubic that interpolates it at the four Chebyshev nodes of the
// interval, coefficients from csrc/exp2_poly.py, relative error < 1e-4). Operates on a pair.
__device__ __forceinline__ void exp2_poly2(float x0, float x1, float& p0, float& p1) {
  constexpr float kMagic = 12582912.f;   // 1.5 * 2^23: adding it rounds to an integer in the low bits
  x0 = fmaxf(x0, -125.f);
  x1 = fmaxf(x1, -125.f);
  const uint64_t x2 = f2_pack(x0, x1);
  const uint64_t t2 = f2_add(x2, f2_pack(kMagic, kMagic));
  const uint64_t n2 = f2_add(t2, f2_pack(-kMagic, -kMagic));
  const uint64_t fr = f2_fma(n2, f2_pack(-1.f, -1.f), x2);
  uint64_t q = f2_fma(f2_pack(0.05583828315138817f, 0.05583828315138817f), fr,
                      f2_pack(0.2426394820213318f, 0.2426394820213318f));
  q = f2_fma(q, fr, f2_pack(0.6931367516517639f, 0.6931367516517639f));
  q = f2_fma(q, fr, f2_pack(0.9999245405197144f, 0.9999245405197144f));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t2, t0, t1);
  // add n to the exponent field: the low mantissa bits of t hold n (two's complement)
  p0 = __int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23));
  p1 = __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23));
}

// Destination token of an output row: perm's entry if it lies in the unit, else -1 (the row is
// not stored) with SS_EINDEX recorded.
__device__ __forceinline__ int dst_token(int perm_t, int N, int* status) {
  if ((unsigned)perm_t < (unsigned)N) return perm_t;
  record_bad_index(status);
  return -1;
}

// Work item = (unit * heads + head, 128-row query tile), numbered head-major so that the CTAs
// running at the same time share the K/V of a few heads in L2.
struct Item {
  int uh, q0, q_last;
  KeyTiles tiles;
};
__device__ __forceinline__ Item item_of(int it, int nq, const AttnParams& P) {
  Item I;
  I.uh = it / nq;
  const int qt = it - I.uh * nq;
  I.q0 = qt * kBM;
  I.q_last = min(I.q0 + kBM, P.N) - 1;
  I.tiles = key_tiles(I.q0, I.q_last, qt, I.uh, P);
  return I;
}

// Persistent: one CTA per SM walks the items it, it + gridDim.x, ... . The key tiles of an item
// are split between two softmax warpgroups (tile n goes to group n % 2), so the MMA pipe
// alternates between them: while one group turns its S tile into probabilities, the tensor core
// runs the other group's P*V and the next Q*K^T. Each group keeps its own running max m, sum l
// and accumulator O (in TMEM); at the end of an item the two partial results of every row are
// merged and scattered. Q is double-buffered, so the next item's Q*K^T starts while this item's
// last tiles and its epilogue are still running.
//   warp 0        TMA producer (Q per item; K and V tiles into a ring of stages)
//   warp 1        TMEM allocator and Q*K^T issuer
//   warp 2        P*V issuer
//   warp 3        idle (completes the producer warpgroup for the register split)
//   warps 4-7     softmax group 0 (one thread per query row = TMEM lane)
//   warps 8-11    softmax group 1
// TMEM columns (AttnTmem): S0 [0,128), S1 [128,256); dh 64: O0 [256,320), O1 [320,384),
// P0 [384,448), P1 [448,512); dh 80: O0 [256,336), O1 [384,464) and P_w over the first 64
// columns of S_w. P is bf16, two per column: the A operand of P*V. Keeping P apart from S (when
// it fits) lets Q*K^T of tile n+2 start while P*V of tile n still reads P.
// Barrier phases count uses across items: every role walks the same items and tiles in order.
template <int DH>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
           const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tq_tail,
           const __grid_constant__ CUtensorMap tk_tail, const __grid_constant__ CUtensorMap tv_tail,
           const AttnParams P, int* status) {
  using S = AttnSmem<DH>;
  using T = AttnTmem<DH>;
  constexpr int NS = S::kStages;
  constexpr bool kSplitHandoff = T::kSeparateP;   // P handed to P*V in two halves
  constexpr bool kHasTail = S::kTail > 0;
  // Epilogue: dh 80 lets group 1 merge and emit each item while group 0 moves on to the next
  // (measured faster there: ViT-H 284 -> 273 us); dh 64 keeps both groups on the merge (the
  // one-group form measured slower: ViT-B 52.8 -> 55.2 us).
  constexpr bool kOneGroupEpi = DH == 80;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  float* s_m = reinterpret_cast<float*>(smem + S::kML);   // [2][128] group 0's, by item parity
  float* s_l = s_m + 2 * kBM;                              // [2][128]
  int* s_dst = reinterpret_cast<int*>(smem + S::kDst);     // [128] destination token or -1
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* q_full = bars + 0;                 // [2] Q buffer landed
  uint64_t* q_empty = q_full + 2;              // [2] Q*K^T of the buffer's item done
  uint64_t* kv_full = q_empty + 2;             // [NS] K and V of a stage landed
  uint64_t* kv_empty = kv_full + NS;           // [NS] P*V of the stage's tile done (K, V free)
  uint64_t* s_full = kv_empty + NS;            // [2] S_w computed
  uint64_t* s_free = s_full + 2;               // [2] S_w read into registers by its group
  uint64_t* p_full = s_free + 2;               // [2][2] half h of P_w written (O_w rescaled first)
  uint64_t* o_done = p_full + 4;               // an item's last P*V done
  // [2] by item parity: group 0's m, l of the item written. Two, so that group 0 (which moves on
  // to the next item at once) cannot complete a second phase before group 1 has waited the first.
  uint64_t* ml_ready = o_done + 1;
  uint64_t* o_free = ml_ready + 2;             // O0, O1 of the item read (next item may reuse them)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_free + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = (P.N + kBM - 1) / kBM;
  const int n_items = nq * P.U * P.heads;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 128);
      mbar_init(p_full + 2 * i, 128);
      mbar_init(p_full + 2 * i + 1, 128);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    mbar_init(o_done, 1);
    if constexpr (kOneGroupEpi) {
      mbar_init(ml_ready, 128);
      mbar_init(ml_ready + 1, 128);
      mbar_init(o_free, 128);
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();   // Q, K, V and perm come from the work before this launch
  griddep_launch();

  // An mbarrier wait whose result gates the next instruction costs ~150 cycles even when the
  // phase has already completed, so the two MMA streams get their own issuing threads: one for
  // Q*K^T, one for P*V. Their data dependencies all go through the barriers above.
  if (warp < 4) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0 && lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      bool ok = true;
      int gn = 0;   // tiles loaded so far (all items)
      for (int it = blockIdx.x, li = 0; ok && it < n_items; it += gridDim.x, ++li) {
        const Item I = item_of(it, nq, P);
        const int qb = li & 1;
        if (li >= 2 && !(ok = mbar_wait(q_empty + qb, ((li >> 1) - 1) & 1, abort, status))) break;
        uint8_t* qbuf = smem + S::kQ + qb * S::kTileBytes;
        mbar_expect_tx(q_full + qb, S::kMain + S::kTailBytes);
        tma_load_3d(qbuf, &tq, q_full + qb, 0, I.q0, I.uh);
        if (kHasTail) tma_load_3d(qbuf + S::kMain, &tq_tail, q_full + qb, 64, I.q0, I.uh);
        const int nt = I.tiles.count();
        for (int n = 0; n < nt; ++n, ++gn) {
          const int st = gn % NS;
          const int c0 = I.tiles.tile(n) * kBN;
          if (gn >= NS && !(ok = mbar_wait(kv_empty + st, ((gn / NS) - 1) & 1, abort, status)))
            break;
          uint8_t* kb = smem + S::kK + st * S::kTileBytes;
          uint8_t* vb = smem + S::kV + st * S::kTileBytes;
          mbar_expect_tx(kv_full + st, 2 * (S::kMain + S::kTailBytes));
          tma_load_3d(kb, &tk, kv_full + st, 0, c0, I.uh);
          if (kHasTail) tma_load_3d(kb + S::kMain, &tk_tail, kv_full + st, 64, c0, I.uh);
          tma_load_3d(vb, &tv, kv_full + st, 0, c0, I.uh);
          if (kHasTail) tma_load_3d(vb + S::kMain, &tv_tail, kv_full + st, 64, c0, I.uh);
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------ Q*K^T issuer ------------------------------
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      bool ok = true;
      int gn = 0;
      int uses[2] = {0, 0};     // tiles computed into S_w so far
      int last[2] = {0, 0};     // global index of the tile that last used S_w
      for (int it = blockIdx.x, li = 0; ok && it < n_items; it += gridDim.x, ++li) {
        const Item I = item_of(it, nq, P);
        const int qb = li & 1;
        if (!(ok = mbar_wait(q_full + qb, (li >> 1) & 1, abort, status))) break;
        const uint32_t q_addr = smem_u32(smem + S::kQ + qb * S::kTileBytes);
        const int nt = I.tiles.count();
        for (int n = 0; n < nt; ++n, ++gn) {
          const int st = gn % NS, w = n & 1;
          if (uses[w] > 0) {
            // S_w is reusable once its previous tile's S is in its group's registers (P apart
            // from S), or once that tile's P*V is done (P over S).
            if constexpr (T::kSeparateP)
              ok = mbar_wait(s_free + w, (uses[w] - 1) & 1, abort, status);
            else
              ok = mbar_wait(kv_empty + last[w] % NS, (last[w] / NS) & 1, abort, status);
            if (!ok) break;
          }
          if (!(ok = mbar_wait(kv_full + st, (gn / NS) & 1, abort, status))) break;
          tc_fence_after();
          const uint32_t k_addr = smem_u32(smem + S::kK + st * S::kTileBytes);
          const uint32_t d = tmem + T::kS + w * T::kSStride;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ss(d, smem_desc(q_addr + kk * 32, 16, 1024, kSwizzle128B),
                         smem_desc(k_addr + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, kk > 0);
          if (kHasTail)
            umma_bf16_ss(d, smem_desc(q_addr + S::kMain, 16, 256, kSwizzle32B),
                         smem_desc(k_addr + S::kMain, 16, 256, kSwizzle32B), idesc_qk, 1);
          umma_commit(s_full + w);
          ++uses[w];
          last[w] = gn;
        }
        if (!ok) break;
        umma_commit(q_empty + qb);   // the Q buffer is free once this item's Q*K^T are done
      }
    } else if (warp == 2 && lane == 0) {
      // ------------------------------ P*V issuer --------------------------------
      // P_w of tile n exists only after S of tile n, which followed that stage's K/V landing
      // (observed by the Q*K^T issuer), so V is ready whenever P is.
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, 64, false, true);
      constexpr uint32_t idesc_pv_tail = idesc_bf16_f32(kBM, 16, false, true);
      bool ok = true;
      int gn = 0;
      int uses[2] = {0, 0};   // P_w handed over so far (p_full phases)
      for (int it = blockIdx.x, li = 0; ok && it < n_items; it += gridDim.x, ++li) {
        const int nt = item_of(it, nq, P).tiles.count();
        // The item's first P*V into O_w overwrites it: the previous item's epilogue must have
        // read O0 and O1.
        if (kOneGroupEpi && li > 0 && !(ok = mbar_wait(o_free, (li - 1) & 1, abort, status)))
          break;
        for (int n = 0; n < nt; ++n, ++gn) {
          const int st = gn % NS, w = n & 1;
          const uint32_t v_addr = smem_u32(smem + S::kV + st * S::kTileBytes);
          const uint32_t a = tmem + T::kP + w * T::kPStride;   // P_w
          const uint32_t d = tmem + T::kO + w * T::kOStride;
          // The first tile of each group overwrites O_w: released by o_free above, or (two-group
          // epilogue) by the group itself, which read the previous item's O before handing over
          // this P.
          const uint32_t acc = n >= 2;
          // P arrives in two halves (keys 0-63, 64-127): the first half's MMAs run while the
          // softmax still computes the second.
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            if (kk % (kBN / 32) == 0) {
              if (!(ok = mbar_wait(p_full + 2 * w + kk / (kBN / 32), uses[w] & 1, abort, status)))
                break;
              tc_fence_after();
            }
            umma_bf16_ts(d, a + kk * 8, smem_desc(v_addr + kk * 2048, kBN * 128, 1024, kSwizzle128B),
                         idesc_pv, acc | (kk > 0));
            if (kHasTail)
              umma_bf16_ts(d + 64, a + kk * 8,
                           smem_desc(v_addr + S::kMain + kk * 512, kBN * 32, 256, kSwizzle32B),
                           idesc_pv_tail, acc | (kk > 0));
          }
          if (!ok) break;
          ++uses[w];
          umma_commit(kv_empty + st);   // Q*K^T of this tile finished before its P existed
        }
        if (!ok) break;
        umma_commit(o_done);   // phase = the item's parity in this CTA's sequence
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------ softmax groups ----------------------------
    const int grp = (warp - 4) >> 2;                    // 0 or 1
    const int row = 32 * (warp & 3) + lane;             // TMEM lane == query row
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t t_s = tmem + T::kS + grp * T::kSStride + lane_off;
    const uint32_t t_p = tmem + T::kP + grp * T::kPStride + lane_off;
    const uint32_t t_o = tmem + T::kO + grp * T::kOStride + lane_off;
    const int b4 = P.b * kStripes;
    const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
    bool ok = true;
    int gn0 = 0;           // global index of the item's first tile
    int uses = 0;          // tiles of this group so far (s_full phases)
    bool s_ready = false;  // the next s_full phase was already seen complete (non-blocking test)
    int g_last = -1;       // global index of this group's previous tile (any item), -1: none
    for (int it = blockIdx.x, li = 0; it < n_items; it += gridDim.x, ++li) {
      const Item I = item_of(it, nq, P);
      const int nt = I.tiles.count();
      const int qrow = I.q0 + row;
      // Destination token of the row: loaded now, used in the epilogue (the load's latency
      // overlaps the item's tiles).
      const bool store = qrow < P.N;
      const int u_i = I.uh / P.heads, h_i = I.uh - u_i * P.heads;
      const int perm_t =
          store ? __ldg(P.perm + (size_t)u_i * P.N + blockmajor_to_canonical(qrow, P.b, P.L)) : 0;
      const int a_q = min(qrow, P.N - 1) / b4;
      const int s_q = band_start(a_q, P.W, P.nb);
      const int band_lo = s_q * b4, band_hi = (s_q + P.W) * b4, glob_hi = P.g * b4;
      float m_ref = -INFINITY, l_run = 0.f;
      int j = 0;
      for (int n = grp; ok && n < nt; n += 2, ++j) {
        // Warp-collective wait: either every lane goes on to the .sync.aligned TMEM ops or none.
        if (!__all_sync(0xffffffffu, s_ready))
          ok = __all_sync(0xffffffffu, mbar_wait(s_full + grp, uses & 1, abort, status));
        ++uses;
        if (!ok) break;
        tc_fence_after();
        float sv[kBN];
        {
          uint32_t r[128];
          tmem_ld128(t_s, r);
#pragma unroll
          for (int i = 0; i < kBN; ++i) sv[i] = __uint_as_float(r[i]);
        }
        // Has P*V of this group's previous tile (in this item or the last) released P_w? Tested
        // now, used after the row max, so the test's latency is hidden behind the max.
        // (With the two-group epilogue both groups waited for the previous item's P*V, so only
        // this item's earlier tiles count.)
        int gprev = n >= 2 ? gn0 + n - 2 : -1;
        if constexpr (kOneGroupEpi) {
          gprev = g_last;
          g_last = gn0 + n;
        }
        bool prev_pv_done = true;
        if constexpr (T::kSeparateP) {
          tc_fence_before();
          mbar_arrive(s_free + grp);   // S_w may now be overwritten by the next Q*K^T into it
          if (gprev >= 0) prev_pv_done = mbar_test(kv_empty + gprev % NS, (gprev / NS) & 1);
        }
        const int c0 = I.tiles.tile(n) * kBN;
        const bool full = tile_full(c0, P);
        if (!full) {
          // The row's kept keys in this tile are two runs, [0, e0) and [s1, e1) relative to c0:
          // turned into four 32-bit column masks, so the per-key test has no branch.
          const int e0 = min(glob_hi, P.N) - c0, s1 = band_lo - c0, e1 = min(band_hi, P.N) - c0;
          uint32_t km[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) km[k] = run_bits(0, e0, 32 * k) | run_bits(s1, e1, 32 * k);
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            sv[i] = (km[i >> 5] >> (i & 31)) & 1u ? sv[i] : -INFINITY;
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
        const float x_max = fmaxf(fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5])),
                                  fmaxf(mx[6], mx[7])) *
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
        // The group's previous P*V must be done before P_w is rewritten and O_w rescaled (with P
        // over S it already is: this S was computed after that P*V).
        if constexpr (T::kSeparateP) {
          if (gprev >= 0) {
            if (!__all_sync(0xffffffffu, prev_pv_done)) {
              ok = __all_sync(0xffffffffu,
                              mbar_wait(kv_empty + gprev % NS, (gprev / NS) & 1, abort, status));
              if (!ok) break;
            }
            tc_fence_after();
          }
        }
        // P row as bf16 pairs (column i holds keys 2i, 2i+1), written to P_w (its own columns, or
        // over S_w, whose row is already in registers) in two halves of 32 columns. 2^x runs on
        // MUFU in f32 (measured faster here than packed-f16 MUFU or the FMA-pipe exp2_poly2, which
        // full tiles can route kPolyPairs of every 16 pairs to). Masked keys give ex2(-inf) = 0.
        auto softmax_row = [&](auto poly_tag) {
          constexpr bool kPoly = decltype(poly_tag)::value;
#pragma unroll
          for (int half = 0; half < 2; ++half) {
            uint32_t pw[32];
#pragma unroll
            for (int i2 = 0; i2 < 32; ++i2) {
              const int i = 64 * half + 2 * i2;
              float x0, x1, p0, p1;
              f2_unpack(f2_fma(f2_pack(sv[i], sv[i + 1]), scale2, nref2), x0, x1);
              if (kPoly && (i2 & 15) < kPolyPairs) {
                exp2_poly2(x0, x1, p0, p1);
              } else {
                p0 = ex2_mufu(x0);
                p1 = ex2_mufu(x1);
              }
              if (i2 & 1)
                sum2b = f2_add(sum2b, f2_pack(p0, p1));
              else
                sum2a = f2_add(sum2a, f2_pack(p0, p1));
              pw[i2] = pack_bf16_pos(p0, p1);   // p >= 0: integer-pipe rounding
            }
            tmem_st32_async(t_p + 32 * half, pw);
            if constexpr (kSplitHandoff) {
              // Each half is handed over as soon as it is written.
              if (half == 0 && rescale && j > 0) {
                // O_w holds the group's earlier tiles (their P*V completed: waited above); it is
                // rescaled before this tile's first P*V accumulates into it.
#pragma unroll 1
                for (int c = 0; c < (DH + 31) / 32; ++c) {
                  uint32_t o[32];
                  tmem_ld32(t_o + c * 32, o);
#pragma unroll
                  for (int i = 0; i < 32; ++i)
                    o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
                  tmem_st32_async(t_o + c * 32, o);
                }
              }
              tmem_st_wait();   // P (and O) complete in TMEM before the arrive releases it
              tc_fence_before();
              mbar_arrive(p_full + 2 * grp + half);
            }
          }
        };
        if (full)
          softmax_row(std::integral_constant<bool, true>());
        else
          softmax_row(std::integral_constant<bool, false>());
        // Is S of this group's next tile already there? Tested here, where the result is not
        // needed at once, instead of by a blocking wait at the top of the next iteration.
        s_ready = mbar_test(s_full + grp, uses & 1);
        float sa0, sa1;
        f2_unpack(f2_add(sum2a, sum2b), sa0, sa1);
        l_run += sa0 + sa1;
        if constexpr (!kSplitHandoff) {
          // Both halves go together (the split costs the dh 80 variant registers it does not
          // have): P written, then O_w rescaled if needed (its earlier P*V completed before this
          // S was committed), then the hand-over.
          tmem_st_wait();
          if (rescale && j > 0) {
#pragma unroll 1
            for (int c = 0; c < (DH + 31) / 32; ++c) {
              uint32_t o[32];
              tmem_ld32(t_o + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32(t_o + c * 32, o);
            }
          }
          tc_fence_before();
          mbar_arrive(p_full + 2 * grp);
          mbar_arrive(p_full + 2 * grp + 1);
        }
      }
      if constexpr (kOneGroupEpi) {
        // ---- merge both groups' partial rows and scatter them to out[u, perm[p], h, :] ----
        // Group 1 merges and emits the item; group 0 hands over its row max and sum and goes on to
        // the next item at once (its first P*V there waits for o_free, i.e. for group 1 to have
        // read O0 and O1). Every wait and barrier below is passed also after a failed wait.
        const int mb = li & 1;   // this item's m, l buffer
        if (grp == 0) {
          s_m[mb * kBM + row] = m_ref;
          s_l[mb * kBM + row] = l_run;
          mbar_arrive(ml_ready + mb);
        } else {
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(ml_ready + mb, (li >> 1) & 1, abort, status));
          if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, li & 1, abort, status));
          tc_fence_after();
          const float m0 = s_m[mb * kBM + row], l0 = s_l[mb * kBM + row];
          const float m1 = m_ref, l1 = l_run;
          const float mm = fmaxf(m0, m1);
          const float a0 = (m0 == -INFINITY) ? 0.f : ex2_mufu(m0 - mm);
          const float a1 = (m1 == -INFINITY) ? 0.f : ex2_mufu(m1 - mm);
          const float L = l0 * a0 + l1 * a1;
          const float inv = L > 0.f ? 1.f / L : 0.f;
          const float f0 = a0 * inv, f1 = a1 * inv;
          const bool has0 = nt > 0, has1 = nt > 1;   // a group with no tile has a stale O
          // The previous item's copy-out is finished before the staging rows are rewritten.
          named_barrier(2, 128);
          // Normalised row -> shared staging (rows padded by 16 bytes against bank conflicts); then
          // the group copies whole rows out, so that each warp store covers contiguous rows.
          const uint32_t stage_row = smem_u32(smem + S::kStage) + row * S::kStageStride;
          if (ok) {
            const uint32_t o0 = tmem + T::kO + lane_off;
            const uint32_t o1 = o0 + T::kOStride;
            auto emit8 = [&](const uint32_t* u0, const uint32_t* u1, int col) {
              float v[8];
  #pragma unroll
              for (int i = 0; i < 8; ++i)
                v[i] = (has0 ? __uint_as_float(u0[i]) * f0 : 0.f) +
                       (has1 ? __uint_as_float(u1[i]) * f1 : 0.f);
              st_shared_v4(stage_row + col * 2, pack_bf16(v[0], v[1]), pack_bf16(v[2], v[3]),
                           pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
            };
  #pragma unroll 1
            for (int c = 0; c < DH / 32; ++c) {   // 32 columns of O0 and O1 at a time
              uint32_t x0[32], x1[32];
              tmem_ld32_pair(o0 + c * 32, o1 + c * 32, x0, x1);
  #pragma unroll
              for (int e = 0; e < 4; ++e) emit8(x0 + 8 * e, x1 + 8 * e, c * 32 + 8 * e);
            }
            if constexpr (DH % 32) {   // dh 80: columns 64..79
  #pragma unroll
              for (int c = (DH / 32) * 32; c < DH; c += 8) {
                uint32_t x0[8], x1[8];
                tmem_ld8_pair(o0 + c, o1 + c, x0, x1);
                emit8(x0, x1, c);
              }
            }
            s_dst[row] = store ? dst_token(perm_t, P.N, status) : -1;
          }
          tc_fence_before();
          mbar_arrive(o_free);   // O0, O1 read: the next item's first P*V may overwrite them
          named_barrier(2, 128);
          if (ok) {
            constexpr int kCpr = DH / 8;                  // 16-byte chunks per row
            const int tid = threadIdx.x - 256;            // 0..127: group 1
            const uint32_t stage = smem_u32(smem + S::kStage);
            uint8_t* out_uh = reinterpret_cast<uint8_t*>(P.out) +
                              ((size_t)u_i * P.N * P.heads + h_i) * DH * 2;
  #pragma unroll 2
            for (int k = 0; k < kBM * kCpr / 128; ++k) {
              const int q = tid + 128 * k;
              const int r = q / kCpr, c = q - r * kCpr;
              const int t = s_dst[r];
              if (t >= 0) {
                const uint4 v = ld_shared_v4(stage + r * S::kStageStride + c * 16);
                *reinterpret_cast<uint4*>(out_uh + (size_t)t * P.heads * DH * 2 + c * 16) = v;
              }
            }
          }
        }
      } else {
        // ---- merge both groups' partial rows and scatter them to out[u, perm[p], h, :] ----
        // Every softmax thread passes both named barriers once per item, also after a failed wait.
        s_m[grp * kBM + row] = m_ref;
        s_l[grp * kBM + row] = l_run;
        if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done, li & 1, abort, status));
        tc_fence_after();
        named_barrier(1, 256);
        constexpr int kCols = DH / 2;   // this group's output columns [grp*kCols, (grp+1)*kCols)
        uint32_t x0[32], x1[32], y0[8], y1[8];   // columns 0-31 and (dh 80) 32-39 of O0, O1
        float m0 = 0.f, m1 = 0.f, l0 = 0.f, l1 = 0.f;
        if (ok) {
          m0 = s_m[row];
          m1 = s_m[kBM + row];
          l0 = s_l[row];
          l1 = s_l[kBM + row];
          const uint32_t o0 = tmem + T::kO + lane_off + grp * kCols;
          const uint32_t o1 = o0 + T::kOStride;
          tmem_ld32_pair(o0, o1, x0, x1);
          if constexpr (kCols > 32) tmem_ld8_pair(o0 + 32, o1 + 32, y0, y1);
        }
        // Both groups have read O0 and O1 (and m, l) before either hands the next item's first P
        // to the P*V issuer, whose first MMA into O_w overwrites it.
        tc_fence_before();
        named_barrier(1, 256);
        // Normalised half-row -> shared staging; then the 256 threads copy whole rows out, so
        // that each warp store covers four contiguous 128-byte rows (dh 64) instead of 32 rows.
        const uint32_t stage_row = smem_u32(smem + S::kStage) + row * S::kStageStride;
        if (ok) {
          const float mm = fmaxf(m0, m1);
          const float a0 = (m0 == -INFINITY) ? 0.f : ex2_mufu(m0 - mm);
          const float a1 = (m1 == -INFINITY) ? 0.f : ex2_mufu(m1 - mm);
          const float L = l0 * a0 + l1 * a1;
          const float inv = L > 0.f ? 1.f / L : 0.f;
          const float f0 = a0 * inv, f1 = a1 * inv;
          // A group with no tile in this item has a stale O: select, do not multiply by zero.
          const bool has0 = nt > 0, has1 = nt > 1;
  #pragma unroll
          for (int c = 0; c < kCols / 8; ++c) {
            float v[8];
  #pragma unroll
            for (int i = 0; i < 8; ++i) {
              const uint32_t u0 = c < 4 ? x0[8 * c + i] : y0[i];
              const uint32_t u1 = c < 4 ? x1[8 * c + i] : y1[i];
              v[i] = (has0 ? __uint_as_float(u0) * f0 : 0.f) + (has1 ? __uint_as_float(u1) * f1 : 0.f);
            }
            st_shared_v4(stage_row + grp * kCols * 2 + c * 16, pack_bf16(v[0], v[1]),
                         pack_bf16(v[2], v[3]), pack_bf16(v[4], v[5]), pack_bf16(v[6], v[7]));
          }
          if (grp == 0) s_dst[row] = store ? dst_token(perm_t, P.N, status) : -1;
        }
        named_barrier(1, 256);
        if (ok) {
          constexpr int kCpr = DH / 8;                  // 16-byte chunks per row
          const int tid = threadIdx.x - 128;            // 0..255
          const uint32_t stage = smem_u32(smem + S::kStage);
          uint8_t* out_uh = reinterpret_cast<uint8_t*>(P.out) +
                            ((size_t)u_i * P.N * P.heads + h_i) * DH * 2;
  #pragma unroll
          for (int k = 0; k < kBM * kCpr / 256; ++k) {
            const int q = tid + 256 * k;
            const int r = q / kCpr, c = q - r * kCpr;
            const int t = s_dst[r];
            if (t >= 0) {
              const uint4 v = ld_shared_v4(stage + r * S::kStageStride + c * 16);
              *reinterpret_cast<uint4*>(out_uh + (size_t)t * P.heads * DH * 2 + c * 16) = v;
            }
          }
        }
      }
      gn0 += nt;
    }
  }
  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------------------------------------
// Short items (windowed blocks: about two key tiles per item): whole items per softmax group.
// ---------------------------------------------------------------------------------------------
// With two key tiles per item, splitting an item's tiles between the two groups (k_attn) leaves
// each group one tile per item, then a wait for both P*V and a merged epilogue behind two
// CTA-wide barriers: the exposed latencies dominate. Here the CTA takes its items in pairs (A =
// its item 2p, B = its item 2p+1); group 0 runs A and group 1 runs B, each a whole item with its
// own Q buffer, S, P and O, each normalising and scattering its own rows (no merge). The pair's
// key tiles go through one K/V ring in the order A_0, B_0, A_1, B_1, ... (kInterleave) or
// A_0, A_1, ..., B_0, B_1, ... . Head dim 64 (the windowed configurations).
struct AttnPairSmem {
  static constexpr int kTileBytes = kBM * 128;                  // 128 rows x 64 bf16
  static constexpr int kStages = 4;                             // depth of the K/V ring
  static constexpr int kQ = 0;                                  // Q of A, Q of B
  static constexpr int kK = 2 * kTileBytes;
  static constexpr int kV = kK + kStages * kTileBytes;
  static constexpr int kStageStride = 64 * 2 + 16;              // padded output staging rows
  static constexpr int kStage = kV + kStages * kTileBytes;      // [2 groups][128 rows]
  static constexpr int kDst = kStage + 2 * kBM * kStageStride;  // [2 groups][128] tokens
  static constexpr int kBar = kDst + 2 * kBM * 4;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;
  static_assert(kAlloc <= 227 * 1024, "attention shared memory above the per-CTA limit");
};

// Position of tile n of the pair's item g in the pair's ring order.
template <bool kInterleave>
__device__ __forceinline__ int pair_tile_index(int g, int n, int ntA, int ntB) {
  if (kInterleave) return min(n, ntA) + min(n, ntB) + (g == 1 && n < ntA ? 1 : 0);
  return g == 0 ? n : ntA + n;
}

template <bool kInterleave>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_pairs(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                 const __grid_constant__ CUtensorMap tv, const AttnParams P, int* status) {
  using S = AttnPairSmem;
  using T = AttnTmem<64>;
  constexpr int NS = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  int* s_dst = reinterpret_cast<int*>(smem + S::kDst);     // [2][128] destination token or -1
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* q_full = bars + 0;                 // [2] Q of group g's item landed
  uint64_t* q_empty = q_full + 2;              // [2] Q*K^T of group g's item done
  uint64_t* kv_full = q_empty + 2;             // [NS]
  uint64_t* kv_empty = kv_full + NS;           // [NS] P*V of the stage's tile done
  uint64_t* s_full = kv_empty + NS;            // [2] S_g computed
  uint64_t* s_free = s_full + 2;               // [2] S_g read into registers
  uint64_t* p_full = s_free + 2;               // [2][2] half h of P_g written
  uint64_t* o_done = p_full + 4;               // [2] last P*V of group g's item done
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(o_done + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nq = (P.N + kBM - 1) / kBM;
  const int n_items = nq * P.U * P.heads;
  const int G = gridDim.x;

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(q_full + i, 1);
      mbar_init(q_empty + i, 1);
      mbar_init(s_full + i, 1);
      mbar_init(s_free + i, 128);
      mbar_init(p_full + 2 * i, 128);
      mbar_init(p_full + 2 * i + 1, 128);
      mbar_init(o_done + i, 1);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  griddep_wait();   // Q, K, V and perm come from the work before this launch
  griddep_launch();

  // Every role walks the pairs p = 0, 1, ... with item A = blockIdx.x + 2pG and B = A + G; every
  // item has at least one key tile (its own band).
  if (warp < 4) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0 && lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      bool ok = true;
      int gn0 = 0;   // ring index of the pair's first tile
      for (int p = 0, itA = blockIdx.x; ok && itA < n_items; ++p, itA += 2 * G) {
        const bool hasB = itA + G < n_items;
        const Item A = item_of(itA, nq, P);
        Item B = A;
        if (hasB) B = item_of(itA + G, nq, P);
        const int ntA = A.tiles.count(), ntB = hasB ? B.tiles.count() : 0;
        if (p >= 1 && !(ok = mbar_wait(q_empty + 0, (p - 1) & 1, abort, status))) break;
        mbar_expect_tx(q_full + 0, S::kTileBytes);
        tma_load_3d(smem + S::kQ, &tq, q_full + 0, 0, A.q0, A.uh);
        if (hasB) {
          if (p >= 1 && !(ok = mbar_wait(q_empty + 1, (p - 1) & 1, abort, status))) break;
          mbar_expect_tx(q_full + 1, S::kTileBytes);
          tma_load_3d(smem + S::kQ + S::kTileBytes, &tq, q_full + 1, 0, B.q0, B.uh);
        }
        for (int j = 0; ok && j < ntA + ntB; ++j) {
          // tile j of the ring order -> (item, tile)
          int g, n;
          if (kInterleave) {
            const int both = 2 * min(ntA, ntB);
            if (j < both) {
              g = j & 1;
              n = j >> 1;
            } else {
              g = ntA > ntB ? 0 : 1;
              n = (j - both) + min(ntA, ntB);
            }
          } else {
            g = j < ntA ? 0 : 1;
            n = j < ntA ? j : j - ntA;
          }
          const int gn = gn0 + j, st = gn % NS;
          if (gn >= NS && !(ok = mbar_wait(kv_empty + st, ((gn / NS) - 1) & 1, abort, status)))
            break;
          const int c0 = (g ? B.tiles.tile(n) : A.tiles.tile(n)) * kBN;
          const int uh = g ? B.uh : A.uh;
          mbar_expect_tx(kv_full + st, 2 * S::kTileBytes);
          tma_load_3d(smem + S::kK + st * S::kTileBytes, &tk, kv_full + st, 0, c0, uh);
          tma_load_3d(smem + S::kV + st * S::kTileBytes, &tv, kv_full + st, 0, c0, uh);
        }
        gn0 += ntA + ntB;
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------ Q*K^T issuer ------------------------------
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      bool ok = true;
      int gn0 = 0;
      int uses[2] = {0, 0};   // tiles computed into S_g so far
      for (int p = 0, itA = blockIdx.x; ok && itA < n_items; ++p, itA += 2 * G) {
        const bool hasB = itA + G < n_items;
        const int ntA = item_of(itA, nq, P).tiles.count();
        const int ntB = hasB ? item_of(itA + G, nq, P).tiles.count() : 0;
        bool q_in0 = false, q_in1 = false;
        for (int j = 0; ok && j < ntA + ntB; ++j) {
          int g, n;
          if (kInterleave) {
            const int both = 2 * min(ntA, ntB);
            g = j < both ? (j & 1) : (ntA > ntB ? 0 : 1);
            n = j < both ? (j >> 1) : (j - both) + min(ntA, ntB);
          } else {
            g = j < ntA ? 0 : 1;
            n = j < ntA ? j : j - ntA;
          }
          bool& q_in = g ? q_in1 : q_in0;
          if (!q_in) {
            if (!(ok = mbar_wait(q_full + g, p & 1, abort, status))) break;
            q_in = true;
          }
          const int gn = gn0 + j, st = gn % NS;
          const int ug = g ? uses[1] : uses[0];
          // S_g is reusable once its previous tile's S is in its group's registers.
          if (ug > 0 && !(ok = mbar_wait(s_free + g, (ug - 1) & 1, abort, status))) break;
          if (!(ok = mbar_wait(kv_full + st, (gn / NS) & 1, abort, status))) break;
          tc_fence_after();
          const uint32_t q_addr = smem_u32(smem + S::kQ + g * S::kTileBytes);
          const uint32_t k_addr = smem_u32(smem + S::kK + st * S::kTileBytes);
          const uint32_t d = tmem + T::kS + g * T::kSStride;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_ss(d, smem_desc(q_addr + kk * 32, 16, 1024, kSwizzle128B),
                         smem_desc(k_addr + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, kk > 0);
          umma_commit(s_full + g);
          if (g) ++uses[1]; else ++uses[0];
          if (n == (g ? ntB : ntA) - 1) umma_commit(q_empty + g);   // the item's Q is free
        }
        gn0 += ntA + ntB;
      }
    } else if (warp == 2 && lane == 0) {
      // ------------------------------ P*V issuer --------------------------------
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, 64, false, true);
      bool ok = true;
      int gn0 = 0;
      int uses[2] = {0, 0};   // P_g handed over so far (p_full phases)
      for (int p = 0, itA = blockIdx.x; ok && itA < n_items; ++p, itA += 2 * G) {
        const bool hasB = itA + G < n_items;
        const int ntA = item_of(itA, nq, P).tiles.count();
        const int ntB = hasB ? item_of(itA + G, nq, P).tiles.count() : 0;
        for (int j = 0; ok && j < ntA + ntB; ++j) {
          int g, n;
          if (kInterleave) {
            const int both = 2 * min(ntA, ntB);
            g = j < both ? (j & 1) : (ntA > ntB ? 0 : 1);
            n = j < both ? (j >> 1) : (j - both) + min(ntA, ntB);
          } else {
            g = j < ntA ? 0 : 1;
            n = j < ntA ? j : j - ntA;
          }
          const int gn = gn0 + j, st = gn % NS;
          const int ug = g ? uses[1] : uses[0];
          const uint32_t v_addr = smem_u32(smem + S::kV + st * S::kTileBytes);
          const uint32_t a = tmem + T::kP + g * T::kPStride;
          const uint32_t d = tmem + T::kO + g * T::kOStride;
          // An item's first tile overwrites O_g: its group read the previous item's O in the
          // epilogue before handing over this P.
          const uint32_t acc = n > 0;
#pragma unroll
          for (int kk = 0; kk < kBN / 16; ++kk) {
            if (kk % (kBN / 32) == 0) {
              if (!(ok = mbar_wait(p_full + 2 * g + kk / (kBN / 32), ug & 1, abort, status)))
                break;
              tc_fence_after();
            }
            umma_bf16_ts(d, a + kk * 8, smem_desc(v_addr + kk * 2048, kBN * 128, 1024, kSwizzle128B),
                         idesc_pv, acc | (kk > 0));
          }
          if (!ok) break;
          if (g) ++uses[1]; else ++uses[0];
          umma_commit(kv_empty + st);
          if (n == (g ? ntB : ntA) - 1) umma_commit(o_done + g);   // the item's O is complete
        }
        gn0 += ntA + ntB;
      }
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------ softmax groups ----------------------------
    const int grp = (warp - 4) >> 2;                    // 0: the pairs' A items, 1: their B items
    const int row = 32 * (warp & 3) + lane;             // TMEM lane == query row
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t t_s = tmem + T::kS + grp * T::kSStride + lane_off;
    const uint32_t t_p = tmem + T::kP + grp * T::kPStride + lane_off;
    const uint32_t t_o = tmem + T::kO + grp * T::kOStride + lane_off;
    const uint32_t bar = 2 + grp;                       // the group's named barrier
    const uint32_t stage_row = smem_u32(smem + S::kStage) + (grp * kBM + row) * S::kStageStride;
    int* dst_tok = s_dst + grp * kBM;
    const int b4 = P.b * kStripes;
    const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
    bool ok = true;
    int gn0 = 0;           // ring index of the pair's first tile
    int uses = 0;          // tiles of this group so far (s_full phases)
    bool s_ready = false;  // the next s_full phase was already seen complete
    for (int p = 0, itA = blockIdx.x; itA < n_items; ++p, itA += 2 * G) {
      const int itB = itA + G;
      const bool hasB = itB < n_items;
      if (grp == 1 && !hasB) break;                    // the CTA's last pair has no B
      const Item I = item_of(grp ? itB : itA, nq, P);
      const int nt = I.tiles.count();
      const int nt_other = grp ? item_of(itA, nq, P).tiles.count()
                               : (hasB ? item_of(itB, nq, P).tiles.count() : 0);
      const int ntA = grp ? nt_other : nt, ntB = grp ? nt : nt_other;
      const int qrow = I.q0 + row;
      const bool store = qrow < P.N;
      const int u_i = I.uh / P.heads, h_i = I.uh - u_i * P.heads;
      const int perm_t =
          store ? __ldg(P.perm + (size_t)u_i * P.N + blockmajor_to_canonical(qrow, P.b, P.L)) : 0;
      const int a_q = min(qrow, P.N - 1) / b4;
      const int s_q = band_start(a_q, P.W, P.nb);
      const int band_lo = s_q * b4, band_hi = (s_q + P.W) * b4, glob_hi = P.g * b4;
      float m_ref = -INFINITY, l_run = 0.f;
      for (int n = 0; ok && n < nt; ++n) {
        if (!__all_sync(0xffffffffu, s_ready))
          ok = __all_sync(0xffffffffu, mbar_wait(s_full + grp, uses & 1, abort, status));
        ++uses;
        if (!ok) break;
        tc_fence_after();
        float sv[kBN];
        {
          uint32_t r[128];
          tmem_ld128(t_s, r);
#pragma unroll
          for (int i = 0; i < kBN; ++i) sv[i] = __uint_as_float(r[i]);
        }
        // P*V of the item's previous tile must be done before P_g is rewritten (the previous
        // item's are: the epilogue waited for them). Tested now, waited for after the row max.
        const int gprev = n >= 1 ? gn0 + pair_tile_index<kInterleave>(grp, n - 1, ntA, ntB) : 0;
        tc_fence_before();
        mbar_arrive(s_free + grp);   // S_g may now be overwritten by the next Q*K^T into it
        const bool prev_pv_done = n == 0 || mbar_test(kv_empty + gprev % NS, (gprev / NS) & 1);
        const int c0 = I.tiles.tile(n) * kBN;
        if (!tile_full(c0, P)) {
          const int e0 = min(glob_hi, P.N) - c0, s1 = band_lo - c0, e1 = min(band_hi, P.N) - c0;
          uint32_t km[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) km[k] = run_bits(0, e0, 32 * k) | run_bits(s1, e1, 32 * k);
#pragma unroll
          for (int i = 0; i < kBN; ++i)
            sv[i] = (km[i >> 5] >> (i & 31)) & 1u ? sv[i] : -INFINITY;
        }
        float mx[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmax3(sv[k], sv[k + 8], sv[k + 16]);
#pragma unroll
        for (int t = 3; t + 1 < 16; t += 2)
#pragma unroll
          for (int k = 0; k < 8; ++k) mx[k] = fmax3(mx[k], sv[k + 8 * t], sv[k + 8 * t + 8]);
#pragma unroll
        for (int k = 0; k < 8; ++k) mx[k] = fmaxf(mx[k], sv[k + 8 * 15]);
        const float x_max = fmaxf(fmaxf(fmax3(mx[0], mx[1], mx[2]), fmax3(mx[3], mx[4], mx[5])),
                                  fmaxf(mx[6], mx[7])) *
                            P.scale_log2;
        // Lazy rescale of the reference max, as in k_attn.
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
        uint64_t sum2a = 0, sum2b = 0;
        if (n >= 1) {
          if (!__all_sync(0xffffffffu, prev_pv_done)) {
            ok = __all_sync(0xffffffffu,
                            mbar_wait(kv_empty + gprev % NS, (gprev / NS) & 1, abort, status));
            if (!ok) break;
          }
          tc_fence_after();
        }
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t pw[32];
#pragma unroll
          for (int i2 = 0; i2 < 32; ++i2) {
            const int i = 64 * half + 2 * i2;
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(sv[i], sv[i + 1]), scale2, nref2), x0, x1);
            const float p0 = ex2_mufu(x0), p1 = ex2_mufu(x1);
            if (i2 & 1)
              sum2b = f2_add(sum2b, f2_pack(p0, p1));
            else
              sum2a = f2_add(sum2a, f2_pack(p0, p1));
            pw[i2] = pack_bf16_pos(p0, p1);
          }
          tmem_st32_async(t_p + 32 * half, pw);
          if (half == 0 && rescale && n > 0) {
            // O_g holds the item's earlier tiles (their P*V completed: waited above).
#pragma unroll 1
            for (int c = 0; c < 2; ++c) {
              uint32_t o[32];
              tmem_ld32(t_o + c * 32, o);
#pragma unroll
              for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
              tmem_st32_async(t_o + c * 32, o);
            }
          }
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(p_full + 2 * grp + half);
        }
        s_ready = mbar_test(s_full + grp, uses & 1);
        float sa0, sa1;
        f2_unpack(f2_add(sum2a, sum2b), sa0, sa1);
        l_run += sa0 + sa1;
      }
      // ---- the group's item: normalise its rows and scatter them to out[u, perm[p], h, :] ----
      // The group's threads all pass both named barriers once per item, also after a failed
      // wait.
      if (ok) ok = __all_sync(0xffffffffu, mbar_wait(o_done + grp, p & 1, abort, status));
      tc_fence_after();
      named_barrier(bar, 128);   // the group's previous copy-out is done with the staging rows
      if (ok) {
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        uint32_t x0[32], x1[32];
        tmem_ld32_pair(t_o, t_o + 32, x0, x1);
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const uint32_t* u = c < 4 ? x0 + 8 * c : x1 + 8 * (c - 4);
          st_shared_v4(stage_row + c * 16,
                       pack_bf16(__uint_as_float(u[0]) * inv, __uint_as_float(u[1]) * inv),
                       pack_bf16(__uint_as_float(u[2]) * inv, __uint_as_float(u[3]) * inv),
                       pack_bf16(__uint_as_float(u[4]) * inv, __uint_as_float(u[5]) * inv),
                       pack_bf16(__uint_as_float(u[6]) * inv, __uint_as_float(u[7]) * inv));
        }
        dst_tok[row] = store ? dst_token(perm_t, P.N, status) : -1;
      }
      tc_fence_before();   // O_g is read before the next item's first P goes to P*V
      named_barrier(bar, 128);
      if (ok) {
        constexpr int kCpr = 8;                          // 16-byte chunks per 64-column row
        const int tid = threadIdx.x - 128 * (1 + grp);   // 0..127 within the group
        const uint32_t stage = smem_u32(smem + S::kStage) + grp * kBM * S::kStageStride;
        uint8_t* out_uh =
            reinterpret_cast<uint8_t*>(P.out) + ((size_t)u_i * P.N * P.heads + h_i) * 64 * 2;
#pragma unroll 4
        for (int k = 0; k < kBM * kCpr / 128; ++k) {
          const int q = tid + 128 * k;
          const int r = q / kCpr, c = q - r * kCpr;
          const int t = dst_tok[r];
          if (t >= 0) {
            const uint4 v = ld_shared_v4(stage + r * S::kStageStride + c * 16);
            *reinterpret_cast<uint4*>(out_uh + (size_t)t * P.heads * 64 * 2 + c * 16) = v;
          }
        }
      }
      gn0 += ntA + ntB;
    }
  }
  tc_fence_before();
  cta_sync_converged();
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
  const int items = ((p.N + kBM - 1) / kBM) * p.U * p.heads;
  dim3 grid(std::max(1, std::min(items, p.sms)));
  return launch_pdl(k_attn<DH>, grid, dim3(kAttnThreads), S::kAlloc, st, *tq, *tk, *tv, *tq_tail,
                    *tk_tail, *tv_tail, p, status);
}

static cudaError_t launch_attn_pairs(const CUtensorMap* tq, const CUtensorMap* tk,
                                     const CUtensorMap* tv, const AttnParams& p, int* status,
                                     cudaStream_t st) {
  using S = AttnPairSmem;
  auto kernel = k_attn_pairs<kPairInterleave>;
  cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, S::kAlloc);
  if (e != cudaSuccess) return e;
  const int items = ((p.N + kBM - 1) / kBM) * p.U * p.heads;
  dim3 grid(std::max(1, std::min((items + 1) / 2, p.sms)));
  return launch_pdl(kernel, grid, dim3(kAttnThreads), S::kAlloc, st, *tq, *tk, *tv, p, status);
}

cudaError_t launch_attn(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* tq_tail, const CUtensorMap* tk_tail,
                        const CUtensorMap* tv_tail, const AttnParams& p, int dh, int* status,
                        cudaStream_t st) {
  if (dh == 64) {
    // Short items (at most kPairTiles key tiles per query tile, as in windowed blocks) go to the
    // whole-item-per-group kernel.
    const int nq = (p.N + kBM - 1) / kBM;
    int nt_max = 0;
    for (int qt = 0; qt < nq; ++qt)
      nt_max = std::max(nt_max,
                        key_tiles(qt * kBM, std::min(qt * kBM + kBM, p.N) - 1, qt, 0, p).count());
    if (nt_max <= kPairTiles) return launch_attn_pairs(tq, tk, tv, p, status, st);
    return launch_attn_dh<64>(tq, tk, tv, tq, tk, tv, p, status, st);
  }
  if (dh == 80) return launch_attn_dh<80>(tq, tk, tv, tq_tail, tk_tail, tv_tail, p, status, st);
  return cudaErrorInvalidValue;
}

cudaError_t set_wait_limit_attn(uint64_t ns) { return set_wait_limit_here(ns); }

}  // namespace ss
