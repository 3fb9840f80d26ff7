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
                                                       int heads, int b, int L,
                                                       int* status) {
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

// ---------------------------------------------------------------------------------------------
// Pair kernel: two query tiles that share their key tiles
// ---------------------------------------------------------------------------------------------
// A pair is the query tiles 2k and 2k+1 (rows [256k, 256k + 256)) of one (unit, head). With
// b = 64 (every 64 x 64-token global block) those 256 rows are one offset block, so both tiles
// keep exactly the same key tiles; otherwise each row masks the tiles of the pair's union list
// that it does not keep. Softmax group A owns tile 2k and group B tile 2k+1 for the whole pair:
// each K/V tile is loaded once and feeds both groups' Q*K^T and P*V, and no partial row is ever
// merged between the groups.
// The groups run unsynchronised with each other: each exponentiates as soon as its own S is read
// and its previous P*V is done. (Making them take turns on the SFU, B starting a tile's
// exponentials when A was half way through them, measured 4% slower at ViT-H: the waits cost more
// than the contention they avoid.) The shared S buffer in TMEM orders them loosely: the Q*K^T of
// one group's tile goes into it as soon as the other group has read its own S out.
// Work is pieces: the pairs of the full rounds of CTAs are whole pieces; the pairs of a partial
// last round are cut into `tail_split` key ranges each, so that round spreads over every CTA; each
// group of such a piece writes its (O, m, l) to a global slot, and k_merge_pieces combines them.
//   warp 0        TMA producer: Q_A, Q_B per piece; K and V tiles into a ring of stages
//   warp 1        TMEM allocator and Q*K^T issuer (both groups)
//   warp 2        P*V issuer (both groups)
//   warp 3        output storer: each group's normalised rows, staged as a tile in shared
//                 memory, go by one TMA store to the permuted output Op (block-major, like Q)
//   warps 4-7     softmax group A (one thread per query row = TMEM lane), and its epilogue
//   warps 8-11    softmax group B, and its epilogue
// TMEM columns: S [0,128) (shared), P_A [128,192), P_B [192,256) (64 columns of bf16 pairs each),
// O_A from 256, O_B from 320 (head dim 64) or 352 (head dim 80).
// V stays in its gathered [key, dh] layout as the MN-major B operand of P*V: at head dim 80 its
// tile is two 128-byte-swizzled 64-column atoms, the second loaded from column 64 with the
// columns past 80 filled with zeros, so one N = 80 MMA per 16 keys covers the whole head.
constexpr int kMaxSplit = 4;

template <int DH>
struct PairTmem {
  static constexpr uint32_t kS = 0;
  static constexpr uint32_t kP = 128, kPStride = 64;
  static constexpr uint32_t kO = 256, kOStride = DH <= 64 ? 64 : 96;
  static constexpr uint32_t kBq = 384;   // relative-position variant: A of the bias MMA, 64 per group
  static_assert(kO + kOStride + DH <= 512, "TMEM columns");
};

// kRelPos: the decomposed relative-position variant (head dim 64). The bias is one more MMA into
// S per tile and group: A = the group's per-row bias slices (Hu + Wu fp16 values per row, in TMEM
// columns 384 + 64g), B = the key tile's one-hot matrix E [128 keys x 128] (fp16 1.0 at columns
// Hu-1-kh and Hu+Wu-1-kw of key (kh, kw)), loaded by TMA with K and V. E makes the stage 64 KB, so
// the ring is two stages deep.
constexpr int kRelPosCols = 128;                               // E columns (Hu + Wu <= 128)
template <int DH, bool kRelPos = false>
struct PairSmem {
  static constexpr int kTail = DH - 64;                        // 0 or 16 columns
  static constexpr int kQKMain = kBM * 128;                    // 128 rows x 64 bf16, 128B swizzle
  static constexpr int kQKTail = kTail ? kBM * kTail * 2 : 0;  // 128 rows x 16 bf16, 32B swizzle
  static constexpr int kQK = kQKMain + kQKTail;                // one Q or K tile
  static constexpr int kVAtom = kBN * 128;                     // 128 keys x 64 bf16, 128B swizzle
  static constexpr int kV = kTail ? 2 * kVAtom : kVAtom;
  static constexpr int kE = kRelPos ? kBN * kRelPosCols * 2 : 0;   // two 128B-swizzled atoms
  static constexpr int kStageBytes = kQK + kV + kE;
  static constexpr int kStages = kRelPos ? 2 : (DH == 64 ? 5 : 3);   // depth of the K/V ring
  static constexpr int kQ = 0;                                 // Q_A, then Q_B
  static constexpr int kKV = 2 * kQK;
  // Output staging, used by the groups in turn: one 128-row tile of O in the layout of a Q tile
  // (128-byte-swizzled 64 columns, then the 32-byte-swizzled tail at head dim 80), the box layout
  // of the TMA store that writes it.
  static constexpr int kStage = kKV + kStages * kStageBytes;
  static constexpr int kBar = kStage + kQK;
  static constexpr int kBytes = kBar + 512;
  static constexpr int kAlloc = kBytes + 1024;                 // slack to align the base to 1024
  static_assert(kQK % 1024 == 0 && kStageBytes % 1024 == 0 && kKV % 1024 == 0,
                "tiles must stay 1024-byte aligned for the 128-byte swizzle");
  static_assert(kAlloc <= 227 * 1024, "pair kernel shared memory above the per-CTA limit");
};

// Piece i: pieces [0, whole) are the whole pairs 0..whole-1; piece whole + v is key range
// v % tail_split of pair whole + v / tail_split. Pairs are numbered head-major (all pairs of one
// (unit, head) together), so concurrently running CTAs share K/V in L2.
struct Piece {
  int pair, uh, qA, qB, n0, n1;
  int tail;          // index among the split pieces (their slots), or -1 for a whole pair
  KeyTiles tiles;
};
__host__ __device__ __forceinline__ int pairs_per_head(int N) {
  return ((N + kBM - 1) / kBM + 1) / 2;
}
__device__ __forceinline__ Piece piece_of(int i, int npairs, const AttnParams& P) {
  Piece c;
  int j = 0, ns = 1;
  if (i < P.whole) {
    c.pair = i;
    c.tail = -1;
  } else {
    c.tail = i - P.whole;
    c.pair = P.whole + c.tail / P.tail_split;
    j = c.tail - (c.pair - P.whole) * P.tail_split;
    ns = P.tail_split;
  }
  c.uh = c.pair / npairs;
  const int pq = c.pair - c.uh * npairs;
  c.qA = pq * 2 * kBM;
  c.qB = c.qA + kBM;
  c.tiles = key_tiles(c.qA, min(c.qA + 2 * kBM, P.N) - 1, pq, c.uh, P);
  const int nt = c.tiles.count();
  c.n0 = j * nt / ns;
  c.n1 = (j + 1) * nt / ns;
  return c;
}
// Every row of the pair keeps every key of the tile: the pair lies in one offset block
// (4b % 256 == 0) and the tile is whole.
__device__ __forceinline__ bool pair_tile_full(int c0, const AttnParams& P) {
  return (P.b * kStripes) % (2 * kBM) == 0 && c0 + kBN <= P.N;
}

// If the CTA gave up a wait, a bounded pause lets its copies and MMAs still in flight land before
// its shared memory and TMEM are released.
__device__ __forceinline__ void abort_drain(volatile int* abort) {
  if (*abort) {
    const uint64_t t0 = globaltimer_ns();
    while (globaltimer_ns() - t0 < 50000ull) {
    }
  }
}

// Row `row` of O (TMEM, DH fp32 columns at t_o) into registers: every 16-column load issued
// before the one wait (a TMEM load takes a few hundred cycles; one after another they add up).
template <int DH>
__device__ __forceinline__ void load_o_row(uint32_t t_o, uint32_t (&o)[DH]) {
#pragma unroll
  for (int cc = 0; cc < DH / 16; ++cc)
    tmem_ld16_nowait(t_o + cc * 16, *reinterpret_cast<uint32_t(*)[16]>(o + 16 * cc));
  tmem_ld_wait();
}
template <int DH, bool kRelPos>
__global__ void __launch_bounds__(kAttnThreads, 1)
    k_attn_pair(const __grid_constant__ CUtensorMap tq, const __grid_constant__ CUtensorMap tk,
                const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tq_tail,
                const __grid_constant__ CUtensorMap tk_tail, const __grid_constant__ CUtensorMap to,
                const __grid_constant__ CUtensorMap to_tail, const __grid_constant__ CUtensorMap te,
                const AttnParams P, int* status) {
  using S = PairSmem<DH, kRelPos>;
  using T = PairTmem<DH>;
  constexpr int NS = S::kStages;
  constexpr bool kHasTail = S::kTail > 0;
  static_assert(!(kRelPos && kHasTail), "the relative-position variant is built for head dim 64");
  static_assert(!kRelPos || T::kBq == T::kO + 2 * T::kOStride, "bias columns follow O_B");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + S::kBar);
  uint64_t* q_full = bars + 0;               // [2] Q_g of the piece landed
  uint64_t* q_empty = q_full + 2;            // [2] the piece's Q*K^T of group g done
  uint64_t* kv_full = q_empty + 2;           // [NS] K and V of a stage landed
  uint64_t* kv_empty = kv_full + NS;         // [NS] both groups' P*V of the stage's tile done
  uint64_t* s_full = kv_empty + NS;          // [2] group g's S computed
  uint64_t* s_free = s_full + 2;             // S read into registers by the group it was for
  uint64_t* p_full = s_free + 2;             // [2][2] half h of P_g written (O_g rescaled first)
  uint64_t* pv_done = p_full + 4;            // [2] P_g * V of a tile done
  uint64_t* stage_free = pv_done + 2;        // the staging tile read by its TMA store
  uint64_t* staged = stage_free + 1;         // a group's rows are in the staging tile
  uint64_t* bq_full = staged + 1;            // [2] relative-position variant: group g's bias rows
                                             // of the piece are in TMEM
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bq_full + 2);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int npairs = pairs_per_head(P.N);
  const int n_pieces = P.whole + (npairs * P.U * P.heads - P.whole) * P.tail_split;

  if (threadIdx.x == 0) {
    for (int g = 0; g < 2; ++g) {
      mbar_init(q_full + g, 1);
      mbar_init(q_empty + g, 1);
      mbar_init(s_full + g, 1);
      if (g == 0) mbar_init(s_free, 128);
      mbar_init(p_full + 2 * g, 128);
      mbar_init(p_full + 2 * g + 1, 128);
      mbar_init(pv_done + g, 1);
    }
    for (int i = 0; i < NS; ++i) {
      mbar_init(kv_full + i, 1);
      mbar_init(kv_empty + i, 1);
    }
    mbar_init(stage_free, 1);
    mbar_init(staged, 128);
    mbar_init(bq_full + 0, 128);
    mbar_init(bq_full + 1, 128);
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

  if (warp < 4) {
    setmaxnreg_dec<kRegsProducer>();
    if (warp == 0 && lane == 0) {
      // ------------------------------ TMA producer ------------------------------
      tma_prefetch_desc(&tq);
      tma_prefetch_desc(&tk);
      tma_prefetch_desc(&tv);
      bool ok = true;
      int gn = 0;   // tiles loaded so far (all pieces)
      for (int i = blockIdx.x, li = 0; ok && i < n_pieces; i += gridDim.x, ++li) {
        const Piece c = piece_of(i, npairs, P);
        for (int g = 0; g < 2; ++g) {
          if (li > 0 && !(ok = mbar_wait(q_empty + g, (li - 1) & 1, abort, status))) break;
          // A pair whose second tile lies past N loads tile A's rows again (never stored).
          const int q0 = (g == 1 && c.qB < P.N) ? c.qB : c.qA;
          uint8_t* qb = smem + S::kQ + g * S::kQK;
          mbar_expect_tx(q_full + g, S::kQK);
          tma_load_3d(qb, &tq, q_full + g, 0, q0, c.uh);
          if (kHasTail) tma_load_3d(qb + S::kQKMain, &tq_tail, q_full + g, 64, q0, c.uh);
        }
        for (int n = c.n0; ok && n < c.n1; ++n, ++gn) {
          const int st = gn % NS;
          if (gn >= NS && !(ok = mbar_wait(kv_empty + st, ((gn / NS) - 1) & 1, abort, status)))
            break;
          const int c0 = c.tiles.tile(n) * kBN;
          uint8_t* kb = smem + S::kKV + st * S::kStageBytes;
          uint8_t* vb = kb + S::kQK;
          mbar_expect_tx(kv_full + st, S::kStageBytes);
          tma_load_3d(kb, &tk, kv_full + st, 0, c0, c.uh);
          if (kHasTail) tma_load_3d(kb + S::kQKMain, &tk_tail, kv_full + st, 64, c0, c.uh);
          tma_load_3d(vb, &tv, kv_full + st, 0, c0, c.uh);
          // head dim 80: columns 64..127 of V; 80..127 lie outside the tensor and read as zero
          if (kHasTail) tma_load_3d(vb + S::kVAtom, &tv, kv_full + st, 64, c0, c.uh);
          if constexpr (kRelPos) {   // the key tile's one-hot matrix (per unit, not per head)
            uint8_t* eb = vb + S::kV;
            const int u_c = c.uh / P.heads;
            tma_load_3d(eb, &te, kv_full + st, 0, c0, u_c);
            tma_load_3d(eb + kBN * 128, &te, kv_full + st, 64, c0, u_c);
          }
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ------------------------------ Q*K^T issuer ------------------------------
      constexpr uint32_t idesc_qk = idesc_bf16_f32(kBM, kBN, false, false);
      bool ok = true;
      int gn = 0;
      for (int i = blockIdx.x, li = 0; ok && i < n_pieces; i += gridDim.x, ++li) {
        const Piece c = piece_of(i, npairs, P);
        if (!(ok = mbar_wait(q_full + 0, li & 1, abort, status))) break;
        if (!(ok = mbar_wait(q_full + 1, li & 1, abort, status))) break;
        if constexpr (kRelPos) {   // both groups' bias rows of this piece are in TMEM
          if (!(ok = mbar_wait(bq_full + 0, li & 1, abort, status))) break;
          if (!(ok = mbar_wait(bq_full + 1, li & 1, abort, status))) break;
          tc_fence_after();
        }
        for (int n = c.n0; ok && n < c.n1; ++n, ++gn) {
          const int st = gn % NS;
          if (!(ok = mbar_wait(kv_full + st, (gn / NS) & 1, abort, status))) break;
          const uint32_t k_addr = smem_u32(smem + S::kKV + st * S::kStageBytes);
          for (int g = 0; g < 2; ++g) {
            // S is reusable once the group it last held S for has read it (use 2 * gn + g - 1).
            const int use = 2 * gn + g;
            if (use > 0 && !(ok = mbar_wait(s_free, (use - 1) & 1, abort, status))) break;
            tc_fence_after();
            const uint32_t q_addr = smem_u32(smem + S::kQ + g * S::kQK);
            const uint32_t d = tmem + T::kS;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d, smem_desc(q_addr + kk * 32, 16, 1024, kSwizzle128B),
                           smem_desc(k_addr + kk * 32, 16, 1024, kSwizzle128B), idesc_qk, kk > 0);
            if (kHasTail)
              umma_bf16_ss(d, smem_desc(q_addr + S::kQKMain, 16, 256, kSwizzle32B),
                           smem_desc(k_addr + S::kQKMain, 16, 256, kSwizzle32B), idesc_qk, 1);
            if constexpr (kRelPos) {
              // S += Bq_g E^T: each key's two bias terms, summed by the tensor core (fp16 x 1.0).
              const uint32_t e_addr = k_addr + S::kQK + S::kV;
              for (int kk = 0; kk < P.rel_ksteps; ++kk)
                umma_bf16_ts(d, tmem + T::kBq + g * 64 + kk * 8,
                             smem_desc(e_addr + (kk >> 2) * (kBN * 128) + (kk & 3) * 32, 16, 1024,
                                       kSwizzle128B),
                             idesc_f16_f32(kBM, kBN, false, false), 1u);
            }
            umma_commit(s_full + g);
          }
        }
        if (!ok) break;
        umma_commit(q_empty + 0);   // the Q buffers are free once the piece's Q*K^T are done
        umma_commit(q_empty + 1);
      }
    } else if (warp == 2 && lane == 0) {
      // ------------------------------ P*V issuer --------------------------------
      // P_g of a tile exists only after S_g of it, which followed the stage's K/V landing
      // (observed by the Q*K^T issuer), so V is ready whenever P is. A piece's first P_g * V
      // overwrites O_g: its group read the previous piece's O_g before handing over this P.
      constexpr uint32_t idesc_pv = idesc_bf16_f32(kBM, DH, false, true);
      bool ok = true;
      int gn = 0;
      for (int i = blockIdx.x; ok && i < n_pieces; i += gridDim.x) {
        const Piece c = piece_of(i, npairs, P);
        for (int n = c.n0; ok && n < c.n1; ++n, ++gn) {
          const int st = gn % NS;
          const uint32_t v_addr = smem_u32(smem + S::kKV + st * S::kStageBytes + S::kQK);
          for (int g = 0; ok && g < 2; ++g) {
            const uint32_t a = tmem + T::kP + g * T::kPStride;
            const uint32_t d = tmem + T::kO + g * T::kOStride;
#pragma unroll
            for (int kk = 0; kk < kBN / 16; ++kk) {
              if (kk % (kBN / 32) == 0) {
                // P arrives in two halves (keys 0-63, 64-127): the first half's MMAs run while
                // the softmax still computes the second.
                if (!(ok = mbar_wait(p_full + 2 * g + kk / (kBN / 32), gn & 1, abort, status)))
                  break;
                tc_fence_after();
              }
              umma_bf16_ts(d, a + kk * 8,
                           smem_desc(v_addr + kk * 2048, S::kVAtom, 1024, kSwizzle128B), idesc_pv,
                           (n > c.n0 || kk > 0) ? 1u : 0u);
            }
            if (!ok) break;
            umma_commit(pv_done + g);
          }
          if (!ok) break;
          umma_commit(kv_empty + st);
        }
      }
    } else if (warp == 3 && lane == 0) {
      // ------------------------------ output storer -----------------------------
      // Each whole piece's staged tiles (group A's, then B's: the order the groups stage them)
      // go by TMA to rows q0 .. q0+127 of matrix u*heads+h of Op; rows past N are not written.
      bool ok = true;
      int use = 0;
      for (int i = blockIdx.x; ok && i < n_pieces; i += gridDim.x) {
        const Piece c = piece_of(i, npairs, P);
        if (c.tail >= 0 && P.tail_split > 1) continue;   // split pieces store their own rows
        for (int g = 0; ok && g < 2; ++g, ++use) {
          if (!(ok = mbar_wait(staged, use & 1, abort, status))) break;
          const int q0 = g ? c.qB : c.qA;
          if (q0 < P.N) {
            tma_store_3d(&to, smem + S::kStage, 0, q0, c.uh);
            if (kHasTail) tma_store_3d(&to_tail, smem + S::kStage + S::kQKMain, 64, q0, c.uh);
            bulk_commit();
          }
          bulk_wait_read();          // the staging tile has been read out
          mbar_arrive(stage_free);   // it may be rewritten
        }
      }
      bulk_wait_all();   // every store has completed before the CTA exits
    }
  } else {
    setmaxnreg_inc<kRegsSoftmax>();
    // ------------------------------ softmax groups ----------------------------
    const int grp = (warp - 4) >> 2;                    // 0: tile A of the pair, 1: tile B
    const int row = 32 * (warp & 3) + lane;             // TMEM lane == query row
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const uint32_t t_s = tmem + T::kS + lane_off;
    const uint32_t t_p = tmem + T::kP + grp * T::kPStride + lane_off;
    const uint32_t t_o = tmem + T::kO + grp * T::kOStride + lane_off;
    const int b4 = P.b * kStripes;
    const uint64_t scale2 = f2_pack(P.scale_log2, P.scale_log2);
    constexpr int kSlot = (DH + 2) * kBM;               // floats of one group's partial
    bool ok = true;
    int gn = 0;            // tiles of this group so far (all pieces): the phase count
    bool s_ready = false;  // the next s_full phase was already seen complete (non-blocking test)
    int stage_uses = 0;    // this group's uses of the staging rows (they alternate with the other's)
    for (int i = blockIdx.x; ok && i < n_pieces; i += gridDim.x) {
      const Piece c = piece_of(i, npairs, P);
      const int u_i = c.uh / P.heads, h_i = c.uh - u_i * P.heads;
      const int qrow = (grp ? c.qB : c.qA) + row;
      const int a_q = min(qrow, P.N - 1) / b4;
      const int s_q = band_start(a_q, P.W, P.nb);
      const int band_lo = s_q * b4, band_hi = (s_q + P.W) * b4, glob_hi = P.g * b4;
      float m_ref = -INFINITY, l_run = 0.f;
      if constexpr (kRelPos) {
        // This row's bias slices into TMEM (A of the bias MMA): entries qh .. qh+Hu-1 of its Rh
        // products, then qw .. qw+Wu-1 of its Rw products (the row of the bias GEMM), so that key
        // (kh, kw) meets them at columns Hu-1-kh and Hu+Wu-1-kw of E. The previous piece's bias
        // MMAs of this group are complete: this thread has read every S they fed.
        const int qr = min(qrow, P.N - 1);
        const int tok = __ldg(P.perm + (size_t)u_i * P.N + blockmajor_to_canonical(qr, P.b, P.L));
        const int t = (unsigned)tok < (unsigned)P.N ? tok : 0;
        const int qh = t / P.rel_w, qw = t - qh * P.rel_w;
        const uint16_t* g = P.rel_tab + ((size_t)c.uh * P.N + qr) * P.rel_ld;
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
          uint32_t w[32];
#pragma unroll
          for (int e2 = 0; e2 < 32; ++e2) {
            uint32_t lohi[2];
#pragma unroll
            for (int s2 = 0; s2 < 2; ++s2) {
              const int e = 64 * half + 2 * e2 + s2;
              uint16_t h = 0;
              if (e < P.rel_h) h = __ldg(g + qh + e);
              else if (e < P.rel_h + P.rel_w) h = __ldg(g + 2 * P.rel_h - 1 + qw + (e - P.rel_h));
              lohi[s2] = h;
            }
            w[e2] = lohi[0] | (lohi[1] << 16);
          }
          tmem_st32_async(tmem + T::kBq + grp * 64 + half * 32 + lane_off, w);
        }
        tmem_st_wait();
        tc_fence_before();
        mbar_arrive(bq_full + grp);
      }
      for (int n = c.n0; ok && n < c.n1; ++n, ++gn) {
        const int j = n - c.n0;
        // Warp-collective wait: either every lane goes on to the .sync.aligned TMEM ops or none.
        if (!__all_sync(0xffffffffu, s_ready))
          ok = __all_sync(0xffffffffu, mbar_wait(s_full + grp, gn & 1, abort, status));
        if (!ok) break;
        tc_fence_after();
        float sv[kBN];
        {
          uint32_t r[128];
          tmem_ld128(t_s, r);
#pragma unroll
          for (int k = 0; k < kBN; ++k) sv[k] = __uint_as_float(r[k]);
        }
        tc_fence_before();
        mbar_arrive(s_free);   // S is in registers: the other group's Q*K^T may overwrite it
        // Has this group's previous P * V released P_g and O_g? Tested now, waited for below.
        bool prev_pv_done = gn == 0 || mbar_test(pv_done + grp, (gn - 1) & 1);
        const int c0 = c.tiles.tile(n) * kBN;
        if (!pair_tile_full(c0, P)) {
          // The row's kept keys in this tile are two runs, [0, e0) and [s1, e1) relative to c0:
          // turned into four 32-bit column masks, so the per-key test has no branch.
          const int e0 = min(glob_hi, P.N) - c0, s1 = band_lo - c0, e1 = min(band_hi, P.N) - c0;
          uint32_t km[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) km[k] = run_bits(0, e0, 32 * k) | run_bits(s1, e1, 32 * k);
#pragma unroll
          for (int k = 0; k < kBN; ++k) sv[k] = (km[k >> 5] >> (k & 31)) & 1u ? sv[k] : -INFINITY;
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
        // TMEM is rescaled on few tiles. The decision is warp-wide (TMEM ops are warp-collective).
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
        // The exponents x = s*scale - ref, in place (two per packed FMA), so that the loop below
        // holds little besides the exponentials. Masked keys give -inf.
        {
          const uint64_t nref2 = f2_pack(-ref, -ref);
#pragma unroll
          for (int k = 0; k < kBN; k += 2)
            f2_unpack(f2_fma(f2_pack(sv[k], sv[k + 1]), scale2, nref2), sv[k], sv[k + 1]);
        }
        // P_g and O_g are free once this group's previous P * V is done.
        if (gn > 0) {
          if (!__all_sync(0xffffffffu, prev_pv_done)) {
            ok = __all_sync(0xffffffffu, mbar_wait(pv_done + grp, (gn - 1) & 1, abort, status));
            if (!ok) break;
          }
          tc_fence_after();
        }
        // P as bf16 pairs (column i holds keys 2i, 2i+1), 16 columns at a time; each 64-key half
        // is handed to the P*V issuer as soon as it is in TMEM. 2^x on the SFU in fp32 (as fast
        // per value as its packed forms, and exact to fp32 input); ex2(-inf) = 0 for masked keys.
        uint64_t sum2a = 0, sum2b = 0;   // two packed partial sums (bit pattern 0 = +0.0f pair)
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t pw[16];
#pragma unroll
          for (int i2 = 0; i2 < 16; ++i2) {
            const int k = 32 * cc + 2 * i2;
            const float p0 = ex2_mufu(sv[k]), p1 = ex2_mufu(sv[k + 1]);
            if (i2 & 1)
              sum2b = f2_add(sum2b, f2_pack(p0, p1));
            else
              sum2a = f2_add(sum2a, f2_pack(p0, p1));
            pw[i2] = pack_bf16_pos(p0, p1);   // p >= 0: integer-pipe rounding
          }
          tmem_st16_async(t_p + 16 * cc, pw);
          if (cc == 1 && rescale && j > 0) {
            // O_g holds the piece's earlier tiles (their P*V completed, above); it is rescaled
            // before this tile's first P*V accumulates into it.
#pragma unroll 1
            for (int oc = 0; oc < DH / 16; ++oc) {
              uint32_t o[16];
              tmem_ld16(t_o + oc * 16, o);
#pragma unroll
              for (int k = 0; k < 16; ++k) o[k] = __float_as_uint(__uint_as_float(o[k]) * alpha);
              tmem_st16_async(t_o + oc * 16, o);
            }
          }
          if (cc & 1) {
            tmem_st_wait();   // this half of P (and O) is in TMEM before the arrive releases it
            tc_fence_before();
            mbar_arrive(p_full + 2 * grp + (cc >> 1));
          }
        }
        if (!ok) break;
        // Is S of this group's next tile already there? Tested here, where the result is not
        // needed at once, instead of by a blocking wait at the top of the next iteration.
        s_ready = mbar_test(s_full + grp, (gn + 1) & 1);
        float sa0, sa1;
        f2_unpack(f2_add(sum2a, sum2b), sa0, sa1);
        l_run += sa0 + sa1;
      }
      if (!ok) break;
      // ---- the piece's rows: O_g is final once the piece's last P_g * V is done ----
      ok = __all_sync(0xffffffffu, mbar_wait(pv_done + grp, (gn - 1) & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      if (c.tail < 0 || P.tail_split == 1) {
        uint32_t o[DH];
        load_o_row<DH>(t_o, o);
        tc_fence_before();   // O_g read before the next piece's first P goes to P*V
        // Normalised row -> the staging tile, once the TMA store of its previous contents (the
        // other group's rows, or this group's a piece ago) has read them; warp 3 then stores it.
        const int use = 2 * stage_uses + grp;
        ++stage_uses;
        if (use > 0 &&
            !(ok = __all_sync(0xffffffffu, mbar_wait(stage_free, (use - 1) & 1, abort, status))))
          break;
        const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
        if (P.ml && qrow < P.N) P.ml[(size_t)c.uh * P.N + qrow] = make_float2(m_ref, l_run);
        const uint32_t tile = smem_u32(smem + S::kStage);
#pragma unroll
        for (int cc = 0; cc < DH / 8; ++cc) {
          // 16-byte chunk cc of the row, at its place in the swizzled box: 128-byte rows with the
          // chunk index XORed with row % 8 (columns 0..63), 32-byte rows with it XORed with
          // (row / 4) % 2 (the tail, columns 64..79).
          const uint32_t addr = cc < 8 ? tile + row * 128 + ((cc ^ (row & 7)) << 4)
                                       : tile + S::kQKMain + row * 32 + (((cc - 8) ^ ((row >> 2) & 1)) << 4);
          st_shared_v4(addr,
                       pack_bf16(__uint_as_float(o[8 * cc + 0]) * inv, __uint_as_float(o[8 * cc + 1]) * inv),
                       pack_bf16(__uint_as_float(o[8 * cc + 2]) * inv, __uint_as_float(o[8 * cc + 3]) * inv),
                       pack_bf16(__uint_as_float(o[8 * cc + 4]) * inv, __uint_as_float(o[8 * cc + 5]) * inv),
                       pack_bf16(__uint_as_float(o[8 * cc + 6]) * inv, __uint_as_float(o[8 * cc + 7]) * inv));
        }
        fence_proxy_async_smem();   // visible to the TMA store
        mbar_arrive(staged);
        continue;
      }
      // Split pair: this piece's O_g (relative to its m) column-major, so that a warp's 32 rows
      // of one column are one 128-byte line, then m and l; k_merge_pieces combines the pair's
      // pieces after this launch.
      {
        float* slot = P.partial + ((size_t)c.tail * 2 + grp) * kSlot + row;
        uint32_t o[DH];
        load_o_row<DH>(t_o, o);
        tc_fence_before();
#pragma unroll
        for (int e = 0; e < DH; ++e) slot[e * kBM] = __uint_as_float(o[e]);
        slot[DH * kBM] = m_ref;
        slot[(DH + 1) * kBM] = l_run;
      }
    }
  }
  tc_fence_before();
  abort_drain(abort);
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
        if (P.ml && store) P.ml[(size_t)I.uh * P.N + qrow] = make_float2(m_ref, l_run);
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

template <int DH, bool kRelPos = false>
static cudaError_t launch_attn_pair(const CUtensorMap* tq, const CUtensorMap* tk,
                                    const CUtensorMap* tv, const CUtensorMap* tq_tail,
                                    const CUtensorMap* tk_tail, const CUtensorMap* to,
                                    const CUtensorMap* to_tail, const CUtensorMap* te,
                                    const AttnParams& p, int* status, cudaStream_t st) {
  using S = PairSmem<DH, kRelPos>;
  auto kernel = k_attn_pair<DH, kRelPos>;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       S::kAlloc);
  if (e != cudaSuccess) return e;
  const int pieces = p.whole + (pairs_per_head(p.N) * p.U * p.heads - p.whole) * p.tail_split;
  dim3 grid(std::max(1, std::min(pieces, p.sms)));
  return launch_pdl(kernel, grid, dim3(kAttnThreads), S::kAlloc, st, *tq, *tk, *tv, *tq_tail,
                    *tk_tail, *to, *to_tail, *te, p, status);
}

// Short items: every query tile has at most kPairTiles key tiles (the windowed blocks).
static bool short_items(const AttnParams& p) {
  const int nq = (p.N + kBM - 1) / kBM;
  int nt_max = 0;
  for (int qt = 0; qt < nq; ++qt)
    nt_max = std::max(nt_max, key_tiles(qt * kBM, std::min(qt * kBM + kBM, p.N) - 1, qt, 0, p).count());
  return nt_max <= kPairTiles;
}

AttnPlan attn_plan(const AttnParams& p, int dh, int sms, bool force_pair) {
  AttnPlan r = {};
  r.pair_kernel = force_pair || p.rel_tab != nullptr || !(dh == 64 && short_items(p));
  if (!r.pair_kernel) return r;
  const int npairs = pairs_per_head(p.N);
  r.pairs = npairs * p.U * p.heads;
  r.whole = r.pairs;
  r.tail_split = 1;
  int nt_min = 1 << 30, nt_max = 0;
  for (int pq = 0; pq < npairs; ++pq) {
    const int q0 = pq * 2 * kBM;
    const int nt = key_tiles(q0, std::min(q0 + 2 * kBM, p.N) - 1, pq, 0, p).count();
    nt_min = std::min(nt_min, nt);
    nt_max = std::max(nt_max, nt);
  }
  // The pairs of a partial last round (r of them) are split into s pieces each, s = how many
  // times r fits the CTAs (at most kMaxSplit, and every piece keeps a tile), when that shortens
  // the busiest CTA: full rounds of whole pairs plus one split piece, against one more round of
  // whole pairs (each piece costs about one tile of pipeline fill and drain; the merge about one).
  const int rem = r.pairs % sms;
  if (rem > 0) {
    const int s = std::min(std::min(kMaxSplit, nt_min), sms / rem);
    const long long full = r.pairs / sms;
    const long long cost_whole = (full + 1) * (nt_max + 1);
    const long long cost_split = full * (nt_max + 1) + (nt_max + s - 1) / s + 2;
    if (s > 1 && cost_split < cost_whole) {
      r.whole = r.pairs - rem;
      r.tail_split = s;
      r.partial_bytes = (size_t)rem * s * 2 * (dh + 2) * kBM * sizeof(float);
    }
  }
  return r;
}

// ---------------------------------------------------------------------------------------------
// Merge of split pairs: the pieces' (O, m, l) of each row, combined in piece order, normalised and
// written to the row of Op.
// ---------------------------------------------------------------------------------------------
// One CTA per (split pair, group, 8-column chunk), one thread per row: O = sum_j 2^(m_j - M) O_j,
// l = sum_j 2^(m_j - M) l_j with M = max_j m_j; Op row chunk = bf16(O / l). A row whose pieces kept
// no key (every m_j = -inf) is written as zeros. (A CTA per chunk, rather than per row block, keeps
// enough loads in flight: one CTA per row block ran latency-bound at a tenth of the L2 bandwidth.)
template <int DH>
__global__ void __launch_bounds__(kBM) k_merge_pieces(const float* __restrict__ partial,
                                                      uint16_t* __restrict__ operm, AttnParams P) {
  griddep_wait();
  griddep_launch();
  constexpr int kSlot = (DH + 2) * kBM;
  constexpr int kChunks = DH / 8;
  const int cc = blockIdx.x % kChunks, pg = blockIdx.x / kChunks;
  const int tp = pg >> 1, grp = pg & 1, row = threadIdx.x;
  const int pair = P.whole + tp;
  const int npairs = pairs_per_head(P.N);
  const int uh = pair / npairs, pq = pair - uh * npairs;
  const int qrow = pq * 2 * kBM + grp * kBM + row;
  if (qrow >= P.N) return;
  const int ns = P.tail_split;
  const float* first = partial + ((size_t)tp * ns * 2 + grp) * kSlot + row;
  float m[kMaxSplit], l[kMaxSplit];
  float M = -INFINITY;
#pragma unroll
  for (int j = 0; j < kMaxSplit; ++j) {
    const float* sj = first + (size_t)j * 2 * kSlot;
    m[j] = j < ns ? __ldg(sj + DH * kBM) : -INFINITY;
    l[j] = j < ns ? __ldg(sj + (DH + 1) * kBM) : 0.f;
    M = fmaxf(M, m[j]);
  }
  float v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) v[e] = 0.f;
  float Lsum = 0.f;
#pragma unroll
  for (int j = 0; j < kMaxSplit; ++j) {
    const float f = m[j] == -INFINITY ? 0.f : exp2f(m[j] - M);
    Lsum += f * l[j];
    const float* sj = first + (size_t)j * 2 * kSlot + (size_t)cc * 8 * kBM;
#pragma unroll
    for (int e = 0; e < 8; ++e) v[e] += (j < ns ? __ldg(sj + e * kBM) : 0.f) * f;
  }
  const float inv = Lsum > 0.f ? 1.f / Lsum : 0.f;
  uint4 w;
  w.x = pack_bf16(v[0] * inv, v[1] * inv);
  w.y = pack_bf16(v[2] * inv, v[3] * inv);
  w.z = pack_bf16(v[4] * inv, v[5] * inv);
  w.w = pack_bf16(v[6] * inv, v[7] * inv);
  reinterpret_cast<uint4*>(operm + ((size_t)uh * P.N + qrow) * DH)[cc] = w;
  if (P.ml && cc == 0) P.ml[(size_t)uh * P.N + qrow] = make_float2(M, Lsum);
}

cudaError_t launch_attn(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* tq_tail, const CUtensorMap* tk_tail,
                        const CUtensorMap* to, const CUtensorMap* to_tail, const AttnParams& p,
                        int dh, int* status, cudaStream_t st, const CUtensorMap* te) {
  if (p.rel_tab) {
    if (dh != 64 || !te) return cudaErrorInvalidValue;
    return launch_attn_pair<64, true>(tq, tk, tv, tq, tk, to, to, te, p, status, st);
  }
  if (dh == 64 && short_items(p)) return launch_attn_pairs(tq, tk, tv, p, status, st);
  if (dh == 64) return launch_attn_pair<64>(tq, tk, tv, tq, tk, to, to, tq, p, status, st);
  if (dh == 80)
    return launch_attn_pair<80>(tq, tk, tv, tq_tail, tk_tail, to, to_tail, tq, p, status, st);
  return cudaErrorInvalidValue;
}

cudaError_t launch_merge_pieces(const AttnParams& p, int dh, cudaStream_t st) {
  const int split_pairs = pairs_per_head(p.N) * p.U * p.heads - p.whole;
  if (p.tail_split <= 1 || split_pairs <= 0) return cudaSuccess;
  const dim3 grid(2 * split_pairs * (dh / 8));
  if (dh == 64) return launch_pdl(k_merge_pieces<64>, grid, dim3(kBM), 0, st, p.partial, p.operm, p);
  if (dh == 80) return launch_pdl(k_merge_pieces<80>, grid, dim3(kBM), 0, st, p.partial, p.operm, p);
  return cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------------------------
// Un-permute: out[u, perm[p], h, :] = Op[u*heads + h, q(p), :] (the pair kernel's output order)
// ---------------------------------------------------------------------------------------------
// One warp per block-major position q of a unit: the warp resolves the token t = perm[u][p(q)],
// reads the position's row of every head matrix (heads * CPR 16-byte chunks) and writes them as
// token t's one contiguous heads * dh row of out. All of a lane's loads are in flight before its
// stores. CPR = 16-byte chunks per head, KPL = chunks per lane.
template <int CPR, int KPL>
__global__ void __launch_bounds__(256) k_unpermute_out(const uint16_t* __restrict__ op,
                                                       const int32_t* __restrict__ perm,
                                                       uint16_t* __restrict__ out, int N,
                                                       int heads, int b, int L, int* status) {
  griddep_wait();
  griddep_launch();
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qpos = blockIdx.x * 8 + warp;
  if (qpos >= N) return;
  const int tok = __ldg(perm + (size_t)u * N + blockmajor_to_canonical(qpos, b, L));
  if ((unsigned)tok >= (unsigned)N) {   // not a token of this unit: skip the row, report it
    if (lane == 0) record_bad_index(status);
    return;
  }
  const int per_tok = heads * CPR;
  const size_t plane = (size_t)N * CPR;   // 16-byte chunks per (unit, head) matrix
  const uint4* src = reinterpret_cast<const uint4*>(op) + (size_t)u * heads * plane +
                     (size_t)qpos * CPR;
  uint4* dst = reinterpret_cast<uint4*>(out) + ((size_t)u * N + tok) * per_tok;
  uint4 buf[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int cidx = e * 32 + lane;
    if (cidx < per_tok) {
      const int h = cidx / CPR, cc = cidx - h * CPR;
      buf[e] = __ldg(src + h * plane + cc);
    }
  }
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int cidx = e * 32 + lane;
    if (cidx < per_tok) dst[cidx] = buf[e];
  }
}

cudaError_t launch_unpermute_out(const uint16_t* op, const int32_t* perm, uint16_t* out, int U,
                                 int N, int heads, int dh, int b, int* status, cudaStream_t st) {
  dim3 grid((N + 7) / 8, U);
  const int L = N / kStripes;
  const int per_tok = heads * (dh / 8);
  if (per_tok > 32 * 10) return cudaErrorInvalidValue;   // heads * dh > 2560
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, grid, dim3(256), 0, st, op, perm, out, N, heads, b, L, status);
  };
  if (dh == 64) return per_tok <= 32 * 8 ? go(k_unpermute_out<8, 8>) : go(k_unpermute_out<8, 10>);
  if (dh == 80) return go(k_unpermute_out<10, 10>);
  return cudaErrorInvalidValue;
}

cudaError_t set_wait_limit_attn(uint64_t ns) { return set_wait_limit_here(ns); }

}  // namespace ss
