// S4: Residual-Consistency MLP on tcgen05 / TMEM.
//
// SparseSAM Dutch technical summary, "Residual-Consistency MLP": tokens are split by the
// permutation order into a keep-set and a residual set; the MLP runs on the top-K keep-set only and
// the residual set passes the block unchanged. Here that is three launches:
//   1. gather the kept rows of x into a dense [B*K, C] operand,
//   2. H = GELU(Xk W1^T + b1)   (tcgen05 GEMM, bias + erf-GELU + bf16 rounding in the epilogue),
//   3. x[keep] += H W2^T + b2   (tcgen05 GEMM, epilogue adds the residual row and stores it back
//                                into x in place; kept rows are distinct, so no atomics).
// Rows outside the keep-set are never touched.
//
// GEMM: C[M, N] = A[M, Kd] B[N, Kd]^T, A and B K-major bf16 in 128B-swizzled 64-wide K blocks
// loaded by TMA into a multi-stage ring; one thread issues 128 x BN x 16 MMAs into a TMEM fp32
// accumulator; eight epilogue warps read it back with tcgen05.ld (one row per thread, two warps
// per TMEM lane quadrant, each on half of the columns).
#include "common.cuh"
#include "kernels.h"

namespace ss {

// One warp per kept row: resolve the row's token, then copy its C bf16 (C/8 16-byte chunks) with
// all of a lane's loads in flight before its stores. CTA 0 also zeroes the GEMMs' k-split
// counters (`zero`, `nzero` ints), which the two GEMM launches that follow expect at zero.
// late_wait: the caller guarantees that keep and x are already final when this launch starts
// (earlier launches of the same call waited for the work that wrote them) and that nothing still
// running reads xk or the counters. The copy then runs at once, in the previous launch's tail,
// and every thread takes the dependency wait at its end, so this launch still completes after the
// previous one for everything that follows.
__global__ void __launch_bounds__(256) k_gather_rows(const uint16_t* __restrict__ x,
                                                     const int32_t* __restrict__ keep,
                                                     uint16_t* __restrict__ xk, int B, int T,
                                                     int K, int C, int* __restrict__ zero,
                                                     int nzero, int late_wait, int* status) {
  if (!late_wait) griddep_wait();
  griddep_launch();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  const int m = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  const int t = m < B * K ? __ldg(keep + m) : 0;
  if (m < B * K && (unsigned)t >= (unsigned)T && lane == 0) record_bad_index(status);
  if (m < B * K && (unsigned)t < (unsigned)T) {   // a keep entry outside the image is skipped
    const int b = m / K;
    const int cpr = C / 8;
    const uint4* src = reinterpret_cast<const uint4*>(x + ((size_t)b * T + t) * C);
    uint4* dst = reinterpret_cast<uint4*>(xk) + (size_t)m * cpr;
    for (int c0 = 0; c0 < cpr; c0 += 256) {
      uint4 buf[8];
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (c0 + e * 32 + lane < cpr) buf[e] = __ldg(src + c0 + e * 32 + lane);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (c0 + e * 32 + lane < cpr) dst[c0 + e * 32 + lane] = buf[e];
    }
  }
  if (late_wait) griddep_wait();
}

cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* keep, uint16_t* xk, int B, int T,
                               int K, int C, int* zero, int nzero, int* status, cudaStream_t st,
                               bool late_wait) {
  const int rows = B * K;
  return launch_pdl(k_gather_rows, dim3((rows + 7) / 8), dim3(256), 0, st, x, keep, xk, B, T, K, C,
                    zero, nzero, late_wait ? 1 : 0, status);
}

// Persistent warp-specialised GEMM. Work unit = (m-tile, n-tile, k-split); CTA c takes units
// c, c + grid, c + 2*grid, ... The accumulator is double-buffered in TMEM, so the epilogue of one
// unit overlaps the mainloop of the next.
//   warp 0      TMA producer (A and B k-blocks into a multi-stage ring, across units)
//   warp 1      TMEM allocator and tcgen05.mma issuer
//   warps 2-3   idle (complete the first warpgroup for the register split)
//   warps 4-11  epilogue: warp w reads TMEM lanes 32*(w%4).. and one half of the tile's columns
// A k-split unit writes its fp32 partial tile to its own slot; the last unit of a tile to finish
// (an atomic counter per tile) sums the slots in split order and applies the epilogue, so the
// result does not depend on which split finished last.
constexpr int kGemmThreads = 384;
constexpr int kEpiThreads = 256;
// Register split (launch: 384 threads x 168): producer warpgroup 56, epilogue warpgroups 224.
constexpr uint32_t kGemmRegsProducer = 56, kGemmRegsEpilogue = 224;
static_assert(128 * kGemmRegsProducer + 256 * kGemmRegsEpilogue <= 384 * 168,
              "GEMM register split too large");

// KSUB 64-wide K sub-blocks per pipeline stage: each full/empty handshake (an mbarrier wait costs
// ~150 cycles of latency on the thread that gates on it) then covers KSUB x 4 MMAs.
template <int BN, int KSUB>
struct GemmCfg {
  static constexpr int kABytes = 128 * 128;       // 128 rows x 64 bf16 per sub-block
  static constexpr int kBBytes = BN * 128;        // BN rows x 64 bf16 per sub-block
  static constexpr int kStageBytes = KSUB * (kABytes + kBBytes);
  static constexpr int kStages = (192 * 1024) / kStageBytes;
  static constexpr int kBar = kStages * kStageBytes;
  static constexpr int kAlloc = kBar + 512 + 1024;
  // two accumulators; TMEM is allocated in powers of two columns
  static constexpr int kTmemCols = 2 * BN <= 128 ? 128 : 2 * BN <= 256 ? 256 : 512;
  static constexpr int kHalf = BN / 2;            // columns per epilogue warp
  static_assert(kStages >= 2, "at least two stages");
};

__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }
__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// GELU(z) = z/2 (1 + erf(z / sqrt 2)), with erf from Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (|error| <= 1.5e-7, far below the bf16 rounding of the
// result): for x >= 0, erfc(x) = (a1 t + a2 t^2 + a3 t^3 + a4 t^4 + a5 t^5) e^(-x^2), t = 1/(1 + p x).
// Then GELU(z) = z/2 erfc(|z|/sqrt 2) for z < 0 and z/2 (2 - erfc(|z|/sqrt 2)) for z >= 0, which
// keeps the relative accuracy of the small negative tail. Two MUFU ops (reciprocal, 2^x) per value;
// the rest runs on a pair of values at once in packed fp32x2 arithmetic (the same roundings as
// scalar operations), halving the FMA-pipe instructions of the fc1 epilogue.
__device__ __forceinline__ void gelu_erf2(float& z0, float& z1) {
  const uint64_t x = f2_mul(f2_pack(fabsf(z0), fabsf(z1)),
                            f2_pack(0.70710678118654752f, 0.70710678118654752f));
  float d0, d1;
  f2_unpack(f2_fma(f2_pack(0.3275911f, 0.3275911f), x, f2_pack(1.0f, 1.0f)), d0, d1);
  const uint64_t t = f2_pack(rcp_mufu(d0), rcp_mufu(d1));
  uint64_t q = f2_fma(f2_pack(1.061405429f, 1.061405429f), t, f2_pack(-1.453152027f, -1.453152027f));
  q = f2_fma(q, t, f2_pack(1.421413741f, 1.421413741f));
  q = f2_fma(q, t, f2_pack(-0.284496736f, -0.284496736f));
  q = f2_fma(q, t, f2_pack(0.254829592f, 0.254829592f));
  float a0, a1;   // -x^2 log2(e)
  f2_unpack(f2_mul(f2_mul(x, x), f2_pack(-1.4426950408889634f, -1.4426950408889634f)), a0, a1);
  const uint64_t erfc = f2_mul(f2_mul(t, q), f2_pack(ex2_mufu(a0), ex2_mufu(a1)));
  float e0, e1, m0, m1;   // erfc and 2 - erfc
  f2_unpack(erfc, e0, e1);
  f2_unpack(f2_fma(erfc, f2_pack(-1.0f, -1.0f), f2_pack(2.0f, 2.0f)), m0, m1);
  const uint64_t w = f2_pack(z0 >= 0.f ? m0 : e0, z1 >= 0.f ? m1 : e1);
  f2_unpack(f2_mul(f2_mul(f2_pack(z0, z1), f2_pack(0.5f, 0.5f)), w), z0, z1);
}

struct GemmShape {
  int M, N, Kd;
  int m_tiles, n_tiles, splits, kb_total;
  int paired;              // two k-splits, every unit resident at once: each finishes half
  int units, whole;        // units; those from `whole` on are tail halves (see GemmPlan::tail)
  float* partial;          // splits > 1: [tiles][splits][BN][128] fp32, column-major tiles;
                           // paired: [tiles][2 halves][BN/2][128]; tail: [tail tiles][2][BN/2][128]
  int* counters;           // [tiles][2], zero on entry (splits > 1)
};

// The epilogue of one output row m (< M) in chunks of 32 columns. The row's destination (and, for
// kind 1, the keep lookup behind it) is resolved once per unit; a chunk's bias and residual words
// are loaded before its accumulator values are needed, so their latency overlaps those reads.
// Kind 1: a keep entry outside the image gives no row (nullptr: the row is skipped) and records
// SS_EINDEX; so does, for kind 2, a permuted position outside the unit. Kind 2's row is the unit
// row's (block-major) place in the gathered Q at head 0; kind 3's a pad token has no row (skipped, no error).
__device__ __forceinline__ uint16_t* epi_row(const GemmEpilogue& ep, const GemmShape& g, int m,
                                             int* status) {
  if (ep.kind == 0 || ep.kind == 4) return ep.out + (size_t)m * g.N;
  if (ep.kind == 2) {
    const int N = ep.ur.N;
    const int u = m / N;
    const int p = __ldg(ep.inv + m);
    if ((unsigned)p >= (unsigned)N) {
      record_bad_index(status);
      return nullptr;
    }
    return ep.out + ((size_t)u * ep.heads * N + canonical_to_blockmajor(p, ep.b, ep.L)) * ep.dh;
  }
  if (ep.kind == 3) {
    const long long src = unit_row_src(ep.ur, m);
    return src < 0 ? nullptr : ep.x + (size_t)src * g.N;
  }
  const int b = m / ep.K_per_image;
  const int t = __ldg(ep.keep + m);
  if ((unsigned)t >= (unsigned)ep.T) {
    record_bad_index(status);
    return nullptr;
  }
  return ep.x + ((size_t)b * ep.T + t) * g.N;
}
struct Epi32In {
  uint4 b[4], x[4];   // bias and (kind 1) residual bf16 words of 32 columns
};
__device__ __forceinline__ void epi_load(const GemmEpilogue& ep, const uint16_t* row, int n,
                                         Epi32In& in) {
  if (ep.bias) {
    const uint4* bp = reinterpret_cast<const uint4*>(ep.bias + n);
#pragma unroll
    for (int q = 0; q < 4; ++q) in.b[q] = __ldg(bp + q);
  }
  if (ep.kind == 1 || ep.kind == 3) {
    const uint4* xp = reinterpret_cast<const uint4*>(row + n);
#pragma unroll
    for (int q = 0; q < 4; ++q) in.x[q] = xp[q];
  }
}
// v0, v1 += the two bf16 values of w (packed fp32x2 add).
__device__ __forceinline__ void f2_add_bf16(float& v0, float& v1, uint32_t w) {
  f2_unpack(f2_add(f2_pack(v0, v1), f2_pack(bf16_lo(w), bf16_hi(w))), v0, v1);
}
// Kind 0: row[n..n+32) = bf16(GELU(v + bias)). Kinds 1, 3: row[n..n+32) = bf16(x + v + bias).
// Kind 2: bf16(v + bias), each 16 columns (within one head: dh is a multiple of 16) to its place.
// Kind 4: row[n..n+32) = fp16(v * scale).
__device__ __forceinline__ void epi_store(const GemmEpilogue& ep, uint16_t* row, int n,
                                          const Epi32In& in, float (&v)[32]) {
  if (ep.kind == 4) {
    uint4* d = reinterpret_cast<uint4*>(row + n);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const __half2 h = __floats2half2_rn(v[q * 8 + 2 * e] * ep.scale, v[q * 8 + 2 * e + 1] * ep.scale);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      d[q] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return;
  }
  if (ep.bias) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w[4] = {in.b[q].x, in.b[q].y, in.b[q].z, in.b[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) f2_add_bf16(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1], w[e]);
    }
  }
  if (ep.kind == 2) {
#pragma unroll
    for (int j = 0; j < 2; ++j) {
      const int c = n + 16 * j;
      const int which = c / ep.C, r = c - which * ep.C, h = r / ep.dh, d = r - h * ep.dh;
      uint4* dst = reinterpret_cast<uint4*>(row + which * ep.which_stride +
                                            (size_t)h * ep.ur.N * ep.dh + d);
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const float* f = v + 16 * j + 8 * q;
        uint4 w;
        w.x = pack_bf16(f[0], f[1]);
        w.y = pack_bf16(f[2], f[3]);
        w.z = pack_bf16(f[4], f[5]);
        w.w = pack_bf16(f[6], f[7]);
        dst[q] = w;
      }
    }
    return;
  }
  if (ep.kind == 0) {
#pragma unroll
    for (int i = 0; i < 16; ++i) gelu_erf2(v[2 * i], v[2 * i + 1]);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w[4] = {in.x[q].x, in.x[q].y, in.x[q].z, in.x[q].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) f2_add_bf16(v[q * 8 + 2 * e], v[q * 8 + 2 * e + 1], w[e]);
    }
  }
  uint4* d = reinterpret_cast<uint4*>(row + n);
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint4 w;
    w.x = pack_bf16(v[q * 8 + 0], v[q * 8 + 1]);
    w.y = pack_bf16(v[q * 8 + 2], v[q * 8 + 3]);
    w.z = pack_bf16(v[q * 8 + 4], v[q * 8 + 5]);
    w.w = pack_bf16(v[q * 8 + 6], v[q * 8 + 7]);
    d[q] = w;
  }
}

template <int BN, int KSUB>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb,
           const GemmShape g, const GemmEpilogue ep, int* status) {
  using G = GemmCfg<BN, KSUB>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kBar);
  uint64_t* empty = full + G::kStages;
  uint64_t* acc_full = empty + G::kStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;        // [2]
  uint64_t* epi_bar = acc_empty + 2;         // epilogue-warps rendezvous (bounded, unlike bar.sync)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(epi_bar + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);
  volatile int* s_last = reinterpret_cast<volatile int*>(tmem_slot + 2);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int units = g.units;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G::kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(acc_full + b, 1);
      mbar_init(acc_empty + b, kEpiThreads);
    }
    mbar_init(epi_bar, kEpiThreads);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, G::kTmemCols);
  tc_fence_before();
  cta_sync_converged();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // A and the epilogue's x come from the work before this launch; the producer waits for it
  // itself, after requesting the B (weight) tiles that do not depend on it.
  const bool producer = warp == 0 && lane == 0;
  if (!producer) {
    griddep_wait();
    griddep_launch();
  }

  // Unit u -> tile (m, n), k-split s and its k-block range; pair: finished with its partner
  // split (paired protocol), slot: the pair's partial and counter slot.
  auto decode = [&](int u, int& m, int& n, int& s, int& kb0, int& kb1, int& slot, bool& pair) {
    if (u < g.whole) {
      m = u % g.m_tiles;
      const int r = u / g.m_tiles;
      n = r % g.n_tiles;
      s = r / g.n_tiles;
      kb0 = (int)((long long)s * g.kb_total / g.splits);
      kb1 = (int)((long long)(s + 1) * g.kb_total / g.splits);
      slot = n * g.m_tiles + m;
      pair = g.paired;
    } else {
      // tail: units whole + 2i and whole + 2i + 1 are the two k-halves of tile whole + i
      const int v = u - g.whole, t = g.whole + (v >> 1);
      m = t % g.m_tiles;
      n = t / g.m_tiles;
      s = v & 1;
      kb0 = s ? g.kb_total / 2 : 0;
      kb1 = s ? g.kb_total : g.kb_total / 2;
      slot = v >> 1;
      pair = true;
    }
  };

  if (warp < 4) {
    setmaxnreg_dec<kGemmRegsProducer>();
    if (producer) {
      tma_prefetch_desc(&ta);
      tma_prefetch_desc(&tb);
      // B tiles of the first unit's first stages, before the wait for the previous work.
      int pre = 0;
      if (blockIdx.x < units) {
        int m, n, s, kb0, kb1, slot;
        bool pair;
        decode(blockIdx.x, m, n, s, kb0, kb1, slot, pair);
        const int nst = (kb1 - kb0) / KSUB, rot = blockIdx.x % nst;
        pre = nst < G::kStages ? nst : G::kStages;
        for (int j = 0; j < pre; ++j) {
          const int kb = kb0 + ((j + rot) % nst) * KSUB;
          uint8_t* sb = smem + j * G::kStageBytes + KSUB * G::kABytes;
          mbar_expect_tx(full + j, G::kStageBytes);
#pragma unroll
          for (int q = 0; q < KSUB; ++q)
            tma_load_2d(sb + q * G::kBBytes, &tb, full + j, (kb + q) * 64, n * BN);
        }
      }
      griddep_wait();
      griddep_launch();
      int it = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x) {
        int m, n, s, kb0, kb1, slot;
        bool pair;
        decode(u, m, n, s, kb0, kb1, slot, pair);
        const int nst = (kb1 - kb0) / KSUB, rot = u % nst;
        for (int j = 0; j < nst; ++j, ++it) {
          const int kb = kb0 + ((j + rot) % nst) * KSUB;   // rotated start: spread over L2 slices
          const int st = it % G::kStages;
          if (it >= G::kStages &&
              !(ok = mbar_wait(empty + st, ((it / G::kStages) - 1) & 1, abort, status)))
            break;
          uint8_t* sa = smem + st * G::kStageBytes;
          uint8_t* sb = sa + KSUB * G::kABytes;
          const bool b_done = it < pre;   // B of this stage requested before the wait
          if (!b_done) mbar_expect_tx(full + st, G::kStageBytes);
#pragma unroll
          for (int q = 0; q < KSUB; ++q) {
            tma_load_2d(sa + q * G::kABytes, &ta, full + st, (kb + q) * 64, m * 128);
            if (!b_done) tma_load_2d(sb + q * G::kBBytes, &tb, full + st, (kb + q) * 64, n * BN);
          }
        }
      }
    } else if (warp == 1 && lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      int it = 0, i = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < units; u += gridDim.x, ++i) {
        int m, n, s, kb0, kb1, slot;
        bool pair;
        decode(u, m, n, s, kb0, kb1, slot, pair);
        const int buf = i & 1;
        if (i >= 2 && !(ok = mbar_wait(acc_empty + buf, ((i >> 1) - 1) & 1, abort, status))) break;
        tc_fence_after();
        const uint32_t d = tmem + buf * BN;
        const int nst = (kb1 - kb0) / KSUB;
        bool ready = mbar_test(full + it % G::kStages, (it / G::kStages) & 1);
        for (int j = 0; j < nst; ++j, ++it) {
          const int st = it % G::kStages;
          if (!__builtin_expect(ready, 1) &&
              !(ok = mbar_wait(full + st, (it / G::kStages) & 1, abort, status)))
            break;
          // test the next stage now: its latency hides behind this stage's MMA issue
          if (j + 1 < nst) ready = mbar_test(full + (it + 1) % G::kStages, ((it + 1) / G::kStages) & 1);
          tc_fence_after();
          const uint32_t a_addr = smem_u32(smem + st * G::kStageBytes);
          const uint32_t b_addr = a_addr + KSUB * G::kABytes;
#pragma unroll
          for (int q = 0; q < KSUB; ++q)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_ss(d, smem_desc(a_addr + q * G::kABytes + kk * 32, 16, 1024, kSwizzle128B),
                           smem_desc(b_addr + q * G::kBBytes + kk * 32, 16, 1024, kSwizzle128B),
                           idesc, (j > 0 || q > 0 || kk > 0) ? 1u : 0u);
          umma_commit(empty + st);
        }
        if (ok) umma_commit(acc_full + buf);
      }
    }
  } else {
    setmaxnreg_inc<kGemmRegsEpilogue>();
    // ------------------------------ epilogue warps ----------------------------
    const int ew = warp - 4;                              // 0..7
    const int row = 32 * (warp & 3) + lane;               // TMEM lane
    const int col0 = (ew >> 2) * G::kHalf;                // this warp's half of the columns
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    uint32_t epi_phase = 0;
    // All epilogue threads meet here; a wait that gives up ends every caller's unit loop.
    auto epi_sync = [&]() -> bool {
      mbar_arrive(epi_bar);
      const bool r = mbar_wait(epi_bar, epi_phase, abort, status);
      epi_phase ^= 1;
      return r;
    };
    int i = 0;
    for (int u = blockIdx.x; u < units; u += gridDim.x, ++i) {
      int m_t, n_t, s, kb0, kb1, slot;
      bool pair;
      decode(u, m_t, n_t, s, kb0, kb1, slot, pair);
      const int buf = i & 1;
      const bool ok = __all_sync(0xffffffffu, mbar_wait(acc_full + buf, (i >> 1) & 1, abort, status));
      if (!ok) break;
      tc_fence_after();
      const int m = m_t * 128 + row;
      const int tile = n_t * g.m_tiles + m_t;
      const uint32_t t_acc = tmem + buf * BN + lane_off + col0;
      uint16_t* drow = m < g.M ? epi_row(ep, g, m, status) : nullptr;
      if (g.splits == 1 && !pair) {
#pragma unroll 1
        for (int c = 0; c < G::kHalf / 32; ++c) {
          const int n = n_t * BN + col0 + c * 32;
          Epi32In in;
          if (drow) epi_load(ep, drow, n, in);
          uint32_t r[32];
          tmem_ld32(t_acc + c * 32, r);
          if (c == G::kHalf / 32 - 1) {
            tc_fence_before();
            mbar_arrive(acc_empty + buf);   // accumulator fully read: MMA may reuse it
          }
          if (drow) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]);
            epi_store(ep, drow, n, in, v);
          }
        }
      } else if (pair) {
        // Two k-splits of the tile run at the same time in two CTAs; split s finishes column half
        // s. All eight epilogue warps take part in both jobs, 32-column chunk by chunk (warp group
        // hg takes chunks hg, hg + 2, ...): first they hand the partner's half of their rows to the
        // partner as an fp32 partial (column-major: a warp's 32 rows of one column are one
        // 128-byte line) and count themselves on that half's counter; then each waits for the
        // partner's eight warps and adds its partial to its own half's chunks (acc_s +
        // partial_(1-s): for two terms the same sum as p0 + p1 in either order) and applies the
        // epilogue.
        constexpr int kChunks = G::kHalf / 32;
        const int hg = ew >> 2, other = 1 - s;
        const uint32_t t_row = tmem + buf * BN + lane_off;
        float* part_out = g.partial + ((size_t)slot * 2 + other) * 128 * G::kHalf + row;
        float* part_in = g.partial + ((size_t)slot * 2 + s) * 128 * G::kHalf + row;
        int* count_out = g.counters + slot * 2 + other;
        int* count_in = g.counters + slot * 2 + s;
#pragma unroll 1
        for (int c = hg; c < kChunks; c += 2) {
          uint32_t r[32];
          tmem_ld32(t_row + other * G::kHalf + c * 32, r);
#pragma unroll
          for (int e = 0; e < 32; ++e)
            part_out[(size_t)(c * 32 + e) * 128] = __uint_as_float(r[e]);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) add_release(count_out, 1);   // this warp's share of the partner's half
        // Every lane acquires the counter itself before reading the partial.
        if (!__all_sync(0xffffffffu, wait_counter_geq(count_in, 8, abort, status))) break;
#pragma unroll 1
        for (int c = hg; c < kChunks; c += 2) {
          const int n = n_t * BN + s * G::kHalf + c * 32;
          Epi32In in;
          float w[32];
          if (drow) {
            epi_load(ep, drow, n, in);
#pragma unroll
            for (int e = 0; e < 32; ++e) w[e] = __ldcg(part_in + (size_t)(c * 32 + e) * 128);
          }
          uint32_t r[32];
          tmem_ld32(t_row + s * G::kHalf + c * 32, r);
          if (drow) {
            float v[32];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __uint_as_float(r[e]) + w[e];
            epi_store(ep, drow, n, in, v);
          }
        }
        tc_fence_before();
        mbar_arrive(acc_empty + buf);   // this warp's reads of the accumulator are done
        // The last of the sixteen arrivals on this half's counter (the partner's eight writer
        // arrivals, then this CTA's eight warps once finished) re-arms it for a later GEMM.
        if (lane == 0 && atomicAdd(count_in, 1) == 15) atomicExch(count_in, 0);
      } else {
        // Write this split's partial tile (column-major, so a warp's 32 rows of one column are
        // one 128-byte line), then let the last split of the tile finish it.
        float* slot = g.partial + ((size_t)tile * g.splits + s) * 128 * BN + (size_t)col0 * 128 + row;
#pragma unroll 1
        for (int c = 0; c < G::kHalf / 32; ++c) {
          uint32_t r[32];
          tmem_ld32(t_acc + c * 32, r);
          if (c == G::kHalf / 32 - 1) {
            tc_fence_before();
            mbar_arrive(acc_empty + buf);
          }
#pragma unroll
          for (int e = 0; e < 32; ++e) slot[(size_t)(c * 32 + e) * 128] = __uint_as_float(r[e]);
        }
        __threadfence();
        if (!epi_sync()) break;
        if (threadIdx.x == 128) *s_last = atomicAdd(g.counters + tile, 1) == g.splits - 1;
        if (!epi_sync()) break;
        if (*s_last) {
          __threadfence();
          if (drow) {
            const float* base =
                g.partial + (size_t)tile * g.splits * 128 * BN + (size_t)col0 * 128 + row;
#pragma unroll 1
            for (int c = 0; c < G::kHalf / 32; ++c) {
              const int n = n_t * BN + col0 + c * 32;
              Epi32In in;
              epi_load(ep, drow, n, in);
              // Split 0's values and split 1's are loaded before either is added (64 loads in
              // flight); further splits follow in the same fixed order: a deterministic sum.
              const float* src = base + (size_t)c * 32 * 128;
              float v[32];
#pragma unroll
              for (int e = 0; e < 32; ++e) v[e] = __ldcg(src + (size_t)e * 128);
              for (int sp = 1; sp < g.splits; ++sp) {
                const float* s2 = src + (size_t)sp * 128 * BN;
                float w[32];
#pragma unroll
                for (int e = 0; e < 32; ++e) w[e] = __ldcg(s2 + (size_t)e * 128);
#pragma unroll
                for (int e = 0; e < 32; ++e) v[e] += w[e];
              }
              epi_store(ep, drow, n, in, v);
            }
          }
          if (threadIdx.x == 128) g.counters[tile] = 0;
        }
        if (!epi_sync()) break;   // s_last is reused by the next unit
      }
    }
  }
  tc_fence_before();
  cta_sync_converged();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

GemmPlan gemm_plan(int M, int N, int Kd, int sms) {
  GemmPlan p;
  const int m_tiles = (M + 127) / 128;
  const int kb = Kd / 64;
  // Pick the tile width and k-split with the smallest makespan, counted in operand bytes that
  // the busiest CTA moves from L2 into shared memory (the measured bound of these GEMMs: one
  // 64-wide k-block of a 128 x BN tile reads 128 + BN rows of 128 B). Rounds of (tile, split)
  // units over the CTAs, times k-blocks per unit, times (128 + BN); a k-split adds the unit's fp32
  // partial tile written (4 BN rows' worth) and, for the unit that finishes the tile, all `s`
  // partials read back. Splits only for long K (>= 24 k-blocks).
  // Without a k-split, a last partial round of R <= sms/2 tiles runs as 2R k-halves (the tail),
  // which costs half a unit plus the pair's partial exchange.
  long long best = -1;
  p.bn = 64;
  p.splits = 1;
  p.tail = 0;
  for (int bn : {256, 192, 128, 64}) {
    if (N % bn) continue;
    const int n_tiles = N / bn;
    for (int s = 1; s <= 8; ++s) {
      if (s > 1 && (kb < 24 || kb / s < 4)) break;
      const long long units = (long long)m_tiles * n_tiles * s;
      long long rounds = (units + sms - 1) / sms;
      const long long kb_unit = (kb + s - 1) / s;
      const long long partial = s > 1 ? (rounds + s) * 4LL * bn : 0;
      long long cost = rounds * kb_unit * (128 + bn) + partial;
      int tail = 0;
      if (s == 1) {
        tail = gemm_tail(m_tiles * n_tiles, kb, sms);
        if (tail) cost = (rounds - 1) * kb * (128 + bn) + (kb / 2) * (128 + bn) + 2 * 4LL * bn;
      }
      if (best < 0 || cost < best) {
        best = cost;
        p.bn = bn;
        p.splits = s;
        p.tail = tail;
      }
    }
  }
  p.m_tiles = m_tiles;
  p.n_tiles = N / p.bn;
  p.units = m_tiles * p.n_tiles * p.splits + p.tail;
  return p;
}

// Only for long K: the halves save kb/2 k-blocks of mainloop, while the pair's partial exchange
// and the unchanged epilogue of the last unit cost a fixed amount (measured on B200: a loss at 12
// k-blocks, about even at 16 and 20, a clear gain at 80).
constexpr int kTailMinKb = 24;
int gemm_tail(int tiles, int kb, int sms) {
  const int r = tiles % sms;
  return tiles > sms && r > 0 && 2 * r <= sms && kb >= kTailMinKb && kb % 2 == 0 ? r : 0;
}

size_t gemm_partial_bytes(const GemmPlan& p) {
  if (p.splits == 1) return (size_t)p.tail * 128 * p.bn * 4;
  return (size_t)p.m_tiles * p.n_tiles * p.splits * 128 * p.bn * 4;
}

template <int BN, int KSUB>
static cudaError_t launch_gemm_bn(const CUtensorMap* ta, const CUtensorMap* tb, const GemmPlan& p,
                                  int M, int N, int Kd, const GemmEpilogue& ep, float* partial,
                                  int* counters, int sms, int* status, cudaStream_t st) {
  using G = GemmCfg<BN, KSUB>;
  cudaError_t e = cudaFuncSetAttribute(k_gemm<BN, KSUB>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, G::kAlloc);
  if (e != cudaSuccess) return e;
  GemmShape g;
  g.M = M;
  g.N = N;
  g.Kd = Kd;
  g.m_tiles = p.m_tiles;
  g.n_tiles = p.n_tiles;
  g.splits = p.splits;
  g.kb_total = Kd / 64;
  g.partial = partial;
  g.counters = counters;
  // The tail as planned holds only for the SM count it was planned for (its partial workspace
  // is sized by it); on another count the last round runs whole tiles.
  const int tiles = p.m_tiles * p.n_tiles;
  const int tail =
      p.splits == 1 && p.tail > 0 && gemm_tail(tiles, g.kb_total, sms) == p.tail ? p.tail : 0;
  g.units = tiles * p.splits + tail;
  g.whole = tiles * p.splits - tail;
  const int grid = g.units < sms ? g.units : sms;
  // Every unit has its own CTA (one per SM, all resident together), so the two splits of a tile
  // can wait for each other; the tail halves all run in the last round, every CTA's earlier units
  // waiting on nothing.
  g.paired = p.splits == 2 && g.units <= grid;
  return launch_pdl(k_gemm<BN, KSUB>, dim3(grid), dim3(kGemmThreads), G::kAlloc, st, *ta, *tb, g, ep,
                    status);
}

cudaError_t launch_gemm(const CUtensorMap* ta, const CUtensorMap* tb, const GemmPlan& p, int M,
                        int N, int Kd, const GemmEpilogue& ep, float* partial, int* counters,
                        int sms, int* status, cudaStream_t st) {
  // Two sub-blocks per stage when every unit's k-range splits evenly (BN 192 and 256 keep one:
  // their 80 and 96 KB double stages would leave only two stages).
  const int kb = Kd / 64;
  const bool two = p.bn <= 128 && kb % p.splits == 0 && (kb / p.splits) % 2 == 0 &&
                   (p.tail == 0 || (kb / 2) % 2 == 0);
  switch (p.bn) {
    case 64:
      return two ? launch_gemm_bn<64, 2>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st)
                 : launch_gemm_bn<64, 1>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st);
    case 128:
      return two ? launch_gemm_bn<128, 2>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st)
                 : launch_gemm_bn<128, 1>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st);
    case 192:
      return launch_gemm_bn<192, 1>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st);
    case 256:
      return launch_gemm_bn<256, 1>(ta, tb, p, M, N, Kd, ep, partial, counters, sms, status, st);
  }
  return cudaErrorInvalidValue;
}

cudaError_t set_wait_limit_mlp(uint64_t ns) { return set_wait_limit_here(ns); }

}  // namespace ss
