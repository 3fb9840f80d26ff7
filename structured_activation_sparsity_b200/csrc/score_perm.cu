// S1 Sobel score and S2 stripe-sort permutation kernels.
//
// S1 follows the SparseSAM Dutch technical summary, "Op Gradiënten Gebaseerde Ordening" (a
// parameter-free Sobel operator's gradient magnitude per token). S2 follows "Stripe-Sort
// Permutatie" (sort by that score, read the sorted list as a matrix, transpose, flatten).
//
// The sort is done by rank counting rather than a comparison network: rank(t) = number of tokens
// that come before t in the stable descending order. With N <= 16384 tokens per unit that is N^2
// independent compares spread over the whole GPU (32 target tokens per CTA, 8 warps splitting the
// other tokens), no synchronisation beyond one CTA-level reduction, and the result is the stable
// order by construction. Each rank is scattered straight into perm, inv and the keep list.
#include "common.cuh"
#include "kernels.h"

namespace ss {

// Squared Sobel gradient magnitude from the 3 x 3 neighbourhood (rows m, 0, p = y-1, y, y+1;
// columns m, 0, p = x-1, x, x+1). Each step is one fp64 round-to-nearest operation, in a fixed
// order, never fused, so every caller gets the same bits.
__device__ __forceinline__ double sobel_of(double l_mm, double l_m0, double l_mp, double l_0m,
                                           double l_0p, double l_pm, double l_p0, double l_pp) {
  double gx = __dadd_rn(__dadd_rn(__dsub_rn(l_mp, l_mm), __dmul_rn(2.0, __dsub_rn(l_0p, l_0m))),
                        __dsub_rn(l_pp, l_pm));
  double gy = __dadd_rn(__dadd_rn(__dsub_rn(l_pm, l_mm), __dmul_rn(2.0, __dsub_rn(l_p0, l_m0))),
                        __dsub_rn(l_pp, l_mp));
  return __dadd_rn(__dmul_rn(gx, gx), __dmul_rn(gy, gy));
}
// Of pixel (y, x) of an H x W image, replicate border.
__device__ __forceinline__ double sobel_at(const float* __restrict__ img, int H, int W, int y,
                                           int x) {
  int ym = y > 0 ? y - 1 : 0, yp = y < H - 1 ? y + 1 : H - 1;
  int xm = x > 0 ? x - 1 : 0, xp = x < W - 1 ? x + 1 : W - 1;
  return sobel_of(img[ym * W + xm], img[ym * W + x], img[ym * W + xp], img[y * W + xm],
                  img[y * W + xp], img[yp * W + xm], img[yp * W + x], img[yp * W + xp]);
}

__global__ void __launch_bounds__(256) k_sobel_score(const float* __restrict__ lum,
                                                     double* __restrict__ score, int B, int H,
                                                     int W) {
  griddep_wait();
  griddep_launch();
  int idx = blockIdx.x * blockDim.x + threadIdx.x;
  int per = H * W;
  if (idx >= B * per) return;
  int b = idx / per;
  int r = idx - b * per;
  int y = r / W, x = r - (r / W) * W;
  score[idx] = sobel_at(lum + (size_t)b * per, H, W, y, x);
}

// Order-preserving 64-bit key of a double: for any non-NaN a, b, a < b exactly when
// key(a) < key(b) as unsigned integers, and -0.0 and +0.0 share one key (they compare equal, so the
// stable sort keeps their enumeration order). Negative values have their bits inverted (so a more
// negative value gets a smaller key), non-negative values get the sign bit set (so they sit above
// every negative one).
__device__ __forceinline__ unsigned long long order_key(double v) {
  unsigned long long u = (unsigned long long)__double_as_longlong(v);
  if (u == 0x8000000000000000ull) u = 0ull;   // -0.0 -> +0.0
  return (u >> 63) ? ~u : (u | 0x8000000000000000ull);
}
// The double whose order_key is k (for -0.0, +0.0).
__device__ __forceinline__ double key_value(unsigned long long k) {
  return __longlong_as_double((long long)((k >> 63) ? (k & 0x7fffffffffffffffull) : ~k));
}

// Unit-local token t -> its score's order key.
struct UnitMap {
  int window_mode;   // 0: unit = image, t = raster index; 1: unit = window, t = window raster
  int Hg, Wg, ws, wpr, nwin;
  // Image b and pixel (y, x) of unit-local token t; false for a window's pad token.
  __device__ __forceinline__ bool locate(int u, int t, int& b, int& y, int& x) const {
    if (!window_mode) {
      b = u;
      y = t / Wg;
      x = t - y * Wg;
      return true;
    }
    b = u / nwin;
    const int w = u - b * nwin;
    const int wy = w / wpr, wx = w - (w / wpr) * wpr;
    y = wy * ws + t / ws;
    x = wx * ws + t % ws;
    return y < Hg && x < Wg;
  }
  __device__ __forceinline__ unsigned long long key(const double* score, int u, int t) const {
    int b, y, x;
    if (!locate(u, t, b, y, x)) return order_key(0.0);   // pad token: +0.0
    return order_key(score[((size_t)b * Hg + y) * Wg + x]);
  }
  // The same key computed from the luminance (S1 fused into S2).
  __device__ __forceinline__ unsigned long long key_lum(const float* lum, int u, int t) const {
    int b, y, x;
    if (!locate(u, t, b, y, x)) return order_key(0.0);
    return order_key(sobel_at(lum + (size_t)b * Hg * Wg, Hg, Wg, y, x));
  }
};

// grid (ceil(N/(32*TG)), units), block 32 * WARPS, dynamic smem N * 8 bytes (16-byte aligned).
// Each CTA ranks TG groups of 32 target tokens; its WARPS warps split the unit's keys and count,
// for the 32 targets of a group at once, the keys that come before each target. More groups per
// CTA mean fewer CTAs filling the same keys (worth it once the grid exceeds a couple of waves).
// FROM_LUM: the keys are the Sobel scores computed here from `lum` (S1 fused into S2); each CTA
// also stores the scores of its target tokens into `score_out`, so every real token's score is
// written once.
template <int WARPS, bool FROM_LUM, int TG = 1>
__global__ void __launch_bounds__(32 * WARPS) k_stripe_rank(const double* __restrict__ score,
                                                            const float* __restrict__ lum,
                                                            double* __restrict__ score_out,
                                                            UnitMap m, int N, int K,
                                                            int32_t* __restrict__ perm,
                                                            int32_t* __restrict__ inv,
                                                            int32_t* __restrict__ keep) {
  extern __shared__ __align__(16) unsigned long long s_key[];
  __shared__ int s_cnt[TG][WARPS][32];
  griddep_wait();
  griddep_launch();
  const int u = blockIdx.y;
  if (FROM_LUM && !m.window_mode && (m.Wg & 3) == 0) {
    // The whole image's keys, four horizontally adjacent pixels per thread from one 3 x 6
    // neighbourhood (18 loads and conversions for four keys instead of 32).
    const float* img = lum + (size_t)u * N;
    const int W = m.Wg, H = m.Hg, qpr = W >> 2;
    for (int q = threadIdx.x; q < N / 4; q += blockDim.x) {
      const int y = q / qpr, x0 = (q - y * qpr) * 4;
      const int rows[3] = {y > 0 ? y - 1 : 0, y, y < H - 1 ? y + 1 : H - 1};
      double l[3][6];
#pragma unroll
      for (int r = 0; r < 3; ++r)
#pragma unroll
        for (int c = 0; c < 6; ++c) {
          const int x = min(max(x0 - 1 + c, 0), W - 1);
          l[r][c] = img[rows[r] * W + x];
        }
      ulonglong2 k2[2];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const double v = sobel_of(l[0][k], l[0][k + 1], l[0][k + 2], l[1][k], l[1][k + 2],
                                  l[2][k], l[2][k + 1], l[2][k + 2]);
        const unsigned long long key = order_key(v);
        if (k & 1) k2[k >> 1].y = key; else k2[k >> 1].x = key;
      }
      reinterpret_cast<ulonglong2*>(s_key)[2 * q] = k2[0];       // y*W + x0 is a multiple of 4
      reinterpret_cast<ulonglong2*>(s_key)[2 * q + 1] = k2[1];
    }
  } else
  // Fill the unit's keys: eight independent loads in flight per thread before any store.
  for (int t0 = threadIdx.x; t0 < N; t0 += 8 * blockDim.x) {
    unsigned long long k8[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int t = t0 + e * blockDim.x;
      k8[e] = t >= N ? 0ull : FROM_LUM ? m.key_lum(lum, u, t) : m.key(score, u, t);
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const int t = t0 + e * blockDim.x;
      if (t < N) s_key[t] = k8[e];
    }
  }
  cta_sync_converged();

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = (((N + WARPS - 1) / WARPS) + 1) & ~1;   // even: pairs stay 16-byte aligned
  const int lo = min(N, warp * chunk), hi = min(N, lo + chunk);
  const ulonglong2* s_pair = reinterpret_cast<const ulonglong2*>(s_key);
#pragma unroll 1
  for (int gi = 0; gi < TG; ++gi) {
    const int t = (blockIdx.x * TG + gi) * 32 + lane;
    const int tt = t < N ? t : N - 1;
    const unsigned long long kt = s_key[tt];
    // Tokens before tt count when their key is >= kt (ties broken by the lower index), tokens
    // after it only when strictly greater: two runs, no per-element index compare. Keys are read
    // in pairs (one 16-byte shared load, the same address across the warp: a broadcast); four
    // independent counters keep the compare chains short.
    const int mid = max(lo, min(hi, tt));
    int c0 = 0, c1 = 0, c2 = 0, c3 = 0;
    int o = lo;
    for (; o + 4 <= mid; o += 4) {
      const ulonglong2 p = s_pair[o >> 1], q = s_pair[(o >> 1) + 1];
      c0 += p.x >= kt;
      c1 += p.y >= kt;
      c2 += q.x >= kt;
      c3 += q.y >= kt;
    }
    for (; o < mid; ++o) c0 += s_key[o] >= kt;
    if ((o & 1) && o < hi) c1 += s_key[o++] > kt;   // back to an even index
    for (; o + 4 <= hi; o += 4) {
      const ulonglong2 p = s_pair[o >> 1], q = s_pair[(o >> 1) + 1];
      c0 += p.x > kt;
      c1 += p.y > kt;
      c2 += q.x > kt;
      c3 += q.y > kt;
    }
    for (; o < hi; ++o) c0 += s_key[o] > kt;
    s_cnt[gi][warp][lane] = (c0 + c1) + (c2 + c3);
  }
  cta_sync_converged();
  if (warp < TG) {
    const int t = (blockIdx.x * TG + warp) * 32 + lane;
    if (t < N) {
      const unsigned long long kt = s_key[t];
      int r = 0;
#pragma unroll
      for (int w = 0; w < WARPS; ++w) r += s_cnt[warp][w][lane];
      const int L = N / kStripes;
      const int pos = (r % kStripes) * L + r / kStripes;   // stripe transpose
      if (perm) perm[(size_t)u * N + pos] = t;
      if (inv) inv[(size_t)u * N + t] = pos;
      if (keep && r < K) keep[(size_t)u * K + r] = t;
      if (FROM_LUM && score_out) {
        int b, y, x;
        if (m.locate(u, t, b, y, x)) score_out[((size_t)b * m.Hg + y) * m.Wg + x] = key_value(kt);
      }
    }
  }
}

cudaError_t launch_sobel_score(const float* lum, double* score, int B, int H, int W,
                               cudaStream_t st) {
  int n = B * H * W;
  return launch_pdl(k_sobel_score, dim3((n + 255) / 256), dim3(256), 0, st, lum, score, B, H, W);
}

cudaError_t launch_stripe_rank(const double* score, const float* lum, double* score_out,
                               int window_mode, int B, int Hg, int Wg, int ws, int units, int N,
                               int K, int32_t* perm, int32_t* inv, int32_t* keep,
                               cudaStream_t st) {
  UnitMap m;
  m.window_mode = window_mode;
  m.Hg = Hg;
  m.Wg = Wg;
  m.ws = ws;
  m.wpr = window_mode ? (Wg + ws - 1) / ws : 1;
  m.nwin = window_mode ? m.wpr * ((Hg + ws - 1) / ws) : 1;
  size_t smem = (size_t)N * sizeof(unsigned long long);
  // Long units split their keys over 32 warps per CTA (a shorter count per warp), short ones
  // over 8 (more CTAs per SM). When one group of 32 targets per CTA would take more than one wave
  // of CTAs (two per SM at 32 warps), each CTA ranks four groups against the keys it filled once.
  const bool big = (long long)units * ((N + 31) / 32) > 2LL * 148;
  auto go = [&](auto kernel, int warps, int tg) -> cudaError_t {
    cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    const dim3 grid((N + 32 * tg - 1) / (32 * tg), units);
    return launch_pdl(kernel, grid, dim3(32 * warps), smem, st, score, lum, score_out, m, N, K,
                      perm, inv, keep);
  };
  if (N >= 2048 && big)
    return lum ? go(k_stripe_rank<32, true, 4>, 32, 4) : go(k_stripe_rank<32, false, 4>, 32, 4);
  if (lum)
    return N >= 2048 ? go(k_stripe_rank<32, true>, 32, 1) : go(k_stripe_rank<8, true>, 8, 1);
  return N >= 2048 ? go(k_stripe_rank<32, false>, 32, 1) : go(k_stripe_rank<8, false>, 8, 1);
}

// ---------------------------------------------------------------------------------------------
// Variants: random scores (the random-permutation ablation) and update magnitudes (a keep
// criterion). Both produce scores that the ranking kernel above turns into perm / keep.
// ---------------------------------------------------------------------------------------------
// Output n of the SplitMix64 generator (Steele, Lea and Flood, "Fast splittable pseudorandom
// number generators", OOPSLA 2014) from state `seed`: the state after n + 1 steps of the golden
// gamma, through the generator's output mix.
__device__ __forceinline__ unsigned long long splitmix64_at(unsigned long long seed,
                                                           unsigned long long n) {
  unsigned long long z = seed + (n + 1ull) * 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// score[i] = (output i >> 11) * 2^-53, uniform in [0, 1), for i < n (= images * tokens).
__global__ void __launch_bounds__(256) k_random_score(double* __restrict__ score, long long n,
                                                      unsigned long long seed) {
  griddep_wait();
  griddep_launch();
  const long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (i < n) score[i] = (double)(splitmix64_at(seed, (unsigned long long)i) >> 11) * 0x1p-53;
}

// mag[r] = sum over c = 0..C-1, in that order, of delta[r, c]^2 (one fp64 round-to-nearest
// operation per multiply and per add, never fused): one thread per token row, 16-byte loads.
__global__ void __launch_bounds__(128) k_update_magnitude(const uint16_t* __restrict__ delta,
                                                          double* __restrict__ mag, long long rows,
                                                          int C) {
  griddep_wait();
  griddep_launch();
  const long long r = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (r >= rows) return;
  const uint4* src = reinterpret_cast<const uint4*>(delta + r * C);
  double acc = 0.0;
  for (int c8 = 0; c8 < C / 8; ++c8) {
    const uint4 w = __ldg(src + c8);
    const uint32_t v[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const double lo = (double)__uint_as_float(v[e] << 16);
      const double hi = (double)__uint_as_float(v[e] & 0xFFFF0000u);
      acc = __dadd_rn(acc, __dmul_rn(lo, lo));
      acc = __dadd_rn(acc, __dmul_rn(hi, hi));
    }
  }
  mag[r] = acc;
}

cudaError_t launch_random_score(double* score, long long n, unsigned long long seed,
                                cudaStream_t st) {
  return launch_pdl(k_random_score, dim3((unsigned)((n + 255) / 256)), dim3(256), 0, st, score, n,
                    seed);
}

cudaError_t launch_update_magnitude(const uint16_t* delta, double* mag, long long rows, int C,
                                    cudaStream_t st) {
  return launch_pdl(k_update_magnitude, dim3((unsigned)((rows + 127) / 128)), dim3(128), 0, st,
                    delta, mag, rows, C);
}

}  // namespace ss
