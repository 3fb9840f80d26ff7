// Geometry and static-pattern arithmetic of Stripe-Sort attention, for host and device.
//
// SparseSAM Dutch technical summary, "Statisch Sparsiteitspatroon": the stripe permutation splits
// the N x N attention matrix into a 4 x 4 mosaic of sub-maps, each banded around its diagonal, plus
// a small global keep-set; the SparseSAM README's `ratio` is the computed fraction (density). The
// pages give no constants. This file implements one reading: block size b = largest divisor of
// L = N/4 with b <= 64 and L/b >= 4; a band of W offset blocks starting at
// clamp(a - (W-1)/2, 0, nb - W); offset block 0 kept by every query; W chosen so the realised
// density is nearest to the requested one (ties to the smaller W).
#pragma once

#include <math.h>
#include <stdint.h>

#ifdef __CUDACC__
#define SS_HD __host__ __device__ __forceinline__
#else
#define SS_HD inline
#endif

namespace ss {

constexpr int kStripes = 4;
constexpr int kMaxBlock = 64;
constexpr int kGlobalBlocks = 1;

SS_HD int block_size_for(int L) {
  for (int b = (L < kMaxBlock ? L : kMaxBlock); b >= 1; --b)
    if (L % b == 0 && L / b >= 4) return b;
  return 0;
}

SS_HD int band_start(int a, int W, int nb) {
  int s = a - (W - 1) / 2;
  if (s < 0) s = 0;
  if (s > nb - W) s = nb - W;
  return s;
}

// Kept key offset blocks of query offset block a: [s, s+W) united with [0, g).
SS_HD bool block_kept(int a, int a_key, int W, int nb, int g) {
  if (a_key < g) return true;
  int s = band_start(a, W, nb);
  return a_key >= s && a_key < s + W;
}

SS_HD int row_count(int a, int W, int nb, int g) {
  int s = band_start(a, W, nb);
  int below = g < s ? g : s;                 // [0, g) blocks left of the band
  int above = g - (s + W) > 0 ? g - (s + W) : 0;
  return W + below + above;
}

inline int pattern_nnz(int W, int nb, int g) {
  int n = 0;
  for (int a = 0; a < nb; ++a) n += row_count(a, W, nb, g);
  return n;
}

// Band width whose density nnz/nb^2 is nearest to `density`; ties go to the smaller W.
inline int choose_band(int nb, int g, double density) {
  int best = 1;
  double best_err = -1.0;
  for (int W = 1; W <= nb; ++W) {
    double rho = (double)pattern_nnz(W, nb, g) / (double)(nb * nb);
    double err = fabs(rho - density);
    if (best_err < 0.0 || err < best_err) {
      best_err = err;
      best = W;
    }
  }
  return best;
}

// K = ceil(density * tokens - 1e-9) in double.
inline int keep_count(double density, int tokens) {
  volatile double prod = density * (double)tokens;   // keep the product and the guard separate
  return (int)ceil(prod - 1e-9);
}

// Block-major position q of the gathered sequence -> canonical permuted position p.
// The gathered layout stores offset block a of all 4 stripes contiguously:
//   q = a*(4b) + j*b + r   <->   p = j*L + a*b + r.
SS_HD int blockmajor_to_canonical(int q, int b, int L) {
  int b4 = b * kStripes;
  int a = q / b4;
  int rem = q - a * b4;
  int j = rem / b;
  int r = rem - j * b;
  return j * L + a * b + r;
}

// The inverse: canonical permuted position p -> block-major position q.
SS_HD int canonical_to_blockmajor(int p, int b, int L) {
  int j = p / L;
  int rem = p - j * L;
  int a = rem / b;
  int r = rem - a * b;
  return a * (b * kStripes) + j * b + r;
}

}  // namespace ss
