// The encoder block's LayerNorms (SAM's ViT block: pre-norm before the attention and before the
// MLP), as row kernels that also place the rows: LN1 writes the block's attention units (window
// partition with zero pad rows, or the image as it is), LN2 gathers and normalises the RC-MLP's
// kept rows. Both are HBM-bound: one read and one write of each row, statistics in registers.
#include "common.cuh"
#include "kernels.h"

namespace ss {

constexpr float kLnEps = 1e-6f;

// One warp per output row; lane l holds chunks l, l + 32, ... (KPL of them) of the row's C/8
// 16-byte chunks. Mean, then the sum of squared deviations from it (two passes over registers),
// each reduced over the warp in fp32.
template <int KPL>
__global__ void __launch_bounds__(256) k_ln_rows(const uint16_t* __restrict__ x,
                                                 const uint16_t* __restrict__ w,
                                                 const uint16_t* __restrict__ b,
                                                 uint16_t* __restrict__ out, long long rows, int C,
                                                 UnitRows ur, const int32_t* __restrict__ keep,
                                                 int K, int* __restrict__ zero, int nzero,
                                                 int* status) {
  griddep_wait();
  griddep_launch();
  if (blockIdx.x == 0)
    for (int i = threadIdx.x; i < nzero; i += blockDim.x) zero[i] = 0;
  const long long m = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (m >= rows) return;
  long long src;
  if (keep) {
    const long long img = m / K;
    const int t = __ldg(keep + m);
    if ((unsigned)t >= (unsigned)ur.T) {
      if (lane == 0) record_bad_index(status);
      return;
    }
    src = img * ur.T + t;
  } else {
    src = unit_row_src(ur, m);
  }
  const int cpr = C / 8;
  uint4* dst = reinterpret_cast<uint4*>(out + (size_t)m * C);
  if (src < 0) {   // a pad token of a windowed block: a zero row
#pragma unroll
    for (int e = 0; e < KPL; ++e)
      if (e * 32 + lane < cpr) dst[e * 32 + lane] = make_uint4(0, 0, 0, 0);
    return;
  }
  const uint4* xr = reinterpret_cast<const uint4*>(x + (size_t)src * C);
  uint4 raw[KPL];
#pragma unroll
  for (int e = 0; e < KPL; ++e) raw[e] = make_uint4(0, 0, 0, 0);
#pragma unroll
  for (int e = 0; e < KPL; ++e)
    if (e * 32 + lane < cpr) raw[e] = __ldg(xr + e * 32 + lane);
  float f[KPL][8];
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const uint32_t u[4] = {raw[e].x, raw[e].y, raw[e].z, raw[e].w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      f[e][2 * j] = __uint_as_float(u[j] << 16);
      f[e][2 * j + 1] = __uint_as_float(u[j] & 0xFFFF0000u);
    }
    if (e * 32 + lane < cpr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) s += f[e][j];
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  const float mean = s / (float)C;
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    if (e * 32 + lane < cpr) {
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const float d = f[e][j] - mean;
        ss += d * d;
      }
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, o);
  const float rstd = 1.0f / sqrtf(ss / (float)C + kLnEps);
  const uint4* wr = reinterpret_cast<const uint4*>(w);
  const uint4* br = reinterpret_cast<const uint4*>(b);
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int c = e * 32 + lane;
    if (c >= cpr) continue;
    const uint4 wv = __ldg(wr + c), bv = __ldg(br + c);
    const uint32_t wu[4] = {wv.x, wv.y, wv.z, wv.w}, bu[4] = {bv.x, bv.y, bv.z, bv.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const float y0 = (f[e][2 * j] - mean) * rstd * __uint_as_float(wu[j] << 16) +
                       __uint_as_float(bu[j] << 16);
      const float y1 = (f[e][2 * j + 1] - mean) * rstd * __uint_as_float(wu[j] & 0xFFFF0000u) +
                       __uint_as_float(bu[j] & 0xFFFF0000u);
      o[j] = pack_bf16(y0, y1);
    }
    dst[c] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_ln_rows(const uint16_t* x, const uint16_t* w, const uint16_t* b, uint16_t* out,
                           long long rows, int C, const UnitRows& ur, const int32_t* keep, int K,
                           int* zero, int nzero, int* status, cudaStream_t st) {
  if (C % 8 != 0 || C > 8 * 32 * 8) return cudaErrorInvalidValue;
  const int kpl = (C / 8 + 31) / 32;
  const dim3 grid((unsigned)((rows + 7) / 8)), block(256);
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, grid, block, 0, st, x, w, b, out, rows, C, ur, keep, K, zero, nzero,
                      status);
  };
  switch (kpl) {
    case 1: return go(k_ln_rows<1>);
    case 2: return go(k_ln_rows<2>);
    case 3: return go(k_ln_rows<3>);
    case 4: return go(k_ln_rows<4>);
    case 5: return go(k_ln_rows<5>);
    default: return go(k_ln_rows<8>);
  }
}

}  // namespace ss
