// Inputs of the relative-position variant of the attention (SAM's decomposed relative positions:
// the score of query (qh, qw) and key (kh, kw) gains q . Rh[qh - kh + Hu - 1] + q . Rw[qw - kw +
// Wu - 1]). The products q . R[r] for every table row r are one tcgen05 GEMM of the gathered Q
// against the two tables stacked (epilogue kind 4); this launch packs those tables into the GEMM's
// B operand and writes, for every key position of every unit, its one-hot row: the attention adds
// a key's two terms to its score with one more MMA (the query rows' bias slices times the key
// tile's one-hot matrix).
#include "common.cuh"
#include "kernels.h"

namespace ss {

// blockIdx.y < U: unit y's one-hot rows, one thread per 16-byte chunk (8 columns) of a row q <
// npad: fp16 1.0 (0x3C00) at columns Hu-1-kh and Hu+Wu-1-kw of the key at block-major position q,
// zeros elsewhere and in the rows past N. blockIdx.y == U: the packed tables, one thread per
// 16-byte chunk of rpack [nr, dh]: rows 0..2Hu-2 = rel_h, then 2Wu-1 rows of rel_w, then zeros.
__global__ void __launch_bounds__(256) k_relpos_prep(const uint16_t* __restrict__ rel_h,
                                                     const uint16_t* __restrict__ rel_w,
                                                     uint16_t* __restrict__ rpack, int dh, int nr,
                                                     const int32_t* __restrict__ perm,
                                                     uint16_t* __restrict__ onehot, int U, int N,
                                                     int npad, int Hu, int Wu, int b, int L,
                                                     int* status) {
  griddep_wait();
  griddep_launch();
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if ((int)blockIdx.y == U) {
    const int cpr = dh / 8;
    if (t >= nr * cpr) return;
    const int r = t / cpr, c = t - r * cpr;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (r < 2 * Hu - 1)
      v = __ldg(reinterpret_cast<const uint4*>(rel_h) + (size_t)r * cpr + c);
    else if (r < 2 * Hu - 1 + 2 * Wu - 1)
      v = __ldg(reinterpret_cast<const uint4*>(rel_w) + (size_t)(r - (2 * Hu - 1)) * cpr + c);
    reinterpret_cast<uint4*>(rpack)[(size_t)r * cpr + c] = v;
    return;
  }
  constexpr int kChunks = kRelPosOneHotCols / 8;
  const int u = blockIdx.y;
  if (t >= npad * kChunks) return;
  const int q = t / kChunks, j = t - q * kChunks;
  int ch = -1, cw = -1;
  if (q < N) {
    const int tok = __ldg(perm + (size_t)u * N + blockmajor_to_canonical(q, b, L));
    if ((unsigned)tok >= (unsigned)N) {
      if (j == 0) record_bad_index(status);
    } else {
      const int kh = tok / Wu, kw = tok - kh * Wu;
      ch = Hu - 1 - kh;
      cw = Hu + Wu - 1 - kw;
    }
  }
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const int c0 = 8 * j + 2 * e;
    w[e] = (c0 == ch || c0 == cw ? 0x3C00u : 0u) | (c0 + 1 == ch || c0 + 1 == cw ? 0x3C000000u : 0u);
  }
  reinterpret_cast<uint4*>(onehot)[((size_t)u * npad + q) * kChunks + j] =
      make_uint4(w[0], w[1], w[2], w[3]);
}

cudaError_t launch_relpos_prep(const uint16_t* rel_h, const uint16_t* rel_w, uint16_t* rpack,
                               int dh, int nr, const int32_t* perm, uint16_t* onehot, int U, int N,
                               int npad, int Hu, int Wu, int b, int* status, cudaStream_t st) {
  const int per = std::max(npad * (kRelPosOneHotCols / 8), nr * dh / 8);
  const dim3 grid((per + 255) / 256, U + 1);
  return launch_pdl(k_relpos_prep, grid, dim3(256), 0, st, rel_h, rel_w, rpack, dh, nr, perm,
                    onehot, U, N, npad, Hu, Wu, b, N / kStripes, status);
}

}  // namespace ss
