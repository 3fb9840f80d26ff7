// Inputs of the relative-position variant of the attention (SAM's decomposed relative positions:
// the score of query (qh, qw) and key (kh, kw) gains q . Rh[qh - kh + Hu - 1] + q . Rw[qw - kw +
// Wu - 1]). The products q . R[r] for every table row r are one tcgen05 GEMM of the gathered Q
// against the two tables stacked (epilogue kind 4); this launch packs those tables into the GEMM's
// B operand and writes, for every key position of every unit, the byte offsets at which the
// attention's softmax threads find the key's two terms in their row's bias slices.
#include "common.cuh"
#include "kernels.h"

namespace ss {

// blockIdx.y < U: unit y's key offsets, one thread per block-major position q < npad (positions
// past N get offset 0; their keys are masked). blockIdx.y == U: the packed tables, one thread per
// 16-byte chunk of rpack [nr, dh]: rows 0..2Hu-2 = rel_h, then 2Wu-1 rows of rel_w, then zeros.
__global__ void __launch_bounds__(256) k_relpos_prep(const uint16_t* __restrict__ rel_h,
                                                     const uint16_t* __restrict__ rel_w,
                                                     uint16_t* __restrict__ rpack, int dh, int nr,
                                                     const int32_t* __restrict__ perm,
                                                     uint16_t* __restrict__ keyoff, int U, int N,
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
  const int u = blockIdx.y;
  if (t >= npad) return;
  uint16_t off = 0;
  if (t < N) {
    const int tok = __ldg(perm + (size_t)u * N + blockmajor_to_canonical(t, b, L));
    if ((unsigned)tok >= (unsigned)N) {
      record_bad_index(status);
    } else {
      const int kh = tok / Wu, kw = tok - kh * Wu;
      off = (uint16_t)(((Hu - 1 - kh) * 2) | (((Hu + Wu - 1 - kw) * 2) << 8));
    }
  }
  keyoff[(size_t)u * npad + t] = off;
}

cudaError_t launch_relpos_prep(const uint16_t* rel_h, const uint16_t* rel_w, uint16_t* rpack,
                               int dh, int nr, const int32_t* perm, uint16_t* keyoff, int U, int N,
                               int npad, int Hu, int Wu, int b, int* status, cudaStream_t st) {
  const int per = std::max(npad, nr * dh / 8);
  const dim3 grid((per + 255) / 256, U + 1);
  return launch_pdl(k_relpos_prep, grid, dim3(256), 0, st, rel_h, rel_w, rpack, dh, nr, perm,
                    keyoff, U, N, npad, Hu, Wu, b, N / kStripes, status);
}

}  // namespace ss
