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
// accumulator; four epilogue warps read it back with tcgen05.ld (one row per thread).
#include "common.cuh"
#include "kernels.h"

namespace ss {

__global__ void __launch_bounds__(256) k_gather_rows(const uint16_t* __restrict__ x,
                                                     const int32_t* __restrict__ keep,
                                                     uint16_t* __restrict__ xk, int B, int T,
                                                     int K, int C) {
  const int cpr = C / 8;
  const int total = B * K * cpr;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < total; i += gridDim.x * blockDim.x) {
    const int m = i / cpr, c = i - (i / cpr) * cpr;
    const int b = m / K;
    const int t = min(max(__ldg(keep + m), 0), T - 1);   // never leave the image
    reinterpret_cast<uint4*>(xk)[(size_t)m * cpr + c] =
        __ldg(reinterpret_cast<const uint4*>(x + ((size_t)b * T + t) * C) + c);
  }
}

cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* keep, uint16_t* xk, int B, int T,
                               int K, int C, cudaStream_t st) {
  const int total = B * K * (C / 8);
  int blocks = (total + 255) / 256;
  if (blocks > 148 * 16) blocks = 148 * 16;
  k_gather_rows<<<blocks, 256, 0, st>>>(x, keep, xk, B, T, K, C);
  return cudaGetLastError();
}

constexpr int kGemmThreads = 192;

template <int BN>
struct GemmCfg {
  static constexpr int kStages = BN == 256 ? 3 : 4;
  static constexpr int kABytes = 128 * 128;       // 128 rows x 64 bf16
  static constexpr int kBBytes = BN * 128;        // BN rows x 64 bf16
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kBar = kStages * kStageBytes;
  static constexpr int kAlloc = kBar + 256 + 1024;
  static constexpr int kTmemCols = BN < 32 ? 32 : BN;
};

__device__ __forceinline__ float bf16_to_f(uint16_t v) { return __uint_as_float(uint32_t(v) << 16); }

__device__ __forceinline__ float gelu_erf(float z) {
  return 0.5f * z * (1.0f + erff(z * 0.70710678118654752f));
}

template <int BN>
__global__ void __launch_bounds__(kGemmThreads, 1)
    k_gemm(const __grid_constant__ CUtensorMap ta, const __grid_constant__ CUtensorMap tb, int M,
           int N, int Kd, const GemmEpilogue ep, int* status) {
  using G = GemmCfg<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + G::kBar);
  uint64_t* empty = full + G::kStages;
  uint64_t* acc_full = empty + G::kStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_full + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * 128, n0 = blockIdx.y * BN;
  const int kblocks = Kd / 64;

  if (threadIdx.x == 0) {
    for (int i = 0; i < G::kStages; ++i) {
      mbar_init(full + i, 1);
      mbar_init(empty + i, 1);
    }
    mbar_init(acc_full, 1);
    *abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_slot, G::kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      tma_prefetch_desc(&ta);
      tma_prefetch_desc(&tb);
      for (int kb = 0; kb < kblocks; ++kb) {
        const int st = kb % G::kStages;
        if (kb >= G::kStages &&
            !mbar_wait(empty + st, ((kb / G::kStages) - 1) & 1, abort, status))
          break;
        uint8_t* sa = smem + st * G::kStageBytes;
        mbar_expect_tx(full + st, G::kStageBytes);
        tma_load_2d(sa, &ta, full + st, kb * 64, m0);
        tma_load_2d(sa + G::kABytes, &tb, full + st, kb * 64, n0);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(128, BN, false, false);
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb) {
        const int st = kb % G::kStages;
        if (!(ok = mbar_wait(full + st, (kb / G::kStages) & 1, abort, status))) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(smem + st * G::kStageBytes);
        const uint32_t b_addr = a_addr + G::kABytes;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16_ss(tmem, smem_desc(a_addr + kk * 32, 16, 1024, kSwizzle128B),
                       smem_desc(b_addr + kk * 32, 16, 1024, kSwizzle128B), idesc,
                       (kb | kk) != 0);
        umma_commit(empty + st);
      }
      if (ok) umma_commit(acc_full);
    }
  } else {
    const int row = 32 * (warp & 3) + lane;
    const uint32_t lane_off = uint32_t(32 * (warp & 3)) << 16;
    const int m = m0 + row;
    const bool ok = mbar_wait(acc_full, 0, abort, status);
    tc_fence_after();
    if (ok) {
      uint16_t* dst_row = nullptr;
      if (ep.kind == 0) {
        dst_row = ep.out + (size_t)m * N;
      } else if (m < M) {
        const int b = m / ep.K_per_image;
        const int t = min(max(__ldg(ep.keep + m), 0), ep.T - 1);
        dst_row = ep.x + ((size_t)b * ep.T + t) * N;
      }
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        tmem_ld32(tmem + lane_off + c * 32, r);
                if (m >= M) continue;
        const int n = n0 + c * 32;
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          v[i] = __uint_as_float(r[i]);
          if (ep.bias) v[i] += bf16_to_f(__ldg(ep.bias + n + i));
        }
        uint4* d = reinterpret_cast<uint4*>(dst_row + n);
        if (ep.kind == 0) {
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = gelu_erf(v[i]);
        } else {
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 xv = d[q];
            const uint32_t w[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              v[q * 8 + 2 * e] += __uint_as_float(w[e] << 16);
              v[q * 8 + 2 * e + 1] += __uint_as_float(w[e] & 0xFFFF0000u);
            }
          }
        }
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
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, G::kTmemCols);
  }
}

template <int BN>
static cudaError_t launch_gemm_bn(const CUtensorMap* ta, const CUtensorMap* tb, int M, int N,
                                  int Kd, const GemmEpilogue& ep, int* status, cudaStream_t st) {
  using G = GemmCfg<BN>;
  cudaError_t e =
      cudaFuncSetAttribute(k_gemm<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, G::kAlloc);
  if (e != cudaSuccess) return e;
  dim3 grid((M + 127) / 128, N / BN);
  k_gemm<BN><<<grid, kGemmThreads, G::kAlloc, st>>>(*ta, *tb, M, N, Kd, ep, status);
  return cudaGetLastError();
}

cudaError_t launch_gemm(const CUtensorMap* ta, const CUtensorMap* tb, int M, int N, int Kd, int BN,
                        const GemmEpilogue& ep, int* status, cudaStream_t st) {
  switch (BN) {
    case 64: return launch_gemm_bn<64>(ta, tb, M, N, Kd, ep, status, st);
    case 128: return launch_gemm_bn<128>(ta, tb, M, N, Kd, ep, status, st);
    case 256: return launch_gemm_bn<256>(ta, tb, M, N, Kd, ep, status, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace ss
