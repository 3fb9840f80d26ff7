// The partial-token-count variant for Perception-Encoder-style encoders (SparseSAM README,
// "Zero-shot CLIP on ImageNet-1k": apply_pe(model.visual, "sparsesam_partial", ratio, group_size=4,
// start_block, mlp_merge); "kernels/": FA2 with RoPE fused). Such an encoder's sequence is `prefix`
// extra tokens (the class token) followed by the Hg x Wg patch tokens, and its attention rotates q
// and k of the patch tokens by a 2-D RoPE. Here:
//   - the Stripe-Sort pattern covers the patch tokens (their count is a multiple of the stripe
//     count), which also attend every prefix key;
//   - each prefix query attends every key (dense);
//   - the RoPE rotation is fused into the patch tokens' gather into the permuted layout.
// The patch rows' attention over their kept patch keys runs in the regular attention kernels,
// which also leave each row's softmax statistics (m, l); k_prefix_merge then folds the prefix keys
// into those rows exactly (one more online-softmax step) while scattering them to the output, and
// k_prefix_rows computes the dense prefix rows.
#include "common.cuh"
#include "kernels.h"

namespace ss {

// 2-D RoPE of one bf16 pair (lo = channel d, hi = channel d + 1) by angle phi, in fp32.
__device__ __forceinline__ uint32_t rope_pair(uint32_t w, float cs, float sn) {
  const float a = __uint_as_float(w << 16), b = __uint_as_float(w & 0xFFFF0000u);
  return pack_bf16(a * cs - b * sn, a * sn + b * cs);
}

// Gather of the patch tokens (source rows prefix + tok of each unit) into the block-major
// permuted layout, q and k rotated: channel pair (d, d+1) of a head, d even, takes the angle
// pos * base^(-i / (dh/4)) with i = (d mod dh/2) / 2 and pos = the token's row for d < dh/2, its
// column otherwise (rope_log2_base = log2(base); 0: no rotation). Layout as k_gather_qkv.
template <int CPR, int KPL>
__global__ void __launch_bounds__(256) k_gather_rope(const uint16_t* __restrict__ q,
                                                     const uint16_t* __restrict__ k,
                                                     const uint16_t* __restrict__ v,
                                                     const int32_t* __restrict__ perm,
                                                     uint16_t* __restrict__ qp,
                                                     uint16_t* __restrict__ kp,
                                                     uint16_t* __restrict__ vp, int N, int heads,
                                                     int b, int L, int prefix, int grid_w,
                                                     float rope_log2_base, int* status) {
  griddep_wait();
  griddep_launch();
  constexpr int DH = CPR * 8, HALF = DH / 2, QUART = DH / 4;
  __shared__ float2 s_rot[8][DH / 2];   // per warp: (cos, sin) of the token's dh/2 channel pairs
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qpos = blockIdx.x * 8 + warp;
  if (qpos >= N) return;
  const int p = blockmajor_to_canonical(qpos, b, L);
  const int tok = __ldg(perm + (size_t)u * N + p);
  if ((unsigned)tok >= (unsigned)N) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  const int per_tok = heads * CPR;
  const size_t plane = (size_t)N * CPR;
  const size_t src_row = ((size_t)u * (N + prefix) + prefix + tok) * per_tok;
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
  const int y = tok / grid_w, x = tok - y * grid_w;
  if (rope_log2_base != 0.f) {
    // The token's dh/2 angles (the same for every head), one or two per lane, shared by the warp.
    for (int pr = lane; pr < DH / 2; pr += 32) {
      const int d = 2 * pr;
      const bool col = d >= HALF;
      const int i = (d - (col ? HALF : 0)) >> 1;
      const float theta = exp2f(-(float)i * rope_log2_base / (float)QUART);
      float sn, cs;
      sincosf((float)(col ? x : y) * theta, &sn, &cs);
      s_rot[warp][pr] = make_float2(cs, sn);
    }
    __syncwarp();
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int c = e * 32 + lane;
      if (c >= per_tok) continue;
      const int cc = c % CPR;
      uint32_t* wq = reinterpret_cast<uint32_t*>(&buf[0][e]);
      uint32_t* wk = reinterpret_cast<uint32_t*>(&buf[1][e]);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float2 r = s_rot[warp][cc * 4 + j];
        wq[j] = rope_pair(wq[j], r.x, r.y);
        wk[j] = rope_pair(wk[j], r.x, r.y);
      }
    }
  }
#pragma unroll
  for (int t = 0; t < 3; ++t)
#pragma unroll
    for (int e = 0; e < KPL; ++e) {
      const int c = e * 32 + lane;
      if (c < per_tok) {
        const int h = c / CPR, cc = c - h * CPR;
        dst[t][h * plane + cc] = buf[t][e];
      }
    }
}

cudaError_t launch_gather_rope(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const int32_t* perm, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                               int U, int N, int heads, int dh, int b, int prefix, int grid_w,
                               float rope_log2_base, int* status, cudaStream_t st) {
  const dim3 grid((N + 7) / 8, U);
  const int L = N / kStripes;
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, grid, dim3(256), 0, st, q, k, v, perm, qp, kp, vp, N, heads, b, L,
                      prefix, grid_w, rope_log2_base, status);
  };
  const int per_tok = heads * (dh / 8);
  if (per_tok > 32 * 8) return cudaErrorInvalidValue;
  if (dh == 64) return per_tok <= 128 ? go(k_gather_rope<8, 4>) : go(k_gather_rope<8, 8>);
  if (dh == 80) return per_tok <= 160 ? go(k_gather_rope<10, 5>) : go(k_gather_rope<10, 8>);
  return cudaErrorInvalidValue;
}

// One warp per block-major patch position of a unit: for each head, the row's attention over its
// kept patch keys (po, normalised, with its (m, l)) and the prefix keys j < prefix (unrotated
// k[u, j]) are combined in one more online-softmax step, with s_j = q_rot . k_j:
//   M = max(m, s_j * scale_log2), a = l * 2^(m - M), c_j = 2^(s_j * scale_log2 - M),
//   out[u, prefix + tok] = (po * a + sum_j c_j v_j) / (a + sum_j c_j).
// The dot products are summed per head by shuffles at head dim 64 (a head's 8 chunks sit in 8
// adjacent lanes of one slot), through shared memory at head dim 80 (a head's 10 chunks may span
// two of a lane's slots).
template <int CPR, int KPL>
__global__ void __launch_bounds__(256) k_prefix_merge(const uint16_t* __restrict__ po,
                                                      const float2* __restrict__ ml,
                                                      const uint16_t* __restrict__ qp,
                                                      const uint16_t* __restrict__ k,
                                                      const uint16_t* __restrict__ v,
                                                      const int32_t* __restrict__ perm,
                                                      uint16_t* __restrict__ out, int N, int heads,
                                                      int b, int L, int prefix, float scale_log2,
                                                      int* status) {
  griddep_wait();
  griddep_launch();
  __shared__ float s_dot[8][kMaxPrefixHeads][kMaxPrefix];
  const int u = blockIdx.y;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int qpos = blockIdx.x * 8 + warp;
  for (int i = lane; i < kMaxPrefixHeads * kMaxPrefix; i += 32) (&s_dot[warp][0][0])[i] = 0.f;
  __syncwarp();
  if (qpos >= N) return;
  const int p = blockmajor_to_canonical(qpos, b, L);
  const int tok = __ldg(perm + (size_t)u * N + p);
  if ((unsigned)tok >= (unsigned)N) {
    if (lane == 0) record_bad_index(status);
    return;
  }
  const int per_tok = heads * CPR;
  const size_t plane = (size_t)N * CPR;
  const uint4* qrow = reinterpret_cast<const uint4*>(qp) + (size_t)u * heads * plane +
                      (size_t)qpos * CPR;
  const uint4* orow = reinterpret_cast<const uint4*>(po) + ((size_t)u * N + tok) * per_tok;
  const uint4* kbase = reinterpret_cast<const uint4*>(k) + (size_t)u * (N + prefix) * per_tok;
  const uint4* vbase = reinterpret_cast<const uint4*>(v) + (size_t)u * (N + prefix) * per_tok;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    // Every lane takes part in every iteration (the shuffles below need the whole warp); lanes
    // past the row's chunks contribute zeros and write nothing.
    const int c = e * 32 + lane;
    const bool active = c < per_tok;
    const int h = active ? c / CPR : 0, cc = active ? c - h * CPR : 0;
    uint32_t qw[4] = {0u, 0u, 0u, 0u};
    if (active) {
      const uint4 qv = __ldg(qrow + h * plane + cc);
      qw[0] = qv.x;
      qw[1] = qv.y;
      qw[2] = qv.z;
      qw[3] = qv.w;
    }
    for (int j = 0; j < prefix; ++j) {
      float d = 0.f;
      if (active) {
        const uint4 kv = __ldg(kbase + (size_t)j * per_tok + c);
        const uint32_t kw[4] = {kv.x, kv.y, kv.z, kv.w};
#pragma unroll
        for (int t = 0; t < 4; ++t)
          d += __uint_as_float(qw[t] << 16) * __uint_as_float(kw[t] << 16) +
               __uint_as_float(qw[t] & 0xFFFF0000u) * __uint_as_float(kw[t] & 0xFFFF0000u);
      }
      if constexpr (CPR == 8) {
        // a head's 8 chunks sit in 8 adjacent lanes of this slot: reduce among them
        d += __shfl_xor_sync(0xffffffffu, d, 1);
        d += __shfl_xor_sync(0xffffffffu, d, 2);
        d += __shfl_xor_sync(0xffffffffu, d, 4);
        if (active && (lane & 7) == 0) s_dot[warp][h][j] = d;
      } else {
        if (active) atomicAdd(&s_dot[warp][h][j], d);
      }
    }
  }
  __syncwarp();
  uint4* orow_out = reinterpret_cast<uint4*>(out) + ((size_t)u * (N + prefix) + prefix + tok) * per_tok;
#pragma unroll
  for (int e = 0; e < KPL; ++e) {
    const int c = e * 32 + lane;
    if (c >= per_tok) continue;
    const int h = c / CPR;
    const float2 st = __ldg(ml + ((size_t)u * heads + h) * N + qpos);
    float M = st.x, cj[kMaxPrefix];
    for (int j = 0; j < prefix; ++j) M = fmaxf(M, s_dot[warp][h][j] * scale_log2);
    const float a = st.x == -INFINITY ? 0.f : st.y * exp2f(st.x - M);
    float den = a;
    for (int j = 0; j < prefix; ++j) {
      cj[j] = exp2f(s_dot[warp][h][j] * scale_log2 - M);
      den += cj[j];
    }
    const uint4 ov = __ldg(orow + c);
    const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w};
    float acc[8];
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      acc[2 * t] = __uint_as_float(ow[t] << 16) * a;
      acc[2 * t + 1] = __uint_as_float(ow[t] & 0xFFFF0000u) * a;
    }
    for (int j = 0; j < prefix; ++j) {
      const uint4 vv = __ldg(vbase + (size_t)j * per_tok + c);
      const uint32_t vw[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        acc[2 * t] += __uint_as_float(vw[t] << 16) * cj[j];
        acc[2 * t + 1] += __uint_as_float(vw[t] & 0xFFFF0000u) * cj[j];
      }
    }
    const float inv = den > 0.f ? 1.f / den : 0.f;
    orow_out[c] = make_uint4(pack_bf16(acc[0] * inv, acc[1] * inv), pack_bf16(acc[2] * inv, acc[3] * inv),
                             pack_bf16(acc[4] * inv, acc[5] * inv), pack_bf16(acc[6] * inv, acc[7] * inv));
  }
}

cudaError_t launch_prefix_merge(const uint16_t* po, const float2* ml, const uint16_t* qp,
                                const uint16_t* k, const uint16_t* v, const int32_t* perm,
                                uint16_t* out, int U, int N, int heads, int dh, int b, int prefix,
                                float scale_log2, int* status, cudaStream_t st) {
  const dim3 grid((N + 7) / 8, U);
  const int L = N / kStripes;
  auto go = [&](auto kernel) {
    return launch_pdl(kernel, grid, dim3(256), 0, st, po, ml, qp, k, v, perm, out, N, heads, b, L,
                      prefix, scale_log2, status);
  };
  const int per_tok = heads * (dh / 8);
  if (per_tok > 32 * 8 || heads > kMaxPrefixHeads || prefix > kMaxPrefix)
    return cudaErrorInvalidValue;
  if (dh == 64) return per_tok <= 128 ? go(k_prefix_merge<8, 4>) : go(k_prefix_merge<8, 8>);
  if (dh == 80) return per_tok <= 160 ? go(k_prefix_merge<10, 5>) : go(k_prefix_merge<10, 8>);
  return cudaErrorInvalidValue;
}

// One CTA per (unit, head, prefix token j): the prefix query (unrotated) against every key of the
// unit -- the prefix keys (unrotated) and the N rotated patch keys of the gathered layout (their
// order does not matter to a dense softmax) -- with its scores held in shared memory.
template <int DH>
__global__ void __launch_bounds__(256) k_prefix_rows(const uint16_t* __restrict__ q,
                                                     const uint16_t* __restrict__ k,
                                                     const uint16_t* __restrict__ v,
                                                     const uint16_t* __restrict__ kp,
                                                     const uint16_t* __restrict__ vp,
                                                     uint16_t* __restrict__ out, int N, int heads,
                                                     int prefix, float scale_log2) {
  griddep_wait();
  griddep_launch();
  extern __shared__ float s_score[];                  // [prefix + N]
  __shared__ float s_q[DH];
  __shared__ float s_red[8];
  __shared__ float2 s_acc[8][DH / 2];
  const int j = blockIdx.x % prefix, uh = blockIdx.x / prefix;
  const int u = uh / heads, h = uh - u * heads;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int n_keys = prefix + N;
  const size_t tok_stride = (size_t)heads * DH;       // elements per token row of q, k, v, out
  const uint16_t* src0 = q + ((size_t)u * n_keys + j) * tok_stride + (size_t)h * DH;
  for (int d = tid; d < DH; d += 256) s_q[d] = __uint_as_float(uint32_t(src0[d]) << 16);
  __syncthreads();
  auto key_row = [&](const uint16_t* base_pre, const uint16_t* base_patch, int t) {
    return t < prefix ? base_pre + ((size_t)u * n_keys + t) * tok_stride + (size_t)h * DH
                      : base_patch + ((size_t)uh * N + (t - prefix)) * DH;
  };
  float mx = -INFINITY;
  for (int t = tid; t < n_keys; t += 256) {
    const uint4* kr = reinterpret_cast<const uint4*>(key_row(k, kp, t));
    float d = 0.f;
#pragma unroll
    for (int c = 0; c < DH / 8; ++c) {
      const uint4 w4 = __ldg(kr + c);
      const uint32_t w[4] = {w4.x, w4.y, w4.z, w4.w};
#pragma unroll
      for (int e = 0; e < 4; ++e)
        d += s_q[8 * c + 2 * e] * __uint_as_float(w[e] << 16) +
             s_q[8 * c + 2 * e + 1] * __uint_as_float(w[e] & 0xFFFF0000u);
    }
    s_score[t] = d * scale_log2;
    mx = fmaxf(mx, d * scale_log2);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane == 0) s_red[warp] = mx;
  __syncthreads();
  float M = s_red[0];
  for (int w = 1; w < 8; ++w) M = fmaxf(M, s_red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int t = tid; t < n_keys; t += 256) {
    const float e = exp2f(s_score[t] - M);
    s_score[t] = e;
    sum += e;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane == 0) s_red[warp] = sum;
  __syncthreads();
  float Ls = 0.f;
  for (int w = 0; w < 8; ++w) Ls += s_red[w];
  // Output: warp w sums p_t v_t over the keys t = w, w + 8, ...; lane l holds the channel pairs
  // l and l + 32 (one coalesced 4-byte load per pair and key); the 8 warps' sums then meet.
  constexpr int DP = DH / 2;
  float2 acc[2] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f)};
  for (int t = warp; t < n_keys; t += 8) {
    const float pt = s_score[t];
    const uint32_t* vr = reinterpret_cast<const uint32_t*>(key_row(v, vp, t));
#pragma unroll
    for (int r2 = 0; r2 < 2; ++r2) {
      const int pr = lane + 32 * r2;
      if (pr < DP) {
        const uint32_t w = __ldg(vr + pr);
        acc[r2].x += pt * __uint_as_float(w << 16);
        acc[r2].y += pt * __uint_as_float(w & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int r2 = 0; r2 < 2; ++r2)
    if (lane + 32 * r2 < DP) s_acc[warp][lane + 32 * r2] = acc[r2];
  __syncthreads();
  if (tid < DP) {
    float2 a = make_float2(0.f, 0.f);
    for (int w = 0; w < 8; ++w) {
      a.x += s_acc[w][tid].x;
      a.y += s_acc[w][tid].y;
    }
    const float inv = Ls > 0.f ? 1.f / Ls : 0.f;
    reinterpret_cast<uint32_t*>(out + ((size_t)u * n_keys + j) * tok_stride + (size_t)h * DH)[tid] =
        pack_bf16(a.x * inv, a.y * inv);
  }
}

cudaError_t launch_prefix_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const uint16_t* kp, const uint16_t* vp, uint16_t* out, int U, int N,
                               int heads, int dh, int prefix, float scale_log2, cudaStream_t st) {
  if (prefix <= 0) return cudaSuccess;
  const dim3 grid((unsigned)(U * heads * prefix));
  const size_t smem = (size_t)(prefix + N) * sizeof(float);
  if (smem > kMaxPrefixRowsSmem) return cudaErrorInvalidValue;
  auto go = [&](auto kernel) {
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kMaxPrefixRowsSmem);
    if (e != cudaSuccess) return e;
    return launch_pdl(kernel, grid, dim3(256), smem, st, q, k, v, kp, vp, out, N, heads, prefix,
                      scale_log2);
  };
  if (dh == 64) return go(k_prefix_rows<64>);
  if (dh == 80) return go(k_prefix_rows<80>);
  return cudaErrorInvalidValue;
}

}  // namespace ss
