// Host-side launchers of the library's kernels (internal to the library).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "pattern.h"
#include "sparsesam.h"

namespace ss {

constexpr int kMaxRankTokens = 16384;   // tokens per unit the rank kernel holds in shared memory

// The bounded-wait limit of each source file's kernels (see c_wait_limit_ns), current device.
cudaError_t set_wait_limit_attn(uint64_t ns);
cudaError_t set_wait_limit_mlp(uint64_t ns);

// sparsesam_rcmlp's argument checks (same codes, same order) and its workspace bytes in *need.
int rcmlp_validate(const ss_cfg* cfg, const uint16_t* x, int32_t C, int32_t hidden,
                   const uint16_t* w1, const uint16_t* b1, const uint16_t* w2, const uint16_t* b2,
                   const int32_t* keep, int32_t K, size_t* need);

cudaError_t launch_sobel_score(const float* lum, double* score, int B, int H, int W,
                               cudaStream_t st);

// Ranks the unit's tokens by score. With lum non-null the scores are computed from lum (S1 fused
// in) instead of read from `score`, and written to score_out (when non-null).
cudaError_t launch_stripe_rank(const double* score, const float* lum, double* score_out,
                               int window_mode, int B, int Hg, int Wg, int ws, int units, int N,
                               int K, int32_t* perm, int32_t* inv, int32_t* keep,
                               cudaStream_t st);

// score[i] = SplitMix64 output i from `seed`, as a uniform double in [0, 1), i < n.
cudaError_t launch_random_score(double* score, long long n, unsigned long long seed,
                                cudaStream_t st);
// mag[r] = sum over c in order of delta[r, c]^2 in fp64, for rows r < rows of C bf16 (C % 8 == 0).
cudaError_t launch_update_magnitude(const uint16_t* delta, double* mag, long long rows, int C,
                                    cudaStream_t st);

// Gathers q, k, v [U, N, heads, dh] into the block-major permuted layout [U*heads, N, dh].
cudaError_t launch_gather_qkv(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                              const int32_t* perm, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                              int U, int N, int heads, int dh, int b, int* status,
                              cudaStream_t st);

struct AttnParams {
  const int32_t* perm;   // [U, N]
  uint16_t* out;         // [U, N, heads, dh]
  int U, N, heads, L, b, nb, W, g;
  float scale_log2;      // log2(e) / sqrt(dh)
  int sms;               // persistent CTAs to launch (one per SM)
  int whole;             // pair kernel: pairs processed whole (the rest are split)
  int tail_split;        // pair kernel: pieces per split pair
  float* partial;        // per split piece and group, fp32 O [dh][128], m [128], l [128]
  uint16_t* operm;       // pair kernel output: [U*heads, N, dh] in block-major permuted order
  float2* ml;            // null, or [U*heads, N] (block-major): each row's running max m and
                         // sum l of 2^(s*scale_log2 - m) over its kept keys, s = q.k
  // Decomposed relative-position bias (null rel_tab: none; head dim 64). rel_tab [U*heads*N,
  // rel_ld] fp16 in block-major row order: the row's q . Rh[r] * sqrt(dh) at column r <
  // 2*rel_h - 1, then q . Rw[r] * sqrt(dh) from column 2*rel_h - 1 (rel_h x rel_w: the unit
  // grid); the key tiles' one-hot matrices come by the launch's `te` map over [U, npad, 128] fp16;
  // rel_ksteps = the bias MMA's K steps of 16 columns, ceil((rel_h + rel_w) / 16).
  const uint16_t* rel_tab;
  int rel_ld, rel_h, rel_w, rel_ksteps;
};
// Which attention kernel a shape takes, and the scratch beyond the gathered Q, K, V it needs
// (planned for `sms` CTAs).
struct AttnPlan {
  bool pair_kernel;      // the pair kernel (else the short-item kernel)
  int pairs, whole, tail_split;
  size_t partial_bytes;
};
AttnPlan attn_plan(const AttnParams& p, int dh, int sms, bool force_pair = false);
constexpr int kRelPosOneHotCols = 128;   // columns of a one-hot row (Hu + Wu <= 128)
// The relative-position variant's inputs: the tables stacked into rpack [nr, dh] (the bias GEMM's
// B operand) and every key position's one-hot row of E [U, npad, 128] fp16 (1.0 at columns
// Hu-1-kh and Hu+Wu-1-kw; zero rows past N).
cudaError_t launch_relpos_prep(const uint16_t* rel_h, const uint16_t* rel_w, uint16_t* rpack,
                               int dh, int nr, const int32_t* perm, uint16_t* onehot, int U, int N,
                               int npad, int Hu, int Wu, int b, int* status, cudaStream_t st);
// Block-sparse attention over the gathered sequences (tensor maps over [U*heads, N, dh]; the
// tails cover columns 64..79 at head dim 80). The pair kernel writes its output, permuted, through
// `to` / `to_tail` (maps over p.operm laid out like Q), except the rows of split pairs, which
// launch_merge_pieces writes from the pieces' partials; launch_unpermute_out then scatters Op to
// p.out. The short-item kernel writes p.out itself.
cudaError_t launch_attn(const CUtensorMap* tq, const CUtensorMap* tk, const CUtensorMap* tv,
                        const CUtensorMap* tq_tail, const CUtensorMap* tk_tail,
                        const CUtensorMap* to, const CUtensorMap* to_tail, const AttnParams& p,
                        int dh, int* status, cudaStream_t st, const CUtensorMap* te = nullptr);
// Rows of Op for the split pairs: the pieces' (O, m, l) in p.partial combined and normalised
// (nothing when the plan splits no pair).
cudaError_t launch_merge_pieces(const AttnParams& p, int dh, cudaStream_t st);
// out[u, perm[u][p(q)], h, :] = op[u*heads + h, q, :] for every block-major position q.
cudaError_t launch_unpermute_out(const uint16_t* op, const int32_t* perm, uint16_t* out, int U,
                                 int N, int heads, int dh, int b, int* status, cudaStream_t st);

// The partial-token-count variant (prefix tokens before the patch tokens, 2-D RoPE on the patch
// tokens' q and k). q, k, v, out: [U, prefix + N, heads, dh].
constexpr int kMaxPrefix = 4;            // prefix (class) tokens per unit
constexpr int kMaxPrefixHeads = 32;
constexpr size_t kMaxPrefixRowsSmem = 64 * 1024;   // scores of one dense prefix row: prefix + N <= 16384
// Patch tokens (rows prefix + perm[u][p]) into the gathered layout, q and k rotated
// (rope_log2_base = log2 of the RoPE base; 0: none).
cudaError_t launch_gather_rope(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const int32_t* perm, uint16_t* qp, uint16_t* kp, uint16_t* vp,
                               int U, int N, int heads, int dh, int b, int prefix, int grid_w,
                               float rope_log2_base, int* status, cudaStream_t st);
// Patch rows: po [U, N, heads, dh] (attention over the kept patch keys, token order) with its
// (m, l) in ml (block-major) merged with the prefix keys, written to out rows prefix + tok.
cudaError_t launch_prefix_merge(const uint16_t* po, const float2* ml, const uint16_t* qp,
                                const uint16_t* k, const uint16_t* v, const int32_t* perm,
                                uint16_t* out, int U, int N, int heads, int dh, int b, int prefix,
                                float scale_log2, int* status, cudaStream_t st);
// Prefix rows: dense attention of each prefix query over all prefix + N keys.
cudaError_t launch_prefix_rows(const uint16_t* q, const uint16_t* k, const uint16_t* v,
                               const uint16_t* kp, const uint16_t* vp, uint16_t* out, int U, int N,
                               int heads, int dh, int prefix, float scale_log2, cudaStream_t st);

// Gathers the kept rows of x [B, T, C] into xk [B*K, C]; zeroes zero[0, nzero). late_wait: keep
// and x are known final at launch (see k_gather_rows), the copy need not wait for the previous
// launch.
cudaError_t launch_gather_rows(const uint16_t* x, const int32_t* keep, uint16_t* xk, int B, int T,
                               int K, int C, int* zero, int nzero, int* status, cudaStream_t st,
                               bool late_wait = false);

// Rows of an encoder block's attention units: row m = u*N + i is token i (enumeration order) of
// unit u. Global blocks: unit u is image u, in raster order. Windowed blocks: the grid is padded
// bottom/right to whole windows of `window` x `window`, unit u = b*windows + w is window w (row-major
// over the padded grid) of image b, its tokens row-major; a token in the padding has no image row.
struct UnitRows {
  int N, T;               // tokens per unit, tokens per image
  int grid_w, grid_h;
  int window;             // 0: global
  int win_per_row, windows;
};
// The image row b*T + t of unit row m, or -1 for a pad token.
__host__ __device__ inline long long unit_row_src(const UnitRows& r, long long m) {
  const long long u = m / r.N;
  const int i = (int)(m - u * r.N);
  if (!r.window) return u * r.T + i;
  const long long b = u / r.windows;
  const int w = (int)(u - b * r.windows);
  const int y = (w / r.win_per_row) * r.window + i / r.window;
  const int x = (w % r.win_per_row) * r.window + i % r.window;
  if (y >= r.grid_h || x >= r.grid_w) return -1;
  return b * r.T + (long long)y * r.grid_w + x;
}

// LayerNorm of rows, bf16 in and out, fp32 statistics: out[m] = (x[src] - mean) / sqrt(var + eps)
// * w + b over the C channels of the source row, or zeros where there is none. keep == null: the
// source of row m < rows is unit_row_src(ur, m) (a block's LN1 over its units, pads zero); else
// it is image m / K's token keep[m] (LN2 over the kept rows; an entry outside the image records
// SS_EINDEX and its row is left unwritten). CTA 0 also zeroes zero[0, nzero).
cudaError_t launch_ln_rows(const uint16_t* x, const uint16_t* w, const uint16_t* b, uint16_t* out,
                           long long rows, int C, const UnitRows& ur, const int32_t* keep, int K,
                           int* zero, int nzero, int* status, cudaStream_t st);

struct GemmEpilogue {
  int kind;                 // 0: out = bf16(GELU(acc + bias)) into out[M, N]
                            // 1: x[b, keep[m], n] = bf16(x + acc + bias)
                            // 2: the q|k|v columns of unit row m into the block-major permuted
                            //    layout: out[which][(u*heads + h)*N + q(inv[m]), d] =
                            //    bf16(acc + bias), q(p) the block-major position of permuted
                            //    position p (pattern block size b, stripe length L)
                            // 3: x[unit_row_src(ur, m), n] = bf16(x + acc + bias), pad rows skipped
                            // 4: out[M, N] = fp16(acc * scale) (the relative-position products)
  const uint16_t* bias;     // [N] or null
  uint16_t* out;            // kind 0; kind 2: gathered Q (K and V follow at which_stride)
  uint16_t* x;              // kind 1: [B, T, N]; kind 3: [B*T, N]
  const int32_t* keep;      // kind 1: [B*K]
  int K_per_image, T;       // kind 1
  const int32_t* inv;       // kind 2: [U*N] permuted position of each unit row
  long long which_stride;   // kind 2: elements from the gathered Q to K (and K to V)
  int heads, dh, C;         // kind 2: C = heads*dh columns per q, k, v
  int b, L;                 // kind 2: the pattern's block size and stripe length
  float scale;              // kind 4
  UnitRows ur;              // kinds 2 (N) and 3
};
// Tile width and k-split of C[M, N] = A[M, Kd] * B[N, Kd]^T for `sms` persistent CTAs.
// tail: without a k-split, the tiles of a last, partial round of units that are each split in two
// along K (two CTAs, finished as a pair), so that round takes half a unit (0: none).
struct GemmPlan {
  int bn, splits, m_tiles, n_tiles, units, tail;
};
GemmPlan gemm_plan(int M, int N, int Kd, int sms);
// Tiles of the tail for `tiles` whole tiles of kb k-blocks over `sms` CTAs (0: no tail).
int gemm_tail(int tiles, int kb, int sms);
// fp32 partial-tile bytes the plan needs (0 without a k-split); plus one int counter per tile.
size_t gemm_partial_bytes(const GemmPlan& p);
// C = A B^T on tcgen05 with the given epilogue. partial / counters: workspace for k-splits
// (counters zero on entry). B must not be written by the launch directly before this one: its
// first tiles are requested before the kernel's dependency wait (weights are the caller's).
cudaError_t launch_gemm(const CUtensorMap* ta, const CUtensorMap* tb, const GemmPlan& p, int M,
                        int N, int Kd, const GemmEpilogue& ep, float* partial, int* counters,
                        int sms, int* status, cudaStream_t st);

}  // namespace ss
