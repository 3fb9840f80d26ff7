/*
 * sparsesam.h -- C ABI of the SparseSAM encoder-block hot path on B200 (sm_100a).
 *
 * SparseSAM ("SparseSAM: Structured Sparsification of Activations in Segment Anything Models")
 * accelerates SAM's ViT encoder with two training-free steps: Stripe-Sort attention and the
 * Residual-Consistency MLP. This library runs the four steps of one encoder block's hot path:
 *
 *   sparsesam_score  S1  Sobel gradient score per token
 *   sparsesam_perm   S2  stable sort by score + stripe transpose -> permutation; top-K keep list
 *   sparsesam_score_perm  S1 + S2 in one pass (the same results, one launch fewer)
 *   sparsesam_block       S1..S4 in one call with one workspace
 *   sparsesam_encoder_block  a full encoder block: LN1, qkv, S3, proj, residual, LN2 + S4
 *   sparsesam_encoder_stack  the encoder's blocks in order over one ranking of the tokens
 *   sparsesam_attn   S3  static block-sparse attention over the permuted sequence
 *   sparsesam_attn_relpos    S3 with SAM's decomposed relative-position bias fused
 *   sparsesam_attn_partial   S3 for prefix + patch sequences with 2-D RoPE (PE-style encoders)
 *   sparsesam_rcmlp  S4  fc1-GELU-fc2 on the kept tokens, added to the residual in place
 *   sparsesam_random_perm     S2 over random scores (the random-permutation ablation)
 *   sparsesam_keep_by_update  the keep-set by update magnitude (another keep criterion)
 *
 * Conventions shared by every call
 *   - Pointers marked (device) are device memory owned by the caller; nothing is allocated or
 *     freed by these calls. Pointers marked (host) are host memory.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream). Every GPU call is
 *     asynchronous on it and never synchronises; results are ready when the stream is.
 *   - Arguments are validated on the host before any launch. On a validation error nothing is
 *     launched and the call returns a negative SS_E* code; sparsesam_strerror() names it.
 *   - bf16 tensors are passed as uint16_t bit patterns (IEEE bfloat16).
 *   - A device-side wait that gives up (it never should) records SS_ETIMEOUT in a device status
 *     word, makes the kernel return early and leaves the context usable; sparsesam_device_status()
 *     reads and clears that word. Every perm / keep index a kernel reads is range-checked: one
 *     outside its unit (perm) or image (keep) records SS_EINDEX in the same word and the row it
 *     would have addressed is skipped (no access outside the caller's tensors).
 *
 * Layouts (shared by the calls; U = attention units, N = tokens per unit)
 *   global mode: U = batch, N = grid_h*grid_w (raster order).
 *   window mode: the grid is padded bottom/right to a multiple of `window` and split into
 *                windows in row-major window order; U = batch*windows, N = window^2, a window's
 *                tokens in window-local raster order (pads included).
 *   lum   fp32 [batch, grid_h, grid_w]
 *   score fp64 [batch, grid_h*grid_w]               (pads are not stored; they score +0.0)
 *   perm  int32 [U, N]  perm[u][p] = unit-local token at permuted position p
 *   inv   int32 [U, N]  inv[u][perm[u][p]] = p
 *   keep  int32 [batch, K]  image-raster token ids of the K top-ranked tokens, in rank order
 *   q,k,v,out bf16 [U, N, heads, head_dim]
 *   x     bf16 [batch, grid_h*grid_w, C]  (never padded)
 */
#ifndef SPARSESAM_H
#define SPARSESAM_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Return codes. */
#define SS_OK            0
#define SS_EINVAL       (-1)  /* a null pointer, a non-positive size, density outside (0,1]      */
#define SS_EUNSUPPORTED (-2)  /* a valid shape this build does not run (head_dim, N % 4, C % 64) */
#define SS_EWORKSPACE   (-3)  /* workspace pointer null/misaligned or smaller than required     */
#define SS_ECUDA        (-4)  /* a CUDA runtime/driver call failed (launch, tensor-map encode)   */
#define SS_ETIMEOUT     (-5)  /* a device-side wait gave up (read via sparsesam_device_status)   */
#define SS_EINDEX       (-6)  /* a perm or keep index outside its unit or image reached a kernel;
                                 the access was skipped (read via sparsesam_device_status)       */

#define SS_GLOBAL 0
#define SS_WINDOW 1

/* One encoder block's shape. The SparseSAM README's registry call apply_sam(encoder, "sparsesam",
 * ratio) takes the density as `ratio` ("ratio=0.5  # density 50%"); here it is `density`. */
typedef struct {
  int32_t batch;      /* images                                                   */
  int32_t grid_h;     /* token grid rows of one image (64 for SAM at 1024 px)      */
  int32_t grid_w;     /* token grid columns                                       */
  int32_t mode;       /* SS_GLOBAL or SS_WINDOW                                    */
  int32_t window;     /* window side in tokens (SAM: 14); ignored in global mode   */
  int32_t heads;      /* attention heads                                          */
  int32_t head_dim;   /* 64 or 80                                                  */
  double  density;    /* fraction of attention and of MLP tokens computed, (0, 1]  */
} ss_cfg;

/* The static pattern a config implies (Stripe-Sort attention; SparseSAM Dutch technical summary,
 * "Statisch Sparsiteitspatroon": a 4x4 mosaic of sub-maps, each with a banded diagonal, plus a small
 * global keep-set). Offset block a of stripe j holds permuted positions j*L + a*b ... + b-1. */
typedef struct {
  int32_t units;        /* U                                                      */
  int32_t unit_tokens;  /* N                                                      */
  int32_t stripes;      /* 4                                                      */
  int32_t L;            /* N / 4, the stripe length                               */
  int32_t b;            /* block size: largest divisor of L with b <= 64, L/b >= 4 */
  int32_t nb;           /* offset blocks per stripe, L / b                        */
  int32_t W;            /* band width in offset blocks                            */
  int32_t g;            /* global offset blocks (1)                               */
  int32_t nnz;          /* kept (query offset block, key offset block) pairs      */
  int32_t keep;         /* K = ceil(density * grid_h*grid_w - 1e-9), per image    */
  double  rho;          /* realised attention density nnz / nb^2                 */
} ss_pattern;

/* Host only. Fills *out for cfg. Band width W is the one in [1, nb] whose density is nearest to
 * cfg->density (ties: smaller W). Returns SS_OK or SS_EINVAL / SS_EUNSUPPORTED. */
int sparsesam_pattern(const ss_cfg* cfg, ss_pattern* out);

/* Host only. The kept key offset blocks of every query offset block as CSR: row_ptr[nb+1] and
 * col_idx[nnz] (host, caller-owned, cap = capacity of col_idx). Row a lists, ascending, the
 * offset blocks in [s, s+W) united with [0, g), s = clamp(a - (W-1)/2, 0, nb - W). All 16
 * sub-maps (query stripe i, key stripe j) share this list. Returns SS_OK, SS_EINVAL (null / cap
 * too small) or SS_EUNSUPPORTED. */
int sparsesam_blocklist(const ss_cfg* cfg, int32_t* row_ptr, int32_t* col_idx, int32_t cap);

/* S1 (SparseSAM Dutch technical summary, "Methodologie" 1, "Op Gradiënten Gebaseerde Ordening":
 * a parameter-free Sobel operator's gradient magnitude as the information-density proxy).
 * lum (device) fp32 [batch, grid_h, grid_w] -> score (device) fp64 [batch, grid_h*grid_w]:
 *   gx = ((l[y-1,x+1]-l[y-1,x-1]) + 2*(l[y,x+1]-l[y,x-1])) + (l[y+1,x+1]-l[y+1,x-1])
 *   gy = ((l[y+1,x-1]-l[y-1,x-1]) + 2*(l[y+1,x]-l[y-1,x])) + (l[y+1,x+1]-l[y-1,x+1])
 *   score = gx*gx + gy*gy
 * with clamp-to-edge borders, each step one fp64 round-to-nearest operation, no FMA. Bit-exact. */
int sparsesam_score(const ss_cfg* cfg, const float* lum, double* score, void* stream);

/* S2 (same summary, "Stripe-Sort Permutatie": sort the tokens by score, read the sorted list as a
 * matrix, transpose it and flatten it). Per unit: stable sort descending by score (equal scores:
 * lower enumeration index first) giving ranked tokens t_0..t_{N-1}; then perm[j*L + k] = t_{4k+j}.
 * score (device) -> perm, inv (device) int32 [U, N]; keep (device) int32 [batch, K]: the first K
 * tokens of each image's own ranking over its real tokens (window mode: per image, not per
 * window). Any of perm/inv/keep may be NULL to skip it (not all three). Scores may be any
 * non-NaN doubles (negative, zero of either sign, infinite): they rank by value, and -0.0 ties with
 * +0.0. A NaN score gives an unspecified (but in-bounds) permutation. */
int sparsesam_perm(const ss_cfg* cfg, const double* score, int32_t* perm, int32_t* inv,
                   int32_t* keep, void* stream);

/* S1 and S2 in one pass: the same results as sparsesam_score(cfg, lum, score) followed by
 * sparsesam_perm(cfg, score, perm, inv, keep), bit for bit, with one launch fewer (global mode:
 * one launch in all; window mode with keep: two). Each ranking CTA computes its unit's Sobel
 * scores itself and writes its own tokens' scores to score. lum, score (device) as for
 * sparsesam_score, both non-NULL; perm, inv, keep as for sparsesam_perm. */
int sparsesam_score_perm(const ss_cfg* cfg, const float* lum, double* score, int32_t* perm,
                         int32_t* inv, int32_t* keep, void* stream);

/* The random-permutation ablation (the SparseSAM README's registry variant `sparsesam_random`):
 * S2 over random scores instead of the Sobel ranking. score (device, non-NULL) fp64
 * [batch, grid_h*grid_w] receives score[b][t] = (X >> 11) * 2^-53, uniform in [0, 1), where X is
 * output b*grid_h*grid_w + t of the SplitMix64 generator started from state `seed` (Steele, Lea
 * and Flood, OOPSLA 2014: output n = mix(seed + (n + 1) * 0x9E3779B97F4A7C15)); then
 * sparsesam_perm(cfg, score, perm, inv, keep) runs on them (perm, inv, keep as there). */
int sparsesam_random_perm(const ss_cfg* cfg, uint64_t seed, double* score, int32_t* perm,
                          int32_t* inv, int32_t* keep, void* stream);

/* The keep-set by update magnitude (Dutch summary, "Methodologie" 2, "Selectieve Berekening": the
 * MLP runs on the top-K tokens with high feature dissimilarity or update magnitude). delta (device)
 * bf16 [batch, grid_h*grid_w, C], 16-byte aligned, C % 8 == 0: each token's update (e.g. the
 * block's attention output). mag (device) fp64 [batch, grid_h*grid_w] receives
 * sum over c = 0..C-1 (in that order, one fp64 rounding per multiply and per add) of
 * delta[b,t,c]^2; keep (device) int32 [batch, K] the first K tokens of each image's stable
 * descending ranking by mag (equal magnitudes: lower token first), 0 <= K <= grid_h*grid_w, for
 * sparsesam_rcmlp(..., keep, K, ...). K = 0 launches nothing. */
int sparsesam_keep_by_update(const ss_cfg* cfg, const uint16_t* delta, int32_t C, int32_t K,
                             double* mag, int32_t* keep, void* stream);

/* Bytes of device workspace sparsesam_attn needs for cfg (0 on an invalid cfg). */
size_t sparsesam_attn_workspace(const ss_cfg* cfg);

/* S3 (same summary, "Statisch Sparsiteitspatroon"; a FlashAttention-2-style kernel over a static
 * pattern). For every unit and head: Qp = q[perm], Kp = k[perm], Vp = v[perm];
 * Op[p] = softmax over the kept keys p' of (Qp[p].Kp[p'] / sqrt(head_dim)) applied to Vp;
 * out[perm[p]] = Op[p]. q, k, v (device, read only), perm (device) from sparsesam_perm, out
 * (device, may not alias q/k/v). bf16 operands, fp32 accumulation and softmax, probabilities rounded
 * to bf16 before the second product. ws (device, 256-byte aligned) >= sparsesam_attn_workspace(cfg)
 * bytes of scratch; its contents on entry do not matter. */
int sparsesam_attn(const ss_cfg* cfg, const uint16_t* q, const uint16_t* k, const uint16_t* v,
                   const int32_t* perm, uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* S3 without its gather: the attention kernel alone, over the permuted Q, K, V that an earlier
 * sparsesam_attn (or sparsesam_block) call with the same cfg and perm left in ws. ws holds three
 * bf16 arrays of sparsesam_attn_workspace(cfg)/3 bytes each (Q, then K, then V), each laid out as
 * [U*heads][N][head_dim]: row q of matrix u*heads+h is the token perm[u][j*L + a*b + r] for the
 * block-major position q = a*4b + j*b + r (offset block a of stripe j; L, b from the pattern).
 * out, perm and the results as for sparsesam_attn. For re-running the attention on prepared
 * operands (and timing the kernel by itself). */
int sparsesam_attn_gathered(const ss_cfg* cfg, const void* ws, size_t ws_bytes,
                            const int32_t* perm, uint16_t* out, void* stream);

/* Bytes of device workspace sparsesam_attn_relpos needs (0 on an invalid cfg). */
size_t sparsesam_attn_relpos_workspace(const ss_cfg* cfg);

/* S3 with SAM's decomposed relative-position bias fused (SparseSAM README, folder layout:
 * "kernels/ ... FA2 + rel-pos"): the score of query token (qh, qw) and key token (kh, kw) of a
 * unit is q.k/sqrt(head_dim) + q.rel_h[qh-kh+Hu-1] + q.rel_w[qw-kw+Wu-1] (q unscaled), over the
 * same kept keys as sparsesam_attn. The unit grid Hu x Wu is grid_h x grid_w (global mode) or
 * window x window (window mode; pad tokens have window coordinates). rel_h (device) bf16
 * [2*Hu-1, head_dim], rel_w (device) bf16 [2*Wu-1, head_dim], 16-byte aligned, shared by the
 * heads. Everything else as sparsesam_attn. The products q.rel_h[r] and q.rel_w[r] are computed
 * on the tensor cores in fp32 and kept in fp16 (scaled by sqrt(head_dim)); the attention adds a
 * key's two terms to its fp32 score with one more tensor-core product (the row's bias values
 * times the key tile's one-hot matrix). Head dim 64 only and Hu + Wu <= 128 (SS_EUNSUPPORTED
 * otherwise): a query row's bias values fill its group's 64 spare TMEM columns. ws (device,
 * 256-byte aligned) >= sparsesam_attn_relpos_workspace(cfg) bytes. */
int sparsesam_attn_relpos(const ss_cfg* cfg, const uint16_t* q, const uint16_t* k,
                          const uint16_t* v, const int32_t* perm, const uint16_t* rel_h,
                          const uint16_t* rel_w, uint16_t* out, void* ws, size_t ws_bytes,
                          void* stream);

/* Bytes of device workspace sparsesam_attn_partial needs (0 on invalid arguments). */
size_t sparsesam_attn_partial_workspace(const ss_cfg* cfg, int32_t prefix);

/* S3 for Perception-Encoder-style sequences: the SparseSAM README's `sparsesam_partial` variant
 * ("Zero-shot CLIP on ImageNet-1k": apply_pe(model.visual, "sparsesam_partial", ratio,
 * group_size=4, ...), with the RoPE of its "kernels/" directory fused). A unit's sequence is
 * `prefix` extra tokens (e.g. the class token; 0 <= prefix <= 4) followed by the grid_h x grid_w
 * patch tokens in raster order: q, k, v, out (device) bf16 [batch, prefix + grid_h*grid_w, heads,
 * head_dim]. cfg must be in global mode; perm (device) int32 [batch, grid_h*grid_w] is the patch
 * tokens' stripe-sort permutation (sparsesam_perm of the patch grid's scores).
 *   - RoPE (rope_base > 1; 0 = none): q and k of patch token (y, x) are rotated pairwise: channels
 *     (d, d+1) of a head, d even, by the angle pos * rope_base^(-i/(head_dim/4)), where
 *     i = (d mod head_dim/2) / 2 and pos = y for d < head_dim/2, x otherwise (an axial 2-D RoPE:
 *     the first half of the channels encodes the row, the second the column). Prefix tokens are
 *     not rotated. Rotation in fp32 from the bf16 inputs, rounded to bf16.
 *   - Patch query rows: softmax of (q.k)/sqrt(head_dim) over their kept patch keys (the static
 *     pattern over the patch tokens, as sparsesam_attn) and every prefix key.
 *   - Prefix query rows: softmax over every key of the unit (dense).
 * fp32 softmax; ws (device, 256-byte aligned) >= sparsesam_attn_partial_workspace(cfg, prefix)
 * bytes. Errors: as sparsesam_attn; SS_EUNSUPPORTED for window mode, more than 32 heads or more
 * than 16384 tokens; SS_EINVAL for prefix or rope_base out of range. */
int sparsesam_attn_partial(const ss_cfg* cfg, int32_t prefix, float rope_base, const uint16_t* q,
                           const uint16_t* k, const uint16_t* v, const int32_t* perm,
                           uint16_t* out, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sparsesam_rcmlp needs for K kept tokens per image (0 on invalid
 * arguments). */
size_t sparsesam_rcmlp_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden, int32_t K);

/* S4 (same summary, "Residual-Consistency MLP": only the top-K keep-set runs through the MLP; the
 * residual set bypasses it unchanged). In place on x (device) bf16 [batch, grid_h*grid_w, C]:
 * for each image b and kept token t = keep[b][r], r < K:
 *   x[b,t,:] = bf16( x[b,t,:] + (w2 . GELU(w1 . x[b,t,:] + b1) + b2) ),  GELU(z) = z/2 (1+erf(z/sqrt2))
 * every other row is left bit-for-bit untouched. w1 bf16 [hidden, C], w2 bf16 [C, hidden]
 * (row-major, PyTorch nn.Linear weight layout); b1 [hidden], b2 [C] bf16 or NULL (zero); x, w1,
 * w2, b1 and b2 16-byte aligned. keep
 * (device) int32 [batch, K] with distinct rows per image: the keep list sparsesam_perm writes
 * (K = the pattern's `keep`, from the density) or one from another criterion
 * (sparsesam_keep_by_update, sparsesam_random_perm), 0 <= K <= grid_h*grid_w; K = 0 launches
 * nothing.
 * C and hidden must be multiples of 64. bf16 operands, fp32 accumulation; the hidden activation
 * is rounded to bf16 between the two products. ws (device, 256-byte aligned) >=
 * sparsesam_rcmlp_workspace bytes. */
int sparsesam_rcmlp(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden,
                    const uint16_t* w1, const uint16_t* b1, const uint16_t* w2, const uint16_t* b2,
                    const int32_t* keep, int32_t K, void* ws, size_t ws_bytes, void* stream);

/* Bytes of device workspace sparsesam_block needs (0 on an invalid cfg). */
size_t sparsesam_block_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden);

/* S1..S4 of one encoder block in one call: sparsesam_score_perm(cfg, lum, score, perm, inv, keep),
 * then sparsesam_attn(cfg, q, k, v, perm, out), then sparsesam_rcmlp(cfg, x, C, hidden, w1, b1,
 * w2, b2, keep), with one workspace: the same launches and results, bit for bit. Arguments and
 * their layouts, alignment and error codes as in those calls (lum, score, perm, keep, out
 * non-NULL; inv may be NULL); in addition out may not overlap x (SS_EINVAL), since S4's row gather
 * is allowed to start before S3 has finished. ws (device, 256-byte aligned) >=
 * sparsesam_block_workspace(cfg, C, hidden) bytes; its contents on entry do not matter. */
int sparsesam_block(const ss_cfg* cfg, const float* lum, const uint16_t* q, const uint16_t* k,
                    const uint16_t* v, uint16_t* x, int32_t C, int32_t hidden, const uint16_t* w1,
                    const uint16_t* b1, const uint16_t* w2, const uint16_t* b2, double* score,
                    int32_t* perm, int32_t* inv, int32_t* keep, uint16_t* out, void* ws,
                    size_t ws_bytes, void* stream);

/* One encoder block's weights (device pointers, bf16, 16-byte aligned; Linear weights in the
 * PyTorch nn.Linear [out, in] layout, row-major). The Linear biases may be NULL (zero); the
 * LayerNorm weight and bias may not. */
typedef struct {
  const uint16_t* ln1_w;    /* [C]        LayerNorm before the attention */
  const uint16_t* ln1_b;    /* [C] */
  const uint16_t* w_qkv;    /* [3C, C]    rows: q (C), k (C), v (C); within each, head-major */
  const uint16_t* b_qkv;    /* [3C] */
  const uint16_t* w_proj;   /* [C, C]     the attention's output projection */
  const uint16_t* b_proj;   /* [C] */
  const uint16_t* ln2_w;    /* [C]        LayerNorm before the MLP */
  const uint16_t* ln2_b;    /* [C] */
  const uint16_t* w1;       /* [hidden, C] */
  const uint16_t* b1;       /* [hidden] */
  const uint16_t* w2;       /* [C, hidden] */
  const uint16_t* b2;       /* [C] */
} ss_block_weights;

/* Bytes of device workspace sparsesam_encoder_block needs for K kept tokens per image (0 on
 * invalid arguments). */
size_t sparsesam_encoder_block_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden, int32_t K);

/* One full SparseSAM encoder block, in place on x (device) bf16 [batch, grid_h*grid_w, C]. The
 * pages patch SparseSAM into SAM's image encoder (README, "SparseSAM": on top of the original
 * checkpoints), so the block is SAM's pre-norm ViT block with S3 as its attention and S4 as its MLP:
 *   a  = S3 attention of qkv(LN1(x)) over the cfg's units (window mode: the normalised grid padded
 *        bottom/right with zero rows to whole windows), heads = cfg->heads, head_dim = C / heads;
 *   x1 = x + proj(a)   (rows of pad tokens dropped);
 *   x  = x1, and for each kept token t of image b: x[b,t] = x1[b,t] + fc2(GELU(fc1(LN2(x1[b,t])))).
 * LayerNorm: (v - mean) / sqrt(var + 1e-6) * weight + bias with the biased variance, fp32
 * statistics. perm, inv (device) int32 [U, N]: the cfg's stripe-sort permutation and its inverse
 * (sparsesam_score_perm with the same cfg); keep (device) int32 [batch, K], 0 <= K <=
 * grid_h*grid_w, as for sparsesam_rcmlp. C = heads * head_dim (head_dim 64 or 80), C and hidden
 * multiples of 64. bf16 operands and activations between the steps (LN outputs, q/k/v, the
 * attention output, x1, the MLP's hidden activation), fp32 accumulation and softmax. ws (device,
 * 256-byte aligned) >= sparsesam_encoder_block_workspace(cfg, C, hidden, K) bytes; its contents on
 * entry do not matter. Errors: SS_EINVAL (NULL or misaligned pointer, C != heads*head_dim, K out
 * of range), SS_EUNSUPPORTED (head_dim, C or hidden not a multiple of 64, N % 4, sizes beyond the
 * launch limits), SS_EWORKSPACE; a perm/inv/keep entry out of range records SS_EINDEX and skips
 * that row. */
int sparsesam_encoder_block(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden,
                            const ss_block_weights* w, const int32_t* perm, const int32_t* inv,
                            const int32_t* keep, int32_t K, void* ws, size_t ws_bytes,
                            void* stream);

/* Bytes of device workspace sparsesam_encoder_stack needs (0 on invalid arguments). */
size_t sparsesam_encoder_stack_workspace(const ss_cfg* cfg, int32_t C, int32_t hidden);

/* The encoder's n_blocks blocks in order, in place on x (device) bf16 [batch, grid_h*grid_w, C].
 * The tokens are ranked once (Dutch summary, "Methodologie": one precomputed permutation set is
 * reused by every layer; here S1 + S2 of lum): the global blocks (is_global[i] != 0) use the whole-image stripe-sort permutation, the
 * windowed blocks the per-window permutations (window = cfg->window) of the same scores, and every
 * block the keep-set of K = ceil(density * grid_h*grid_w) tokens per image. cfg->mode is ignored.
 * w (host) [n_blocks] and is_global (host) [n_blocks]; each block as sparsesam_encoder_block.
 * ws (device, 256-byte aligned) >= sparsesam_encoder_stack_workspace(cfg, C, hidden) bytes; it
 * holds the scores, both permutations, the keep list and one block's workspace, reused by every
 * block. Errors as for sparsesam_encoder_block, for either geometry. */
int sparsesam_encoder_stack(const ss_cfg* cfg, const float* lum, uint16_t* x, int32_t C,
                            int32_t hidden, int32_t n_blocks, const ss_block_weights* w,
                            const uint8_t* is_global, void* ws, size_t ws_bytes, void* stream);

/* S4 without a caller-provided workspace. The SparseSAM pages have no counterpart to this call;
 * it exists for callers that cannot allocate device memory where they run the block: hosts whose
 * allocator owns all device memory and gives plug-ins none, and latency-bound loops that must not
 * pay cudaMalloc's implicit device-wide synchronisation. Same arguments, semantics and results as sparsesam_rcmlp,
 * minus ws/ws_bytes: the scratch lives in a 32 MiB array inside this library (a file-scope
 * __device__ array that every GPU loading the library holds until the process exits).
 *   - Arguments are checked as sparsesam_rcmlp checks them (same codes); then, before any CUDA
 *     call, SS_EWORKSPACE when sparsesam_rcmlp_workspace(cfg, C, hidden, K) exceeds 32 MiB (e.g.
 *     the SAM ViT-B global block, 28 MB, fits; batch 4 does not).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 *   - The first call on a device looks up the array's device address (cudaGetSymbolAddress, with
 *     that device current). The address is kept
 *     for the process; after a cudaDeviceReset of that device it is stale (so is the status
 *     word's address that every call looks up the same way), and the library must not be used on
 *     that device again.
 *   - All calls on a device share the one array and leave their contents in it; nothing needs
 *     clearing because each call writes every scratch byte before reading it. Calls whose GPU
 *     execution overlaps (different streams, no ordering between them) race on the array. */
int sparsesam_rcmlp_noalloc(const ss_cfg* cfg, uint16_t* x, int32_t C, int32_t hidden,
                            const uint16_t* w1, const uint16_t* b1, const uint16_t* w2,
                            const uint16_t* b2, const int32_t* keep, int32_t K, void* stream);

/* Reads (and clears) the device status word that bounded device waits and index checks write.
 * Synchronises the given stream. *status receives SS_OK, SS_ETIMEOUT or SS_EINDEX. Returns SS_OK or
 * SS_ECUDA. */
int sparsesam_device_status(int32_t* status, void* stream);

/* Test support for the failure path of the bounded device waits (no counterpart on the pages).
 * sparsesam_set_wait_limit_ns sets, on the current device, how long a device wait may take before
 * it gives up (default 500 ms; 0 restores the default). sparsesam_wait_selftest launches one CTA
 * that waits on an mbarrier no thread arrives on (`which` = 0) or on a global counter nothing
 * increments (`which` = 1), through the same bounded waits the kernels use, so that the wait runs
 * out and records SS_ETIMEOUT in the status word; with `which` = 2 or 3 the barrier is arrived on /
 * the counter is set first, so the wait succeeds and records nothing. Nothing else is in flight in
 * that CTA. Both return SS_OK, SS_EINVAL or SS_ECUDA. */
int sparsesam_set_wait_limit_ns(uint64_t ns);
int sparsesam_wait_selftest(int32_t which, void* stream);

/* Kernel launches this library has issued since it was loaded (host counter). */
uint64_t sparsesam_launch_count(void);

/* Per-launch tracing. While enabled, each kernel launch is bracketed by two CUDA events on its
 * stream (at most `capacity` launches are recorded). sparsesam_trace_stop synchronises the events,
 * and sparsesam_trace_get(i, ...) returns the i-th launch's kernel name and duration in ms.
 * Returns the number of records (stop) or SS_OK / SS_EINVAL / SS_ECUDA. */
int sparsesam_trace_start(int32_t capacity);
int sparsesam_trace_stop(void);
int sparsesam_trace_get(int32_t i, const char** name, float* ms);

/* Static text for a return code. */
const char* sparsesam_strerror(int code);

#ifdef __cplusplus
}
#endif
#endif /* SPARSESAM_H */
