"""Float64 CPU oracle of the SparseSAM encoder-block hot path.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import, call or execute this module: only
the tests, the smoke check and the benchmark's CPU-baseline / reference legs do. It shares no code
with the CUDA library and imports nothing from it.

What it computes, step by step, as the SparseSAM pages describe it (the pages give prose only; each
open choice takes the plainest reading, listed beside each function):

  S1 score  -- SparseSAM technical summary (Dutch), "Methodologie" 1, "Op Gradiënten Gebaseerde
               Ordening"; Japanese summary "手法" 1, 勾配に基づく順序付け: a parameter-free Sobel
               operator gives the local gradient magnitude of each token.
  S2 perm   -- same sections, "Stripe-Sort Permutatie": sort the tokens by that score, treat the
               sorted list as a matrix, transpose it and flatten it.
  S3 attn   -- same sections, "Statisch Sparsiteitspatroon": the permutation splits the N x N
               attention matrix into a 4 x 4 mosaic of sub-maps, each banded around its diagonal,
               plus a small global keep-set; SparseSAM README, "apply_sam(..., ratio=0.5)  # density
               50%": the knob is the computed fraction.
  S4 rcmlp  -- Dutch summary "Methodologie" 2, "Residual-Consistency MLP": the MLP runs on the top-K
               keep-set only; the residual set passes through unchanged.

Pins (tests/test_oracle_pins.py): closed forms, invariants, library routines and brute force.
The pattern's constants -- block-size rule, one global offset block, the nearest-density band width --
are a reading of silent pages: their implementation is pinned by hand-derived counts, but against the
pages themselves they are parity unpinned (the pages print no worked example).

All arithmetic is IEEE float64. S1 uses one RN operation per step in a fixed order (numpy never fuses
multiply-add), so its results are bit-reproducible.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np
from scipy.special import erf

STRIPES = 4          # "4 x 4 mosaic" (Dutch summary, Statisch Sparsiteitspatroon); group_size=4 (README, PE example)
MAX_BLOCK = 64       # reading: block size is the largest divisor of L that is <= 64 with >= 4 blocks
GLOBAL_BLOCKS = 1    # reading: the global keep-set is offset block 0 of every stripe


# ---------------------------------------------------------------------------------------------
# S1: Sobel score
# ---------------------------------------------------------------------------------------------
def sobel_score(lum: np.ndarray) -> np.ndarray:
    """Squared Sobel gradient magnitude per token, float64 [B, Hg*Wg] in raster order.

    Reading: replicate (clamp-to-edge) border, so a constant image scores exactly 0; the squared
    magnitude gx^2 + gy^2 orders tokens as the magnitude does, so no square root; no normalisation.
    Operation order (each a single float64 RN op):
      gx = ((l[y-1,x+1] - l[y-1,x-1]) + 2*(l[y,x+1] - l[y,x-1])) + (l[y+1,x+1] - l[y+1,x-1])
      gy = ((l[y+1,x-1] - l[y-1,x-1]) + 2*(l[y+1,x] - l[y-1,x])) + (l[y+1,x+1] - l[y-1,x+1])
      s  = gx*gx + gy*gy
    """
    lum = np.asarray(lum)
    assert lum.ndim == 3
    B, H, W = lum.shape
    l = lum.astype(np.float64)
    out = np.empty((B, H * W), dtype=np.float64)
    for b in range(B):
        img = l[b]

        def at(dy, dx):
            ys = np.clip(np.arange(H) + dy, 0, H - 1)
            xs = np.clip(np.arange(W) + dx, 0, W - 1)
            return img[ys][:, xs]

        gx = ((at(-1, 1) - at(-1, -1)) + 2.0 * (at(0, 1) - at(0, -1))) + (at(1, 1) - at(1, -1))
        gy = ((at(1, -1) - at(-1, -1)) + 2.0 * (at(1, 0) - at(-1, 0))) + (at(1, 1) - at(-1, 1))
        out[b] = (gx * gx + gy * gy).reshape(-1)
    return out


# ---------------------------------------------------------------------------------------------
# Units: which tokens an attention unit holds, in its enumeration (raster) order
# ---------------------------------------------------------------------------------------------
@dataclass(frozen=True)
class Geometry:
    batch: int
    grid_h: int
    grid_w: int
    mode: str = "global"      # "global" | "window"
    window: int = 14

    @property
    def padded(self):
        if self.mode == "global":
            return self.grid_h, self.grid_w
        ws = self.window
        return -(-self.grid_h // ws) * ws, -(-self.grid_w // ws) * ws

    @property
    def windows(self) -> int:
        if self.mode == "global":
            return 1
        hp, wp = self.padded
        return (hp // self.window) * (wp // self.window)

    @property
    def units(self) -> int:
        return self.batch * self.windows

    @property
    def unit_tokens(self) -> int:
        return self.grid_h * self.grid_w if self.mode == "global" else self.window ** 2


def unit_members(geo: Geometry):
    """For every unit, (image index, array of raster token ids of the image or -1 for a pad token).

    Global mode: the whole image in row-major order. Window mode (SAM's windowed blocks): the grid
    is padded bottom/right to a multiple of the window and cut into windows in row-major window
    order; a window enumerates its tokens row-major.
    """
    units = []
    if geo.mode == "global":
        for b in range(geo.batch):
            units.append((b, np.arange(geo.grid_h * geo.grid_w)))
        return units
    ws = geo.window
    hp, wp = geo.padded
    for b in range(geo.batch):
        for wy in range(hp // ws):
            for wx in range(wp // ws):
                ids = np.full(ws * ws, -1, dtype=np.int64)
                for r in range(ws):
                    for c in range(ws):
                        y, x = wy * ws + r, wx * ws + c
                        if y < geo.grid_h and x < geo.grid_w:
                            ids[r * ws + c] = y * geo.grid_w + x
                units.append((b, ids))
    return units


def unit_scores(score: np.ndarray, geo: Geometry) -> np.ndarray:
    """[U, N] float64 scores of each unit's tokens in enumeration order; pad tokens score +0.0."""
    out = np.zeros((geo.units, geo.unit_tokens), dtype=np.float64)
    for u, (b, ids) in enumerate(unit_members(geo)):
        real = ids >= 0
        out[u, real] = score[b, ids[real]]
    return out


# ---------------------------------------------------------------------------------------------
# S2: stable sort and stripe transpose
# ---------------------------------------------------------------------------------------------
def ranked_order(s: np.ndarray) -> np.ndarray:
    """Enumeration indices sorted by score, descending; equal scores keep lower index first.

    Reading: descending (the keep-set is the "top-K"); a stable sort on the raster enumeration.
    """
    s = np.asarray(s, dtype=np.float64)
    return np.argsort(-s, kind="stable")


def stripe_transpose(ranked: np.ndarray, stripes: int = STRIPES):
    """Stripe-sort permutation from a ranked list.

    The ranked list is read row-major as an (L, S) matrix, transposed to (S, L) and flattened, so
    position p = j*L + k holds rank S*k + j. Returns (perm, inv): perm[p] = enumeration index at
    permuted position p, inv[perm[p]] = p.
    """
    n = ranked.shape[0]
    assert n % stripes == 0, "token count must be a multiple of the stripe count"
    L = n // stripes
    perm = ranked.reshape(L, stripes).T.reshape(-1).copy()
    inv = np.empty_like(perm)
    inv[perm] = np.arange(n)
    return perm.astype(np.int32), inv.astype(np.int32)


def stripe_sort(score: np.ndarray, geo: Geometry):
    """perm, inv int32 [U, N] for every attention unit (S2)."""
    us = unit_scores(score, geo)
    perms = np.empty(us.shape, dtype=np.int32)
    invs = np.empty(us.shape, dtype=np.int32)
    for u in range(us.shape[0]):
        perms[u], invs[u] = stripe_transpose(ranked_order(us[u]))
    return perms, invs


# ---------------------------------------------------------------------------------------------
# S3: static pattern
# ---------------------------------------------------------------------------------------------
def block_size(L: int) -> int:
    """Largest divisor b of L with b <= 64 and L/b >= 4 (reading of the unstated block size)."""
    for b in range(min(MAX_BLOCK, L), 0, -1):
        if L % b == 0 and L // b >= 4:
            return b
    raise ValueError(f"stripe length {L} too short for a 4-block pattern")


def band_start(a: int, W: int, nb: int) -> int:
    """First offset block of the width-W band of row a: the window is shifted inward at the edges."""
    return min(max(a - (W - 1) // 2, 0), nb - W)


def kept_offset_blocks(a: int, W: int, nb: int, g: int = GLOBAL_BLOCKS) -> list[int]:
    """Key offset blocks a' kept for query offset block a: Band_W(a) united with [0, g)."""
    s = band_start(a, W, nb)
    return sorted(set(range(s, s + W)) | set(range(g)))


def density_of(W: int, nb: int, g: int = GLOBAL_BLOCKS) -> float:
    return sum(len(kept_offset_blocks(a, W, nb, g)) for a in range(nb)) / float(nb * nb)


@dataclass(frozen=True)
class Pattern:
    N: int
    L: int
    b: int
    nb: int
    W: int
    g: int
    rho: float
    row_ptr: np.ndarray   # CSR over query offset blocks a: kept key offset blocks
    col_idx: np.ndarray


def pattern(N: int, density: float) -> Pattern:
    """The static pattern for an N-token unit at the requested density.

    The band width W in [1, nb] is the one whose realised density is nearest to the request; a tie
    goes to the smaller W. The same offset-block pattern holds in all 16 sub-maps of the mosaic.
    """
    if not (0.0 < density <= 1.0):
        raise ValueError("density must lie in (0, 1]")
    assert N % STRIPES == 0
    L = N // STRIPES
    b = block_size(L)
    nb = L // b
    best_W, best_err = None, None
    for W in range(1, nb + 1):
        err = abs(density_of(W, nb) - density)
        if best_err is None or err < best_err:
            best_W, best_err = W, err
    W = best_W
    rows = [kept_offset_blocks(a, W, nb) for a in range(nb)]
    row_ptr = np.zeros(nb + 1, dtype=np.int32)
    row_ptr[1:] = np.cumsum([len(r) for r in rows])
    col_idx = np.array([c for r in rows for c in r], dtype=np.int32)
    return Pattern(N, L, b, nb, W, GLOBAL_BLOCKS, density_of(W, nb), row_ptr, col_idx)


def position_offset_block(N: int, b: int) -> np.ndarray:
    """Offset block a of every permuted position p = j*L + a*b + r."""
    L = N // STRIPES
    return (np.arange(N) % L) // b


def attention(q, k, v, perm, density: float) -> np.ndarray:
    """Stripe-Sort attention, float64 [U, N, heads, dh].

    Qp = Q[perm], Kp = K[perm], Vp = V[perm]; each permuted query row takes a softmax (with its max
    subtracted, summed in float64, no online rescaling) of Qp.Kp/sqrt(dh) over its kept keys only,
    then out[perm[p]] = Op[p].
    """
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    U, N, H, D = q.shape
    pat = pattern(N, density)
    blk = position_offset_block(N, pat.b)
    scale = 1.0 / math.sqrt(D)
    out = np.empty((U, N, H, D), dtype=np.float64)
    for u in range(U):
        pm = perm[u]
        qp = q[u][pm].transpose(1, 0, 2)   # [H, N, D]
        kp = k[u][pm].transpose(1, 0, 2)
        vp = v[u][pm].transpose(1, 0, 2)
        for a in range(pat.nb):
            rows = np.nonzero(blk == a)[0]
            kept = pat.col_idx[pat.row_ptr[a]:pat.row_ptr[a + 1]]
            keys = np.nonzero(np.isin(blk, kept))[0]
            s = np.matmul(qp[:, rows], kp[:, keys].transpose(0, 2, 1)) * scale
            s = s - s.max(axis=2, keepdims=True)
            e = np.exp(s)
            p = e / e.sum(axis=2, keepdims=True)
            o = np.matmul(p, vp[:, keys])                # [H, rows, D]
            out[u, pm[rows]] = o.transpose(1, 0, 2)
    return out


# ---------------------------------------------------------------------------------------------
# S4: Residual-Consistency MLP
# ---------------------------------------------------------------------------------------------
def keep_count(density: float, tokens: int) -> int:
    """K = ceil(d*N - 1e-9) in float64: the top-K keep-set size over an image's real tokens."""
    if not (0.0 < density <= 1.0):
        raise ValueError("density must lie in (0, 1]")
    return int(math.ceil(density * tokens - 1e-9))


def keep_list(score: np.ndarray, density: float) -> np.ndarray:
    """int32 [B, K]: the K highest-scoring tokens of each image, in rank order (per-image sort)."""
    B, T = score.shape
    K = keep_count(density, T)
    out = np.empty((B, K), dtype=np.int32)
    for b in range(B):
        out[b] = ranked_order(score[b])[:K]
    return out


def gelu(z: np.ndarray) -> np.ndarray:
    """Exact (erf) GELU: z/2 * (1 + erf(z/sqrt(2)))."""
    return 0.5 * z * (1.0 + erf(z / math.sqrt(2.0)))


def rcmlp(x, w1, b1, w2, b2, keep) -> np.ndarray:
    """y = x; y[t] = x[t] + (W2 GELU(W1 x[t] + b1) + b2) for every kept token t of each image.

    x [B, T, C]; w1 [hidden, C]; w2 [C, hidden]; b1/b2 may be None (zero). Rows outside the keep
    set are copied unchanged.
    """
    x = np.asarray(x, dtype=np.float64)
    w1 = np.asarray(w1, dtype=np.float64)
    w2 = np.asarray(w2, dtype=np.float64)
    b1 = np.zeros(w1.shape[0]) if b1 is None else np.asarray(b1, dtype=np.float64)
    b2 = np.zeros(w2.shape[0]) if b2 is None else np.asarray(b2, dtype=np.float64)
    y = x.copy()
    for b in range(x.shape[0]):
        rows = np.asarray(keep[b], dtype=np.int64)
        if rows.size == 0:
            continue
        xs = x[b, rows]
        h = gelu(xs @ w1.T + b1)
        y[b, rows] = xs + (h @ w2.T + b2)
    return y


def keep_top(score: np.ndarray, K: int) -> np.ndarray:
    """int32 [B, K]: the K first tokens of each image's stable descending ranking by `score`
    (ties: lower token index first) -- the keep list of any keep criterion given as a score."""
    B, T = score.shape
    assert 0 <= K <= T
    out = np.empty((B, K), dtype=np.int32)
    for b in range(B):
        out[b] = ranked_order(score[b])[:K]
    return out


# ---------------------------------------------------------------------------------------------
# Variants: the random-permutation ablation and the update-magnitude keep criterion
# ---------------------------------------------------------------------------------------------
_GOLDEN_GAMMA = np.uint64(0x9E3779B97F4A7C15)


def splitmix64(seed: int, n: np.ndarray) -> np.ndarray:
    """Output n (n = 0, 1, ...) of the SplitMix64 generator started from state `seed` (Steele,
    Lea and Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014): the state after
    n + 1 steps, seed + (n + 1) * gamma, through the generator's output mix. uint64 arithmetic
    wraps modulo 2^64."""
    n = np.asarray(n, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = np.uint64(seed) + (n + np.uint64(1)) * _GOLDEN_GAMMA
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def random_scores(batch: int, tokens: int, seed: int) -> np.ndarray:
    """float64 [B, T] uniform in [0, 1): token t of image b draws output b*T + t of SplitMix64
    from `seed`, keeps its top 53 bits and scales them by 2^-53.

    Reading of the README's registry variant `sparsesam_random`: the stripe-sort permutation (and
    keep list) built from a random token order instead of the Sobel ranking -- the same sort,
    transpose and pattern, over these scores."""
    idx = np.arange(batch * tokens, dtype=np.uint64)
    u = splitmix64(seed, idx) >> np.uint64(11)
    return (u.astype(np.float64) * 2.0 ** -53).reshape(batch, tokens)


def update_magnitude(delta) -> np.ndarray:
    """float64 [B, T]: sum over channels c = 0, 1, ..., C-1, in that order, of delta[b, t, c]^2.

    Reading of the Dutch summary's "Selectieve Berekening" (the MLP runs on the top-K tokens "with
    high feature dissimilarity or update magnitude"): a token's update magnitude is the squared
    norm of the update its row receives (e.g. the block's attention output); the keep-set is
    keep_top(update_magnitude(delta), K). Each square of a bf16 value is exact in float64; the
    sum is rounded step by step in channel order."""
    d = np.asarray(delta, dtype=np.float64)
    acc = np.zeros(d.shape[:2], dtype=np.float64)
    for c in range(d.shape[2]):
        acc = acc + d[:, :, c] * d[:, :, c]
    return acc


# ---------------------------------------------------------------------------------------------
# Decomposed relative-position bias (SAM's attention), fused into S3
# ---------------------------------------------------------------------------------------------
# SparseSAM README, folder layout: "kernels/ fused cutlass-DSL CUDA kernels (FA2 + rel-pos / RoPE)".
# SAM's image-encoder attention (Kirillov et al., "Segment Anything", 2023, following MViTv2's
# decomposed relative positions) adds to the scaled score of query token (qh, qw) and key token
# (kh, kw) of a Hu x Wu unit grid the bias q . Rh[qh - kh + Hu - 1] + q . Rw[qw - kw + Wu - 1],
# with q unscaled and tables Rh [2Hu - 1, dh], Rw [2Wu - 1, dh] of the unit's size. Readings: the
# unit grid is the image (global blocks) or the window (windowed blocks; pad tokens have window
# coordinates like any other); the bias applies to the kept keys of the pattern only.


def unit_grid(geo: Geometry):
    """(Hu, Wu): the grid of one attention unit, whose tokens enumerate row-major."""
    return (geo.grid_h, geo.grid_w) if geo.mode == "global" else (geo.window, geo.window)


def relpos_bias(q, rel_h, rel_w, Hu: int, Wu: int) -> np.ndarray:
    """float64 [U, heads, N, N]: bias[u, h, i, j] of query token i and key token j (unit-local
    enumeration order) = q[u,i,h] . rel_h[yi - yj + Hu - 1] + q[u,i,h] . rel_w[xi - xj + Wu - 1]."""
    q = np.asarray(q, dtype=np.float64)
    rh = np.asarray(rel_h, dtype=np.float64)
    rw = np.asarray(rel_w, dtype=np.float64)
    U, N, H, D = q.shape
    assert N == Hu * Wu and rh.shape == (2 * Hu - 1, D) and rw.shape == (2 * Wu - 1, D)
    y, x = np.arange(N) // Wu, np.arange(N) % Wu
    qh = np.einsum("unhd,rd->uhnr", q, rh)                 # q . rel_h[r] for every r
    qw = np.einsum("unhd,rd->uhnr", q, rw)
    ridx_h = y[:, None] - y[None, :] + Hu - 1               # [N (query), N (key)]
    ridx_w = x[:, None] - x[None, :] + Wu - 1
    rows = np.arange(N)[:, None]
    return qh[:, :, rows, ridx_h] + qw[:, :, rows, ridx_w]


def attention_relpos(q, k, v, perm, density: float, geo: Geometry, rel_h, rel_w) -> np.ndarray:
    """Stripe-Sort attention with the decomposed relative-position bias, float64 [U, N, heads, dh]:
    each permuted query row's softmax over its kept keys of q.k/sqrt(dh) + bias (relpos_bias)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    U, N, H, D = q.shape
    Hu, Wu = unit_grid(geo)
    bias = relpos_bias(q, rel_h, rel_w, Hu, Wu)             # [U, H, N, N], token order
    pat = pattern(N, density)
    blk = position_offset_block(N, pat.b)
    scale = 1.0 / math.sqrt(D)
    out = np.empty((U, N, H, D), dtype=np.float64)
    for u in range(U):
        pm = np.asarray(perm[u], dtype=np.int64)
        qp = q[u][pm].transpose(1, 0, 2)
        kp = k[u][pm].transpose(1, 0, 2)
        vp = v[u][pm].transpose(1, 0, 2)
        bp = bias[u][:, pm][:, :, pm]                       # permuted rows and columns
        for a in range(pat.nb):
            rows = np.nonzero(blk == a)[0]
            kept = pat.col_idx[pat.row_ptr[a]:pat.row_ptr[a + 1]]
            keys = np.nonzero(np.isin(blk, kept))[0]
            s = np.matmul(qp[:, rows], kp[:, keys].transpose(0, 2, 1)) * scale
            s = s + bp[:, rows][:, :, keys]
            s = s - s.max(axis=2, keepdims=True)
            e = np.exp(s)
            o = np.matmul(e / e.sum(axis=2, keepdims=True), vp[:, keys])
            out[u, pm[rows]] = o.transpose(1, 0, 2)
    return out


# ---------------------------------------------------------------------------------------------
# The partial-token-count variant: prefix tokens + patch tokens, 2-D RoPE
# ---------------------------------------------------------------------------------------------
# SparseSAM README, "Zero-shot CLIP on ImageNet-1k": the Perception Encoder is patched with
# `sparsesam_partial` (group_size=4); its "kernels/" directory fuses RoPE into the attention.
# Readings of what the pages leave open: the sequence is `prefix` extra tokens (the class token)
# followed by the patch tokens in raster order; the stripe-sort pattern covers the patch tokens
# only; patch queries also attend every prefix key, prefix queries attend every key; the RoPE is
# axial 2-D (Su et al., "RoFormer", 2021, extended per axis): the first half of a head's channels
# rotates with the token's row, the second half with its column, pair i of a half at frequency
# base^(-i / (dh/4)); prefix tokens are not rotated.


def rope_2d(x, grid_h: int, grid_w: int, base: float) -> np.ndarray:
    """x [U, T, heads, dh] of patch tokens in raster order, rotated (float64): channels (d, d+1),
    d = half*dh/2 + 2i, turn by pos * base^(-i/(dh/4)), pos = row (half 0) or column (half 1)."""
    x = np.asarray(x, dtype=np.float64)
    U, T, H, D = x.shape
    assert T == grid_h * grid_w and D % 4 == 0
    half, quart = D // 2, D // 4
    pos = (np.arange(T) // grid_w, np.arange(T) % grid_w)
    out = x.copy()
    for axis in (0, 1):
        for i in range(quart):
            d = axis * half + 2 * i
            phi = pos[axis] * float(base) ** (-i / quart)
            c, s = np.cos(phi)[None, :, None], np.sin(phi)[None, :, None]
            a, b = x[:, :, :, d], x[:, :, :, d + 1]
            out[:, :, :, d] = a * c - b * s
            out[:, :, :, d + 1] = a * s + b * c
    return out


def attention_partial(q, k, v, perm, density: float, prefix: int, grid_h: int, grid_w: int,
                      rope_base: float) -> np.ndarray:
    """Stripe-Sort attention over prefix + patch sequences, float64 [U, prefix + T, heads, dh].

    Patch queries: softmax over their kept patch keys (the pattern over the T patch tokens, perm
    [U, T] their stripe-sort permutation) and every prefix key. Prefix queries: softmax over all
    keys. q and k of patch tokens are rotated by rope_2d first (rope_base 0: no rotation)."""
    q = np.asarray(q, dtype=np.float64).copy()
    k = np.asarray(k, dtype=np.float64).copy()
    v = np.asarray(v, dtype=np.float64)
    U, NT, H, D = q.shape
    T = NT - prefix
    if rope_base:
        q[:, prefix:] = rope_2d(q[:, prefix:], grid_h, grid_w, rope_base)
        k[:, prefix:] = rope_2d(k[:, prefix:], grid_h, grid_w, rope_base)
    pat = pattern(T, density)
    blk = position_offset_block(T, pat.b)
    scale = 1.0 / math.sqrt(D)

    def softmax_rows(s):
        s = s - s.max(axis=-1, keepdims=True)
        e = np.exp(s)
        return e / e.sum(axis=-1, keepdims=True)

    out = np.empty((U, NT, H, D), dtype=np.float64)
    for u in range(U):
        pm = np.asarray(perm[u], dtype=np.int64)
        qp = q[u, prefix + pm].transpose(1, 0, 2)          # [H, T, D]
        kp = k[u, prefix + pm].transpose(1, 0, 2)
        vp = v[u, prefix + pm].transpose(1, 0, 2)
        kx = k[u, :prefix].transpose(1, 0, 2)              # [H, prefix, D]
        vx = v[u, :prefix].transpose(1, 0, 2)
        for a in range(pat.nb):
            rows = np.nonzero(blk == a)[0]
            kept = pat.col_idx[pat.row_ptr[a]:pat.row_ptr[a + 1]]
            keys = np.nonzero(np.isin(blk, kept))[0]
            kk = np.concatenate([kp[:, keys], kx], axis=1)
            vv = np.concatenate([vp[:, keys], vx], axis=1)
            p = softmax_rows(np.matmul(qp[:, rows], kk.transpose(0, 2, 1)) * scale)
            out[u, prefix + pm[rows]] = np.matmul(p, vv).transpose(1, 0, 2)
        for j in range(prefix):
            s = np.einsum("hd,thd->ht", q[u, j], k[u]) * scale   # [H, NT]
            out[u, j] = np.einsum("ht,thd->hd", softmax_rows(s), v[u])
    return out


# ---------------------------------------------------------------------------------------------
# The full encoder block around S3 and S4, and the encoder stack
# ---------------------------------------------------------------------------------------------
# The pages patch SparseSAM into SAM's image encoder without retraining (README, "SparseSAM":
# "patched on top of the original checkpoints"), so the block around S3 and S4 is SAM's ViT block
# (Kirillov et al., "Segment Anything", 2023, image encoder: a ViT with 14x14 windowed blocks and a
# few global blocks): pre-norm, x = x + proj(attn(LN1(x))), x = x + MLP(LN2(x)). Readings of what
# the pages leave open: LayerNorm eps 1e-6 (SAM's encoder); the windowed blocks pad the normalised
# grid bottom/right with zero rows up to a multiple of the window and crop the attention branch
# back before the residual add; the qkv projection's 3C output columns are ordered (q|k|v, head,
# channel); the relative-position bias is left out (it is a separate row); the RC-MLP keeps its
# residual rows exactly (Dutch summary, "Residual-Consistency MLP"), so the MLP branch, LN2
# included, runs on the kept rows only.
LN_EPS = 1e-6


def layer_norm(x, weight, bias, eps: float = LN_EPS) -> np.ndarray:
    """LayerNorm over the last axis in float64: (x - mean) / sqrt(var + eps) * weight + bias, with
    the mean and the (biased) variance of each row."""
    x = np.asarray(x, dtype=np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * np.asarray(weight, np.float64) + np.asarray(bias, np.float64)


def to_units(x: np.ndarray, geo: Geometry) -> np.ndarray:
    """[B, T, C] -> [U, N, C]: each attention unit's rows in enumeration order (unit_members); a
    pad token's row is zero."""
    out = np.zeros((geo.units, geo.unit_tokens, x.shape[-1]), dtype=np.float64)
    for u, (b, ids) in enumerate(unit_members(geo)):
        real = ids >= 0
        out[u, real] = x[b, ids[real]]
    return out


def from_units(a: np.ndarray, geo: Geometry) -> np.ndarray:
    """[U, N, C] -> [B, T, C]: the rows of real tokens back at their image positions (pads
    dropped)."""
    out = np.zeros((geo.batch, geo.grid_h * geo.grid_w, a.shape[-1]), dtype=np.float64)
    for u, (b, ids) in enumerate(unit_members(geo)):
        real = ids >= 0
        out[b, ids[real]] = a[u, real]
    return out


@dataclass
class BlockParams:
    """One encoder block's weights (torch Linear convention: w [out, in]). Biases may be None."""
    ln1_w: np.ndarray
    ln1_b: np.ndarray
    w_qkv: np.ndarray      # [3C, C]
    b_qkv: np.ndarray
    w_proj: np.ndarray     # [C, C]
    b_proj: np.ndarray
    ln2_w: np.ndarray
    ln2_b: np.ndarray
    w1: np.ndarray         # [hidden, C]
    b1: np.ndarray
    w2: np.ndarray         # [C, hidden]
    b2: np.ndarray


def _lin(x, w, b):
    y = x @ np.asarray(w, np.float64).T
    return y if b is None else y + np.asarray(b, np.float64)


def encoder_block(x, prm: BlockParams, perm, keep, geo: Geometry, heads: int,
                  density: float) -> np.ndarray:
    """One SparseSAM encoder block, float64 [B, T, C]:
        a  = Stripe-Sort attention (S3) of qkv(LN1(x)) over the block's units,
        x1 = x + proj(a)                      (pad rows cropped),
        y  = x1; y[t] = x1[t] + MLP(LN2(x1[t])) for t in keep (S4's keep-set).
    perm: [U, N] of the block's geometry (window or global); keep: [B, K]."""
    x = np.asarray(x, dtype=np.float64)
    C = x.shape[-1]
    dh = C // heads
    xu = to_units(layer_norm(x, prm.ln1_w, prm.ln1_b), geo)
    qkv = _lin(xu, prm.w_qkv, prm.b_qkv)                                 # [U, N, 3C]
    U, N, _ = qkv.shape
    q, k, v = (qkv[..., i * C:(i + 1) * C].reshape(U, N, heads, dh) for i in range(3))
    a = attention(q, k, v, perm, density).reshape(U, N, C)
    x1 = x + from_units(_lin(a, prm.w_proj, prm.b_proj), geo)
    y = x1.copy()
    for b in range(x.shape[0]):
        rows = np.asarray(keep[b], dtype=np.int64)
        if rows.size == 0:
            continue
        h = gelu(_lin(layer_norm(x1[b, rows], prm.ln2_w, prm.ln2_b), prm.w1, prm.b1))
        y[b, rows] = x1[b, rows] + _lin(h, prm.w2, prm.b2)
    return y


def encoder_stack(x, blocks, lum, grid_window: int, global_blocks, heads: int,
                  density: float) -> np.ndarray:
    """The encoder's blocks in order over x [B, T, C]. One Sobel score per image ranks its tokens
    once (S1); the global blocks take the image's stripe-sort permutation, the windowed blocks the
    per-window permutations of the same scores, and every block the same keep-set (S2, S4).
    global_blocks: indices of the global-attention blocks; the others are windowed."""
    B, Hg, Wg = np.asarray(lum).shape
    score = sobel_score(lum)
    geo_g = Geometry(B, Hg, Wg, "global", grid_window)
    geo_w = Geometry(B, Hg, Wg, "window", grid_window)
    perm_g, _ = stripe_sort(score, geo_g)
    perm_w, _ = stripe_sort(score, geo_w)
    keep = keep_list(score, density)
    y = np.asarray(x, dtype=np.float64)
    for i, prm in enumerate(blocks):
        g = i in global_blocks
        y = encoder_block(y, prm, perm_g if g else perm_w, keep, geo_g if g else geo_w, heads,
                          density)
    return y


# ---------------------------------------------------------------------------------------------
# The whole block, for the smoke check and the CPU baseline
# ---------------------------------------------------------------------------------------------
def hot_path(lum, q, k, v, x, w1, b1, w2, b2, geo: Geometry, density: float):
    """S1..S4 in order; returns (score, perm, inv, keep, attn_out, mlp_out)."""
    score = sobel_score(lum)
    perm, inv = stripe_sort(score, geo)
    keep = keep_list(score, density)
    out = attention(q, k, v, perm, density)
    y = rcmlp(x, w1, b1, w2, b2, keep)
    return score, perm, inv, keep, out, y
