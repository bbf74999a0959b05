"""Plain, slow CPU oracle for retained-mass block-sparse attention over 3D video tokens.

TEST INFRASTRUCTURE ONLY.  This module is imported by tests/, by the smoke check in
__graft_entry__.py and by the CPU-baseline leg of bench.py -- never by the library.
It shares no code, table or helper with the CUDA path and imports nothing from it.

Everything here is numpy in float64 unless a step turns floating point into an
integer or a code, where it works in the precision stated at that step.  Each
function cites the passage it follows:

* [LoSA]  "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion
  Acceleration", Abstract: exact block attention masses measured at one dense step;
  per head and query block, the smallest key/value block set whose mass meets a
  retained-mass threshold (99% by default); the frozen block lists reused by the
  attention of all later steps.
* [FPS]   "FPSAttention: Training-Aware FP8 and Sparsity Co-Design for Fast Video
  Diffusion", Abstract, innovation 1: one 3D tile granularity shared by the sparsity
  block and the FP8 quantisation scale.
* [SVG2]  "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
  Semantic-Aware Permutation", Abstract: top-p dynamic budget control (the same
  per-row retained-mass selection).

Readings taken where the pages are silent (each is listed with its reason in the
design notes of the repository):

R1  tile order: tiles are 4x4x4 tokens, enumerated row-major over the tile grid
    (tt, th, tw); inside a tile, row-major over (dt, dh, dw).  Padded positions
    (outside the valid T x H x W grid) hold zeros.
R2  block mass of (query block i, kv block j) = mean over the valid queries of
    block i of the softmax probability mass falling on the valid keys of block j;
    pad keys are excluded from the softmax; a block with no valid query has an
    all-zero mass row.  Each row of valid masses then sums to 1.
R3  the selection compares masses as integers: q_j = rint(m_j * 2^40) from the
    float32 mass; target = ceil(tau * sum(q)) with tau * sum(q) one IEEE float64
    multiply (tau is the float32 threshold widened exactly); blocks are ranked by
    (q descending, index ascending); the kept set is the shortest prefix whose sum
    reaches the target; kept indices are emitted ascending.
R4  the sparse attention renormalises over the kept blocks only (no correction term);
    pad query rows and rows with no kept valid key output zeros (log-sum-exp -inf).
R5  FP8: one scale per (batch, head, 64-token tile): s = absmax / 448 in float32
    (s = 1 when absmax = 0); codes = e4m3 round-to-nearest-even with saturation to
    +-448 of (x / s) computed in float32.  The oracle attends over the dequantised
    values and does not model the quantisation of P.
"""
from __future__ import annotations

import functools
import math
from dataclasses import dataclass

import numpy as np

TILE = 4          # tile edge in tokens along t, h and w
TILE_TOKENS = 64  # tokens per tile
FP_SCALE = 2.0 ** 40


@dataclass(frozen=True)
class Grid:
    """Valid grid (T, H, W) and padded grid (Tp, Hp, Wp); padded sizes are multiples of 4."""
    T: int
    H: int
    W: int
    Tp: int
    Hp: int
    Wp: int

    def __post_init__(self):
        for v, p in ((self.T, self.Tp), (self.H, self.Hp), (self.W, self.Wp)):
            if v < 1 or p < v or p % TILE:
                raise ValueError("padded extents must cover the grid and be multiples of 4")

    @property
    def S(self):
        return self.T * self.H * self.W

    @property
    def Np(self):
        return self.Tp * self.Hp * self.Wp


# --------------------------------------------------------------------------- permute
@functools.lru_cache(maxsize=16)
def _tile_slot_source_cached(g: "Grid") -> np.ndarray:
    return _tile_slot_source(g)


def tile_slot_source(g: Grid) -> np.ndarray:
    """Cached copy of the slot map (see _tile_slot_source)."""
    return _tile_slot_source_cached(g).copy()


def _tile_slot_source(g: Grid) -> np.ndarray:
    """For every tile-major slot p, the raster token index it holds, or -1 for a pad slot.

    [FPS] unified 3D tile-wise granularity; order per reading R1.  Written as the plain
    triple loop over padded positions.
    """
    nth, ntw = g.Hp // TILE, g.Wp // TILE
    src = np.full(g.Np, -1, dtype=np.int64)
    for t in range(g.Tp):
        for h in range(g.Hp):
            for w in range(g.Wp):
                tile = ((t // TILE) * nth + h // TILE) * ntw + w // TILE
                inner = ((t % TILE) * TILE + h % TILE) * TILE + w % TILE
                if t < g.T and h < g.H and w < g.W:
                    src[tile * TILE_TOKENS + inner] = (t * g.H + h) * g.W + w
    return src


def valid_slots(g: Grid) -> np.ndarray:
    return _tile_slot_source_cached(g) >= 0


def permute_forward(x: np.ndarray, g: Grid) -> np.ndarray:
    """Raster [B, S, Hh, D] -> tile-major [B, Hh, Np, D]; pad slots zero.  [FPS], R1."""
    B, S, Hh, D = x.shape
    if S != g.S:
        raise ValueError("token count does not match the grid")
    src = tile_slot_source(g)
    out = np.zeros((B, Hh, g.Np, D), dtype=x.dtype)
    for p in range(g.Np):
        if src[p] >= 0:
            out[:, :, p, :] = x[:, src[p], :, :]
    return out


def permute_inverse(y: np.ndarray, g: Grid) -> np.ndarray:
    """Tile-major [B, Hh, Np, D] -> raster [B, S, Hh, D]; pad slots dropped.  [FPS], R1."""
    B, Hh, Np, D = y.shape
    if Np != g.Np:
        raise ValueError("slot count does not match the padded grid")
    src = tile_slot_source(g)
    out = np.zeros((B, g.S, Hh, D), dtype=y.dtype)
    for p in range(g.Np):
        if src[p] >= 0:
            out[:, src[p], :, :] = y[:, :, p, :]
    return out


# --------------------------------------------------------------------------- block mass
def _softmax_rows(logits: np.ndarray) -> np.ndarray:
    z = logits - logits.max(axis=1, keepdims=True)
    e = np.exp(z)
    return e / e.sum(axis=1, keepdims=True)


def block_mass_row(qt, kt, g: Grid, b: int, h: int, i: int, q_block: int, kv_block: int,
                   scale: float) -> np.ndarray:
    """Mass of query block i of head (b, h) over every kv block: float64 [Np // kv_block].

    [LoSA] the block masses are measured exactly on one dense step; definition per
    reading R2.
    qt, kt: tile-major [B, Hh, Np, D] arrays (any float dtype; widened to float64).
    """
    valid = valid_slots(g)
    n_kb = g.Np // kv_block
    rows = np.arange(i * q_block, (i + 1) * q_block)
    rows = rows[valid[rows]]
    mass = np.zeros(n_kb, dtype=np.float64)
    if rows.size == 0:
        return mass
    keys = np.nonzero(valid)[0]
    q = qt[b, h, rows, :].astype(np.float64)
    k = kt[b, h, keys, :].astype(np.float64)
    p = _softmax_rows(scale * (q @ k.T))            # [nq, nkeys], rows sum to 1
    per_key = p.sum(axis=0)                         # summed over the block's queries
    np.add.at(mass, keys // kv_block, per_key)      # each key's mass into its block
    return mass / rows.size


def block_mass(qt, kt, g: Grid, q_block: int, kv_block: int, scale: float) -> np.ndarray:
    """All block masses, float64 [B, Hh, Np // q_block, Np // kv_block].  [LoSA], R2."""
    B, Hh = qt.shape[0], qt.shape[1]
    n_qb, n_kb = g.Np // q_block, g.Np // kv_block
    out = np.zeros((B, Hh, n_qb, n_kb), dtype=np.float64)
    for b in range(B):
        for h in range(Hh):
            for i in range(n_qb):
                out[b, h, i] = block_mass_row(qt, kt, g, b, h, i, q_block, kv_block, scale)
    return out


# --------------------------------------------------------------------------- top-p select
def fixed_point_masses(m_row) -> np.ndarray:
    """float32 masses -> int64 q = rint(m * 2^40) (exact: a power-of-two scale, then RNE)."""
    m = np.asarray(m_row, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(m)) or np.any(m < 0) or np.any(m > 4096.0):
        raise ValueError("masses must be finite and in [0, 4096]")
    return np.rint(m * FP_SCALE).astype(np.int64)


def topp_target(total: int, tau) -> int:
    """ceil(tau * total) with tau the float32 threshold widened to float64 (one multiply)."""
    return int(math.ceil(float(np.float64(np.float32(tau))) * float(np.float64(total))))


def topp_select_row(m_row, tau) -> np.ndarray:
    """Smallest kv-block set whose mass reaches tau of the row's total.

    [LoSA] per head and query block, the fewest kv blocks whose mass reaches the
    threshold; [SVG2] top-p budget control.
    Greedy on the descending order is minimal: any k blocks hold at most the k largest
    masses.  Ties between equal masses go to the lower block index (reading R3).
    Returns the kept block indices ascending (int64).
    """
    q = fixed_point_masses(m_row)
    target = topp_target(int(q.sum()), tau)
    order = sorted(range(q.size), key=lambda j: (-int(q[j]), j))
    acc, k = 0, 0
    while acc < target:
        acc += int(q[order[k]])
        k += 1
    return np.array(sorted(order[:k]), dtype=np.int64)


def topp_select(mass_rows, tau):
    """CSR (row_ptr int64 [R+1], col_idx int64 [nnz]) of the per-row selections."""
    mass_rows = np.asarray(mass_rows, dtype=np.float32)
    kept = [topp_select_row(r, tau) for r in mass_rows.reshape(-1, mass_rows.shape[-1])]
    row_ptr = np.zeros(len(kept) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(x) for x in kept])
    col_idx = np.concatenate(kept) if kept else np.zeros(0, np.int64)
    return row_ptr, col_idx.astype(np.int64)


# --------------------------------------------------------------------------- attention
def masked_attention_query(qt, kt, vt, g: Grid, b: int, h: int, p: int, q_block: int,
                           kv_block: int, row_ptr, col_idx, scale: float):
    """Output row and log-sum-exp of query slot p of head (b, h) over its kept blocks.

    [LoSA] attention over the frozen block lists; normalisation per reading R4.
    Returns (o float64 [D], lse float64); lse is natural-log units.
    """
    D = vt.shape[-1]
    valid = valid_slots(g)
    if not valid[p]:
        return np.zeros(D), -math.inf
    Hh = qt.shape[1]
    n_qb = g.Np // q_block
    r = (b * Hh + h) * n_qb + p // q_block
    blocks = np.asarray(col_idx[int(row_ptr[r]):int(row_ptr[r + 1])], dtype=np.int64)
    keys = (blocks[:, None] * kv_block + np.arange(kv_block)[None, :]).reshape(-1)
    keys = keys[valid[keys]]
    if keys.size == 0:
        return np.zeros(D), -math.inf
    q = qt[b, h, p, :].astype(np.float64)
    k = kt[b, h, keys, :].astype(np.float64)
    v = vt[b, h, keys, :].astype(np.float64)
    logits = scale * (k @ q)
    mx = logits.max()
    e = np.exp(logits - mx)
    z = e.sum()
    return (e / z) @ v, float(mx + math.log(z))


def masked_attention(qt, kt, vt, g: Grid, q_block, kv_block, row_ptr, col_idx, scale,
                     queries=None):
    """Output rows for a list of (b, h, p) query slots (all slots when None).

    Returns (o float64 [n, D], lse float64 [n]) in the order of `queries`, or the full
    tile-major (o [B, Hh, Np, D], lse [B, Hh, Np]) when queries is None.
    """
    B, Hh, Np, D = qt.shape
    full = queries is None
    if full:
        queries = [(b, h, p) for b in range(B) for h in range(Hh) for p in range(Np)]
    o = np.zeros((len(queries), D))
    lse = np.zeros(len(queries))
    for n, (b, h, p) in enumerate(queries):
        o[n], lse[n] = masked_attention_query(qt, kt, vt, g, b, h, p, q_block, kv_block,
                                              row_ptr, col_idx, scale)
    if full:
        return o.reshape(B, Hh, Np, D), lse.reshape(B, Hh, Np)
    return o, lse


# --------------------------------------------------------------------------- FP8 e4m3
def e4m3_decode_table() -> np.ndarray:
    """Value of each of the 256 e4m3 codes (OCP 8-bit floating point, E4M3 variant):
    1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits; exponent 0 is subnormal
    (m/8 * 2^-6); exponent 15 with mantissa 7 is NaN; there are no infinities."""
    out = np.zeros(256, dtype=np.float64)
    for c in range(256):
        sign = -1.0 if c >> 7 else 1.0
        e = (c >> 3) & 0xF
        m = c & 0x7
        if e == 0xF and m == 0x7:
            out[c] = math.nan
        elif e == 0:
            out[c] = sign * (m / 8.0) * 2.0 ** -6
        else:
            out[c] = sign * (1.0 + m / 8.0) * 2.0 ** (e - 7)
    return out


def e4m3_encode(x) -> np.ndarray:
    """float32 -> e4m3 code: round to nearest, ties to even code, saturate to +-448.

    The sign of a value that rounds to zero is kept (code 0x80 for negative zero).
    """
    x = np.asarray(x, dtype=np.float32).astype(np.float64)
    if not np.all(np.isfinite(x)):
        raise ValueError("non-finite input")
    table = e4m3_decode_table()
    mags = table[:127]                       # codes 0..126: 0 .. 448, increasing
    a = np.abs(x)
    a_sat = np.minimum(a, 448.0)
    hi = np.searchsorted(mags, a_sat, side="left")      # mags[hi-1] < a <= mags[hi]
    hi = np.minimum(hi, 126)
    exact = mags[hi] == a_sat
    lo = np.maximum(hi - 1, 0)
    d_lo = a_sat - mags[lo]
    d_hi = mags[hi] - a_sat
    pick_hi = (d_hi < d_lo) | ((d_hi == d_lo) & (hi % 2 == 0))
    code = np.where(exact, hi, np.where(pick_hi, hi, lo)).astype(np.uint8)
    neg = np.signbit(x)
    return np.where(neg, code | 0x80, code).astype(np.uint8)


def quant_e4m3_tiles(xt):
    """Per-(batch, head, 64-token tile) scale and e4m3 codes of a tile-major tensor.

    [FPS] FP8 with the 3D tile as the quantisation unit; reading R5.  xt is
    [B, Hh, Np, D] (pad slots zero).  Returns (codes uint8 [B, Hh, Np, D],
    scales float32 [B, Hh, Np // 64]).
    """
    x32 = np.asarray(xt, dtype=np.float32)
    B, Hh, Np, D = x32.shape
    tiles = x32.reshape(B, Hh, Np // TILE_TOKENS, TILE_TOKENS, D)
    absmax = np.abs(tiles).max(axis=(3, 4)).astype(np.float32)
    scales = np.where(absmax == 0, np.float32(1.0), absmax / np.float32(448.0)).astype(np.float32)
    y = (tiles / scales[..., None, None]).astype(np.float32)
    codes = e4m3_encode(y).reshape(B, Hh, Np, D)
    return codes, scales


def dequant_e4m3_tiles(codes, scales) -> np.ndarray:
    """codes [B, Hh, Np, D] and scales [B, Hh, Np // 64] -> float64 values."""
    table = e4m3_decode_table()
    v = table[np.asarray(codes, dtype=np.int64)]
    B, Hh, Np, D = v.shape
    s = np.repeat(np.asarray(scales, dtype=np.float64), TILE_TOKENS, axis=2)
    return v * s[..., None]


# --------------------------------------------------------------------------- static patterns
# "Sparse-vDiT: Unleashing the Power of Sparse Attention to Accelerate Video Diffusion
# Transformers", Abstract: recurring diagonal, multi-diagonal and vertical-stripe attention
# structures.  "GRAT" (grouping attention for large images/videos), Abstract: queries of a
# group share keys restricted to surrounding blocks or to criss-cross regions.
#
# Readings (the pages name the structures only): everything is at kv-block (= tile)
# granularity in tile-major order; a query block covers its own tiles (one for 64-token
# blocks, two for 128-token blocks) and keeps kv block j when the predicate holds for any
# of them.
#   DIAGONAL        |j - u| <= w
#   MULTI_DIAGONAL  |j - (u + k L)| <= w for some k in [-K, K], k != 0; L defaults to the
#                   tiles of one temporal layer (Hp/4 * Wp/4): the same place in other frames
#   VERTICAL_STRIPE j % stride == offset (the same kv blocks for every query block)
#   SURROUNDING     |jt - ut| <= rt and |jh - uh| <= rh and |jw - uw| <= rw (tile coords)
#   CRISS_CROSS     tile j shares at least two of its three tile coordinates with u
# The kept set is the union over the enabled kinds.
PAT_DIAGONAL = 1
PAT_MULTI_DIAGONAL = 2
PAT_VERTICAL_STRIPE = 4
PAT_SURROUNDING = 8
PAT_CRISS_CROSS = 16


def _tile_coords(g: Grid, j: int):
    nth, ntw = g.Hp // TILE, g.Wp // TILE
    return j // (nth * ntw), (j // ntw) % nth, j % ntw


def pattern_keeps(g: Grid, q_block: int, i: int, j: int, kinds: int, diag_width=0,
                  multi_count=0, multi_period=0, stripe_stride=0, stripe_offset=0,
                  radius=(0, 0, 0)) -> bool:
    """Whether query block i keeps kv block j under the enabled structured patterns."""
    per = q_block // TILE_TOKENS
    L = multi_period if multi_period > 0 else (g.Hp // TILE) * (g.Wp // TILE)
    jt, jh, jw = _tile_coords(g, j)
    if kinds & PAT_VERTICAL_STRIPE and stripe_stride > 0 and j % stripe_stride == stripe_offset:
        return True
    for u in range(i * per, (i + 1) * per):
        if kinds & PAT_DIAGONAL and abs(j - u) <= diag_width:
            return True
        if kinds & PAT_MULTI_DIAGONAL:
            for k in range(-multi_count, multi_count + 1):
                if k != 0 and abs(j - (u + k * L)) <= diag_width:
                    return True
        ut, uh, uw = _tile_coords(g, u)
        if kinds & PAT_SURROUNDING and abs(jt - ut) <= radius[0] and abs(jh - uh) <= radius[1] \
                and abs(jw - uw) <= radius[2]:
            return True
        if kinds & PAT_CRISS_CROSS and (int(jt == ut) + int(jh == uh) + int(jw == uw)) >= 2:
            return True
    return False


def pattern_csr(g: Grid, q_block: int, batch: int, heads: int, kinds: int, **params):
    """CSR (row_ptr, col_idx) of the structured pattern, identical for every (b, h)."""
    n_qb, n_kb = g.Np // q_block, g.Np // 64
    rows = []
    for i in range(n_qb):
        rows.append([j for j in range(n_kb) if pattern_keeps(g, q_block, i, j, kinds, **params)])
    kept = [r for _ in range(batch * heads) for r in rows]
    row_ptr = np.zeros(len(kept) + 1, dtype=np.int64)
    row_ptr[1:] = np.cumsum([len(r) for r in kept])
    col_idx = np.array([j for r in kept for j in r], dtype=np.int64)
    return row_ptr, col_idx


# --------------------------------------------------------------------------- pooled estimate
# "Sparse VideoGen2", Abstract: top-p dynamic budget control over cluster-level attention;
# the related-work entry on head-wise adaptive sparse attention (online top-p).  Reading R8:
# with the 4x4x4 tiles as the clusters, a kv block is represented by the mean of its valid
# keys and weighted by its number of valid keys, a query block by the mean of its valid
# queries, and the estimated block mass is the softmax over kv blocks of those block-level
# logits, each weighted by its key count:
#   M_est[i, j] = n_j exp(scale qbar_i . kbar_j) / sum_j' n_j' exp(scale qbar_i . kbar_j')
# Blocks without valid keys get 0; query blocks without valid queries get an all-zero row.
def pooled_block_mass(qt, kt, g: Grid, q_block: int, kv_block: int, scale: float) -> np.ndarray:
    """Estimated block masses float64 [B, Hh, Np // q_block, Np // kv_block] (reading R8)."""
    B, Hh = qt.shape[0], qt.shape[1]
    valid = valid_slots(g)
    n_qb, n_kb = g.Np // q_block, g.Np // kv_block
    out = np.zeros((B, Hh, n_qb, n_kb), dtype=np.float64)
    n_keys = np.array([valid[j * kv_block:(j + 1) * kv_block].sum() for j in range(n_kb)], float)
    for b in range(B):
        for h in range(Hh):
            k = kt[b, h].astype(np.float64)
            kbar = np.zeros((n_kb, k.shape[-1]))
            for j in range(n_kb):
                rows = np.arange(j * kv_block, (j + 1) * kv_block)
                rows = rows[valid[rows]]
                if rows.size:
                    kbar[j] = k[rows].mean(axis=0)
            q = qt[b, h].astype(np.float64)
            for i in range(n_qb):
                rows = np.arange(i * q_block, (i + 1) * q_block)
                rows = rows[valid[rows]]
                if rows.size == 0:
                    continue
                qbar = q[rows].mean(axis=0)
                logits = scale * (kbar @ qbar)
                keep = n_keys > 0
                z = logits[keep] - logits[keep].max()
                w = n_keys[keep] * np.exp(z)
                out[b, h, i, keep] = w / w.sum()
    return out


# --------------------------------------------------------------------------- semantic clusters
# "Sparse VideoGen2", Abstract: semantic-aware permutation -- tokens are clustered by
# k-means on their vectors and reordered so that each cluster is contiguous, with no
# padding; cluster representatives identify the critical clusters (top-p dynamic budget
# control) and the attention runs over the densified layout.  Reading R10:
#   * per (batch, head), queries and keys are clustered separately by Lloyd's k-means from
#     given initial centroids for a fixed number of rounds; a round assigns every token to
#     the nearest centroid (squared Euclidean distance, ties to the lowest index) and then
#     replaces each centroid by the mean of its tokens (an empty cluster keeps its centroid);
#   * the assignment is the definition itself: squared Euclidean distance sum_d (x_d - c_d)^2
#     in float64, first minimum (lowest index) on ties; the means are float64 too.  A
#     device computing the distance in lower precision may pick another centroid only
#     where two distances agree to that precision: tests compare labels where the oracle's
#     minimum is unique at the device's precision and check the others for validity;
#   * cluster order: clusters by index, tokens of one cluster in their raster order;
#   * cluster-level estimate as in R8 with clusters for tiles: weights n_j exp(s qc_i . kc_j)
#     over the key clusters, normalised per query cluster (qc, kc the final centroids);
#   * the selection is R3 applied to those rows; a query token attends to every key of the
#     key clusters selected for its cluster, softmax renormalised over them (R4).
def kmeans_distances(x, centroids) -> np.ndarray:
    """Squared Euclidean distance [N, C] of every row of x to every centroid, float64,
    summed over the coordinates as written in the definition."""
    x = np.asarray(x, dtype=np.float64)
    c = np.asarray(centroids, dtype=np.float64)
    d = np.empty((x.shape[0], c.shape[0]))
    for j in range(c.shape[0]):
        diff = x - c[j][None, :]
        d[:, j] = (diff * diff).sum(axis=1)
    return d


def kmeans_assign(x, centroids) -> np.ndarray:
    """Nearest centroid of every row of x (reading R10): the first minimum of the float64
    squared distances, i.e. the lowest index among equidistant centroids."""
    return np.argmin(kmeans_distances(x, centroids), axis=1).astype(np.int64)


def kmeans_lloyd(x, init, rounds: int):
    """(labels, centroids float64 [C, D], counts) after `rounds` assign-then-update rounds."""
    x = np.asarray(x, dtype=np.float64)
    c = np.array(init, dtype=np.float64)
    labels = np.zeros(x.shape[0], dtype=np.int64)
    for _ in range(rounds):
        labels = kmeans_assign(x, c)
        for j in range(c.shape[0]):
            member = labels == j
            if member.any():
                c[j] = x[member].mean(axis=0)
    counts = np.bincount(labels, minlength=c.shape[0])
    return labels, c, counts


def cluster_layout(labels, n_clusters: int):
    """(starts, token_of_slot, slot_of_token): clusters in index order, tokens of a cluster
    in raster order (a stable sort by cluster id)."""
    labels = np.asarray(labels, dtype=np.int64)
    counts = np.bincount(labels, minlength=n_clusters)
    starts = np.concatenate([[0], np.cumsum(counts)[:-1]]).astype(np.int64)
    token_of_slot = np.argsort(labels, kind="stable").astype(np.int64)
    slot_of_token = np.empty_like(token_of_slot)
    slot_of_token[token_of_slot] = np.arange(labels.size)
    return starts, token_of_slot, slot_of_token


def cluster_mass(qc, q_counts, kc, k_counts, scale: float) -> np.ndarray:
    """Estimated mass [Cq, Ck] of key cluster j for query cluster i (reading R10)."""
    qc = np.asarray(qc, dtype=np.float64)
    kc = np.asarray(kc, dtype=np.float64)
    nk = np.asarray(k_counts, dtype=np.float64)
    out = np.zeros((qc.shape[0], kc.shape[0]))
    keep = nk > 0
    if not keep.any():
        return out
    for i in range(qc.shape[0]):
        if q_counts[i] == 0:
            continue
        logits = scale * (kc[keep] @ qc[i])
        w = nk[keep] * np.exp(logits - logits.max())
        out[i, keep] = w / w.sum()
    return out


def cluster_attention(q, k, v, q_starts, q_counts, k_starts, k_counts, row_ptr, col_idx,
                      scale: float, rows=None) -> np.ndarray:
    """Attention in cluster order [S, D]: the queries of cluster i attend to the keys of the
    key clusters col_idx[row_ptr[i]:row_ptr[i+1]] (reading R10).  `rows` restricts the
    computation to those query slots (others stay zero)."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    out = np.zeros((q.shape[0], v.shape[1]))
    want = None if rows is None else set(int(r) for r in rows)
    for i in range(len(q_starts)):
        keys = np.concatenate([np.arange(k_starts[j], k_starts[j] + k_counts[j])
                               for j in col_idx[row_ptr[i]:row_ptr[i + 1]]] or [np.zeros(0, int)])
        keys = keys.astype(np.int64)
        for p in range(int(q_starts[i]), int(q_starts[i] + q_counts[i])):
            if want is not None and p not in want:
                continue
            if keys.size == 0:
                continue
            logits = scale * (k[keys] @ q[p])
            w = np.exp(logits - logits.max())
            out[p] = (w / w.sum()) @ v[keys]
    return out
