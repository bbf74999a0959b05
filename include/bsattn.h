/*
 * bsattn.h -- C ABI of libbsattn.so: retained-mass block-sparse self-attention over a
 * long 3D video token sequence, written for NVIDIA B200 (sm_100a).
 *
 * The method: one dense calibration call measures the exact softmax attention mass of
 * every (head, query block, key/value block) pair; for each head and query block the
 * smallest key/value block set whose mass reaches a threshold (99% by default) is kept;
 * later calls attend only over those frozen block lists.
 *   - "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion
 *     Acceleration", Abstract (masses, threshold, frozen lists).
 *   - "FPSAttention: Training-Aware FP8 and Sparsity Co-Design for Fast Video
 *     Diffusion", Abstract, innovation 1 (the 3D tile as the unit of sparsity and of
 *     the FP8 scale).
 *   - "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via
 *     Semantic-Aware Permutation", Abstract (top-p dynamic budget control).
 *
 * Conventions shared by every call
 *   - Every tensor pointer is a DEVICE pointer owned by the caller.  The library
 *     allocates no memory and keeps no global state (the one exception is the fixed
 *     scratch array of bsa_topp_select_noalloc, below); scratch space is the caller's
 *     workspace (`ws`), sized by bsa_workspace_bytes().  A workspace serves one call at a
 *     time: calls that may overlap (other streams) need workspaces of their own.
 *   - Every call is asynchronous and ordered on `stream` (NULL = legacy default
 *     stream).  A call returns after launching; results are ready when the stream is.
 *   - Arguments are checked on the host before anything is launched.  A bad argument
 *     returns a non-zero status and launches nothing.  Checks that need device data
 *     (CSR contents, mass values, pipeline time limits) set bits in the status word at
 *     the head of the workspace; read them with bsa_device_status().
 *   - Errors cross the ABI only as bsa_status codes: no exceptions, no printing, no
 *     exit, no trap.
 *   - Layouts.  raster: [B, S, Hh, D] with S = T*H*W and token s = (t*H + h)*W + w.
 *     tile-major: [B, Hh, Np, D] with Np = Tp*Hp*Wp; slot p = tile*64 + inner, where
 *     tile = ((t/4)*(Hp/4) + h/4)*(Wp/4) + w/4 and inner = ((t%4)*4 + h%4)*4 + w%4.
 *     Slots outside the valid T x H x W grid are pad slots.  Query block i is slots
 *     [i*q_block, (i+1)*q_block); kv block j is slots [j*64, (j+1)*64), one tile.
 *   - Sizes: head_dim in {64, 128}; q_block in {64, 128}; kv_block = 64; Tp, Hp, Wp
 *     multiples of 4 covering T, H, W; B*Hh*Np*D < 2^31 elements per tensor is not
 *     required (64-bit offsets are used), but B*Hh*(Np/q_block) rows must fit int32.
 *     Also Np = Tp*Hp*Wp < 2^30 and a multiple of q_block, at most 4096 kv blocks per head
 *     (Np/64 <= 4096), and R*(Np/64) < 2^31 with R = B*Hh*(Np/q_block) (CSR offsets are
 *     int32).  Inconsistent extents (a size below 1, a padded extent below its valid one
 *     or not a multiple of 4, Np not a multiple of q_block) return BSA_ERR_INVALID_ARG;
 *     a consistent shape beyond these limits returns BSA_ERR_UNSUPPORTED; either way
 *     bsa_workspace_bytes gives 0.
 *   - Pointers to bf16 / fp32 / e4m3 tensors must be 16-byte aligned.
 */
#ifndef BSATTN_H
#define BSATTN_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define BSA_API __attribute__((visibility("default")))
#else
#define BSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* bsa_stream_t;

typedef enum {
  BSA_OK = 0,
  BSA_ERR_INVALID_ARG = 1,   /* null pointer, bad size, bad alignment, bad threshold */
  BSA_ERR_UNSUPPORTED = 2,   /* shape outside the supported set (head_dim, block sizes) */
  BSA_ERR_CAPACITY = 3,      /* workspace or col_idx capacity too small */
  BSA_ERR_CUDA = 4,          /* a CUDA runtime / driver call failed */
  BSA_ERR_TIMEOUT = 5,       /* a device pipeline wait hit its time limit and gave up */
  BSA_ERR_DEVICE_INPUT = 6,  /* device data failed a check (CSR order/range, mass values) */
  BSA_ERR_IO = 7             /* a list file is missing, unwritable, truncated or corrupt */
} bsa_status;

typedef enum { BSA_BF16 = 0, BSA_FP32 = 1, BSA_E4M3 = 2 } bsa_dtype;

typedef enum {
  BSA_OP_BLOCK_MASS = 0,
  BSA_OP_TOPP_SELECT = 1,
  BSA_OP_FWD = 2,
  BSA_OP_PATTERN = 3,
  BSA_OP_POOLED_MASS = 4
} bsa_op;

/* Structured kv-block patterns for bsa_pattern_csr (bit flags, combined by union). */
typedef enum {
  BSA_PAT_DIAGONAL = 1,         /* |j - u| <= diag_width                                   */
  BSA_PAT_MULTI_DIAGONAL = 2,   /* |j - (u + k*L)| <= diag_width, 0 < |k| <= multi_count   */
  BSA_PAT_VERTICAL_STRIPE = 4,  /* j % stripe_stride == stripe_offset, for every row        */
  BSA_PAT_SURROUNDING = 8,      /* tile of j within (radius_t, radius_h, radius_w) of u     */
  BSA_PAT_CRISS_CROSS = 16      /* tile of j shares at least two tile coordinates with u    */
} bsa_pattern_kind;

typedef struct {
  uint32_t kinds;               /* OR of bsa_pattern_kind */
  int32_t diag_width;           /* half width of every diagonal band, in blocks (>= 0) */
  int32_t multi_count;          /* extra diagonals on each side (>= 0) */
  int32_t multi_period;         /* L in blocks; <= 0 means the tiles of one temporal layer */
  int32_t stripe_stride;        /* > 0 enables stripes */
  int32_t stripe_offset;        /* 0 <= offset < stride */
  int32_t radius_t, radius_h, radius_w;  /* >= 0, in tiles */
} bsa_pattern;

typedef struct {
  int32_t batch, heads, head_dim; /* B, Hh, D */
  int32_t T, H, W;                /* valid token grid */
  int32_t Tp, Hp, Wp;             /* padded grid, multiples of 4 */
  int32_t q_block, kv_block;      /* tokens per query block (64 | 128), per kv block (64) */
} bsa_shape;

/* Bytes of workspace that `op` needs for `shape` (0 on an invalid shape).  Every
 * workspace starts with a 256-byte status header; the rest is scratch whose contents
 * do not persist meaningfully between calls. */
BSA_API size_t bsa_workspace_bytes(const bsa_shape* shape, int op);

/* Zero the status header of a workspace (stream-ordered).  Call once before the first
 * use of a workspace and after reading an error. */
BSA_API bsa_status bsa_clear_status(void* ws, bsa_stream_t stream);

/* Synchronise `stream`, then report the status header of `ws`: BSA_OK, or the first
 * error class recorded by a device-side check (TIMEOUT before DEVICE_INPUT before
 * CAPACITY).  The header is left as it is. */
BSA_API bsa_status bsa_device_status(const void* ws, bsa_stream_t stream);

/* Raw status header words (flags, detail) for diagnostics; synchronises `stream`. */
BSA_API bsa_status bsa_device_status_words(const void* ws, uint32_t out_words[4], bsa_stream_t stream);

BSA_API const char* bsa_status_string(bsa_status status);

/* The compute capability the library's kernels were compiled for, as the CUDA runtime
 * reports it for a kernel of the loaded library (cudaFuncGetAttributes binaryVersion:
 * major*10 + minor, 100 for sm_100a).  Needs a CUDA device; BSA_ERR_CUDA otherwise. */
BSA_API bsa_status bsa_kernel_binary_version(int32_t* version);

/* 3D tile permutation ("FPSAttention", Abstract, innovation 1: unified 3D tile-wise
 * granularity).  inverse = 0: raster src [B,S,Hh,D] -> tile-major dst [B,Hh,Np,D],
 * pad slots written as zero.  inverse = 1: tile-major src -> raster dst, pad slots
 * dropped.  dtype BSA_BF16 or BSA_FP32 (elements copied bit for bit).  src and dst
 * must not overlap. */
BSA_API bsa_status bsa_tile_permute(const bsa_shape* shape, bsa_dtype dtype, int inverse,
                            const void* src, void* dst, bsa_stream_t stream);

/* Permutation fused with per-tile FP8 quantisation ("FPSAttention", Abstract: FP8
 * quantisation at the 3D tile granularity).  src: raster bf16 [B,S,Hh,D].  dst:
 * tile-major e4m3 codes [B,Hh,Np,D].  tile_scales: fp32 [B,Hh,Np/64], one per
 * (batch, head, 64-token tile): s = absmax/448 in fp32 (1 when the tile is all zero);
 * code = e4m3 round-to-nearest-even, saturating, of x/s computed in fp32. */
BSA_API bsa_status bsa_tile_permute_quant_e4m3(const bsa_shape* shape, const void* src_bf16,
                                       uint8_t* dst, float* tile_scales, bsa_stream_t stream);

/* Exact block attention masses at a dense step ("LoSA", Abstract: the masses of all
 * block pairs are measured exactly on one early step that runs dense attention).  q, k: tile-major bf16 [B,Hh,Np,D] with
 * zero pad slots.  mass: fp32 [B,Hh,Np/q_block,Np/64]; mass[b,h,i,j] is the mean over
 * the valid queries of block i of the softmax(softmax_scale * q.k) probability on the
 * valid keys of block j (pad keys excluded).  Rows of a block with no valid query are
 * zero.  One dense pass on tcgen05 tensor cores: every probability computed once against a
 * lazily raised reference max, unnormalised block sums per row kept in the workspace and
 * normalised by the row sums at the end.  Workspace: bsa_workspace_bytes(shape, BSA_OP_BLOCK_MASS) -- the
 * status header, a 256-byte slice pool, and 192 slices of 256 x Np/64 fp32, each held by
 * one live CTA at a time (claimed from the pool when the CTA starts, freed when it ends). */
BSA_API bsa_status bsa_block_mass(const bsa_shape* shape, const void* q, const void* k,
                          float softmax_scale, float* mass, void* ws, size_t ws_bytes,
                          bsa_stream_t stream);

/* Fused calibration step: the dense attention output and the exact block masses in one
 * call ("LoSA", Abstract: the calibration step is a dense attention step on which the
 * block masses are measured).  One dense pass: each probability is formed once (against a
 * lazily raised reference max, O rescaled when it moves) and used for both the masses (as
 * bsa_block_mass) and out = P V.  q, k, v: tile-major bf16 [B,Hh,Np,D].  out: bf16
 * tile-major (pad query slots zero); lse (nullable): fp32 [B,Hh,Np] natural log; mass:
 * fp32 [B,Hh,Np/q_block,Np/64].  Workspace as for BSA_OP_BLOCK_MASS. */
BSA_API bsa_status bsa_dense_fwd_mass(const bsa_shape* shape, const void* q, const void* k,
                                      const void* v, float softmax_scale, void* out, float* lse,
                                      float* mass, void* ws, size_t ws_bytes,
                                      bsa_stream_t stream);

/* Pooled estimate of the block masses, for per-step ("online") selection without a dense
 * pass ("Sparse VideoGen2", Abstract: top-p dynamic budget control on attention between
 * token clusters).  With the 4x4x4 tiles as clusters: qbar_i = mean of the valid queries
 * of query block i, kbar_j = mean of the valid keys of kv block j, n_j = its valid keys;
 * mass_est[b,h,i,j] = n_j exp(s qbar_i.kbar_j) / sum_j' n_j' exp(s qbar_i.kbar_j'), with
 * s = softmax_scale; 0 for blocks without valid keys; zero rows for query blocks without
 * valid queries.  Feed the result to bsa_topp_select.  q, k: tile-major bf16; mass_est:
 * fp32 [B,Hh,Np/q_block,Np/64].  Workspace: bsa_workspace_bytes(shape,
 * BSA_OP_POOLED_MASS). */
BSA_API bsa_status bsa_pooled_mass(const bsa_shape* shape, const void* q, const void* k,
                                   float softmax_scale, float* mass_est, void* ws,
                                   size_t ws_bytes, bsa_stream_t stream);

/* Retained-mass (top-p) block selection ("LoSA", Abstract: per head and query block,
 * the fewest kv blocks whose mass reaches the threshold are kept; "Sparse VideoGen2",
 * Abstract: top-p dynamic budget control).  mass: fp32 [R, Np/64] with
 * R = B*Hh*(Np/q_block), values finite in [0, 4096] (others are flagged DEVICE_INPUT and
 * count as 0) with each row summing to less than 2^22 (block masses are probabilities; a
 * row sums to 1).  Per row, masses become integers
 * q = rint(m * 2^40); target = ceil(threshold * sum q) (one fp64 multiply); blocks are
 * ranked by (q desc, index asc) and the shortest prefix reaching the target is kept.
 * Output CSR: row_ptr int32 [R+1] (row_ptr[0] = 0), col_idx int32 ascending within a
 * row.  threshold in (0, 1].  col_capacity = entries available at col_idx; R*(Np/64)
 * always suffices.  If the selection needs more, row_ptr is still complete, col_idx
 * holds what fits and the status header records CAPACITY. */
BSA_API bsa_status bsa_topp_select(const bsa_shape* shape, const float* mass, float threshold,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                           void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Allocation-free variant of bsa_topp_select.  No counterpart in the papers: this is an
 * interface for callers that cannot give the library a workspace -- for example a plugin
 * inside a serving engine whose memory planner owns all device memory and forbids ad-hoc
 * cudaMalloc, or code on a latency-critical path where cudaMalloc's implicit device
 * synchronisation would stall the stream.  Inputs, outputs and results are exactly those
 * of bsa_topp_select; only the scratch (per-row counts and kept bitmaps) differs: it lives
 * in a fixed 16 MiB array in the library's own device memory, which every GPU that loads
 * the library holds until the process exits.  This call allocates nothing (no cudaMalloc,
 * no cudaFree, no allocating library routine).
 *   - Size limit: R*4 rounded up to 256 bytes, plus R*ceil((Np/64)/32)*4 bytes, must fit in
 *     16 MiB (R = B*Hh*Np/q_block); larger problems return BSA_ERR_CAPACITY and launch
 *     nothing.  The 720p 40-head shape needs 10.6 MB.
 *   - Set-up: the array's device address depends on the CUDA context (each context that
 *     loads the library has its own copy, and a device reset reloads it elsewhere), so the
 *     first call in each context -- the device's primary context, a driver-API context of
 *     the caller's own, or the new context after a device reset -- looks the address up
 *     (cudaGetSymbolAddress, with that context current) and caches it under the context's
 *     unique ID.  Make that first call before any stream capture.
 *   - Every call shares the one array and leaves its contents behind; each call rewrites
 *     all of the scratch it reads, so nothing needs clearing, but calls that overlap on the
 *     GPU (different streams, or several host threads) race on it and must be serialised
 *     by the caller.
 *   - status: null, or a caller-owned device buffer of 4 uint32 words that receives the
 *     device-side flags (same encoding as a workspace status header; zero it first). */
BSA_API bsa_status bsa_topp_select_noalloc(const bsa_shape* shape, const float* mass,
                                           float threshold, int32_t* row_ptr, int32_t* col_idx,
                                           int64_t col_capacity, uint32_t* status,
                                           bsa_stream_t stream);

/* Frozen lists on disk ("LoSA", Abstract: the block indices selected at the calibration
 * step are frozen and reused for all remaining steps -- they are the method's only state,
 * so a run can resume after the calibration with the very same lists).  HOST pointers,
 * owned by the caller; these calls touch no device memory and launch nothing.
 * File: magic "BSALISTS", version 1, the bsa_shape, the threshold (float32, kept for the
 * record), R and nnz (int64), row_ptr int32 [R+1], col_idx int32 [nnz], then a 64-bit
 * FNV-1a hash of everything before it; little-endian.
 *   bsa_lists_save: row_ptr [R+1] and col_idx [row_ptr[R]] as a selection produces them
 *     (row_ptr[0] = 0, non-decreasing, each row's indices strictly ascending in
 *     [0, Np/64)), else BSA_ERR_INVALID_ARG; written to `path`.tmp and renamed, so `path`
 *     never holds half a file; BSA_ERR_IO if it cannot be written.
 *   bsa_lists_read_header: the stored shape, threshold and nnz (any output may be NULL),
 *     so the caller can size col_idx.
 *   bsa_lists_load: `shape` must equal the stored one (else BSA_ERR_INVALID_ARG) and
 *     col_capacity >= nnz (else BSA_ERR_CAPACITY); a missing, truncated, altered (hash) or
 *     malformed file returns BSA_ERR_IO.  The caller's buffers are written only on
 *     BSA_OK. */
BSA_API bsa_status bsa_lists_save(const char* path, const bsa_shape* shape, float threshold,
                                  const int32_t* row_ptr, const int32_t* col_idx);
BSA_API bsa_status bsa_lists_read_header(const char* path, bsa_shape* shape, float* threshold,
                                         int64_t* nnz);
BSA_API bsa_status bsa_lists_load(const char* path, const bsa_shape* shape, float* threshold,
                                  int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity);

/* Static structured kv-block lists ("Sparse-vDiT", Abstract: diagonal, multi-diagonal and
 * vertical-stripe attention structures; "GRAT", Abstract: key regions restricted to
 * surrounding blocks or criss-cross lines).  Blocks are 4x4x4 tiles in tile-major order;
 * u ranges over the tile(s) of query block i (one for q_block 64, two for 128); kv block j
 * is kept when any enabled kind holds for some u.  Output CSR as bsa_topp_select (same
 * lists for every batch and head; ascending within a row).  Workspace:
 * bsa_workspace_bytes(shape, BSA_OP_PATTERN). */
BSA_API bsa_status bsa_pattern_csr(const bsa_shape* shape, const bsa_pattern* pattern,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Block-sparse attention forward over frozen CSR block lists ("LoSA", Abstract: the
 * frozen block indices are reused for all remaining steps).  For each query slot of
 * row r = (b*Hh + h)*(Np/q_block) + p/q_block: softmax(softmax_scale * q.k) over the
 * valid keys of the kv blocks col_idx[row_ptr[r] .. row_ptr[r+1]) only, times v.
 * q, k, v: tile-major [B,Hh,Np,D]; dtype BSA_BF16 (q_scales etc. NULL) or BSA_E4M3
 * (codes plus fp32 per-tile scales [B,Hh,Np/64] from bsa_tile_permute_quant_e4m3).
 * col_idx must be strictly ascending within each row and < Np/64 (checked on the
 * device; violations set DEVICE_INPUT and the row attends to the set of its indices).
 * out: bf16 tile-major [B,Hh,Np,D]; pad query slots and rows with no kept valid key
 * are written as zero.  lse (nullable): fp32 [B,Hh,Np], natural-log log-sum-exp of
 * the kept logits (-inf where out is zero). */
BSA_API bsa_status bsa_fwd(const bsa_shape* shape, bsa_dtype dtype,
                   const void* q, const void* k, const void* v,
                   const float* q_scales, const float* k_scales, const float* v_scales,
                   const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale,
                   void* out, float* lse, void* ws, size_t ws_bytes, bsa_stream_t stream);

/* ------------------------------------------------------------------------------------
 * Semantic-aware permutation ("Sparse VideoGen2: Accelerate Video Generation with Sparse
 * Attention via Semantic-Aware Permutation", Abstract: tokens are clustered by k-means on
 * their vectors and reordered so that every cluster is contiguous, without padding; the
 * cluster representatives identify the critical clusters under top-p budget control, and
 * the attention runs on the densified layout).  Per (batch, head), queries and keys are
 * clustered separately: n_q_clusters query clusters, n_k_clusters key clusters.
 *
 * Layouts: raster tokens [B, S, Hh, D] bf16; cluster order [B, Hh, S, D] bf16, where the
 * tokens of cluster c of head (b, h) occupy slots [starts[b,h,c], starts + counts) in
 * raster order; per-head int32 arrays [B, Hh, S] or [B, Hh, C]; centroids fp32
 * [B, Hh, C, D].  All pointers are device pointers owned by the caller; tensors of bf16
 * rows must be 16-byte aligned, int32 and fp32 arrays 4-byte aligned. */
/* Limits: batch, heads >= 1 (else BSA_ERR_INVALID_ARG, as for a size below 1); head_dim,
 * n_tokens and the cluster counts as below, B*Hh*S*(D/8) < 2^31 and
 * B*Hh*n_q_clusters*n_k_clusters < 2^31 (flat indices fit 31 bits), else
 * BSA_ERR_UNSUPPORTED; the workspace-size calls give 0 for a shape outside them. */
typedef struct {
  int32_t batch, heads;
  int32_t head_dim;                    /* 64 or 128 */
  int32_t n_tokens;                    /* S, 1 .. 2^24 */
  int32_t n_q_clusters, n_k_clusters;  /* 1 .. 1024 each */
} bsa_cluster_shape;

/* Bytes of workspace for bsa_kmeans / bsa_cluster_layout with n_clusters clusters. */
BSA_API size_t bsa_kmeans_workspace_bytes(const bsa_cluster_shape* shape, int32_t n_clusters);
/* Bytes of workspace for bsa_cluster_fwd. */
BSA_API size_t bsa_cluster_fwd_workspace_bytes(const bsa_cluster_shape* shape);
/* Bytes of workspace for bsa_topp_select_rows. */
BSA_API size_t bsa_topp_rows_workspace_bytes(int64_t rows, int32_t cols);

/* Lloyd's k-means over the S tokens of every (batch, head), `rounds` rounds of: assign
 * every token to the nearest centroid (argmin_c |c|^2 - 2 x.c in fp32, ties to the lowest
 * c), then replace every centroid by the mean of its tokens, summed in cluster order in
 * fp32 (deterministic); a cluster with no token keeps its centroid.  x: raster bf16.
 * centroids: in = initial, out = final (the means of the last assignment).  labels:
 * int32 [B, Hh, S], the last assignment; counts: int32 [B, Hh, n_clusters]. */
BSA_API bsa_status bsa_kmeans(const bsa_cluster_shape* shape, int32_t n_clusters, const void* x,
                              int32_t rounds, float* centroids, int32_t* labels, int32_t* counts,
                              void* ws, size_t ws_bytes, bsa_stream_t stream);

/* Cluster order of every (batch, head) from labels in [0, n_clusters): counts, starts
 * (exclusive scan of counts), token_of_slot [B,Hh,S] (raster token held by each slot; -1
 * for slots left over by out-of-range labels, which raise DEVICE_INPUT) and slot_of_token
 * [B,Hh,S] (-1 for such tokens).  A stable counting sort: tokens of a cluster keep their
 * raster order. */
BSA_API bsa_status bsa_cluster_layout(const bsa_cluster_shape* shape, int32_t n_clusters,
                                      const int32_t* labels, int32_t* counts, int32_t* starts,
                                      int32_t* token_of_slot, int32_t* slot_of_token, void* ws,
                                      size_t ws_bytes, bsa_stream_t stream);

/* Row gather into cluster order (inverse = 0): dst[b,h,p,:] = src[b, token_of_slot[b,h,p],
 * h, :] (zeros for a -1 slot); or scatter back (inverse = 1): dst[b, token_of_slot[b,h,p],
 * h, :] = src[b,h,p,:] (raster rows no slot points at are left untouched). */
BSA_API bsa_status bsa_cluster_permute(const bsa_cluster_shape* shape, int inverse,
                                       const int32_t* token_of_slot, const void* src, void* dst,
                                       bsa_stream_t stream);

/* Cluster-level estimate of the attention mass, to feed bsa_topp_select_rows:
 * mass[b,h,i,j] = n_j exp(s qc_i.kc_j) / sum_j' n_j' exp(s qc_i.kc_j') with s =
 * softmax_scale, qc/kc the query/key centroids (fp32 [B,Hh,C,D]) and n_j = k_counts; 0
 * for key clusters without tokens; zero rows for query clusters without tokens.
 * mass: fp32 [B, Hh, n_q_clusters, n_k_clusters]. */
BSA_API bsa_status bsa_cluster_mass(const bsa_cluster_shape* shape, const float* q_centroids,
                                    const int32_t* q_counts, const float* k_centroids,
                                    const int32_t* k_counts, float softmax_scale, float* mass,
                                    bsa_stream_t stream);

/* bsa_topp_select on any rows x cols fp32 matrix (same rule, same precondition on the
 * values): CSR of the smallest column set of each row reaching threshold of its mass.
 * cols <= 4096, rows * cols < 2^31. */
BSA_API bsa_status bsa_topp_select_rows(const float* mass, int64_t rows, int32_t cols,
                                        float threshold, int32_t* row_ptr, int32_t* col_idx,
                                        int64_t col_capacity, void* ws, size_t ws_bytes,
                                        bsa_stream_t stream);

/* Attention in cluster order: every query of cluster i of head (b, h) attends to all keys
 * of the key clusters col_idx[row_ptr[r] .. row_ptr[r+1]), r = (b*Hh + h)*n_q_clusters + i
 * (strictly ascending, < n_k_clusters; checked on the device), softmax(softmax_scale q.k)
 * renormalised over those keys.  q, k, v: cluster order bf16 [B,Hh,S,D] (q by the query
 * clustering, k and v by the key clustering); q_starts/q_counts and k_starts/k_counts:
 * int32 [B,Hh,C] cluster extents (checked to lie inside [0, S) on the device).  out: bf16
 * cluster order [B,Hh,S,D]; lse (nullable) fp32 [B,Hh,S]; rows of a cluster with no kept
 * key are zero (lse -inf).  The tensor-core kernel of bsa_fwd, walking each selected key
 * cluster in runs of <= 64 keys that start at the cluster's first slot. */
BSA_API bsa_status bsa_cluster_fwd(const bsa_cluster_shape* shape, const void* q, const void* k,
                                   const void* v, const int32_t* q_starts, const int32_t* q_counts,
                                   const int32_t* k_starts, const int32_t* k_counts,
                                   const int32_t* row_ptr, const int32_t* col_idx,
                                   float softmax_scale, void* out, float* lse, void* ws,
                                   size_t ws_bytes, bsa_stream_t stream);

/* Self-test of the failure detection every pipelined kernel relies on.  Launches one
 * small CTA in which one thread waits on a shared-memory barrier that nothing ever
 * completes, with the same bounded wait the kernels use but a limit of limit_ns
 * (1e3 .. 1e10 ns): the wait gives up, records TIMEOUT (detail 0x1FF) in the status
 * header of ws and raises the CTA's abort flag; a second warp waiting on the same barrier
 * with a longer limit then gives up through the abort flag.  Nothing faults or hangs: the
 * kernel ends by itself after ~limit_ns and the context stays usable.  Words 8..10 of the
 * header receive (first wait completed?, second wait completed?, abort flag seen), so a
 * healthy run reads TIMEOUT from bsa_device_status and (0, 0, 1) there.  ws: >= 256
 * bytes, 16-byte aligned. */
BSA_API bsa_status bsa_selftest_wait(void* ws, size_t ws_bytes, int64_t limit_ns,
                                     bsa_stream_t stream);

/* bsa_fwd on the raster layout, the tile permutation fused into the kernel: q, k, v and
 * out are bf16 [B, S, Hh, D] in token order (S = T*H*W).  The kernel loads every 4x4x4
 * tile of a head with one 5D TMA box over the raster tensor (the box's shared-memory
 * image is the tile-major block; positions outside the valid grid read as zeros, which are
 * the pad slots) and writes each query row straight to its token.  Lists, schedule and
 * arithmetic are those of bsa_fwd: the result equals bsa_tile_permute(inverse) of bsa_fwd
 * on tile-permuted inputs.  lse (nullable): fp32 [B, Hh, S] in token order.  Workspace as
 * for BSA_OP_FWD.  bf16 only. */
BSA_API bsa_status bsa_fwd_raster(const bsa_shape* shape, const void* q, const void* k,
                                  const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                  float softmax_scale, void* out, float* lse, void* ws,
                                  size_t ws_bytes, bsa_stream_t stream);

/* Library build identification (static string). */
BSA_API const char* bsa_version(void);

#ifdef __cplusplus
}
#endif

#endif /* BSATTN_H */
