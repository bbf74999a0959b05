// Internal interface between the C ABI (api.cu) and the kernel files.
#pragma once

#include "bsa_common.cuh"

namespace bsa {

// Division by a per-launch constant as a multiply and a shift ("Division by Invariant
// Integers using Multiplication", Granlund and Montgomery, 1994): for 0 <= n < 2^31 and
// 1 <= d < 2^31, with l = ceil(log2 d) and m = ceil(2^(32+l) / d) (below 2^34),
// floor(n / d) = floor(n * m / 2^(32+l)) exactly, and n * m fits 64 bits.  A division by
// a runtime value would otherwise run on the conversion/reciprocal pipe, which the
// softmax loops need for their exponentials.
struct FastDiv {
  unsigned long long m;
  int shift;  // 32 + l
};

inline FastDiv make_fastdiv(int d) {
  int l = 0;
  while ((1ull << l) < static_cast<unsigned long long>(d)) ++l;
  FastDiv f;
  f.m = ((1ull << (32 + l)) + static_cast<unsigned long long>(d) - 1ull) /
        static_cast<unsigned long long>(d);
  f.shift = 32 + l;
  return f;
}

__host__ __device__ __forceinline__ int fdiv(int n, const FastDiv& f) {
  return static_cast<int>((static_cast<unsigned long long>(static_cast<unsigned>(n)) * f.m) >>
                          f.shift);
}

// Token grid of one (batch, head) slice.
struct GridDims {
  int T, H, W;     // valid grid
  int Tp, Hp, Wp;  // padded grid (multiples of 4)
  int nth, ntw;    // tiles along h and w (Hp/4, Wp/4)
  int S, Np;       // valid tokens, padded slots
  FastDiv div_ntw, div_nth, div_W, div_H;  // division by ntw, nth, W, H
};

// Attention problem in tile-major layout.
struct AttnDims {
  GridDims g;
  int batch, heads, head_dim;
  int q_block;     // 64 or 128
  int n_qb, n_kb;  // query blocks, kv blocks (64 slots each) per head
  int n_cta_per_head;  // ceil(Np / 256): CTAs covering one head's query slots
};

// ---------------------------------------------------------------- grid geometry
// Slot p of the tile-major order: tile = p / 64, inner = p % 64; tiles run row-major over
// (t/4, h/4, w/4), inner slots row-major over (t%4, h%4, w%4).

// Coordinates of tile j (w fastest, then h, then t).
__device__ __forceinline__ void tile_coords(const GridDims& g, int j, int& tw, int& th, int& tt) {
  const int rest = fdiv(j, g.div_ntw);
  tw = j - rest * g.ntw;
  tt = fdiv(rest, g.div_nth);
  th = rest - tt * g.nth;
}

// Raster token index held by slot p, or -1 for a pad slot.
__device__ __forceinline__ int slot_to_token(const GridDims& g, int p) {
  const int tile = p >> 6, inner = p & 63;
  int tw, th, tt;
  tile_coords(g, tile, tw, th, tt);
  const int t = tt * 4 + (inner >> 4);
  const int h = th * 4 + ((inner >> 2) & 3);
  const int w = tw * 4 + (inner & 3);
  if (t >= g.T || h >= g.H || w >= g.W) return -1;
  return (t * g.H + h) * g.W + w;
}

__device__ __forceinline__ int token_to_slot(const GridDims& g, int s) {
  const int rest = fdiv(s, g.div_W);
  const int w = s - rest * g.W;
  const int t = fdiv(rest, g.div_H);
  const int h = rest - t * g.H;
  const int tile = ((t >> 2) * g.nth + (h >> 2)) * g.ntw + (w >> 2);
  return tile * 64 + (((t & 3) * 4 + (h & 3)) * 4 + (w & 3));
}

__device__ __forceinline__ bool slot_valid(const GridDims& g, int p) {
  return slot_to_token(g, p) >= 0;
}

// Valid-slot mask of tile j: bit i set when slot i of the tile lies inside the grid.
__device__ __forceinline__ uint64_t tile_valid_mask(const GridDims& g, int j) {
  int tw, th, tt;
  tile_coords(g, j, tw, th, tt);
  const int vt = min(4, max(0, g.T - 4 * tt));
  const int vh = min(4, max(0, g.H - 4 * th));
  const int vw = min(4, max(0, g.W - 4 * tw));
  const uint64_t row4 = (1ull << vw) - 1ull;
  uint64_t m16 = 0;
  for (int i = 0; i < vh; ++i) m16 |= row4 << (4 * i);
  uint64_t m64 = 0;
  for (int i = 0; i < vt; ++i) m64 |= m16 << (16 * i);
  return m64;
}

// The same mask from the tile's coordinates (no division).
__device__ __forceinline__ uint64_t tile_valid_mask_at(const GridDims& g, int tw, int th, int tt) {
  const int vt = min(4, max(0, g.T - 4 * tt));
  const int vh = min(4, max(0, g.H - 4 * th));
  const int vw = min(4, max(0, g.W - 4 * tw));
  const uint64_t row4 = (1ull << vw) - 1ull;
  uint64_t m16 = 0;
  for (int i = 0; i < vh; ++i) m16 |= row4 << (4 * i);
  uint64_t m64 = 0;
  for (int i = 0; i < vt; ++i) m64 |= m16 << (16 * i);
  return m64;
}

// Moves tile coordinates (w fastest, then h, then t) forward by `by` tiles.
__device__ __forceinline__ void tile_advance(const GridDims& g, int by, int& tw, int& th, int& tt) {
  tw += by;
  while (tw >= g.ntw) {
    tw -= g.ntw;
    if (++th == g.nth) {
      th = 0;
      ++tt;
    }
  }
}

__device__ __forceinline__ bool tile_has_pad(const GridDims& g, int j) {
  int tw, th, tt;
  tile_coords(g, j, tw, th, tt);
  return 4 * tt + 4 > g.T || 4 * th + 4 > g.H || 4 * tw + 4 > g.W;
}

__device__ __forceinline__ void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

cudaError_t launch_tile_permute(const GridDims& g, int batch, int heads, int row_bytes,
                                int inverse, const void* src, void* dst, cudaStream_t stream);

cudaError_t launch_tile_permute_quant_e4m3(const GridDims& g, int batch, int heads, int head_dim,
                                           const void* src, uint8_t* dst, float* scales,
                                           cudaStream_t stream);

// Structured patterns (mirrors bsa_pattern in the C header).
enum : uint32_t {
  PAT_DIAGONAL = 1u,
  PAT_MULTI_DIAGONAL = 2u,
  PAT_VERTICAL_STRIPE = 4u,
  PAT_SURROUNDING = 8u,
  PAT_CRISS_CROSS = 16u,
};
struct PatternParams {
  uint32_t kinds;
  int diag_width, multi_count, multi_period, stripe_stride, stripe_offset;
  int radius_t, radius_h, radius_w;
};
cudaError_t launch_pattern_csr(const AttnDims& a, const PatternParams& pp, int32_t* row_ptr,
                               int32_t* col_idx, long long col_capacity, void* ws,
                               cudaStream_t stream);

// Per-row kept bitmaps + counts -> CSR (exclusive scan, then warp-per-row compaction).
cudaError_t launch_bitmap_to_csr(const int32_t* counts, const uint32_t* bitmaps, long long rows,
                                 int words, int32_t* row_ptr, int32_t* col_idx,
                                 long long col_capacity, uint32_t* status, cudaStream_t stream);

// Top-p selection.  Workspace layout after the status header: counts int32 [R],
// bitmaps uint32 [R][words].
size_t topp_scratch_bytes(long long rows, int n_kb);
cudaError_t launch_topp_select(const float* mass, long long rows, int n_kb, float threshold,
                               int32_t* row_ptr, int32_t* col_idx, long long col_capacity,
                               void* ws, cudaStream_t stream);

// Allocation-free selection: scratch in a fixed device array owned by the library
// (kNoAllocScratchBytes per device); status is a caller buffer of 4 words or null.
size_t topp_noalloc_capacity_bytes();
cudaError_t launch_topp_select_noalloc(const float* mass, long long rows, int n_kb, float threshold,
                                       int32_t* row_ptr, int32_t* col_idx, long long col_capacity,
                                       uint32_t* status, cudaStream_t stream);

// Block-sparse forward.  Scratch after the status header: per-CTA schedule.
size_t fwd_scratch_bytes(const AttnDims& a);

cudaError_t launch_bsattn_fwd(const AttnDims& a, int fp8, const void* q, const void* k,
                              const void* v, const float* q_scales, const float* k_scales,
                              const float* v_scales, const int32_t* row_ptr,
                              const int32_t* col_idx, float softmax_scale, void* out, float* lse,
                              void* ws, cudaStream_t stream);

// Dense calibration pass.
// Scratch of the calibration kernels: kMassSlots slices of 256 rows x n_kb fp32 row-block
// sums after a 256-byte pool bitmap (one bit per slice, cleared by the launcher).  A CTA
// claims a free slice when it starts and frees it when it ends, so live CTAs never share a
// slice; with one CTA per SM (their shared memory admits no second) and more slices than
// SMs, a claim always finds a free slice.
constexpr int kMassSlots = 192;
constexpr size_t kMassPoolBytes = 256;

// Claim a free slice (bit of `pool`), or -1 after kWaitLimitNs without one (TIMEOUT recorded).
__device__ __forceinline__ int claim_mass_slice(uint32_t* pool, uint32_t* status) {
  constexpr int kWords = kMassSlots / 32;
  const int w0 = static_cast<int>(blockIdx.x % kWords);
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    for (int i = 0; i < kWords; ++i) {
      const int w = (w0 + i) % kWords;
      uint32_t v = *reinterpret_cast<volatile uint32_t*>(pool + w);
      while (v != 0xffffffffu) {
        const int b = __ffs(~v) - 1;
        const uint32_t old = atomicOr(pool + w, 1u << b);
        if (!(old & (1u << b))) {
          __threadfence();  // the previous holder's accesses come before ours
          return w * 32 + b;
        }
        v = old | (1u << b);
      }
    }
    if (globaltimer_ns() - t0 > kWaitLimitNs) {
      record_status(status, FLAG_TIMEOUT, DETAIL_MASS_SLICE, blockIdx.x, 0u);
      return -1;
    }
  }
}

__device__ __forceinline__ void release_mass_slice(uint32_t* pool, int slice) {
  if (slice < 0) return;
  __threadfence();  // this CTA's accesses to the slice come before the next holder's
  atomicAnd(pool + (slice >> 5), ~(1u << (slice & 31)));
}

size_t mass_scratch_bytes(const AttnDims& a);
cudaError_t mass_grid(const AttnDims& a, int* grid);
cudaError_t launch_block_mass(const AttnDims& a, const void* q, const void* k, float softmax_scale,
                              float* mass, void* ws, cudaStream_t stream);

// Fused calibration: dense attention output and block masses in one call.
cudaError_t launch_calib_dense_mass(const AttnDims& a, const void* q, const void* k, const void* v,
                                    float softmax_scale, void* out, float* lse, float* mass,
                                    void* ws, cudaStream_t stream);

// Pooled (block-level) estimate of the block masses.
size_t pooled_scratch_bytes(const AttnDims& a);
cudaError_t launch_pooled_mass(const AttnDims& a, const void* q, const void* k, float softmax_scale,
                               float* mass, void* ws, cudaStream_t stream);

// Semantic-aware clustering (one clustering of S tokens into C clusters per (batch, head)).
struct ClusterDims {
  int batch, heads, head_dim;
  int S;  // tokens per (batch, head)
  int C;  // clusters
};
size_t cluster_scratch_bytes(const ClusterDims& cd);
cudaError_t launch_kmeans(const ClusterDims& cd, const void* x, int rounds, float* centroids,
                          int32_t* labels, int32_t* counts, void* ws, cudaStream_t stream);
cudaError_t launch_cluster_layout(const ClusterDims& cd, const int32_t* labels, int32_t* counts,
                                  int32_t* starts, int32_t* token_of_slot, int32_t* slot_of_token,
                                  void* ws, cudaStream_t stream);
cudaError_t launch_cluster_permute(const ClusterDims& cd, int inverse, const int32_t* token_of_slot,
                                   const void* src, void* dst, cudaStream_t stream);
cudaError_t launch_cluster_mass(int batch, int heads, int head_dim, int n_qc, int n_kc,
                                const float* qc, const int32_t* q_counts, const float* kc,
                                const int32_t* k_counts, float softmax_scale, float* mass,
                                cudaStream_t stream);

// Attention in cluster order.  Scratch after the status header: per query cluster, its
// runs of <= 64 keys, and the CTA offsets of the clusters.
int cluster_max_entries(int S, int n_kc);
int cluster_ctas_per_head(int S, int n_qc);
size_t cluster_fwd_scratch_bytes(int bhn, int S, int n_qc, int n_kc);
cudaError_t launch_cluster_fwd(int batch, int heads, int head_dim, int S, int n_qc, int n_kc,
                               const void* q, const void* k, const void* v,
                               const int32_t* q_starts, const int32_t* q_counts,
                               const int32_t* k_starts, const int32_t* k_counts,
                               const int32_t* row_ptr, const int32_t* col_idx,
                               float softmax_scale, void* out, float* lse, void* ws,
                               cudaStream_t stream);

// Raster tokens of one batch as 4x4x4-tile boxes (see api.cu).
cudaError_t encode_tmap_raster_tiles(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                                     int elem_bytes, int D, int heads, int W, int H, int T);
// Block-sparse forward reading Q/K/V from and writing O to the raster layout.
cudaError_t launch_bsattn_fwd_raster(const AttnDims& a, const void* q, const void* k,
                                     const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                     float softmax_scale, void* out, float* lse, void* ws,
                                     cudaStream_t stream);

// Failure-detection self-test (bounded wait on a barrier nothing completes).
cudaError_t launch_selftest_wait(void* ws, uint64_t limit_ns, cudaStream_t stream);
cudaError_t kernel_binary_version(int* version);

// Encode a rank-3 bf16/e4m3 tensor map over [bh][Np][D] with a (box_d x box_rows x 1) box
// and 128-byte swizzle.
cudaError_t encode_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                           int elem_bytes, int D, int Np, int bh, int box_d, int box_rows);

// Same with explicit extents (innermost first), byte strides of dims 1 and 2, and box.
cudaError_t encode_tmap_3d_strided(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                                   const unsigned long long dims[3],
                                   const unsigned long long strides_bytes[2],
                                   const unsigned box[3]);

}  // namespace bsa
