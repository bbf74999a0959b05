// Semantic-aware clustering of tokens: k-means, the cluster order, and the cluster-level
// estimate of the attention mass.
//
// "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via Semantic-Aware
// Permutation", Abstract: tokens are clustered by k-means on their vectors and reordered so
// that each cluster occupies consecutive positions, without padding; the cluster
// representatives identify the critical clusters for the top-p budget control.
//
// Per (batch, head) one clustering of S tokens into C clusters:
//   kmeans_split_kernel    centroids -> three bf16 parts (hi, mid, lo) and |c|^2.
//   kmeans_assign_tc_kernel label = argmin_c (|c|^2 - 2 x.c), ties to the lowest c: x.c on
//                          the tensor cores as x.hi + x.mid + x.lo (tcgen05, fp32 accumulate
//                          in TMEM), 128 tokens per CTA, argmin by one thread per TMEM lane.
//   layout_hist_kernel     per chunk of 1024 tokens, the tokens of each cluster.
//   layout_scan_kernel     per head: cluster sizes, cluster starts (exclusive scan) and each
//                          chunk's first slot inside every cluster.
//   layout_scatter_kernel  one warp per chunk walks its tokens in order: rank among equal
//                          labels by __match_any_sync, so the order is stable.
//   kmeans_update_kernel   centroid = sum of the cluster's tokens / size: 8 warps (32 for
//                          clusters of 1,024 tokens or more on average) over fixed segments
//                          of the cluster order, partial sums added in a fixed order
//                          (deterministic); empty clusters keep theirs.
//   cluster_gather/scatter row copies between raster [B, S, Hh, D] and cluster order
//                          [B, Hh, S, D].
//   cluster_mass_kernel    one CTA per (bh, 8 query clusters): logits with each key centroid row
//                          read once per group, then a weighted softmax per row.
#include "bsa_kernels.cuh"

namespace bsa {

namespace {

constexpr int kLayoutChunk = 1024;  // tokens per histogram chunk
constexpr int kScatterWarps = 8;

}  // namespace

// ---- assignment on the tensor cores
// Every centroid is split into three bf16 parts, hi = bf16(c), mid = bf16(c - hi),
// lo = bf16(c - hi - mid), whose sum is c to within ~2^-24 relative; x is bf16, so the
// tensor cores form x.hi + x.mid + x.lo from exact products with fp32 accumulation: the
// dot products of the fp32 centroids to float32 accuracy.  dist = |c|^2 - 2 x.c is then
// reduced per token (one thread per TMEM lane), ties to the lowest centroid index.

// One warp per (bh, padded centroid row): the three parts [bh][part][c_pad][D] and |c|^2
// (lanes over d, then a fixed xor-shuffle tree).  Rows c >= C are zero.
template <int D>
__global__ void __launch_bounds__(256) kmeans_split_kernel(ClusterDims cd, int c_pad,
                                                           const float* __restrict__ cent,
                                                           __nv_bfloat16* __restrict__ parts,
                                                           float* __restrict__ norms) {
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<long long>(cd.batch) * cd.heads * c_pad) return;  // warp-uniform
  const int bh = static_cast<int>(w / c_pad);
  const int c = static_cast<int>(w - static_cast<long long>(bh) * c_pad);
  const long long plane = static_cast<long long>(c_pad) * D;
  __nv_bfloat16* out = parts + static_cast<long long>(bh) * 3 * plane + static_cast<long long>(c) * D;
  float n = 0.f;
#pragma unroll
  for (int d = lane; d < D; d += 32) {
    const float v = c < cd.C ? cent[(static_cast<long long>(bh) * cd.C + c) * D + d] : 0.f;
    const __nv_bfloat16 hi = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(hi);
    const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
    const __nv_bfloat16 lo = __float2bfloat16_rn(r1 - __bfloat162float(mid));
    out[d] = hi;
    out[plane + d] = mid;
    out[2 * plane + d] = lo;
    n = fmaf(v, v, n);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) n += __shfl_xor_sync(0xffffffffu, n, o);
  if (lane == 0) norms[static_cast<long long>(bh) * c_pad + c] = n;
}

constexpr int kTcRows = 128;     // tokens per CTA = TMEM lanes
constexpr int kTcStages = 2;     // centroid-part ring (two stages: two CTAs fit an SM at n_tile 256)
constexpr int kTcThreads = 160;  // warps 0-3: distances and argmin; warp 4: TMA + MMA

template <int D>
struct AssignSmem {
  static constexpr int kChunks = D / 64;         // 128-byte chunks of a bf16 row
  static constexpr int kXChunk = kTcRows * 128;  // one chunk of the token tile
  static size_t bytes(int n_tile, int c_pad) {
    return 1024 + kChunks * kXChunk + static_cast<size_t>(kTcStages) * n_tile * 128 +
           static_cast<size_t>(c_pad) * 4 + 256;
  }
};

// One CTA per (bh, 128 tokens).  The token tile is loaded once; the parts of each tile of
// n_tile centroids stream through a 2-stage ring as (part, 64-dim chunk) steps, each step
// 4 MMAs of K = 16 into TMEM buffer (tile & 1); the epilogue warps reduce a finished buffer
// while the next tile accumulates in the other.  The CTA allocates only the TMEM columns
// it uses (tmem_cols), so CTAs overlap on an SM.
template <int D>
__global__ void __launch_bounds__(kTcThreads, 1) kmeans_assign_tc_kernel(
    const __grid_constant__ CUtensorMap tm_x, const __grid_constant__ CUtensorMap tm_c,
    ClusterDims cd, int n_tile, int c_pad, uint32_t tmem_cols, const float* __restrict__ norms,
    int32_t* __restrict__ labels, uint32_t* status) {
  using L = AssignSmem<D>;
  constexpr int CH = L::kChunks;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int bstage = n_tile * 128;
  uint8_t* xs = smem;
  uint8_t* bs = smem + CH * L::kXChunk;
  float* sn = reinterpret_cast<float*>(bs + kTcStages * bstage);
  uint64_t* bars = reinterpret_cast<uint64_t*>(sn + c_pad);  // c_pad is a multiple of 16
  uint64_t* bar_x = bars;
  uint64_t* bar_full = bars + 1;
  uint64_t* bar_empty = bar_full + kTcStages;
  uint64_t* bar_acc = bar_empty + kTcStages;  // [2] accumulator complete
  uint64_t* bar_drained = bar_acc + 2;        // [2] epilogue done with the buffer
  uint64_t* bar_drain = bar_drained + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_bh = (cd.S + kTcRows - 1) / kTcRows;
  const int bh = blockIdx.x / per_bh;
  const int s0 = (blockIdx.x - bh * per_bh) * kTcRows;
  const int b = bh / cd.heads, h = bh - b * cd.heads;
  const int n_tiles = c_pad / n_tile;
  const int per_tile = 3 * CH;  // ring steps per centroid tile
  const int T = n_tiles * per_tile;

  if (threadIdx.x == 0) {
    mbar_init(bar_x, 1);
    for (int i = 0; i < kTcStages; ++i) {
      mbar_init(bar_full + i, 1);
      mbar_init(bar_empty + i, 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar_acc + i, 1);
      mbar_init(bar_drained + i, 4);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  for (int i = threadIdx.x; i < c_pad; i += kTcThreads) sn[i] = norms[static_cast<long long>(bh) * c_pad + i];
  if (warp == 4) tmem_alloc(tmem_slot, tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 4) {
    if (lane == 0) {
      prefetch_tensormap(&tm_x);
      prefetch_tensormap(&tm_c);
      auto load_step = [&](int k) {  // centroid tile k / per_tile, part, 64-dim chunk
        const int st = k % kTcStages;
        const int n = k / per_tile, part = (k / CH) % 3, ch = k % CH;
        mbar_arrive_expect_tx(bar_full + st, bstage);
        tma_load_3d(bs + st * bstage, &tm_c, bar_full + st, ch * 64, n * n_tile, bh * 3 + part);
      };
      mbar_arrive_expect_tx(bar_x, CH * L::kXChunk);
      for (int ch = 0; ch < CH; ++ch)
        tma_load_3d(xs + ch * L::kXChunk, &tm_x, bar_x, ch * 64, h, b * cd.S + s0);
      for (int k = 0; k < T && k < kTcStages; ++k) load_step(k);
      const uint32_t idesc = make_idesc(1u, 0u, 128u, static_cast<uint32_t>(n_tile));
      const uint64_t x_desc0 = make_sdesc_sw128(smem_u32(xs), 16, 1024);
      const uint64_t b_desc0 = make_sdesc_sw128(smem_u32(bs), 16, 1024);
      bool ok = mbar_wait(bar_x, 0, abort_flag, status, DETAIL_WAIT_Q);
      for (int k = 0; k < T && ok; ++k) {
        const int st = k % kTcStages;
        const int n = k / per_tile, kin = k - n * per_tile, ch = k % CH;
        const int buf = n & 1;
        if (kin == 0 && n >= 2 &&
            !mbar_wait(bar_drained + buf, ((n - 2) >> 1) & 1, abort_flag, status, DETAIL_WAIT_O_FULL)) {
          ok = false;
          break;
        }
        if (!mbar_wait(bar_full + st, (k / kTcStages) & 1, abort_flag, status, DETAIL_WAIT_K_FULL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint64_t xd = x_desc0 + static_cast<uint64_t>((ch * L::kXChunk) >> 4);
        const uint64_t bd = b_desc0 + static_cast<uint64_t>((st * bstage) >> 4);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // 16 dims (32 bytes) per MMA inside the chunk
          mma_f16_ss(tmem + buf * n_tile, xd + 2 * kk, bd + 2 * kk, idesc, (kin > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar_empty + st);
        if (kin == per_tile - 1) mma_commit(bar_acc + buf);
        // refill the stage of step k - 1 (its MMAs were issued before this step's)
        if (k >= 1 && k - 1 + kTcStages < T) {
          const int st2 = (k - 1) % kTcStages;
          if (!mbar_wait(bar_empty + st2, ((k - 1) / kTcStages) & 1, abort_flag, status,
                         DETAIL_WAIT_K_EMPTY)) {
            ok = false;
            break;
          }
          load_step(k - 1 + kTcStages);
        }
      }
      // Whatever happened, let every issued MMA finish before TMEM is released.
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, status, DETAIL_WAIT_O_FULL);
    }
  } else {
    // ------------------------------------------------ distances and argmin, one token per thread
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    float best = INFINITY;
    int best_c = 0;
    bool ok = true;
    for (int n = 0; n < n_tiles; ++n) {
      const int buf = n & 1;
      const bool got = ok && __all_sync(0xffffffffu, mbar_wait(bar_acc + buf, (n >> 1) & 1, abort_flag,
                                                                status, DETAIL_WAIT_S_FULL));
      ok = got;
      tc_fence_after();
      if (got) {
        for (int c0 = 0; c0 < n_tile; c0 += 32) {
          float v[32];
          tmem_ld32(lane_base + buf * n_tile + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const int idx = n * n_tile + c0 + j;
            const float dist = fmaf(-2.f, v[j], sn[idx]);
            if (idx < cd.C && dist < best) {  // strict: the lowest index wins a tie
              best = dist;
              best_c = idx;
            }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_drained + buf);
    }
    const int s = s0 + warp * 32 + lane;
    if (s < cd.S && ok) labels[static_cast<long long>(bh) * cd.S + s] = best_c;
  }
  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, tmem_cols);
  }
}

// Tokens of each cluster in every chunk of kLayoutChunk tokens: hist[bh][chunk][C].
// Labels outside [0, C) are flagged and left out of the order.
__global__ void __launch_bounds__(256) layout_hist_kernel(ClusterDims cd,
                                                          const int32_t* __restrict__ labels,
                                                          int32_t* __restrict__ hist,
                                                          uint32_t* status) {
  extern __shared__ int32_t sh_hist[];
  const int nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  const int bh = blockIdx.x / nchunks;
  const int chunk = blockIdx.x - bh * nchunks;
  for (int c = threadIdx.x; c < cd.C; c += blockDim.x) sh_hist[c] = 0;
  __syncthreads();
  const int s0 = chunk * kLayoutChunk;
  const int s1 = min(cd.S, s0 + kLayoutChunk);
  const int32_t* lb = labels + static_cast<long long>(bh) * cd.S;
  for (int s = s0 + threadIdx.x; s < s1; s += blockDim.x) {
    const int l = lb[s];
    if (l < 0 || l >= cd.C) {
      record_status(status, FLAG_DEVICE_INPUT, DETAIL_CLUSTER_RANGE, static_cast<uint32_t>(bh),
                    static_cast<uint32_t>(s));
      continue;
    }
    atomicAdd(&sh_hist[l], 1);
  }
  __syncthreads();
  int32_t* out = hist + (static_cast<long long>(bh) * nchunks + chunk) * cd.C;
  for (int c = threadIdx.x; c < cd.C; c += blockDim.x) out[c] = sh_hist[c];
}

// Per head (one CTA, one thread per cluster): turns hist into each chunk's first slot inside
// every cluster (in place), and writes counts and starts.
__global__ void __launch_bounds__(1024) layout_scan_kernel(ClusterDims cd, int32_t* __restrict__ hist,
                                                           int32_t* __restrict__ counts,
                                                           int32_t* __restrict__ starts) {
  __shared__ int warp_tot[32];
  const int bh = blockIdx.x;
  const int c = threadIdx.x;
  const int nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  int32_t* hb = hist + static_cast<long long>(bh) * nchunks * cd.C;
  // eight chunks' counts are loaded before any is written back, so a head's scan costs
  // nchunks / 8 memory round trips rather than nchunks
  constexpr int kU = 8;
  int run = 0;
  if (c < cd.C) {
    for (int k0 = 0; k0 < nchunks; k0 += kU) {
      int n[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        n[u] = k0 + u < nchunks ? hb[static_cast<long long>(k0 + u) * cd.C + c] : 0;
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        if (k0 + u < nchunks) hb[static_cast<long long>(k0 + u) * cd.C + c] = run;
        run += n[u];
      }
    }
  }
  // exclusive scan of the cluster sizes over the CTA
  int incl = run;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane_id() >= static_cast<uint32_t>(o)) incl += y;
  }
  if (lane_id() == 31) warp_tot[c >> 5] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < (c >> 5); ++w) before += warp_tot[w];
  const int start = before + incl - run;
  if (c < cd.C) {
    counts[static_cast<long long>(bh) * cd.C + c] = run;
    starts[static_cast<long long>(bh) * cd.C + c] = start;
    for (int k0 = 0; k0 < nchunks; k0 += kU) {
      int f[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u)
        f[u] = k0 + u < nchunks ? hb[static_cast<long long>(k0 + u) * cd.C + c] : 0;
#pragma unroll
      for (int u = 0; u < kU; ++u)
        if (k0 + u < nchunks) hb[static_cast<long long>(k0 + u) * cd.C + c] = f[u] + start;
    }
  }
}

// One warp per chunk: slot of every token = its chunk's first slot in its cluster + the
// number of earlier tokens of the chunk with the same label.
__global__ void __launch_bounds__(32 * kScatterWarps) layout_scatter_kernel(
    ClusterDims cd, const int32_t* __restrict__ labels, const int32_t* __restrict__ first,
    int32_t* __restrict__ token_of_slot, int32_t* __restrict__ slot_of_token) {
  extern __shared__ int32_t sh_next[];  // [kScatterWarps][C]
  const int nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  const long long wid = static_cast<long long>(blockIdx.x) * kScatterWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (wid >= static_cast<long long>(cd.batch) * cd.heads * nchunks) return;  // warp-uniform
  const int bh = static_cast<int>(wid / nchunks);
  const int chunk = static_cast<int>(wid - static_cast<long long>(bh) * nchunks);
  int32_t* next = sh_next + (threadIdx.x >> 5) * cd.C;
  const int32_t* fb = first + (static_cast<long long>(bh) * nchunks + chunk) * cd.C;
  for (int c = lane; c < cd.C; c += 32) next[c] = fb[c];
  __syncwarp();
  const int32_t* lb = labels + static_cast<long long>(bh) * cd.S;
  int32_t* tos = token_of_slot + static_cast<long long>(bh) * cd.S;
  int32_t* sot = slot_of_token + static_cast<long long>(bh) * cd.S;
  const int s0 = chunk * kLayoutChunk;
  const int s1 = min(cd.S, s0 + kLayoutChunk);
  for (int g = s0; g < s1; g += 32) {
    const int s = g + lane;
    int l = s < s1 ? lb[s] : -1;
    if (l < 0 || l >= cd.C) l = -1;  // left out (flagged by the histogram)
    const unsigned peers = __match_any_sync(0xffffffffu, l);
    const int rank = __popc(peers & ((1u << lane) - 1u));
    int slot = -1;
    if (l >= 0) slot = next[l] + rank;
    __syncwarp();
    if (l >= 0 && rank == 0) next[l] += __popc(peers);
    __syncwarp();
    if (s < s1) {
      sot[s] = slot;
      if (slot >= 0 && slot < cd.S) tos[slot] = s;
    }
  }
}

// centroid[bh][c] = mean of the cluster's tokens.  One CTA of 8 warps per (bh, cluster):
// warp w sums the w-th of 8 contiguous segments of the cluster's slots (lane l holds dims
// D/32 * l ..), the 8 partial sums are added in warp order: a fixed summation order
// (deterministic).  An empty cluster keeps its centroid.
template <int D, int W>
__global__ void __launch_bounds__(32 * W) kmeans_update_kernel(ClusterDims cd,
                                                            const __nv_bfloat16* __restrict__ x,
                                                            const int32_t* __restrict__ token_of_slot,
                                                            const int32_t* __restrict__ starts,
                                                            const int32_t* __restrict__ counts,
                                                            float* __restrict__ cent) {
  constexpr int PER = D / 32;  // dims per lane: 4 (D = 128) or 2 (D = 64)
  __shared__ float part[W][D];
  const int bh = blockIdx.x / cd.C;
  const int c = blockIdx.x - bh * cd.C;
  const int b = bh / cd.heads, h = bh - b * cd.heads;
  const int n = counts[static_cast<long long>(bh) * cd.C + c];
  if (n <= 0) return;  // uniform over the CTA
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int st = starts[static_cast<long long>(bh) * cd.C + c];
  const int seg = (n + W - 1) / W;
  const int lo = min(n, warp * seg), hi = min(n, lo + seg);
  const int32_t* tos = token_of_slot + static_cast<long long>(bh) * cd.S + st;
  const __nv_bfloat16* xb = x + static_cast<long long>(b) * cd.S * cd.heads * D + h * D + lane * PER;
  const long long row = static_cast<long long>(cd.heads) * D;
  float acc[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) acc[e] = 0.f;
  // 8 tokens' loads in flight, then their adds in slot order (the same sums as one token
  // at a time)
  constexpr int kBatch = 8;
  for (int i0 = lo; i0 < hi; i0 += kBatch) {
    uint32_t w[kBatch][PER / 2];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i = i0 + u;
      if (i < hi) {
        const __nv_bfloat16* r = xb + tos[i] * row;
        if constexpr (PER == 4) {
          const uint2 v = *reinterpret_cast<const uint2*>(r);
          w[u][0] = v.x;
          w[u][1] = v.y;
        } else {
          w[u][0] = *reinterpret_cast<const uint32_t*>(r);
        }
      } else {
#pragma unroll
        for (int e = 0; e < PER / 2; ++e) w[u][e] = 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      if (i0 + u >= hi) break;
#pragma unroll
      for (int e = 0; e < PER / 2; ++e) {
        acc[2 * e] += __uint_as_float(w[u][e] << 16);
        acc[2 * e + 1] += __uint_as_float(w[u][e] & 0xFFFF0000u);
      }
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) part[warp][lane * PER + e] = acc[e];
  __syncthreads();
  if (threadIdx.x < D) {
    float sum = 0.f;
#pragma unroll
    for (int w = 0; w < W; ++w) sum += part[w][threadIdx.x];
    cent[(static_cast<long long>(bh) * cd.C + c) * D + threadIdx.x] = __fdiv_rn(sum, static_cast<float>(n));
  }
}

// Row copies: forward dst[bh][p] = src[b][token_of_slot[bh][p]][h] (zeros for an empty
// slot); inverse dst[b][token_of_slot[bh][p]][h] = src[bh][p].  16 bytes per lane.
template <int D>
__global__ void __launch_bounds__(256) cluster_permute_kernel(ClusterDims cd, int inverse,
                                                              const int32_t* __restrict__ tos,
                                                              const __nv_bfloat16* __restrict__ src,
                                                              __nv_bfloat16* __restrict__ dst) {
  constexpr int kVec = D / 8;  // uint4 per row
  const long long rows = static_cast<long long>(cd.batch) * cd.heads * cd.S;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       i < rows * kVec; i += stride) {
    const long long r = i / kVec;
    const int v = static_cast<int>(i - r * kVec);
    const int bh = static_cast<int>(r / cd.S);
    const int p = static_cast<int>(r - static_cast<long long>(bh) * cd.S);
    const int b = bh / cd.heads, h = bh - b * cd.heads;
    const int t = tos[r];
    const bool ok = t >= 0 && t < cd.S;
    const long long raster = ((static_cast<long long>(b) * cd.S + (ok ? t : 0)) * cd.heads + h) * D;
    const long long perm = (static_cast<long long>(bh) * cd.S + p) * D;
    if (!inverse) {
      uint4 w = make_uint4(0u, 0u, 0u, 0u);
      if (ok) w = reinterpret_cast<const uint4*>(src + raster)[v];
      reinterpret_cast<uint4*>(dst + perm)[v] = w;
    } else if (ok) {
      reinterpret_cast<uint4*>(dst + raster)[v] = reinterpret_cast<const uint4*>(src + perm)[v];
    }
  }
}

// Cluster-level estimate: M[i][j] = n_j exp(s qc_i . kc_j) / sum_j' n_j' exp(s qc_i . kc_j').
// One CTA of 8 warps per (bh, group of kMassGroup query clusters).  Logits: warp w takes key
// clusters w, w + 8, ...; its lanes read a key centroid row once, coalesced, and form its
// dot products with every query centroid of the group (lanes over d, a fixed xor-shuffle
// tree), so each key row is read once per group instead of once per query cluster.  Then
// warp q normalises row q of the group (weighted softmax over the key clusters).
constexpr int kMassGroup = 8;
constexpr int kMassMaxKc = 1024;
constexpr int kMassMaxD = 128;

__global__ void __launch_bounds__(256) cluster_mass_kernel(int heads, int D, int n_qc, int n_kc,
                                                           const float* __restrict__ qc,
                                                           const int32_t* __restrict__ q_counts,
                                                           const float* __restrict__ kc,
                                                           const int32_t* __restrict__ k_counts,
                                                           float scale_log2, float* __restrict__ mass) {
  __shared__ float sq[kMassGroup][kMassMaxD];
  __shared__ float lg[kMassGroup][kMassMaxKc];
  const int groups = (n_qc + kMassGroup - 1) / kMassGroup;
  const int bh = blockIdx.x / groups;
  const int i0 = (blockIdx.x - bh * groups) * kMassGroup;
  const int ng = min(kMassGroup, n_qc - i0);  // query clusters in this group
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const long long qrow0 = static_cast<long long>(bh) * n_qc + i0;
  for (int e = tid; e < kMassGroup * D; e += 256) {
    const int q = e / D, d = e - q * D;
    sq[q][d] = q < ng ? qc[(qrow0 + q) * D + d] : 0.f;
  }
  __syncthreads();
  const float* kb = kc + static_cast<long long>(bh) * n_kc * D;
  const int32_t* nk = k_counts + static_cast<long long>(bh) * n_kc;
  for (int j = warp; j < n_kc; j += 8) {
    float acc[kMassGroup];
#pragma unroll
    for (int q = 0; q < kMassGroup; ++q) acc[q] = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float kv = kb[static_cast<long long>(j) * D + d];
#pragma unroll
      for (int q = 0; q < kMassGroup; ++q) acc[q] = fmaf(sq[q][d], kv, acc[q]);
    }
#pragma unroll
    for (int q = 0; q < kMassGroup; ++q)
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) acc[q] += __shfl_xor_sync(0xffffffffu, acc[q], o);
    if (lane < kMassGroup) {
      float v = acc[0];
#pragma unroll
      for (int q = 1; q < kMassGroup; ++q) v = lane == q ? acc[q] : v;
      lg[lane][j] = nk[j] > 0 ? v * scale_log2 : -INFINITY;
    }
  }
  __syncthreads();
  if (warp >= ng) return;
  float* out = mass + (qrow0 + warp) * n_kc;
  if (q_counts[qrow0 + warp] <= 0) {  // an empty query cluster: all-zero row
    for (int j = lane; j < n_kc; j += 32) out[j] = 0.f;
    return;
  }
  float* row = lg[warp];
  float mx = -INFINITY;
  for (int j = lane; j < n_kc; j += 32) mx = fmaxf(mx, row[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  float sum = 0.f;
  for (int j = lane; j < n_kc; j += 32) {
    const float w = mx == -INFINITY ? 0.f : static_cast<float>(max(nk[j], 0)) * exp2f(row[j] - mx);
    row[j] = w;
    sum += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  for (int j = lane; j < n_kc; j += 32) out[j] = row[j] * inv;
}

// ---------------------------------------------------------------------------------------
// Workspace after the status header: hist int32 [BH][nchunks][C], starts int32 [BH][C],
// token_of_slot int32 [BH][S], slot_of_token int32 [BH][S] (k-means only uses the last
// three internally; the layout call writes them to the caller's arrays instead).
static size_t al256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

// Centroid tile of the tensor-core assignment: all clusters in one MMA when C <= 256; a
// multiple of 32 so the epilogue reads whole 32-column groups of it.
static int assign_n_tile(int C) { return C >= 256 ? 256 : ((C + 31) / 32) * 32; }
static int assign_c_pad(int C) {
  const int n = assign_n_tile(C);
  return ((C + n - 1) / n) * n;
}

// Workspace after the status header: hist, starts, token_of_slot, slot_of_token (the
// cluster order), then the centroid parts bf16 [BH][3][c_pad][D] and norms fp32 [BH][c_pad].
size_t cluster_scratch_bytes(const ClusterDims& cd) {
  const size_t bhn = static_cast<size_t>(cd.batch) * cd.heads;
  const size_t nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  const size_t c_pad = static_cast<size_t>(assign_c_pad(cd.C));
  return al256(bhn * nchunks * cd.C * 4) + al256(bhn * cd.C * 4) + 2 * al256(bhn * cd.S * 4) +
         al256(bhn * 3 * c_pad * cd.head_dim * 2) + al256(bhn * c_pad * 4);
}

template <int D>
static cudaError_t launch_assign(const ClusterDims& cd, const void* x, const float* centroids,
                                 __nv_bfloat16* parts, float* norms, int32_t* labels,
                                 uint32_t* status, cudaStream_t stream) {
  const long long bhn = static_cast<long long>(cd.batch) * cd.heads;
  const int n_tile = assign_n_tile(cd.C), c_pad = assign_c_pad(cd.C);
  kmeans_split_kernel<D><<<static_cast<unsigned>((bhn * c_pad + 7) / 8), 256, 0, stream>>>(
      cd, c_pad, centroids, parts, norms);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // tokens: raster [B, S, Hh, D] as (D, Hh, B*S) with a 64 x 1 x 128 box
  CUtensorMap tx, tc;
  const unsigned long long xdims[3] = {static_cast<unsigned long long>(D),
                                       static_cast<unsigned long long>(cd.heads),
                                       static_cast<unsigned long long>(cd.batch) * cd.S};
  const unsigned long long xstr[2] = {static_cast<unsigned long long>(D) * 2,
                                      static_cast<unsigned long long>(cd.heads) * D * 2};
  const unsigned xbox[3] = {64u, 1u, static_cast<unsigned>(kTcRows)};
  e = encode_tmap_3d_strided(&tx, x, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, xdims, xstr, xbox);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tc, parts, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, c_pad,
                     static_cast<int>(bhn * 3), 64, n_tile);
  if (e != cudaSuccess) return e;
  const size_t smem = AssignSmem<D>::bytes(n_tile, c_pad);
  e = cudaFuncSetAttribute(kmeans_assign_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const unsigned ctas = static_cast<unsigned>(bhn * ((cd.S + kTcRows - 1) / kTcRows));
  // TMEM: one accumulator of n_tile columns, two when there are several centroid tiles,
  // rounded up to a power of two, so several CTAs can share an SM's 512 columns.
  const int need = (c_pad / n_tile > 1) ? 2 * n_tile : n_tile;
  uint32_t cols = 32;
  while (cols < static_cast<uint32_t>(need)) cols <<= 1;
  kmeans_assign_tc_kernel<D><<<ctas, kTcThreads, smem, stream>>>(tx, tc, cd, n_tile, c_pad, cols,
                                                                 norms, labels, status);
  return cudaGetLastError();
}

static cudaError_t layout_into(const ClusterDims& cd, const int32_t* labels, int32_t* counts,
                               int32_t* starts, int32_t* tos, int32_t* sot, int32_t* hist,
                               uint32_t* status, cudaStream_t stream) {
  const long long bhn = static_cast<long long>(cd.batch) * cd.heads;
  const int nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  cudaError_t e = cudaMemsetAsync(tos, 0xFF, static_cast<size_t>(bhn) * cd.S * 4, stream);
  if (e != cudaSuccess) return e;
  layout_hist_kernel<<<static_cast<unsigned>(bhn * nchunks), 256, cd.C * 4, stream>>>(cd, labels, hist,
                                                                                      status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  layout_scan_kernel<<<static_cast<unsigned>(bhn), 1024, 0, stream>>>(cd, hist, counts, starts);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const long long warps = bhn * nchunks;
  layout_scatter_kernel<<<static_cast<unsigned>((warps + kScatterWarps - 1) / kScatterWarps),
                          32 * kScatterWarps, kScatterWarps * cd.C * 4, stream>>>(cd, labels, hist,
                                                                                  tos, sot);
  return cudaGetLastError();
}

cudaError_t launch_cluster_layout(const ClusterDims& cd, const int32_t* labels, int32_t* counts,
                                  int32_t* starts, int32_t* token_of_slot, int32_t* slot_of_token,
                                  void* ws, cudaStream_t stream) {
  if (cd.batch * cd.heads == 0 || cd.S == 0) return cudaSuccess;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  int32_t* hist = reinterpret_cast<int32_t*>(base + kStatusBytes);
  return layout_into(cd, labels, counts, starts, token_of_slot, slot_of_token, hist, status, stream);
}

cudaError_t launch_kmeans(const ClusterDims& cd, const void* x, int rounds, float* centroids,
                          int32_t* labels, int32_t* counts, void* ws, cudaStream_t stream) {
  const long long bhn = static_cast<long long>(cd.batch) * cd.heads;
  if (bhn == 0 || cd.S == 0 || rounds <= 0) return cudaSuccess;
  const int nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  uint8_t* p = base + kStatusBytes;
  int32_t* hist = reinterpret_cast<int32_t*>(p);
  p += al256(static_cast<size_t>(bhn) * nchunks * cd.C * 4);
  int32_t* starts = reinterpret_cast<int32_t*>(p);
  p += al256(static_cast<size_t>(bhn) * cd.C * 4);
  int32_t* tos = reinterpret_cast<int32_t*>(p);
  p += al256(static_cast<size_t>(bhn) * cd.S * 4);
  int32_t* sot = reinterpret_cast<int32_t*>(p);
  p += al256(static_cast<size_t>(bhn) * cd.S * 4);
  __nv_bfloat16* parts = reinterpret_cast<__nv_bfloat16*>(p);
  p += al256(static_cast<size_t>(bhn) * 3 * assign_c_pad(cd.C) * cd.head_dim * 2);
  float* norms = reinterpret_cast<float*>(p);
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const unsigned upd_ctas = static_cast<unsigned>(bhn * cd.C);
  for (int r = 0; r < rounds; ++r) {
    cudaError_t e = cd.head_dim == 128
                        ? launch_assign<128>(cd, x, centroids, parts, norms, labels, status, stream)
                        : launch_assign<64>(cd, x, centroids, parts, norms, labels, status, stream);
    if (e != cudaSuccess) return e;
    e = layout_into(cd, labels, counts, starts, tos, sot, hist, status, stream);
    if (e != cudaSuccess) return e;
    // large clusters (1,024 tokens or more on average) get 32 warps, smaller ones 8
    const bool wide = cd.S >= 1024LL * cd.C;
    if (cd.head_dim == 128) {
      if (wide)
        kmeans_update_kernel<128, 32><<<upd_ctas, 1024, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
      else
        kmeans_update_kernel<128, 8><<<upd_ctas, 256, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
    } else {
      if (wide)
        kmeans_update_kernel<64, 32><<<upd_ctas, 1024, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
      else
        kmeans_update_kernel<64, 8><<<upd_ctas, 256, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_cluster_permute(const ClusterDims& cd, int inverse, const int32_t* token_of_slot,
                                   const void* src, void* dst, cudaStream_t stream) {
  const long long rows = static_cast<long long>(cd.batch) * cd.heads * cd.S;
  if (rows == 0) return cudaSuccess;
  const long long items = rows * (cd.head_dim / 8);
  const long long want = (items + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < 148LL * 16 ? want : 148LL * 16);
  const __nv_bfloat16* s = static_cast<const __nv_bfloat16*>(src);
  __nv_bfloat16* d = static_cast<__nv_bfloat16*>(dst);
  if (cd.head_dim == 128)
    cluster_permute_kernel<128><<<grid, 256, 0, stream>>>(cd, inverse, token_of_slot, s, d);
  else
    cluster_permute_kernel<64><<<grid, 256, 0, stream>>>(cd, inverse, token_of_slot, s, d);
  return cudaGetLastError();
}

cudaError_t launch_cluster_mass(int batch, int heads, int head_dim, int n_qc, int n_kc,
                                const float* qc, const int32_t* q_counts, const float* kc,
                                const int32_t* k_counts, float softmax_scale, float* mass,
                                cudaStream_t stream) {
  const long long rows = static_cast<long long>(batch) * heads * n_qc;
  if (rows == 0 || n_kc == 0) return cudaSuccess;
  if (head_dim > kMassMaxD || n_kc > kMassMaxKc) return cudaErrorNotSupported;
  const long long ctas = static_cast<long long>(batch) * heads * ((n_qc + kMassGroup - 1) / kMassGroup);
  cluster_mass_kernel<<<static_cast<unsigned>(ctas), 256, 0, stream>>>(
      heads, head_dim, n_qc, n_kc, qc, q_counts, kc, k_counts, softmax_scale * 1.4426950408889634f,
      mass);
  return cudaGetLastError();
}

}  // namespace bsa
