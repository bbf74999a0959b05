// Semantic-aware clustering of tokens: k-means, the cluster order, and the cluster-level
// estimate of the attention mass.
//
// "Sparse VideoGen2: Accelerate Video Generation with Sparse Attention via Semantic-Aware
// Permutation", Abstract: tokens are clustered by k-means on their vectors and reordered so
// that each cluster occupies consecutive positions, without padding; the cluster
// representatives identify the critical clusters for the top-p budget control.
//
// Per (batch, head) one clustering of S tokens into C clusters:
//   kmeans_assign_kernel   label = argmin_c (|c|^2 - 2 x.c) in float32, ties to the lowest c;
//                          four tokens per thread, centroids staged 16 at a time in shared
//                          memory and read as broadcasts (each feeds 32 FMAs).
//   layout_hist_kernel     per chunk of 1024 tokens, the tokens of each cluster.
//   layout_scan_kernel     per head: cluster sizes, cluster starts (exclusive scan) and each
//                          chunk's first slot inside every cluster.
//   layout_scatter_kernel  one warp per chunk walks its tokens in order: rank among equal
//                          labels by __match_any_sync, so the order is stable.
//   kmeans_update_kernel   centroid = sum of the cluster's tokens in cluster order / size,
//                          a fixed summation order (deterministic); empty clusters keep theirs.
//   cluster_gather/scatter row copies between raster [B, S, Hh, D] and cluster order
//                          [B, Hh, S, D].
//   cluster_mass_kernel    one CTA per (bh, query cluster): weighted softmax over key clusters.
#include "bsa_kernels.cuh"

namespace bsa {

namespace {

constexpr int kAsgThreads = 128;
constexpr int kAsgChunk = 16;   // centroids per shared-memory stage
constexpr int kAsgTokens = 4;   // tokens per thread
constexpr int kLayoutChunk = 1024;  // tokens per histogram chunk
constexpr int kScatterWarps = 8;

// Eight bf16 values (little-endian pairs in four words) to float: a bf16 is the upper half
// of the float with the same bits.
__device__ __forceinline__ void bf16x8_to_float(const uint4& raw, float* f) {
  const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kAsgThreads) kmeans_assign_kernel(
    const __nv_bfloat16* __restrict__ x, ClusterDims cd, const float* __restrict__ cent,
    int32_t* __restrict__ labels) {
  constexpr int TPT = kAsgTokens;  // tokens per thread: each centroid broadcast feeds 4 x 8 FMAs
  __shared__ __align__(16) float cs[kAsgChunk][D];
  __shared__ float cn[kAsgChunk];
  const int per_bh = (cd.S + kAsgThreads * TPT - 1) / (kAsgThreads * TPT);
  const int bh = blockIdx.x / per_bh;
  const int s0 = (blockIdx.x - bh * per_bh) * kAsgThreads * TPT + threadIdx.x;
  const int b = bh / cd.heads, h = bh - b * cd.heads;
  const __nv_bfloat16* xr[TPT];
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    const int s = s0 + u * kAsgThreads;
    xr[u] = x + ((static_cast<long long>(b) * cd.S + (s < cd.S ? s : 0)) * cd.heads + h) * D;
  }
  const float* cb = cent + static_cast<long long>(bh) * cd.C * D;
  float best[TPT];
  int best_c[TPT];
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    best[u] = INFINITY;
    best_c[u] = 0;
  }
  for (int c0 = 0; c0 < cd.C; c0 += kAsgChunk) {
    const int nc = min(kAsgChunk, cd.C - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < kAsgChunk * D; i += kAsgThreads) {
      const int j = i / D, d = i - j * D;
      cs[j][d] = j < nc ? cb[static_cast<long long>(c0 + j) * D + d] : 0.f;
    }
    __syncthreads();
    {  // |c|^2: 8 lanes per centroid; lane p sums dims 8m + p, m = 0 .. D/8 - 1, starting at
       // m = j mod 4 so the warp's four centroids fall in distinct banks; fixed order.
      constexpr int kPart = D / 8;
      const int j = threadIdx.x >> 3, part = threadIdx.x & 7;
      float n = 0.f;
#pragma unroll 4
      for (int m = 0; m < kPart; ++m) {
        const float c = cs[j][8 * ((m + (j & 3)) % kPart) + part];
        n = fmaf(c, c, n);
      }
      n += __shfl_xor_sync(0xffffffffu, n, 1);
      n += __shfl_xor_sync(0xffffffffu, n, 2);
      n += __shfl_xor_sync(0xffffffffu, n, 4);
      if (part == 0) cn[j] = n;
    }
    __syncthreads();
    float acc[TPT][kAsgChunk];
#pragma unroll
    for (int u = 0; u < TPT; ++u)
#pragma unroll
      for (int j = 0; j < kAsgChunk; ++j) acc[u][j] = 0.f;
#pragma unroll 1
    for (int d = 0; d < D; d += 8) {
      float xv[TPT][8];
#pragma unroll
      for (int u = 0; u < TPT; ++u) bf16x8_to_float(*reinterpret_cast<const uint4*>(xr[u] + d), xv[u]);
#pragma unroll
      for (int j = 0; j < kAsgChunk; ++j) {
        const float4 c0v = *reinterpret_cast<const float4*>(&cs[j][d]);
        const float4 c1v = *reinterpret_cast<const float4*>(&cs[j][d + 4]);
#pragma unroll
        for (int u = 0; u < TPT; ++u) {
          float a = acc[u][j];
          a = fmaf(xv[u][0], c0v.x, a);
          a = fmaf(xv[u][1], c0v.y, a);
          a = fmaf(xv[u][2], c0v.z, a);
          a = fmaf(xv[u][3], c0v.w, a);
          a = fmaf(xv[u][4], c1v.x, a);
          a = fmaf(xv[u][5], c1v.y, a);
          a = fmaf(xv[u][6], c1v.z, a);
          a = fmaf(xv[u][7], c1v.w, a);
          acc[u][j] = a;
        }
      }
    }
#pragma unroll
    for (int j = 0; j < kAsgChunk; ++j) {
#pragma unroll
      for (int u = 0; u < TPT; ++u) {
        const float dist = fmaf(-2.f, acc[u][j], cn[j]);
        if (j < nc && dist < best[u]) {  // strict: the lowest index wins a tie
          best[u] = dist;
          best_c[u] = c0 + j;
        }
      }
    }
  }
#pragma unroll
  for (int u = 0; u < TPT; ++u) {
    const int s = s0 + u * kAsgThreads;
    if (s < cd.S) labels[static_cast<long long>(bh) * cd.S + s] = best_c[u];
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
  int run = 0;
  if (c < cd.C) {
    for (int k = 0; k < nchunks; ++k) {
      const int n = hb[static_cast<long long>(k) * cd.C + c];
      hb[static_cast<long long>(k) * cd.C + c] = run;
      run += n;
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
    for (int k = 0; k < nchunks; ++k) hb[static_cast<long long>(k) * cd.C + c] += start;
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

// centroid[bh][c] = mean of the cluster's tokens, summed in cluster order: 4 partial sums by
// slot index mod 4, combined in a fixed order.  One CTA of D threads per (bh, cluster).
template <int D>
__global__ void __launch_bounds__(D) kmeans_update_kernel(ClusterDims cd,
                                                          const __nv_bfloat16* __restrict__ x,
                                                          const int32_t* __restrict__ token_of_slot,
                                                          const int32_t* __restrict__ starts,
                                                          const int32_t* __restrict__ counts,
                                                          float* __restrict__ cent) {
  const int bh = blockIdx.x / cd.C;
  const int c = blockIdx.x - bh * cd.C;
  const int b = bh / cd.heads, h = bh - b * cd.heads;
  const int d = threadIdx.x;
  const int n = counts[static_cast<long long>(bh) * cd.C + c];
  if (n <= 0) return;  // empty cluster: keeps its centroid
  const int st = starts[static_cast<long long>(bh) * cd.C + c];
  const int32_t* tos = token_of_slot + static_cast<long long>(bh) * cd.S + st;
  const __nv_bfloat16* xb = x + static_cast<long long>(b) * cd.S * cd.heads * D + h * D + d;
  const long long row = static_cast<long long>(cd.heads) * D;
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  int i = 0;
  for (; i + 4 <= n; i += 4) {
#pragma unroll
    for (int u = 0; u < 4; ++u) acc[u] += __bfloat162float(xb[tos[i + u] * row]);
  }
  for (; i < n; ++i) acc[i & 3] += __bfloat162float(xb[tos[i] * row]);
  const float sum = (acc[0] + acc[1]) + (acc[2] + acc[3]);
  cent[(static_cast<long long>(bh) * cd.C + c) * D + d] = __fdiv_rn(sum, static_cast<float>(n));
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
// One CTA of 256 threads per (bh, query cluster); logits in shared memory (<= 1024).
__global__ void __launch_bounds__(256) cluster_mass_kernel(int heads, int D, int n_qc, int n_kc,
                                                           const float* __restrict__ qc,
                                                           const int32_t* __restrict__ q_counts,
                                                           const float* __restrict__ kc,
                                                           const int32_t* __restrict__ k_counts,
                                                           float scale_log2, float* __restrict__ mass) {
  __shared__ float sq[128];
  __shared__ float lg[1024];
  __shared__ float red[8];
  const int bh = blockIdx.x / n_qc;
  const int i = blockIdx.x - bh * n_qc;
  const int tid = threadIdx.x;
  float* out = mass + static_cast<long long>(blockIdx.x) * n_kc;
  if (q_counts[static_cast<long long>(bh) * n_qc + i] <= 0) {
    for (int j = tid; j < n_kc; j += 256) out[j] = 0.f;
    return;
  }
  for (int d = tid; d < D; d += 256) sq[d] = qc[static_cast<long long>(blockIdx.x) * D + d];
  __syncthreads();
  const float* kb = kc + static_cast<long long>(bh) * n_kc * D;
  const int32_t* nk = k_counts + static_cast<long long>(bh) * n_kc;
  float mx = -INFINITY;
  for (int j = tid; j < n_kc; j += 256) {
    float acc = 0.f;
    for (int d = 0; d < D; ++d) acc = fmaf(sq[d], kb[static_cast<long long>(j) * D + d], acc);
    const float l = nk[j] > 0 ? acc * scale_log2 : -INFINITY;
    lg[j] = l;
    mx = fmaxf(mx, l);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (lane_id() == 0) red[tid >> 5] = mx;
  __syncthreads();
  mx = red[0];
#pragma unroll
  for (int w = 1; w < 8; ++w) mx = fmaxf(mx, red[w]);
  __syncthreads();
  float sum = 0.f;
  for (int j = tid; j < n_kc; j += 256) {
    const float w = mx == -INFINITY ? 0.f : static_cast<float>(max(nk[j], 0)) * exp2f(lg[j] - mx);
    lg[j] = w;
    sum += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  if (lane_id() == 0) red[tid >> 5] = sum;
  __syncthreads();
  sum = ((red[0] + red[1]) + (red[2] + red[3])) + ((red[4] + red[5]) + (red[6] + red[7]));
  const float inv = sum > 0.f ? 1.f / sum : 0.f;
  for (int j = tid; j < n_kc; j += 256) out[j] = lg[j] * inv;
}

// ---------------------------------------------------------------------------------------
// Workspace after the status header: hist int32 [BH][nchunks][C], starts int32 [BH][C],
// token_of_slot int32 [BH][S], slot_of_token int32 [BH][S] (k-means only uses the last
// three internally; the layout call writes them to the caller's arrays instead).
static size_t al256(size_t n) { return (n + 255) & ~static_cast<size_t>(255); }

size_t cluster_scratch_bytes(const ClusterDims& cd) {
  const size_t bhn = static_cast<size_t>(cd.batch) * cd.heads;
  const size_t nchunks = (cd.S + kLayoutChunk - 1) / kLayoutChunk;
  return al256(bhn * nchunks * cd.C * 4) + al256(bhn * cd.C * 4) + 2 * al256(bhn * cd.S * 4);
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
  const __nv_bfloat16* xb = static_cast<const __nv_bfloat16*>(x);
  const unsigned asg_ctas =
      static_cast<unsigned>(bhn * ((cd.S + kAsgThreads * kAsgTokens - 1) / (kAsgThreads * kAsgTokens)));
  const unsigned upd_ctas = static_cast<unsigned>(bhn * cd.C);
  for (int r = 0; r < rounds; ++r) {
    if (cd.head_dim == 128)
      kmeans_assign_kernel<128><<<asg_ctas, kAsgThreads, 0, stream>>>(xb, cd, centroids, labels);
    else
      kmeans_assign_kernel<64><<<asg_ctas, kAsgThreads, 0, stream>>>(xb, cd, centroids, labels);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = layout_into(cd, labels, counts, starts, tos, sot, hist, status, stream);
    if (e != cudaSuccess) return e;
    if (cd.head_dim == 128)
      kmeans_update_kernel<128><<<upd_ctas, 128, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
    else
      kmeans_update_kernel<64><<<upd_ctas, 64, 0, stream>>>(cd, xb, tos, starts, counts, centroids);
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
  cluster_mass_kernel<<<static_cast<unsigned>(rows), 256, 0, stream>>>(
      heads, head_dim, n_qc, n_kc, qc, q_counts, kc, k_counts, softmax_scale * 1.4426950408889634f,
      mass);
  return cudaGetLastError();
}

}  // namespace bsa
