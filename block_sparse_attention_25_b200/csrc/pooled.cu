// Pooled (block-level) estimate of the block masses, for per-step ("online") top-p
// selection without a dense pass.
//
// "Sparse VideoGen2", Abstract: top-p dynamic budget control on attention between token
// clusters; with 4x4x4 tiles as the clusters, a kv block is represented by the mean of its
// valid keys and weighted by their number, a query block by the mean of its valid queries:
//   M_est[i, j] = n_j exp(scale qbar_i . kbar_j) / sum_j' n_j' exp(scale qbar_i . kbar_j').
// The result feeds bsa_topp_select like the exact masses do.
//
// Kernels (fp32 CUDA-core math: the estimate is ~Np^2/4096 * D multiply-adds per head):
//   pool_tiles_kernel   one warp per (bh, tile): sums of the valid rows of Q and K.
//   pooled_logits_kernel one CTA per (bh, 8 query blocks): qbar from the tile sums, kbar
//                        in chunks of 32 tiles staged in shared memory (rows padded to
//                        D+1 floats, so 32 threads reading 32 rows hit 32 banks); writes
//                        the log2-domain logits into the output tensor.
//   pooled_softmax_kernel one warp per row: weighted softmax in place.
#include "bsa_kernels.cuh"

namespace bsa {

// Valid rows of tile j (popcount of its slot mask).
__device__ __forceinline__ int tile_valid_count(const GridDims& g, int j) {
  return __popcll(tile_valid_mask(g, j));
}

template <int D>
__global__ void __launch_bounds__(256) pool_tiles_kernel(const __nv_bfloat16* __restrict__ q,
                                                         const __nv_bfloat16* __restrict__ k,
                                                         GridDims g, long long tiles,
                                                         float* __restrict__ qsum,
                                                         float* __restrict__ ksum) {
  constexpr int PER = D / 32;  // dims per lane (4 or 2)
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= tiles) return;
  const int lane = threadIdx.x & 31;
  const int ntiles = g.Np / 64;
  const int j = static_cast<int>(w % ntiles);
  const uint64_t vm = tile_valid_mask(g, j);
  const __nv_bfloat16* qt = q + w * 64 * D + lane * PER;
  const __nv_bfloat16* kt = k + w * 64 * D + lane * PER;
  float aq[PER], ak[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) aq[e] = ak[e] = 0.f;
  for (int r = 0; r < 64; ++r) {
    if (!((vm >> r) & 1ull)) continue;
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      aq[e] += __bfloat162float(qt[r * D + e]);
      ak[e] += __bfloat162float(kt[r * D + e]);
    }
  }
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    qsum[w * D + lane * PER + e] = aq[e];
    ksum[w * D + lane * PER + e] = ak[e];
  }
}

// Logits in log2 units: scale * log2(e) * qbar_i . kbar_j, -inf for tiles without valid keys
// (the softmax kernel adds log2(n_j)).  One thread per (query block, kv tile) of a chunk.
template <int D>
__global__ void __launch_bounds__(256) pooled_logits_kernel(const float* __restrict__ qsum,
                                                            const float* __restrict__ ksum,
                                                            AttnDims a, float scale_log2,
                                                            float* __restrict__ out) {
  __shared__ float sq[8][D];
  __shared__ float sk[32][D + 1];
  __shared__ float s_inv[8];     // 1 / valid queries of each query block (0 if none)
  __shared__ float s_kinv[32];   // 1 / valid keys of each tile of the chunk (0 if none)
  const int groups = (a.n_qb + 7) / 8;
  const int bh = blockIdx.x / groups;
  const int i0 = (blockIdx.x % groups) * 8;
  const int tid = threadIdx.x;
  const int per = a.q_block / 64;  // tiles per query block
  const long long tbase = static_cast<long long>(bh) * a.n_kb;
  if (tid < 8) {
    const int i = i0 + tid;
    int cnt = 0;
    if (i < a.n_qb)
      for (int u = i * per; u < (i + 1) * per; ++u) cnt += tile_valid_count(a.g, u);
    s_inv[tid] = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
  }
  __syncthreads();
  // qbar of the CTA's 8 query blocks (0 for a block without valid queries)
  for (int x = tid; x < 8 * D; x += 256) {
    const int qi = x / D, d = x % D;
    const int i = i0 + qi;
    float sum = 0.f;
    if (i < a.n_qb)
      for (int u = i * per; u < (i + 1) * per; ++u) sum += qsum[(tbase + u) * D + d];
    sq[qi][d] = sum * s_inv[qi];
  }
  const int qi = tid >> 5, jl = tid & 31;
  const int i = i0 + qi;
  for (int j0 = 0; j0 < a.n_kb; j0 += 32) {
    __syncthreads();
    if (tid < 32) {
      const int j = j0 + tid;
      const int cnt = j < a.n_kb ? tile_valid_count(a.g, j) : 0;
      s_kinv[tid] = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
    }
    __syncthreads();
    for (int x = tid; x < 32 * D; x += 256) {
      const int r = x / D, d = x % D;
      const int j = j0 + r;
      sk[r][d] = j < a.n_kb ? ksum[(tbase + j) * D + d] * s_kinv[r] : 0.f;
    }
    __syncthreads();
    const int j = j0 + jl;
    if (i < a.n_qb && j < a.n_kb) {
      float acc0 = 0.f, acc1 = 0.f;
#pragma unroll 8
      for (int d = 0; d < D; d += 2) {
        acc0 = fmaf(sq[qi][d], sk[jl][d], acc0);
        acc1 = fmaf(sq[qi][d + 1], sk[jl][d + 1], acc1);
      }
      out[(static_cast<long long>(bh) * a.n_qb + i) * a.n_kb + j] =
          s_kinv[jl] > 0.f ? (acc0 + acc1) * scale_log2 : -INFINITY;
    }
  }
}

// In place: row of log2 logits -> n_j 2^(s_j - max) / sum.  Rows of query blocks without
// valid queries become zero.
__global__ void __launch_bounds__(256) pooled_softmax_kernel(AttnDims a, long long rows,
                                                             float* __restrict__ m) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const int i = static_cast<int>(r % a.n_qb);
  const int per = a.q_block / 64;
  int nq = 0;
  for (int u = i * per; u < (i + 1) * per; ++u) nq += tile_valid_count(a.g, u);
  float* row = m + r * a.n_kb;
  float mx = -INFINITY;
  for (int j = lane; j < a.n_kb; j += 32) mx = fmaxf(mx, row[j]);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
  if (nq == 0 || mx == -INFINITY) {  // no valid query, or no valid key in the head
    for (int j = lane; j < a.n_kb; j += 32) row[j] = 0.f;
    return;
  }
  float sum = 0.f;
  for (int j = lane; j < a.n_kb; j += 32) {
    const float w = static_cast<float>(tile_valid_count(a.g, j)) * exp2f(row[j] - mx);
    row[j] = w;
    sum += w;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
  const float inv = 1.f / sum;
  for (int j = lane; j < a.n_kb; j += 32) row[j] *= inv;
}

size_t pooled_scratch_bytes(const AttnDims& a) {
  return 2 * static_cast<size_t>(a.batch) * a.heads * a.n_kb * a.head_dim * sizeof(float);
}

cudaError_t launch_pooled_mass(const AttnDims& a, const void* q, const void* k, float softmax_scale,
                               float* mass, void* ws, cudaStream_t stream) {
  const long long tiles = 1LL * a.batch * a.heads * a.n_kb;
  const long long rows = 1LL * a.batch * a.heads * a.n_qb;
  if (tiles == 0) return cudaSuccess;
  float* qsum = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  float* ksum = qsum + tiles * a.head_dim;
  const float sl2 = softmax_scale * 1.4426950408889634f;
  const unsigned pool_ctas = static_cast<unsigned>((tiles + 7) / 8);
  const unsigned logit_ctas = static_cast<unsigned>(1LL * a.batch * a.heads * ((a.n_qb + 7) / 8));
  const unsigned sm_ctas = static_cast<unsigned>((rows + 7) / 8);
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  if (a.head_dim == 128) {
    pool_tiles_kernel<128><<<pool_ctas, 256, 0, stream>>>(qb, kb, a.g, tiles, qsum, ksum);
    pooled_logits_kernel<128><<<logit_ctas, 256, 0, stream>>>(qsum, ksum, a, sl2, mass);
  } else {
    pool_tiles_kernel<64><<<pool_ctas, 256, 0, stream>>>(qb, kb, a.g, tiles, qsum, ksum);
    pooled_logits_kernel<64><<<logit_ctas, 256, 0, stream>>>(qsum, ksum, a, sl2, mass);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  pooled_softmax_kernel<<<sm_ctas, 256, 0, stream>>>(a, rows, mass);
  return cudaGetLastError();
}

}  // namespace bsa
