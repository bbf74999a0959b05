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
//   pooled_logits_kernel a register-tiled qbar . kbar product per (bh): 64 x 64 logits per
//                        CTA, 4 x 4 per thread; writes the log2-domain logits into the
//                        output tensor.
//   pooled_softmax_kernel one warp per row: weighted softmax in place.
#include <algorithm>

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
// (the softmax kernel adds log2(n_j)).  A register-tiled product per (bh): a CTA of 256
// threads computes a 128 x 128 tile of (query block, kv block) logits, 8 x 8 per thread
// (rows 4ty..4ty+3 and 64+4ty.., columns likewise, so each 16-byte shared load of a warp is
// conflict-free); the head dimension is staged 16 at a time in shared memory as
// [d][block].  qbar and kbar are formed while staging: sums of the block's tiles times
// 1 / valid count (0 for an empty block).  Every logit sums over d in order 0..D-1
// (deterministic).
constexpr int kLgTile = 128;
constexpr int kLgK = 16;

template <int D>
__global__ void __launch_bounds__(256) pooled_logits_kernel(const float* __restrict__ qsum,
                                                            const float* __restrict__ ksum,
                                                            AttnDims a, float scale_log2,
                                                            float* __restrict__ out) {
  __shared__ __align__(16) float sa[kLgK][kLgTile];
  __shared__ __align__(16) float sb[kLgK][kLgTile];
  __shared__ float s_qinv[kLgTile];
  __shared__ float s_kinv[kLgTile];
  const int ti = (a.n_qb + kLgTile - 1) / kLgTile;
  const int tj = (a.n_kb + kLgTile - 1) / kLgTile;
  const int per_bh = ti * tj;
  const int bh = blockIdx.x / per_bh;
  const int rem = blockIdx.x - bh * per_bh;
  const int i0 = (rem / tj) * kLgTile;
  const int j0 = (rem % tj) * kLgTile;
  const int tid = threadIdx.x;
  const int per = a.q_block / 64;  // tiles per query block
  const long long tbase = static_cast<long long>(bh) * a.n_kb;
  if (tid < kLgTile) {
    const int i = i0 + tid;
    int cnt = 0;
    if (i < a.n_qb)
      for (int u = i * per; u < (i + 1) * per; ++u) cnt += tile_valid_count(a.g, u);
    s_qinv[tid] = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
  } else {
    const int j = j0 + tid - kLgTile;
    const int cnt = j < a.n_kb ? tile_valid_count(a.g, j) : 0;
    s_kinv[tid - kLgTile] = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
  }
  const int ty = tid >> 4, tx = tid & 15;
  float acc[8][8];
#pragma unroll
  for (int r = 0; r < 8; ++r)
#pragma unroll
    for (int c = 0; c < 8; ++c) acc[r][c] = 0.f;
  for (int d0 = 0; d0 < D; d0 += kLgK) {
    __syncthreads();
    // stage 128 blocks x 16 dims of qbar and kbar, transposed to [d][block]: two 16-byte
    // loads of four consecutive dims per thread and matrix (128 x 16 = 2 x 256 x 4)
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int f = tid + 256 * h;
      const int blk = f >> 2, dq = (f & 3) * 4;
      const int i = i0 + blk, j = j0 + blk;
      float4 qv = make_float4(0.f, 0.f, 0.f, 0.f), kv = qv;
      if (i < a.n_qb) {
        for (int u = i * per; u < (i + 1) * per; ++u) {
          const float4 t = *reinterpret_cast<const float4*>(qsum + (tbase + u) * D + d0 + dq);
          qv.x += t.x;
          qv.y += t.y;
          qv.z += t.z;
          qv.w += t.w;
        }
        const float fq = s_qinv[blk];
        qv = make_float4(qv.x * fq, qv.y * fq, qv.z * fq, qv.w * fq);
      }
      if (j < a.n_kb) {
        const float4 t = *reinterpret_cast<const float4*>(ksum + (tbase + j) * D + d0 + dq);
        const float fk = s_kinv[blk];
        kv = make_float4(t.x * fk, t.y * fk, t.z * fk, t.w * fk);
      }
      sa[dq + 0][blk] = qv.x;
      sa[dq + 1][blk] = qv.y;
      sa[dq + 2][blk] = qv.z;
      sa[dq + 3][blk] = qv.w;
      sb[dq + 0][blk] = kv.x;
      sb[dq + 1][blk] = kv.y;
      sb[dq + 2][blk] = kv.z;
      sb[dq + 3][blk] = kv.w;
    }
    __syncthreads();
#pragma unroll
    for (int d = 0; d < kLgK; ++d) {
      const float4 a0 = *reinterpret_cast<const float4*>(&sa[d][4 * ty]);
      const float4 a1 = *reinterpret_cast<const float4*>(&sa[d][64 + 4 * ty]);
      const float4 b0 = *reinterpret_cast<const float4*>(&sb[d][4 * tx]);
      const float4 b1 = *reinterpret_cast<const float4*>(&sb[d][64 + 4 * tx]);
      const float ar[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float br[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int r = 0; r < 8; ++r)
#pragma unroll
        for (int c = 0; c < 8; ++c) acc[r][c] = fmaf(ar[r], br[c], acc[r][c]);
    }
  }
  const bool vec = (a.n_kb & 3) == 0;  // rows start 16-byte aligned
#pragma unroll
  for (int r = 0; r < 8; ++r) {
    const int i = i0 + (r < 4 ? 4 * ty + r : 64 + 4 * ty + r - 4);
    if (i >= a.n_qb) continue;
    float* orow = out + (static_cast<long long>(bh) * a.n_qb + i) * a.n_kb;
#pragma unroll
    for (int g = 0; g < 2; ++g) {
      const int cl = 64 * g + 4 * tx;  // first of four columns inside the tile
      const int j = j0 + cl;
      float v[4];
#pragma unroll
      for (int c = 0; c < 4; ++c)
        v[c] = s_kinv[cl + c] > 0.f ? acc[r][4 * g + c] * scale_log2 : -INFINITY;
      if (vec && j + 3 < a.n_kb) {
        *reinterpret_cast<float4*>(orow + j) = make_float4(v[0], v[1], v[2], v[3]);
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (j + c < a.n_kb) orow[j + c] = v[c];
      }
    }
  }
}

// In place: row of log2 logits -> n_j 2^(s_j - max) / sum.  Rows of query blocks without
// valid queries become zero.  A warp per row, looping over rows; rows of up to
// 32 * kSmPerLane kv blocks stay in registers (one read, one write) with the weights n_j
// from a per-CTA table; longer rows take three passes over memory.  Both give the same
// per-lane order of operations, hence the same results.
constexpr int kSmPerLane = 72;
__global__ void __launch_bounds__(256) pooled_softmax_kernel(AttnDims a, long long rows,
                                                             float* __restrict__ m) {
  __shared__ float wt[32 * kSmPerLane];
  const bool in_regs = a.n_kb <= 32 * kSmPerLane;
  if (in_regs) {
    for (int j = threadIdx.x; j < a.n_kb; j += blockDim.x)
      wt[j] = static_cast<float>(tile_valid_count(a.g, j));
    __syncthreads();
  }
  const int lane = threadIdx.x & 31;
  const int per = a.q_block / 64;
  const int nu = (a.n_kb + 31) >> 5;
  for (long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5); r < rows;
       r += static_cast<long long>(gridDim.x) * 8) {
    const int i = static_cast<int>(r % a.n_qb);
    int nq = 0;
    for (int u = i * per; u < (i + 1) * per; ++u) nq += tile_valid_count(a.g, u);
    float* row = m + r * a.n_kb;
    if (in_regs) {
      float v[kSmPerLane];
      float mx = -INFINITY;
#pragma unroll
      for (int u = 0; u < kSmPerLane; ++u) {
        const int j = lane + 32 * u;
        v[u] = (u < nu && j < a.n_kb) ? row[j] : -INFINITY;
        mx = fmaxf(mx, v[u]);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (nq == 0 || mx == -INFINITY) {  // no valid query, or no valid key in the head
#pragma unroll
        for (int u = 0; u < kSmPerLane; ++u) {
          const int j = lane + 32 * u;
          if (u < nu && j < a.n_kb) row[j] = 0.f;
        }
        continue;
      }
      float sum = 0.f;
#pragma unroll
      for (int u = 0; u < kSmPerLane; ++u) {
        const int j = lane + 32 * u;
        if (u < nu && j < a.n_kb) {
          v[u] = wt[j] * exp2f(v[u] - mx);
          sum += v[u];
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, o);
      const float inv = 1.f / sum;
#pragma unroll
      for (int u = 0; u < kSmPerLane; ++u) {
        const int j = lane + 32 * u;
        if (u < nu && j < a.n_kb) row[j] = v[u] * inv;
      }
    } else {
      float mx = -INFINITY;
      for (int j = lane; j < a.n_kb; j += 32) mx = fmaxf(mx, row[j]);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
      if (nq == 0 || mx == -INFINITY) {
        for (int j = lane; j < a.n_kb; j += 32) row[j] = 0.f;
        continue;
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
  }
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
  const unsigned logit_ctas = static_cast<unsigned>(1LL * a.batch * a.heads *
                                                    ((a.n_qb + kLgTile - 1) / kLgTile) *
                                                    ((a.n_kb + kLgTile - 1) / kLgTile));
  // a warp per row, CTAs looping over rows: the weight table is built once per CTA
  const unsigned sm_ctas = static_cast<unsigned>(std::min<long long>((rows + 7) / 8, 148LL * 8));
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
