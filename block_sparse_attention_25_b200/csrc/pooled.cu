// Pooled (block-level) estimate of the block masses, for per-step ("online") top-p
// selection without a dense pass.
//
// "Sparse VideoGen2", Abstract: top-p dynamic budget control on attention between token
// clusters; with 4x4x4 tiles as the clusters, a kv block is represented by the mean of its
// valid keys and weighted by their number, a query block by the mean of its valid queries:
//   M_est[i, j] = n_j exp(scale qbar_i . kbar_j) / sum_j' n_j' exp(scale qbar_i . kbar_j').
// The result feeds bsa_topp_select like the exact masses do.
//
// Kernels:
//   pool_tiles_kernel    one warp per (bh, tile): sums of the valid rows of Q and K, 16-byte
//                        loads with eight rows in flight per lane.
//   pooled_split_kernel  qbar_i and kbar_j (sums times 1 / valid count, fp32), each cut
//                        into three bf16 parts hi + mid + lo (the fp32 value to ~2^-24),
//                        laid out as rows of six D-wide segments so that one bf16 product
//                        of a q row and a k row sums the six terms
//                        hi.hi + hi.mid + mid.hi + hi.lo + lo.hi + mid.mid.
//   pooled_logits_tc_kernel  that product on the tensor cores: a 128 x 128 tile of
//                        (query block, kv block) logits per CTA, K = 6 D, TMA-fed
//                        128-byte-swizzled stages, fp32 accumulator in TMEM; writes the
//                        log2-domain logits (-inf for tiles without valid keys).
//   pooled_softmax_kernel one warp per row: weighted softmax in place.
#include <algorithm>

#include "bsa_kernels.cuh"

namespace bsa {

// Valid rows of tile j (popcount of its slot mask).
__device__ __forceinline__ int tile_valid_count(const GridDims& g, int j) {
  return __popcll(tile_valid_mask(g, j));
}

// One warp per (bh, tile): sums of the tile's valid rows of Q and of K.  A lane reads 8
// dims (16 bytes) of a row; the warp's lane groups (two for D = 128, four for D = 64) take
// rows r = group (mod groups), each lane with eight rows' loads in flight before they are
// added.  The groups' partial sums are combined at the end by a fixed xor tree, so the
// result does not depend on timing.
template <int D>
__global__ void __launch_bounds__(256) pool_tiles_kernel(const __nv_bfloat16* __restrict__ q,
                                                         const __nv_bfloat16* __restrict__ k,
                                                         GridDims g, long long tiles,
                                                         float* __restrict__ qsum,
                                                         float* __restrict__ ksum) {
  constexpr int LPR = D / 8;         // lanes per row (16 for D = 128, 8 for D = 64)
  constexpr int RPI = 32 / LPR;      // rows per warp instruction (2 or 4)
  constexpr int kU = 8;              // row loads in flight per lane
  const long long w = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (w >= tiles) return;
  const int lane = threadIdx.x & 31;
  const int ntiles = g.Np / 64;
  const int j = static_cast<int>(w % ntiles);
  const uint64_t vm = tile_valid_mask(g, j);
  const int sub = lane / LPR;        // which of the instruction's rows
  const int d0 = (lane % LPR) * 8;
  const __nv_bfloat16* qt = q + w * 64 * D + d0;
  const __nv_bfloat16* kt = k + w * 64 * D + d0;
  float aq[8], ak[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) aq[e] = ak[e] = 0.f;
  for (int r0 = 0; r0 < 64; r0 += RPI * kU) {
    uint4 vq[kU], vk[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int r = r0 + u * RPI + sub;
      const bool ok = r < 64 && ((vm >> r) & 1ull);
      vq[u] = ok ? *reinterpret_cast<const uint4*>(qt + r * D) : make_uint4(0u, 0u, 0u, 0u);
      vk[u] = ok ? *reinterpret_cast<const uint4*>(kt + r * D) : make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const uint32_t wq[4] = {vq[u].x, vq[u].y, vq[u].z, vq[u].w};
      const uint32_t wk[4] = {vk[u].x, vk[u].y, vk[u].z, vk[u].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        aq[2 * e] += __uint_as_float(wq[e] << 16);
        aq[2 * e + 1] += __uint_as_float(wq[e] & 0xFFFF0000u);
        ak[2 * e] += __uint_as_float(wk[e] << 16);
        ak[2 * e + 1] += __uint_as_float(wk[e] & 0xFFFF0000u);
      }
    }
  }
  // combine the row groups in a fixed order (xor tree over the lanes holding the same dims)
#pragma unroll
  for (int o = LPR; o < 32; o <<= 1)
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      aq[e] += __shfl_xor_sync(0xffffffffu, aq[e], o);
      ak[e] += __shfl_xor_sync(0xffffffffu, ak[e], o);
    }
  if (sub == 0) {
    float4* oq = reinterpret_cast<float4*>(qsum + w * D + d0);
    float4* okk = reinterpret_cast<float4*>(ksum + w * D + d0);
    oq[0] = make_float4(aq[0], aq[1], aq[2], aq[3]);
    oq[1] = make_float4(aq[4], aq[5], aq[6], aq[7]);
    okk[0] = make_float4(ak[0], ak[1], ak[2], ak[3]);
    okk[1] = make_float4(ak[4], ak[5], ak[6], ak[7]);
  }
}

// qbar / kbar rows, split for the tensor cores: row r of qs is query block i of head bh
// (r = bh * n_qb + i), row r of ks kv block j (r = bh * n_kb + j); each row holds six
// D-wide bf16 segments, q: [hi, hi, mid, hi, lo, mid], k: [hi, mid, hi, lo, hi, mid].  A
// block without valid rows is all zeros.  One thread per (row, 8 dims): two 16-byte loads
// of the sums, six 16-byte stores.
template <int D>
__global__ void __launch_bounds__(256) pooled_split_kernel(const float* __restrict__ qsum,
                                                           const float* __restrict__ ksum,
                                                           AttnDims a,
                                                           __nv_bfloat16* __restrict__ qs,
                                                           __nv_bfloat16* __restrict__ ks) {
  constexpr int G = D / 8;  // 8-dim groups per row
  const long long bhn = static_cast<long long>(a.batch) * a.heads;
  const long long nq = bhn * a.n_qb, nk = bhn * a.n_kb;
  const long long idx = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long row = idx / G;
  const int d0 = static_cast<int>(idx - row * G) * 8;
  if (row >= nq + nk) return;
  float x[8];
  __nv_bfloat16* dst;
  const bool isq = row < nq;
  if (isq) {
    const long long bh = row / a.n_qb;
    const int i = static_cast<int>(row - bh * a.n_qb);
    const int per = a.q_block / 64;  // tiles per query block
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = 0.f;
    int cnt = 0;
    for (int u = i * per; u < (i + 1) * per; ++u) {
      const float4* src = reinterpret_cast<const float4*>(qsum + (bh * a.n_kb + u) * D + d0);
      const float4 v0 = src[0], v1 = src[1];
      x[0] += v0.x; x[1] += v0.y; x[2] += v0.z; x[3] += v0.w;
      x[4] += v1.x; x[5] += v1.y; x[6] += v1.z; x[7] += v1.w;
      cnt += tile_valid_count(a.g, u);
    }
    const float inv = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = cnt > 0 ? x[e] * inv : 0.f;
    dst = qs + row * (6 * D) + d0;
  } else {
    const long long rk = row - nq;
    const long long bh = rk / a.n_kb;
    const int j = static_cast<int>(rk - bh * a.n_kb);
    const int cnt = tile_valid_count(a.g, j);
    const float inv = cnt > 0 ? 1.f / static_cast<float>(cnt) : 0.f;
    const float4* src = reinterpret_cast<const float4*>(ksum + (bh * a.n_kb + j) * D + d0);
    const float4 v0 = src[0], v1 = src[1];
    const float t[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = cnt > 0 ? t[e] * inv : 0.f;
    dst = ks + rk * (6 * D) + d0;
  }
  uint4 hi, mid, lo;
  uint32_t* ph = reinterpret_cast<uint32_t*>(&hi);
  uint32_t* pm = reinterpret_cast<uint32_t*>(&mid);
  uint32_t* pl = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
  for (int e = 0; e < 8; e += 2) {
    float h2[2], m2[2], l2[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const __nv_bfloat16 hb = __float2bfloat16_rn(x[e + u]);
      const float r1 = x[e + u] - __bfloat162float(hb);  // exact
      const __nv_bfloat16 mb = __float2bfloat16_rn(r1);
      const __nv_bfloat16 lb = __float2bfloat16_rn(r1 - __bfloat162float(mb));
      h2[u] = __bfloat162float(hb);
      m2[u] = __bfloat162float(mb);
      l2[u] = __bfloat162float(lb);
    }
    // the parts are bf16 values already, so packing them back is exact
    ph[e / 2] = pack_bf16x2(h2[0], h2[1]);
    pm[e / 2] = pack_bf16x2(m2[0], m2[1]);
    pl[e / 2] = pack_bf16x2(l2[0], l2[1]);
  }
  const uint4 seg[6] = {hi, isq ? hi : mid, isq ? mid : hi, isq ? hi : lo, isq ? lo : hi, mid};
#pragma unroll
  for (int t = 0; t < 6; ++t) *reinterpret_cast<uint4*>(dst + t * D) = seg[t];
}

// Logits in log2 units: scale * log2(e) * qbar_i . kbar_j, -inf for tiles without valid keys
// (the softmax kernel adds log2(n_j)).  One CTA of 128 threads per 128 x 128 tile: thread 0
// of warp 0 issues the TMA loads of 64-column (128-byte) chunks of the split rows into a
// kPlStages-deep ring, thread 0 of warp 1 the MMAs (M = N = 128, K = 16 each) into one
// fp32 TMEM accumulator, and all four warps read it back (a thread per query block).
constexpr int kPlStages = 3;
constexpr int kPlStage = 2 * 128 * 128;  // A and B chunks of one stage, bytes
constexpr int kPlAlloc = kPlStages * kPlStage + 1024 + 1024;

template <int D>
__global__ void __launch_bounds__(128) pooled_logits_tc_kernel(
    const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
    AttnDims a, float scale_log2, float* __restrict__ out, uint32_t* status) {
  constexpr int KC = 6 * D / 64;  // 128-byte chunks along the product's K
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kPlStages * kPlStage);
  uint64_t* bar_full = bars;
  uint64_t* bar_empty = bars + kPlStages;
  uint64_t* bar_acc = bars + 2 * kPlStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_acc + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* jvalid = const_cast<int*>(abort_flag) + 1;  // [128]

  const int ti = (a.n_qb + 127) / 128;
  const int tj = (a.n_kb + 127) / 128;
  const int per_bh = ti * tj;
  const int bh = blockIdx.x / per_bh;
  const int rem = blockIdx.x - bh * per_bh;
  const int i0 = (rem / tj) * 128;
  const int j0 = (rem % tj) * 128;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kPlStages; ++st) {
      mbar_init(bar_full + st, 1);
      mbar_init(bar_empty + st, 1);
    }
    mbar_init(bar_acc, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  {
    const int j = j0 + threadIdx.x;
    jvalid[threadIdx.x] = (j < a.n_kb && tile_valid_count(a.g, j) > 0) ? 1 : 0;
  }
  if (warp == 0) tmem_alloc(tmem_slot, 128);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0 && lane == 0) {
    // ------------------------------------------------------------ TMA producer
    prefetch_tensormap(&tm_a);
    prefetch_tensormap(&tm_b);
    for (int kc = 0; kc < KC; ++kc) {
      const int st = kc % kPlStages;
      if (kc >= kPlStages && !mbar_wait(bar_empty + st, ((kc / kPlStages) - 1) & 1, abort_flag,
                                        status, DETAIL_WAIT_K_EMPTY))
        break;
      uint8_t* sa = smem + st * kPlStage;
      mbar_arrive_expect_tx(bar_full + st, kPlStage);
      tma_load_3d(sa, &tm_a, bar_full + st, kc * 64, i0, bh);
      tma_load_3d(sa + 128 * 128, &tm_b, bar_full + st, kc * 64, j0, bh);
    }
  } else if (warp == 1 && lane == 0) {
    // ------------------------------------------------------------ MMA issuer
    const uint32_t idesc = make_idesc(1u, 0u, 128u, 128u);
    for (int kc = 0; kc < KC; ++kc) {
      const int st = kc % kPlStages;
      if (!mbar_wait(bar_full + st, (kc / kPlStages) & 1, abort_flag, status, DETAIL_WAIT_K_FULL))
        break;
      tc_fence_after();
      const uint32_t sa = smem_u32(smem + st * kPlStage);
      const uint64_t ad = make_sdesc_sw128(sa, 16, 1024);
      const uint64_t bd = make_sdesc_sw128(sa + 128 * 128, 16, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)
        mma_f16_ss(tmem, ad + static_cast<uint64_t>((kk * 32) >> 4),
                   bd + static_cast<uint64_t>((kk * 32) >> 4), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
      mma_commit(bar_empty + st);
    }
    // Whatever happened, every issued MMA completes before the accumulator is read or
    // the tensor memory released.
    mma_commit(bar_acc);
    mbar_wait_drain(bar_acc, 0, status, DETAIL_WAIT_O_FULL);
  }
  __syncwarp();
  // ------------------------------------------------------------ epilogue
  const bool got = __all_sync(0xffffffffu,
                              mbar_wait(bar_acc, 0, abort_flag, status, DETAIL_WAIT_O_FULL));
  tc_fence_after();
  const int i = i0 + warp * 32 + lane;
  const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
  float* orow = out + (static_cast<long long>(bh) * a.n_qb + i) * a.n_kb;
  const bool vec = (a.n_kb & 3) == 0;  // rows start 16-byte aligned
#pragma unroll 1
  for (int c0 = 0; c0 < 128; c0 += 32) {
    float v[32];
    tmem_ld32(lane_base + c0, v);
    tmem_ld_wait();
    if (!got || i >= a.n_qb) continue;
#pragma unroll
    for (int c = 0; c < 32; ++c) v[c] = jvalid[c0 + c] ? v[c] * scale_log2 : -INFINITY;
    const int j = j0 + c0;
    if (vec && j + 31 < a.n_kb) {
#pragma unroll
      for (int c = 0; c < 32; c += 4)
        *reinterpret_cast<float4*>(orow + j + c) = make_float4(v[c], v[c + 1], v[c + 2], v[c + 3]);
    } else {
#pragma unroll
      for (int c = 0; c < 32; ++c)
        if (j + c < a.n_kb) orow[j + c] = v[c];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 128);
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

// Scratch after the status header: per-tile sums qsum, ksum fp32 [bh][n_kb][D], then the
// split rows qs bf16 [bh][n_qb][6D] and ks bf16 [bh][n_kb][6D] (16-byte aligned rows).
size_t pooled_scratch_bytes(const AttnDims& a) {
  const size_t bhn = static_cast<size_t>(a.batch) * a.heads;
  return 2 * bhn * a.n_kb * a.head_dim * sizeof(float) +
         bhn * (static_cast<size_t>(a.n_qb) + a.n_kb) * 6 * a.head_dim * sizeof(__nv_bfloat16);
}

template <int D>
static cudaError_t launch_pooled_logits(const AttnDims& a, const float* qsum, const float* ksum,
                                        __nv_bfloat16* qs, __nv_bfloat16* ks, float sl2,
                                        float* mass, uint32_t* status, cudaStream_t stream) {
  const long long bhn = 1LL * a.batch * a.heads;
  const long long rows = bhn * (a.n_qb + a.n_kb);
  pooled_split_kernel<D><<<static_cast<unsigned>((rows * (D / 8) + 255) / 256), 256, 0, stream>>>(
      qsum, ksum, a, qs, ks);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap ta, tb;
  e = encode_tmap_3d(&ta, qs, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 6 * D, a.n_qb,
                     static_cast<int>(bhn), 64, 128);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tb, ks, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 6 * D, a.n_kb,
                     static_cast<int>(bhn), 64, 128);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(pooled_logits_tc_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           kPlAlloc);
  if (e != cudaSuccess) return e;
  const unsigned ctas = static_cast<unsigned>(bhn * ((a.n_qb + 127) / 128) * ((a.n_kb + 127) / 128));
  pooled_logits_tc_kernel<D><<<ctas, 128, kPlAlloc, stream>>>(ta, tb, a, sl2, mass, status);
  return cudaGetLastError();
}

cudaError_t launch_pooled_mass(const AttnDims& a, const void* q, const void* k, float softmax_scale,
                               float* mass, void* ws, cudaStream_t stream) {
  const long long tiles = 1LL * a.batch * a.heads * a.n_kb;
  const long long rows = 1LL * a.batch * a.heads * a.n_qb;
  if (tiles == 0) return cudaSuccess;
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  float* qsum = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  float* ksum = qsum + tiles * a.head_dim;
  __nv_bfloat16* qs = reinterpret_cast<__nv_bfloat16*>(ksum + tiles * a.head_dim);
  __nv_bfloat16* ks = qs + rows * 6 * a.head_dim;
  const float sl2 = softmax_scale * 1.4426950408889634f;
  const unsigned pool_ctas = static_cast<unsigned>((tiles + 7) / 8);
  // a warp per row, CTAs looping over rows: the weight table is built once per CTA
  const unsigned sm_ctas = static_cast<unsigned>(std::min<long long>((rows + 7) / 8, 148LL * 8));
  const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q);
  const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k);
  cudaError_t e;
  if (a.head_dim == 128) {
    pool_tiles_kernel<128><<<pool_ctas, 256, 0, stream>>>(qb, kb, a.g, tiles, qsum, ksum);
    e = launch_pooled_logits<128>(a, qsum, ksum, qs, ks, sl2, mass, status, stream);
  } else {
    pool_tiles_kernel<64><<<pool_ctas, 256, 0, stream>>>(qb, kb, a.g, tiles, qsum, ksum);
    e = launch_pooled_logits<64>(a, qsum, ksum, qs, ks, sl2, mass, status, stream);
  }
  if (e != cudaSuccess) return e;
  pooled_softmax_kernel<<<sm_ctas, 256, 0, stream>>>(a, rows, mass);
  return cudaGetLastError();
}

}  // namespace bsa
