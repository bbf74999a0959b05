// Dense calibration pass: exact softmax attention mass of every (query block, kv block)
// pair, sm_100a.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: the method measures exact block attention masses at one early dense step.
//
// mass[b,h,i,j] = mean over the valid queries q of block i of
//                 sum over the valid keys k of block j of softmax_k(scale * q.k).
//
// One CTA owns 256 query slots (two M=128 tiles) and walks every kv block once, two blocks
// (N = 128 keys) per step: S = Q K^T on the tensor cores, then per row and kv block j
//   e[r,j] = sum over the keys of block j of exp2(S*c - m_r),
// with m_r a lazy reference max: it is raised only when a block's max exceeds it by more
// than kRescaleLog2 (every exponential then stays <= 2^kRescaleLog2, far from overflow).
// On such a raise -- rare: only a row whose early blocks are far below its later ones --
// the row's sum and the block sums it has already written are multiplied by
// exp2(m_old - m_new) in place.  Every exponential of the calibration is computed once.
// e[r,j] goes to the CTA's slice of the workspace; at the end of the CTA
//   mass[i,j] = (1 / valid queries of i) * sum over the rows r of query block i of
//               e[r,j] * exp2(m_r,half(j) - m_r) / l_r,
// in a fixed order (deterministic), where the two threads of a row (one per column half)
// each kept their own reference max m_r,half and sum.
// The slice is claimed from a pool when the CTA starts and given back when it ends, so no
// two live CTAs ever write the same slice, wherever and whenever they run.
// Warp roles (576 threads): warps 0-7 and 10-17 own the rows, two threads per row: warps
// 0-3 / 4-7 take the first kv block of each step of tile 0 / 1, warps 10-13 / 14-17 the
// second (a warp reads the TMEM lane quarter of its sub-partition, warp % 4); warp 8 is
// the TMA producer (K only), warp 9 the MMA issuer and TMEM owner.  Four row warps per
// sub-partition keep the exponential unit fed.  TMEM holds two S buffers per tile
// (4 x 128 columns), so the tensor core computes step s+1 while step s is reduced.
#include "bsa_kernels.cuh"

namespace bsa {

namespace mass {
constexpr int kThreads = 576;
constexpr int kRowsPerCta = 256;
// 18 warps: 5 share sub-partitions 0 and 1, whose 16K-register files then allow 96
// registers per thread.
constexpr int kMaxRegs = 96;
// Lazy reference max (log2 units): exponentials stay <= 2^64 and a row's sum below
// 2^64 * keys, so fp32 cannot overflow for any sequence length the ABI admits.
constexpr float kRescaleLog2 = 64.0f;
}  // namespace mass

struct MassParams {
  AttnDims a;
  float* mass;
  uint32_t* status;
  float* scratch;  // [kMassSlots][n_kb][256] unnormalised row-block sums
  uint32_t* pool;  // kMassSlots bits: slices held by live CTAs
  float scale_log2;
};

template <int D>
struct MassSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kQTile = 128 * D * 2;
  static constexpr int kKStage = 128 * D * 2;
  static constexpr int kKStages = (D == 128) ? 4 : 6;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = 2 * kQTile;
  static constexpr int kRedOff = kKOff + kKStages * kKStage;   // float [2 half][256] row weights
  static constexpr int kXchOff = kRedOff + 2 * 256 * 4;         // float [2 tile][2 half][128 row][2]
  static constexpr int kBarOff = kXchOff + 2 * 2 * 128 * 2 * 4;
  static constexpr int kBytes = kBarOff + 512;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __maxnreg__(mass::kMaxRegs)
    block_mass_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k, const MassParams p) {
  using L = MassSmem<D>;
  constexpr int KS = L::kKStages;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte-swizzled operand tiles need 1024-byte alignment in the shared window.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_kempty = bar_kfull + KS;
  uint64_t* bar_sfull = bar_kempty + KS;  // [tile][buf] = 4
  uint64_t* bar_sempty = bar_sfull + 4;   // [tile][buf] = 4
  uint64_t* bar_drain = bar_sempty + 4;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* nvalid_sm = reinterpret_cast<int*>(tmem_slot + 2);  // [2 half][2 tile][4 warp]
  int* slice_sm = reinterpret_cast<int*>(tmem_slot + 20);  // this CTA's scratch slice
  float* row_w = reinterpret_cast<float*>(smem + L::kRedOff);  // [half][row] weight of e
  float* xch = reinterpret_cast<float*>(smem + L::kXchOff);

  const AttnDims& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int bh = cta / a.n_cta_per_head;
  const int row0 = (cta - bh * a.n_cta_per_head) * mass::kRowsPerCta;
  const int nsteps = (a.n_kb + 1) >> 1;  // two kv blocks per step

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(bar_kfull + i, 1);
      mbar_init(bar_kempty + i, 1);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(bar_sfull + i, 1);
      mbar_init(bar_sempty + i, 256);
    }
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    *slice_sm = claim_mass_slice(p.pool, p.status);
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 8) {
    if (lane == 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      mbar_arrive_expect_tx(bar_q, 2 * L::kQTile);
      for (int t = 0; t < 2; ++t)
        for (int ch = 0; ch < L::kChunks; ++ch)
          tma_load_3d(smem + L::kQOff + t * L::kQTile + ch * (128 * 128), &tm_q, bar_q, ch * 64,
                      row0 + t * 128, bh);
      for (int s = 0; s < nsteps; ++s) {
        const int nb = (2 * s + 1 < a.n_kb) ? 2 : 1;
        const int ks = s % KS;
        if (s >= KS && !mbar_wait(bar_kempty + ks, ((s / KS) - 1) & 1, abort_flag, p.status,
                                  DETAIL_WAIT_K_EMPTY))
          break;
        mbar_arrive_expect_tx(bar_kfull + ks, nb * 64 * D * 2);
        uint8_t* kst = smem + L::kKOff + ks * L::kKStage;
        for (int ch = 0; ch < L::kChunks; ++ch) {
          tma_load_3d(kst + ch * (128 * 128), &tm_k, bar_kfull + ks, ch * 64, 2 * s * 64, bh);
          if (nb == 2)
            tma_load_3d(kst + ch * (128 * 128) + 64 * 128, &tm_k, bar_kfull + ks, ch * 64,
                        (2 * s + 1) * 64, bh);
        }
      }
    }
  } else if (warp == 9) {
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + L::kQOff);
      const uint32_t k_base = smem_u32(smem + L::kKOff);
      bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, DETAIL_WAIT_Q);
      for (int s = 0; s < nsteps && ok; ++s) {
        const int nb = (2 * s + 1 < a.n_kb) ? 2 : 1;
        const int ks = s % KS;
        const int buf = s & 1;
        const uint32_t idesc = make_idesc(1u, 0u, 128u, static_cast<uint32_t>(nb * 64));
        if (!mbar_wait(bar_kfull + ks, (s / KS) & 1, abort_flag, p.status, DETAIL_WAIT_K_FULL)) {
          ok = false;
          break;
        }
        const uint32_t kb = k_base + ks * L::kKStage;
        for (int t = 0; t < 2; ++t) {
          if (s >= 2 && !mbar_wait(bar_sempty + 2 * t + buf, ((s >> 1) - 1) & 1, abort_flag,
                                   p.status, DETAIL_WAIT_P_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t qb = q_base + t * L::kQTile;
          const uint32_t s_tmem = tmem + (2 * t + buf) * 128;
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t off = (kk >> 2) * (128 * 128) + (kk & 3) * 32;
            mma_f16_ss(s_tmem, make_sdesc_sw128(qb + off, 16, 1024),
                       make_sdesc_sw128(kb + off, 16, 1024), idesc, kk > 0 ? 1u : 0u);
          }
          mma_commit(bar_sfull + 2 * t + buf);
        }
        if (!ok) break;
        mma_commit(bar_kempty + ks);
      }
      mma_commit(bar_drain);
      mbar_wait_drain(bar_drain, 0, p.status, DETAIL_WAIT_O_FULL);
    }
  } else {
    const int h = warp >= 10 ? 1 : 0;           // which kv block of each step (column half)
    const int t = (h ? warp - 10 : warp) >> 2;  // query tile
    const int wq = warp & 3;                    // TMEM lane quarter = the warp's sub-partition
    const int row = wq * 32 + lane;
    const int local = t * 128 + row;
    const int slot = row0 + local;
    const bool q_valid = slot < a.g.Np && slot_valid(a.g, slot);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const float c = p.scale_log2;
    const int gbar = 1 + 2 * t + h;  // named barrier of the 4 warps of (tile, half)
    // valid queries per warp (for the per-query-block means at the end)
    const int wcount = __popc(__ballot_sync(0xffffffffu, q_valid));
    if (lane == 0) nvalid_sm[(h * 2 + t) * 4 + wq] = wcount;
    named_bar_sync(gbar, 128);
    // this CTA's scratch slice: [n_kb][256] row-block sums (none: the claim timed out, no
    // masses are written and the status header says so)
    const int slice = *slice_sm;
    const bool have_slice = slice >= 0;
    float* sc = p.scratch + static_cast<size_t>(have_slice ? slice : 0) * 256 * a.n_kb;

    float m_ref = -INFINITY, l_run = 0.f;  // this half's reference max (log2 units) and sum
    bool ok = true;
    // tile coordinates of this half's kv block 2*s + h, advanced incrementally (no
    // division inside the loop: integer division shares the pipe of the exponentials)
    int tw = 0, th = 0, tt = 0;
    tile_advance(a.g, h, tw, th, tt);
    for (int s = 0; s < nsteps; ++s) {
      const int nb = (2 * s + 1 < a.n_kb) ? 2 : 1;
      const bool mine = h < nb;  // this half has a kv block in this step
      const int buf = s & 1;
      // A warp that gives up keeps stepping (without touching TMEM) so that every warp of
      // the group passes the same named barriers.
      bool got = ok ? mbar_wait(bar_sfull + 2 * t + buf, (s >> 1) & 1, abort_flag, p.status,
                                DETAIL_WAIT_S_FULL)
                    : false;
      got = __all_sync(0xffffffffu, got);
      ok = got;
      if (got) {
        float sv[64];
        tc_fence_after();
        if (mine) {
          const uint32_t s_addr = lane_base + (2 * t + buf) * 128 + 64 * h;
          tmem_ld64(s_addr, sv);  // one load instruction (107.7 vs 108.4 ms at 720p)
          tmem_ld_wait();
        }
        tc_fence_before();
        mbar_arrive(bar_sempty + 2 * t + buf);
        if (mine) {
          // Pad keys -> -inf (same for every row).
          if (4 * tt + 4 > a.g.T || 4 * th + 4 > a.g.H || 4 * tw + 4 > a.g.W) {
            const uint64_t mk = tile_valid_mask_at(a.g, tw, th, tt);
            const uint32_t mw[2] = {static_cast<uint32_t>(mk), static_cast<uint32_t>(mk >> 32)};
#pragma unroll
            for (int i = 0; i < 64; ++i) sv[i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? sv[i] : -INFINITY;
          }
          float mx[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) mx[i] = sv[i];
#pragma unroll
          for (int i = 8; i < 64; ++i) mx[i & 7] = fmaxf(mx[i & 7], sv[i]);
          const float mb = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                 fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                           c;  // c > 0, so -inf stays -inf
          if (mb > m_ref + mass::kRescaleLog2) {
            // Raise the reference (the first block always does).  Sums formed against the
            // old one are scaled to the new; nothing was formed while it was -inf.
            if (m_ref != -INFINITY) {
              const float f = fast_exp2(m_ref - mb);
              l_run *= f;
              if (have_slice)
                for (int j = h; j < 2 * s; j += 2) sc[static_cast<size_t>(j) * 256 + local] *= f;
            }
            m_ref = mb;
          }
          float e = 0.f;
          if (m_ref != -INFINITY) {
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int i = 0; i < 64; ++i) acc[i & 3] += fast_exp2(fmaf(sv[i], c, -m_ref));
            e = (acc[0] + acc[1]) + (acc[2] + acc[3]);
          }
          l_run += e;
          if (have_slice) sc[static_cast<size_t>(2 * s + h) * 256 + local] = e;
        }
      }
      tile_advance(a.g, 2, tw, th, tt);
    }

    // ------------------------------------------------------------ masses
    // The halves' (reference max, sum) pairs -> the row's max m and sum l; half h's block
    // sums are weighted by exp2(m_h - m) / l.  Then mass[i, j] = (1 / valid queries of i) *
    // sum_r e[r, j] * weight_r,half(j) over the rows of query block i, in row order, by all
    // 512 row threads over the CTA's (query block, kv block) outputs.
    xch[((t * 2 + h) * 128 + row) * 2] = m_ref;
    xch[((t * 2 + h) * 128 + row) * 2 + 1] = l_run;
    named_bar_sync(5 + t, 256);
    {
      const float m0 = xch[((t * 2 + 0) * 128 + row) * 2];
      const float m1 = xch[((t * 2 + 1) * 128 + row) * 2];
      const float mr = fmaxf(m0, m1);
      const float f0 = m0 == -INFINITY ? 0.f : fast_exp2(m0 - mr);
      const float f1 = m1 == -INFINITY ? 0.f : fast_exp2(m1 - mr);
      const float l = xch[((t * 2 + 0) * 128 + row) * 2 + 1] * f0 +
                      xch[((t * 2 + 1) * 128 + row) * 2 + 1] * f1;
      row_w[h * 256 + local] = (q_valid && ok && l > 0.f) ? (h ? f1 : f0) / l : 0.f;
    }
    named_bar_sync(7, 512);  // every row's block sums and 1 / l_r are written
    if (have_slice) {
      const int rt = (h ? warp - 10 : warp) * 32 + lane + 256 * h;  // 0 .. 511
      const int warps_per_qb = a.q_block / 32;  // 2 or 4
      const int nq_cta = mass::kRowsPerCta / a.q_block;
      const int qb0 = row0 / a.q_block;
      for (int o = rt; o < nq_cta * a.n_kb; o += 512) {
        const int qi = o / a.n_kb;
        const int j = o - qi * a.n_kb;
        const int qb = qb0 + qi;
        if (qb >= a.n_qb) continue;
        int nvq = 0;
        for (int w = 0; w < warps_per_qb; ++w) {
          const int r0 = qi * a.q_block + 32 * w;  // first row of the warp's 32 in the CTA
          nvq += nvalid_sm[(r0 >> 7) * 4 + ((r0 & 127) >> 5)];
        }
        const float* col = sc + static_cast<size_t>(j) * 256 + qi * a.q_block;
        const float* w = row_w + (j & 1) * 256 + qi * a.q_block;  // block j is half j & 1's
        float tot = 0.f;
        for (int r = 0; r < a.q_block; r += 4) {
          const float4 ev = *reinterpret_cast<const float4*>(col + r);
          tot += ev.x * w[r];
          tot += ev.y * w[r + 1];
          tot += ev.z * w[r + 2];
          tot += ev.w * w[r + 3];
        }
        p.mass[(static_cast<long long>(bh) * a.n_qb + qb) * a.n_kb + j] =
            nvq > 0 ? tot / static_cast<float>(nvq) : 0.f;
      }
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
  if (threadIdx.x == 0) release_mass_slice(p.pool, *slice_sm);
}

// Scratch after the status header: the slice pool's bitmap, then kMassSlots slices of
// n_kb x 256 fp32 row-block sums.
size_t mass_scratch_bytes(const AttnDims& a) {
  return kMassPoolBytes +
         static_cast<size_t>(kMassSlots) * 256 * static_cast<size_t>(a.n_kb) * sizeof(float);
}

template <int D>
static cudaError_t launch_mass(const AttnDims& a, const void* q, const void* k,
                               const MassParams& prm, long long ctas, cudaStream_t stream) {
  using L = MassSmem<D>;
  CUtensorMap tq, tk;
  const int bh = a.batch * a.heads;
  cudaError_t e = encode_tmap_3d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.g.Np, bh, 64, 128);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.g.Np, bh, 64, 64);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(block_mass_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::kAlloc);
  if (e != cudaSuccess) return e;
  // one CTA per SM, so the live CTAs (at most the SM count) never exhaust the kMassSlots
  // slices and no claim waits
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, block_mass_kernel<D>, mass::kThreads,
                                                    L::kAlloc);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorInvalidConfiguration;
  e = cudaMemsetAsync(prm.pool, 0, kMassPoolBytes, stream);
  if (e != cudaSuccess) return e;
  block_mass_kernel<D><<<static_cast<unsigned>(ctas), mass::kThreads, L::kAlloc, stream>>>(tq, tk,
                                                                                          prm);
  return cudaGetLastError();
}

cudaError_t launch_block_mass(const AttnDims& a, const void* q, const void* k, float softmax_scale,
                              float* mass_out, void* ws, cudaStream_t stream) {
  const long long ctas = static_cast<long long>(a.batch) * a.heads * a.n_cta_per_head;
  if (ctas == 0) return cudaSuccess;
  MassParams prm;
  prm.a = a;
  prm.mass = mass_out;
  prm.status = static_cast<uint32_t*>(ws);
  prm.pool = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  prm.scratch = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes + kMassPoolBytes);
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (a.head_dim == 128) return launch_mass<128>(a, q, k, prm, ctas, stream);
  return launch_mass<64>(a, q, k, prm, ctas, stream);
}

}  // namespace bsa
