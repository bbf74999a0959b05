// Fused calibration step: the dense attention output and the exact block masses in one
// call, sm_100a.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: the calibration step runs dense attention and measures the exact block masses
// on it.  Computing them separately costs a QK^T pass for the masses plus a QK^T and a PV
// pass for the output; here one walk over the kv blocks does both:
//   S = Q K^T, P = exp2(S*c - m_r) with m_r a lazy reference max (raised only when a step's
//   max exceeds it by more than kRescaleLog2), every probability computed once: stored to
//   TMEM as bf16 for O += P V, summed per kv block into the CTA's workspace slice, and into
//   the row sum l_r.  When m_r is raised -- rare -- the row's O, its sum and the block sums
//   it has already written are multiplied by exp2(m_old - m_new);
//   end: O / l_r, and mass[i,j] = (1 / valid queries of i) * sum over the rows of query
//   block i of e[r,j] / l_r in a fixed order, as in bsa_block_mass.
//
// Layout, roles and pipeline follow the block-sparse forward (attn_fwd.cu): 256 query
// slots per CTA in two M=128 tiles, 384 threads (warps 0-7 row owners, warp 8 TMA, warp 9
// MMA, warps 10-11 completing the producer warpgroup, which hands registers to the row
// owners), TMEM S0 S1 O0 O1 with P stored over S; the MMA order is PV_t(s-1), S_t(s), the
// PV in two halves: the first kv block's keys as soon as their P is stored (P_part).
#include "bsa_kernels.cuh"

namespace bsa {

namespace calib {
constexpr int kThreads = 384;
constexpr int kRowsPerCta = 256;
// Launched at 168 registers a thread (three warps per sub-partition); the producer
// warpgroup gives some back: 2*128*kRegsRows + 128*kRegsProducer <= 384*168.
constexpr int kRegsLaunch = 168;
constexpr int kRegsRows = 184;
constexpr int kRegsProducer = 136;
static_assert(2 * 128 * kRegsRows + 128 * kRegsProducer <= kThreads * kRegsLaunch,
              "register shares must fit the launch total");
// Lazy reference max (log2 units): P <= 2^16, so O = sum P V stays far inside fp32 range.
constexpr float kRescaleLog2 = 16.0f;
}  // namespace calib

struct CalibParams {
  AttnDims a;
  __nv_bfloat16* out;
  float* lse;
  float* mass;
  uint32_t* status;
  float* scratch;  // [kMassSlots][n_kb][256] unnormalised row-block sums
  uint32_t* pool;  // kMassSlots bits: slices held by live CTAs
  float scale_log2;
};

template <int D>
struct CalibSmem {
  static constexpr int kChunks = D / 64;
  static constexpr int kQTile = 128 * D * 2;
  static constexpr int kKVStage = 128 * D * 2;
  static constexpr int kKStages = (D == 128) ? 3 : 4;
  static constexpr int kVStages = (D == 128) ? 2 : 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = 2 * kQTile;
  static constexpr int kVOff = kKOff + kKStages * kKVStage;
  static constexpr int kRedOff = kVOff + kVStages * kKVStage;  // float [256] 1 / row sum
  static constexpr int kBarOff = kRedOff + 256 * 4;
  static constexpr int kBytes = kBarOff + 512;
  static constexpr int kAlloc = kBytes + 1024;
};

template <int D>
__global__ void __launch_bounds__(calib::kThreads, 1)
    calib_dense_mass_kernel(const __grid_constant__ CUtensorMap tm_q,
                            const __grid_constant__ CUtensorMap tm_k,
                            const __grid_constant__ CUtensorMap tm_v, const CalibParams p) {
  using L = CalibSmem<D>;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* bar_q = bars;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_kempty = bar_kfull + KS;
  uint64_t* bar_vfull = bar_kempty + KS;
  uint64_t* bar_vempty = bar_vfull + VS;
  uint64_t* bar_sfull = bar_vempty + VS;  // [2]
  uint64_t* bar_pfull = bar_sfull + 2;    // [2] P_t stored
  uint64_t* bar_ppart = bar_pfull + 2;    // [2] P_t of the step's first kv block stored
  uint64_t* bar_ofull = bar_ppart + 2;
  uint64_t* bar_drain = bar_ofull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* nvalid_sm = reinterpret_cast<int*>(tmem_slot + 2);  // [2 tile][4 warp]
  int* slice_sm = reinterpret_cast<int*>(tmem_slot + 12);  // this CTA's scratch slice
  float* inv_l_sm = reinterpret_cast<float*>(smem + L::kRedOff);

  const AttnDims& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int bh = cta / a.n_cta_per_head;
  const int row0 = (cta - bh * a.n_cta_per_head) * calib::kRowsPerCta;
  const int nsteps = (a.n_kb + 1) >> 1;  // two kv blocks per step

  if (threadIdx.x == 0) {
    mbar_init(bar_q, 1);
    for (int i = 0; i < KS; ++i) {
      mbar_init(bar_kfull + i, 1);
      mbar_init(bar_kempty + i, 1);
    }
    for (int i = 0; i < VS; ++i) {
      mbar_init(bar_vfull + i, 1);
      mbar_init(bar_vempty + i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull + t, 1);
      mbar_init(bar_pfull + t, 128);
      mbar_init(bar_ppart + t, 128);
    }
    mbar_init(bar_ofull, 1);
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

  if (warp >= 8) {
    warpgroup_reg_dec<calib::kRegsProducer>();
    if (warp == 8) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
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
          uint8_t* kst = smem + L::kKOff + ks * L::kKVStage;
          for (int ch = 0; ch < L::kChunks; ++ch) {
            tma_load_3d(kst + ch * (128 * 128), &tm_k, bar_kfull + ks, ch * 64, 2 * s * 64, bh);
            if (nb == 2)
              tma_load_3d(kst + ch * (128 * 128) + 64 * 128, &tm_k, bar_kfull + ks, ch * 64,
                          (2 * s + 1) * 64, bh);
          }
          const int vs = s % VS;
          if (s >= VS && !mbar_wait(bar_vempty + vs, ((s / VS) - 1) & 1, abort_flag, p.status,
                                    DETAIL_WAIT_V_EMPTY))
            break;
          mbar_arrive_expect_tx(bar_vfull + vs, nb * 64 * D * 2);
          uint8_t* vst = smem + L::kVOff + vs * L::kKVStage;
          for (int ch = 0; ch < L::kChunks; ++ch) {
            tma_load_3d(vst + ch * (128 * 128), &tm_v, bar_vfull + vs, ch * 64, 2 * s * 64, bh);
            if (nb == 2)
              tma_load_3d(vst + ch * (128 * 128) + 64 * 128, &tm_v, bar_vfull + vs, ch * 64,
                          (2 * s + 1) * 64, bh);
          }
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0) {
        const uint64_t q_desc0 = make_sdesc_sw128(smem_u32(smem + L::kQOff), 16, 1024);
        const uint64_t k_desc0 = make_sdesc_sw128(smem_u32(smem + L::kKOff), 16, 1024);
        const uint64_t v_desc0 = make_sdesc_sw128(smem_u32(smem + L::kVOff), 128 * 128, 1024);
        const uint32_t idesc_pv = make_idesc(1u, 1u, 128u, static_cast<uint32_t>(D));
        bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, DETAIL_WAIT_Q);
        auto issue_pv = [&](int t, int u, int half) {
          // O_t (+)= P_t V over the keys of step u's first (half 0) or second (half 1) kv
          // block, 16 keys per MMA.
          const int nbp = (2 * u + 1 < a.n_kb) ? 2 : 1;
          const uint64_t vd = v_desc0 + static_cast<uint64_t>(((u % VS) * L::kKVStage) >> 4);
          const uint32_t p_tmem = tmem + t * 128;
          const uint32_t o_tmem = tmem + 256 + t * D;
          if (half >= nbp) return;
  #pragma unroll
          for (int kk = 4 * half; kk < 4 * half + 4; ++kk)
            mma_f16_ts(o_tmem, p_tmem + kk * 8, vd + static_cast<uint64_t>((kk * 2048) >> 4),
                       idesc_pv, (u > 0 || kk > 0) ? 1u : 0u);
        };
        // PV of step u for tile t: the first block's keys at P_part, the rest at P_full.
        auto pv_step = [&](int t, int u) -> bool {
          if (!mbar_wait(bar_ppart + t, u & 1, abort_flag, p.status, DETAIL_WAIT_P_PART))
            return false;
          if (t == 0 && !mbar_wait(bar_vfull + (u % VS), (u / VS) & 1, abort_flag, p.status,
                                   DETAIL_WAIT_V_FULL))
            return false;
          tc_fence_after();
          issue_pv(t, u, 0);
          if (!mbar_wait(bar_pfull + t, u & 1, abort_flag, p.status, DETAIL_WAIT_P_FULL))
            return false;
          tc_fence_after();
          issue_pv(t, u, 1);
          return true;
        };
        for (int s = 0; s < nsteps && ok; ++s) {
          const int nb = (2 * s + 1 < a.n_kb) ? 2 : 1;
          const int ks = s % KS;
          const uint32_t idesc_qk = make_idesc(1u, 0u, 128u, static_cast<uint32_t>(nb * 64));
          if (!mbar_wait(bar_kfull + ks, (s / KS) & 1, abort_flag, p.status, DETAIL_WAIT_K_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = k_desc0 + static_cast<uint64_t>((ks * L::kKVStage) >> 4);
          for (int t = 0; t < 2; ++t) {
            if (s > 0) {
              // the previous step's PV; it also frees S_t (P is stored over it), and S_t(s)
              // issued after it completes after it
              if (!pv_step(t, s - 1)) {
                ok = false;
                break;
              }
              if (t == 1) mma_commit(bar_vempty + ((s - 1) % VS));
            }
            tc_fence_after();
            const uint64_t qd = q_desc0 + static_cast<uint64_t>((t * L::kQTile) >> 4);
            const uint32_t s_tmem = tmem + t * 128;
  #pragma unroll
            for (int kk = 0; kk < D / 16; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
              mma_f16_ss(s_tmem, qd + off, kd + off, idesc_qk, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_sfull + t);
          }
          if (!ok) break;
          mma_commit(bar_kempty + ks);
        }
        if (ok) {
          const int u = nsteps - 1;
          for (int t = 0; t < 2 && ok; ++t) ok = pv_step(t, u);
          if (ok) mma_commit(bar_ofull);
        }
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0, p.status, DETAIL_WAIT_O_FULL);
      }
    }
  } else {
    warpgroup_reg_inc<calib::kRegsRows>();
    // ------------------------------------------------------------ row owners
    const int t = warp >> 2;
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const int local = t * 128 + row;
    const int slot = row0 + local;
    const bool in_range = slot < a.g.Np;
    const bool q_valid = in_range && slot_valid(a.g, slot);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128;
    const uint32_t o_addr = lane_base + 256 + t * D;
    const float c = p.scale_log2;
    const int wcount = __popc(__ballot_sync(0xffffffffu, q_valid));
    if (lane == 0) nvalid_sm[t * 4 + wq] = wcount;
    named_bar_sync(1 + t, 128);
    // this CTA's scratch slice: [n_kb][256] row-block sums (none: the claim timed out, no
    // masses are written and the status header says so)
    const int slice = *slice_sm;
    const bool have_slice = slice >= 0;
    float* sc = p.scratch + static_cast<size_t>(have_slice ? slice : 0) * 256 * a.n_kb;

    float m_ref = -INFINITY, l_run = 0.f;  // reference max (log2 units) and sum against it
    bool ok = true;
    for (int s = 0; s < nsteps; ++s) {
      const int nb = (2 * s + 1 < a.n_kb) ? 2 : 1;
      // A warp that gives up keeps stepping (without touching TMEM) so that the row warps
      // all reach the barrier before the masses.
      bool got = ok ? mbar_wait(bar_sfull + t, s & 1, abort_flag, p.status, DETAIL_WAIT_S_FULL)
                    : false;
      got = __all_sync(0xffffffffu, got);
      ok = got;
      if (!got) continue;
      tc_fence_after();
      float sv[128];
      tmem_ld32(s_addr + 0, sv + 0);
      tmem_ld32(s_addr + 32, sv + 32);
      if (nb == 2) {
        tmem_ld32(s_addr + 64, sv + 64);
        tmem_ld32(s_addr + 96, sv + 96);
      }
      tmem_ld_wait();
      // pad keys and the absent half of a 1-block step -> -inf
      const int j0 = 2 * s;
      const uint64_t mk0 = tile_has_pad(a.g, j0) ? tile_valid_mask(a.g, j0) : ~0ull;
      const uint64_t mk1 =
          nb == 2 ? (tile_has_pad(a.g, j0 + 1) ? tile_valid_mask(a.g, j0 + 1) : ~0ull) : 0ull;
      if ((mk0 & mk1) != ~0ull) {
        const uint32_t mw[4] = {static_cast<uint32_t>(mk0), static_cast<uint32_t>(mk0 >> 32),
                                static_cast<uint32_t>(mk1), static_cast<uint32_t>(mk1 >> 32)};
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? sv[i] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = sv[i];
#pragma unroll
      for (int i = 8; i < 128; ++i) mx[i & 7] = fmaxf(mx[i & 7], sv[i]);
      const float m_new = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                                fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]))) *
                          c;  // c > 0, so -inf stays -inf
      float factor = 1.f;
      bool resc = false;
      if (m_new > m_ref + calib::kRescaleLog2) {  // the first step with a valid key always
        if (m_ref != -INFINITY) {
          factor = fast_exp2(m_ref - m_new);
          resc = true;
        }
        m_ref = m_new;
      }
      // P = exp2(S*c - m) stored over S_t as bf16 pairs; the first kv block's P releases
      // its half of PV unless this warp must first rescale its rows of O (then both halves
      // are released at the end).  A row with no valid key so far has every P = 0.
      const float m_use = (m_ref == -INFINITY) ? 0.f : m_ref;
      const bool warp_resc = __any_sync(0xffffffffu, resc);
      float acc[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        if (ch >= 2 && nb == 1) break;
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float p0 = fast_exp2(fmaf(sv[32 * ch + 2 * i], c, -m_use));
          const float p1 = fast_exp2(fmaf(sv[32 * ch + 2 * i + 1], c, -m_use));
          acc[ch >> 1][i & 1] += p0 + p1;
          pk[i] = pack_bf16x2(p0, p1);
        }
        BSA_TMEM_ST_X16(s_addr + 16 * ch, pk);
        if (ch == 1 && !warp_resc) {  // the first kv block's P: its half of PV may start
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar_ppart + t);
        }
      }
      const float e0 = acc[0][0] + acc[0][1];
      const float e1 = acc[1][0] + acc[1][1];
      l_run = fmaf(l_run, factor, e0 + e1);
      if (have_slice) {
        if (resc)  // the block sums formed against the old reference
          for (int j = 0; j < j0; ++j) sc[static_cast<size_t>(j) * 256 + local] *= factor;
        sc[static_cast<size_t>(j0) * 256 + local] = e0;
        if (nb == 2) sc[static_cast<size_t>(j0 + 1) * 256 + local] = e1;
      }
      if (warp_resc) {
        // O_t is quiescent: the PV of the previous step completed before S_full fired.
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          float ov[32];
          tmem_ld32(o_addr + c0, ov);
          tmem_ld_wait();
          uint32_t r[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(ov[i] * factor);
          BSA_TMEM_ST_X16(o_addr + c0, r);
          BSA_TMEM_ST_X16(o_addr + c0 + 16, (r + 16));
        }
      }
      tmem_st_wait();
      tc_fence_before();
      if (warp_resc) mbar_arrive(bar_ppart + t);
      mbar_arrive(bar_pfull + t);
    }

    // ------------------------------------------------------------ epilogue
    bool have_o = ok && nsteps > 0;
    if (have_o) {
      have_o = __all_sync(0xffffffffu,
                          mbar_wait(bar_ofull, 0, abort_flag, p.status, DETAIL_WAIT_O_FULL));
      tc_fence_after();
    }
    const float inv_l = (q_valid && l_run > 0.f) ? 1.f / l_run : 0.f;
    __nv_bfloat16* orow = p.out + (static_cast<long long>(bh) * a.g.Np + slot) * D;
#pragma unroll 1
    for (int c0 = 0; c0 < D; c0 += 32) {
      float ov[32];
      if (have_o) {
        tmem_ld32(o_addr + c0, ov);
        tmem_ld_wait();
      } else {
#pragma unroll
        for (int i = 0; i < 32; ++i) ov[i] = 0.f;
      }
      if (in_range) {
        uint4 w[4];
        uint32_t* wp = reinterpret_cast<uint32_t*>(w);
#pragma unroll
        for (int i = 0; i < 16; ++i) wp[i] = pack_bf16x2(ov[2 * i] * inv_l, ov[2 * i + 1] * inv_l);
        uint4* dst = reinterpret_cast<uint4*>(orow + c0);
#pragma unroll
        for (int i = 0; i < 4; ++i) dst[i] = w[i];
      }
    }
    if (p.lse != nullptr && in_range)
      p.lse[static_cast<long long>(bh) * a.g.Np + slot] =
          (q_valid && l_run > 0.f) ? (m_ref + log2f(l_run)) * 0.6931471805599453f : -INFINITY;

    // ------------------------------------------------------------ masses
    // mass[i, j] = (1 / valid queries of i) * sum_r e[r, j] / l_r over the rows of query
    // block i, in row order, by the 256 row threads over the CTA's outputs.
    inv_l_sm[local] = (q_valid && ok && l_run > 0.f) ? 1.f / l_run : 0.f;
    named_bar_sync(7, 256);  // every row's block sums and 1 / l_r are written
    if (have_slice) {
      const int rt = warp * 32 + lane;  // 0 .. 255
      const int warps_per_qb = a.q_block / 32;  // 2 or 4
      const int nq_cta = calib::kRowsPerCta / a.q_block;
      const int qb0 = row0 / a.q_block;
      for (int o = rt; o < nq_cta * a.n_kb; o += 256) {
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
        float tot = 0.f;
        for (int r = 0; r < a.q_block; r += 4) {
          const float4 ev = *reinterpret_cast<const float4*>(col + r);
          tot += ev.x * inv_l_sm[qi * a.q_block + r];
          tot += ev.y * inv_l_sm[qi * a.q_block + r + 1];
          tot += ev.z * inv_l_sm[qi * a.q_block + r + 2];
          tot += ev.w * inv_l_sm[qi * a.q_block + r + 3];
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

template <int D>
static cudaError_t launch_calib(const AttnDims& a, const void* q, const void* k, const void* v,
                                const CalibParams& prm, long long ctas, cudaStream_t stream) {
  using L = CalibSmem<D>;
  CUtensorMap tq, tk, tv;
  const int bh = a.batch * a.heads;
  cudaError_t e = encode_tmap_3d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.g.Np, bh, 64, 128);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.g.Np, bh, 64, 64);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.g.Np, bh, 64, 64);
  if (e != cudaSuccess) return e;
  // the register split between warpgroups needs the kernel launched at exactly kRegsLaunch
  cudaFuncAttributes attr;
  e = cudaFuncGetAttributes(&attr, calib_dense_mass_kernel<D>);
  if (e != cudaSuccess) return e;
  if (attr.numRegs != calib::kRegsLaunch) return cudaErrorInvalidConfiguration;
  e = cudaFuncSetAttribute(calib_dense_mass_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           L::kAlloc);
  if (e != cudaSuccess) return e;
  // one CTA per SM, so the live CTAs (at most the SM count) never exhaust the kMassSlots
  // slices and no claim waits
  int per_sm = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, calib_dense_mass_kernel<D>,
                                                    calib::kThreads, L::kAlloc);
  if (e != cudaSuccess) return e;
  if (per_sm != 1) return cudaErrorInvalidConfiguration;
  e = cudaMemsetAsync(prm.pool, 0, kMassPoolBytes, stream);
  if (e != cudaSuccess) return e;
  calib_dense_mass_kernel<D><<<static_cast<unsigned>(ctas), calib::kThreads, L::kAlloc, stream>>>(
      tq, tk, tv, prm);
  return cudaGetLastError();
}

cudaError_t launch_calib_dense_mass(const AttnDims& a, const void* q, const void* k, const void* v,
                                    float softmax_scale, void* out, float* lse, float* mass,
                                    void* ws, cudaStream_t stream) {
  const long long ctas = static_cast<long long>(a.batch) * a.heads * a.n_cta_per_head;
  if (ctas == 0) return cudaSuccess;
  CalibParams prm;
  prm.a = a;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.mass = mass;
  prm.status = static_cast<uint32_t*>(ws);
  prm.pool = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(ws) + kStatusBytes);
  prm.scratch = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + kStatusBytes + kMassPoolBytes);
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (a.head_dim == 128) return launch_calib<128>(a, q, k, v, prm, ctas, stream);
  return launch_calib<64>(a, q, k, v, prm, ctas, stream);
}

}  // namespace bsa
