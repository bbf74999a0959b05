// Block-sparse flash-attention forward over frozen CSR kv-block lists on CTA pairs, sm_100a.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: the block indices selected at the calibration step are frozen and reused by
// the attention of all remaining steps; softmax runs over the kept blocks only.
//
// Same arithmetic and schedule as bsattn_fwd_kernel (attn_fwd.cu): 256 query slots of one
// (batch, head) walk the union of their query blocks' kv lists two kv blocks (128 keys) per
// step, keys a row's query block did not keep masked, online softmax with a lazy reference
// max.  What changes is the hardware mapping: the 256 slots are two 128-row tiles on two
// SMs of a cluster (a CTA pair), and every tensor-core operation is a pair MMA
// (tcgen05 cta_group::2, M = 256) issued by the first CTA:
//   S = Q K^T   A = Q, 128 rows from each CTA's shared memory;  B = K, each CTA holding
//               one of the step's two kv blocks (64 keys x 128 dims);
//   O += P V    A = P from each CTA's tensor memory;  B = V, each CTA holding 64 of the
//               128 head dims of the step's 128 keys.
// So each SM loads half of every K and V tile, and with one tile per SM its tensor memory
// holds two S buffers: S(s+1) = Q K(s+1)^T runs while the softmax works on S(s), and the
// chain softmax -> PV -> next QK^T of one tile no longer sets the step time.
//
// Per CTA (192 threads):
//   warps 0-3  softmax and epilogue, one thread per row (TMEM lane) of the CTA's tile
//   warp 4     TMA producer: the CTA's Q tile once, its halves of K and V every step
//   warp 5     tensor memory owner; in the pair's first CTA also the MMA issuer
// Tensor memory (512 columns per SM): S0 [0,128)  S1 [128,256)  O [256,384).
// Barriers: Q / K / V "full" and P "full" live in the first CTA (both CTAs' copies and
// softmax warps arrive there); S "full", K / V "empty", PV "done" and O "full" exist in
// both CTAs, completed by multicast commits of the pair MMAs.
// A step with one kv block (an odd list's tail) loads that block twice and masks the copy,
// so every pair MMA has N = 128.
#include "bsa_kernels.cuh"

namespace bsa {

namespace pair {
constexpr int kThreads = 192;
constexpr int kRows = 128;                 // query rows per CTA (one tile)
constexpr int kKStages = 4;
constexpr int kVStages = 4;
constexpr float kRescaleLog2 = 8.0f;
constexpr uint16_t kBoth = 0x3;            // multicast mask: both CTAs of the pair

// Shared memory (bf16, D = 128): byte offsets from the 1024-aligned base.
constexpr int kQBytes = kRows * 256;       // 128 rows x 128 dims: two 64-dim swizzle chunks
constexpr int kKBytes = 64 * 256;          // one kv block x 128 dims: two chunks of 64 rows
constexpr int kVBytes = 128 * 128;         // 128 keys x this CTA's 64 dims
constexpr int kQOff = 0;
constexpr int kKOff = kQOff + kQBytes;
constexpr int kVOff = kKOff + kKStages * kKBytes;
constexpr int kBarOff = kVOff + kVStages * kVBytes;
constexpr int kBytes = kBarOff + 512;
constexpr int kAlloc = kBytes + 1024;
}  // namespace pair

struct PairParams {
  AttnDims a;
  const int32_t* counts;
  const uint32_t* entries;
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
  float scale_log2;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair::kThreads, 1)
    bsattn_fwd_pair_kernel(const __grid_constant__ CUtensorMap tm_q,
                           const __grid_constant__ CUtensorMap tm_k,
                           const __grid_constant__ CUtensorMap tm_v, const PairParams p) {
  using namespace pair;
  constexpr int KS = kKStages, VS = kVStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kBarOff);
  uint64_t* bar_q = bars;                   // first CTA: both Q tiles loaded
  uint64_t* bar_kfull = bars + 1;           // [KS] first CTA: both K halves loaded
  uint64_t* bar_kempty = bar_kfull + KS;    // [KS] each CTA: its K slot free again
  uint64_t* bar_vfull = bar_kempty + KS;    // [VS]
  uint64_t* bar_vempty = bar_vfull + VS;    // [VS]
  uint64_t* bar_sfull = bar_vempty + VS;    // [2] each CTA: S buffer b computed
  uint64_t* bar_pfull = bar_sfull + 2;      // [2] first CTA: P of buffer b stored (8 warps)
  uint64_t* bar_pvdone = bar_pfull + 2;     // each CTA: the latest PV has completed
  uint64_t* bar_ofull = bar_pvdone + 1;     // each CTA: the last PV has completed
  uint64_t* bar_drain = bar_ofull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const AttnDims& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();        // 0: issues the pair MMAs
  const int grp = blockIdx.x >> 1;                // 256-slot group = schedule entry list
  const int bh = grp / a.n_cta_per_head;
  const int row0 = (grp - bh * a.n_cta_per_head) * 256 + static_cast<int>(rank) * kRows;
  const int n_ent = p.counts[grp];
  const uint32_t* ent = p.entries + static_cast<long long>(grp) * a.n_kb;
  const int nsteps = (n_ent + 1) >> 1;

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
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_sfull + b, 1);
      mbar_init(bar_pfull + b, 8);  // four softmax warps in each CTA
    }
    mbar_init(bar_pvdone, 1);
    mbar_init(bar_ofull, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) tmem_alloc_pair(tmem_slot, 512);
  tc_fence_before();
  // both CTAs' barriers exist before either signals the other's
  cluster_sync_all();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // the first CTA's copy of a barrier, as a shared::cluster address
  auto first = [](uint64_t* bar) { return mapa_shared(smem_u32(bar), 0); };

  if (warp == 4) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0 && nsteps > 0) {
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      if (rank == 0) mbar_arrive_expect_tx(bar_q, 2 * kQBytes);
      for (int ch = 0; ch < 2; ++ch)
        tma_load_3d_pair(smem + kQOff + ch * (kRows * 128), &tm_q, first(bar_q), ch * 64, row0, bh);
      for (int s = 0; s < nsteps; ++s) {
        const int nb = (2 * s + 1 < n_ent) ? 2 : 1;
        const int j0 = static_cast<int>(ent[2 * s] >> 5);
        const int j1 = nb == 2 ? static_cast<int>(ent[2 * s + 1] >> 5) : j0;  // copy, masked
        const int ks = s % KS;
        if (s >= KS && !mbar_wait_cluster(bar_kempty + ks, ((s / KS) - 1) & 1, abort_flag,
                                          p.status, DETAIL_WAIT_K_EMPTY))
          break;
        if (rank == 0) mbar_arrive_expect_tx(bar_kfull + ks, 2 * kKBytes);
        uint8_t* kst = smem + kKOff + ks * kKBytes;
        const int jk = rank == 0 ? j0 : j1;  // this CTA's kv block of the step
        for (int ch = 0; ch < 2; ++ch)
          tma_load_3d_pair(kst + ch * (64 * 128), &tm_k, first(bar_kfull + ks), ch * 64, jk * 64, bh);
        const int vs = s % VS;
        if (s >= VS && !mbar_wait_cluster(bar_vempty + vs, ((s / VS) - 1) & 1, abort_flag,
                                          p.status, DETAIL_WAIT_V_EMPTY))
          break;
        if (rank == 0) mbar_arrive_expect_tx(bar_vfull + vs, 2 * kVBytes);
        uint8_t* vst = smem + kVOff + vs * kVBytes;
        const int dv = static_cast<int>(rank) * 64;  // this CTA's head dims
        tma_load_3d_pair(vst, &tm_v, first(bar_vfull + vs), dv, j0 * 64, bh);
        tma_load_3d_pair(vst + 64 * 128, &tm_v, first(bar_vfull + vs), dv, j1 * 64, bh);
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ MMA issuer (first CTA)
    if (rank == 0 && lane == 0 && nsteps > 0) {
      const uint64_t q_desc0 = make_sdesc_sw128(smem_u32(smem + kQOff), 16, 1024);
      const uint64_t k_desc0 = make_sdesc_sw128(smem_u32(smem + kKOff), 16, 1024);
      const uint64_t v_desc0 = make_sdesc_sw128(smem_u32(smem + kVOff), kVBytes, 1024);
      const uint32_t idesc_qk = make_idesc(1u, 0u, 256u, 128u);  // bf16, B K-major
      const uint32_t idesc_pv = make_idesc(1u, 1u, 256u, 128u);  // bf16, B MN-major
      bool ok = mbar_wait_cluster(bar_q, 0, abort_flag, p.status, DETAIL_WAIT_Q);
      // O += P(u) V(u): P in the S buffer of step u (bf16 pairs, 8 columns per 16 keys)
      auto issue_pv = [&](int u) -> bool {
        if (!mbar_wait_cluster(bar_pfull + (u & 1), (u >> 1) & 1, abort_flag, p.status,
                               DETAIL_WAIT_P_FULL))
          return false;
        const int vs = u % VS;
        if (!mbar_wait_cluster(bar_vfull + vs, (u / VS) & 1, abort_flag, p.status,
                               DETAIL_WAIT_V_FULL))
          return false;
        tc_fence_after();
        const uint64_t vd = v_desc0 + static_cast<uint64_t>((vs * kVBytes) >> 4);
        const uint32_t p_tmem = tmem + (u & 1) * 128;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_f16_ts_pair(tmem + 256, p_tmem + kk * 8,
                          vd + static_cast<uint64_t>((kk * 16 * 128) >> 4), idesc_pv,
                          (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit_pair(bar_vempty + vs, kBoth);
        mma_commit_pair(bar_pvdone, kBoth);
        return true;
      };
      for (int s = 0; s < nsteps && ok; ++s) {
        const int ks = s % KS;
        if (!mbar_wait_cluster(bar_kfull + ks, (s / KS) & 1, abort_flag, p.status,
                               DETAIL_WAIT_K_FULL)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // S(s) into buffer s & 1; its previous reader, PV(s - 2), was issued before
        const uint64_t kd = k_desc0 + static_cast<uint64_t>((ks * kKBytes) >> 4);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          // K (= head dim) advances 32 bytes per MMA inside each 128-byte swizzle chunk
          const uint64_t qoff = static_cast<uint64_t>(((kk >> 2) * (kRows * 128) + (kk & 3) * 32) >> 4);
          const uint64_t koff = static_cast<uint64_t>(((kk >> 2) * (64 * 128) + (kk & 3) * 32) >> 4);
          mma_f16_ss_pair(tmem + (s & 1) * 128, q_desc0 + qoff, kd + koff, idesc_qk,
                          kk > 0 ? 1u : 0u);
        }
        mma_commit_pair(bar_sfull + (s & 1), kBoth);
        mma_commit_pair(bar_kempty + ks, kBoth);
        if (s > 0) ok = issue_pv(s - 1);
      }
      if (ok) ok = issue_pv(nsteps - 1);
      if (ok) mma_commit_pair(bar_ofull, kBoth);
      // Whatever happened, every issued MMA completes before tensor memory is released.
      mma_commit_pair(bar_drain, 0x1);
      mbar_wait_drain(bar_drain, 0, p.status, DETAIL_WAIT_O_FULL);
    }
  } else {
    // ------------------------------------------------------------ softmax warps
    const int row = warp * 32 + lane;      // TMEM lane = row of this CTA's tile
    const int slot = row0 + row;
    const int qsel = (static_cast<int>(rank) * kRows + warp * 32) / a.q_block;  // keep bit
    const bool in_range = slot < a.g.Np;
    const bool q_valid = in_range && slot_valid(a.g, slot);
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(warp * 32) << 16);
    const uint32_t o_addr = lane_base + 256;
    const float c = p.scale_log2;
    float m_run = -INFINITY;  // reference max, scaled log2 units
    float l_run = 0.f;
    bool ok = true;
    int pv_waited = 0;        // PV(0 .. pv_waited-1) are known complete
    auto wait_pv = [&](int u) -> bool {  // PV(u) complete; phases are waited in order
      bool good = true;
      while (pv_waited <= u && good) {
        good = __all_sync(0xffffffffu, mbar_wait_cluster(bar_pvdone, pv_waited & 1, abort_flag,
                                                         p.status, DETAIL_WAIT_O_FULL));
        if (good) ++pv_waited;
      }
      return good;
    };
    uint32_t e0n = nsteps > 0 ? ld_early_u32(ent) : 0u;
    uint32_t e1n = n_ent > 1 ? ld_early_u32(ent + 1) : 0u;
    for (int s = 0; s < nsteps; ++s) {
      const int nb = (2 * s + 1 < n_ent) ? 2 : 1;
      const uint32_t e0 = e0n, e1 = e1n;
      if (s + 1 < nsteps) {
        e0n = ld_early_u32(ent + 2 * s + 2);
        e1n = (2 * s + 3 < n_ent) ? ld_early_u32(ent + 2 * s + 3) : 0u;
      }
      const uint32_t s_addr = lane_base + (s & 1) * 128;
      const bool got = __all_sync(
          0xffffffffu, mbar_wait_cluster(bar_sfull + (s & 1), (s >> 1) & 1, abort_flag, p.status,
                                         DETAIL_WAIT_S_FULL));
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      // The blocks of the step this warp's query block keeps (warp-uniform); the rest
      // contribute P = 0 with no exponentials.
      const bool k0 = (e0 >> qsel) & 1u;
      const bool k1 = nb == 2 && ((e1 >> qsel) & 1u);
      float sv[128];
      if (k0) {
        tmem_ld32(s_addr + 0, sv + 0);
        tmem_ld32(s_addr + 32, sv + 32);
      }
      if (k1) {
        tmem_ld32(s_addr + 64, sv + 64);
        tmem_ld32(s_addr + 96, sv + 96);
      }
      tmem_ld_wait();
      if (k0 && ((e0 >> 4) & 1u)) {  // pad keys -> -inf
        const uint64_t mk = tile_valid_mask(a.g, static_cast<int>(e0 >> 5));
        const uint32_t mw[2] = {static_cast<uint32_t>(mk), static_cast<uint32_t>(mk >> 32)};
#pragma unroll
        for (int i = 0; i < 64; ++i) sv[i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? sv[i] : -INFINITY;
      }
      if (k1 && ((e1 >> 4) & 1u)) {
        const uint64_t mk = tile_valid_mask(a.g, static_cast<int>(e1 >> 5));
        const uint32_t mw[2] = {static_cast<uint32_t>(mk), static_cast<uint32_t>(mk >> 32)};
#pragma unroll
        for (int i = 0; i < 64; ++i)
          sv[64 + i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? sv[64 + i] : -INFINITY;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) mx[i] = -INFINITY;
      if (k0) {
#pragma unroll
        for (int i = 0; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], sv[i]);
      }
      if (k1) {
#pragma unroll
        for (int i = 64; i < 128; ++i) mx[4 + (i & 3)] = fmaxf(mx[4 + (i & 3)], sv[i]);
      }
      const float mh = fmaxf(fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])),
                             fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7])));
      const float m_new = mh == -INFINITY ? -INFINITY : mh * c;  // c > 0
      float factor = 1.f;
      bool resc = false;
      if (m_new > m_run + kRescaleLog2 || (m_run == -INFINITY && m_new != -INFINITY)) {
        if (m_run != -INFINITY) {
          factor = fast_exp2(m_run - m_new);
          resc = true;
        }
        m_run = m_new;
      }
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int ch = 0; ch < 4; ++ch) {
        uint32_t pk[16];
        if (ch < 2 ? k0 : k1) {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(sv[32 * ch + 2 * i], c, -m_use));
            const float p1 = fast_exp2(fmaf(sv[32 * ch + 2 * i + 1], c, -m_use));
            ls[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        BSA_TMEM_ST_X16(s_addr + 16 * ch, pk);
      }
      l_run = fmaf(l_run, factor, (ls[0] + ls[1]) + (ls[2] + ls[3]));
      if (__any_sync(0xffffffffu, resc)) {
        // O must hold every earlier step before it is rescaled: PV(s - 1) complete
        if (s > 0 && !wait_pv(s - 1)) {
          ok = false;
          break;
        }
        tc_fence_after();
#pragma unroll 1
        for (int c0 = 0; c0 < 128; c0 += 32) {
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
      // PV(s - 1) completes (in practice long since) before P(s) is released: PV(s) cannot
      // be issued, so "PV done" is never two phases ahead of the phase waited for here.
      if (s > 0 && !wait_pv(s - 1)) {
        ok = false;
        break;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(first(bar_pfull + (s & 1)));
    }

    // ------------------------------------------------------------ epilogue
    const float inv_l = (l_run > 0.f && q_valid) ? 1.f / l_run : 0.f;
    bool have_o = ok && nsteps > 0;
    if (have_o) {
      have_o = __all_sync(0xffffffffu, mbar_wait_cluster(bar_ofull, 0, abort_flag, p.status,
                                                         DETAIL_WAIT_O_FULL));
      tc_fence_after();
    }
    __nv_bfloat16* orow = p.out + (static_cast<long long>(bh) * a.g.Np + slot) * 128;
#pragma unroll 1
    for (int c0 = 0; c0 < 128; c0 += 32) {
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
          (l_run > 0.f && q_valid) ? (m_run + __log2f(l_run)) * 0.6931471805599453f : -INFINITY;
  }

  // Both CTAs are done with the pair's tensor memory (the first CTA's MMAs have drained)
  // before either releases its columns.
  __syncwarp();
  tc_fence_before();
  cluster_sync_all();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, 512);
  }
}

cudaError_t launch_bsattn_fwd_pair(const AttnDims& a, const void* q, const void* k, const void* v,
                                   const int32_t* counts, const uint32_t* entries,
                                   float softmax_scale, void* out, float* lse, uint32_t* status,
                                   long long groups, cudaStream_t stream) {
  CUtensorMap tq, tk, tv;
  const int bhn = a.batch * a.heads;
  cudaError_t e = encode_tmap_3d(&tq, q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, a.g.Np, bhn, 64, 128);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tk, k, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, a.g.Np, bhn, 64, 64);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tv, v, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, 128, a.g.Np, bhn, 64, 64);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bsattn_fwd_pair_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           pair::kAlloc);
  if (e != cudaSuccess) return e;
  PairParams prm;
  prm.a = a;
  prm.counts = counts;
  prm.entries = entries;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  bsattn_fwd_pair_kernel<<<static_cast<unsigned>(2 * groups), pair::kThreads, pair::kAlloc,
                           stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

}  // namespace bsa
