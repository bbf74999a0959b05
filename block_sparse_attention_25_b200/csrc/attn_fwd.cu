// Block-sparse flash-attention forward over frozen CSR kv-block lists, sm_100a.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: the block indices selected at the calibration step are frozen and reused by
// the attention of all remaining steps; softmax runs over the kept blocks only.
// "FPSAttention", Abstract: FP8 e4m3 operands with one scale per 3D tile.
//
// Work decomposition
//   One CTA owns 256 consecutive query slots of one (batch, head): two M=128 tiles, so
//   every K/V tile fetched into shared memory feeds two tensor-core tiles.  The CTA walks
//   the sorted union of its query blocks' kv lists (built by bsattn_schedule_kernel) two
//   kv blocks (N = 128 keys) per step; keys of a block that a query block did not keep
//   are masked to -inf for that block's rows.
//
// Warp roles (384 threads; warps 10-11 only complete the producer warpgroup)
//   warps 0-3  softmax for Q tile 0, one thread per query row (TMEM lanes 0..127)
//   warps 4-7  softmax for Q tile 1
//   warp 8     TMA producer: Q once, then K and V of every step into rings
//   warp 9     tcgen05.mma issuer (one thread) and TMEM owner
//
// Tensor memory (512 columns x 128 lanes x 32 bit)
//   S0 [0,128)  S1 [128,256)  O0 [256,256+D)  O1 [256+D,256+2D)
//   P_t (bf16 pairs) overwrites the first 64 columns of S_t once S_t has been read.
//
// Per step s, the MMA thread issues for t = 0, 1:  O_t += P_t(s-1) V(s-1);  S_t(s) = Q_t K(s)^T
// and commits S_full[t] after both, so when softmax t sees S_t(s) the previous PV into O_t
// has completed and O_t may be rescaled in place.  The PV is issued in two halves: the
// first kv block's keys as soon as their P is stored (P_part), the rest at P_full.
// Rescaling is lazy: the running max used for exponentiation moves only when a row's max
// grows by more than 8 (log2 units), so P <= 256 and, for smooth attention, O is almost
// never touched (a threshold of 16 for bf16 measured the same: rescales are already rare).
#include "bsa_kernels.cuh"

namespace bsa {

namespace fwd {

// 12 warps = 3 warpgroups: two softmax warpgroups (one per Q tile) and one producer
// warpgroup (TMA warp, MMA warp, two idle warps).  Launched at 168 registers a thread (three
// warps share each sub-partition's 16K registers), the producer warpgroup gives registers
// back and the softmax warpgroups take them: 2*128*184 + 128*136 = 384*168 (the split with
// the fewest spills over the variants).
constexpr int kThreads = 384;
constexpr int kRegsLaunch = 168;
constexpr int kRegsSoftmax = 184;
constexpr int kRegsProducer = 136;
static_assert(2 * 128 * kRegsSoftmax + 128 * kRegsProducer <= kThreads * kRegsLaunch,
              "register shares must fit the launch total");
constexpr int kRowsPerCta = 256;
constexpr float kRescaleLog2 = 8.0f;

// Schedule entry: (j << 5) | (has_pad_keys << 4) | keep bits for the CTA's <= 4 query blocks.
__device__ __forceinline__ int entry_block(uint32_t e) { return static_cast<int>(e >> 5); }

// Cluster order: an entry is a run of 1..64 consecutive keys, (first slot << 7) | length.
__device__ __forceinline__ int entry_start(uint32_t e) { return static_cast<int>(e >> 7); }
__device__ __forceinline__ uint64_t entry_len_mask(uint32_t e) {
  const uint32_t len = e & 127u;
  return len >= 64u ? ~0ull : ((1ull << len) - 1ull);
}

}  // namespace fwd

// Build, per CTA, the ascending union of its query blocks' kv lists with keep bits.
// One 256-thread CTA per attention CTA.  Validates the CSR rows it reads.
__global__ void __launch_bounds__(256) bsattn_schedule_kernel(AttnDims a,
                                                              const int32_t* __restrict__ row_ptr,
                                                              const int32_t* __restrict__ col_idx,
                                                              int32_t* __restrict__ counts,
                                                              uint32_t* __restrict__ entries,
                                                              const float* __restrict__ v_scales,
                                                              float* __restrict__ sigma,
                                                              uint32_t* status) {
  __shared__ uint32_t bm[4][128];  // up to 4096 kv blocks per query block
  __shared__ int warp_tot[8];
  __shared__ float warp_max[8];
  const int cta = blockIdx.x;
  const int bh = cta / a.n_cta_per_head;
  const int c = cta - bh * a.n_cta_per_head;
  const int nq = fwd::kRowsPerCta / a.q_block;
  const int tid = threadIdx.x;
  for (int i = tid; i < 4 * 128; i += 256) (&bm[0][0])[i] = 0u;
  __syncthreads();
  for (int slot = 0; slot < nq; ++slot) {
    const int qb = c * nq + slot;
    if (qb >= a.n_qb) break;
    const long long r = static_cast<long long>(bh) * a.n_qb + qb;
    const int beg = row_ptr[r], end = row_ptr[r + 1];
    if (beg < 0 || end < beg || end - beg > a.n_kb) {
      if (tid == 0) record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_ROWPTR, static_cast<uint32_t>(r), 0u);
      continue;
    }
    for (int e = beg + tid; e < end; e += 256) {
      const int j = col_idx[e];
      if (j < 0 || j >= a.n_kb) {
        record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_RANGE, static_cast<uint32_t>(r), static_cast<uint32_t>(e));
        continue;
      }
      if (e > beg && col_idx[e - 1] >= j)
        record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_ORDER, static_cast<uint32_t>(r), static_cast<uint32_t>(e));
      atomicOr(&bm[slot][j >> 5], 1u << (j & 31));
    }
  }
  __syncthreads();
  uint32_t* out = entries + static_cast<long long>(cta) * a.n_kb;
  const float* vsc = v_scales ? v_scales + static_cast<long long>(bh) * a.n_kb : nullptr;
  float vmax = 0.f;
  int base = 0;
  for (int j0 = 0; j0 < a.n_kb; j0 += 256) {
    const int j = j0 + tid;
    uint32_t keep = 0;
    if (j < a.n_kb) {
#pragma unroll
      for (int s = 0; s < 4; ++s) keep |= ((bm[s][j >> 5] >> (j & 31)) & 1u) << s;
    }
    const bool any = keep != 0;
    const uint32_t bal = __ballot_sync(0xffffffffu, any);
    const int wpos = __popc(bal & ((1u << lane_id()) - 1u));
    if (lane_id() == 0) warp_tot[tid >> 5] = __popc(bal);
    __syncthreads();
    int before = 0, tot = 0;
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      if (w < (tid >> 5)) before += warp_tot[w];
      tot += warp_tot[w];
    }
    if (any) {
      const uint32_t pad = tile_has_pad(a.g, j) ? 1u : 0u;
      out[base + before + wpos] = (static_cast<uint32_t>(j) << 5) | (pad << 4) | keep;
      if (vsc) vmax = fmaxf(vmax, vsc[j]);
    }
    base += tot;
    __syncthreads();
  }
  if (tid == 0) counts[cta] = base;
  if (sigma != nullptr) {
    // Largest V tile scale over the CTA's list: P is quantised relative to it.
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) vmax = fmaxf(vmax, __shfl_xor_sync(0xffffffffu, vmax, o));
    if (lane_id() == 0) warp_max[tid >> 5] = vmax;
    __syncthreads();
    if (tid == 0) {
      float m = 0.f;
      for (int w = 0; w < 8; ++w) m = fmaxf(m, warp_max[w]);
      sigma[cta] = m > 0.f ? m : 1.f;
    }
  }
}

struct FwdParams {
  AttnDims a;
  const int32_t* counts;
  const uint32_t* entries;
  const float* q_scales;  // e4m3 only: per (bh, 64-token tile)
  const float* k_scales;
  const float* v_scales;
  const float* sigma;     // e4m3 only: per CTA, max V tile scale over its list
  __nv_bfloat16* out;
  float* lse;
  uint32_t* status;
  float scale_log2;  // softmax_scale * log2(e)
  // cluster order only (tokens of a query cluster are consecutive slots; the CTAs of one
  // head cover its clusters 256 rows at a time, cta_base[bh][c] = first CTA of cluster c)
  int S;            // slots per (batch, head)
  int n_qc;         // query clusters per (batch, head)
  int cap;          // CTAs launched per (batch, head); those past cta_base[bh][n_qc] exit
  int max_ent;      // entry capacity per query cluster
  const int32_t* q_starts;
  const int32_t* q_counts;
  const int32_t* cta_base;   // [bh][n_qc + 1]
  const int32_t* ent_counts; // [bh][n_qc]
  // raster layout only: the batch of this launch and its first CTA (one launch per batch)
  int raster_b;
  int cta_offset;
};

// Shared-memory plan.  Every operand row is cut into 128-byte swizzle chunks (64 bf16 or
// 128 e4m3 elements); a 128-row tile of one chunk is 16 KB.
template <int D, bool FP8>
struct FwdSmem {
  static constexpr int kElem = FP8 ? 1 : 2;
  static constexpr int kRowBytes = D * kElem;
  static constexpr int kChunks = kRowBytes / 128;
  static constexpr int kChunkElems = 128 / kElem;
  static constexpr int kQTile = 128 * kRowBytes;     // one 128-row Q tile
  static constexpr int kKVStage = 128 * kRowBytes;   // two 64-row kv blocks
  static constexpr int kKStages = (kRowBytes == 256) ? 3 : 4;
  static constexpr int kVStages = (kRowBytes == 256) ? 2 : 4;
  static constexpr int kQOff = 0;
  static constexpr int kKOff = kQOff + 2 * kQTile;
  static constexpr int kVOff = kKOff + kKStages * kKVStage;
  static constexpr int kBarOff = kVOff + kVStages * kKVStage;
  static constexpr int kBytes = kBarOff + 512;
  static constexpr int kAlloc = kBytes + 1024;  // slack for 1024-byte alignment
  // P of a step is released to the PV MMAs in kParts key ranges of 128 / kParts keys (bf16
  // P is stored 32 keys at a time, e4m3 P 64 keys at a time).  Two ranges (one kv block
  // each): four 32-key ranges measured 3% slower, each release costing the softmax a wait
  // for its tensor-memory stores.
  static constexpr int kParts = 2;
  static constexpr int kChunksPerPart = 4 / kParts;  // bf16 32-key chunks per part
};

// e4m3 P is stored as P * (s_v / sigma) * kPScale: with the lazy rescale P <= 256, so the
// largest code is 256 * 1.75 = 448, the e4m3 maximum.
constexpr float kPScale = 1.75f;

template <int D, bool FP8, bool VARLEN, bool RASTER = false>
__global__ void __launch_bounds__(fwd::kThreads, 1)
    bsattn_fwd_kernel(const __grid_constant__ CUtensorMap tm_q,
                      const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const FwdParams p) {
  using L = FwdSmem<D, FP8>;
  constexpr int CE = L::kChunkElems;
  constexpr int KS = L::kKStages, VS = L::kVStages;
  extern __shared__ uint8_t smem_raw[];
  // 128-byte-swizzled operand tiles need 1024-byte alignment in the shared window.
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::kBarOff);
  uint64_t* bar_q = bars + 0;
  uint64_t* bar_kfull = bars + 1;
  uint64_t* bar_kempty = bar_kfull + KS;
  uint64_t* bar_vfull = bar_kempty + KS;
  uint64_t* bar_vempty = bar_vfull + VS;
  uint64_t* bar_sfull = bar_vempty + VS;  // [2]
  uint64_t* bar_pfull = bar_sfull + 2;    // [2]
  uint64_t* bar_ppart = bar_pfull + 2;    // [2][3] P of the step's first key ranges stored
  uint64_t* bar_ofull = bar_ppart + 6;
  uint64_t* bar_drain = bar_ofull + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bar_drain + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const AttnDims& a = p.a;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int cta = blockIdx.x + (RASTER ? p.cta_offset : 0);
  int bh, row0, n_ent, rows_here;
  const uint32_t* ent;
  if constexpr (VARLEN) {
    // Which query cluster, and which 256 rows of it, this CTA owns.
    bh = cta / p.cap;
    const int local_cta = cta - bh * p.cap;
    const int32_t* base = p.cta_base + static_cast<long long>(bh) * (p.n_qc + 1);
    if (local_cta >= base[p.n_qc]) return;  // uniform: before any barrier or allocation
    int lo = 0, hi = p.n_qc - 1;              // last cluster with base <= local_cta
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (base[mid] <= local_cta) lo = mid; else hi = mid - 1;
    }
    const int tile = local_cta - base[lo];
    const long long qrow = static_cast<long long>(bh) * p.n_qc + lo;
    const int qs = p.q_starts[qrow], qn = p.q_counts[qrow];
    row0 = qs + tile * fwd::kRowsPerCta;
    rows_here = min(fwd::kRowsPerCta, qn - tile * fwd::kRowsPerCta);
    n_ent = p.ent_counts[qrow];
    ent = p.entries + qrow * p.max_ent;
    if (qs < 0 || qn < 0 || qs > p.S - qn) {  // the cluster's slots must lie inside the head
      if (threadIdx.x == 0)
        record_status(p.status, FLAG_DEVICE_INPUT, DETAIL_CLUSTER_RANGE, static_cast<uint32_t>(qrow), 0u);
      rows_here = 0;
      n_ent = 0;
    }
  } else {
    bh = cta / a.n_cta_per_head;
    row0 = (cta - bh * a.n_cta_per_head) * fwd::kRowsPerCta;
    rows_here = fwd::kRowsPerCta;
    n_ent = p.counts[cta];
    ent = p.entries + static_cast<long long>(cta) * a.n_kb;
  }
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
    for (int t = 0; t < 2; ++t) {
      mbar_init(bar_sfull + t, 1);
      mbar_init(bar_pfull + t, 128);
      for (int q = 0; q < 3; ++q) mbar_init(bar_ppart + 3 * t + q, 128);
    }
    mbar_init(bar_ofull, 1);
    mbar_init(bar_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 9) tmem_alloc(tmem_slot, 512);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // Raster layout: tile u of head h as one 5D box (dims, head, w, h, t) of this batch's
  // tensor map; tiles past the padded grid and slots past the valid grid read as zeros.
  const int head = bh - (bh / a.heads) * a.heads;
  auto raster_tile = [&](uint8_t* dst, const CUtensorMap* map, uint64_t* bar, int ch, int u) {
    int tw, th, tt;
    tile_coords(a.g, u, tw, th, tt);
    tma_load_5d(dst, map, bar, ch * CE, head, tw * 4, th * 4, tt * 4);
  };
  if (warp >= 8) {
    warpgroup_reg_dec<fwd::kRegsProducer>();
    if (warp == 8) {
      // ------------------------------------------------------------ TMA producer
      if (lane == 0 && nsteps > 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        mbar_arrive_expect_tx(bar_q, 2 * L::kQTile);
        for (int t = 0; t < 2; ++t)
          for (int ch = 0; ch < L::kChunks; ++ch) {
            uint8_t* dq = smem + L::kQOff + t * L::kQTile + ch * (128 * 128);
            if constexpr (RASTER) {  // a 128-row Q tile is two 4x4x4 tiles
              raster_tile(dq, &tm_q, bar_q, ch, (row0 + t * 128) >> 6);
              raster_tile(dq + 64 * 128, &tm_q, bar_q, ch, ((row0 + t * 128) >> 6) + 1);
            } else {
              tma_load_3d(dq, &tm_q, bar_q, ch * CE, row0 + t * 128, bh);
            }
          }
        for (int s = 0; s < nsteps; ++s) {
          const int nb = (2 * s + 1 < n_ent) ? 2 : 1;
          // first key row of each of the step's (one or two) 64-row boxes
          const int j0 = VARLEN ? fwd::entry_start(ent[2 * s]) : fwd::entry_block(ent[2 * s]) * 64;
          const int j1 = nb == 2 ? (VARLEN ? fwd::entry_start(ent[2 * s + 1])
                                           : fwd::entry_block(ent[2 * s + 1]) * 64)
                                 : 0;
          const int ks = s % KS;
          if (s >= KS && !mbar_wait(bar_kempty + ks, ((s / KS) - 1) & 1, abort_flag, p.status,
                                    DETAIL_WAIT_K_EMPTY))
            break;
          mbar_arrive_expect_tx(bar_kfull + ks, nb * 64 * L::kRowBytes);
          uint8_t* kst = smem + L::kKOff + ks * L::kKVStage;
          for (int ch = 0; ch < L::kChunks; ++ch) {
            if constexpr (RASTER) {
              raster_tile(kst + ch * (128 * 128), &tm_k, bar_kfull + ks, ch, j0 >> 6);
              if (nb == 2) raster_tile(kst + ch * (128 * 128) + 64 * 128, &tm_k, bar_kfull + ks, ch, j1 >> 6);
            } else {
              tma_load_3d(kst + ch * (128 * 128), &tm_k, bar_kfull + ks, ch * CE, j0, bh);
              if (nb == 2)
                tma_load_3d(kst + ch * (128 * 128) + 64 * 128, &tm_k, bar_kfull + ks, ch * CE,
                            j1, bh);
            }
          }
          const int vs = s % VS;
          if (s >= VS && !mbar_wait(bar_vempty + vs, ((s / VS) - 1) & 1, abort_flag, p.status,
                                    DETAIL_WAIT_V_EMPTY))
            break;
          mbar_arrive_expect_tx(bar_vfull + vs, nb * 64 * L::kRowBytes);
          uint8_t* vst = smem + L::kVOff + vs * L::kKVStage;
          for (int ch = 0; ch < L::kChunks; ++ch) {
            if constexpr (RASTER) {
              raster_tile(vst + ch * (128 * 128), &tm_v, bar_vfull + vs, ch, j0 >> 6);
              if (nb == 2) raster_tile(vst + ch * (128 * 128) + 64 * 128, &tm_v, bar_vfull + vs, ch, j1 >> 6);
            } else {
              tma_load_3d(vst + ch * (128 * 128), &tm_v, bar_vfull + vs, ch * CE, j0, bh);
              if (nb == 2)
                tma_load_3d(vst + ch * (128 * 128) + 64 * 128, &tm_v, bar_vfull + vs, ch * CE,
                            j1, bh);
            }
          }
        }
      }
    } else if (warp == 9) {
      // ------------------------------------------------------------ MMA issuer
      if (lane == 0 && nsteps > 0) {
        const uint32_t q_base = smem_u32(smem + L::kQOff);
        const uint32_t k_base = smem_u32(smem + L::kKOff);
        const uint32_t v_base = smem_u32(smem + L::kVOff);
        constexpr uint32_t kFmt = FP8 ? 0u : 1u;  // e4m3 / bf16
        const uint32_t idesc_pv = make_idesc(kFmt, 1u, 128u, static_cast<uint32_t>(D));
        bool ok = mbar_wait(bar_q, 0, abort_flag, p.status, DETAIL_WAIT_Q);
        // Shared-memory descriptors: built once; the start-address field is the low bits, so
        // a byte offset inside the operand region is added as offset >> 4.
        const uint64_t q_desc0 = make_sdesc_sw128(q_base, 16, 1024);
        const uint64_t k_desc0 = make_sdesc_sw128(k_base, 16, 1024);
        const uint64_t v_desc0 = make_sdesc_sw128(v_base, 128 * 128, 1024);
        auto issue_pv = [&](int t, int sp, int part) {
          // O_t (+)= P_t(sp) V(sp) over key range `part` of the step (kParts ranges of 128 /
          // kParts keys).  One MMA takes 32 bytes of K: 16 keys (bf16) or 32 keys (e4m3), i.e. 8
          // TMEM columns of P and 16 or 32 rows (2 or 4 swizzle atoms) of V.
          constexpr int kKeysPerMma = 32 / L::kElem;
          constexpr int kMmas = 128 / kKeysPerMma;  // for a 2-block step
          constexpr int kPerPart = kMmas / L::kParts;
          const int kk0 = part * kPerPart;
          const int nmma = min(kk0 + kPerPart, (2 * sp + 1 < n_ent) ? kMmas : kMmas / 2);
          const uint64_t vd = v_desc0 + static_cast<uint64_t>(((sp % VS) * L::kKVStage) >> 4);
          const uint32_t p_tmem = tmem + t * 128;
          const uint32_t o_tmem = tmem + 256 + t * D;
  #pragma unroll
          for (int kk = 0; kk < kMmas; ++kk) {
            if (kk < kk0) continue;
            if (kk >= nmma) break;
            const uint64_t bdesc = vd + static_cast<uint64_t>((kk * kKeysPerMma * 128) >> 4);
            if constexpr (FP8)
              mma_f8_ts(o_tmem, p_tmem + kk * 8, bdesc, idesc_pv, (sp > 0 || kk > 0) ? 1u : 0u);
            else
              mma_f16_ts(o_tmem, p_tmem + kk * 8, bdesc, idesc_pv, (sp > 0 || kk > 0) ? 1u : 0u);
          }
        };
        for (int s = 0; s < nsteps && ok; ++s) {
          const int ks = s % KS;
          const int nb = (2 * s + 1 < n_ent) ? 2 : 1;
          const uint32_t idesc_qk = make_idesc(kFmt, 0u, 128u, static_cast<uint32_t>(nb * 64));
          if (!mbar_wait(bar_kfull + ks, (s / KS) & 1, abort_flag, p.status, DETAIL_WAIT_K_FULL)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t kd = k_desc0 + static_cast<uint64_t>((ks * L::kKVStage) >> 4);
          for (int t = 0; t < 2; ++t) {
            if (s > 0) {
              // PV of the previous step range by range, each as soon as its P is stored, while
              // the softmax still works on the later keys.
              if (t == 0 && !mbar_wait(bar_vfull + ((s - 1) % VS), ((s - 1) / VS) & 1, abort_flag,
                                       p.status, DETAIL_WAIT_V_FULL)) {
                ok = false;
                break;
              }
              for (int q = 0; q < L::kParts && ok; ++q) {
                const bool last = q + 1 == L::kParts;
                ok = mbar_wait(last ? bar_pfull + t : bar_ppart + 3 * t + q, (s - 1) & 1,
                               abort_flag, p.status, last ? DETAIL_WAIT_P_FULL : DETAIL_WAIT_P_PART);
                if (!ok) break;
                tc_fence_after();
                issue_pv(t, s - 1, q);
              }
              if (!ok) break;
              if (t == 1) mma_commit(bar_vempty + ((s - 1) % VS));
            }
            const uint64_t qd = q_desc0 + static_cast<uint64_t>((t * L::kQTile) >> 4);
            const uint32_t s_tmem = tmem + t * 128;
            // K (= head dim) advances 32 bytes per MMA inside each 128-byte swizzle chunk.
  #pragma unroll
            for (int kk = 0; kk < L::kRowBytes / 32; ++kk) {
              const uint64_t off = static_cast<uint64_t>(((kk >> 2) * (128 * 128) + (kk & 3) * 32) >> 4);
              const uint64_t adesc = qd + off;
              const uint64_t bdesc = kd + off;
              if constexpr (FP8)
                mma_f8_ss(s_tmem, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
              else
                mma_f16_ss(s_tmem, adesc, bdesc, idesc_qk, kk > 0 ? 1u : 0u);
            }
            mma_commit(bar_sfull + t);
          }
          if (!ok) break;
          mma_commit(bar_kempty + ks);
        }
        if (ok) {
          const int sl = nsteps - 1;
          for (int t = 0; t < 2 && ok; ++t) {
            if (t == 0 && !mbar_wait(bar_vfull + (sl % VS), (sl / VS) & 1, abort_flag, p.status,
                                     DETAIL_WAIT_V_FULL)) {
              ok = false;
              break;
            }
            for (int q = 0; q < L::kParts && ok; ++q) {
              const bool last = q + 1 == L::kParts;
              ok = mbar_wait(last ? bar_pfull + t : bar_ppart + 3 * t + q, sl & 1, abort_flag,
                             p.status, last ? DETAIL_WAIT_P_FULL : DETAIL_WAIT_P_PART);
              if (!ok) break;
              tc_fence_after();
              issue_pv(t, sl, q);
            }
          }
          if (ok) mma_commit(bar_ofull);
        }
        // Whatever happened, let every issued MMA finish before TMEM is released.
        mma_commit(bar_drain);
        mbar_wait_drain(bar_drain, 0, p.status, DETAIL_WAIT_O_FULL);
      }
    }
  } else {
    warpgroup_reg_inc<fwd::kRegsSoftmax>();
    // ------------------------------------------------------------ softmax warps
    const int t = warp >> 2;           // Q tile
    const int wq = warp & 3;           // TMEM lane quarter
    const int row = wq * 32 + lane;    // row inside the tile
    const int local = t * 128 + row;   // row inside the CTA
    const int slot = row0 + local;     // query slot inside the head
    const int qsel = VARLEN ? 0 : local / a.q_block;
    // in_range: the row is this CTA's to write; q_valid: it holds a token
    // raster layout: the token a slot holds (-1 for a pad slot); only tokens are written
    const int token = (RASTER && slot < a.g.Np) ? slot_to_token(a.g, slot) : -1;
    const bool in_range = VARLEN ? local < rows_here : (RASTER ? token >= 0 : slot < a.g.Np);
    const bool q_valid = VARLEN ? in_range : (in_range && slot_valid(a.g, slot));
    const long long head_slots = VARLEN ? p.S : a.g.Np;
    const uint32_t lane_base = tmem + (static_cast<uint32_t>(wq * 32) << 16);
    const uint32_t s_addr = lane_base + t * 128;
    const uint32_t o_addr = lane_base + 256 + t * D;
    const float c = p.scale_log2;
    // e4m3: logits carry the Q tile scale of this row and the K tile scale of each block.
    float cq = c;
    float sig = 1.f;
    if constexpr (FP8) {
      const long long tbase = static_cast<long long>(bh) * a.n_kb;
      cq = c * (in_range ? p.q_scales[tbase + (slot >> 6)] : 0.f);
      sig = p.sigma[cta];
    }
    float m_run = -INFINITY;  // running max, scaled log2 units
    float l_run = 0.f;
    bool ok = true;

    uint32_t e0n = nsteps > 0 ? ld_early_u32(ent) : 0u;
    uint32_t e1n = n_ent > 1 ? ld_early_u32(ent + 1) : 0u;
    for (int s = 0; s < nsteps; ++s) {
      const int nb = (2 * s + 1 < n_ent) ? 2 : 1;
      const uint32_t e0 = e0n, e1 = e1n;
      if (s + 1 < nsteps) {
        e0n = ld_early_u32(ent + 2 * s + 2);
        e1n = (2 * s + 3 < n_ent) ? ld_early_u32(ent + 2 * s + 3) : 0u;
      }
      const bool got = __all_sync(
          0xffffffffu, mbar_wait(bar_sfull + t, s & 1, abort_flag, p.status, DETAIL_WAIT_S_FULL));
      if (!got) {
        ok = false;
        break;
      }
      tc_fence_after();
      float sv[128];
      if constexpr (FP8) {
        // one 64-column load per kv block (e4m3: 141.7 vs 143.1 ms at 720p; bf16 measured
        // 0.5% slower with it, so it keeps the 32-column loads)
        tmem_ld64(s_addr + 0, sv + 0);
        if (nb == 2) tmem_ld64(s_addr + 64, sv + 64);
      } else {
        tmem_ld32(s_addr + 0, sv + 0);
        tmem_ld32(s_addr + 32, sv + 32);
        if (nb == 2) {
          tmem_ld32(s_addr + 64, sv + 64);
          tmem_ld32(s_addr + 96, sv + 96);
        }
      }
      tmem_ld_wait();
      // Column masks (warp-uniform: a warp's rows share one query block).  A block this
      // query block did not keep, or a pad key, or the absent half of a 1-block step -> -inf.
      uint64_t mk0 = 0ull, mk1 = 0ull;
      if constexpr (VARLEN) {  // every row keeps every run; a short run masks its tail
        mk0 = fwd::entry_len_mask(e0);
        if (nb == 2) mk1 = fwd::entry_len_mask(e1);
      } else {
        if ((e0 >> qsel) & 1u) mk0 = ((e0 >> 4) & 1u) ? tile_valid_mask(a.g, fwd::entry_block(e0)) : ~0ull;
        if (nb == 2 && ((e1 >> qsel) & 1u))
          mk1 = ((e1 >> 4) & 1u) ? tile_valid_mask(a.g, fwd::entry_block(e1)) : ~0ull;
      }
      if ((mk0 & mk1) != ~0ull) {
        const uint32_t mw[4] = {static_cast<uint32_t>(mk0), static_cast<uint32_t>(mk0 >> 32),
                                static_cast<uint32_t>(mk1), static_cast<uint32_t>(mk1 >> 32)};
#pragma unroll
        for (int i = 0; i < 128; ++i) sv[i] = ((mw[i >> 5] >> (i & 31)) & 1u) ? sv[i] : -INFINITY;
      }
      // log2-domain multiplier of each half (block) of the step
      float fb0 = c, fb1 = c, pv0 = 1.f, pv1 = 1.f;
      if constexpr (FP8) {
        const long long tbase = static_cast<long long>(bh) * a.n_kb;
        const int j0 = fwd::entry_block(e0), j1 = fwd::entry_block(e1);
        fb0 = cq * p.k_scales[tbase + j0];
        fb1 = nb == 2 ? cq * p.k_scales[tbase + j1] : 0.f;
        pv0 = p.v_scales[tbase + j0] / sig * kPScale;
        pv1 = nb == 2 ? p.v_scales[tbase + j1] / sig * kPScale : 0.f;
      }
      float mx[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = sv[i];
#pragma unroll
      for (int i = 4; i < 64; ++i) mx[i & 3] = fmaxf(mx[i & 3], sv[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[4 + i] = sv[64 + i];
#pragma unroll
      for (int i = 68; i < 128; ++i) mx[4 + (i & 3)] = fmaxf(mx[4 + (i & 3)], sv[i]);
      const float mh0 = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3]));
      const float mh1 = fmaxf(fmaxf(mx[4], mx[5]), fmaxf(mx[6], mx[7]));
      // multipliers are > 0, so the scaled max is the max of the scaled half maxima
      const float m_new = fmaxf(mh0 == -INFINITY ? -INFINITY : mh0 * fb0,
                                mh1 == -INFINITY ? -INFINITY : mh1 * fb1);
      float factor = 1.f;
      bool resc = false;
      if (m_new > m_run + fwd::kRescaleLog2 || (m_run == -INFINITY && m_new != -INFINITY)) {
        if (m_run != -INFINITY) {
          factor = fast_exp2(m_run - m_new);
          resc = true;
        }
        m_run = m_new;
      }
      // P = exp2(S*f - m), stored over S_t as it is produced: bf16 pairs, 16 columns per 32
      // keys; or e4m3 quads (P scaled by the block's V scale), 16 columns per 64 keys.  As
      // each key range's P is stored, its barrier lets the MMA start that part of PV --
      // unless this warp must first rescale its rows of O: then every part is released at
      // the end.  Every part barrier is arrived at once per step (absent keys included).
      const float m_use = (m_run == -INFINITY) ? 0.f : m_run;
      const bool warp_resc = __any_sync(0xffffffffu, resc);
      auto release_part = [&](int q) {
        if (!warp_resc) {
          tmem_st_wait();
          tc_fence_before();
          mbar_arrive(bar_ppart + 3 * t + q);
        }
      };
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
      if constexpr (!FP8) {
#pragma unroll
        for (int ch = 0; ch < 4; ++ch) {
          if (ch >= 2 && nb == 1) break;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float p0 = fast_exp2(fmaf(sv[32 * ch + 2 * i], c, -m_use));
            const float p1 = fast_exp2(fmaf(sv[32 * ch + 2 * i + 1], c, -m_use));
            ls[i & 3] += p0 + p1;
            pk[i] = pack_bf16x2(p0, p1);
          }
          BSA_TMEM_ST_X16(s_addr + 16 * ch, pk);
          if ((ch + 1) % L::kChunksPerPart == 0 && (ch + 1) / L::kChunksPerPart < L::kParts)
            release_part((ch + 1) / L::kChunksPerPart - 1);
        }
      } else {
#pragma unroll
        for (int b = 0; b < 2; ++b) {
          if (b == 1 && nb == 1) break;
          const float fb = b ? fb1 : fb0;
          const float pv = b ? pv1 : pv0;
          uint32_t pk[16];
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            float pq[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              pq[u] = fast_exp2(fmaf(sv[64 * b + 4 * i + u], fb, -m_use));
              ls[u] += pq[u];
            }
            const uint32_t lo = pack_e4m3x2(pq[0] * pv, pq[1] * pv);
            const uint32_t hi = pack_e4m3x2(pq[2] * pv, pq[3] * pv);
            pk[i] = lo | (hi << 16);
          }
          BSA_TMEM_ST_X16(s_addr + 16 * b, pk);
          if (b == 0) release_part(0);
        }
      }
      // factor is 1 unless this row's reference max moved; it scales only the old sum.
      l_run = fmaf(l_run, factor, (ls[0] + ls[1]) + (ls[2] + ls[3]));
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
      if (warp_resc) {
        for (int q = 0; q + 1 < L::kParts; ++q) mbar_arrive(bar_ppart + 3 * t + q);
      } else if (!FP8 && L::kParts == 4 && nb == 1) {
        mbar_arrive(bar_ppart + 3 * t + 2);  // keys 64-95: absent in a one-block step
      }
      mbar_arrive(bar_pfull + t);
    }

    // ------------------------------------------------------------ epilogue
    // e4m3: O was accumulated from P * s_v / sigma * kPScale and V / s_v.
    const float o_mult = FP8 ? sig / kPScale : 1.f;
    const float inv_l = (l_run > 0.f && q_valid) ? o_mult / l_run : 0.f;
    bool have_o = ok && nsteps > 0;
    if (have_o) {
      have_o = __all_sync(0xffffffffu,
                          mbar_wait(bar_ofull, 0, abort_flag, p.status, DETAIL_WAIT_O_FULL));
      tc_fence_after();
    }
    __nv_bfloat16* orow =
        RASTER ? p.out + ((static_cast<long long>(p.raster_b) * a.g.S + (token < 0 ? 0 : token)) *
                              a.heads + head) * D
               : p.out + (static_cast<long long>(bh) * head_slots + slot) * D;
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
    if (p.lse != nullptr && in_range) {
      const float lse = (l_run > 0.f && q_valid) ? (m_run + __log2f(l_run)) * 0.6931471805599453f
                                                 : -INFINITY;
      if constexpr (RASTER)
        p.lse[static_cast<long long>(bh) * a.g.S + token] = lse;
      else
        p.lse[static_cast<long long>(bh) * head_slots + slot] = lse;
    }
  }

  __syncwarp();
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Scratch after the status header: counts int32 [ctas], sigma fp32 [ctas] (e4m3 only),
// entries uint32 [ctas][n_kb].
size_t fwd_scratch_bytes(const AttnDims& a) {
  const long long ctas = static_cast<long long>(a.batch) * a.heads * a.n_cta_per_head;
  const size_t counts = (static_cast<size_t>(ctas) * 4 + 255) & ~static_cast<size_t>(255);
  return 2 * counts + static_cast<size_t>(ctas) * a.n_kb * 4;
}

// The register split between warpgroups assumes the kernel is launched at exactly
// fwd::kRegsLaunch registers a thread; with fewer, the softmax warpgroups' increase could
// never be satisfied, so such a build is refused before any launch.
template <typename Kernel>
static cudaError_t check_fwd_registers(Kernel kernel) {
  cudaFuncAttributes attr;
  const cudaError_t e = cudaFuncGetAttributes(&attr, kernel);
  if (e != cudaSuccess) return e;
  return attr.numRegs == fwd::kRegsLaunch ? cudaSuccess : cudaErrorInvalidConfiguration;
}

template <int D, bool FP8, bool VARLEN>
static cudaError_t launch_fwd(const AttnDims& a, int rows_per_head, const void* q, const void* k,
                              const void* v, const FwdParams& prm, long long ctas,
                              cudaStream_t stream) {
  using L = FwdSmem<D, FP8>;
  CUtensorMap tq, tk, tv;
  const int bh = a.batch * a.heads;
  const CUtensorMapDataType dt = FP8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
  const int eb = L::kElem, ce = L::kChunkElems;
  cudaError_t e = encode_tmap_3d(&tq, q, dt, eb, D, rows_per_head, bh, ce, 128);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tk, k, dt, eb, D, rows_per_head, bh, ce, 64);
  if (e != cudaSuccess) return e;
  e = encode_tmap_3d(&tv, v, dt, eb, D, rows_per_head, bh, ce, 64);
  if (e != cudaSuccess) return e;
  e = check_fwd_registers(bsattn_fwd_kernel<D, FP8, VARLEN>);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bsattn_fwd_kernel<D, FP8, VARLEN>,
                           cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  bsattn_fwd_kernel<D, FP8, VARLEN>
      <<<static_cast<unsigned>(ctas), fwd::kThreads, L::kAlloc, stream>>>(tq, tk, tv, prm);
  return cudaGetLastError();
}

cudaError_t launch_bsattn_fwd(const AttnDims& a, int fp8, const void* q, const void* k,
                              const void* v, const float* q_scales, const float* k_scales,
                              const float* v_scales, const int32_t* row_ptr,
                              const int32_t* col_idx, float softmax_scale, void* out, float* lse,
                              void* ws, cudaStream_t stream) {
  if (fp8 && a.head_dim != 128) return cudaErrorNotSupported;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const long long ctas = static_cast<long long>(a.batch) * a.heads * a.n_cta_per_head;
  if (ctas == 0) return cudaSuccess;
  const size_t counts_bytes = (static_cast<size_t>(ctas) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* counts = reinterpret_cast<int32_t*>(base + kStatusBytes);
  float* sigma = reinterpret_cast<float*>(base + kStatusBytes + counts_bytes);
  uint32_t* entries = reinterpret_cast<uint32_t*>(base + kStatusBytes + 2 * counts_bytes);
  bsattn_schedule_kernel<<<static_cast<unsigned>(ctas), 256, 0, stream>>>(
      a, row_ptr, col_idx, counts, entries, fp8 ? v_scales : nullptr, fp8 ? sigma : nullptr,
      status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  FwdParams prm;
  prm.a = a;
  prm.counts = counts;
  prm.entries = entries;
  prm.q_scales = q_scales;
  prm.k_scales = k_scales;
  prm.v_scales = v_scales;
  prm.sigma = sigma;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.S = 0;
  prm.n_qc = 0;
  prm.cap = 0;
  prm.max_ent = 0;
  prm.q_starts = prm.q_counts = prm.cta_base = prm.ent_counts = nullptr;
  prm.raster_b = 0;
  prm.cta_offset = 0;
  if (fp8) return launch_fwd<128, true, false>(a, a.g.Np, q, k, v, prm, ctas, stream);
  if (a.head_dim == 128) return launch_fwd<128, false, false>(a, a.g.Np, q, k, v, prm, ctas, stream);
  return launch_fwd<64, false, false>(a, a.g.Np, q, k, v, prm, ctas, stream);
}

// ---------------------------------------------------------------------------------------
// Raster layout: Q, K, V and O are [B, S, Hh, D] bf16 in token order.  The kernel loads each
// 4x4x4 tile with one 5D TMA box (whose shared-memory image is the tile-major block) and
// writes each query row to its token; the lists, schedule and arithmetic are those of
// bsa_fwd, so the result equals bsa_fwd on tile-permuted inputs, permuted back.
template <int D>
static cudaError_t launch_fwd_raster(const AttnDims& a, const void* q, const void* k,
                                     const void* v, FwdParams prm, cudaStream_t stream) {
  using L = FwdSmem<D, false>;
  cudaError_t e = check_fwd_registers(bsattn_fwd_kernel<D, false, false, true>);
  if (e != cudaSuccess) return e;
  e = cudaFuncSetAttribute(bsattn_fwd_kernel<D, false, false, true>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, L::kAlloc);
  if (e != cudaSuccess) return e;
  const long long per_batch = static_cast<long long>(a.g.S) * a.heads * D;  // elements
  for (int b = 0; b < a.batch; ++b) {  // 5D maps cover one batch
    CUtensorMap tq, tk, tv;
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(q) + b * per_batch;
    const __nv_bfloat16* kb = static_cast<const __nv_bfloat16*>(k) + b * per_batch;
    const __nv_bfloat16* vb = static_cast<const __nv_bfloat16*>(v) + b * per_batch;
    e = encode_tmap_raster_tiles(&tq, qb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.heads, a.g.W,
                                 a.g.H, a.g.T);
    if (e != cudaSuccess) return e;
    e = encode_tmap_raster_tiles(&tk, kb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.heads, a.g.W,
                                 a.g.H, a.g.T);
    if (e != cudaSuccess) return e;
    e = encode_tmap_raster_tiles(&tv, vb, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, D, a.heads, a.g.W,
                                 a.g.H, a.g.T);
    if (e != cudaSuccess) return e;
    prm.raster_b = b;
    prm.cta_offset = b * a.heads * a.n_cta_per_head;
    const unsigned ctas = static_cast<unsigned>(a.heads * a.n_cta_per_head);
    bsattn_fwd_kernel<D, false, false, true><<<ctas, fwd::kThreads, L::kAlloc, stream>>>(tq, tk, tv, prm);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return cudaSuccess;
}

cudaError_t launch_bsattn_fwd_raster(const AttnDims& a, const void* q, const void* k,
                                     const void* v, const int32_t* row_ptr, const int32_t* col_idx,
                                     float softmax_scale, void* out, float* lse, void* ws,
                                     cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const long long ctas = static_cast<long long>(a.batch) * a.heads * a.n_cta_per_head;
  if (ctas == 0) return cudaSuccess;
  const size_t counts_bytes = (static_cast<size_t>(ctas) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* counts = reinterpret_cast<int32_t*>(base + kStatusBytes);
  uint32_t* entries = reinterpret_cast<uint32_t*>(base + kStatusBytes + 2 * counts_bytes);
  bsattn_schedule_kernel<<<static_cast<unsigned>(ctas), 256, 0, stream>>>(
      a, row_ptr, col_idx, counts, entries, nullptr, nullptr, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  FwdParams prm{};
  prm.a = a;
  prm.counts = counts;
  prm.entries = entries;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  if (a.head_dim == 128) return launch_fwd_raster<128>(a, q, k, v, prm, stream);
  return launch_fwd_raster<64>(a, q, k, v, prm, stream);
}

// ---------------------------------------------------------------------------------------
// Cluster order ("Sparse VideoGen2", Abstract: semantic-aware permutation, densified layout
// without padding).  Q, K and V are [B, Hh, S, D] with the tokens of every cluster in
// consecutive slots; query cluster c of head bh owns slots [q_starts, q_starts + q_counts)
// and attends to the key clusters listed in CSR row bh * n_qc + c.

// Per (bh, query cluster): the runs of <= 64 keys covering its selected key clusters, in
// list order.  One CTA per CSR row; validates the row like bsattn_schedule_kernel.  Selected
// key clusters whose slot ranges touch (consecutive clusters of the cluster order, empty
// ones between them included) form one span, cut into 64-key runs from its start, so only
// a span's last run is partial: the keys attended are the same, with fewer masked columns.
__global__ void __launch_bounds__(256) cluster_schedule_kernel(
    int n_rows, int n_kc, int max_ent, int S, const int32_t* __restrict__ row_ptr,
    const int32_t* __restrict__ col_idx, const int32_t* __restrict__ k_starts,
    const int32_t* __restrict__ k_counts, int32_t* __restrict__ ent_counts,
    uint32_t* __restrict__ entries, uint32_t* status) {
  __shared__ int st_sm[256], cn_sm[256];
  const int r = blockIdx.x;
  const int bh = r / n_rows;  // n_rows = query clusters per head
  const int tid = threadIdx.x;
  const int beg = row_ptr[r], end = row_ptr[r + 1];
  if (beg < 0 || end < beg || end - beg > n_kc) {
    if (tid == 0) {
      record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_ROWPTR, static_cast<uint32_t>(r), 0u);
      ent_counts[r] = 0;
    }
    return;
  }
  uint32_t* out = entries + static_cast<long long>(r) * max_ent;
  // walk state (thread 0): current span [span_s, span_e), next run start nb, runs written
  int span_e = -1, nb = 0, pos = 0;
  auto emit = [&](int start, int len) {
    if (pos < max_ent) out[pos] = (static_cast<uint32_t>(start) << 7) | static_cast<uint32_t>(len);
    ++pos;
  };
  for (int e0 = beg; e0 < end; e0 += 256) {
    const int e = e0 + tid;
    int start = 0, cnt = 0;
    if (e < end) {
      const int kc = col_idx[e];
      if (kc < 0 || kc >= n_kc) {
        record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_RANGE, static_cast<uint32_t>(r),
                      static_cast<uint32_t>(e));
      } else {
        if (e > beg && col_idx[e - 1] >= kc)
          record_status(status, FLAG_DEVICE_INPUT, DETAIL_CSR_ORDER, static_cast<uint32_t>(r),
                        static_cast<uint32_t>(e));
        start = k_starts[static_cast<long long>(bh) * n_kc + kc];
        cnt = k_counts[static_cast<long long>(bh) * n_kc + kc];
        if (start < 0 || cnt < 0 || start > S - cnt) {  // runs must lie inside the head
          record_status(status, FLAG_DEVICE_INPUT, DETAIL_CLUSTER_RANGE, static_cast<uint32_t>(r),
                        static_cast<uint32_t>(e));
          start = 0;
          cnt = 0;
        }
      }
    }
    st_sm[tid] = start;
    cn_sm[tid] = cnt;
    __syncthreads();
    if (tid == 0) {
      const int n = min(256, end - e0);
      for (int i = 0; i < n; ++i) {
        const int a0 = st_sm[i], c0 = cn_sm[i];
        if (c0 == 0) continue;
        if (a0 != span_e) {  // a new span: the previous one's partial run first
          if (span_e >= 0 && nb < span_e) emit(nb, span_e - nb);
          nb = a0;
        }
        span_e = a0 + c0;
        for (; nb + 64 <= span_e; nb += 64) emit(nb, 64);
      }
    }
    __syncthreads();
  }
  if (tid == 0) {
    if (span_e >= 0 && nb < span_e) emit(nb, span_e - nb);
    if (pos > max_ent) {
      record_status(status, FLAG_CAPACITY, DETAIL_COL_CAPACITY, static_cast<uint32_t>(r), 0u);
      pos = max_ent;
    }
    ent_counts[r] = pos;
  }
}

// cta_base[bh][c] = first CTA of query cluster c (256 rows per CTA); [bh][n_qc] = total.
__global__ void __launch_bounds__(1024) cluster_cta_base_kernel(int n_qc,
                                                                const int32_t* __restrict__ q_counts,
                                                                int32_t* __restrict__ cta_base) {
  __shared__ int warp_tot[32];
  const int bh = blockIdx.x;
  const int tid = threadIdx.x;
  int base = 0;
  for (int c0 = 0; c0 < n_qc; c0 += 1024) {
    const int c = c0 + tid;
    const int n = c < n_qc ? max(q_counts[static_cast<long long>(bh) * n_qc + c], 0) : 0;
    const int tiles = (n + fwd::kRowsPerCta - 1) / fwd::kRowsPerCta;
    int incl = tiles;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane_id() >= static_cast<uint32_t>(o)) incl += y;
    }
    if (lane_id() == 31) warp_tot[tid >> 5] = incl;
    __syncthreads();
    int before = 0, tot = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < (tid >> 5)) before += warp_tot[w];
      tot += warp_tot[w];
    }
    if (c < n_qc) cta_base[static_cast<long long>(bh) * (n_qc + 1) + c] = base + before + incl - tiles;
    base += tot;
    __syncthreads();
  }
  if (tid == 0) cta_base[static_cast<long long>(bh) * (n_qc + 1) + n_qc] = base;
}

int cluster_max_entries(int S, int n_kc) { return (S + 63) / 64 + n_kc; }
int cluster_ctas_per_head(int S, int n_qc) { return n_qc + (S + fwd::kRowsPerCta - 1) / fwd::kRowsPerCta; }

// Scratch after the status header: ent_counts int32 [BH * n_qc], cta_base int32
// [BH * (n_qc + 1)], entries uint32 [BH * n_qc][max_ent].
size_t cluster_fwd_scratch_bytes(int bhn, int S, int n_qc, int n_kc) {
  const size_t a = (static_cast<size_t>(bhn) * n_qc * 4 + 255) & ~static_cast<size_t>(255);
  const size_t b = (static_cast<size_t>(bhn) * (n_qc + 1) * 4 + 255) & ~static_cast<size_t>(255);
  return a + b + static_cast<size_t>(bhn) * n_qc * cluster_max_entries(S, n_kc) * 4;
}

cudaError_t launch_cluster_fwd(int batch, int heads, int head_dim, int S, int n_qc, int n_kc,
                               const void* q, const void* k, const void* v,
                               const int32_t* q_starts, const int32_t* q_counts,
                               const int32_t* k_starts, const int32_t* k_counts,
                               const int32_t* row_ptr, const int32_t* col_idx,
                               float softmax_scale, void* out, float* lse, void* ws,
                               cudaStream_t stream) {
  const int bhn = batch * heads;
  if (bhn == 0 || S == 0) return cudaSuccess;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const size_t a_bytes = (static_cast<size_t>(bhn) * n_qc * 4 + 255) & ~static_cast<size_t>(255);
  const size_t b_bytes = (static_cast<size_t>(bhn) * (n_qc + 1) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* ent_counts = reinterpret_cast<int32_t*>(base + kStatusBytes);
  int32_t* cta_base = reinterpret_cast<int32_t*>(base + kStatusBytes + a_bytes);
  uint32_t* entries = reinterpret_cast<uint32_t*>(base + kStatusBytes + a_bytes + b_bytes);
  const int max_ent = cluster_max_entries(S, n_kc);
  cluster_schedule_kernel<<<static_cast<unsigned>(bhn * n_qc), 256, 0, stream>>>(
      n_qc, n_kc, max_ent, S, row_ptr, col_idx, k_starts, k_counts, ent_counts, entries, status);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  cluster_cta_base_kernel<<<static_cast<unsigned>(bhn), 1024, 0, stream>>>(n_qc, q_counts, cta_base);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  AttnDims a{};
  a.batch = batch;
  a.heads = heads;
  a.head_dim = head_dim;
  a.q_block = 64;
  FwdParams prm{};
  prm.a = a;
  prm.entries = entries;
  prm.out = static_cast<__nv_bfloat16*>(out);
  prm.lse = lse;
  prm.status = status;
  prm.scale_log2 = softmax_scale * 1.4426950408889634f;
  prm.S = S;
  prm.n_qc = n_qc;
  prm.cap = cluster_ctas_per_head(S, n_qc);
  prm.max_ent = max_ent;
  prm.q_starts = q_starts;
  prm.q_counts = q_counts;
  prm.cta_base = cta_base;
  prm.ent_counts = ent_counts;
  const long long ctas = static_cast<long long>(bhn) * prm.cap;
  if (head_dim == 128) return launch_fwd<128, false, true>(a, S, q, k, v, prm, ctas, stream);
  return launch_fwd<64, false, true>(a, S, q, k, v, prm, ctas, stream);
}

}  // namespace bsa
