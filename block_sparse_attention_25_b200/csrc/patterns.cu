// Static structured kv-block lists (CSR) for the block-sparse forward.
//
// "Sparse-vDiT", Abstract: diagonal, multi-diagonal and vertical-stripe attention
// structures recur across layers and heads.  "GRAT", Abstract: queries of a group attend
// to a shared, structured key region: surrounding blocks or criss-cross lines.
// Block granularity is the 4x4x4 tile in tile-major order (one kv block per tile); a
// query block covers its own tile(s) and keeps kv block j when any enabled predicate
// holds for one of them (union over kinds).  The lists are the same for every (batch,
// head); each CSR row is still written out so the forward sees an ordinary CSR.
//
// One warp per distinct CSR row (the n_qb rows of one (batch, head)): 32 kv blocks per
// ballot -> kept bitmap + count in the workspace; a copy kernel repeats them for the other
// (batch, head) pairs; then the selection's scan and compaction kernels turn the bitmaps
// into row_ptr/col_idx.
#include "bsa_kernels.cuh"

namespace bsa {

__device__ __forceinline__ bool pattern_keep(const PatternParams& pp, int nth, int ntw, int per,
                                             int i, int j) {
  if ((pp.kinds & PAT_VERTICAL_STRIPE) && pp.stripe_stride > 0 &&
      j % pp.stripe_stride == pp.stripe_offset)
    return true;
  const int jt = j / (nth * ntw), jh = (j / ntw) % nth, jw = j % ntw;
  for (int u = i * per; u < (i + 1) * per; ++u) {
    const int d = j - u;
    if ((pp.kinds & PAT_DIAGONAL) && abs(d) <= pp.diag_width) return true;
    if (pp.kinds & PAT_MULTI_DIAGONAL) {
      for (int k = 1; k <= pp.multi_count; ++k) {
        if (abs(d - k * pp.multi_period) <= pp.diag_width) return true;
        if (abs(d + k * pp.multi_period) <= pp.diag_width) return true;
      }
    }
    const int ut = u / (nth * ntw), uh = (u / ntw) % nth, uw = u % ntw;
    if ((pp.kinds & PAT_SURROUNDING) && abs(jt - ut) <= pp.radius_t &&
        abs(jh - uh) <= pp.radius_h && abs(jw - uw) <= pp.radius_w)
      return true;
    if ((pp.kinds & PAT_CRISS_CROSS) && (int(jt == ut) + int(jh == uh) + int(jw == uw)) >= 2)
      return true;
  }
  return false;
}

__global__ void __launch_bounds__(256) pattern_rows_kernel(PatternParams pp, int nth, int ntw,
                                                           int q_block, int n_qb, int n_kb,
                                                           long long rows,
                                                           int32_t* __restrict__ counts,
                                                           uint32_t* __restrict__ bitmaps,
                                                           int words) {
  const long long r = static_cast<long long>(blockIdx.x) * 8 + (threadIdx.x >> 5);
  if (r >= rows) return;
  const int lane = threadIdx.x & 31;
  const int i = static_cast<int>(r % n_qb);
  const int per = q_block / 64;
  uint32_t* out = bitmaps + r * words;
  int kept = 0;
  for (int j0 = 0; j0 < n_kb; j0 += 32) {
    const int j = j0 + lane;
    const bool keep = j < n_kb && pattern_keep(pp, nth, ntw, per, i, j);
    const unsigned b = __ballot_sync(0xffffffffu, keep);
    if (lane == 0) out[j0 >> 5] = b;
    kept += __popc(b);
  }
  if (lane == 0) counts[r] = kept;
}

// Rows [n_qb, rows): the counts and bitmap words of row r % n_qb.  One thread per word.
__global__ void __launch_bounds__(256) pattern_repeat_kernel(long long rows, int n_qb, int words,
                                                             int32_t* __restrict__ counts,
                                                             uint32_t* __restrict__ bitmaps) {
  const long long w = static_cast<long long>(blockIdx.x) * 256 + threadIdx.x;
  const long long total = (rows - n_qb) * words;
  if (w >= total) return;
  const long long r = n_qb + w / words;
  const int k = static_cast<int>(w - (r - n_qb) * words);
  const int src = static_cast<int>(r % n_qb);
  bitmaps[r * words + k] = bitmaps[static_cast<long long>(src) * words + k];
  if (k == 0) counts[r] = counts[src];
}

cudaError_t launch_pattern_csr(const AttnDims& a, const PatternParams& pp_in, int32_t* row_ptr,
                               int32_t* col_idx, long long col_capacity, void* ws,
                               cudaStream_t stream) {
  PatternParams pp = pp_in;
  if (pp.multi_period <= 0) pp.multi_period = a.g.nth * a.g.ntw;
  const long long rows = 1LL * a.batch * a.heads * a.n_qb;
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const int words = (a.n_kb + 31) / 32;
  const size_t counts_bytes = (static_cast<size_t>(rows) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* counts = reinterpret_cast<int32_t*>(base + kStatusBytes);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(base + kStatusBytes + counts_bytes);
  if (rows == 0) return cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), stream);
  // the lists are the same for every (batch, head): evaluate the n_qb rows of the first
  // one and repeat them
  pattern_rows_kernel<<<static_cast<unsigned>((a.n_qb + 7) / 8), 256, 0, stream>>>(
      pp, a.g.nth, a.g.ntw, a.q_block, a.n_qb, a.n_kb, a.n_qb, counts, bitmaps, words);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  if (rows > a.n_qb) {
    const long long total = (rows - a.n_qb) * words;
    pattern_repeat_kernel<<<static_cast<unsigned>((total + 255) / 256), 256, 0, stream>>>(
        rows, a.n_qb, words, counts, bitmaps);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  return launch_bitmap_to_csr(counts, bitmaps, rows, words, row_ptr, col_idx, col_capacity,
                              status, stream);
}

}  // namespace bsa
