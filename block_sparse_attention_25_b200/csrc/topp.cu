// Retained-mass (top-p) block selection into CSR lists.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: for each head and query block keep the smallest key/value block set whose
// attention mass meets the threshold.  "Sparse VideoGen2", Abstract: top-p dynamic
// budget control is the same per-row operator.
//
// Per row the masses become integers q = rint(m * 2^40) and the target is
// ceil(tau * sum q) (one fp64 multiply).  The shortest prefix of the (q desc, index asc)
// order that reaches the target is found without sorting: an exact quickselect over the
// row's values (64-bit integer sums reduced over a warp) finds the value t* of the last
// kept element and the sum A of everything above it; all blocks with q > t*
// are kept, plus the ceil((target - A) / t*) lowest-index blocks with q == t*.  Integer
// arithmetic makes the result independent of reduction order, so it is bit-identical to
// a sequential sort-and-scan.
//
// Kernels: (1) select, one warp per row -> kept bitmap + count in the workspace;
// (2) exclusive scan of the counts -> row_ptr; (3) compaction, one warp per row ->
// col_idx ascending.
#include <mutex>

#include "bsa_kernels.cuh"

namespace bsa {


// One warp per row, kSelWarps rows per CTA, warp-synchronous (no CTA barriers).
// Shared memory per warp: the row's fixed-point masses (n_kb uint64) and the candidate
// list (n_kb uint32 row indices).
constexpr int kSelWarps = 4;
constexpr int kBatch = 8;  // elements per lane loaded back to back in each pass over a row

__device__ __forceinline__ unsigned long long warp_sum_u64(unsigned long long v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
// Per row: the masses become integers in shared memory, then a quickselect finds the value
// t* of the last kept element and the sum A of everything above it.  Each round takes a
// pivot p (median of three candidates), sums the candidates above p and counts those equal
// to it (exact 64-bit integer sums, reduced over the warp), and either stops (t* = p), or
// keeps only the candidates above p, or adds everything >= p to A and keeps only those
// below p.  Every round removes the pivot's value from the candidates, so the loop ends;
// the candidate list (row indices) is compacted in place, so the work is about four passes
// over the row whatever its value range.  The final pass walks the row 32 blocks at a time,
// so a ballot of the keep decisions is one bitmap word, in index order (ties go to the
// lower index).
__device__ __forceinline__ unsigned long long median3(unsigned long long a, unsigned long long b,
                                                      unsigned long long c) {
  const unsigned long long lo = a < b ? a : b, hi = a < b ? b : a;
  return c < lo ? lo : (c > hi ? hi : c);
}

__global__ void __launch_bounds__(32 * kSelWarps) topp_select_rows_kernel(
    const float* __restrict__ mass, long long rows, int n_kb, double tau,
    int32_t* __restrict__ counts, uint32_t* __restrict__ bitmaps, int words, uint32_t* status) {
  extern __shared__ unsigned long long sel_smem[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const long long r = static_cast<long long>(blockIdx.x) * kSelWarps + warp;
  if (r >= rows) return;
  unsigned long long* qrow = sel_smem + static_cast<size_t>(warp) * (n_kb + (n_kb + 1) / 2);
  uint32_t* cand = reinterpret_cast<uint32_t*>(qrow + n_kb);  // candidate row indices
  const float* row = mass + r * n_kb;
  const unsigned lt_mask = (1u << lane) - 1u;

  // fixed-point masses into shared memory, and their sum.  Each lane issues kBatch loads
  // before using any of them, so a row costs a few memory round trips, not n_kb / 32.
  unsigned long long sum = 0;
  bool bad = false;
  for (int j0 = 0; j0 < n_kb; j0 += 32 * kBatch) {
    float m[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + 32 * u + lane;
      m[u] = j < n_kb ? __ldcs(row + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j0 + 32 * u + lane;
      if (j < n_kb) {
        unsigned long long q = 0;
        // valid: finite and 0 <= m <= 4096 (NaN fails both comparisons)
        if (m[u] >= 0.f && m[u] <= 4096.f)
          q = static_cast<unsigned long long>(
              __double2ll_rn(static_cast<double>(m[u]) * 1099511627776.0));
        else
          bad = true;
        qrow[j] = q;
        sum += q;
      }
    }
  }
  if (bad) record_status(status, FLAG_DEVICE_INPUT, DETAIL_MASS_VALUE, static_cast<uint32_t>(r), 0u);
  sum = warp_sum_u64(sum);
  const unsigned long long target =
      static_cast<unsigned long long>(ceil(__dmul_rn(tau, static_cast<double>(sum))));
  __syncwarp();

  // Invariant: every element outside the candidates is either above them (kept; its sum is
  // in A < target) or below them (dropped), and the last kept element is a candidate.  The
  // host admits 0 < tau <= 1, so target <= sum and the invariant holds from the start.
  unsigned long long A = 0, tstar = 0;
  if (target > 0) {
    int nc = n_kb;
    bool all = true;  // the candidates are still the whole row (cand not yet written)
    unsigned long long p = median3(qrow[0], qrow[n_kb >> 1], qrow[n_kb - 1]);
    while (true) {
      // sum of the candidates above p and the count of those equal to it
      unsigned long long sgt = 0;
      uint32_t ceq = 0;
      for (int j0 = 0; j0 < nc; j0 += 32 * kBatch) {
        unsigned long long qv[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + 32 * u + lane;
          qv[u] = j < nc ? qrow[all ? j : static_cast<int>(cand[j])] : 0ull;
        }
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + 32 * u + lane;
          if (j < nc) {
            if (qv[u] > p) sgt += qv[u];
            else if (qv[u] == p) ++ceq;
          }
        }
      }
      sgt = warp_sum_u64(sgt);
      const unsigned long long neq = static_cast<unsigned long long>(__reduce_add_sync(0xffffffffu, ceq));
      bool above;
      if (A + sgt >= target) {
        above = true;                  // the crossing lies above p
      } else if (A + sgt + neq * p >= target) {
        A += sgt;                      // the crossing is one of the elements equal to p
        tstar = p;
        break;
      } else {
        A += sgt + neq * p;            // everything >= p is kept
        above = false;
      }
      // compact the candidates on the kept side of p, in place: a batch is read into
      // registers before any of it is written, and writes land below the batch's end
      int kept_nc = 0;
      for (int j0 = 0; j0 < nc; j0 += 32 * kBatch) {
        uint32_t idx[kBatch];
        bool sel[kBatch];
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const int j = j0 + 32 * u + lane;
          idx[u] = j < nc ? (all ? static_cast<uint32_t>(j) : cand[j]) : 0u;
          const unsigned long long q = j < nc ? qrow[idx[u]] : 0ull;
          sel[u] = j < nc && (above ? q > p : q < p);
        }
        __syncwarp();
#pragma unroll
        for (int u = 0; u < kBatch; ++u) {
          const unsigned bal = __ballot_sync(0xffffffffu, sel[u]);
          if (sel[u]) cand[kept_nc + __popc(bal & lt_mask)] = idx[u];
          kept_nc += __popc(bal);
        }
        __syncwarp();
      }
      nc = kept_nc;
      all = false;
      if (nc == 0) {  // unreachable while the invariant holds; ends the loop regardless
        tstar = p;
        break;
      }
      p = median3(qrow[cand[0]], qrow[cand[nc >> 1]], qrow[cand[nc - 1]]);
    }
  }

  // Keep q > t*, and the c lowest-index blocks with q == t*.
  const unsigned long long c = target > 0 ? (target - A + tstar - 1) / tstar : 0ull;
  unsigned long long ties_before = 0;
  unsigned long long kept = 0;
  uint32_t* out_bits = bitmaps + r * words;
  for (int j1 = 0; j1 < n_kb; j1 += 32 * kBatch) {
    unsigned long long qv[kBatch];
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j = j1 + 32 * u + lane;
      qv[u] = j < n_kb ? qrow[j] : 0ull;
    }
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int j0 = j1 + 32 * u;
      if (j0 >= n_kb) break;  // warp-uniform
      const int j = j0 + lane;
      const unsigned long long q = qv[u];
      const bool is_tie = target > 0 && j < n_kb && q == tstar;
      const unsigned tb = __ballot_sync(0xffffffffu, is_tie);
      const unsigned long long rank = ties_before + __popc(tb & lt_mask);
      const bool keep = target > 0 && j < n_kb && (q > tstar || (is_tie && rank < c));
      const unsigned kb = __ballot_sync(0xffffffffu, keep);
      if (lane == 0) out_bits[j0 >> 5] = kb;
      ties_before += __popc(tb);
      kept += __popc(kb);
    }
  }
  if (lane == 0) counts[r] = static_cast<int32_t>(kept);
}

// Exclusive scan of counts[0..R) into row_ptr[0..R] with one 1024-thread CTA.
__global__ void __launch_bounds__(1024) topp_scan_kernel(const int32_t* __restrict__ counts,
                                                         long long rows,
                                                         int32_t* __restrict__ row_ptr) {
  __shared__ long long warp_tot[32];
  const int tid = threadIdx.x;
  const long long per = (rows + 1023) / 1024;
  const long long lo = tid * per;
  const long long hi = min(rows, lo + per);
  long long s = 0;
  for (long long i = lo; i < hi; ++i) s += counts[i];
  long long inc = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, inc, o);
    if ((tid & 31) >= o) inc += n;
  }
  if ((tid & 31) == 31) warp_tot[tid >> 5] = inc;
  __syncthreads();
  long long before = 0;
  for (int i = 0; i < (tid >> 5); ++i) before += warp_tot[i];
  long long run = before + inc - s;
  for (long long i = lo; i < hi; ++i) {
    row_ptr[i] = static_cast<int32_t>(run);
    run += counts[i];
  }
  if (tid == 1023) {
    long long total = 0;
    for (int i = 0; i < 32; ++i) total += warp_tot[i];
    row_ptr[rows] = static_cast<int32_t>(total);
  }
}

// One warp per row: compact the kept bitmap into ascending col_idx, staging 32 words
// (1024 blocks) at a time in shared memory so the global writes are contiguous.
__global__ void __launch_bounds__(256) topp_fill_kernel(const uint32_t* __restrict__ bitmaps,
                                                        int words, long long rows,
                                                        const int32_t* __restrict__ row_ptr,
                                                        int32_t* __restrict__ col_idx,
                                                        long long capacity, uint32_t* status) {
  __shared__ int32_t stage[8][1024];
  const int w = threadIdx.x >> 5;
  const int lane = lane_id();
  const long long r = static_cast<long long>(blockIdx.x) * 8 + w;
  if (r >= rows) return;
  const uint32_t* bits = bitmaps + r * words;
  long long pos = row_ptr[r];
  bool overflow = false;
  for (int w0 = 0; w0 < words; w0 += 32) {
    const uint32_t word = (w0 + lane < words) ? bits[w0 + lane] : 0u;
    const int pc = __popc(word);
    int inc = pc;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int n = __shfl_up_sync(0xffffffffu, inc, o);
      if (lane >= o) inc += n;
    }
    const int chunk = __shfl_sync(0xffffffffu, inc, 31);
    int k = inc - pc;
    uint32_t wb = word;
    while (wb) {
      const int b = __ffs(wb) - 1;
      wb &= wb - 1;
      stage[w][k++] = (w0 + lane) * 32 + b;
    }
    __syncwarp();
    for (int i = lane; i < chunk; i += 32) {
      if (pos + i < capacity) col_idx[pos + i] = stage[w][i];
      else overflow = true;
    }
    __syncwarp();
    pos += chunk;
  }
  if (overflow) record_status(status, FLAG_CAPACITY, DETAIL_COL_CAPACITY, static_cast<uint32_t>(r), 0u);
}

static cudaError_t launch_select_rows(const float* mass, long long rows, int n_kb, float threshold,
                                      int32_t* counts, uint32_t* bitmaps, int words,
                                      uint32_t* status, cudaStream_t stream) {
  const size_t smem = static_cast<size_t>(kSelWarps) * (n_kb + (n_kb + 1) / 2) * sizeof(unsigned long long);
  cudaError_t e = cudaFuncSetAttribute(topp_select_rows_kernel,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const long long ctas = (rows + kSelWarps - 1) / kSelWarps;
  topp_select_rows_kernel<<<static_cast<unsigned>(ctas), 32 * kSelWarps, smem, stream>>>(
      mass, rows, n_kb, static_cast<double>(threshold), counts, bitmaps, words, status);
  return cudaGetLastError();
}

cudaError_t launch_bitmap_to_csr(const int32_t* counts, const uint32_t* bitmaps, long long rows,
                                 int words, int32_t* row_ptr, int32_t* col_idx,
                                 long long col_capacity, uint32_t* status, cudaStream_t stream) {
  topp_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topp_fill_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      bitmaps, words, rows, row_ptr, col_idx, col_capacity, status);
  return cudaGetLastError();
}

size_t topp_scratch_bytes(long long rows, int n_kb) {
  const long long words = (n_kb + 31) / 32;
  const size_t counts = static_cast<size_t>(rows) * 4;
  const size_t counts_al = (counts + 255) & ~static_cast<size_t>(255);
  return counts_al + static_cast<size_t>(rows) * words * 4;
}

cudaError_t launch_topp_select(const float* mass, long long rows, int n_kb, float threshold,
                               int32_t* row_ptr, int32_t* col_idx, long long col_capacity,
                               void* ws, cudaStream_t stream) {
  uint8_t* base = static_cast<uint8_t*>(ws);
  uint32_t* status = reinterpret_cast<uint32_t*>(base);
  const int words = (n_kb + 31) / 32;
  const size_t counts_bytes = (static_cast<size_t>(rows) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* counts = reinterpret_cast<int32_t*>(base + kStatusBytes);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(base + kStatusBytes + counts_bytes);
  if (rows == 0) {
    return cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), stream);
  }
  cudaError_t e = launch_select_rows(mass, rows, n_kb, threshold, counts, bitmaps, words, status,
                                     stream);
  if (e != cudaSuccess) return e;
  topp_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topp_fill_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      bitmaps, words, rows, row_ptr, col_idx, col_capacity, status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------------------
// Allocation-free variant of the selection.
//
// Some callers cannot hand the library a workspace: a plugin inside a serving engine whose
// memory planner reserves all device memory up front and forbids ad-hoc cudaMalloc, code
// on a latency-critical path where cudaMalloc's implicit synchronisation would stall the
// stream, or a runtime that owns every device allocation through its own pool.  For them
// the selection's scratch (per-row counts and kept bitmaps) lives in a fixed array in the
// library's own device memory, sized for the largest shapes this library targets.
namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;  // 16 MiB per device

// Every GPU that loads the library holds this array until the process exits.  In host
// code its name is only a host-side stand-in; the device address comes from
// cudaGetSymbolAddress below.
static __device__ __align__(256) uint8_t g_topp_noalloc_scratch[kNoAllocScratchBytes];

// The array's device address belongs to the CUDA context the module was loaded into: another
// context on the same device (a driver-API context of the caller's own) sees the array at
// another address, and a device reset unloads the module, so an address found before the
// reset may no longer belong to the library.  The address is therefore cached per context,
// keyed by the context's unique ID (cuCtxGetId: never reused within a process, unlike the
// context handle), so the first call in every context -- a new one after a device reset
// included -- looks it up with that context current.
using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_fn(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) == cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    return reinterpret_cast<Fn>(p);
  return nullptr;
}

constexpr int kMaxContexts = 64;
std::mutex g_noalloc_mu;
unsigned long long g_noalloc_ctx_id[kMaxContexts] = {0};
void* g_noalloc_addr[kMaxContexts] = {nullptr};
int g_noalloc_n = 0;     // entries in use
int g_noalloc_next = 0;  // entry replaced next once all are in use

// Device address of the scratch array in the current context.
cudaError_t noalloc_scratch_address(void** out) {
  static CtxGetCurrentFn get_ctx = nullptr;
  static CtxGetIdFn get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    get_ctx = driver_fn<CtxGetCurrentFn>("cuCtxGetCurrent");
    get_id = driver_fn<CtxGetIdFn>("cuCtxGetId");
  });
  if (get_ctx == nullptr || get_id == nullptr) return cudaErrorInitializationError;
  CUcontext ctx = nullptr;
  if (get_ctx(&ctx) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  if (ctx == nullptr) {
    // No context current on this thread yet: the runtime's lookup makes the current
    // device's primary context current.
    void* p = nullptr;
    const cudaError_t e0 = cudaGetSymbolAddress(&p, g_topp_noalloc_scratch);
    if (e0 != cudaSuccess) return e0;
    if (get_ctx(&ctx) != CUDA_SUCCESS || ctx == nullptr) return cudaErrorDeviceUninitialized;
  }
  unsigned long long id = 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return cudaErrorDeviceUninitialized;
  cudaError_t e = cudaSuccess;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  for (int i = 0; i < g_noalloc_n; ++i)
    if (g_noalloc_ctx_id[i] == id) {
      *out = g_noalloc_addr[i];
      return cudaSuccess;
    }
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_topp_noalloc_scratch);
  if (e != cudaSuccess) return e;
  int slot = g_noalloc_n < kMaxContexts ? g_noalloc_n++ : g_noalloc_next++ % kMaxContexts;
  g_noalloc_ctx_id[slot] = id;
  g_noalloc_addr[slot] = p;
  *out = p;
  return cudaSuccess;
}

}  // namespace

size_t topp_noalloc_capacity_bytes() { return kNoAllocScratchBytes; }

cudaError_t launch_topp_select_noalloc(const float* mass, long long rows, int n_kb, float threshold,
                                       int32_t* row_ptr, int32_t* col_idx, long long col_capacity,
                                       uint32_t* status, cudaStream_t stream) {
  void* scratch = nullptr;
  cudaError_t e = noalloc_scratch_address(&scratch);
  if (e != cudaSuccess) return e;
  if (rows == 0) return cudaMemsetAsync(row_ptr, 0, sizeof(int32_t), stream);
  // Same layout as the workspace scratch: counts int32 [rows] (256-byte aligned), then
  // bitmaps uint32 [rows][words].  Both are fully rewritten by every call.
  const int words = (n_kb + 31) / 32;
  const size_t counts_bytes = (static_cast<size_t>(rows) * 4 + 255) & ~static_cast<size_t>(255);
  int32_t* counts = static_cast<int32_t*>(scratch);
  uint32_t* bitmaps = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(scratch) + counts_bytes);
  e = launch_select_rows(mass, rows, n_kb, threshold, counts, bitmaps, words, status, stream);
  if (e != cudaSuccess) return e;
  topp_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topp_fill_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      bitmaps, words, rows, row_ptr, col_idx, col_capacity, status);
  return cudaGetLastError();
}

}  // namespace bsa
