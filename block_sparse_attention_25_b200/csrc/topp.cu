// Retained-mass (top-p) block selection into CSR lists.
//
// "LoSA: Near-Lossless Sparse Attention for Training-Free Video Diffusion Acceleration",
// Abstract: for each head and query block keep the smallest key/value block set whose
// attention mass meets the threshold.  "Sparse VideoGen2", Abstract: top-p dynamic
// budget control is the same per-row operator.
//
// Per row the masses become integers q = rint(m * 2^40) and the target is
// ceil(tau * sum q) (one fp64 multiply).  The shortest prefix of the (q desc, index asc)
// order that reaches the target is found without sorting: an exact MSB-first radix
// select on q (8-bit digits, per-digit sums in shared memory) finds the value t* of the
// last kept element and the sum A of everything above it; all blocks with q > t* are
// kept, plus the ceil((target - A) / t*) lowest-index blocks with q == t*.  Integer
// arithmetic makes the result independent of reduction order, so it is bit-identical to
// a sequential sort-and-scan.
//
// Kernels: (1) select, one 256-thread CTA per row -> kept bitmap + count in the
// workspace; (2) exclusive scan of the counts -> row_ptr; (3) compaction, one warp per
// row -> col_idx ascending.
#include <mutex>

#include "bsa_kernels.cuh"

namespace bsa {

constexpr int kToppThreads = 256;
constexpr int kToppMaxKb = 4096;
constexpr int kToppMaxE = kToppMaxKb / kToppThreads;  // elements per thread

__device__ __forceinline__ unsigned long long warp_incl_scan_u64(unsigned long long v) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long n = __shfl_up_sync(0xffffffffu, v, o);
    if (static_cast<int>(lane_id()) >= o) v += n;
  }
  return v;
}

// Block-wide inclusive scan of one uint64 per thread (256 threads).  Returns the
// inclusive value; *total receives the block total.
__device__ __forceinline__ unsigned long long block_incl_scan_u64(unsigned long long v,
                                                                  unsigned long long* sm8,
                                                                  unsigned long long* total) {
  const int w = threadIdx.x >> 5;
  unsigned long long inc = warp_incl_scan_u64(v);
  if (lane_id() == 31) sm8[w] = inc;
  __syncthreads();
  unsigned long long before = 0, tot = 0;
#pragma unroll
  for (int i = 0; i < kToppThreads / 32; ++i) {
    const unsigned long long s = sm8[i];
    if (i < w) before += s;
    tot += s;
  }
  __syncthreads();
  *total = tot;
  return inc + before;
}

__device__ __forceinline__ unsigned long long block_max_u64(unsigned long long v,
                                                            unsigned long long* sm8) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long n = __shfl_xor_sync(0xffffffffu, v, o);
    v = n > v ? n : v;
  }
  if (lane_id() == 0) sm8[threadIdx.x >> 5] = v;
  __syncthreads();
  unsigned long long m = 0;
#pragma unroll
  for (int i = 0; i < kToppThreads / 32; ++i) m = sm8[i] > m ? sm8[i] : m;
  __syncthreads();
  return m;
}

__global__ void __launch_bounds__(kToppThreads) topp_select_rows_kernel(
    const float* __restrict__ mass, int n_kb, double tau, int32_t* __restrict__ counts,
    uint32_t* __restrict__ bitmaps, int words, uint32_t* status) {
  __shared__ float sm_m[kToppMaxKb];
  __shared__ unsigned long long h_sum[256];
  __shared__ unsigned long long sm8[kToppThreads / 32];
  __shared__ uint32_t sm_bits[kToppMaxKb / 32];
  __shared__ int sh_first;

  const long long r = blockIdx.x;
  const int tid = threadIdx.x;
  const float* row = mass + r * n_kb;
  for (int j = tid; j < n_kb; j += kToppThreads) sm_m[j] = row[j];
  for (int j = tid; j < words; j += kToppThreads) sm_bits[j] = 0u;
  __syncthreads();

  // Contiguous ownership: thread tid holds blocks [tid*E, tid*E + n_mine).
  const int E = (n_kb + kToppThreads - 1) / kToppThreads;
  const int first = tid * E;
  const int n_mine = max(0, min(E, n_kb - first));
  unsigned long long q[kToppMaxE];
  unsigned long long my_sum = 0, my_max = 0;
  bool bad = false;
#pragma unroll
  for (int e = 0; e < kToppMaxE; ++e) {
    q[e] = 0ull;
    if (e < n_mine) {
      const float m = sm_m[first + e];
      // valid: finite and 0 <= m <= 4096 (NaN fails both comparisons)
      if (m >= 0.f && m <= 4096.f) {
        q[e] = static_cast<unsigned long long>(__double2ll_rn(static_cast<double>(m) * 1099511627776.0));
      } else {
        bad = true;
      }
      my_sum += q[e];
      my_max = q[e] > my_max ? q[e] : my_max;
    }
  }
  if (bad) record_status(status, FLAG_DEVICE_INPUT, DETAIL_MASS_VALUE, static_cast<uint32_t>(r), 0u);

  unsigned long long S;
  (void)block_incl_scan_u64(my_sum, sm8, &S);
  const unsigned long long Mx = block_max_u64(my_max, sm8);
  const unsigned long long target =
      static_cast<unsigned long long>(ceil(__dmul_rn(tau, static_cast<double>(S))));

  unsigned long long tstar = 0, A = 0;
  if (target > 0) {
    const int nbits = 64 - __clzll(static_cast<long long>(Mx));
    int shift = ((nbits + 7) / 8 - 1) * 8;
    if (shift < 0) shift = 0;
    unsigned long long prefix = 0;
    for (; shift >= 0; shift -= 8) {
      h_sum[tid] = 0ull;
      __syncthreads();
      const unsigned long long hi = prefix >> (shift + 8);
#pragma unroll
      for (int e = 0; e < kToppMaxE; ++e) {
        if (e < n_mine && (q[e] >> (shift + 8)) == hi) {
          atomicAdd(&h_sum[(q[e] >> shift) & 255ull], q[e]);
        }
      }
      __syncthreads();
      // Thread tid looks at digit 255 - tid (descending); inclusive scan from the top.
      const unsigned long long v = h_sum[255 - tid];
      unsigned long long tot;
      const unsigned long long inc = block_incl_scan_u64(v, sm8, &tot);
      if (tid == 0) sh_first = kToppThreads;
      __syncthreads();
      if (A + inc >= target) atomicMin(&sh_first, tid);
      __syncthreads();
      const int f = sh_first;
      // Broadcast the sum strictly above the crossing digit from thread f.
      if (tid == f) {
        h_sum[0] = A + inc - v;  // reuse slot 0 (the histogram is read already)
        sm8[0] = static_cast<unsigned long long>(255 - f);
      }
      __syncthreads();
      A = h_sum[0];
      prefix |= sm8[0] << shift;
      __syncthreads();
    }
    tstar = prefix;
  }

  // Keep q > t*, and the lowest-index c elements with q == t*.
  unsigned long long c = 0;
  if (target > 0) c = (target - A + tstar - 1) / tstar;
  int my_eq = 0, my_gt = 0;
#pragma unroll
  for (int e = 0; e < kToppMaxE; ++e) {
    if (e < n_mine && target > 0) {
      my_gt += q[e] > tstar;
      my_eq += q[e] == tstar;
    }
  }
  unsigned long long tot_eq;
  const unsigned long long eq_incl = block_incl_scan_u64(static_cast<unsigned long long>(my_eq), sm8, &tot_eq);
  unsigned long long tot_gt;
  (void)block_incl_scan_u64(static_cast<unsigned long long>(my_gt), sm8, &tot_gt);
  unsigned long long rank = eq_incl - my_eq;
  if (target > 0) {
#pragma unroll
    for (int e = 0; e < kToppMaxE; ++e) {
      if (e < n_mine) {
        bool keep = q[e] > tstar;
        if (q[e] == tstar) {
          keep = rank < c;
          ++rank;
        }
        if (keep) atomicOr(&sm_bits[(first + e) >> 5], 1u << ((first + e) & 31));
      }
    }
  }
  __syncthreads();
  uint32_t* out_bits = bitmaps + r * words;
  for (int j = tid; j < words; j += kToppThreads) out_bits[j] = sm_bits[j];
  if (tid == 0) counts[r] = static_cast<int32_t>(target > 0 ? tot_gt + c : 0ull);
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
  topp_select_rows_kernel<<<static_cast<unsigned>(rows), kToppThreads, 0, stream>>>(
      mass, n_kb, static_cast<double>(threshold), counts, bitmaps, words, status);
  cudaError_t e = cudaGetLastError();
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

constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_addr[kMaxDevices] = {nullptr};

// Device address of the scratch array for the current device, looked up once per device
// (with that device current) and cached.
cudaError_t noalloc_scratch_address(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (g_noalloc_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topp_noalloc_scratch);
    if (e != cudaSuccess) return e;
    g_noalloc_addr[dev] = p;
  }
  *out = g_noalloc_addr[dev];
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
  topp_select_rows_kernel<<<static_cast<unsigned>(rows), kToppThreads, 0, stream>>>(
      mass, n_kb, static_cast<double>(threshold), counts, bitmaps, words, status);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topp_scan_kernel<<<1, 1024, 0, stream>>>(counts, rows, row_ptr);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  topp_fill_kernel<<<static_cast<unsigned>((rows + 7) / 8), 256, 0, stream>>>(
      bitmaps, words, rows, row_ptr, col_idx, col_capacity, status);
  return cudaGetLastError();
}

}  // namespace bsa
