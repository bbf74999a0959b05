// C ABI of libbsattn.so: argument checks, workspace layout, tensor-map encoding and
// kernel launches.  See include/bsattn.h for the contract of every entry point.
#include <cstring>
#include <mutex>

#include "../../include/bsattn.h"
#include "bsa_kernels.cuh"

namespace bsa {

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

cudaError_t encode_tmap_3d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                           int elem_bytes, int D, int Np, int bh, int box_d, int box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorInitializationError;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(Np),
                              static_cast<cuuint64_t>(bh)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(D) * elem_bytes,
                                 static_cast<cuuint64_t>(Np) * D * elem_bytes};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box_d), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_tmap_3d_strided(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                                   const unsigned long long dims[3],
                                   const unsigned long long strides_bytes[2],
                                   const unsigned box[3]) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorInitializationError;
  const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
  const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
  const cuuint32_t bx[3] = {box[0], box[1], box[2]};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  const CUresult r = fn(map, dtype, 3, const_cast<void*>(base), d, st, bx, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Raster tokens [S = T*H*W][Hh][D] of one batch as a 5D map (D, Hh, W, H, T) with a
// (64, 1, 4, 4, 4) box: one box is one 4x4x4 tile of one head, 64 rows of 64 elements in
// (t, h, w) row-major order, coordinates past (W, H, T) read as zeros.
cudaError_t encode_tmap_raster_tiles(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                                     int elem_bytes, int D, int heads, int W, int H, int T) {
  EncodeTiledFn fn = encode_fn();
  if (fn == nullptr) return cudaErrorInitializationError;
  const cuuint64_t row = static_cast<cuuint64_t>(D) * elem_bytes;
  const cuuint64_t dims[5] = {static_cast<cuuint64_t>(D), static_cast<cuuint64_t>(heads),
                              static_cast<cuuint64_t>(W), static_cast<cuuint64_t>(H),
                              static_cast<cuuint64_t>(T)};
  const cuuint64_t strides[4] = {row, row * heads, row * heads * W, row * heads * W * H};
  const cuuint32_t box[5] = {static_cast<cuuint32_t>(128 / elem_bytes), 1u, 4u, 4u, 4u};
  const cuuint32_t estr[5] = {1u, 1u, 1u, 1u, 1u};
  const CUresult r = fn(map, dtype, 5, const_cast<void*>(base), dims, strides, box, estr,
                        CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                        CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace bsa

using bsa::AttnDims;
using bsa::GridDims;
using bsa::ClusterDims;

namespace {

// Host-side shape checks shared by every entry point.
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

bsa_status check_shape(const bsa_shape* s, bool attention) {
  if (s == nullptr) return BSA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->heads < 1 || s->head_dim < 1) return BSA_ERR_INVALID_ARG;
  if (s->T < 1 || s->H < 1 || s->W < 1) return BSA_ERR_INVALID_ARG;
  if (s->Tp < s->T || s->Hp < s->H || s->Wp < s->W) return BSA_ERR_INVALID_ARG;
  if ((s->Tp & 3) || (s->Hp & 3) || (s->Wp & 3)) return BSA_ERR_INVALID_ARG;
  const long long np = 1LL * s->Tp * s->Hp * s->Wp;
  if (np >= (1LL << 30)) return BSA_ERR_UNSUPPORTED;
  if (s->head_dim != 64 && s->head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (attention) {
    if (s->kv_block != 64) return BSA_ERR_UNSUPPORTED;
    if (s->q_block != 64 && s->q_block != 128) return BSA_ERR_UNSUPPORTED;
    if (np % s->q_block) return BSA_ERR_INVALID_ARG;
    const long long rows = 1LL * s->batch * s->heads * (np / s->q_block);
    if (rows >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
    if (np / 64 > 4096) return BSA_ERR_UNSUPPORTED;  // selection and schedule bitmaps
    // CSR offsets are int32
    if (rows * (np / 64) >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  }
  return BSA_OK;
}

}  // namespace

namespace bsa {
bsa_status check_attention_shape(const bsa_shape* s) { return check_shape(s, true); }
}  // namespace bsa

namespace {

GridDims make_grid(const bsa_shape* s) {
  GridDims g;
  g.T = s->T;
  g.H = s->H;
  g.W = s->W;
  g.Tp = s->Tp;
  g.Hp = s->Hp;
  g.Wp = s->Wp;
  g.nth = s->Hp / 4;
  g.ntw = s->Wp / 4;
  g.S = s->T * s->H * s->W;
  g.Np = s->Tp * s->Hp * s->Wp;
  g.div_ntw = bsa::make_fastdiv(g.ntw);
  g.div_nth = bsa::make_fastdiv(g.nth);
  g.div_W = bsa::make_fastdiv(g.W);
  g.div_H = bsa::make_fastdiv(g.H);
  return g;
}

AttnDims make_attn(const bsa_shape* s) {
  AttnDims a;
  a.g = make_grid(s);
  a.batch = s->batch;
  a.heads = s->heads;
  a.head_dim = s->head_dim;
  a.q_block = s->q_block;
  a.n_qb = a.g.Np / s->q_block;
  a.n_kb = a.g.Np / 64;
  a.n_cta_per_head = (a.g.Np + 255) / 256;
  return a;
}

bsa_status from_cuda(cudaError_t e) { return e == cudaSuccess ? BSA_OK : BSA_ERR_CUDA; }

size_t workspace_bytes(const bsa_shape* s, int op) {
  if (check_shape(s, true) != BSA_OK) return 0;
  const AttnDims a = make_attn(s);
  switch (op) {
    case BSA_OP_BLOCK_MASS:
      return bsa::kStatusBytes + bsa::mass_scratch_bytes(a);
    case BSA_OP_TOPP_SELECT:
      return bsa::kStatusBytes +
             bsa::topp_scratch_bytes(1LL * a.batch * a.heads * a.n_qb, a.n_kb);
    case BSA_OP_FWD:
      return bsa::kStatusBytes + bsa::fwd_scratch_bytes(a);
    case BSA_OP_POOLED_MASS:
      return bsa::kStatusBytes + bsa::pooled_scratch_bytes(a);
    case BSA_OP_PATTERN:
      return bsa::kStatusBytes +
             bsa::topp_scratch_bytes(1LL * a.batch * a.heads * a.n_qb, a.n_kb);
    default:
      return 0;
  }
}

}  // namespace

extern "C" {

const char* bsa_version(void) { return "bsattn 0.1 sm_100a"; }

bsa_status bsa_kernel_binary_version(int32_t* version) {
  if (version == nullptr) return BSA_ERR_INVALID_ARG;
  int v = 0;
  const cudaError_t e = bsa::kernel_binary_version(&v);
  if (e != cudaSuccess) return from_cuda(e);
  *version = v;
  return BSA_OK;
}

const char* bsa_status_string(bsa_status st) {
  switch (st) {
    case BSA_OK: return "ok";
    case BSA_ERR_INVALID_ARG: return "invalid argument";
    case BSA_ERR_UNSUPPORTED: return "unsupported shape";
    case BSA_ERR_CAPACITY: return "capacity too small";
    case BSA_ERR_CUDA: return "CUDA error";
    case BSA_ERR_TIMEOUT: return "device wait timed out";
    case BSA_ERR_DEVICE_INPUT: return "device-side input check failed";
    case BSA_ERR_IO: return "list file missing, unreadable or corrupt";
  }
  return "unknown status";
}

size_t bsa_workspace_bytes(const bsa_shape* shape, int op) { return workspace_bytes(shape, op); }

bsa_status bsa_clear_status(void* ws, bsa_stream_t stream) {
  if (ws == nullptr) return BSA_ERR_INVALID_ARG;
  return from_cuda(cudaMemsetAsync(ws, 0, bsa::kStatusBytes, stream));
}

bsa_status bsa_device_status_words(const void* ws, uint32_t out_words[4], bsa_stream_t stream) {
  if (ws == nullptr || out_words == nullptr) return BSA_ERR_INVALID_ARG;
  cudaError_t e = cudaMemcpyAsync(out_words, ws, 4 * sizeof(uint32_t), cudaMemcpyDeviceToHost, stream);
  if (e == cudaSuccess) e = cudaStreamSynchronize(stream);
  return from_cuda(e);
}

bsa_status bsa_device_status(const void* ws, bsa_stream_t stream) {
  uint32_t w[4] = {0, 0, 0, 0};
  const bsa_status st = bsa_device_status_words(ws, w, stream);
  if (st != BSA_OK) return st;
  if (w[0] & bsa::FLAG_TIMEOUT) return BSA_ERR_TIMEOUT;
  if (w[0] & bsa::FLAG_DEVICE_INPUT) return BSA_ERR_DEVICE_INPUT;
  if (w[0] & bsa::FLAG_CAPACITY) return BSA_ERR_CAPACITY;
  return BSA_OK;
}

bsa_status bsa_tile_permute(const bsa_shape* shape, bsa_dtype dtype, int inverse, const void* src,
                            void* dst, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, false);
  if (st != BSA_OK) return st;
  if (src == nullptr || dst == nullptr || !bsa::aligned16(src) || !bsa::aligned16(dst))
    return BSA_ERR_INVALID_ARG;
  if (dtype != BSA_BF16 && dtype != BSA_FP32) return BSA_ERR_UNSUPPORTED;
  if (inverse != 0 && inverse != 1) return BSA_ERR_INVALID_ARG;
  const GridDims g = make_grid(shape);
  const int row_bytes = shape->head_dim * (dtype == BSA_BF16 ? 2 : 4);
  return from_cuda(bsa::launch_tile_permute(g, shape->batch, shape->heads, row_bytes, inverse, src,
                                            dst, stream));
}

bsa_status bsa_tile_permute_quant_e4m3(const bsa_shape* shape, const void* src_bf16, uint8_t* dst,
                                       float* tile_scales, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, false);
  if (st != BSA_OK) return st;
  if (src_bf16 == nullptr || dst == nullptr || tile_scales == nullptr ||
      !bsa::aligned16(src_bf16) || !bsa::aligned16(dst) ||
      (reinterpret_cast<uintptr_t>(tile_scales) & 3u))
    return BSA_ERR_INVALID_ARG;
  const long long ntiles = 1LL * shape->batch * shape->heads * (1LL * shape->Tp * shape->Hp * shape->Wp / 64);
  if (ntiles >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  const GridDims g = make_grid(shape);
  return from_cuda(bsa::launch_tile_permute_quant_e4m3(g, shape->batch, shape->heads,
                                                       shape->head_dim, src_bf16, dst,
                                                       tile_scales, stream));
}

bsa_status bsa_block_mass(const bsa_shape* shape, const void* q, const void* k, float softmax_scale,
                          float* mass, void* ws, size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || mass == nullptr || ws == nullptr || !bsa::aligned16(q) ||
      !bsa::aligned16(k) || !bsa::aligned16(ws) || (reinterpret_cast<uintptr_t>(mass) & 3u))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_BLOCK_MASS)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  return from_cuda(bsa::launch_block_mass(a, q, k, softmax_scale, mass, ws, stream));
}

bsa_status bsa_dense_fwd_mass(const bsa_shape* shape, const void* q, const void* k, const void* v,
                              float softmax_scale, void* out, float* lse, float* mass, void* ws,
                              size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || mass == nullptr ||
      ws == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(v) || !bsa::aligned16(out) ||
      !bsa::aligned16(ws) || (reinterpret_cast<uintptr_t>(mass) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_BLOCK_MASS)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  return from_cuda(
      bsa::launch_calib_dense_mass(a, q, k, v, softmax_scale, out, lse, mass, ws, stream));
}

bsa_status bsa_pooled_mass(const bsa_shape* shape, const void* q, const void* k,
                           float softmax_scale, float* mass_est, void* ws, size_t ws_bytes,
                           bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || mass_est == nullptr || ws == nullptr ||
      !bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(mass_est) & 3u))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale >= 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_POOLED_MASS)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  return from_cuda(bsa::launch_pooled_mass(a, q, k, softmax_scale, mass_est, ws, stream));
}

bsa_status bsa_topp_select(const bsa_shape* shape, const float* mass, float threshold,
                           int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, void* ws,
                           size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (mass == nullptr || row_ptr == nullptr || ws == nullptr || !bsa::aligned16(ws) ||
      (reinterpret_cast<uintptr_t>(mass) & 3u) || !aligned4(row_ptr) || !aligned4(col_idx))
    return BSA_ERR_INVALID_ARG;
  if (col_capacity < 0 || (col_capacity > 0 && col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  if (!(threshold > 0.f && threshold <= 1.f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_TOPP_SELECT)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  const long long rows = 1LL * a.batch * a.heads * a.n_qb;
  return from_cuda(bsa::launch_topp_select(mass, rows, a.n_kb, threshold, row_ptr, col_idx,
                                           col_capacity, ws, stream));
}

bsa_status bsa_pattern_csr(const bsa_shape* shape, const bsa_pattern* pattern, int32_t* row_ptr,
                           int32_t* col_idx, int64_t col_capacity, void* ws, size_t ws_bytes,
                           bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (pattern == nullptr || row_ptr == nullptr || ws == nullptr || !bsa::aligned16(ws) ||
      !aligned4(row_ptr) || !aligned4(col_idx))
    return BSA_ERR_INVALID_ARG;
  if (col_capacity < 0 || (col_capacity > 0 && col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  const uint32_t all = BSA_PAT_DIAGONAL | BSA_PAT_MULTI_DIAGONAL | BSA_PAT_VERTICAL_STRIPE |
                       BSA_PAT_SURROUNDING | BSA_PAT_CRISS_CROSS;
  if (pattern->kinds & ~all) return BSA_ERR_INVALID_ARG;
  if (pattern->diag_width < 0 || pattern->multi_count < 0 || pattern->stripe_stride < 0 ||
      pattern->radius_t < 0 || pattern->radius_h < 0 || pattern->radius_w < 0)
    return BSA_ERR_INVALID_ARG;
  if (pattern->stripe_stride > 0 &&
      (pattern->stripe_offset < 0 || pattern->stripe_offset >= pattern->stripe_stride))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_PATTERN)) return BSA_ERR_CAPACITY;
  bsa::PatternParams pp;
  pp.kinds = pattern->kinds;
  pp.diag_width = pattern->diag_width;
  pp.multi_count = pattern->multi_count;
  pp.multi_period = pattern->multi_period;
  pp.stripe_stride = pattern->stripe_stride;
  pp.stripe_offset = pattern->stripe_offset;
  pp.radius_t = pattern->radius_t;
  pp.radius_h = pattern->radius_h;
  pp.radius_w = pattern->radius_w;
  const AttnDims a = make_attn(shape);
  return from_cuda(bsa::launch_pattern_csr(a, pp, row_ptr, col_idx, col_capacity, ws, stream));
}

bsa_status bsa_topp_select_noalloc(const bsa_shape* shape, const float* mass, float threshold,
                                   int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity,
                                   uint32_t* status, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (mass == nullptr || row_ptr == nullptr || (reinterpret_cast<uintptr_t>(mass) & 3u) ||
      !aligned4(row_ptr) || !aligned4(col_idx) || (status != nullptr && (reinterpret_cast<uintptr_t>(status) & 3u)))
    return BSA_ERR_INVALID_ARG;
  if (col_capacity < 0 || (col_capacity > 0 && col_idx == nullptr)) return BSA_ERR_INVALID_ARG;
  if (!(threshold > 0.f && threshold <= 1.f)) return BSA_ERR_INVALID_ARG;
  const AttnDims a = make_attn(shape);
  const long long rows = 1LL * a.batch * a.heads * a.n_qb;
  // The scratch is the library's fixed per-device array: larger problems are refused.
  if (bsa::topp_scratch_bytes(rows, a.n_kb) > bsa::topp_noalloc_capacity_bytes())
    return BSA_ERR_CAPACITY;
  return from_cuda(bsa::launch_topp_select_noalloc(mass, rows, a.n_kb, threshold, row_ptr, col_idx,
                                                   col_capacity, status, stream));
}

bsa_status bsa_fwd(const bsa_shape* shape, bsa_dtype dtype, const void* q, const void* k,
                   const void* v, const float* q_scales, const float* k_scales,
                   const float* v_scales, const int32_t* row_ptr, const int32_t* col_idx,
                   float softmax_scale, void* out, float* lse, void* ws, size_t ws_bytes,
                   bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || row_ptr == nullptr || col_idx == nullptr ||
      out == nullptr || ws == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(v) || !bsa::aligned16(out) ||
      !bsa::aligned16(ws) || (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)) ||
      !aligned4(row_ptr) || !aligned4(col_idx))
    return BSA_ERR_INVALID_ARG;
  if (dtype == BSA_E4M3) {
    if (q_scales == nullptr || k_scales == nullptr || v_scales == nullptr) return BSA_ERR_INVALID_ARG;
    if ((reinterpret_cast<uintptr_t>(q_scales) | reinterpret_cast<uintptr_t>(k_scales) |
         reinterpret_cast<uintptr_t>(v_scales)) & 3u)
      return BSA_ERR_INVALID_ARG;
    if (shape->head_dim != 128) return BSA_ERR_UNSUPPORTED;
  } else if (dtype != BSA_BF16) {
    return BSA_ERR_UNSUPPORTED;
  }
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_FWD)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  const cudaError_t e =
      bsa::launch_bsattn_fwd(a, dtype == BSA_E4M3 ? 1 : 0, q, k, v, q_scales, k_scales, v_scales,
                             row_ptr, col_idx, softmax_scale, out, lse, ws, stream);
  if (e == cudaErrorNotSupported) return BSA_ERR_UNSUPPORTED;
  return from_cuda(e);
}

}  // extern "C"

// ---------------------------------------------------------------- semantic clusters
namespace {

bsa_status check_cluster_shape(const bsa_cluster_shape* s) {
  if (s == nullptr) return BSA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->heads < 1 || s->n_tokens < 1 || s->n_q_clusters < 1 ||
      s->n_k_clusters < 1)
    return BSA_ERR_INVALID_ARG;
  if (s->head_dim != 64 && s->head_dim != 128) return BSA_ERR_UNSUPPORTED;
  if (s->n_tokens > (1 << 24) || s->n_q_clusters > 1024 || s->n_k_clusters > 1024)
    return BSA_ERR_UNSUPPORTED;
  const long long bh = 1LL * s->batch * s->heads;
  // every per-head array and every flat row index fits in 31 bits
  if (bh * s->n_tokens * (s->head_dim / 8) >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if (bh * s->n_q_clusters * s->n_k_clusters >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  return BSA_OK;
}

ClusterDims cluster_dims(const bsa_cluster_shape* s, int C) {
  ClusterDims cd;
  cd.batch = s->batch;
  cd.heads = s->heads;
  cd.head_dim = s->head_dim;
  cd.S = s->n_tokens;
  cd.C = C;
  return cd;
}

}  // namespace

extern "C" {

size_t bsa_kmeans_workspace_bytes(const bsa_cluster_shape* shape, int32_t n_clusters) {
  if (check_cluster_shape(shape) != BSA_OK || n_clusters < 1 || n_clusters > 1024) return 0;
  return bsa::kStatusBytes + bsa::cluster_scratch_bytes(cluster_dims(shape, n_clusters));
}

size_t bsa_cluster_fwd_workspace_bytes(const bsa_cluster_shape* shape) {
  if (check_cluster_shape(shape) != BSA_OK) return 0;
  return bsa::kStatusBytes + bsa::cluster_fwd_scratch_bytes(shape->batch * shape->heads,
                                                            shape->n_tokens, shape->n_q_clusters,
                                                            shape->n_k_clusters);
}

size_t bsa_topp_rows_workspace_bytes(int64_t rows, int32_t cols) {
  if (rows < 0 || cols < 1 || cols > 4096 || rows * cols >= (1LL << 31)) return 0;
  return bsa::kStatusBytes + bsa::topp_scratch_bytes(rows, cols);
}

bsa_status bsa_kmeans(const bsa_cluster_shape* shape, int32_t n_clusters, const void* x,
                      int32_t rounds, float* centroids, int32_t* labels, int32_t* counts, void* ws,
                      size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_cluster_shape(shape);
  if (st != BSA_OK) return st;
  if (n_clusters < 1 || n_clusters > 1024) return BSA_ERR_UNSUPPORTED;
  if (rounds < 1 || rounds > 10000) return BSA_ERR_INVALID_ARG;
  if (x == nullptr || centroids == nullptr || labels == nullptr || counts == nullptr ||
      ws == nullptr || !bsa::aligned16(x) || !aligned4(centroids) || !aligned4(labels) ||
      !aligned4(counts) || !bsa::aligned16(ws))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa_kmeans_workspace_bytes(shape, n_clusters)) return BSA_ERR_CAPACITY;
  return from_cuda(bsa::launch_kmeans(cluster_dims(shape, n_clusters), x, rounds, centroids,
                                      labels, counts, ws, stream));
}

bsa_status bsa_cluster_layout(const bsa_cluster_shape* shape, int32_t n_clusters,
                              const int32_t* labels, int32_t* counts, int32_t* starts,
                              int32_t* token_of_slot, int32_t* slot_of_token, void* ws,
                              size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_cluster_shape(shape);
  if (st != BSA_OK) return st;
  if (n_clusters < 1 || n_clusters > 1024) return BSA_ERR_UNSUPPORTED;
  if (labels == nullptr || counts == nullptr || starts == nullptr || token_of_slot == nullptr ||
      slot_of_token == nullptr || ws == nullptr || !aligned4(labels) || !aligned4(counts) ||
      !aligned4(starts) || !aligned4(token_of_slot) || !aligned4(slot_of_token) ||
      !bsa::aligned16(ws))
    return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa_kmeans_workspace_bytes(shape, n_clusters)) return BSA_ERR_CAPACITY;
  return from_cuda(bsa::launch_cluster_layout(cluster_dims(shape, n_clusters), labels, counts,
                                              starts, token_of_slot, slot_of_token, ws, stream));
}

bsa_status bsa_cluster_permute(const bsa_cluster_shape* shape, int inverse,
                               const int32_t* token_of_slot, const void* src, void* dst,
                               bsa_stream_t stream) {
  bsa_status st = check_cluster_shape(shape);
  if (st != BSA_OK) return st;
  if (inverse != 0 && inverse != 1) return BSA_ERR_INVALID_ARG;
  if (token_of_slot == nullptr || src == nullptr || dst == nullptr || !aligned4(token_of_slot) ||
      !bsa::aligned16(src) || !bsa::aligned16(dst) || src == dst)
    return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_cluster_permute(cluster_dims(shape, 1), inverse, token_of_slot, src,
                                               dst, stream));
}

bsa_status bsa_cluster_mass(const bsa_cluster_shape* shape, const float* q_centroids,
                            const int32_t* q_counts, const float* k_centroids,
                            const int32_t* k_counts, float softmax_scale, float* mass,
                            bsa_stream_t stream) {
  bsa_status st = check_cluster_shape(shape);
  if (st != BSA_OK) return st;
  if (q_centroids == nullptr || q_counts == nullptr || k_centroids == nullptr ||
      k_counts == nullptr || mass == nullptr || !aligned4(q_centroids) || !aligned4(q_counts) ||
      !aligned4(k_centroids) || !aligned4(k_counts) || !aligned4(mass))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_cluster_mass(shape->batch, shape->heads, shape->head_dim,
                                            shape->n_q_clusters, shape->n_k_clusters, q_centroids,
                                            q_counts, k_centroids, k_counts, softmax_scale, mass,
                                            stream));
}

bsa_status bsa_topp_select_rows(const float* mass, int64_t rows, int32_t cols, float threshold,
                                int32_t* row_ptr, int32_t* col_idx, int64_t col_capacity, void* ws,
                                size_t ws_bytes, bsa_stream_t stream) {
  if (rows < 0 || cols < 1) return BSA_ERR_INVALID_ARG;
  if (cols > 4096 || rows * cols >= (1LL << 31)) return BSA_ERR_UNSUPPORTED;
  if (mass == nullptr || row_ptr == nullptr || ws == nullptr || !bsa::aligned16(ws) ||
      !aligned4(mass) || !aligned4(row_ptr))
    return BSA_ERR_INVALID_ARG;
  if (col_capacity < 0 || (col_capacity > 0 && (col_idx == nullptr || !aligned4(col_idx))))
    return BSA_ERR_INVALID_ARG;
  if (!(threshold > 0.f && threshold <= 1.f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa_topp_rows_workspace_bytes(rows, cols)) return BSA_ERR_CAPACITY;
  return from_cuda(bsa::launch_topp_select(mass, rows, cols, threshold, row_ptr, col_idx,
                                           col_capacity, ws, stream));
}

bsa_status bsa_cluster_fwd(const bsa_cluster_shape* shape, const void* q, const void* k,
                           const void* v, const int32_t* q_starts, const int32_t* q_counts,
                           const int32_t* k_starts, const int32_t* k_counts,
                           const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale,
                           void* out, float* lse, void* ws, size_t ws_bytes,
                           bsa_stream_t stream) {
  bsa_status st = check_cluster_shape(shape);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || q_starts == nullptr ||
      q_counts == nullptr || k_starts == nullptr || k_counts == nullptr || row_ptr == nullptr ||
      col_idx == nullptr || ws == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(v) || !bsa::aligned16(out) ||
      !bsa::aligned16(ws) || !aligned4(q_starts) || !aligned4(q_counts) || !aligned4(k_starts) ||
      !aligned4(k_counts) || !aligned4(row_ptr) || !aligned4(col_idx) ||
      (lse != nullptr && !aligned4(lse)))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < bsa_cluster_fwd_workspace_bytes(shape)) return BSA_ERR_CAPACITY;
  return from_cuda(bsa::launch_cluster_fwd(shape->batch, shape->heads, shape->head_dim,
                                           shape->n_tokens, shape->n_q_clusters,
                                           shape->n_k_clusters, q, k, v, q_starts, q_counts,
                                           k_starts, k_counts, row_ptr, col_idx, softmax_scale,
                                           out, lse, ws, stream));
}


bsa_status bsa_selftest_wait(void* ws, size_t ws_bytes, int64_t limit_ns, bsa_stream_t stream) {
  if (ws == nullptr || !bsa::aligned16(ws) || ws_bytes < bsa::kStatusBytes) return BSA_ERR_INVALID_ARG;
  if (limit_ns < 1000 || limit_ns > 10000000000LL) return BSA_ERR_INVALID_ARG;
  return from_cuda(bsa::launch_selftest_wait(ws, static_cast<uint64_t>(limit_ns), stream));
}


bsa_status bsa_fwd_raster(const bsa_shape* shape, const void* q, const void* k, const void* v,
                          const int32_t* row_ptr, const int32_t* col_idx, float softmax_scale,
                          void* out, float* lse, void* ws, size_t ws_bytes, bsa_stream_t stream) {
  bsa_status st = check_shape(shape, true);
  if (st != BSA_OK) return st;
  if (q == nullptr || k == nullptr || v == nullptr || out == nullptr || row_ptr == nullptr ||
      col_idx == nullptr || ws == nullptr)
    return BSA_ERR_INVALID_ARG;
  if (!bsa::aligned16(q) || !bsa::aligned16(k) || !bsa::aligned16(v) || !bsa::aligned16(out) ||
      !bsa::aligned16(ws) || (reinterpret_cast<uintptr_t>(row_ptr) & 3u) ||
      (reinterpret_cast<uintptr_t>(col_idx) & 3u) ||
      (lse != nullptr && (reinterpret_cast<uintptr_t>(lse) & 3u)))
    return BSA_ERR_INVALID_ARG;
  if (!(softmax_scale > 0.f) || !(softmax_scale < 1e30f)) return BSA_ERR_INVALID_ARG;
  if (ws_bytes < workspace_bytes(shape, BSA_OP_FWD)) return BSA_ERR_CAPACITY;
  const AttnDims a = make_attn(shape);
  return from_cuda(bsa::launch_bsattn_fwd_raster(a, q, k, v, row_ptr, col_idx, softmax_scale, out,
                                                 lse, ws, stream));
}

}  // extern "C"
