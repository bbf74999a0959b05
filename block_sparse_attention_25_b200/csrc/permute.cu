// 3D tile permutation between raster token order and 4x4x4 tile-major order, and the
// same permutation fused with per-tile e4m3 quantisation.
//
// "FPSAttention: Training-Aware FP8 and Sparsity Co-Design for Fast Video Diffusion",
// Abstract, innovation 1: one 3D tile granularity is the unit of both the sparsity
// block and the FP8 quantisation scale.
//
// Both kernels are HBM-bound copies.  Every thread moves whole 16-byte vectors; one
// (slot, head) row of D elements is a contiguous 128- or 256-byte run on both sides, so
// reads and writes use full 32-byte sectors.
#include "bsa_kernels.cuh"

namespace bsa {

// dst[b][h][p][:] = src[b][token(p)][h][:] (zero for pad slots).  One thread per 16-byte
// vector of the destination, grid-stride, four vectors in flight per thread.  Idx is
// uint32_t when the vector count fits, so the index divisions stay 32-bit.
template <typename Idx>
__global__ void __launch_bounds__(256) tile_permute_fwd_kernel(const uint4* __restrict__ src,
                                                               uint4* __restrict__ dst,
                                                               GridDims g, int heads, int vpr,
                                                               Idx total) {
  const Idx stride = static_cast<Idx>(gridDim.x) * blockDim.x;
  for (Idx base = static_cast<Idx>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
       base += 4 * stride) {
    uint4 val[4];
    Idx idx[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      idx[u] = base + u * stride;
      val[u] = make_uint4(0u, 0u, 0u, 0u);
      if (idx[u] < total) {
        const Idx row = idx[u] / vpr;  // (b*heads + h)*Np + p
        const int v = static_cast<int>(idx[u] - row * vpr);
        const Idx bh = row / g.Np;
        const int p = static_cast<int>(row - bh * g.Np);
        const int h = static_cast<int>(bh % heads);
        const long long b = static_cast<long long>(bh / heads);
        const int tok = slot_to_token(g, p);
        if (tok >= 0) val[u] = __ldg(src + ((b * g.S + tok) * heads + h) * vpr + v);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (idx[u] < total) dst[idx[u]] = val[u];
  }
}

// dst[b][s][h][:] = src[b][h][slot(s)][:].  One thread per 16-byte vector of the raster
// destination.
template <typename Idx>
__global__ void __launch_bounds__(256) tile_permute_inv_kernel(const uint4* __restrict__ src,
                                                               uint4* __restrict__ dst,
                                                               GridDims g, int heads, int vpr,
                                                               Idx total) {
  const Idx stride = static_cast<Idx>(gridDim.x) * blockDim.x;
  for (Idx base = static_cast<Idx>(blockIdx.x) * blockDim.x + threadIdx.x; base < total;
       base += 4 * stride) {
    uint4 val[4];
    Idx idx[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      idx[u] = base + u * stride;
      if (idx[u] < total) {
        const Idx row = idx[u] / vpr;  // (b*S + s)*heads + h
        const int v = static_cast<int>(idx[u] - row * vpr);
        const Idx bs = row / heads;
        const int h = static_cast<int>(row - bs * heads);
        const Idx bb = bs / g.S;
        const int s = static_cast<int>(bs - bb * g.S);
        const long long b = static_cast<long long>(bb);
        const int p = token_to_slot(g, s);
        val[u] = __ldg(src + ((b * heads + h) * g.Np + p) * vpr + v);
      }
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (idx[u] < total) dst[idx[u]] = val[u];
  }
}

// Permute + quantise: one 128-thread CTA per (b, h, 64-token tile).  The tile's 64 x D
// bf16 values are gathered from the raster source into registers, reduced to absmax,
// and written as e4m3 codes x / s, s = absmax / 448 (1 for an all-zero tile).
template <int D>
__global__ void __launch_bounds__(128) tile_permute_quant_e4m3_kernel(
    const uint4* __restrict__ src, uint8_t* __restrict__ dst, float* __restrict__ scales,
    GridDims g, int heads) {
  constexpr int VPR = D / 8;             // 16-byte vectors of 8 bf16 per row
  constexpr int NV = 64 * VPR / 128;     // vectors per thread
  const int tile_lin = blockIdx.x;       // (b*heads + h)*ntiles + tile
  const int ntiles = g.Np >> 6;
  const int tile = tile_lin % ntiles;
  const int bh = tile_lin / ntiles;
  const int h = bh % heads;
  const int b = bh / heads;

  uint4 vals[NV];
  float amax = 0.f;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int vi = threadIdx.x + 128 * i;
    const int r = vi / VPR, c = vi % VPR;
    const int tok = slot_to_token(g, tile * 64 + r);
    vals[i] = make_uint4(0u, 0u, 0u, 0u);
    if (tok >= 0)
      vals[i] = __ldg(src + ((static_cast<long long>(b) * g.S + tok) * heads + h) * VPR + c);
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&vals[i]);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(e[k]);
      amax = fmaxf(amax, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  __shared__ float red[4];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = amax;
  __syncthreads();
  amax = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
  const float s = (amax == 0.f) ? 1.f : __fdiv_rn(amax, 448.f);
  if (threadIdx.x == 0) scales[tile_lin] = s;

  uint8_t* out = dst + (static_cast<long long>(bh) * g.Np + tile * 64) * D;
#pragma unroll
  for (int i = 0; i < NV; ++i) {
    const int vi = threadIdx.x + 128 * i;
    const __nv_bfloat162* e = reinterpret_cast<const __nv_bfloat162*>(&vals[i]);
    uint16_t c[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __bfloat1622float2(e[k]);
      c[k] = pack_e4m3x2(__fdiv_rn(f.x, s), __fdiv_rn(f.y, s));
    }
    uint2 packed;
    packed.x = static_cast<uint32_t>(c[0]) | (static_cast<uint32_t>(c[1]) << 16);
    packed.y = static_cast<uint32_t>(c[2]) | (static_cast<uint32_t>(c[3]) << 16);
    reinterpret_cast<uint2*>(out)[vi] = packed;
  }
}

static int copy_grid(long long total) {
  // Enough CTAs to fill every SM several times over; the loop covers the rest.
  long long want = (total + 4 * 256 - 1) / (4 * 256);
  const long long cap = 148LL * 16;
  return static_cast<int>(want < 1 ? 1 : (want > cap ? cap : want));
}

cudaError_t launch_tile_permute(const GridDims& g, int batch, int heads, int row_bytes,
                                int inverse, const void* src, void* dst, cudaStream_t stream) {
  const int vpr = row_bytes / 16;
  const long long rows = inverse ? static_cast<long long>(batch) * g.S * heads
                                 : static_cast<long long>(batch) * heads * g.Np;
  const long long total = rows * vpr;
  if (total == 0) return cudaSuccess;
  const int grid = copy_grid(total);
  const uint4* in = static_cast<const uint4*>(src);
  uint4* out = static_cast<uint4*>(dst);
  // 32-bit indexing while idx + 4 * stride cannot wrap.
  const bool small = total + 8LL * grid * 256 < (1LL << 32);
  if (inverse) {
    if (small)
      tile_permute_inv_kernel<uint32_t><<<grid, 256, 0, stream>>>(in, out, g, heads, vpr,
                                                                   static_cast<uint32_t>(total));
    else
      tile_permute_inv_kernel<unsigned long long><<<grid, 256, 0, stream>>>(
          in, out, g, heads, vpr, static_cast<unsigned long long>(total));
  } else {
    if (small)
      tile_permute_fwd_kernel<uint32_t><<<grid, 256, 0, stream>>>(in, out, g, heads, vpr,
                                                                   static_cast<uint32_t>(total));
    else
      tile_permute_fwd_kernel<unsigned long long><<<grid, 256, 0, stream>>>(
          in, out, g, heads, vpr, static_cast<unsigned long long>(total));
  }
  return cudaGetLastError();
}

cudaError_t launch_tile_permute_quant_e4m3(const GridDims& g, int batch, int heads, int head_dim,
                                           const void* src, uint8_t* dst, float* scales,
                                           cudaStream_t stream) {
  const long long ntiles = static_cast<long long>(batch) * heads * (g.Np / 64);
  if (ntiles == 0) return cudaSuccess;
  if (head_dim == 128)
    tile_permute_quant_e4m3_kernel<128><<<static_cast<unsigned>(ntiles), 128, 0, stream>>>(
        static_cast<const uint4*>(src), dst, scales, g, heads);
  else
    tile_permute_quant_e4m3_kernel<64><<<static_cast<unsigned>(ntiles), 128, 0, stream>>>(
        static_cast<const uint4*>(src), dst, scales, g, heads);
  return cudaGetLastError();
}

}  // namespace bsa
