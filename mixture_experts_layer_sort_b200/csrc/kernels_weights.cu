// kernels_weights.cu - load-time weight preparation (not on the forward path):
// per (expert, tensor) FP8 scales, e4m3 quantisation, and the tiled storage layout.
//
// Stored layout: tile (e, rb, kb) holds rows [rb*128, rb*128+128) and bytes
// [kb*128, kb*128+128) of expert e's row-major matrix, as 128 rows of 128 bytes,
// 16 KB contiguous; tiles are ordered by e, then rb, then kb. A GEMM stage's weight
// tile is then one contiguous 16 KB read, which spreads over every HBM channel,
// where a row-major tile would be 128 pieces of 128 bytes one row pitch apart.
//
// FP8 ("tensor-quantized", toolboxkart.tech, "AWS SageMaker MoE kernel
// optimizations H200", section "2. FP8 backend routing changes which kernel path
// runs"): one scale per expert tensor s = amax / (the format's largest finite value,
// 448 for E4M3, 57344 for E5M2; 1 for an all-zero tensor), codes = RNE(w / s)
// saturated, the division in IEEE fp32 (fp8_format.cuh).
#include "fp8_format.cuh"
#include "moe_internal.h"

namespace moe {

namespace {

__device__ __forceinline__ long long tiled_offset(const TileGeom& g, long long e, long long r, long long byte) {
  const long long kbn = g.row_bytes / 128;
  const long long slot = g.expert_tiles > 0 ? g.expert_tiles : g.rb_total * kbn;
  const long long tile = e * slot + (g.rb_offset + r / 128) * kbn + byte / 128;
  return (tile * 128 + (r & 127)) * 128 + (byte & 127);
}

// Byte offset, in the row-major side, of byte `b` of row r of expert e.
__device__ __forceinline__ long long rowmajor_offset(const TileGeom& g, long long e, long long r, long long b) {
  return e * g.src_expert_stride + r * g.src_row_stride + g.src_offset + b;
}

// scales[e * stride] = amax of expert e's rows (bf16, row-major side of g; K = row_bytes
// elements per row, the stored layout being FP8) / the format's largest finite value.
__global__ void __launch_bounds__(1024) weight_amax_kernel(int f8, const uint8_t* w, TileGeom g, float* scales,
                                                           int stride) {
  const int e = blockIdx.x;
  if (g.expert_mask != nullptr && g.expert_mask[e] != g.mask_value) return;
  const long long per_row = g.row_bytes / 8;       // 16-byte vectors of 8 bf16 per row
  float m = 0.f;
  for (long long i = threadIdx.x; i < g.rows * per_row; i += blockDim.x) {
    const long long r = i / per_row;
    const long long c = (i - r * per_row) * 16;
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(w + rowmajor_offset(g, e, r, c)));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(p[q]);
      m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
    }
  }
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ float red[32];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = (threadIdx.x < (blockDim.x >> 5)) ? red[threadIdx.x] : 0.f;
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (threadIdx.x == 0) scales[static_cast<size_t>(e) * stride] = fp8_scale_from_amax(__float_as_uint(m), f8);
  }
}

// 8 bf16 -> 8 FP8 codes (8 bytes) per thread, written at their tiled position.
__global__ void __launch_bounds__(256) weight_quant_tiled_kernel(int f8, const uint8_t* w, TileGeom g,
                                                                 const float* scales, int stride, uint8_t* dst) {
  const long long K = g.row_bytes;                 // FP8: one byte per element
  const long long per_row = K / 8;
  const long long total = static_cast<long long>(g.E) * g.rows * per_row;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<long long>(gridDim.x) * 256) {
    const long long row = i / per_row;              // e * rows + r
    const long long c = (i - row * per_row) * 8;
    const long long e = row / g.rows;
    const long long r = row - e * g.rows;
    if (g.expert_mask != nullptr && g.expert_mask[e] != g.mask_value) continue;
    const ScaleDiv dv(__ldg(scales + e * stride));
    // 8 bf16 source values = 16 bytes at column c of the row-major source
    const uint4 u = __ldg(reinterpret_cast<const uint4*>(w + rowmajor_offset(g, e, r, 2 * c)));
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
    unsigned short c2[4];
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 f = __bfloat1622float2(p[q]);
      const float2 d = make_float2(dv(f.x), dv(f.y));
      c2[q] = fp8x2(d, f8);
    }
    uint2 o;
    o.x = static_cast<unsigned>(c2[0]) | (static_cast<unsigned>(c2[1]) << 16);
    o.y = static_cast<unsigned>(c2[2]) | (static_cast<unsigned>(c2[3]) << 16);
    *reinterpret_cast<uint2*>(dst + tiled_offset(g, e, r, c)) = o;
  }
}

// 16-byte vectors between the row-major [E, rows, row_bytes] and the tiled layout.
template <bool kToTiled>
__global__ void __launch_bounds__(256) retile_kernel(const uint8_t* src, TileGeom g, uint8_t* dst) {
  const long long per_row = g.row_bytes / 16;
  const long long total = static_cast<long long>(g.E) * g.rows * per_row;
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < total; i += static_cast<long long>(gridDim.x) * 256) {
    const long long row = i / per_row;
    const long long b = (i - row * per_row) * 16;
    const long long e = row / g.rows;
    const long long r = row - e * g.rows;
    if (g.expert_mask != nullptr && g.expert_mask[e] != g.mask_value) continue;
    const long long t = tiled_offset(g, e, r, b);
    const long long m = rowmajor_offset(g, e, r, b);
    if constexpr (kToTiled) *reinterpret_cast<uint4*>(dst + t) = __ldg(reinterpret_cast<const uint4*>(src + m));
    else *reinterpret_cast<uint4*>(dst + m) = *reinterpret_cast<const uint4*>(src + t);
  }
}

int grid_for(long long work) {
  long long b = (work + 255) / 256;
  if (b > 32ll * sm_count()) b = 32ll * sm_count();
  return static_cast<int>(b < 1 ? 1 : b);
}

}  // namespace

cudaError_t launch_weight_amax(int f8, const __nv_bfloat16* w, const TileGeom& g, float* scales, int stride,
                               cudaStream_t s) {
  weight_amax_kernel<<<g.E, 1024, 0, s>>>(f8, reinterpret_cast<const uint8_t*>(w), g, scales, stride);
  return cudaGetLastError();
}

cudaError_t launch_weight_quant_tiled(int f8, const __nv_bfloat16* w, const TileGeom& g, const float* scales,
                                      int stride, uint8_t* dst, cudaStream_t s) {
  weight_quant_tiled_kernel<<<grid_for(g.E * g.rows * (g.row_bytes / 8)), 256, 0, s>>>(
      f8, reinterpret_cast<const uint8_t*>(w), g, scales, stride, dst);
  return cudaGetLastError();
}

cudaError_t launch_tile_weights(const void* src, const TileGeom& g, void* dst, cudaStream_t s) {
  retile_kernel<true><<<grid_for(g.E * g.rows * (g.row_bytes / 16)), 256, 0, s>>>(
      static_cast<const uint8_t*>(src), g, static_cast<uint8_t*>(dst));
  return cudaGetLastError();
}

cudaError_t launch_untile_weights(const void* src, const TileGeom& g, void* dst, cudaStream_t s) {
  retile_kernel<false><<<grid_for(g.E * g.rows * (g.row_bytes / 16)), 256, 0, s>>>(
      static_cast<const uint8_t*>(src), g, static_cast<uint8_t*>(dst));
  return cudaGetLastError();
}

}  // namespace moe
