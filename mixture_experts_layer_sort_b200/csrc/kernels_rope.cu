// kernels_rope.cu - inverse rotary position embedding fused with per-head FP8
// quantisation, for any number of tokens (a run-time argument: one precompiled kernel
// per head size, nothing specialised or rebuilt per token count).
//
// The pages name this kernel, `_fused_inv_rope_fp8_quant_per_head`, as the one that
// used to be recompiled for every new token count, costing time to first token at
// eight-way tensor parallelism until its variable-length parameters were kept out of
// the specialisation (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200",
// section "3. Removing repeat compilation can reduce first-token delay"; aib.vote,
// "AWS SageMaker MoE kernel optimizations", fourth paragraph). They give only the
// name; what it computes here, per (token t, head h) vector of D values:
//   1. undo the rotation by the angles of position p = positions[t]: for each pair
//      (a', b') and its angle's c = cos, s = sin from the table row p
//      (cos in columns [0, D/2), sin in [D/2, D)):  a = a'c + b's,  b = b'c - a's,
//      each product, sum and difference rounded to fp32 in that order;
//      pairs are (i, i + D/2) (half-split) or (2i, 2i + 1) (interleaved);
//   2. one FP8 scale per vector: s = max|y| / F (F = 448 e4m3, 57344 e5m2; 1 for an
//      all-zero vector), codes = RNE(y / s) saturated, the division in IEEE fp32.
// A position outside [0, max_pos) has no table row: its vector gets codes 0 and a
// NaN scale (no out-of-bounds read).
//
// Layout and roofline: one warp per token; a head vector is spread over D/16 lanes,
// 16 consecutive values (32 bytes in, 16 bytes of codes out) per lane, so that the
// per-vector work (the max reduction, the scale, its reciprocal) is shared by 16 values
// and a warp covers 512/D vectors per pass; the half-split partner of a value sits D/32
// lanes away. The position (one token ahead) and the lane's part of the table row are
// read once per token, and up to four passes of vectors are in flight at once. The kernel moves 2D bytes in
// and D + 4 bytes out per vector, plus 4 + 4D bytes per token: it is HBM-bound.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdio>
#include <type_traits>

#include "../../include/moe_b200.h"
#include "fp8_format.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kRopeThreads = 256;

struct RopeArgs {
  const __nv_bfloat16* x;   // [T, NH, D]
  const int* positions;     // [T]
  const float* cos_sin;     // [max_pos, D]
  uint8_t* codes;           // [T, NH, D]
  float* scales;            // [T, NH]
  long long nvec;           // T * NH
  int NH, max_pos, f8;
  int interleaved;
};

constexpr int kEPL = 16;   // values of a head vector per lane

// n consecutive fp32 values (n a multiple of 4, 16-byte aligned)
template <int n>
__device__ __forceinline__ void load_f32(const float* p, float* v) {
  #pragma unroll
  for (int q = 0; q < n; q += 4) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(p + q));
    v[q] = f.x;
    v[q + 1] = f.y;
    v[q + 2] = f.z;
    v[q + 3] = f.w;
  }
}

constexpr int kRopePasses = 4;   // passes of head vectors per warp in flight

// D values per head vector, L = D / 16 lanes per vector (16 values each), 32 / L vectors
// per pass of a warp; one warp per token: the position (loaded one token ahead) and the
// lane's part of the token's cos/sin row are loaded once, then the token's heads up to
// four passes at a time, all their loads issued before any value is used.
template <int D>
__global__ void __launch_bounds__(kRopeThreads, 2) inv_rope_fp8_kernel(RopeArgs a) {
  constexpr int L = D / kEPL;          // lanes per head vector
  constexpr int HPW = 32 / L;          // head vectors per pass
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int hl = lane / L;             // this lane's head vector in a pass
  const int e0 = (lane % L) * kEPL;    // its values [e0, e0 + 16) of the vector
  const long long gwarp = (static_cast<long long>(blockIdx.x) * kRopeThreads + threadIdx.x) >> 5;
  const long long nwarps = static_cast<long long>(gridDim.x) * (kRopeThreads / 32);
  const float fmax = fp8_max(a.f8);
  // half-split: values i < D/2 pair with i + D/2, which sits L/2 lanes further; a lane
  // of the upper half holds the b' of its pairs. Interleaved: 2i pairs with 2i + 1.
  const bool upper = e0 >= D / 2;
  const int ang0 = a.interleaved ? e0 / 2 : (upper ? e0 - D / 2 : e0);
  const long long T = a.nvec / a.NH;
  int pos_next = gwarp < T ? __ldg(a.positions + gwarp) : 0;
  for (long long t = gwarp; t < T; t += nwarps) {
    const int pos = pos_next;                     // the same for the whole warp
    if (t + nwarps < T) pos_next = __ldg(a.positions + t + nwarps);
    const bool valid = pos >= 0 && pos < a.max_pos;
    float c[kEPL], s[kEPL];                       // interleaved: the first 8 of each
    if (valid) {
      const float* row = a.cos_sin + static_cast<long long>(pos) * D;
      if (a.interleaved) {
        load_f32<kEPL / 2>(row + ang0, c);
        load_f32<kEPL / 2>(row + D / 2 + ang0, s);
      } else {
        load_f32<kEPL>(row + ang0, c);
        load_f32<kEPL>(row + D / 2 + ang0, s);
      }
    }
    for (int h0 = 0; h0 < a.NH; h0 += kRopePasses * HPW) {
      // the raw bf16 values (two 16-byte vectors per pass) until each pass is used
      uint4 xr[kRopePasses][2];
      #pragma unroll
      for (int u = 0; u < kRopePasses; ++u) {
        const int h = h0 + u * HPW + hl;
        if (h < a.NH) {
          const uint4* p = reinterpret_cast<const uint4*>(a.x + (t * a.NH + h) * D + e0);
          xr[u][0] = __ldg(p);
          xr[u][1] = __ldg(p + 1);
        } else {
          xr[u][0] = make_uint4(0u, 0u, 0u, 0u);
          xr[u][1] = xr[u][0];
        }
      }
      #pragma unroll
      for (int u = 0; u < kRopePasses; ++u) {
        if (h0 + u * HPW >= a.NH) break;          // warp-uniform
        const int h = h0 + u * HPW + hl;          // lanes past the last head compute zeros
        float xv[kEPL];
        {
          const __nv_bfloat162* hp = reinterpret_cast<const __nv_bfloat162*>(xr[u]);
          #pragma unroll
          for (int q = 0; q < kEPL / 2; ++q) {
            const float2 f = __bfloat1622float2(hp[q]);
            xv[2 * q] = f.x;
            xv[2 * q + 1] = f.y;
          }
        }
        float y[kEPL];
        if (valid) {
          if (a.interleaved) {
            #pragma unroll
            for (int q = 0; q < kEPL / 2; ++q) {
              const float pa = xv[2 * q], pb = xv[2 * q + 1];
              y[2 * q] = __fadd_rn(__fmul_rn(pa, c[q]), __fmul_rn(pb, s[q]));
              y[2 * q + 1] = __fsub_rn(__fmul_rn(pb, c[q]), __fmul_rn(pa, s[q]));
            }
          } else {
            #pragma unroll
            for (int q = 0; q < kEPL; ++q) {
              const float other = __shfl_xor_sync(0xFFFFFFFFu, xv[q], L / 2);
              const float pa = upper ? other : xv[q];
              const float pb = upper ? xv[q] : other;
              y[q] = upper ? __fsub_rn(__fmul_rn(pb, c[q]), __fmul_rn(pa, s[q]))
                           : __fadd_rn(__fmul_rn(pa, c[q]), __fmul_rn(pb, s[q]));
            }
          }
        } else {   // (valid is the same for the whole warp: the shuffles above stay uniform)
          #pragma unroll
          for (int q = 0; q < kEPL; ++q) y[q] = 0.f;
        }
        float m = 0.f;
        #pragma unroll
        for (int q = 0; q < kEPL; ++q) m = fmaxf(m, fabsf(y[q]));
        #pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
        const float sc = m == 0.f ? 1.f : __fdiv_rn(m, fmax);
        const ScaleDiv dv(sc);   // y / sc, correctly rounded, one reciprocal per vector
        uint4 o;
        unsigned* ow = reinterpret_cast<unsigned*>(&o);
        #pragma unroll
        for (int q = 0; q < kEPL / 4; ++q) {
          const unsigned short lo = fp8x2(make_float2(dv(y[4 * q]), dv(y[4 * q + 1])), a.f8);
          const unsigned short hi = fp8x2(make_float2(dv(y[4 * q + 2]), dv(y[4 * q + 3])), a.f8);
          ow[q] = valid ? (static_cast<unsigned>(lo) | (static_cast<unsigned>(hi) << 16)) : 0u;
        }
        if (h < a.NH) {
          const long long v = t * a.NH + h;
          *reinterpret_cast<uint4*>(a.codes + v * D + e0) = o;
          if (e0 == 0) a.scales[v] = valid ? sc : __int_as_float(0x7FC00000);
        }
      }
    }
  }
}

// The grid is capped at the blocks that are resident at once (a grid-stride loop
// over tokens), so that every warp runs several tokens with its position loads one
// token ahead instead of blocks arriving in waves.
template <int D>
cudaError_t launch_rope(const RopeArgs& a, cudaStream_t s) {
  static const int per_sm = [] {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, inv_rope_fp8_kernel<D>, kRopeThreads, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    return n;
  }();
  const long long per_block = kRopeThreads / 32;   // tokens per block and round
  long long blocks = (a.nvec / a.NH + per_block - 1) / per_block;
  const long long cap = static_cast<long long>(per_sm) * sm_count();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  return launch_kernel(inv_rope_fp8_kernel<D>, dim3(static_cast<unsigned>(blocks)), dim3(kRopeThreads), 0, s, a);
}

bool aligned(const void* p, unsigned bytes) { return (reinterpret_cast<uintptr_t>(p) & (bytes - 1)) == 0; }

}  // namespace

}  // namespace moe

extern "C" int moe_inv_rope_fp8_quant(const void* x, const int* positions, const float* cos_sin, int max_pos,
                                      int num_tokens, int num_heads, int head_dim, int interleaved, int fp8_format,
                                      void* codes, float* scales, void* stream) {
  if (num_tokens < 0 || num_heads < 1 || max_pos < 1 || (interleaved != 0 && interleaved != 1))
    return MOE_ERR_INVALID_ARG;
  if (head_dim != 64 && head_dim != 128 && head_dim != 256) return MOE_ERR_INVALID_ARG;
  if (fp8_format != MOE_DTYPE_FP8_E4M3 && fp8_format != MOE_DTYPE_FP8_E5M2) return MOE_ERR_INVALID_ARG;
  if (num_tokens == 0) return MOE_OK;
  if (!x || !positions || !cos_sin || !codes || !scales) return MOE_ERR_INVALID_ARG;
  if (!moe::aligned(x, 16) || !moe::aligned(cos_sin, 16) || !moe::aligned(codes, 16) || !moe::aligned(positions, 4) ||
      !moe::aligned(scales, 4))
    return MOE_ERR_INVALID_ARG;
  moe::RopeArgs a{};
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.positions = positions;
  a.cos_sin = cos_sin;
  a.codes = static_cast<uint8_t*>(codes);
  a.scales = scales;
  a.nvec = static_cast<long long>(num_tokens) * num_heads;
  a.NH = num_heads;
  a.max_pos = max_pos;
  a.f8 = fp8_format == MOE_DTYPE_FP8_E5M2 ? moe::kFp8E5M2 : moe::kFp8E4M3;
  a.interleaved = interleaved;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  moe::NvtxRange range("moe_inv_rope_fp8_quant");
  cudaError_t e = head_dim == 64 ? moe::launch_rope<64>(a, st)
                                 : (head_dim == 128 ? moe::launch_rope<128>(a, st) : moe::launch_rope<256>(a, st));
  if (e != cudaSuccess) {
    std::fprintf(stderr, "moe_inv_rope_fp8_quant: launch failed: %s\n", cudaGetErrorString(e));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}
