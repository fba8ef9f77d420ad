// kernels_route.cu - router top-k, activation gather/quantise, h quantise and
// finalise.
//
// Router: "a token usually activates only a selected subset" of the experts
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section
// "Why MoE inference needs specialized kernels"). Each token keeps its k largest
// logits, equal logits going to the lower expert id, and weights the selected
// experts by their softmax renormalised over the selection.
//
// FP8: per-tensor ("tensor-quantized", same page, section "2. FP8 backend routing
// changes which kernel path runs") E4M3 or E5M2 codes, s = amax / (the format's
// largest finite value), codes = RNE(v / s) saturated, the division in IEEE fp32
// (fp8_format.cuh).
#include "fp8_format.cuh"

#include "moe_internal.h"
#include "route_common.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kRouteWarps = 8;

// One warp per token (route_token); FP8 layers also fold the token's max |x| into
// the per-tensor amax word.
template <int NPL>
__global__ void __launch_bounds__(kRouteWarps * 32) route_kernel(RouteArgs a) {
  const int t = blockIdx.x * kRouteWarps + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  pdl_wait();
  pdl_trigger();
  // max|h| starts at zero whatever path the previous forward took (gate_up, which folds
  // into it, waits for this kernel to complete)
  if (a.amax_h_reset != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *a.amax_h_reset = 0u;
  if (t >= a.M) return;
  route_token<NPL>(a.logits + static_cast<size_t>(t) * a.E, a.E, a.k, lane, a.topk_ids + static_cast<size_t>(t) * a.k,
                   a.topk_w + static_cast<size_t>(t) * a.k);

  if (a.amax_x != nullptr) {
    // FP8: this token's contribution to max |x|
    const uint4* xr = reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(t) * a.H);
    float m = 0.f;
    for (int i = lane; i < a.H / 8; i += 32) {
      const uint4 v = xr[i];
      const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&v);
      #pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float2 f = __bfloat1622float2(p[q]);
        m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
      }
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) atomicMax(a.amax_x, __float_as_uint(m));
  }
}

// 8 fp32 values -> 8 FP8 codes (RNE, saturating), v[i] / s correctly rounded.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], const ScaleDiv& dv, int f8) {
  uint2 r;
  unsigned short c[4];
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    float2 f = make_float2(dv(v[2 * q]), dv(v[2 * q + 1]));
    c[q] = fp8x2(f, f8);
  }
  r.x = static_cast<unsigned>(c[0]) | (static_cast<unsigned>(c[1]) << 16);
  r.y = static_cast<unsigned>(c[2]) | (static_cast<unsigned>(c[3]) << 16);
  return r;
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4& u, float (&v)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    const float2 f = __bfloat1622float2(p[q]);
    v[2 * q] = f.x;
    v[2 * q + 1] = f.y;
  }
}

// Row copies (gather, h quantise): 128 threads per row, two rows per 256-thread block.
// A thread loads up to 8 of the row's 16-byte vectors (8 bf16 each) before it stores
// any, so a row costs one memory round trip per 8 x 128 vectors, and the per-element
// work (the FP8 division) is spread over 128 threads instead of one warp.
constexpr int kRowThreads = 128;
constexpr int kRowsPerBlock = 256 / kRowThreads;

template <bool kFP8, bool kCoherent>
__device__ __forceinline__ void copy_row(const uint4* __restrict__ src, void* __restrict__ dst, int n8, float s,
                                         int f8, int t) {
  const ScaleDiv dv(s);
  for (int base = t; base < n8; base += kRowThreads * 8) {
    uint4 v[8];
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      if (base + kRowThreads * j < n8) v[j] = kCoherent ? __ldcg(src + base + kRowThreads * j) : __ldg(src + base + kRowThreads * j);
    #pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int i = base + kRowThreads * j;
      if (i < n8) {
        if constexpr (!kFP8) {
          reinterpret_cast<uint4*>(dst)[i] = v[j];
        } else {
          float f[8];
          bf16x8_to_f32(v[j], f);
          reinterpret_cast<uint2*>(dst)[i] = quant8(f, dv, f8);
        }
      }
    }
  }
}

// x_perm row r = the x row of the token of padded pair r (or its FP8 codes). Blocks
// stride over the rows (the grid is capped at a few blocks per SM), so that a
// thread's stores of one row overlap its loads of the next. With `xq` set (large FP8
// batches) the token rows are already quantised and the rows are byte copies.
// (at most 85 registers: a CTA fits next to a grouped-GEMM CTA on one SM)
template <bool kFP8>
__global__ void __launch_bounds__(256, 3) gather_kernel(GatherArgs a) {
  const int t = threadIdx.x % kRowThreads;
  pdl_wait();
  pdl_trigger();
  // independent loads issued together (rows past rows_used hold stale but in-bounds pairs)
  const int used = a.header[kHdrRowsUsed];
  const unsigned amax = (kFP8 && a.xq == nullptr) ? *a.amax_x : 0u;
  const float s = kFP8 ? fp8_scale_from_amax(amax, a.f8) : 1.f;
  const int bound = used < a.rows_bound ? used : a.rows_bound;
  for (int r = blockIdx.x * kRowsPerBlock + threadIdx.x / kRowThreads; r < bound;
       r += gridDim.x * kRowsPerBlock) {
    const int p = a.padded_pairs[r];
    if (p >= a.P) continue;   // a pad row: never read by an output column
    const size_t tok = static_cast<size_t>(p / a.k);
    if constexpr (!kFP8) {
      copy_row<false, false>(reinterpret_cast<const uint4*>(a.x + tok * a.H),
                             static_cast<__nv_bfloat16*>(a.x_perm) + static_cast<size_t>(r) * a.H, a.H / 8, 1.f, 0, t);
    } else if (a.xq != nullptr) {
      copy_row<false, false>(reinterpret_cast<const uint4*>(a.xq + tok * a.H),
                             static_cast<uint8_t*>(a.x_perm) + static_cast<size_t>(r) * a.H, a.H / 16, 1.f, 0, t);
    } else {
      copy_row<true, false>(reinterpret_cast<const uint4*>(a.x + tok * a.H),
                            static_cast<uint8_t*>(a.x_perm) + static_cast<size_t>(r) * a.H, a.H / 8, s, a.f8, t);
    }
  }
}

// A precision per expert: row r of a pair routed to an FP8 expert gets the codes of
// its token's x row in x_perm8; a pair of a bf16 expert gets the bf16 row in x_perm.
__global__ void __launch_bounds__(256) gather_mixed_kernel(GatherArgs a) {
  const int t = threadIdx.x % kRowThreads;
  pdl_wait();
  pdl_trigger();
  const int used = a.header[kHdrRowsUsed];
  const float s = fp8_scale_from_amax(*a.amax_x, a.f8);
  const int bound = used < a.rows_bound ? used : a.rows_bound;
  for (int r = blockIdx.x * kRowsPerBlock + threadIdx.x / kRowThreads; r < bound;
       r += gridDim.x * kRowsPerBlock) {
    const int p = a.padded_pairs[r];
    if (p >= a.P) continue;   // a pad row: never read by an output column
    const size_t tok = static_cast<size_t>(p / a.k);
    const uint4* src = reinterpret_cast<const uint4*>(a.x + tok * a.H);
    if (a.eflags[a.topk_ids[p]] != 0)
      copy_row<true, false>(src, a.x_perm8 + static_cast<size_t>(r) * a.H, a.H / 8, s, a.f8, t);
    else
      copy_row<false, false>(src, static_cast<__nv_bfloat16*>(a.x_perm) + static_cast<size_t>(r) * a.H, a.H / 8,
                             1.f, 0, t);
  }
}

// FP8, large batches: the M token rows of x -> FP8 codes with s_x = amax(x)/F, once
// per token instead of once per (token, slot) pair.
__global__ void __launch_bounds__(256) quant_x_kernel(QuantXArgs a) {
  const int t = threadIdx.x % kRowThreads;
  pdl_wait();
  pdl_trigger();
  const float s = fp8_scale_from_amax(*a.amax_x, a.f8);
  for (int r = blockIdx.x * kRowsPerBlock + threadIdx.x / kRowThreads; r < a.M; r += gridDim.x * kRowsPerBlock)
    copy_row<true, false>(reinterpret_cast<const uint4*>(a.x + static_cast<size_t>(r) * a.H),
                          a.xq + static_cast<size_t>(r) * a.H, a.H / 8, s, a.f8, t);
}

// FP8: h (bf16) -> codes with s_h = amax(h)/F over the valid rows.
__global__ void __launch_bounds__(256) quant_h_kernel(QuantHArgs a) {
  const int t = threadIdx.x % kRowThreads;
  pdl_wait();
  pdl_trigger();
  const int used = a.header[kHdrRowsUsed];
  const float s = fp8_scale_from_amax(*a.amax_h, a.f8);
  const int bound = used < a.rows_bound ? used : a.rows_bound;
  for (int r = blockIdx.x * kRowsPerBlock + threadIdx.x / kRowThreads; r < bound;
       r += gridDim.x * kRowsPerBlock) {
    const int p = a.padded_pairs[r];
    if (p >= a.P) continue;
    if (a.eflags != nullptr && a.eflags[a.topk_ids[p]] == 0) continue;   // a bf16 expert's row
    // h was written by the previous kernel: coherent loads, not the read-only path
    copy_row<true, true>(reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(r) * a.I),
                         a.h_q + static_cast<size_t>(r) * a.I, a.I / 8, s, a.f8, t);
  }
}

// out = bf16(acc); acc = 0 for the next forward; reset the FP8 amax words.
// Four float4 of acc per thread per step, all loaded before any is stored.
__global__ void __launch_bounds__(256) finalize_kernel(FinalizeArgs a) {
  pdl_wait();
  pdl_trigger();
  if (blockIdx.x == 0 && threadIdx.x == 0 && a.amax != nullptr) {
    if (a.last_scales != nullptr) {
      a.last_scales[0] = fp8_scale_from_amax(a.amax[0], a.f8);
      a.last_scales[1] = fp8_scale_from_amax(a.amax[1], a.f8);
    }
    a.amax[0] = 0u;
    a.amax[1] = 0u;
  }
  const long long n4 = a.n / 4;
  float4* acc4 = reinterpret_cast<float4*>(a.acc);
  uint2* out4 = reinterpret_cast<uint2*>(a.out);
  const long long T = static_cast<long long>(gridDim.x) * 256;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
  for (long long i = blockIdx.x * 256ll + threadIdx.x; i < n4; i += 4 * T) {
    float4 v[4];
    #pragma unroll
    for (int j = 0; j < 4; ++j)
      if (i + j * T < n4) v[j] = __ldcg(acc4 + i + j * T);
    #pragma unroll
    for (int j = 0; j < 4; ++j) {
      const long long q = i + j * T;
      if (q < n4) {
        __stcg(acc4 + q, zero);
        const __nv_bfloat162 lo = __floats2bfloat162_rn(v[j].x, v[j].y);
        const __nv_bfloat162 hi = __floats2bfloat162_rn(v[j].z, v[j].w);
        uint2 o;
        o.x = *reinterpret_cast<const unsigned*>(&lo);
        o.y = *reinterpret_cast<const unsigned*>(&hi);
        out4[q] = o;
      }
    }
  }
}

}  // namespace

// The one-row kernels ask for the largest shared-memory carveout, as the grouped GEMMs
// need it: an SM then never has to change its L1 / shared split between the two, and a
// GEMM CTA can start next to one of theirs.
cudaError_t route_configure() {
  const int c = cudaSharedmemCarveoutMaxShared;
  const cudaFuncAttribute at = cudaFuncAttributePreferredSharedMemoryCarveout;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(route_kernel<1>, at, c)) || (e = cudaFuncSetAttribute(route_kernel<2>, at, c)) ||
      (e = cudaFuncSetAttribute(route_kernel<4>, at, c)) || (e = cudaFuncSetAttribute(route_kernel<8>, at, c)) ||
      (e = cudaFuncSetAttribute(route_kernel<16>, at, c)) || (e = cudaFuncSetAttribute(gather_kernel<false>, at, c)) ||
      (e = cudaFuncSetAttribute(gather_kernel<true>, at, c)) || (e = cudaFuncSetAttribute(quant_x_kernel, at, c)) ||
      (e = cudaFuncSetAttribute(quant_h_kernel, at, c)))
    return e;
  return cudaFuncSetAttribute(finalize_kernel, at, c);
}

cudaError_t launch_route(const RouteArgs& a, cudaStream_t s) {
  const int grid = (a.M + kRouteWarps - 1) / kRouteWarps;
  const dim3 g(grid), b(kRouteWarps * 32);
  if (a.E <= 32) return launch_kernel(route_kernel<1>, g, b, 0, s, a);
  if (a.E <= 64) return launch_kernel(route_kernel<2>, g, b, 0, s, a);
  if (a.E <= 128) return launch_kernel(route_kernel<4>, g, b, 0, s, a);
  if (a.E <= 256) return launch_kernel(route_kernel<8>, g, b, 0, s, a);
  return launch_kernel(route_kernel<16>, g, b, 0, s, a);
}

// Row kernels: one block per two rows, or (capped) at most 8 blocks per SM striding
// over the rows. Measured at prefill size on one box: the bf16 gather (14 KB
// row copies) is faster uncapped (127 vs 141 us), the FP8 row kernels (quantising,
// or copying 1-byte rows) capped (x: 116 vs 150 us, h: 68 vs 81 us). At decode sizes
// (at most 8192 padded rows) the gather and the h quantisation run one block per SM, so
// that the grouped GEMM launched after them finds room for its CTAs at once (decode bf16
// M = 16 / 64 and e4m3 M = 32 / 64 1.4-2.5 us faster).
int row_grid(int rows, bool capped) {
  const int g = (rows + kRowsPerBlock - 1) / kRowsPerBlock;
  const int cap = 8 * sm_count();
  return g < 1 ? 1 : ((capped && g > cap) ? cap : g);
}

cudaError_t launch_gather(const GatherArgs& a, bool fp8, cudaStream_t s) {
  if (a.eflags != nullptr)
    return launch_kernel(gather_mixed_kernel, dim3(row_grid(a.rows_bound, true)), dim3(256), 0, s, a);
  int grid = row_grid(a.rows_bound, fp8);
  if (a.rows_bound <= 8192 && grid > sm_count()) grid = sm_count();
  if (fp8) return launch_kernel(gather_kernel<true>, dim3(grid), dim3(256), 0, s, a);
  return launch_kernel(gather_kernel<false>, dim3(grid), dim3(256), 0, s, a);
}

cudaError_t launch_quant_x(const QuantXArgs& a, cudaStream_t s) {
  return launch_kernel(quant_x_kernel, dim3(row_grid(a.M, true)), dim3(256), 0, s, a);
}

cudaError_t launch_quant_h(const QuantHArgs& a, cudaStream_t s) {
  int grid = row_grid(a.rows_bound, true);
  if (a.rows_bound <= 8192 && grid > sm_count()) grid = sm_count();
  return launch_kernel(quant_h_kernel, dim3(grid), dim3(256), 0, s, a);
}

cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s) {
  long long n4 = a.n / 4;
  long long blocks = (n4 + 255) / 256;
  if (blocks < 1) blocks = 1;
  if (blocks > 8ll * sm_count()) blocks = 8ll * sm_count();
  return launch_kernel(finalize_kernel, dim3(static_cast<int>(blocks)), dim3(256), 0, s, a);
}

}  // namespace moe
