// kernels_gemv.cu - the MoE layer for thin batches (up to 16 tokens) on the CUDA cores.
//
// At decode sizes an expert receives one or two tokens: each weight byte then feeds one
// or two multiply-adds, about 1 FLOP per byte, two orders of magnitude below the
// tensor cores' ridge, and the time of the layer is the time to stream the active
// experts' weights. What the tensor-core chain adds on top of that streaming is
// latency: an align launch, a gather, split-K partial sums (a 128-row weight tile over
// the whole reduction is more bytes than one SM should stream alone), and a finalize.
// This path runs the same arithmetic as three launches:
//   plan     route every token (the top-k rule of route_common.cuh), group the pairs
//            by expert (the align kernel's padded groups, kept for inspection) and
//            list the active experts; FP8: amax(x), s_x and the x codes;
//   gate_up  one CTA per (active expert, 8 intermediate features): 8 W_gate and 8 W_up
//            rows times every token of the expert, h = silu(g) * u stored bf16 by
//            pair; FP8: max|h| into the amax word;
//   down     one CTA per (token, 8 or 16 output features): the token's k experts'
//            W_down rows times their h rows, weighted by the routing weights and
//            summed in fp32, written to `out` as bf16 (no atomics, no finalize).
// The routing, the movement of tokens and the combination of the experts' outputs cost
// work around the matrix products, and fusing them cuts the number of GPU operations
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels").
// On Hopper the thin-batch answer was Swap-AB on the tensor cores (aib.vote, "AWS
// SageMaker MoE kernel optimizations", second paragraph); the tensor-core chain keeps it
// for wider batches, and this path replaces it where the product is a matrix-vector
// product.
//
// Every lane of a warp streams 16-byte pieces of the tiled weights (kernels_weights.cu:
// a 128-row x 128-byte tile is 16 KB contiguous, rows in order), so one warp load
// covers 4 consecutive 128-byte rows; the 8 lanes of a row split its 128 bytes and
// meet in a shuffle reduction. Activations sit in shared memory as bf16 values (FP8
// codes decode exactly into bf16), read once per K block and reused for every row the
// lane holds. Products accumulate in fp32; FP8 scales are applied as in the
// tensor-core epilogues (s_gate*s_x, s_up*s_x, routing weight * s_down * s_h).
#include <cuda_fp16.h>

#include <algorithm>

#include "fp8_format.cuh"
#include "moe_internal.h"
#include "route_common.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kPlanThreads = 1024;
constexpr int kGvThreads = 256;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGuRows = 8;                 // W_gate (and W_up) rows per gate_up CTA

enum WFormat : int { kWBf16 = 0, kWE4M3 = 1, kWE5M2 = 2 };

// Ask L2 to fetch `bytes` (a multiple of 16) at a 16-byte aligned global address.
__device__ __forceinline__ void prefetch_l2(const void* p, int bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// Elements in one 16-byte piece of a weight row, and per 128-byte K block.
template <int kW>
struct WTraits {
  static constexpr int kEPL = kW == kWBf16 ? 8 : 16;
  static constexpr int kKPB = kEPL * 8;
};

// 8 bf16 values (16 bytes of shared memory) -> fp32.
__device__ __forceinline__ void bf16x8_f32(const uint4& u, float* f) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
}

// 8 FP8 codes (8 bytes) -> their values as 8 bf16 (exact: every e4m3 and e5m2 value is a
// bf16 value).
__device__ __forceinline__ uint4 fp8x8_to_bf16(uint2 c, int f8) {
  const unsigned w[2] = {c.x, c.y};
  unsigned o[4];
  #pragma unroll
  for (int q = 0; q < 2; ++q) {
    #pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const __nv_fp8x2_storage_t s = static_cast<__nv_fp8x2_storage_t>(w[q] >> (16 * hh));
      const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(s, f8 == kFp8E5M2 ? __NV_E5M2 : __NV_E4M3);
      const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&r));
      const __nv_bfloat162 b = __floats2bfloat162_rn(v.x, v.y);
      o[2 * q + hh] = *reinterpret_cast<const unsigned*>(&b);
    }
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// 8 fp32 values -> 8 FP8 codes, v / s correctly rounded (ScaleDiv), RNE, saturating.
__device__ __forceinline__ uint2 codes8(const float (&v)[8], const ScaleDiv& dv, int f8) {
  unsigned short c[4];
  #pragma unroll
  for (int q = 0; q < 4; ++q) c[q] = fp8x2(make_float2(dv(v[2 * q]), dv(v[2 * q + 1])), f8);
  return make_uint2(static_cast<unsigned>(c[0]) | (static_cast<unsigned>(c[1]) << 16),
                    static_cast<unsigned>(c[2]) | (static_cast<unsigned>(c[3]) << 16));
}

// silu(z) = z / (1 + e^-z), as in the tensor-core gate_up epilogue.
__device__ __forceinline__ float silu_f(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// ------------------------------------------------------------------ route + plan
// One CTA. Warp t routes token t; FP8 layers also take max|x| over the batch and write
// the x codes; then the pairs are grouped by expert in ascending pair id (the rank of
// pair (t, j) inside its expert is the number of earlier tokens routed there: a popcount
// of the expert's token mask), padded to 16 rows like the align kernel, and the active
// experts are listed in ascending id order.
template <int NPL>
__global__ void __launch_bounds__(kPlanThreads, 1) gemv_plan_kernel(GemvArgs a) {
  __shared__ int s_ids[kGemvMaxM * 16];
  __shared__ float s_w[kGemvMaxM * 16];
  __shared__ int s_count[512];
  __shared__ unsigned s_mask[512];
  __shared__ int s_pad[512];
  __shared__ int s_poff[513];
  __shared__ float s_red[kPlanThreads / 32];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int E = a.E, k = a.k, P = a.M * a.k;
  for (int e = tid; e < E; e += kPlanThreads) {
    s_count[e] = 0;
    s_mask[e] = 0u;
  }
  pdl_wait();
  pdl_trigger();
  // the max|h| word of this forward starts at zero (gate_up folds into it)
  if (tid == 0 && a.xq != nullptr) a.amax[1] = 0u;
  if (warp < a.M) route_token<NPL>(a.logits + static_cast<size_t>(warp) * E, E, k, lane, s_ids + warp * k, s_w + warp * k);
  if (a.xq != nullptr) {
    // FP8: s_x = max|x| / F over the whole batch, then every token row's codes
    const int n8 = a.M * a.H / 8;
    const uint4* x8 = reinterpret_cast<const uint4*>(a.x);
    float m = 0.f;
    for (int i = tid; i < n8; i += kPlanThreads) {
      float f[8];
      bf16x8_f32(__ldg(x8 + i), f);
      #pragma unroll
      for (int q = 0; q < 8; ++q) m = fmaxf(m, fabsf(f[q]));
    }
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if (lane == 0) s_red[warp] = m;
    __syncthreads();
    m = 0.f;
    #pragma unroll 8
    for (int w = 0; w < kPlanThreads / 32; ++w) m = fmaxf(m, s_red[w]);
    if (tid == 0) a.amax[0] = __float_as_uint(m);
    const ScaleDiv dv(fp8_scale_from_amax(__float_as_uint(m), a.f8));
    uint2* xq8 = reinterpret_cast<uint2*>(a.xq);
    for (int i = tid; i < n8; i += kPlanThreads) {
      float f[8];
      bf16x8_f32(__ldg(x8 + i), f);
      xq8[i] = codes8(f, dv, a.f8);
    }
  }
  __syncthreads();
  for (int p = tid; p < P; p += kPlanThreads) {
    const int e = s_ids[p];
    a.topk_ids[p] = e;
    a.topk_w[p] = s_w[p];
    atomicAdd(&s_count[e], 1);
    atomicOr(&s_mask[e], 1u << (p / k));
  }
  __syncthreads();
  for (int e = tid; e < E; e += kPlanThreads) s_pad[e] = (s_count[e] + kPadRows - 1) / kPadRows * kPadRows;
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(s_pad, s_poff, E, lane);
  __syncthreads();
  if (warp == 1) {
    // active experts, ascending id: one ballot per 32 experts
    int n_act = 0;
    for (int base = 0; base < E; base += 32) {
      const int e = base + lane;
      const int c = e < E ? s_count[e] : 0;
      const unsigned m = __ballot_sync(0xFFFFFFFFu, c > 0);
      if (c > 0) a.active[n_act + __popc(m & ((1u << lane) - 1u))] = make_int4(e, c, s_poff[e], 0);
      n_act += __popc(m);
    }
    if (lane == 0) a.header[kHdrGemvActive] = n_act;
  }
  for (int p = tid; p < P; p += kPlanThreads) {
    const int e = s_ids[p];
    const int t = p / k;
    a.padded_pairs[s_poff[e] + __popc(s_mask[e] & ((1u << t) - 1u))] = p;
  }
  for (int e = tid; e < E; e += kPlanThreads) {
    for (int r = s_poff[e] + s_count[e]; r < s_poff[e + 1]; ++r) a.padded_pairs[r] = P;
    a.counts[e] = s_count[e];
    a.padded_offsets[e] = s_poff[e];
  }
  if (tid == 0) {
    a.padded_offsets[E] = s_poff[E];
    a.header[kHdrRowsUsed] = s_poff[E];
  }
}


// 8 weights (half `part` of a 16-byte piece for FP8, the whole piece for bf16) -> fp32.
template <int kW>
__device__ __forceinline__ void weights8_f32(const uint4& u, int part, float (&f)[8]) {
  if constexpr (kW == kWBf16) {
    bf16x8_f32(u, f);
  } else {
    const unsigned lo = part == 0 ? u.x : u.z, hi = part == 0 ? u.y : u.w;
    const unsigned w[2] = {lo, hi};
    #pragma unroll
    for (int q = 0; q < 2; ++q) {
      #pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const __nv_fp8x2_storage_t c = static_cast<__nv_fp8x2_storage_t>(w[q] >> (16 * hh));
        const __half2_raw r = __nv_cvt_fp8x2_to_halfraw2(c, kW == kWE5M2 ? __NV_E5M2 : __NV_E4M3);
        const float2 v = __half22float2(*reinterpret_cast<const __half2*>(&r));
        f[4 * q + 2 * hh] = v.x;
        f[4 * q + 2 * hh + 1] = v.y;
      }
    }
  }
}

// ------------------------------------------------------------------ streaming
// Each lane streams its own 16-byte pieces of the weights through a ring of kDepth
// stages in shared memory with cp.async (L2 -> shared, no registers held while in
// flight); a stage holds four pieces per lane, 2 KB per warp, and the ring runs across
// unit boundaries. A lane reads back only what it copied itself, after
// cp.async.wait_group: no barrier sits between the copy and the use. Two CTAs of 8 warps
// per SM keep 16 x 8 KB = 128 KB of weights in flight per SM.
constexpr int kDepth = 4;
constexpr int kCtasPerSm = 2;   // two CTAs of 8 warps per SM: 16 warps to hide the dot products' latency
constexpr int kStageWarp = 4 * 32 * 16;              // bytes of one stage of one warp
constexpr int kRingWarp = kDepth * kStageWarp;       // 8 KB
constexpr int kRingBytes = kGvWarps * kRingWarp;     // 64 KB per CTA

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(src),
               "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// the lane's piece i of ring slot d
__device__ __forceinline__ uint8_t* ring_piece(uint8_t* ring_lane, int d, int i) {
  return ring_lane + d * kStageWarp + i * 512;
}

// ------------------------------------------------------------------ gate_up
// Units (a, g): active expert a, W_gate rows [8g, 8g + 8) and the W_up rows of the same
// features, over the whole reduction, times the expert's tokens in passes of up to 4
// (an expert with more tokens streams its rows once per pass). CTA c takes the
// contiguous range [c*U/G, (c+1)*U/G) of the U = A*I/8 units (one or a few experts,
// whose pairs it keeps in shared memory with every token row of x); warp w takes units
// w, w + 8, ... of the range, K block after K block. In a K block lane l holds 16 bytes
// of gate rows l/8 and l/8 + 4 and of the same up rows. Unit positions advance by 8
// groups with a carry into the next expert (I/8 >= 16 groups per expert).
constexpr int kGuMaxExperts = 16;   // experts one CTA's range may span (host-checked)
constexpr int kGuTokens = 4;        // tokens per pass: the register tile of a lane

template <int kW>
__global__ void __launch_bounds__(kGvThreads, kCtasPerSm) gemv_gate_up_kernel(GemvArgs a) {
  constexpr int kEPL = WTraits<kW>::kEPL, kKPB = WTraits<kW>::kKPB;
  constexpr int NT = kGuTokens;
  extern __shared__ __align__(128) uint8_t gv_smem[];
  __shared__ int4 s_act[kGuMaxExperts];
  __shared__ int s_pairs[kGuMaxExperts * kGemvMaxM];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  uint8_t* ring = gv_smem + warp * kRingWarp + lane * 16;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(gv_smem + kRingBytes);   // [M][H]
  pdl_wait();
  pdl_trigger();
  // the plan was written by the previous kernel: read it from L2
  const int groups = a.I / kGuRows;
  const int U = __ldcg(a.header + kHdrGemvActive) * groups;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = static_cast<int>(static_cast<long long>(c) * U / G);
  const int u1 = static_cast<int>(static_cast<long long>(c + 1) * U / G);
  if (u0 >= u1) return;
  const int a0 = u0 / groups;
  const int R = (u1 - 1) / groups - a0 + 1;
  if (tid < R) s_act[tid] = __ldcg(a.active + a0 + tid);
  __syncthreads();
  const uint64_t pol = l2_policy_evict_first();
  const int nu = warp < u1 - u0 ? (u1 - u0 - warp + kGvWarps - 1) / kGvWarps : 0;
  // the warp's first unit, and its stages: K blocks of every pass of every unit
  const int ar_first = (u0 + warp) / groups, g_first = u0 + warp - ar_first * groups;
  int n_st = 0;
  {
    int ar = ar_first, g = g_first;
    for (int i = 0; i < nu; ++i) {
      n_st += (s_act[ar - a0].y + NT - 1) / NT * a.kb1;
      g += kGvWarps;
      if (g >= groups) {
        g -= groups;
        ++ar;
      }
    }
  }
  int is_ar = ar_first, is_g = g_first, is_pass = 0, is_kb = 0;   // next stage to issue
  auto issue = [&](int s) {
    if (s < n_st) {
      const long long e = s_act[is_ar - a0].x;
      const int f0 = is_g * kGuRows;
      const long long base = e * a.et1 + is_kb;
      const uint8_t* pg = a.w13 + ((base + static_cast<long long>(f0 >> 7) * a.kb1) * kTileRows + (f0 & 127)) * kRowBytes + lane * 16;
      const uint8_t* pu = a.w13 + ((base + static_cast<long long>((a.I + f0) >> 7) * a.kb1) * kTileRows + (f0 & 127)) * kRowBytes + lane * 16;
      const int d = s % kDepth;
      cp_async16(ring_piece(ring, d, 0), pg, pol);
      cp_async16(ring_piece(ring, d, 1), pg + 512, pol);
      cp_async16(ring_piece(ring, d, 2), pu, pol);
      cp_async16(ring_piece(ring, d, 3), pu + 512, pol);
      if (++is_kb == a.kb1) {
        is_kb = 0;
        if (++is_pass == (s_act[is_ar - a0].y + NT - 1) / NT) {
          is_pass = 0;
          is_g += kGvWarps;
          if (is_g >= groups) {
            is_g -= groups;
            ++is_ar;
          }
        }
      }
    }
    cp_async_commit();
  };
  #pragma unroll 1
  for (int s = 0; s < kDepth - 1; ++s) issue(s);
  // the range's pairs, and every token row of x (FP8: the values of its codes) as bf16
  for (int i = tid; i < R * kGemvMaxM; i += kGvThreads) {
    const int r = i / kGemvMaxM, j = i - r * kGemvMaxM;
    if (j < s_act[r].y) s_pairs[i] = __ldcg(a.padded_pairs + s_act[r].z + j);
  }
  const int vecs = a.H / 8;
  for (int i = tid; i < a.M * vecs; i += kGvThreads) {
    uint4 v;
    if constexpr (kW == kWBf16) v = __ldg(reinterpret_cast<const uint4*>(a.x) + i);
    else v = fp8x8_to_bf16(__ldcg(reinterpret_cast<const uint2*>(a.xq) + i), a.f8);
    reinterpret_cast<uint4*>(xs)[i] = v;
  }
  __syncthreads();
  float sx = 1.f;
  if constexpr (kW != kWBf16) sx = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
  float acc[4][NT][2];   // two chains per (row, token): even and odd K elements
  #pragma unroll
  for (int i = 0; i < 4; ++i)
    #pragma unroll
    for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = 0.f;
  int xo[NT];   // x row offsets (elements) of the current pass's tokens
  int c_ar = ar_first, c_g = g_first, c_pass = 0, c_kb = 0;   // stage being computed
  int n = 0, rec = 0;
  float lmax = 0.f;
  const int kq = (lane & 7) * kEPL;   // the lane's first K element inside a K block
  #pragma unroll 1
  for (int s = 0; s < n_st; ++s) {
    issue(s + kDepth - 1);
    cp_async_wait<kDepth - 1>();
    if (c_kb == 0) {   // a new pass: up to NT of the expert's tokens
      rec = c_ar - a0;
      n = s_act[rec].y - NT * c_pass;
      if (n > NT) n = NT;
      #pragma unroll
      for (int j = 0; j < NT; ++j) xo[j] = j < n ? (s_pairs[rec * kGemvMaxM + NT * c_pass + j] / a.k) * a.H : 0;
    }
    const int d = s % kDepth;
    uint4 wv[4];
    #pragma unroll
    for (int i = 0; i < 4; ++i) wv[i] = *reinterpret_cast<const uint4*>(ring_piece(ring, d, i));
    const int k0 = c_kb * kKPB + kq;
    #pragma unroll
    for (int part = 0; part < kEPL / 8; ++part) {
      float w[4][8];
      #pragma unroll
      for (int i = 0; i < 4; ++i) weights8_f32<kW>(wv[i], part, w[i]);
      #pragma unroll
      for (int j = 0; j < NT; ++j) {
        if (j < n) {
          float xv[8];
          bf16x8_f32(*reinterpret_cast<const uint4*>(xs + xo[j] + k0 + 8 * part), xv);
          #pragma unroll
          for (int i = 0; i < 4; ++i)
            #pragma unroll
            for (int q = 0; q < 8; ++q) acc[i][j][q & 1] = fmaf(w[i][q], xv[q], acc[i][j][q & 1]);
        }
      }
    }
    if (++c_kb == a.kb1) {
      // the pass is complete: the 8 lanes of each row meet, then lane 8q writes h of
      // features f0 + q (gate piece 0, up piece 2) and f0 + q + 4 (pieces 1 and 3)
      c_kb = 0;
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        #pragma unroll
        for (int j = 0; j < NT; ++j) {
          float v = acc[i][j][0] + acc[i][j][1];
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
          acc[i][j][0] = v;
        }
      if ((lane & 7) == 0) {
        float sg = 1.f, su = 1.f;
        if constexpr (kW != kWBf16) {
          const int e = s_act[rec].x;
          sg = __ldg(a.w_scales + e * 3 + 0) * sx;
          su = __ldg(a.w_scales + e * 3 + 1) * sx;
        }
        const int q = lane >> 3;
        const int f0 = c_g * kGuRows;
        #pragma unroll
        for (int j = 0; j < NT; ++j) {
          if (j < n) {
            __nv_bfloat16* hrow = a.h + static_cast<size_t>(s_pairs[rec * kGemvMaxM + NT * c_pass + j]) * a.I + f0 + q;
            #pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
              const __nv_bfloat16 hb = __float2bfloat16_rn(silu_f(acc[hf][j][0] * sg) * (acc[2 + hf][j][0] * su));
              hrow[4 * hf] = hb;
              lmax = fmaxf(lmax, fabsf(__bfloat162float(hb)));
            }
          }
        }
      }
      #pragma unroll
      for (int i = 0; i < 4; ++i)
        #pragma unroll
        for (int j = 0; j < NT; ++j) acc[i][j][0] = acc[i][j][1] = 0.f;
      if (++c_pass == (s_act[rec].y + NT - 1) / NT) {
        c_pass = 0;
        c_g += kGvWarps;
        if (c_g >= groups) {
          c_g -= groups;
          ++c_ar;
        }
      }
    }
  }
  cp_async_wait<0>();   // only empty groups remain; nothing may land after the CTA leaves
  if constexpr (kW != kWBf16) {
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o));
    if (lane == 0 && lmax > 0.f) atomicMax(a.amax + 1, __float_as_uint(lmax));
  }
}

// ------------------------------------------------------------------ down
constexpr int kDnRows = 16;

struct DownSmem {
  size_t part, e, sc, h, total;
  __host__ __device__ DownSmem(int units, int tokens, int k, int I) {
    const size_t slots = (static_cast<size_t>(tokens) * k + 3) & ~size_t(3);
    part = kRingBytes;
    e = part + static_cast<size_t>(units) * kGvWarps * kDnRows * 4;
    sc = e + slots * 4;
    h = sc + slots * 4;
    total = h + static_cast<size_t>(tokens) * k * I * 2;
  }
};

__device__ __forceinline__ void fp8_forward_done(const GemvArgs& a) {
  a.last_scales[0] = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
  a.last_scales[1] = fp8_scale_from_amax(__ldcg(a.amax + 1), a.f8);
  a.amax[0] = 0u;
}

template <int kW>
__global__ void __launch_bounds__(kGvThreads, kCtasPerSm) gemv_down_kernel(GemvArgs a) {
  constexpr int kEPL = WTraits<kW>::kEPL, kKPB = WTraits<kW>::kKPB;
  extern __shared__ __align__(128) uint8_t gv_smem[];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int k = a.k;
  const int fgroups = a.H / kDnRows;
  const int U = a.M * fgroups;
  const int G = gridDim.x, c = blockIdx.x;
  const int u0 = static_cast<int>(static_cast<long long>(c) * U / G);
  const int u1 = static_cast<int>(static_cast<long long>(c + 1) * U / G);
  if (u0 >= u1) {
    pdl_wait();
    pdl_trigger();
    if constexpr (kW != kWBf16)
      if (c == 0 && tid == 0) fp8_forward_done(a);
    return;
  }
  const int t0 = u0 / fgroups;
  const int T = (u1 - 1) / fgroups - t0 + 1;
  const int nu = u1 - u0;
  uint8_t* ring = gv_smem + warp * kRingWarp + lane * 16;
  const DownSmem L(a.dn_units, a.dn_tokens, k, a.I);
  float* part = reinterpret_cast<float*>(gv_smem + L.part);
  int* s_e = reinterpret_cast<int*>(gv_smem + L.e);
  float* s_sc = reinterpret_cast<float*>(gv_smem + L.sc);
  __nv_bfloat16* hs = reinterpret_cast<__nv_bfloat16*>(gv_smem + L.h);
  for (int i = tid; i < T * k; i += kGvThreads) {
    s_e[i] = __ldcg(a.topk_ids + t0 * k + i);
    s_sc[i] = __ldcg(a.topk_w + t0 * k + i);
  }
  for (int i = tid; i < nu * kGvWarps * kDnRows; i += kGvThreads) part[i] = 0.f;
  __syncthreads();
  const uint64_t pol = l2_policy_evict_first();
  const int nj = warp < k ? (k - warp + kGvWarps - 1) / kGvWarps : 0;
  const int n_st = nu * nj * a.kb2;
  // next stage to issue: unit (token is_t, features is_f0), slot is_j, K block is_kb;
  // units advance by one feature group with a carry into the next token
  int is_t = t0, is_f0 = (u0 - t0 * fgroups) * kDnRows, is_j = 0, is_kb = 0;
  auto issue = [&](int s) {
    if (s < n_st) {
      const long long e = s_e[(is_t - t0) * k + warp + kGvWarps * is_j];
      const uint8_t* p = a.wd + (((e * a.et2 + static_cast<long long>(is_f0 >> 7) * a.kb2 + is_kb) * kTileRows) + (is_f0 & 127)) * kRowBytes + lane * 16;
      const int d = s % kDepth;
      #pragma unroll
      for (int i = 0; i < 4; ++i) cp_async16(ring_piece(ring, d, i), p + 512 * i, pol);
      if (++is_kb == a.kb2) {
        is_kb = 0;
        if (++is_j == nj) {
          is_j = 0;
          is_f0 += kDnRows;
          if (is_f0 == a.H) {
            is_f0 = 0;
            ++is_t;
          }
        }
      }
    }
    cp_async_commit();
  };
  #pragma unroll 1
  for (int s = 0; s < kDepth - 1; ++s) issue(s);
  if (a.prefetch_kb > 0) {
    const int pk = a.prefetch_kb < a.kb2 ? a.prefetch_kb : a.kb2;
    for (int i = tid; i < nu * k * pk; i += kGvThreads) {
      const int kb = i % pk, r = i / pk;
      const int j = r % k, u = u0 + r / k;
      const int t = u / fgroups;
      const int f0 = (u - t * fgroups) * kDnRows;
      const long long e = s_e[(t - t0) * k + j];
      prefetch_l2(a.wd + (((e * a.et2 + static_cast<long long>(f0 >> 7) * a.kb2 + kb) * kTileRows) + (f0 & 127)) * kRowBytes,
                  kDnRows * kRowBytes);
    }
  }
  pdl_wait();
  pdl_trigger();
  float s_h = 1.f;
  if constexpr (kW != kWBf16) {
    s_h = fp8_scale_from_amax(__ldcg(a.amax + 1), a.f8);
    for (int i = tid; i < T * k; i += kGvThreads) s_sc[i] = s_sc[i] * (__ldg(a.w_scales + s_e[i] * 3 + 2) * s_h);
    if (c == 0 && tid == 0) fp8_forward_done(a);
  }
  {
    const int vecs = a.I / 8;
    const ScaleDiv dv(s_h);
    const uint4* h8 = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(t0) * k * a.I);
    for (int i = tid; i < T * k * vecs; i += kGvThreads) {
      uint4 v = __ldcg(h8 + i);
      if constexpr (kW != kWBf16) {
        float f[8];
        bf16x8_f32(v, f);
        v = fp8x8_to_bf16(codes8(f, dv, a.f8), a.f8);
      }
      reinterpret_cast<uint4*>(hs)[i] = v;
    }
  }
  __syncthreads();
  float acc[4] = {0.f, 0.f, 0.f, 0.f}, y[4][2] = {{0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}, {0.f, 0.f}};
  int ui = 0, jj = 0, kb = 0, t = t0, fg = u0 - t0 * fgroups;   // stage being computed
  const int kq = (lane & 7) * kEPL;
  #pragma unroll 1
  for (int s = 0; s < n_st; ++s) {
    issue(s + kDepth - 1);
    cp_async_wait<kDepth - 1>();
    const int slot = (t - t0) * k + warp + kGvWarps * jj;
    const int d = s % kDepth;
    uint4 wv[4];
    #pragma unroll
    for (int i = 0; i < 4; ++i) wv[i] = *reinterpret_cast<const uint4*>(ring_piece(ring, d, i));
    const __nv_bfloat16* hrow = hs + static_cast<size_t>(slot) * a.I + kb * kKPB + kq;
    #pragma unroll
    for (int p8 = 0; p8 < kEPL / 8; ++p8) {
      float hv[8];
      bf16x8_f32(*reinterpret_cast<const uint4*>(hrow + 8 * p8), hv);
      #pragma unroll
      for (int r = 0; r < 4; ++r) {
        float w[8];
        weights8_f32<kW>(wv[r], p8, w);
        #pragma unroll
        for (int q = 0; q < 8; ++q) y[r][q & 1] = fmaf(w[q], hv[q], y[r][q & 1]);
      }
    }
    if (++kb == a.kb2) {
      kb = 0;
      const float sc = s_sc[slot];
      #pragma unroll
      for (int r = 0; r < 4; ++r) {
        acc[r] = fmaf(sc, y[r][0] + y[r][1], acc[r]);
        y[r][0] = y[r][1] = 0.f;
      }
      if (++jj == nj) {
        jj = 0;
        #pragma unroll
        for (int r = 0; r < 4; ++r) {
          float v = acc[r];
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 4);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 2);
          v += __shfl_xor_sync(0xFFFFFFFFu, v, 1);
          acc[r] = 0.f;
          if ((lane & 7) == 0) part[(ui * kGvWarps + warp) * kDnRows + (lane >> 3) + 4 * r] = v;
        }
        ++ui;
        if (++fg == fgroups) {
          fg = 0;
          ++t;
        }
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  for (int i = tid; i < nu * kDnRows; i += kGvThreads) {
    const int uu = i / kDnRows, row = i - uu * kDnRows;
    float sum = 0.f;
    #pragma unroll
    for (int w = 0; w < kGvWarps; ++w) sum += part[(uu * kGvWarps + w) * kDnRows + row];
    const int u = u0 + uu;
    const int t = u / fgroups;
    a.out[static_cast<size_t>(t) * a.H + (u - t * fgroups) * kDnRows + row] = __float2bfloat16_rn(sum);
  }
}

size_t gate_up_smem(int M, int H) { return kRingBytes + static_cast<size_t>(M) * H * 2; }
size_t down_smem(int units, int tokens, int k, int I) { return DownSmem(units, tokens, k, I).total; }
constexpr size_t kGvSmemMax = 220 * 1024;

void down_shape(int M, int H, int sms, int& units, int& tokens) {
  const int fgroups = H / kDnRows;
  const long long U = static_cast<long long>(M) * fgroups;
  units = static_cast<int>((U + sms - 1) / sms);
  tokens = std::min(M, (units - 1) / fgroups + 2);
}

template <int kW>
cudaError_t launch_gate_up_fmt(const GemvArgs& a, cudaStream_t s) {
  const dim3 grid(a.grid), block(kGvThreads);
  return launch_kernel(gemv_gate_up_kernel<kW>, grid, block, gate_up_smem(a.M, a.H), s, a);
}

template <int kW>
cudaError_t launch_down_fmt(const GemvArgs& a, cudaStream_t s) {
  const dim3 grid(a.grid), block(kGvThreads);
  const size_t smem = down_smem(a.dn_units, a.dn_tokens, a.k, a.I);
  return launch_kernel(gemv_down_kernel<kW>, grid, block, smem, s, a);
}

template <int kW>
cudaError_t configure_fmt() {
  cudaError_t e;
  const int mx = static_cast<int>(kGvSmemMax);
  if ((e = cudaFuncSetAttribute(gemv_gate_up_kernel<kW>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx))) return e;
  return cudaFuncSetAttribute(gemv_down_kernel<kW>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}

}  // namespace

bool gemv_supported(int M, int E, int k, int H, int I, int sms) {
  if (M < 1 || M > kGemvMaxM || k > 16 || E > 512 || sms < 1) return false;
  sms *= kCtasPerSm;
  const long long groups = I / kGuRows;
  const long long U = std::min<long long>(E, static_cast<long long>(M) * k) * groups;
  const long long per_cta = (U + sms - 1) / sms;
  if ((per_cta - 1) / groups + 2 > kGuMaxExperts) return false;
  int units, tokens;
  down_shape(M, H, sms, units, tokens);
  return gate_up_smem(M, H) <= kGvSmemMax && down_smem(units, tokens, k, I) <= kGvSmemMax;
}

size_t gemv_down_plan(GemvArgs& a, int sms) {
  sms *= kCtasPerSm;
  a.grid = sms;
  down_shape(a.M, a.H, sms, a.dn_units, a.dn_tokens);
  return down_smem(a.dn_units, a.dn_tokens, a.k, a.I);
}

cudaError_t gemv_configure() {
  cudaError_t e;
  if ((e = configure_fmt<kWBf16>())) return e;
  if ((e = configure_fmt<kWE4M3>())) return e;
  return configure_fmt<kWE5M2>();
}

cudaError_t launch_gemv_plan(const GemvArgs& a, cudaStream_t s) {
  const dim3 g(1), b(kPlanThreads);
  if (a.E <= 32) return launch_kernel(gemv_plan_kernel<1>, g, b, 0, s, a);
  if (a.E <= 64) return launch_kernel(gemv_plan_kernel<2>, g, b, 0, s, a);
  if (a.E <= 128) return launch_kernel(gemv_plan_kernel<4>, g, b, 0, s, a);
  if (a.E <= 256) return launch_kernel(gemv_plan_kernel<8>, g, b, 0, s, a);
  return launch_kernel(gemv_plan_kernel<16>, g, b, 0, s, a);
}

cudaError_t launch_gemv_gate_up(const GemvArgs& a, int fmt, cudaStream_t s) {
  if (fmt == kWE4M3) return launch_gate_up_fmt<kWE4M3>(a, s);
  if (fmt == kWE5M2) return launch_gate_up_fmt<kWE5M2>(a, s);
  return launch_gate_up_fmt<kWBf16>(a, s);
}

cudaError_t launch_gemv_down(const GemvArgs& a, int fmt, cudaStream_t s) {
  if (fmt == kWE4M3) return launch_down_fmt<kWE4M3>(a, s);
  if (fmt == kWE5M2) return launch_down_fmt<kWE5M2>(a, s);
  return launch_down_fmt<kWBf16>(a, s);
}

}  // namespace moe
