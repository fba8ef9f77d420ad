// kernels_gemv.cu - the MoE layer for thin batches (up to 16 tokens).
//
// At decode sizes an expert receives one or two tokens: each weight byte then feeds one
// or two multiply-adds, about 1 FLOP per byte, two orders of magnitude below the
// tensor cores' ridge, and the time of the layer is the time to stream the active
// experts' weights. What the tcgen05 chain adds on top of that streaming is latency: an
// align launch, a gather, split-K partial sums (a 128-row weight tile over the whole
// reduction is more bytes than one SM should stream alone), and a finalize. This path
// runs the same arithmetic as three launches:
//   plan     route every token (the top-k rule of route_common.cuh), group the pairs
//            by expert (the align kernel's padded groups, kept for inspection) and
//            list the active experts; FP8: amax(x), s_x and the x codes;
//   gate_up  units of (active expert, 8 intermediate features) spread over the warps of
//            two CTAs per SM: 8 W_gate and 8 W_up rows times the expert's tokens, h =
//            silu(g) * u stored bf16 by pair; FP8: max|h| into the amax word;
//   down     units of (token, 16 output features): the token's k experts' W_down rows
//            times their h rows, weighted by the routing weights and summed in fp32,
//            written to `out` as bf16 (no atomics, no finalize).
// The routing, the movement of tokens and the combination of the experts' outputs cost
// work around the matrix products, and fusing them cuts the number of GPU operations
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels"). On Hopper the thin-batch answer was Swap-AB on
// the tensor cores (aib.vote, "AWS SageMaker MoE kernel optimizations", second
// paragraph); the tcgen05 chain keeps it for wider batches, and this path replaces it
// where the product is a matrix-vector product.
//
// The weight rows of a unit are the 16 rows (M) of warp-level tensor-core products
// (mma.sync m16n8k16 on bf16, m16n8k32 on e4m3 / e5m2 codes): one instruction takes a
// 16 x 32-byte slice of the weights, where a multiply-add per weight element would take
// dozens, so a warp's instruction stream keeps up with the bytes it streams. The
// tokens (up to 8) are the N of the product, and the activations (bf16 values or FP8
// codes, exactly the operands of the tcgen05 chain's MMAs) sit in shared memory.
// Products accumulate in fp32; FP8 scales are applied as in the chain's epilogues
// (s_gate*s_x, s_up*s_x, routing weight * s_down * s_h).
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

// 8 bf16 values (16 bytes of shared memory) -> fp32.
__device__ __forceinline__ void bf16x8_f32(const uint4& u, float* f) {
  const unsigned w[4] = {u.x, u.y, u.z, u.w};
  #pragma unroll
  for (int q = 0; q < 4; ++q) {
    f[2 * q] = __uint_as_float(w[q] << 16);
    f[2 * q + 1] = __uint_as_float(w[q] & 0xFFFF0000u);
  }
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


// ------------------------------------------------------------------ streaming
// Each warp streams its unit's weights through a ring of kDepth stages in shared memory
// with cp.async (L2 -> shared, no registers held while in flight). A stage is one
// 128-byte K block of the unit's 16 weight rows (2 KB); every lane copies four 16-byte
// pieces of it, chunk c of row R landing at R*128 + ((c ^ (R & 7)) * 16), so that the
// ldmatrix loads of the tensor-core fragments read eight rows of one chunk from eight
// different bank groups. Per iteration a warp waits for its oldest stage, meets at a
// warp barrier (its lanes' copies of that stage landed; their reads of the stage
// refilled next are done), issues the next stage and multiplies. Two CTAs of 8 warps per
// SM keep 16 x (kD - 1) x 2 KB of weights in flight per SM.
constexpr int kCtasPerSm = 2;
constexpr int kStageWarp = 16 * kRowBytes;           // bytes of one stage of one warp
// ring depth kD (4..6 stages: 8-12 KB per warp, 64-96 KB per CTA), the deepest that lets
// two CTAs share an SM next to the batch's activation rows
template <int kD>
struct Ring {
  static constexpr int kWarp = kD * kStageWarp;
  static constexpr int kBytes = kGvWarps * kWarp;
};

__device__ __forceinline__ void cp_async16(uint32_t smem_dst, const void* src, uint64_t pol) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_dst), "l"(src), "l"(pol)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

// Byte offset, inside a stage, of chunk c (16 bytes) of row R (128 bytes).
__device__ __forceinline__ uint32_t swz(int R, int c) { return R * kRowBytes + ((c ^ (R & 7)) << 4); }

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr)
               : "memory");
}
__device__ __forceinline__ void ldsm_x2(uint32_t addr, uint32_t (&r)[2]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0, %1}, [%2];" : "=r"(r[0]), "=r"(r[1]) : "r"(addr) : "memory");
}

// d (16 x 8, fp32) += a (16 rows x one K step) * b (one K step x 8 columns): a K step is
// 16 bf16 values, or 32 e4m3 / e5m2 codes, of every row (the product of two codes is
// exact in fp32, as in the tensor-core chain's kind::f8f6f4).
template <int kW>
__device__ __forceinline__ void mma_step(float (&d)[4], const uint32_t (&a)[4], const uint32_t (&b)[2]) {
  if constexpr (kW == kWBf16)
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  else if constexpr (kW == kWE4M3)
    asm volatile("mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
  else
    asm volatile("mma.sync.aligned.m16n8k32.row.col.f32.e5m2.e5m2.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
                 "{%0, %1, %2, %3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Activation rows in shared memory: bf16 values (bf16 layers) or FP8 codes, each row
// padded by 16 bytes so that ldmatrix's eight rows fall into different bank groups.
template <int kW>
struct ActRows {
  static constexpr int kEl = kW == kWBf16 ? 2 : 1;
  __host__ __device__ static int stride(int len) { return len * kEl + 16; }   // bytes
};

// ------------------------------------------------------------------ gate_up
// Units (a, g): active expert a, W_gate rows [8g, 8g + 8) and the W_up rows of the same
// features (the 16 rows of one MMA: gate rows 0..7, up rows 8..15), over the whole
// reduction, times the expert's tokens in passes of up to 8 (the MMA's N). CTA c takes
// the contiguous range [c*U/G, (c+1)*U/G) of the U = A*I/8 units (one or a few experts,
// whose pairs it keeps in shared memory with every token row of x: bf16, or FP8 codes);
// warp w takes units w, w + 8, ... of the range, K block after K block. A lane's
// accumulators hold gate and up of the same feature for two tokens, so SwiGLU needs no
// exchange. Unit positions advance by 8 groups with a carry into the next expert (I/8 >=
// 16 groups per expert).
constexpr int kGuMaxExperts = 16;   // experts one CTA's range may span (host-checked)
constexpr int kGuTokens = 8;        // tokens per pass: the N of one MMA

template <int kW, int kD>
__global__ void __launch_bounds__(kGvThreads, kCtasPerSm) gemv_gate_up_kernel(GemvArgs a) {
  constexpr int NT = kGuTokens;
  constexpr int kDepth = kD;
  constexpr int kRingWarp = Ring<kD>::kWarp, kRingBytes = Ring<kD>::kBytes;
  extern __shared__ __align__(128) uint8_t gv_smem[];
  __shared__ int4 s_act[kGuMaxExperts];
  __shared__ int s_pairs[kGuMaxExperts * kGemvMaxM];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const uint32_t ring = smem_u32(gv_smem) + warp * kRingWarp;
  uint8_t* xs = gv_smem + kRingBytes;                  // [M + 1][xstride]: token rows, a zero row
  const int xstride = ActRows<kW>::stride(a.H);
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
  // this lane's four pieces of a stage: rows 4i + lane/8, chunk lane % 8
  uint32_t dst[4];
  #pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = swz(4 * i + (lane >> 3), lane & 7);
  int is_ar = ar_first, is_g = g_first, is_pass = 0, is_kb = 0;   // next stage to issue
  auto issue = [&](int s) {
    if (s < n_st) {
      const long long e = s_act[is_ar - a0].x;
      const int f0 = is_g * kGuRows;
      const long long base = e * a.et1 + is_kb;
      const uint8_t* pg = a.w13 + ((base + static_cast<long long>(f0 >> 7) * a.kb1) * kTileRows + (f0 & 127)) * kRowBytes + lane * 16;
      const uint8_t* pu = a.w13 + ((base + static_cast<long long>((a.I + f0) >> 7) * a.kb1) * kTileRows + (f0 & 127)) * kRowBytes + lane * 16;
      const uint32_t slot = ring + (s % kDepth) * kStageWarp;
      cp_async16(slot + dst[0], pg, pol);
      cp_async16(slot + dst[1], pg + 512, pol);
      cp_async16(slot + dst[2], pu, pol);
      cp_async16(slot + dst[3], pu + 512, pol);
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
  // the range's pairs, every token row of x (bf16, or its FP8 codes) and a zero row
  for (int i = tid; i < R * kGemvMaxM; i += kGvThreads) {
    const int r = i / kGemvMaxM, j = i - r * kGemvMaxM;
    if (j < s_act[r].y) s_pairs[i] = __ldcg(a.padded_pairs + s_act[r].z + j);
  }
  {
    const int rowv = a.H * ActRows<kW>::kEl / 16;   // 16-byte vectors of a row
    const uint4* src = kW == kWBf16 ? reinterpret_cast<const uint4*>(a.x) : reinterpret_cast<const uint4*>(a.xq);
    for (int i = tid; i < (a.M + 1) * rowv; i += kGvThreads) {
      const int m = i / rowv, v = i - m * rowv;
      uint4 val = make_uint4(0u, 0u, 0u, 0u);
      if (m < a.M) val = kW == kWBf16 ? __ldg(src + i) : __ldcg(src + i);
      *reinterpret_cast<uint4*>(xs + m * xstride + v * 16) = val;
    }
  }
  __syncthreads();
  float sx = 1.f;
  if constexpr (kW != kWBf16) sx = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
  const uint32_t xbase = smem_u32(xs);
  const uint32_t zero_row = xbase + a.M * xstride;
  const int a_row = lane & 15, a_hi = lane >> 4;        // A fragments: row, second chunk
  const int b_tok = lane & 7, b_hi = (lane >> 3) & 1;   // B fragments: token, second chunk
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  uint32_t brow = zero_row;   // this lane's token row of the current pass
  int c_ar = ar_first, c_g = g_first, c_pass = 0, c_kb = 0;   // stage being computed
  int n = 0, rec = 0;
  float lmax = 0.f;
  #pragma unroll 1
  for (int s = 0; s < n_st; ++s) {
    cp_async_wait<kDepth - 2>();
    __syncwarp();
    issue(s + kDepth - 1);
    if (c_kb == 0) {   // a new pass: up to NT of the expert's tokens
      rec = c_ar - a0;
      n = s_act[rec].y - NT * c_pass;
      if (n > NT) n = NT;
      brow = b_tok < n ? xbase + (s_pairs[rec * kGemvMaxM + NT * c_pass + b_tok] / a.k) * xstride : zero_row;
    }
    const uint32_t slot = ring + (s % kDepth) * kStageWarp;
    #pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[4], bf[2];
      ldsm_x4(slot + swz(a_row, 2 * ks + a_hi), af);
      ldsm_x2(brow + (c_kb * 8 + 2 * ks + b_hi) * 16, bf);
      mma_step<kW>(d, af, bf);
    }
    if (++c_kb == a.kb1) {
      // the pass is complete: lane (g, t) holds gate and up of feature f0 + g for the
      // pass's tokens 2t and 2t + 1
      c_kb = 0;
      float sg = 1.f, su = 1.f;
      if constexpr (kW != kWBf16) {
        const int e = s_act[rec].x;
        sg = __ldg(a.w_scales + e * 3 + 0) * sx;
        su = __ldg(a.w_scales + e * 3 + 1) * sx;
      }
      const int g = lane >> 2, t2 = 2 * (lane & 3);
      const int f = c_g * kGuRows + g;
      #pragma unroll
      for (int q = 0; q < 2; ++q) {
        if (t2 + q < n) {
          const __nv_bfloat16 hb = __float2bfloat16_rn(silu_f(d[q] * sg) * (d[2 + q] * su));
          a.h[static_cast<size_t>(s_pairs[rec * kGemvMaxM + NT * c_pass + t2 + q]) * a.I + f] = hb;
          lmax = fmaxf(lmax, fabsf(__bfloat162float(hb)));
        }
      }
      d[0] = d[1] = d[2] = d[3] = 0.f;
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
// Units (t, f): token t, output features [16f, 16f + 16) (the 16 rows of one MMA). CTA c
// takes the contiguous range [c*U/G, (c+1)*U/G) of the U = M*H/16 units (a token or two,
// whose routing and h rows it keeps in shared memory: bf16, or the codes of h under s_h
// for FP8). Warp w takes the slots j = w, w + 8 (k <= 16) of every unit of the range: it
// streams the 16 W_down rows of expert e_j over the whole reduction and multiplies them
// by h of pair t*k + j (column 0 of the MMA; the other columns read a zero row). The
// slot's sums, weighted by the routing weight (FP8: * s_down * s_h), meet in shared
// memory when the range is done: out[t, f] in bf16, no atomics. The routing comes from
// the route kernel, two launches back, so the first stages of weights stream in before
// the wait for gate_up.
constexpr int kDnRows = 16;

// Byte offsets of the down kernel's shared memory regions (each 16-byte aligned).
struct DownSmem {
  size_t part, e, sc, h, total;
  __host__ __device__ DownSmem(int units, int tokens, int k, int hstride, int ring_bytes) {
    const size_t slots = (static_cast<size_t>(tokens) * k + 3) & ~size_t(3);
    part = ring_bytes;
    e = part + static_cast<size_t>(units) * kGvWarps * kDnRows * 4;
    sc = e + slots * 4;
    h = sc + slots * 4;
    total = h + (static_cast<size_t>(tokens) * k + 1) * hstride;   // + a zero row
  }
};

__device__ __forceinline__ void fp8_forward_done(const GemvArgs& a) {
  a.last_scales[0] = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
  a.last_scales[1] = fp8_scale_from_amax(__ldcg(a.amax + 1), a.f8);
  a.amax[0] = 0u;
}

template <int kW, int kD>
__global__ void __launch_bounds__(kGvThreads, kCtasPerSm) gemv_down_kernel(GemvArgs a) {
  constexpr int kDepth = kD;
  constexpr int kRingWarp = Ring<kD>::kWarp;
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
  const int hstride = ActRows<kW>::stride(a.I);
  const uint32_t ring = smem_u32(gv_smem) + warp * kRingWarp;
  const DownSmem L(a.dn_units, a.dn_tokens, k, hstride, Ring<kD>::kBytes);
  float* part = reinterpret_cast<float*>(gv_smem + L.part);    // [units][8 warps][16]
  int* s_e = reinterpret_cast<int*>(gv_smem + L.e);            // [tokens * k]
  float* s_sc = reinterpret_cast<float*>(gv_smem + L.sc);      // [tokens * k]
  uint8_t* hs = gv_smem + L.h;                                 // [tokens * k + 1][hstride]
  for (int i = tid; i < T * k; i += kGvThreads) {
    s_e[i] = __ldcg(a.topk_ids + t0 * k + i);
    s_sc[i] = __ldcg(a.topk_w + t0 * k + i);
  }
  for (int i = tid; i < nu * kGvWarps * kDnRows; i += kGvThreads) part[i] = 0.f;
  __syncthreads();
  const uint64_t pol = l2_policy_evict_first();
  const int nj = warp < k ? (k - warp + kGvWarps - 1) / kGvWarps : 0;
  const int n_st = nu * nj * a.kb2;
  uint32_t dst[4];
  #pragma unroll
  for (int i = 0; i < 4; ++i) dst[i] = swz(4 * i + (lane >> 3), lane & 7);
  // next stage to issue: unit (token is_t, features is_f0), slot is_j, K block is_kb;
  // units advance by one feature group with a carry into the next token
  int is_t = t0, is_f0 = (u0 - t0 * fgroups) * kDnRows, is_j = 0, is_kb = 0;
  auto issue = [&](int s) {
    if (s < n_st) {
      const long long e = s_e[(is_t - t0) * k + warp + kGvWarps * is_j];
      const uint8_t* p = a.wd + (((e * a.et2 + static_cast<long long>(is_f0 >> 7) * a.kb2 + is_kb) * kTileRows) + (is_f0 & 127)) * kRowBytes + lane * 16;
      const uint32_t slot = ring + (s % kDepth) * kStageWarp;
      #pragma unroll
      for (int i = 0; i < 4; ++i) cp_async16(slot + dst[i], p + 512 * i, pol);
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
    // L2 requests for the first K blocks of every (unit, slot) of the range, while gate_up
    // may still be running
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
  // h rows of the range's pairs (t0*k ...), written by gate_up: read from L2; FP8: their
  // codes under s_h; then a zero row
  {
    const int vecs = a.I / 8;   // 8 values per step
    const ScaleDiv dv(s_h);
    const uint4* h8 = reinterpret_cast<const uint4*>(a.h + static_cast<size_t>(t0) * k * a.I);
    for (int i = tid; i < T * k * vecs; i += kGvThreads) {
      const int r = i / vecs, v = i - r * vecs;
      const uint4 x = __ldcg(h8 + i);
      if constexpr (kW == kWBf16) {
        *reinterpret_cast<uint4*>(hs + r * hstride + v * 16) = x;
      } else {
        float f[8];
        bf16x8_f32(x, f);
        *reinterpret_cast<uint2*>(hs + r * hstride + v * 8) = codes8(f, dv, a.f8);
      }
    }
    for (int i = tid; i < hstride / 16; i += kGvThreads)
      *reinterpret_cast<uint4*>(hs + T * k * hstride + i * 16) = make_uint4(0u, 0u, 0u, 0u);
  }
  __syncthreads();
  const uint32_t hbase = smem_u32(hs);
  const uint32_t zero_row = hbase + T * k * hstride;
  const int a_row = lane & 15, a_hi = lane >> 4;
  const int b_hi = (lane >> 3) & 1;
  float d[4] = {0.f, 0.f, 0.f, 0.f};
  float acc0 = 0.f, acc1 = 0.f;   // lane (g, 0): features f0 + g and f0 + g + 8 of the unit
  int ui = 0, jj = 0, kb = 0, t = t0;
  int slot = 0;
  uint32_t brow = zero_row;
  #pragma unroll 1
  for (int s = 0; s < n_st; ++s) {
    cp_async_wait<kDepth - 2>();
    __syncwarp();
    issue(s + kDepth - 1);
    if (kb == 0) {   // a new (unit, slot): column 0 is h of its pair
      slot = (t - t0) * k + warp + kGvWarps * jj;
      brow = (lane & 7) == 0 ? hbase + slot * hstride : zero_row;
    }
    const uint32_t sl = ring + (s % kDepth) * kStageWarp;
    #pragma unroll
    for (int ks = 0; ks < 4; ++ks) {
      uint32_t af[4], bf[2];
      ldsm_x4(sl + swz(a_row, 2 * ks + a_hi), af);
      ldsm_x2(brow + (kb * 8 + 2 * ks + b_hi) * 16, bf);
      mma_step<kW>(d, af, bf);
    }
    if (++kb == a.kb2) {   // the slot is complete: column 0, weighted
      kb = 0;
      const float sc = s_sc[slot];
      acc0 = fmaf(sc, d[0], acc0);
      acc1 = fmaf(sc, d[2], acc1);
      d[0] = d[1] = d[2] = d[3] = 0.f;
      if (++jj == nj) {   // the warp's last slot of the unit
        jj = 0;
        if ((lane & 3) == 0) {
          part[(ui * kGvWarps + warp) * kDnRows + (lane >> 2)] = acc0;
          part[(ui * kGvWarps + warp) * kDnRows + (lane >> 2) + 8] = acc1;
        }
        acc0 = acc1 = 0.f;
        ++ui;
        if ((u0 + ui) % fgroups == 0) ++t;
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
    const int tt = u / fgroups;
    a.out[static_cast<size_t>(tt) * a.H + (u - tt * fgroups) * kDnRows + row] = __float2bfloat16_rn(sum);
  }
}

// Activation row stride in shared memory: the row plus 16 bytes (el: bytes per value).
int act_stride(int len, int el) { return len * el + 16; }
size_t gate_up_smem(int M, int H, int el, int depth) {
  return static_cast<size_t>(kGvWarps) * depth * kStageWarp + static_cast<size_t>(M + 1) * act_stride(H, el);
}
size_t down_smem(int units, int tokens, int k, int I, int el, int depth) {
  return DownSmem(units, tokens, k, act_stride(I, el), kGvWarps * depth * kStageWarp).total;
}
// dynamic shared memory of one CTA at most
constexpr size_t kGvSmemMax = 220 * 1024;
// dynamic shared memory of one CTA when two share an SM (228 KB per SM, 1 KB reserved per
// CTA, the kernels' static arrays)
constexpr size_t kTwoPerSm = 111 * 1024;

// The deepest ring (4..6 stages) that keeps two CTAs per SM, given the smem of a depth.
template <class F>
int pick_depth(F smem_at) {
  for (int d = 6; d > 4; --d)
    if (smem_at(d) <= kTwoPerSm) return d;
  return 4;
}

void down_shape(int M, int H, int sms, int& units, int& tokens) {
  const int fgroups = H / kDnRows;
  const long long U = static_cast<long long>(M) * fgroups;
  units = static_cast<int>((U + sms - 1) / sms);
  tokens = std::min(M, (units - 1) / fgroups + 2);
}

template <int kW>
cudaError_t launch_gate_up_fmt(const GemvArgs& a, cudaStream_t s) {
  const dim3 grid(a.grid), block(kGvThreads);
  const int el = ActRows<kW>::kEl;
  const int d = pick_depth([&](int dd) { return gate_up_smem(a.M, a.H, el, dd); });
  const size_t smem = gate_up_smem(a.M, a.H, el, d);
  if (d == 6) return launch_kernel(gemv_gate_up_kernel<kW, 6>, grid, block, smem, s, a);
  if (d == 5) return launch_kernel(gemv_gate_up_kernel<kW, 5>, grid, block, smem, s, a);
  return launch_kernel(gemv_gate_up_kernel<kW, 4>, grid, block, smem, s, a);
}

template <int kW>
cudaError_t launch_down_fmt(const GemvArgs& a, cudaStream_t s) {
  const dim3 grid(a.grid), block(kGvThreads);
  const int el = ActRows<kW>::kEl;
  const int d = pick_depth([&](int dd) { return down_smem(a.dn_units, a.dn_tokens, a.k, a.I, el, dd); });
  const size_t smem = down_smem(a.dn_units, a.dn_tokens, a.k, a.I, el, d);
  if (d == 6) return launch_kernel(gemv_down_kernel<kW, 6>, grid, block, smem, s, a);
  if (d == 5) return launch_kernel(gemv_down_kernel<kW, 5>, grid, block, smem, s, a);
  return launch_kernel(gemv_down_kernel<kW, 4>, grid, block, smem, s, a);
}

template <int kW, int kD>
cudaError_t configure_one() {
  cudaError_t e;
  const int mx = static_cast<int>(kGvSmemMax);
  if ((e = cudaFuncSetAttribute(gemv_gate_up_kernel<kW, kD>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx)))
    return e;
  return cudaFuncSetAttribute(gemv_down_kernel<kW, kD>, cudaFuncAttributeMaxDynamicSharedMemorySize, mx);
}

template <int kW>
cudaError_t configure_fmt() {
  cudaError_t e;
  if ((e = configure_one<kW, 4>())) return e;
  if ((e = configure_one<kW, 5>())) return e;
  return configure_one<kW, 6>();
}

}  // namespace

bool gemv_supported(int M, int E, int k, int H, int I, int sms, bool fp8) {
  const int el = fp8 ? 1 : 2;
  if (M < 1 || M > kGemvMaxM || k > 16 || E > 512 || sms < 1) return false;
  sms *= kCtasPerSm;
  const long long groups = I / kGuRows;
  const long long U = std::min<long long>(E, static_cast<long long>(M) * k) * groups;
  const long long per_cta = (U + sms - 1) / sms;
  if ((per_cta - 1) / groups + 2 > kGuMaxExperts) return false;
  int units, tokens;
  down_shape(M, H, sms, units, tokens);
  return gate_up_smem(M, H, el, 4) <= kGvSmemMax && down_smem(units, tokens, k, I, el, 4) <= kGvSmemMax;
}

size_t gemv_down_plan(GemvArgs& a, int sms) {
  sms *= kCtasPerSm;
  a.grid = sms;
  down_shape(a.M, a.H, sms, a.dn_units, a.dn_tokens);
  return down_smem(a.dn_units, a.dn_tokens, a.k, a.I, a.xq != nullptr ? 1 : 2, 4);
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
