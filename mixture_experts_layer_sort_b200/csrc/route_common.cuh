// route_common.cuh - device helpers shared by the router/align kernels and the
// single-launch decode kernel: per-token top-k routing, a warp-wide exclusive scan
// and the split-K choice.
//
// Routing: "a token usually activates only a selected subset" of the experts
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels"). A token keeps its k largest logits (equal
// logits go to the lower expert id) and weights them by their softmax renormalised
// over the selection.
#pragma once

#include "moe_internal.h"

namespace moe {

// Orderable 32-bit key of a logit: larger key = larger logit, -0.0 equal to +0.0,
// NaN (key 1) below -inf (key 0x007FFFFF); key 0 means "no candidate".
__device__ __forceinline__ unsigned route_key(float v) {
  if (v != v) return 1u;
  unsigned b = __float_as_uint(v);
  if (v == 0.0f) b = 0u;
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}

__device__ __forceinline__ float key_logit(unsigned key) {
  if (key == 1u) return __uint_as_float(0x7FC00000u);
  return __uint_as_float((key & 0x80000000u) ? (key & 0x7FFFFFFFu) : ~key);
}

// One warp routes one token: lane l holds logits l, l+32, ... (NPL of them). Each of
// the k picks takes the largest key over the warp (redux max), then the lowest expert
// id holding that key (redux min); the owning lane then rescans its own few logits.
// Lanes j < k write ids[j] and w[j].
template <int NPL>
__device__ __forceinline__ void route_token(const float* row, int E, int k, int lane, int* ids, float* w) {
  unsigned key[NPL];
  #pragma unroll
  for (int i = 0; i < NPL; ++i) {
    const int e = lane + 32 * i;
    key[i] = (e < E) ? route_key(row[e]) : 0u;
  }
  unsigned best = 0u;
  int best_i = 0;
  #pragma unroll
  for (int i = 0; i < NPL; ++i)
    if (key[i] > best) {
      best = key[i];
      best_i = i;
    }
  int my_id = 0;
  float my_logit = 0.f;
  for (int j = 0; j < k; ++j) {
    const unsigned vmax = __reduce_max_sync(0xFFFFFFFFu, best);
    const unsigned cand = (best == vmax) ? static_cast<unsigned>(lane + 32 * best_i) : 0xFFFFFFFFu;
    const int id = static_cast<int>(__reduce_min_sync(0xFFFFFFFFu, cand));
    if (lane == j) {
      my_id = id;
      my_logit = key_logit(vmax);
    }
    if ((id & 31) == lane) {        // this lane's best was taken: rescan its logits
      #pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (i == best_i) key[i] = 0u;
      best = 0u;
      best_i = 0;
      #pragma unroll
      for (int i = 0; i < NPL; ++i)
        if (key[i] > best) {
          best = key[i];
          best_i = i;
        }
    }
  }
  // slot 0 holds the largest selected logit. When it is -inf, every logit of the
  // row is -inf (or NaN): the row takes the limit of k equal logits, weight 1/k each.
  const float lmax = __shfl_sync(0xFFFFFFFFu, my_logit, 0);
  const bool no_finite = lmax == __uint_as_float(0xFF800000u) || lmax != lmax;
  const float ex = (lane < k) ? (no_finite ? 1.f : expf(my_logit - lmax)) : 0.f;
  float sum = ex;
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(0xFFFFFFFFu, sum, o);
  if (lane < k) {
    ids[lane] = my_id;
    w[lane] = ex / sum;
  }
}

// route_token for any E <= 512 (NPL = logits per lane chosen at run time).
__device__ __forceinline__ void route_token_any(const float* row, int E, int k, int lane, int* ids, float* w) {
  if (E <= 32) route_token<1>(row, E, k, lane, ids, w);
  else if (E <= 64) route_token<2>(row, E, k, lane, ids, w);
  else if (E <= 128) route_token<4>(row, E, k, lane, ids, w);
  else if (E <= 256) route_token<8>(row, E, k, lane, ids, w);
  else route_token<16>(row, E, k, lane, ids, w);
}

constexpr int kSplitOverhead = 2;   // per-unit fixed cost, in K-block equivalents

// Split-K factor of one GEMM, chosen by a whole warp: lane l prices s = l + 1 in
// bytes moved per SM: waves(tiles * s over the SMs) * (K blocks per split + 2) *
// bytes of a K block, plus, for a split, the partial sums it adds to and (gate_up)
// reads back from memory. The cheapest (smallest s on ties) wins; s = 1 when
// splitting is not allowed.
__device__ __forceinline__ int choose_splits_warp(int tiles, int kblocks, int sms, bool allow, int kblock_bytes,
                                  int split_bytes, int lane) {
  const int smax = min(allow ? kMaxSplits : 1, kblocks);
  unsigned long long cost = ~0ull;
  const int s = lane + 1;
  if (tiles > 0 && s <= smax) {
    const unsigned units = static_cast<unsigned>(tiles) * static_cast<unsigned>(s);
    const unsigned waves = (units + sms - 1) / static_cast<unsigned>(sms);
    const unsigned long long per_unit =
        static_cast<unsigned long long>((kblocks + s - 1) / s + kSplitOverhead) * kblock_bytes +
        (s > 1 ? static_cast<unsigned long long>(split_bytes) : 0ull);
    cost = waves * per_unit;
  }
  unsigned long long best = cost;
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long other = __shfl_xor_sync(0xFFFFFFFFu, best, o);
    best = other < best ? other : best;
  }
  const unsigned pick = __reduce_min_sync(0xFFFFFFFFu, cost == best ? static_cast<unsigned>(s) : 0xFFFFFFFFu);
  return (tiles > 0 && best != ~0ull) ? static_cast<int>(pick) : 1;
}

// Exclusive scan of in[0..n) by one warp into out[0..n), the total into out[n]; out
// may be in (each lane reads an element of its own chunk before writing it).
__device__ __forceinline__ void warp_exclusive_scan(const int* in, int* out, int n, int lane) {
  const int chunk = (n + 31) / 32;
  const int lo = lane * chunk;
  const int hi = min(n, lo + chunk);
  int local = 0;
  for (int i = lo; i < hi; ++i) local += in[i];
  int incl = local;
  #pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += y;
  }
  int run = incl - local;
  for (int i = lo; i < hi; ++i) {
    const int v = in[i];
    out[i] = run;
    run += v;
  }
  if (lane == 31) out[n] = incl;
}

}  // namespace moe
