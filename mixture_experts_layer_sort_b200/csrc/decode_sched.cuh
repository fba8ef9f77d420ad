// decode_sched.cuh - the schedule of a decode batch (up to 64 tokens) built by every
// CTA in its own shared memory from the batch's routing: per-expert counts, the stable
// grouping of (token, slot) pairs by expert, padded row offsets, the active experts, and
// the tile counts and split factors of both grouped GEMMs. A kernel that builds it needs
// no align kernel before it and no grid-wide exchange of the routing; it is used by the
// single-launch decode kernel and by the small-batch GEMMs.
//
// Grouping: pair p = t*k + j goes to expert ids[p]; inside an expert pairs keep
// ascending p (the rank of (t, j) in expert e is the number of earlier tokens routed to
// e, one popcount of a 64-bit per-expert token mask). Rows are padded to 16 per expert.
#pragma once

#include "gemm_pipeline.cuh"
#include "route_common.cuh"

namespace moe {

constexpr int kSchedMaxTokens = 64;     // per-expert token masks are 64 bits
constexpr int kSchedMaxPairs = 512;
constexpr int kSchedMaxExperts = 512;
constexpr int kSchedBalancedWaves = 8;  // as in the align kernel

// Up to kMaxE experts; kMaxDone tokens finished by one down unit (at most a unit's
// token rows).
template <int kMaxE, int kMaxDone>
struct SchedT {
  static constexpr int kMaxExperts = kMaxE;
  int ids[kSchedMaxPairs];
  float w[kSchedMaxPairs];
  int count[kMaxE];
  int off[kMaxE + 1];                  // compact offsets of each expert's pairs
  int poff[kMaxE + 1];                 // padded offsets (rows of h)
  int act[kMaxE];                      // active experts, ascending
  int aidx[kMaxE + 1];                 // index of each expert among the active ones
  unsigned mask[kMaxE][2];             // tokens routed to each expert
  int pairs[kSchedMaxPairs];           // pair ids grouped by expert, ascending inside an expert
  int done[kMaxDone];                  // tokens completed by the current down unit
  float red[32];                       // block reduction scratch (one per warp)
  int ndone;
  int nact, T1, S1, T2, S2, n_max, rows_used, flag;
};

// The schedule of the single-launch decode kernel and of the small-batch GEMMs.
using Sched = SchedT<kSchedMaxExperts, kSchedMaxTokens>;

__host__ __device__ constexpr bool sched_supported(int M, int E, int k) {
  return M >= 1 && M <= kSchedMaxTokens && E <= kSchedMaxExperts && M * k <= kSchedMaxPairs;
}

// Tile t of a GEMM from the schedule: tile t = (active expert t / fb, row block t % fb);
// every expert has a single token tile (n_e <= M <= 64).
template <class S>
struct SmemTileFn {
  const S* s;
  int fb;
  __device__ __forceinline__ Tile operator()(int t) const {
    const int ai = t / fb;
    Tile tile;
    tile.expert = s->act[ai];
    tile.fblock = t - ai * fb;
    tile.row_start = s->poff[tile.expert];
    tile.n_valid = s->count[tile.expert];
    return tile;
  }
};

// Zero the counts and token masks (all threads; a barrier must follow before the build).
template <class S>
__device__ __forceinline__ void sched_clear(S* s, int E, int tid, int nthreads) {
  for (int e = tid; e < E; e += nthreads) {
    s->count[e] = 0;
    s->mask[e][0] = 0u;
    s->mask[e][1] = 0u;
  }
}

// Everything after the routing, from s->ids[0..P) (all threads of the CTA; the counts
// and masks cleared and a barrier passed before). Ends without a barrier: the caller
// synchronises before reading the schedule. G = CTAs of the grid; fb1/fb2 tiles across
// the output features and kb1/kb2 K blocks of gate_up/down; uniform = 1 forces one
// split factor per GEMM.
template <class S>
static __device__ void sched_build(S* s, int P, int E, int k, int fb1, int fb2, int kb1, int kb2, int G,
                            int ws1_rows_cap, int uniform, int tid, int nthreads) {
  const int warp = tid >> 5, lane = tid & 31;
  for (int p = tid; p < P; p += nthreads) {
    const int e = s->ids[p];
    const int t = p / k;
    atomicAdd(&s->count[e], 1);
    atomicOr(&s->mask[e][t >> 5], 1u << (t & 31));
  }
  __syncthreads();
  if (warp == 0) {
    warp_exclusive_scan(s->count, s->off, E, lane);
  } else if (warp == 1) {
    for (int e = lane; e < E; e += 32) s->act[e] = (s->count[e] + kPadRows - 1) / kPadRows * kPadRows;
    __syncwarp();
    warp_exclusive_scan(s->act, s->poff, E, lane);
  }
  __syncthreads();
  if (warp == 0) {
    for (int e = lane; e < E; e += 32) s->aidx[e] = s->count[e] > 0 ? 1 : 0;
    __syncwarp();
    warp_exclusive_scan(s->aidx, s->aidx, E, lane);   // in place
    __syncwarp();
    for (int e = lane; e < E; e += 32)
      if (s->count[e] > 0) s->act[s->aidx[e]] = e;
    if (lane == 0) s->nact = s->aidx[E];
  }
  __syncthreads();
  // stable grouping: rank of pair (t, j) inside expert e = tokens t' < t routed to e
  for (int p = tid; p < P; p += nthreads) {
    const int e = s->ids[p];
    const int t = p / k;
    const unsigned lo = t < 32 ? (s->mask[e][0] & ((1u << t) - 1u)) : s->mask[e][0];
    const unsigned hi = t < 32 ? 0u : (s->mask[e][1] & ((1u << (t - 32)) - 1u));
    s->pairs[s->off[e] + __popc(lo) + __popc(hi)] = p;
  }
  if (warp == 0) {
    int m = 0;
    for (int e = lane; e < E; e += 32) m = max(m, s->count[e]);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int A = s->nact;
    const int rows_used = s->poff[E];
    const int n_mean = A > 0 ? (P + A - 1) / A : 0;
    const int t1 = A * fb1;
    // the align kernel's rule: the balanced schedule (0) for one to
    // kSchedBalancedWaves waves of tiles when the partial sums fit, else the cost
    // model's split factor
    const bool allow = rows_used <= ws1_rows_cap;
    const int s1 = (!uniform && allow && t1 >= G && t1 < kSchedBalancedWaves * G)
                       ? 0
                       : choose_splits_warp(t1, kb1, G, allow, 2 * 16384 + n_mean * 128, n_mean * 256 * 4 * 2, lane);
    if (lane == 0) {
      s->n_max = (m + kPadRows - 1) / kPadRows * kPadRows;
      s->rows_used = rows_used;
      s->T1 = t1;
      s->S1 = s1;
    }
  } else if (warp == 1) {
    const int A = s->nact;
    const int n_mean = A > 0 ? (P + A - 1) / A : 0;
    const int t2 = A * fb2;
    const int s2 = (!uniform && t2 >= G && t2 < kSchedBalancedWaves * G)
                       ? 0
                       : choose_splits_warp(t2, kb2, G, true, 16384 + n_mean * 128, n_mean * 128 * 4, lane);
    if (lane == 0) {
      s->T2 = t2;
      s->S2 = s2;
    }
  }
}

// Copies of the schedule for inspection and for the kernels that read the padded
// permutation from global memory (the FP8 h quantiser): counts, padded offsets, the
// padded pair list (pad = P) and the rows in use. One CTA calls it (all its threads).
template <class S>
__device__ __forceinline__ void sched_publish(const S* s, int P, int E, int* counts, int* padded_offsets,
                                              int* padded_pairs, int* header, int tid, int nthreads) {
  for (int e = tid; e < E; e += nthreads) {
    counts[e] = s->count[e];
    padded_offsets[e] = s->poff[e];
    for (int r = s->poff[e]; r < s->poff[e + 1]; ++r) {
      const int j = r - s->poff[e];
      padded_pairs[r] = j < s->count[e] ? s->pairs[s->off[e] + j] : P;
    }
  }
  if (tid == 0) {
    padded_offsets[E] = s->poff[E];
    header[kHdrRowsUsed] = s->rows_used;
  }
}

}  // namespace moe
