// kernels_align.cu - moe_align: group the (token, slot) pairs by expert, pad each
// group to 16 rows, and build the tile lists and split factors of both grouped
// GEMMs. Up to 8192 pairs one thread block does everything; larger batches count
// per chunk of 1024 pairs in blocks of their own, plan in the one block, and place
// each chunk's pairs in its own block again.
//
// "Routing tokens to experts, moving data and combining expert outputs can add
// work around the matrix multiplications" (toolboxkart.tech, "AWS SageMaker MoE
// kernel optimizations H200", section "Why MoE inference needs specialized
// kernels"); the permutation below is that data movement's index map. Pair
// p = t*k + j goes to expert topk_ids[p]; inside an expert pairs keep ascending p.
// The tile list is the "dynamic scheduling" of thin, variable token batches the
// aib.vote page describes ("AWS SageMaker MoE kernel optimizations", third
// paragraph): it is built on the device from the counts, so the host never
// learns the routing and no kernel depends on the token count at compile time.
#include "moe_internal.h"
#include "route_common.cuh"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kAlignThreads = 1024;
// The balanced schedule (split factor 0) serves from one to kBalancedWaves waves of
// tiles. With more, round-robin leaves every CTA within one tile of the mean (< 1/8
// of its work) and the cut tiles would cost more than they save; with less than one
// wave, an equal split of every tile (the cost model's factor) needs fewer partial
// sums for the same balance.
constexpr int kBalancedWaves = 8;
constexpr int kAlignWarps = kAlignThreads / 32;
__global__ void __launch_bounds__(kAlignThreads, 1) align_kernel(AlignArgs a) {
  extern __shared__ int sm[];
  const int E = a.E;
  int* s_count = sm;                    // [E]
  int* s_padded = s_count + E;          // [E]   count rounded up to 16
  int* s_poff = s_padded + E;           // [E+1] padded offsets
  int* s_base = s_poff + E + 1;         // [E]   pairs of e placed by earlier chunks
  int* s_nb = s_base + E;               // [E]   token blocks of e
  int* s_nboff = s_nb + E;              // [E+1]
  int* s_wc = s_nboff + E + 1;          // [32][E] per-warp counts of the current chunk
  // precision per expert: token blocks of the FP8 experts and their offsets, then of the
  // bf16 experts (the FP8 experts' tiles go first in each tile list)
  int* s_nb8 = s_wc + kAlignWarps * E;  // [E]
  int* s_nboff8 = s_nb8 + E;            // [E+1]
  int* s_nbbf = s_nboff8 + E + 1;       // [E]
  int* s_nboffbf = s_nbbf + E;          // [E+1]
  const bool mixed = a.eflags != nullptr;

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;

  // small batches (M <= 64): stable ranks from per-expert token masks (the k experts
  // of a token are distinct, so the rank of pair (t, j) inside its expert is the
  // number of earlier tokens routed there); the per-warp table is reused for them
  const int M = a.P / a.k;
  const bool small = M <= 64;
  unsigned* s_mask = reinterpret_cast<unsigned*>(s_wc);   // [E][2] when small
  for (int e = tid; e < E; e += kAlignThreads) {
    s_count[e] = 0;
    s_base[e] = 0;
    if (small) {
      s_mask[2 * e] = 0u;
      s_mask[2 * e + 1] = 0u;
    }
  }
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const bool chunked = a.chunk_counts != nullptr;
  if (chunked) {
    // counts are the sums of the chunks' counts (written by align_count_kernel)
    for (int e = tid; e < E; e += kAlignThreads) {
      int n = 0;
      for (int c = 0; c < a.chunks; ++c) n += a.chunk_counts[static_cast<size_t>(c) * E + e];
      s_count[e] = n;
    }
  } else {
    for (int p = tid; p < a.P; p += kAlignThreads) {
      const int e = a.topk_ids[p];
      atomicAdd(&s_count[e], 1);
      if (small) {
        const int t = p / a.k;
        atomicOr(&s_mask[2 * e + (t >> 5)], 1u << (t & 31));
      }
    }
  }
  __syncthreads();
  for (int e = tid; e < E; e += kAlignThreads) {
    const int n = s_count[e];
    s_padded[e] = (n + kPadRows - 1) / kPadRows * kPadRows;
    s_nb[e] = (n + a.BN - 1) / a.BN;
    if (mixed) {
      const bool f8 = a.eflags[e] != 0;
      s_nb8[e] = f8 ? s_nb[e] : 0;
      s_nbbf[e] = f8 ? 0 : s_nb[e];
    }
  }
  __syncthreads();
  if (warp == 0) warp_exclusive_scan(s_padded, s_poff, E, lane);
  if (warp == 1) warp_exclusive_scan(s_nb, s_nboff, E, lane);
  if (mixed && warp == 2) warp_exclusive_scan(s_nb8, s_nboff8, E, lane);
  if (mixed && warp == 3) warp_exclusive_scan(s_nbbf, s_nboffbf, E, lane);
  __syncthreads();

  if (small) {
    for (int p = tid; p < a.P; p += kAlignThreads) {
      const int e = a.topk_ids[p];
      const int t = p / a.k;
      const unsigned lo = t < 32 ? (s_mask[2 * e] & ((1u << t) - 1u)) : s_mask[2 * e];
      const unsigned hi = t < 32 ? 0u : (s_mask[2 * e + 1] & ((1u << (t - 32)) - 1u));
      a.padded_pairs[s_poff[e] + __popc(lo) + __popc(hi)] = p;
    }
  }
  if (chunked) {
    // the first padded row of every (chunk, expert) group, for align_scatter_kernel
    for (int e = tid; e < E; e += kAlignThreads) {
      int run = s_poff[e];
      for (int c = 0; c < a.chunks; ++c) {
        const size_t i = static_cast<size_t>(c) * E + e;
        a.chunk_base[i] = run;
        run += a.chunk_counts[i];
      }
    }
  }
  // Otherwise a stable scatter, 1024 pairs per chunk: rank inside the warp from the
  // match mask, plus the counts of earlier warps in this chunk, plus earlier chunks.
  const unsigned lt_mask = (1u << lane) - 1u;
  for (int c0 = 0; !small && !chunked && c0 < a.P; c0 += kAlignThreads) {
    for (int i = tid; i < kAlignWarps * E; i += kAlignThreads) s_wc[i] = 0;
    __syncthreads();
    const int p = c0 + tid;
    const bool valid = p < a.P;
    const int e = valid ? a.topk_ids[p] : 0x7FFFFFFF;
    const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
    const int rank = __popc(peers & lt_mask);
    if (valid && rank == 0) s_wc[warp * E + e] = __popc(peers);
    __syncthreads();
    if (valid) {
      int pos = s_base[e] + rank;
      for (int w = 0; w < warp; ++w) pos += s_wc[w * E + e];
      a.padded_pairs[s_poff[e] + pos] = p;
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kAlignThreads) {
      int tot = 0;
      for (int w = 0; w < kAlignWarps; ++w) tot += s_wc[w * E + ee];
      s_base[ee] += tot;
    }
    __syncthreads();
  }

  for (int e = tid; e < E; e += kAlignThreads) {
    for (int r = s_poff[e] + s_count[e]; r < s_poff[e + 1]; ++r) a.padded_pairs[r] = a.P;
    a.counts[e] = s_count[e];
    a.padded_offsets[e] = s_poff[e];
  }
  if (tid == 0) a.padded_offsets[E] = s_poff[E];

  // Tiles: for expert e, its token blocks b and weight row blocks f, in the
  // order (e, f, b) so that tiles sharing a weight tile are neighbours. The down
  // tiles go in feature slabs: (slab, e, f, b), slab s covering row blocks
  // [s*F/S, (s+1)*F/S). Every tile of a slab adds into the same columns of the fp32
  // accumulator, so with S slabs only 1/S of the accumulator is live in L2 at a time
  // (a large batch's accumulator would otherwise not stay in L2 between the k
  // contributions to each token); the price is reading each expert's h once per slab.
  const int nblocks_all = s_nboff[E];
  // (a layer with a precision per expert keeps one slab: each of its two parts must
  // be one contiguous run of tiles)
  const int S2 = (mixed || a.acc_slabs < 1) ? 1 : a.acc_slabs;
  for (int e = warp; e < E; e += kAlignWarps) {
    const int n = s_count[e];
    const int nb = s_nb[e];
    if (nb == 0) continue;
    const int base = !mixed ? s_nboff[e] : (a.eflags[e] != 0 ? s_nboff8[e] : s_nboff8[E] + s_nboffbf[e]);
    for (int idx = lane; idx < nb * a.fblocks1; idx += 32) {
      const int f = idx / nb, b = idx - f * nb;
      Tile t;
      t.expert = e;
      t.fblock = f;
      t.row_start = s_poff[e] + b * a.BN;
      t.n_valid = min(a.BN, n - b * a.BN);
      a.tiles1[static_cast<size_t>(base) * a.fblocks1 + idx] = t;
    }
    for (int idx = lane; idx < nb * a.fblocks2; idx += 32) {
      const int f = idx / nb, b = idx - f * nb;
      Tile t;
      t.expert = e;
      t.fblock = f;
      t.row_start = s_poff[e] + b * a.BN;
      t.n_valid = min(a.BN, n - b * a.BN);
      const int sl = ((f + 1) * S2 - 1) / a.fblocks2;      // the slab holding row block f
      const int f0 = sl * a.fblocks2 / S2, f1 = (sl + 1) * a.fblocks2 / S2;
      a.tiles2[static_cast<size_t>(nblocks_all) * f0 + static_cast<size_t>(base) * (f1 - f0) + (f - f0) * nb + b] = t;
    }
  }

  // widest token tile (the GEMMs size their stage ring from it) and the split-K
  // factors: warps 0 and 1 of the block
  __syncthreads();
  if (warp == 0) {
    int m = 0;
    for (int e = lane; e < E; e += 32) m = max(m, min(a.BN, s_count[e]));
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int nblocks = s_nboff[E];
    const int rows_used = s_poff[E];
    const int t1 = nblocks * a.fblocks1;
    // mean token rows per tile; gate_up K block = two 16 KB weight tiles + n rows of x;
    // a split gate_up tile adds and reads back n x 256 fp32 partial sums
    const int n_mean = nblocks > 0 ? (a.P + nblocks - 1) / nblocks : 0;
    // balanced schedule (split factor 0) for one to kBalancedWaves waves of tiles when
    // the partial sums fit the workspace; otherwise the cost model's split factor
    const bool allow = rows_used <= a.ws1_rows_cap;
    const bool bal1 = allow && t1 >= a.num_sms && t1 < kBalancedWaves * a.num_sms;
    const int s1 = (!a.uniform_splits && bal1) ? 0
                                     : choose_splits_warp(t1, a.kblocks1, a.num_sms, allow,
                                                          2 * 16384 + n_mean * 128, n_mean * 256 * 4 * 2, lane);
    if (lane == 0) {
      a.header[kHdrMaxRows] = (m + kPadRows - 1) / kPadRows * kPadRows;
      a.header[kHdrRowsUsed] = rows_used;
      a.header[kHdrTiles1] = t1;
      a.header[kHdrSplits1] = s1;
      a.header[kHdrTokenBlocks] = nblocks;
    }
  } else if (mixed && warp >= 2 && warp < 6) {
    // the FP8 part and the bf16 part of each list, each with its own split factor
    // (the rule of warps 0 and 1 below with the part's tiles and K blocks)
    const bool gate = warp < 4, f8 = (warp & 1) == 0;
    const int nb_part = f8 ? s_nboff8[E] : s_nboffbf[E];
    const int nblocks = s_nboff[E];
    const int n_mean = nblocks > 0 ? (a.P + nblocks - 1) / nblocks : 0;
    const int t = nb_part * (gate ? a.fblocks1 : a.fblocks2);
    const int kb = gate ? (f8 ? a.kblocks1_f8 : a.kblocks1) : (f8 ? a.kblocks2_f8 : a.kblocks2);
    const int kbytes = (gate ? 2 * 16384 : 16384) + n_mean * 128;
    const int sbytes = gate ? n_mean * 256 * 4 * 2 : n_mean * 128 * 4;
    const bool allow = !gate || s_poff[E] <= a.ws1_rows_cap;
    const bool bal = allow && t >= a.num_sms && t < kBalancedWaves * a.num_sms;
    const int sp = (!a.uniform_splits && bal) ? 0 : choose_splits_warp(t, kb, a.num_sms, allow, kbytes, sbytes, lane);
    if (lane == 0) {
      const int slot = gate ? (f8 ? kHdrTiles1F8 : kHdrTiles1BF) : (f8 ? kHdrTiles2F8 : kHdrTiles2BF);
      a.header[slot] = t;
      a.header[slot + 1] = sp;
    }
  } else if (warp == 1) {
    const int nblocks = s_nboff[E];
    const int t2 = nblocks * a.fblocks2;
    const int n_mean = nblocks > 0 ? (a.P + nblocks - 1) / nblocks : 0;
    // down: a split only adds more fp32 partial sums to the accumulator
    const bool bal2 = t2 >= a.num_sms && t2 < kBalancedWaves * a.num_sms;
    const int s2 = (!a.uniform_splits && bal2) ? 0
                                     : choose_splits_warp(t2, a.kblocks2, a.num_sms, true, 16384 + n_mean * 128,
                                                          n_mean * 128 * 4, lane);
    if (lane == 0) {
      a.header[kHdrTiles2] = t2;
      a.header[kHdrSplits2] = s2;
    }
  }
}

// Multi-block path, step 1: per-expert pair counts of chunk blockIdx.x.
__global__ void __launch_bounds__(kAlignChunk) align_count_kernel(AlignArgs a) {
  extern __shared__ int hist[];   // [E]
  for (int e = threadIdx.x; e < a.E; e += kAlignChunk) hist[e] = 0;
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int p = blockIdx.x * kAlignChunk + threadIdx.x;
  if (p < a.P) atomicAdd(&hist[a.topk_ids[p]], 1);
  __syncthreads();
  for (int e = threadIdx.x; e < a.E; e += kAlignChunk)
    a.chunk_counts[static_cast<size_t>(blockIdx.x) * a.E + e] = hist[e];
}

// Multi-block path, step 3: place the pairs of chunk blockIdx.x. Row of pair p =
// chunk_base[chunk][e] + (pairs of e earlier in the chunk): earlier warps' counts
// plus the rank inside the warp from the match mask, so the order inside an expert
// stays ascending in p.
__global__ void __launch_bounds__(kAlignChunk) align_scatter_kernel(AlignArgs a) {
  extern __shared__ int wc[];     // [32][E] pairs of e in each warp of the chunk
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = threadIdx.x; i < 32 * a.E; i += kAlignChunk) wc[i] = 0;
  pdl_wait();
  pdl_trigger();
  __syncthreads();
  const int p = blockIdx.x * kAlignChunk + threadIdx.x;
  const bool valid = p < a.P;
  const int e = valid ? a.topk_ids[p] : 0x7FFFFFFF;
  const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
  const int rank = __popc(peers & ((1u << lane) - 1u));
  if (valid && rank == 0) wc[warp * a.E + e] = __popc(peers);
  __syncthreads();
  if (valid) {
    int pos = a.chunk_base[static_cast<size_t>(blockIdx.x) * a.E + e] + rank;
    for (int w = 0; w < warp; ++w) pos += wc[w * a.E + e];
    a.padded_pairs[pos] = p;
  }
}

}  // namespace

size_t align_smem_bytes(int E) { return static_cast<size_t>(10 * E + 4 + kAlignWarps * E) * sizeof(int); }

cudaError_t align_configure() {
  cudaError_t e = cudaFuncSetAttribute(align_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(align_smem_bytes(512)));
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(align_scatter_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, 32 * 512 * 4);
}

cudaError_t launch_align_count(const AlignArgs& a, cudaStream_t s) {
  return launch_kernel(align_count_kernel, dim3(a.chunks), dim3(kAlignChunk), static_cast<size_t>(a.E) * 4, s, a);
}

cudaError_t launch_align_scatter(const AlignArgs& a, cudaStream_t s) {
  return launch_kernel(align_scatter_kernel, dim3(a.chunks), dim3(kAlignChunk), static_cast<size_t>(32) * a.E * 4,
                       s, a);
}

cudaError_t launch_align(const AlignArgs& a, cudaStream_t s) {
  return launch_kernel(align_kernel, dim3(1), dim3(kAlignThreads), align_smem_bytes(a.E), s, a);
}

}  // namespace moe
