// gemm_pipeline.cuh - the warp-specialised tcgen05 pipeline behind both grouped GEMMs
// of the MoE layer, written once and used by the stand-alone grouped kernel
// (kernels_gemm.cu) and by the single-launch decode kernel (kernels_decode.cu).
//
// Orientation: every tile is "swap-AB". The expert's weight rows fill the MMA's
// M = 128 slot and the expert's few tokens are the N dimension (16..256), i.e. the
// kernel computes D^T = W * X^T instead of X * W^T (M = 256 over a CTA pair, kPair
// below, each CTA holding 128 of the rows and half of the tokens). (A B)^T = B^T A^T
// changes no arithmetic (kongchang.com, "MoE Kernel Engineering Optimization Practices on
// Amazon SageMaker AI", section "Swap-AB: Making WGMMA Run at Full Utilization");
// it keeps the tensor-core rows busy when decode gives an expert a handful of
// tokens (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section
// "1. Swap-AB makes better use of the WGMMA tile"; aib.vote, "AWS SageMaker MoE
// kernel optimizations", second paragraph). On sm_100 N reaches 256, so the same
// orientation also covers prefill (~128-256 tokens per expert).
//
// A stage holds two 128-row weight tiles that share one activation tile: the W_gate
// and W_up rows of the same 128 features (gate_up), or two consecutive 128-row
// blocks of W_down (down). Two TMEM accumulators take the two products. The gate_up
// epilogue forms h = silu(g) * u ("fuses scaling, matrix multiplication ... into one
// GPU pass", aib.vote page, third paragraph); the down epilogue scales by the
// routing weight and scatter-adds into the fp32 token accumulator ("expert
// aggregation").
//
// Roles: warp 0 = TMA producer (lane 0 owns the stage barriers and the weight loads,
// the activation rows of a stage are spread over the lanes), warp 1 = TMEM owner and
// MMA issuer, warps 2.. = epilogue: kEpiGroups warps per TMEM lane quadrant (warp % 4),
// which take turns over the 16-column chunks of the accumulators. With token tiles wider
// than 128 columns there is a single accumulator buffer, and the MMAs of the next tile
// wait until the epilogue has read it: more warps per quadrant shorten that wait. Units (a tile,
// or one K range of a split tile) come from a unit source; dependencies of the
// activation operand and completion signals come from hooks, so that one kernel can
// run both GEMMs back to back.
#pragma once

#include "fp8_format.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {
namespace pipe {

// Epilogue warps per TMEM lane quadrant. Measured on one B200 at prefill size (E=256,
// M=4096, one forward): 1 -> 4487 us, 2 -> 4280, 3 -> 4147, 4 -> 4223 (bf16); FP8
// 2724 / 2491 / 2429 / 2422; decode unchanged.
constexpr int kEpiGroups = 3;
constexpr int kEpiThreads = 128 * kEpiGroups;
constexpr int kThreads = 64 + kEpiThreads;
constexpr int kTokenTile = 256;   // widest token tile: the largest N of an M=128 MMA
static_assert(kTokenTile == kTokenBlock, "the align kernel's token blocks are the GEMM token tiles");

// kSmem: dynamic shared memory of the kernel (default 224 KB, one CTA per SM: 3 KB under
// the sm_100 opt-in maximum, so that a CTA of a one-row kernel launched next to it, a
// gather or h quantisation with its own 1 KB reserve, can share the SM and the GEMM's
// first weight loads overlap it under programmatic dependent launch); kTmem: TMEM
// columns it allocates (two accumulator buffers of kTmem / 2 columns). Two kernels whose
// sizes add up to at most one SM's shared memory and TMEM can have CTAs resident on the
// same SM at once.
// kPair: the tiles of a unit are split over a CTA pair (a cluster of two) that runs
// M = 256 MMAs: each CTA holds its own two weight tiles and half of the activation rows,
// the pair's first CTA issues the MMAs, and each CTA's TMEM receives its own rows.
constexpr int kGemmSmem = 229376;
template <bool kFP8, int kSmem = kGemmSmem, int kTmem = 512, bool kPair_ = false>
struct Cfg {
  static constexpr bool kPair = kPair_;
  static constexpr int kATiles = 2;
  static constexpr int kABytes = kTileRows * kRowBytes;             // 16 KB per weight tile
  static constexpr int kTmemCols = kTmem;                            // two buffers x two accumulators
  static constexpr int kBufCols = kTmem / 2;                         // columns of one buffer
  static constexpr int kSmemBytes = kSmem;
  // [0, 1 KB): barriers and flags; [1 KB, 3 KB): two slots of the down epilogue's
  // per-column token row (int, 256 columns each); [3 KB, 5 KB): two slots of its
  // scaled routing weights (float); then the caller's extra bytes, then the ring
  static constexpr int kColTableOffset = 1024;
  static constexpr int kFixedBytes = 6144;
  static constexpr int kMaxStages = 16;
  static constexpr int kKPerBlock = kFP8 ? 128 : 64;                 // elements in one 128-byte row
  static constexpr int kMmaKBytes = 32;                              // K of one MMA = 32 bytes
  static constexpr int kMmasPerBlock = kRowBytes / kMmaKBytes;
  static_assert(2 * kMaxStages * 8 + 40 + 4 + 16 <= kColTableOffset, "barrier area");
  static_assert(kColTableOffset + 2 * 2 * 256 * 4 <= kFixedBytes, "column tables");
  static_assert(kTmem == 256 || kTmem == 512, "TMEM allocation");
};

struct Shared {
  uint8_t* ring;          // stage ring, 1024-aligned
  uint64_t* full;         // [kMaxStages]
  uint64_t* empty;        // [kMaxStages]
  uint64_t* acc_full;     // [2]
  uint64_t* acc_empty;    // [2]
  uint64_t* drain;        // MMA warp, after a failure: completion of every MMA it issued
  uint32_t* tmem_slot;
  int* flags;             // [0] abort, [1] last arriver, [2..3] epilogue wait outcome
  int* col_tok;           // [2][256]
  float* col_w;           // [2][256]
  uint8_t* extra;         // caller's region (1024-aligned), or the ring when none
  int ring_bytes;
};

template <class C>
__device__ __forceinline__ Shared carve(uint8_t* raw, int extra_bytes) {
  Shared s;
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(raw) + 1023) & ~uintptr_t(1023));
  s.full = reinterpret_cast<uint64_t*>(base);
  s.empty = s.full + C::kMaxStages;
  s.acc_full = s.empty + C::kMaxStages;
  s.acc_empty = s.acc_full + 2;
  s.drain = s.acc_empty + 2;
  s.tmem_slot = reinterpret_cast<uint32_t*>(s.drain + 1);
  s.flags = reinterpret_cast<int*>(s.tmem_slot + 1);
  s.col_tok = reinterpret_cast<int*>(base + C::kColTableOffset);
  s.col_w = reinterpret_cast<float*>(base + C::kColTableOffset + 2048);
  const int extra = (extra_bytes + 1023) & ~1023;
  s.extra = base + C::kFixedBytes;
  s.ring = base + C::kFixedBytes + extra;
  s.ring_bytes = C::kSmemBytes - 1024 - C::kFixedBytes - extra;
  return s;
}

// Barrier init (one thread) and TMEM allocation (warp 1), then a CTA-wide sync.
template <class C>
__device__ __forceinline__ uint32_t prologue(const Shared& s, int warp) {
  if (threadIdx.x == 0) {
    // pair: the first CTA's full barriers count both CTAs' bytes (the second CTA's are
    // unused); every CTA's empty barriers take the first CTA's commits
    for (int i = 0; i < C::kMaxStages; ++i) {
      mbar_init(&s.full[i], 1);
      mbar_init(&s.empty[i], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&s.acc_full[b], 1);
      mbar_init(&s.acc_empty[b], (C::kPair ? 2 : 1) * (kEpiThreads / 32));
    }
    mbar_init(s.drain, 1);
    for (int i = 0; i < 4; ++i) s.flags[i] = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    if constexpr (C::kPair) {
      tmem_alloc_pair(s.tmem_slot, C::kTmemCols);
      tmem_relinquish_pair();
    } else {
      tmem_alloc(s.tmem_slot, C::kTmemCols);
      tmem_relinquish();
    }
  }
  tc_fence_before();
  if constexpr (C::kPair) cluster_sync();   // both CTAs' barriers exist before either signals the other
  else __syncthreads();
  tc_fence_after();
  return *s.tmem_slot;
}

template <class C>
__device__ __forceinline__ void teardown(uint32_t tmem, int warp) {
  tc_fence_before();
  if constexpr (C::kPair) cluster_sync();   // neither CTA leaves while the other may still signal it
  else __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    if constexpr (C::kPair) tmem_dealloc_pair(tmem, C::kTmemCols);
    else tmem_dealloc(tmem, C::kTmemCols);
  }
}

// Stage ring: a stage holds the two weight tiles plus n_max rows of activations
// (n_max = widest token tile of the forward), so thin decode batches get a deeper
// ring than prefill. Two TMEM buffers (columns 0 and kBufCols) when a buffer's two
// accumulators fit kBufCols columns (up to 128 tokens with 512 columns, 64 with 256),
// else one buffer of two accumulators kBufCols apart.
struct Ring {
  int n_cap, stage_bytes, stages, nbuf;
  uint32_t up_col, buf_col;
};

template <class C>
__device__ __forceinline__ Ring make_ring(int n_max, int max_stages, int ring_bytes) {
  Ring r;
  // at most kTokenTile tokens, and two accumulators of n_cap columns in the allocation
  // (a unit with more valid rows fails its bounds check and is reported, not run)
  constexpr int kCap = kTokenTile < C::kTmemCols / 2 ? kTokenTile : C::kTmemCols / 2;
  // a pair's N is a multiple of 32, so that each CTA holds whole 16-row boxes of it
  constexpr int kGran = C::kPair ? 32 : 16;
  r.n_cap = n_max < kGran ? kGran : (n_max > kCap ? kCap : ((n_max + kGran - 1) & ~(kGran - 1)));
  r.stage_bytes = (C::kATiles * C::kABytes + (C::kPair ? r.n_cap / 2 : r.n_cap) * kRowBytes + 1023) & ~1023;
  r.stages = ring_bytes / r.stage_bytes;
  if (r.stages > C::kMaxStages) r.stages = C::kMaxStages;
  if (max_stages >= 2 && r.stages > max_stages) r.stages = max_stages;
  r.nbuf = 2 * r.n_cap <= C::kBufCols ? 2 : 1;
  r.up_col = r.nbuf == 2 ? C::kBufCols / 2 : C::kBufCols;
  r.buf_col = C::kBufCols;
  return r;
}

struct Unit {
  Tile t;
  int tile;      // index of the tile (split-K counter)
  int S;         // splits of the tile
  int kb0, kb1;  // K blocks of this unit
  bool ok;       // tile passed its bounds check (every role skips a bad unit alike)
};

__device__ __forceinline__ Unit make_unit_range(const Tile& t, int tile, int kb0, int kb1, int S, int n_cap) {
  Unit x;
  x.t = t;
  x.tile = tile;
  x.S = S;
  x.kb0 = kb0;
  x.kb1 = kb1;
  x.ok = t.n_valid >= 1 && t.n_valid <= n_cap && kb1 > kb0;
  return x;
}

// Split s of S equal K ranges of a tile.
__device__ __forceinline__ Unit make_unit(const Tile& t, int tile, int s, int S, int kblocks, int n_cap) {
  return make_unit_range(t, tile, s * kblocks / S, (s + 1) * kblocks / S, S, n_cap);
}

// Tile t of a tile list in global memory (written by the align kernel).
struct GlobalTileFn {
  const Tile* tiles;
  __device__ __forceinline__ Tile operator()(int t) const { return tiles[t]; }
};

// The units of worker w (of nw: CTAs, or CTA pairs) over T tiles given by a tile function
// (a list in global memory, or a schedule held in shared memory); count() of them,
// unit(i) in the order every role of the CTA walks them. Two ways of dealing them
// out, chosen by S:
//  - S >= 1: each tile is cut into S equal K ranges and the T*S units go round-robin.
//  - S == 0, balanced: the T tiles minus the last one to two waves go round-robin as
//    whole tiles. The K blocks of the remaining tiles are cut into one contiguous
//    range per CTA of equal length (to one K block), so that every CTA streams the
//    same weight bytes whatever T is. A tile whose K blocks fall into the ranges of
//    several CTAs is a split tile with S = that number of CTAs. A CTA takes its range
//    first, so that the split tiles' partial-sum fix-ups overlap the whole tiles.
template <class TileFn>
struct UnitSchedule {
  TileFn tiles;
  int T, S, K;
  int w, nw;               // this worker (a CTA, or a CTA pair) and the number of workers
  int bal_tiles;           // tiles [0, bal_tiles) form the balanced region
  int g_bal;               // CTAs that share it (each with a non-empty range)
  int bal_total;           // its K blocks
  int x0, x1;              // this CTA's K-block range in it
  int n_bal, n_whole;      // this CTA's units: pieces of the range, then whole tiles

  // The balanced region holds fewer than two waves of tiles of at most 256 K blocks,
  // so c * bal_total stays far below 2^31 for any grid of up to a few hundred CTAs.
  __device__ __forceinline__ UnitSchedule(TileFn tiles_, int T_, int S_, int K_, bool pair = false)
      : tiles(tiles_), T(T_), S(S_), K(K_),
        w(pair ? static_cast<int>(blockIdx.x) >> 1 : static_cast<int>(blockIdx.x)),
        nw(pair ? static_cast<int>(gridDim.x) >> 1 : static_cast<int>(gridDim.x)), bal_tiles(0), g_bal(0),
        bal_total(0), x0(0), x1(0), n_bal(0), n_whole(0) {
    if (S != 0 || T <= 0 || K <= 0) return;
    const int G = nw;
    const int c = w;
    const int waves = T / G, rem = T - waves * G;
    bal_tiles = rem == 0 ? 0 : (waves == 0 ? T : rem + G);
    bal_total = bal_tiles * K;
    g_bal = bal_total < G ? bal_total : G;
    if (c < g_bal) {
      x0 = c * bal_total / g_bal;
      x1 = (c + 1) * bal_total / g_bal;
      n_bal = (x1 - 1) / K - x0 / K + 1;
    }
    const int whole = T - bal_tiles;
    n_whole = c < whole ? (whole - 1 - c) / G + 1 : 0;
  }
  // the CTA whose range holds K block x of the balanced region
  __device__ __forceinline__ int owner(int x) const { return ((x + 1) * g_bal - 1) / bal_total; }
  __device__ __forceinline__ int count() const {
    if (S == 0) return n_bal + n_whole;
    const int n = T * S, c = w;
    return c < n ? (n - 1 - c) / nw + 1 : 0;
  }
  __device__ __forceinline__ Unit unit(int i, int n_cap) const {
    if (S != 0) {
      const int u = w + i * nw;
      const int t = u / S;
      return make_unit(tiles(t), t, u - t * S, S, K, n_cap);
    }
    if (i < n_bal) {
      const int t = x0 / K + i;
      const int kb0 = i == 0 ? x0 - t * K : 0;
      const int last = x1 - 1;
      const int kb1 = t == last / K ? last - t * K + 1 : K;
      const int first = t * K;
      const int sharers = owner(first + K - 1) - owner(first) + 1;
      return make_unit_range(tiles(t), t, kb0, kb1, sharers, n_cap);
    }
    const int t = bal_tiles + w + (i - n_bal) * nw;
    return make_unit_range(tiles(t), t, 0, K, 1, n_cap);
  }
};

struct GlobalTiles : UnitSchedule<GlobalTileFn> {
  __device__ __forceinline__ GlobalTiles(const Tile* tiles_, int T_, int S_, int K_, bool pair = false)
      : UnitSchedule<GlobalTileFn>(GlobalTileFn{tiles_}, T_, S_, K_, pair) {}
};

// silu(z) = z / (1 + e^-z) with the fast division (2 ulp): e^-z = inf for z < -88 gives
// z * 0 = -0, the limit; the epilogue rounds the product to bf16 right after.
__device__ __forceinline__ float silu(float z) { return __fdividef(z, 1.f + __expf(-z)); }

// SM cycles a pipeline wait may take before it gives up (GemmArgs::wait_budget, 0 = the
// default of about a second).
__device__ __forceinline__ long long wait_budget(const GemmArgs& a) {
  return a.wait_budget > 0 ? a.wait_budget : (1ll << 31);
}

// ------------------------------------------------------------------------ producer
struct ProducerState {
  int stage = 0;
  uint32_t phase = 0;
  int issued = 0;
  bool failed = false;
};

// Hooks (all lanes call them uniformly):
//   int dep(const Unit&)  - key of the activation operand's dependency
//   bool ready(int dep)   - non-blocking check
//   bool wait(int dep)    - blocking (bounded) wait; false when it gave up
//   bool direct()         - activation rows are single rows of a [tokens, K] tensor
//                           (one-row TMA boxes) instead of 16-row boxes of a permuted one
//   int direct_token(const Unit&, int j) - in direct mode, the tensor row of column j
template <class C, class Src, class Hooks>
__device__ void run_producer(const GemmArgs& a, const CUtensorMap* tm_w, const CUtensorMap* tm_b, const Shared& sh,
                             const Ring& rg, const Src& src, Hooks& hk, ProducerState& ps, volatile int* abort_flag,
                             int lane) {
  const uint64_t pol_w = l2_policy_evict_first();   // weights stream through once
  const uint64_t pol_b = l2_policy_evict_last();    // activations are re-read per tile
  // Activation loads whose dependency is not met yet wait in a queue (their weight
  // loads are already out); the queue is released in order once it fills the ring.
  int npend = 0;
  int pend_stage[C::kMaxStages], pend_kc[C::kMaxStages], pend_row[C::kMaxStages], pend_nb[C::kMaxStages],
      pend_dep[C::kMaxStages];
  // direct mode: x row (token) of activation rows lane, lane+32, lane+64, lane+96 of
  // the current unit; pad rows re-read row 0 (their columns are never stored)
  int tok[4] = {0, 0, 0, 0};
  const bool direct = hk.direct();
  // nb: 16-row boxes, or in direct mode the number of valid rows (rows past them are
  // not loaded: an MMA output column depends on its own activation row only, and the
  // columns of pad rows are never stored)
  auto load_b = [&](int stg, int kc, int row_start, int nb) {
    uint8_t* bdst = sh.ring + stg * rg.stage_bytes + C::kATiles * C::kABytes;
    if constexpr (C::kPair) {
      const uint32_t bar = mapa_shared(smem_u32(&sh.full[stg]), 0);
      for (int j = lane; j < nb; j += 32)
        tma_load_2d_pair(bdst + j * 16 * kRowBytes, tm_b, bar, kc, row_start + 16 * j, pol_b);
    } else if (!direct) {
      for (int j = lane; j < nb; j += 32)
        tma_load_2d(bdst + j * 16 * kRowBytes, tm_b, &sh.full[stg], kc, row_start + 16 * j, pol_b);
    } else {
      #pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int j = lane + 32 * i;
        if (j < nb) tma_load_2d(bdst + j * kRowBytes, tm_b, &sh.full[stg], kc, tok[i], pol_b);
      }
    }
  };
  // issue queued activation loads in order while their dependencies are met
  auto drain = [&](bool block) -> bool {
    int i = 0;
    for (; i < npend; ++i) {
      if (!hk.ready(pend_dep[i])) {
        if (!block) break;
        if (!hk.wait(pend_dep[i])) return false;
      }
      load_b(pend_stage[i], pend_kc[i], pend_row[i], pend_nb[i]);
    }
    for (int j = i; j < npend; ++j) {
      pend_stage[j - i] = pend_stage[j];
      pend_kc[j - i] = pend_kc[j];
      pend_row[j - i] = pend_row[j];
      pend_nb[j - i] = pend_nb[j];
      pend_dep[j - i] = pend_dep[j];
    }
    npend -= i;
    return true;
  };
  // pair: this CTA's weight row blocks sit pair_rb blocks after the first CTA's, and it
  // holds activation rows [N/2, N) of the unit (the first CTA rows [0, N/2))
  const int rank = C::kPair ? static_cast<int>(cluster_ctarank()) : 0;
  const int n_units = src.count();
  for (int i = 0; i < n_units && !ps.failed; ++i) {
    const Unit un = src.unit(i, rg.n_cap);
    if (!un.ok) continue;
    const int half = ((un.t.n_valid + 31) & ~31) >> 1;
    const int nb16 = C::kPair ? half >> 4 : (un.t.n_valid + 15) >> 4;
    const int row0 = un.t.row_start + rank * half;
    // first tiled-weight block of the unit's two weight row blocks; a second block
    // past the end of the tensor reads zeros and is not stored by the epilogue
    const int rb0 = un.t.fblock * a.rb_step + rank * a.pair_rb;
    const int et = a.w_expert_tiles > 0 ? static_cast<int>(a.w_expert_tiles) : a.w_rblocks * a.kblocks;
    const int wtile = un.t.expert * et + rb0 * a.kblocks;
    const int wtile2 = un.t.expert * et + (rb0 + a.second_rb) * a.kblocks;
    // activation rows of a stage: 16-row boxes, or (direct mode) the valid rows alone
    const int nrows = direct ? un.t.n_valid : nb16;
    const uint32_t tx = C::kATiles * C::kABytes + (direct ? un.t.n_valid : nb16 * 16) * kRowBytes;
    const int dep = hk.dep(un);
    for (int kb = un.kb0; kb < un.kb1; ++kb) {
      int ok = 1;
      if (lane == 0) {
        ok = mbar_wait_bounded(&sh.empty[ps.stage], ps.phase ^ 1u, abort_flag, wait_budget(a)) ? 1 : 0;
        if (!ok) {
          report_error(a.err, kErrWaitEmpty);
          *abort_flag = 1;
        } else if constexpr (C::kPair) {
          // both CTAs' loads count on the first CTA's barrier, which expects both halves
          uint8_t* st = sh.ring + ps.stage * rg.stage_bytes;
          const uint32_t bar = mapa_shared(smem_u32(&sh.full[ps.stage]), 0);
          if (rank == 0) mbar_arrive_expect_tx(&sh.full[ps.stage], 2 * tx);
          tma_load_2d_pair(st, tm_w, bar, 0, (wtile + kb) * kTileRows, pol_w);
          tma_load_2d_pair(st + C::kABytes, tm_w, bar, 0, (wtile2 + kb) * kTileRows, pol_w);
        } else {
          uint8_t* st = sh.ring + ps.stage * rg.stage_bytes;
          mbar_arrive_expect_tx(&sh.full[ps.stage], tx);
          tma_load_2d(st, tm_w, &sh.full[ps.stage], 0, (wtile + kb) * kTileRows, pol_w);
          tma_load_2d(st + C::kABytes, tm_w, &sh.full[ps.stage], 0, (wtile2 + kb) * kTileRows, pol_w);
        }
      }
      ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
      if (!ok) {
        ps.failed = true;
        break;
      }
      if (direct && kb == un.kb0) {
        // queued activation loads read the previous unit's token rows: issue them
        // (waiting for their dependency) before the rows change
        if (npend > 0 && !drain(true)) ps.failed = true;
        // the unit's token rows, read while its first weight tiles are in flight
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = lane + 32 * i;
          tok[i] = j < un.t.n_valid ? hk.direct_token(un, j) : 0;
        }
      }
      const int kc = kb * C::kKPerBlock;
      if (!ps.failed && npend > 0 && !drain(false)) ps.failed = true;
      if (!ps.failed && npend == 0 && hk.ready(dep)) {
        load_b(ps.stage, kc, row0, nrows);
      } else if (!ps.failed) {
        pend_stage[npend] = ps.stage;
        pend_kc[npend] = kc;
        pend_row[npend] = row0;
        pend_nb[npend] = nrows;
        pend_dep[npend] = dep;
        if (++npend == rg.stages && !drain(true)) ps.failed = true;
      }
      if (ps.failed) {
        if (lane == 0) {
          report_error(a.err, kErrWaitDep);
          *abort_flag = 1;
        }
        // this stage's weight loads are out: count it, so that producer_quiesce waits
        // for them before the CTA leaves
        ++ps.issued;
        if (++ps.stage == rg.stages) {
          ps.stage = 0;
          ps.phase ^= 1u;
        }
        break;
      }
      ++ps.issued;
      if (++ps.stage == rg.stages) {
        ps.stage = 0;
        ps.phase ^= 1u;
      }
    }
  }
  if (!ps.failed && npend > 0 && !drain(true)) {
    ps.failed = true;
    if (lane == 0) {
      report_error(a.err, kErrWaitDep);
      *abort_flag = 1;
    }
  }
}

// Pair: wait until the MMAs have released every stage this CTA filled, so that no
// arrival of the other CTA's commits is still on its way when the CTA leaves.
template <class C>
__device__ void producer_tail(const Shared& sh, const Ring& rg, const ProducerState& ps, int lane) {
  if (ps.failed || lane != 0) return;
  int zero = 0;
  int st = ps.stage;
  uint32_t ph = ps.phase;
  for (int i = 0; i < rg.stages; ++i) {
    mbar_wait_bounded(&sh.empty[st], ph ^ 1u, &zero, 1ll << 26);
    if (++st == rg.stages) {
      st = 0;
      ph ^= 1u;
    }
  }
}

// After a failure: let the copies already in flight land before shared memory goes away.
template <class C>
__device__ void producer_quiesce(const Shared& sh, const Ring& rg, const ProducerState& ps, int lane) {
  if (!ps.failed || lane != 0) return;
  if constexpr (C::kPair) {
    if (cluster_ctarank() != 0) {
      // its loads count on the other CTA's barriers: give them time to land instead
      const long long t0 = clock64();
      while (clock64() - t0 < (1ll << 17)) {
      }
      return;
    }
  }
  int zero = 0;
  int st = ps.stage, ph = static_cast<int>(ps.phase);
  const int pending = ps.issued < rg.stages ? ps.issued : rg.stages;
  for (int i = 0; i < pending; ++i) {
    if (--st < 0) {
      st = rg.stages - 1;
      ph ^= 1;
    }
    mbar_wait_bounded(&sh.full[st], static_cast<uint32_t>(ph), &zero, 1ll << 26);
  }
}

// ------------------------------------------------------------------------ MMA issuer
struct MmaState {
  int stage = 0;
  uint32_t phase = 0;
  int it = 0;
  bool failed = false;
};

template <class C, bool kFP8, class Src>
__device__ void run_mma(const GemmArgs& a, const Shared& sh, const Ring& rg, const Src& src, MmaState& ms,
                        uint32_t tmem, volatile int* abort_flag) {
  const int n_units = src.count();
  for (int i = 0; i < n_units && !ms.failed; ++i) {
    const Unit un = src.unit(i, rg.n_cap);
    if (!un.ok) continue;
    const uint32_t n_pad = C::kPair ? static_cast<uint32_t>((un.t.n_valid + 31) & ~31)
                                    : static_cast<uint32_t>((un.t.n_valid + 15) & ~15);
    // operand format: bf16 = 1 under kind::f16; the FP8 format code under kind::f8f6f4
    const uint32_t idesc = idesc_make(kFP8 ? static_cast<uint32_t>(a.f8) : 1u, C::kPair ? 256u : 128u, n_pad);
    const int buf = rg.nbuf == 2 ? (ms.it & 1) : 0;
    const uint32_t acc_phase = rg.nbuf == 2 ? ((ms.it >> 1) & 1) : (ms.it & 1);
    const uint32_t d_tmem = tmem + rg.buf_col * buf;
    ++ms.it;
    if (!mbar_wait_bounded(&sh.acc_empty[buf], acc_phase ^ 1u, abort_flag, wait_budget(a), C::kPair)) {
      report_error(a.err, kErrWaitAccEmpty);
      *abort_flag = 1;
      ms.failed = true;
      break;
    }
    tc_fence_after();
    for (int kb = un.kb0; kb < un.kb1; ++kb) {
      if (!mbar_wait_bounded(&sh.full[ms.stage], ms.phase, abort_flag, wait_budget(a))) {
        report_error(a.err, kErrWaitFull);
        *abort_flag = 1;
        ms.failed = true;
        break;
      }
      tc_fence_after();
      const uint32_t a0 = smem_u32(sh.ring + ms.stage * rg.stage_bytes);
      const uint32_t b0 = a0 + C::kATiles * C::kABytes;
      #pragma unroll
      for (int kk = 0; kk < C::kMmasPerBlock; ++kk) {
        const uint32_t koff = kk * C::kMmaKBytes;
        const uint32_t accum = (kb > un.kb0 || kk > 0) ? 1u : 0u;
        const uint64_t bd = sdesc_k_sw128(b0 + koff);
        const uint64_t ad0 = sdesc_k_sw128(a0 + koff);
        const uint64_t ad1 = sdesc_k_sw128(a0 + C::kABytes + koff);
        if constexpr (C::kPair && kFP8) {
          mma_f8_pair(d_tmem, ad0, bd, idesc, accum);
          mma_f8_pair(d_tmem + rg.up_col, ad1, bd, idesc, accum);
        } else if constexpr (C::kPair) {
          mma_bf16_pair(d_tmem, ad0, bd, idesc, accum);
          mma_bf16_pair(d_tmem + rg.up_col, ad1, bd, idesc, accum);
        } else if constexpr (kFP8) {
          mma_f8(d_tmem, ad0, bd, idesc, accum);
          mma_f8(d_tmem + rg.up_col, ad1, bd, idesc, accum);
        } else {
          mma_bf16(d_tmem, ad0, bd, idesc, accum);
          mma_bf16(d_tmem + rg.up_col, ad1, bd, idesc, accum);
        }
      }
      // frees the stage (in both CTAs of a pair) once these MMAs have read it
      if constexpr (C::kPair) mma_commit_pair(&sh.empty[ms.stage]);
      else mma_commit(&sh.empty[ms.stage]);
      if (++ms.stage == rg.stages) {
        ms.stage = 0;
        ms.phase ^= 1u;
      }
    }
    if (ms.failed) break;
    // accumulator complete (in both CTAs of a pair)
    if constexpr (C::kPair) mma_commit_pair(&sh.acc_full[buf]);
    else mma_commit(&sh.acc_full[buf]);
  }
}

// After the MMA thread gave up: make every MMA it issued complete (they write TMEM and
// arrive on stage barriers) before the CTA frees TMEM and leaves. tcgen05.commit
// tracks all earlier MMAs of the thread; the wait is bounded as well.
template <class C>
__device__ __forceinline__ void mma_drain(const Shared& sh, const MmaState& ms) {
  if (!ms.failed) return;
  int zero = 0;
  if constexpr (C::kPair) mma_commit_pair(sh.drain);
  else mma_commit(sh.drain);
  mbar_wait_bounded(sh.drain, 0u, &zero, 1ll << 26);
}

// ------------------------------------------------------------------------ epilogue
struct EpiState {
  int iter = 0;
  float lmax = 0.f;     // FP8 gate_up: max |h| written by this thread
  bool failed = false;
};

// Hooks:
//   column(const Unit&, int j, float scale, int& tok, float& w) - down: token row and
//        scaled routing weight of column j
//   static constexpr bool kSignalTiles; tile_done(const Unit&, int epi_tid, float lmax) -
//        gate_up: called by every epilogue thread once the tile's h rows are written
//        (lmax: the thread's running max |h|, FP8)
//   static constexpr bool kTokenCompletion; down_done(const Unit&, const int* s_tok,
//        int epi_tid) - down: called by every epilogue thread after the unit's adds
template <class C, bool kGateUp, bool kFP8, class Src, class Hooks>
__device__ void run_epilogue(const GemmArgs& a, const Shared& sh, const Ring& rg, const Src& src, Hooks& hk,
                             EpiState& es, uint32_t tmem, volatile int* abort_flag, int warp, int lane) {
  const int q = warp & 3;                       // TMEM lane quadrant of this warp
  const int grp = (warp - 2) >> 2;              // its 16-column chunks: grp + kEpiGroups * m
  const int row = q * 32 + lane;                // weight row inside the tile
  const uint32_t t_lane0 = tmem + (static_cast<uint32_t>(q * 32) << 16);
  const int epi_tid = threadIdx.x - 64;
  // pair: this CTA's rows are the weight row blocks pair_rb after the first CTA's, and
  // both CTAs' epilogues release an accumulator on the first CTA's barrier
  const int rank = C::kPair ? static_cast<int>(cluster_ctarank()) : 0;
  auto release_acc = [&](int b) {
    if constexpr (C::kPair) mbar_arrive_cluster(mapa_shared(smem_u32(&sh.acc_empty[b]), 0));
    else mbar_arrive(&sh.acc_empty[b]);
  };
  float sx = 1.f, sh_scale = 1.f;
  if constexpr (kFP8) {
    // written by other CTAs (or kernels): read from L2, not a possibly stale L1 line
    sx = fp8_scale_from_amax(__ldcg(a.amax_x), a.f8);
    if constexpr (!kGateUp) sh_scale = fp8_scale_from_amax(__ldcg(a.amax_h), a.f8);
  }
  const int n_units = src.count();
  for (int i = 0; i < n_units && !es.failed; ++i) {
    const Unit un = src.unit(i, rg.n_cap);
    if (!un.ok) {
      if (epi_tid == 0) report_error(a.err, kErrBadTile);
      continue;
    }
    // One thread waits; the named barrier hands the outcome to the other epilogue
    // threads, so that all of them leave together if the wait gives up. Flag and column-table
    // slots alternate per unit: no thread can be two units ahead of another.
    volatile int* okf = sh.flags + 2 + (es.iter & 1);
    int* s_tok = sh.col_tok + 256 * (es.iter & 1);
    float* s_w = sh.col_w + 256 * (es.iter & 1);
    if constexpr (!kGateUp) {
      // token row and scaled routing weight of every column, once per unit, while
      // the MMAs still run
      float scale = 1.f;
      if constexpr (kFP8) scale = __ldg(a.w_scales + un.t.expert * 3 + 2) * sh_scale;
      for (int j = epi_tid; j < un.t.n_valid; j += kEpiThreads) hk.column(un, j, scale, s_tok[j], s_w[j]);
    }
    const int buf = rg.nbuf == 2 ? (es.iter & 1) : 0;
    const uint32_t acc_phase = rg.nbuf == 2 ? ((es.iter >> 1) & 1) : (es.iter & 1);
    const uint32_t t_lane = t_lane0 + rg.buf_col * buf;
    ++es.iter;
    if (epi_tid == 0) *okf = mbar_wait_bounded(&sh.acc_full[buf], acc_phase, abort_flag, wait_budget(a)) ? 1 : 0;
    named_bar_sync(1, kEpiThreads);
    if (*okf == 0) {
      if (epi_tid == 0) {
        report_error(a.err, kErrWaitAccFull);
        *abort_flag = 1;
      }
      es.failed = true;
      break;
    }
    tc_fence_after();
    const int n_valid = un.t.n_valid;
    const int e = un.t.expert;
    // this warp's chunks c = grp, grp + kEpiGroups, ... < nchunks; the accumulator is
    // released after the last of them is read (at once when there is none)
    const int nchunks = (n_valid + 15) >> 4;
    const int my_last = nchunks - 1 < grp ? -1 : grp + (nchunks - 1 - grp) / kEpiGroups * kEpiGroups;
    if (my_last < 0) {
      tc_fence_before();
      __syncwarp();
      if (lane == 0) release_acc(buf);
    }

    if constexpr (kGateUp) {
      const int col = (un.t.fblock * a.rb_step + rank * a.pair_rb) * kTileRows + row;
      float sg = 1.f, su = 1.f;
      if constexpr (kFP8) {
        sg = __ldg(a.w_scales + e * 3 + 0) * sx;
        su = __ldg(a.w_scales + e * 3 + 1) * sx;
      }
      const bool split = un.S > 1;
      const size_t ld_ws = static_cast<size_t>(2) * a.I;
      for (int c = grp; c < nchunks; c += kEpiGroups) {
        const int c0 = c * 16;
        float g[16], v[16];
        __syncwarp();
        tmem_ld16(t_lane + c0, g);
        tmem_ld16(t_lane + rg.up_col + c0, v);
        tmem_ld_wait();
        if (c == my_last) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(buf);
        }
        #pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int n = c0 + j;
          if (n < n_valid) {
            const size_t r = static_cast<size_t>(un.t.row_start + n);
            if (split) {
              red_add_f32(a.ws1 + r * ld_ws + col, g[j]);
              red_add_f32(a.ws1 + r * ld_ws + a.I + col, v[j]);
            } else {
              const float hv = silu(g[j] * sg) * (v[j] * su);
              const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
              a.h[r * a.I + col] = hb;
              if constexpr (kFP8) es.lmax = fmaxf(es.lmax, fabsf(__bfloat162float(hb)));
            }
          }
        }
      }
      bool wrote = !split;
      if (split) {
        // the last of the splits of this tile finishes it from the partial sums
        __threadfence();
        named_bar_sync(1, kEpiThreads);
        if (epi_tid == 0) {
          const int ctr = C::kPair ? 2 * un.tile + rank : un.tile;   // a pair's CTAs finish their own rows
          const int old = atomicAdd(a.tile_counters + ctr, 1);
          const int last = (old == un.S - 1) ? 1 : 0;
          if (last) a.tile_counters[ctr] = 0;
          sh.flags[1] = last;
        }
        named_bar_sync(1, kEpiThreads);
        if (sh.flags[1]) {
          wrote = true;
          __threadfence();
          // 8 columns per batch: all 16 loads (L2, bypassing L1) are in flight together;
          // the warps of a quadrant take turns over the batches
          for (int n0 = 8 * grp; n0 < n_valid; n0 += 8 * kEpiGroups) {
            float gs[8], us[8];
            #pragma unroll
            for (int j = 0; j < 8; ++j) {
              gs[j] = 0.f;
              us[j] = 0.f;
              if (n0 + j < n_valid) {
                const float* pg = a.ws1 + static_cast<size_t>(un.t.row_start + n0 + j) * ld_ws + col;
                gs[j] = __ldcg(pg);
                us[j] = __ldcg(pg + a.I);
              }
            }
            #pragma unroll
            for (int j = 0; j < 8; ++j) {
              if (n0 + j < n_valid) {
                const size_t r = static_cast<size_t>(un.t.row_start + n0 + j);
                float* pg = a.ws1 + r * ld_ws + col;
                __stcg(pg, 0.f);
                __stcg(pg + a.I, 0.f);
                const float hv = silu(gs[j] * sg) * (us[j] * su);
                const __nv_bfloat16 hb = __float2bfloat16_rn(hv);
                a.h[r * a.I + col] = hb;
                if constexpr (kFP8) es.lmax = fmaxf(es.lmax, fabsf(__bfloat162float(hb)));
              }
            }
          }
        }
      }
      if constexpr (Hooks::kSignalTiles) {
        if (wrote) hk.tile_done(un, epi_tid, es.lmax);
      }
    } else {
      // rows of the first weight block go to features rb*128 + row, the second block's
      // to (rb + 1)*128 + row, when that block exists (H/128 odd: the last tile has one)
      const int rb = un.t.fblock * a.rb_step + rank * a.pair_rb;
      const int col0 = rb * kTileRows + row;
      const bool has2 = (rb + 1) * kTileRows < a.H;
      for (int c = grp; c < nchunks; c += kEpiGroups) {
        const int c0 = c * 16;
        float y[16], y2[16];
        __syncwarp();
        tmem_ld16(t_lane + c0, y);
        tmem_ld16(t_lane + rg.up_col + c0, y2);
        tmem_ld_wait();
        if (c == my_last) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(buf);
        }
        #pragma unroll
        for (int j = 0; j < 16; ++j)
          if (c0 + j < n_valid) {
            float* dst = a.acc + static_cast<size_t>(s_tok[c0 + j]) * a.H + col0;
            red_add_f32(dst, y[j] * s_w[c0 + j]);
            if (has2) red_add_f32(dst + kTileRows, y2[j] * s_w[c0 + j]);
          }
      }
      if constexpr (Hooks::kTokenCompletion) hk.down_done(un, s_tok, epi_tid);
    }
  }
}

// FP8 gate_up: fold this thread's max |h| into the global amax word.
__device__ __forceinline__ void publish_amax(unsigned* amax, float lmax, int lane) {
  #pragma unroll
  for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o));
  if (lane == 0 && lmax > 0.f) atomicMax(amax, __float_as_uint(lmax));
}

}  // namespace pipe
}  // namespace moe
