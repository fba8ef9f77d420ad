// kernels_gemm.cu - the two grouped GEMMs of the MoE layer on 5th-generation
// tensor cores (tcgen05, accumulators in TMEM, operands staged by TMA).
//
// Orientation: every tile is "swap-AB". The expert's weight rows fill the MMA's
// M = 128 slot and the expert's few tokens are the N dimension (16..BN), i.e.
// the kernel computes D^T = W * X^T instead of X * W^T. The identity
// (A B)^T = B^T A^T changes no arithmetic (kongchang.com, "MoE Kernel
// Engineering Optimization Practices on Amazon SageMaker AI", section "Swap-AB:
// Making WGMMA Run at Full Utilization"); it keeps the tensor-core rows busy
// when decode gives an expert only a handful of tokens (toolboxkart.tech, "AWS
// SageMaker MoE kernel optimizations H200", section "1. Swap-AB makes better use
// of the WGMMA tile"; aib.vote, "AWS SageMaker MoE kernel optimizations", second
// paragraph). On sm_100 the N dimension reaches 256, so the same orientation also
// covers prefill, where an expert holds ~128-256 tokens.
//
// gate_up (GEMM1): per tile, 128 rows of W_gate and the same 128 rows of W_up go
// to two TMEM accumulators [128 x N]; the epilogue forms h = silu(g) * u and
// stores it as bf16 ("fuses scaling, matrix multiplication ... into one GPU pass",
// aib.vote page, third paragraph). down (GEMM2): 128 rows of W_down times h; the
// epilogue multiplies by the routing weight (and the FP8 scales) and
// scatter-adds into the fp32 token accumulator with red.global.add ("expert
// aggregation").
//
// Work units: the tiles from the align kernel, each optionally split along K
// (split-K) so that small decode batches still stream weights through all SMs.
// A persistent grid of one CTA per SM walks units blockIdx.x, +gridDim.x, ...
// Warp roles: warp 0 = TMA producer, warp 1 = TMEM owner + MMA issuer,
// warps 2-5 = epilogue (TMEM lanes 32*(warp%4) .. +31).
#include <cuda_fp8.h>

#include "moe_internal.h"
#include "sm100.cuh"

namespace moe {

namespace {

constexpr int kThreads = 192;
constexpr int kEpiThreads = 128;

template <bool kGateUp, bool kFP8, int BN>
struct Cfg {
  // two 128-row weight tiles per stage share one activation tile: W_gate and W_up
  // rows of the same features (gate_up), or two consecutive 128-row blocks of
  // W_down (down), so each activation byte brought in feeds 256 weight rows
  static constexpr int kATiles = 2;
  static constexpr int kABytes = kTileRows * kRowBytes;            // 16 KB per weight tile
  static constexpr int kAccCols = 2 * BN;
  static constexpr int kTmemCols = 512;   // two accumulator buffers of up to 256 columns
  // shared memory: [alignment slack][1 KB barriers and flags][stage ring]
  static constexpr int kSmemBytes = 232448;                         // the sm_100 opt-in maximum
  // [0, 1 KB): barriers and flags; [1 KB, 3 KB): two slots of the down epilogue's
  // per-column token row (int, 256 columns each); [3 KB, 5 KB): two slots of its
  // scaled routing weights (float); the stage ring starts at 6 KB (1024-aligned)
  static constexpr int kColTableOffset = 1024;
  static constexpr int kColTableBytes = 2 * 2 * 256 * 4;
  static constexpr int kBarrierBytes = 6144;
  static constexpr int kRingBytes = kSmemBytes - 1024 - kBarrierBytes;
  static constexpr int kMaxStages = 16;
  static constexpr int kKPerBlock = kFP8 ? 128 : 64;                // elements in one 128-byte row
  static constexpr int kMmaKBytes = 32;                             // K of one MMA = 32 bytes
  static constexpr int kMmasPerBlock = kRowBytes / kMmaKBytes;
  static_assert(kAccCols <= 512, "TMEM holds 512 columns");
  static_assert(BN % 16 == 0 && BN >= 16 && BN <= 256, "N of an M=128 MMA");
  static_assert(2 * kMaxStages * 8 + 32 + 4 + 16 <= kColTableOffset, "barrier area");
  static_assert(kColTableOffset + kColTableBytes <= kBarrierBytes && kBarrierBytes % 1024 == 0,
                "column tables must end before the 1024-aligned stage ring");
  static_assert(kATiles * kABytes + BN * kRowBytes <= kRingBytes / 2, "at least two stages");
};

// Stage size from the widest token tile of this forward (the align kernel writes it
// to the header): a stage holds the weight tile(s) plus n_max rows of activations,
// so thin decode batches get a deeper ring than prefill.
template <class C>
__device__ __forceinline__ void ring_geometry(int n_max, int BN, int max_stages, int& n_cap, int& stage_bytes,
                                              int& stages) {
  const int n = n_max < 16 ? 16 : (n_max > BN ? BN : ((n_max + 15) & ~15));
  n_cap = n;
  stage_bytes = (C::kATiles * C::kABytes + n * kRowBytes + 1023) & ~1023;
  stages = C::kRingBytes / stage_bytes;
  if (stages > C::kMaxStages) stages = C::kMaxStages;
  if (max_stages >= 2 && stages > max_stages) stages = max_stages;
}

struct Unit {
  Tile t;
  int kb0, kb1;
  bool ok;
};

// A unit whose token tile does not fit the stage (n_cap rows) or the accumulator is
// rejected identically by every role, so no role waits for work another skipped.
__device__ __forceinline__ Unit load_unit(const GemmArgs& a, int u, int S, int n_cap) {
  Unit x;
  x.t = a.tiles[u / S];
  const int s = u - (u / S) * S;
  x.kb0 = s * a.kblocks / S;
  x.kb1 = (s + 1) * a.kblocks / S;
  x.ok = x.t.n_valid >= 1 && x.t.n_valid <= n_cap && x.kb1 > x.kb0;
  return x;
}

__device__ __forceinline__ float silu(float z) { return z / (1.f + __expf(-z)); }

__device__ __forceinline__ float scale_from_amax(unsigned bits) {
  const float amax = __uint_as_float(bits);
  return amax == 0.f ? 1.f : __fdiv_rn(amax, 448.f);
}

template <bool kGateUp, bool kFP8, int BN>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs a, const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_b) {
  using C = Cfg<kGateUp, kFP8, BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* smem = base + C::kBarrierBytes;                         // stage ring, 1024-aligned
  uint64_t* full = reinterpret_cast<uint64_t*>(base);
  uint64_t* empty = full + C::kMaxStages;
  uint64_t* acc_full = empty + C::kMaxStages;   // [2]
  uint64_t* acc_empty = acc_full + 2;           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(acc_empty + 2);
  int* flags = reinterpret_cast<int*>(tmem_slot + 1);   // [0] abort, [1] last arriver, [2..3] wait outcome
  volatile int* abort_flag = flags;
  int* col_tok = reinterpret_cast<int*>(base + C::kColTableOffset);           // [2][256]
  float* col_w = reinterpret_cast<float*>(base + C::kColTableOffset + 2048);  // [2][256]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // TMEM accumulators: buffer b starts at column 256*b. Two buffers let the MMA of
  // the next unit run while the epilogue drains this one; gate_up needs two
  // accumulators (gate, up) per buffer, so it double-buffers only up to 128 tokens.

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kEpiThreads / 32);
    }
    for (int i = 0; i < 4; ++i) flags[i] = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_b);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, C::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // When the previous kernel wrote the tile list, nobody reads it before waiting.
  if (a.wait_first) {
    pdl_wait();
    pdl_trigger();
  }
  int n_cap, stage_bytes, STAGES;
  ring_geometry<C>(a.header[kHdrMaxRows], BN, a.max_stages, n_cap, stage_bytes, STAGES);
  // two accumulators per buffer (one per weight tile), double-buffered up to 128 tokens
  const int nbuf = n_cap <= 128 ? 2 : 1;
  const uint32_t up_col = nbuf == 2 ? 128u : 256u;

  const int T = a.header[a.hdr_tiles];
  const int S = a.header[a.hdr_splits];
  const int units = T * S;

  // Everyone but the producer warp waits for the previous kernel here. The tile list
  // and header come from the align kernel, at least two launches back, so they are
  // complete already (see pdl_wait in sm100.cuh).
  if (warp != 0 && !a.wait_first) {
    pdl_wait();
    pdl_trigger();
  }

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (one warp)
    // Lane 0 owns the stage barriers and issues the weight loads; the activation rows
    // of a stage are spread over the 32 lanes.
    const uint64_t pol_w = l2_policy_evict_first();   // weights stream through once
    const uint64_t pol_b = l2_policy_evict_last();    // activations are re-read per tile
    int stage = 0;
    uint32_t phase = 0;
    int issued = 0;
    bool failed = false;
    // Weights never depend on the previous kernel, activations do: the first
    // STAGES weight loads go out before waiting for it, their activation loads after.
    bool waited = a.wait_first != 0;
    int npend = 0;
    int pend_stage[C::kMaxStages], pend_kc[C::kMaxStages], pend_row[C::kMaxStages], pend_nb[C::kMaxStages];
    // direct mode: x row (token) of activation rows lane, lane+32, lane+64, lane+96 of
    // the current unit; pad rows re-read row 0 (their columns are never stored)
    int tok[4] = {0, 0, 0, 0};
    auto load_b = [&](int stg, int kc, int row_start, int nb) {
      uint8_t* bdst = smem + stg * stage_bytes + C::kATiles * C::kABytes;
      if (a.direct_pairs == nullptr) {
        for (int j = lane; j < nb; j += 32)
          tma_load_2d(bdst + j * 16 * kRowBytes, &tm_b, &full[stg], kc, row_start + 16 * j, pol_b);
      } else {
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = lane + 32 * i;
          if (j < nb * 16) tma_load_2d(bdst + j * kRowBytes, &tm_b, &full[stg], kc, tok[i], pol_b);
        }
      }
    };
    auto release_pending = [&]() {
      pdl_wait();
      pdl_trigger();
      waited = true;
      for (int i = 0; i < npend; ++i) load_b(pend_stage[i], pend_kc[i], pend_row[i], pend_nb[i]);
      npend = 0;
    };
    for (int u = blockIdx.x; u < units && !failed; u += gridDim.x) {
      const Unit un = load_unit(a, u, S, n_cap);
      if (!un.ok) continue;
      const int nb16 = (un.t.n_valid + 15) >> 4;
      // first tiled-weight block of the unit's two weight row blocks; a second block
      // past the end of the tensor reads zeros and is not stored by the epilogue
      const int rb0 = un.t.fblock * a.rb_step;
      const int wtile = (un.t.expert * a.w_rblocks + rb0) * a.kblocks;
      const int wtile_up = (un.t.expert * a.w_rblocks + rb0 + a.second_rb) * a.kblocks;
      const uint32_t tx = C::kATiles * C::kABytes + nb16 * 16 * kRowBytes;
      if (a.direct_pairs != nullptr) {
        #pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int j = lane + 32 * i;
          tok[i] = j < un.t.n_valid ? __ldcg(a.direct_pairs + un.t.row_start + j) / a.k : 0;
        }
      }
      for (int kb = un.kb0; kb < un.kb1; ++kb) {
        int ok = 1;
        if (lane == 0) {
          ok = mbar_wait_bounded(&empty[stage], phase ^ 1u, abort_flag) ? 1 : 0;
          if (!ok) {
            report_error(a.err, kErrWaitEmpty);
            *abort_flag = 1;
          } else {
            uint8_t* st = smem + stage * stage_bytes;
            mbar_arrive_expect_tx(&full[stage], tx);
            tma_load_2d(st, &tm_w, &full[stage], 0, (wtile + kb) * kTileRows, pol_w);
            tma_load_2d(st + C::kABytes, &tm_w, &full[stage], 0, (wtile_up + kb) * kTileRows, pol_w);
          }
        }
        ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
        if (!ok) {
          failed = true;
          break;
        }
        const int kc = kb * C::kKPerBlock;
        if (waited) {
          load_b(stage, kc, un.t.row_start, nb16);
        } else {
          pend_stage[npend] = stage;
          pend_kc[npend] = kc;
          pend_row[npend] = un.t.row_start;
          pend_nb[npend] = nb16;
          if (++npend == STAGES) release_pending();
        }
        ++issued;
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
    }
    if (!waited) release_pending();
    if (failed && lane == 0) {
      // let the copies already in flight land before the CTA's shared memory goes away
      int zero = 0;
      int st = stage, ph = static_cast<int>(phase);
      const int pending = issued < STAGES ? issued : STAGES;
      for (int i = 0; i < pending; ++i) {
        if (--st < 0) {
          st = STAGES - 1;
          ph ^= 1;
        }
        mbar_wait_bounded(&full[st], static_cast<uint32_t>(ph), &zero, 1ll << 26);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const Unit un = load_unit(a, u, S, n_cap);
        if (!un.ok) continue;
        const uint32_t n_pad = static_cast<uint32_t>((un.t.n_valid + 15) & ~15);
        const uint32_t idesc = idesc_make(kFP8 ? 0u : 1u, 128u, n_pad);
        const int buf = nbuf == 2 ? (it & 1) : 0;
        const uint32_t acc_phase = nbuf == 2 ? ((it >> 1) & 1) : (it & 1);
        const uint32_t d_tmem = tmem + 256u * buf;
        ++it;
        if (!mbar_wait_bounded(&acc_empty[buf], acc_phase ^ 1u, abort_flag)) {
          report_error(a.err, kErrWaitAccEmpty);
          *abort_flag = 1;
          break;
        }
        tc_fence_after();
        bool failed = false;
        for (int kb = un.kb0; kb < un.kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, abort_flag)) {
            report_error(a.err, kErrWaitFull);
            *abort_flag = 1;
            failed = true;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(smem + stage * stage_bytes);
          const uint32_t b0 = a0 + C::kATiles * C::kABytes;
          #pragma unroll
          for (int kk = 0; kk < C::kMmasPerBlock; ++kk) {
            const uint32_t koff = kk * C::kMmaKBytes;
            const uint32_t accum = (kb > un.kb0 || kk > 0) ? 1u : 0u;
            const uint64_t bd = sdesc_k_sw128(b0 + koff);
            if constexpr (kFP8) mma_e4m3(d_tmem, sdesc_k_sw128(a0 + koff), bd, idesc, accum);
            else mma_bf16(d_tmem, sdesc_k_sw128(a0 + koff), bd, idesc, accum);
            const uint64_t ad1 = sdesc_k_sw128(a0 + C::kABytes + koff);
            if constexpr (kFP8) mma_e4m3(d_tmem + up_col, ad1, bd, idesc, accum);
            else mma_bf16(d_tmem + up_col, ad1, bd, idesc, accum);
          }
          mma_commit(&empty[stage]);   // frees the stage once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (failed) break;
        mma_commit(&acc_full[buf]);    // accumulator complete
      }
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                       // TMEM lane quadrant of this warp
    const int row = q * 32 + lane;                // weight row inside the tile
    const uint32_t t_lane0 = tmem + (static_cast<uint32_t>(q * 32) << 16);
    const int epi_tid = threadIdx.x - 64;
    int iter = 0;
    float lmax = 0.f;
    float sx = 1.f, sh = 1.f;
    if constexpr (kFP8) {
      sx = scale_from_amax(*a.amax_x);
      if constexpr (!kGateUp) sh = scale_from_amax(*a.amax_h);
    }
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
      const Unit un = load_unit(a, u, S, n_cap);
      if (!un.ok) {
        if (epi_tid == 0) report_error(a.err, kErrBadTile);
        continue;
      }
      // One thread waits; the named barrier hands the outcome to the other 127,
      // so that all of them leave together if the wait gives up. The flag slot
      // alternates per unit: no thread can be two units ahead of another.
      volatile int* okf = flags + 2 + (iter & 1);
      int* s_tok = col_tok + 256 * (iter & 1);
      float* s_w = col_w + 256 * (iter & 1);
      if constexpr (!kGateUp) {
        // token row and scaled routing weight of every column, loaded once per unit
        // while the MMAs still run (slot alternates per unit, like okf)
        float scale = 1.f;
        if constexpr (kFP8) scale = __ldg(a.w_scales + un.t.expert * 3 + 2) * sh;
        for (int j = epi_tid; j < un.t.n_valid; j += kEpiThreads) {
          const int p = __ldg(a.padded_pairs + un.t.row_start + j);
          s_tok[j] = p / a.k;
          s_w[j] = __ldg(a.topk_w + p) * scale;
        }
      }
      const int buf = nbuf == 2 ? (iter & 1) : 0;
      const uint32_t acc_phase = nbuf == 2 ? ((iter >> 1) & 1) : (iter & 1);
      const uint32_t t_lane = t_lane0 + 256u * buf;
      ++iter;
      if (epi_tid == 0) *okf = mbar_wait_bounded(&acc_full[buf], acc_phase, abort_flag) ? 1 : 0;
      named_bar_sync(1, kEpiThreads);
      if (*okf == 0) {
        if (epi_tid == 0) {
          report_error(a.err, kErrWaitAccFull);
          *abort_flag = 1;
        }
        break;
      }
      tc_fence_after();
      const int n_valid = un.t.n_valid;
      const int e = un.t.expert;
      const int col = un.t.fblock * kTileRows + row;

      if constexpr (kGateUp) {
        float sg = 1.f, su = 1.f;
        if constexpr (kFP8) {
          sg = __ldg(a.w_scales + e * 3 + 0) * sx;
          su = __ldg(a.w_scales + e * 3 + 1) * sx;
        }
        const bool split = S > 1;
        const size_t ld_ws = static_cast<size_t>(2) * a.I;
        for (int c0 = 0; c0 < n_valid; c0 += 16) {
          float g[16], v[16];
          __syncwarp();
          tmem_ld16(t_lane + c0, g);
          tmem_ld16(t_lane + up_col + c0, v);
          tmem_ld_wait();
          if (c0 + 16 >= n_valid) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
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
                if constexpr (kFP8) lmax = fmaxf(lmax, fabsf(__bfloat162float(hb)));
              }
            }
          }
        }
        if (split) {
          // the last of the S units of this tile finishes it from the partial sums
          __threadfence();
          named_bar_sync(1, kEpiThreads);
          if (epi_tid == 0) {
            const int tile = u / S;
            const int old = atomicAdd(a.tile_counters + tile, 1);
            const int last = (old == S - 1) ? 1 : 0;
            if (last) a.tile_counters[tile] = 0;
            flags[1] = last;
          }
          named_bar_sync(1, kEpiThreads);
          if (flags[1]) {
            __threadfence();
            // 8 columns per batch: all 16 loads (L2, bypassing L1) are in flight together
            for (int n0 = 0; n0 < n_valid; n0 += 8) {
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
                  if constexpr (kFP8) lmax = fmaxf(lmax, fabsf(__bfloat162float(hb)));
                }
              }
            }
          }
        }
      } else {
        // rows of the first weight block go to features f*256 + row, the second block's
        // to f*256 + 128 + row, when that block exists (H/128 odd: the last tile has one)
        const int col0 = un.t.fblock * 2 * kTileRows + row;
        const bool has2 = (un.t.fblock * 2 + 1) * kTileRows < a.H;
        for (int c0 = 0; c0 < n_valid; c0 += 16) {
          float y[16], y2[16];
          __syncwarp();
          tmem_ld16(t_lane + c0, y);
          tmem_ld16(t_lane + up_col + c0, y2);
          tmem_ld_wait();
          if (c0 + 16 >= n_valid) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&acc_empty[buf]);
          }
          #pragma unroll
          for (int j = 0; j < 16; ++j)
            if (c0 + j < n_valid) {
              float* dst = a.acc + static_cast<size_t>(s_tok[c0 + j]) * a.H + col0;
              red_add_f32(dst, y[j] * s_w[c0 + j]);
              if (has2) red_add_f32(dst + kTileRows, y2[j] * s_w[c0 + j]);
            }
        }
      }
    }
    if constexpr (kGateUp && kFP8) {
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o));
      if (lane == 0 && lmax > 0.f) atomicMax(a.amax_h, __float_as_uint(lmax));
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem, C::kTmemCols);
  }
}

// One tile variant: up to 256 token rows per tile (the largest N of an M=128 MMA).
// Thin batches are not penalised: the stage ring and the TMEM buffering follow the
// widest token tile of the forward at run time (ring_geometry).
constexpr int kTokenTile = 256;

template <bool kGateUp, bool kFP8, int BN>
cudaError_t launch_one(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& b, int grid, cudaStream_t s) {
  using C = Cfg<kGateUp, kFP8, BN>;
  return launch_kernel(grouped_gemm_kernel<kGateUp, kFP8, BN>, dim3(grid), dim3(kThreads),
                       static_cast<size_t>(C::kSmemBytes), s, a, w, b);
}

template <bool kGateUp, bool kFP8, int BN>
cudaError_t configure_one() {
  using C = Cfg<kGateUp, kFP8, BN>;
  return cudaFuncSetAttribute(grouped_gemm_kernel<kGateUp, kFP8, BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              C::kSmemBytes);
}

template <bool kGateUp, bool kFP8>
cudaError_t launch_variant(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& b, int variant, int grid,
                           cudaStream_t s) {
  (void)variant;
  return launch_one<kGateUp, kFP8, kTokenTile>(a, w, b, grid, s);
}

template <bool kGateUp, bool kFP8>
cudaError_t configure_all() {
  return configure_one<kGateUp, kFP8, kTokenTile>();
}

}  // namespace

int variant_bn(int v) {
  (void)v;
  return kTokenTile;
}

cudaError_t gemm_configure() {
  cudaError_t e;
  if ((e = configure_all<true, false>()) != cudaSuccess) return e;
  if ((e = configure_all<true, true>()) != cudaSuccess) return e;
  if ((e = configure_all<false, false>()) != cudaSuccess) return e;
  return configure_all<false, true>();
}

cudaError_t launch_gemm1(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& x, bool fp8, int variant,
                         int grid, cudaStream_t s) {
  return fp8 ? launch_variant<true, true>(a, w, x, variant, grid, s)
             : launch_variant<true, false>(a, w, x, variant, grid, s);
}

cudaError_t launch_gemm2(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& h, bool fp8, int variant,
                         int grid, cudaStream_t s) {
  return fp8 ? launch_variant<false, true>(a, w, h, variant, grid, s)
             : launch_variant<false, false>(a, w, h, variant, grid, s);
}

}  // namespace moe
