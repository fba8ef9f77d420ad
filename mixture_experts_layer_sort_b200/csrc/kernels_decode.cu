// kernels_decode.cu - the whole MoE layer for a decode batch (M <= 64 tokens, bf16 or
// FP8) in ONE persistent, cooperative launch: routing, the grouping of (token, slot)
// pairs by expert, the gate_up GEMM with SwiGLU, the down GEMM with the routing-weight
// scatter-add, and the conversion of the finished token rows to bf16.
//
// Fused MoE kernels "combine routing, data movement and expert calculations into
// fewer GPU operations", cutting launch overhead and intermediate traffic
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels"). At decode sizes the weights of the selected
// experts are the only large traffic, and what decides the time is how soon after the
// launch they start streaming and how little waiting is left once they have arrived.
//
// How one launch replaces the chain, per CTA (one per SM, all resident):
// - Every CTA routes all M tokens itself (the logits are staged in shared memory
//   first, so that the loads overlap) and builds the grouping and both unit schedules
//   in shared memory: no CTA waits for another to learn the routing. The order inside
//   an expert (ascending token, i.e. ascending pair id) comes from a per-expert 64-bit
//   token mask.
// - gate_up streams weights at once. Its activation operand is read straight from
//   the token rows with one-row TMA boxes (no gathered copy): bf16 layers read x;
//   FP8 layers read e4m3/e5m2 codes of x that CTA t writes for token t once every
//   token's max |x| is in (two grid counters the producer waits on, bounded, while
//   the first weight tiles are already in flight).
// - Each finished gate_up tile bumps its expert's "h ready" counter (and, FP8, a
//   global count of finished tiles after folding its max |h| into the amax word).
// - A CTA moves on to its down units as soon as it has issued its gate_up work:
//   W_down streams in while other CTAs finish gate_up. bf16: a down unit's activation
//   loads wait until every gate_up tile of its expert is done. FP8: s_h needs every
//   h row, so once all gate_up tiles are done each CTA converts its share of the h
//   rows to codes, and the down activation loads wait for all shares (the FP8 h
//   quantisation of the chain, without its launch or its extra pass over h).
// - The down epilogue adds into the fp32 accumulator and counts, per token, the K
//   blocks added so far; the CTA that completes a token converts its row to bf16 and
//   re-zeroes it. The last CTA to finish resets the counters.
// All CTAs must be resident at once (they wait on each other): the launch is
// cooperative, one CTA per SM. Every wait is bounded and reports through the error
// word when it gives up.
#include "decode_sched.cuh"
#include "fp8_format.cuh"
#include "gemm_pipeline.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

using namespace pipe;

// Global sync words (zero between launches; the last CTA resets them):
enum SyncSlot : int {
  kSyncDone = 0,       // CTAs that finished everything
  kSyncGateDone = 1,   // FP8: gate_up tiles finished (all experts)
  kSyncXMax = 2,       // FP8: tokens whose max |x| is folded into the amax word
  kSyncXq = 3,         // FP8: token rows of x quantised
  kSyncHq = 4,         // FP8: CTAs that converted their share of h
  kSyncAmaxX = 5,      // FP8: max |x| (float bits)
  kSyncAmaxH = 6,      // FP8: max |h| (float bits)
  kSyncFixed = 8       // then expert_ready [E], then token K-block counts [M]
};

struct DecodeArgs {
  const float* logits;
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  int M, E, k, H, I, P;
  int ws1_rows_cap, max_stages, f8, uniform;
  int* sync;
  uint8_t* xq;             // FP8: [M, H] codes of x
  uint8_t* hq;             // FP8: [rows, I] codes of h (the down GEMM's activation)
  // copies of the routing for inspection (written by CTA 0 at the end)
  int* topk_ids;
  float* topk_w;
  int* counts;
  int* padded_offsets;
  int* padded_pairs;
  int* header;
  float* last_scales;      // FP8: s_x, s_h of this forward
  GemmArgs g1, g2;
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Bounded wait of one thread until *p >= target (acquire); false when it gave up.
__device__ __forceinline__ bool wait_counter(const int* p, int target, volatile int* abort_flag) {
  if (ld_acquire(p) >= target) return true;
  const long long t0 = clock64();
  while (true) {
    __nanosleep(64);
    if (ld_acquire(p) >= target) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > (1ll << 31)) return false;
  }
}

// Warp-uniform: lane 0 checks *p >= target (acquire); every lane gets the answer, and
// on success every lane orders its later TMA reads after the producers' writes.
__device__ __forceinline__ bool warp_poll(const int* p, int target) {
  int v = 0;
  if ((threadIdx.x & 31) == 0) v = ld_acquire(p) >= target ? 1 : 0;
  v = __shfl_sync(0xFFFFFFFFu, v, 0);
  if (v) fence_proxy_async_global();
  return v != 0;
}

// Bounded spin of the producer warp on a condition read by lane 0.
template <class F>
__device__ __forceinline__ bool spin_until(F cond, volatile int* abort_flag) {
  const long long t0 = clock64();
  while (true) {
    int ok = 0;
    if ((threadIdx.x & 31) == 0) ok = cond() ? 1 : 0;
    ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
    if (ok) return true;
    if (*abort_flag) return false;
    if (clock64() - t0 > (1ll << 31)) return false;
    __nanosleep(32);
  }
}

// gate_up: activation rows are token rows of x (bf16) or of its codes (FP8; ready
// once all M rows are written).
template <bool kFP8>
struct GateUpHooks {
  const DecodeArgs* d;
  const Sched* s;
  int* expert_ready;
  volatile int* abort_flag;
  bool xready = !kFP8;
  static constexpr bool kSignalTiles = true;
  static constexpr bool kTokenCompletion = false;
  __device__ __forceinline__ bool direct() const { return true; }
  __device__ __forceinline__ int direct_token(const Unit& un, int j) const {
    return s->pairs[s->off[un.t.expert] + j] / d->k;
  }
  __device__ __forceinline__ int dep(const Unit&) const { return 0; }
  __device__ __forceinline__ bool ready(int) {
    if (!xready) xready = warp_poll(d->sync + kSyncXq, d->M);
    return xready;
  }
  __device__ __forceinline__ bool wait(int dd) {
    if (ready(dd)) return true;
    const int* p = d->sync + kSyncXq;
    const int m = d->M;
    if (!spin_until([p, m]() { return ld_acquire(p) >= m; }, abort_flag)) return false;
    return ready(dd);
  }
  __device__ __forceinline__ void column(const Unit&, int, float, int&, float&) const {}
  // every epilogue thread: its h stores of the tile (and, FP8, its max |h| so far) are
  // visible, also to TMA reads, before the counters move
  __device__ __forceinline__ void tile_done(const Unit& un, int epi_tid, float lmax) {
    if constexpr (kFP8) {
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) lmax = fmaxf(lmax, __shfl_xor_sync(0xFFFFFFFFu, lmax, o));
      if ((threadIdx.x & 31) == 0 && lmax > 0.f)
        atomicMax(reinterpret_cast<unsigned*>(d->sync + kSyncAmaxH), __float_as_uint(lmax));
    }
    fence_proxy_async_global();
    __threadfence();
    named_bar_sync(1, kEpiThreads);
    if (epi_tid == 0) {
      __threadfence();
      atomicAdd(expert_ready + un.t.expert, 1);
      if constexpr (kFP8) atomicAdd(d->sync + kSyncGateDone, 1);
    }
  }
  __device__ __forceinline__ void down_done(const Unit&, const int*, int) {}
};

// down: activation rows of expert e come from h (bf16: complete once all its gate_up
// tiles are done) or from its codes (FP8: complete once every CTA converted its
// share); tokens are converted by whoever adds their last K block.
template <bool kFP8>
struct DownHooks {
  const DecodeArgs* d;
  Sched* s;
  int* expert_ready;
  int* token_cnt;
  int fb1, need, grid;   // gate_up tiles per expert; K blocks added per token; CTAs
  volatile int* abort_flag;
  int last_ready = -1;
  static constexpr bool kSignalTiles = false;
  static constexpr bool kTokenCompletion = true;
  __device__ __forceinline__ bool direct() const { return false; }
  __device__ __forceinline__ int direct_token(const Unit&, int) const { return 0; }
  __device__ __forceinline__ int dep(const Unit& un) const { return kFP8 ? 0 : un.t.expert; }
  __device__ __forceinline__ bool ready(int e) {
    if (e == last_ready) return true;
    const bool v = kFP8 ? warp_poll(d->sync + kSyncHq, grid) : warp_poll(expert_ready + e, fb1);
    if (v) last_ready = e;
    return v;
  }
  __device__ __forceinline__ bool wait(int e) {
    if (ready(e)) return true;
    const int* p = kFP8 ? d->sync + kSyncHq : expert_ready + e;
    const int f = kFP8 ? grid : fb1;
    if (!spin_until([p, f]() { return ld_acquire(p) >= f; }, abort_flag)) return false;
    return ready(e);
  }
  __device__ __forceinline__ void column(const Unit& un, int j, float scale, int& tok, float& w) const {
    const int p = s->pairs[s->off[un.t.expert] + j];
    tok = p / d->k;
    w = s->w[p] * scale;
  }
  __device__ __forceinline__ void tile_done(const Unit&, int, float) {}
  __device__ __forceinline__ void down_done(const Unit& un, const int* s_tok, int epi_tid) {
    __threadfence();                        // this unit's adds happen before the counts move
    named_bar_sync(1, kEpiThreads);
    if (epi_tid == 0) s->ndone = 0;
    named_bar_sync(1, kEpiThreads);
    const int add = un.kb1 - un.kb0;
    for (int j = epi_tid; j < un.t.n_valid; j += kEpiThreads) {
      const int t = s_tok[j];
      if (atomicAdd(token_cnt + t, add) == need - add) s->done[atomicAdd(&s->ndone, 1)] = t;
    }
    named_bar_sync(1, kEpiThreads);
    const int nd = s->ndone;
    if (nd > 0) {
      __threadfence();
      const int H = d->H;
      for (int i = 0; i < nd; ++i) {
        const int t = s->done[i];
        float4* acc4 = reinterpret_cast<float4*>(d->g2.acc + static_cast<size_t>(t) * H);
        uint2* out4 = reinterpret_cast<uint2*>(d->out + static_cast<size_t>(t) * H);
        for (int c = epi_tid; c < H / 4; c += kEpiThreads) {
          const float4 v = __ldcg(acc4 + c);
          __stcg(acc4 + c, make_float4(0.f, 0.f, 0.f, 0.f));
          const __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
          const __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
          uint2 o;
          o.x = *reinterpret_cast<const unsigned*>(&lo);
          o.y = *reinterpret_cast<const unsigned*>(&hi);
          out4[c] = o;
        }
        if (epi_tid == 0) token_cnt[t] = 0;
      }
    }
    named_bar_sync(1, kEpiThreads);         // s->done is reused by the next unit
  }
};

// 8 fp32 values -> 8 FP8 codes (RNE, saturating), v[i] / s correctly rounded.
__device__ __forceinline__ uint2 quant8(const float (&v)[8], const ScaleDiv& dv, int f8) {
  unsigned short c[4];
  #pragma unroll
  for (int q = 0; q < 4; ++q) c[q] = fp8x2(make_float2(dv(v[2 * q]), dv(v[2 * q + 1])), f8);
  uint2 r;
  r.x = static_cast<unsigned>(c[0]) | (static_cast<unsigned>(c[1]) << 16);
  r.y = static_cast<unsigned>(c[2]) | (static_cast<unsigned>(c[3]) << 16);
  return r;
}

// One row of n bf16 values -> codes, by the 128 epilogue threads (n % 8 == 0).
__device__ __forceinline__ void quant_row(const __nv_bfloat16* src, uint8_t* dst, int n, float s, int f8,
                                          int epi_tid) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint2* d2 = reinterpret_cast<uint2*>(dst);
  const ScaleDiv dv(s);
  for (int i = epi_tid; i < n / 8; i += kEpiThreads) {
    const uint4 u = __ldcg(s4 + i);
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
    float f[8];
    #pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float2 v = __bfloat1622float2(p[q]);
      f[2 * q] = v.x;
      f[2 * q + 1] = v.y;
    }
    d2[i] = quant8(f, dv, f8);
  }
}

template <bool kFP8>
__global__ void __launch_bounds__(kThreads, 1)
    fused_decode_kernel(const __grid_constant__ DecodeArgs d, const __grid_constant__ CUtensorMap tm_w13,
                        const __grid_constant__ CUtensorMap tm_wd, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_h) {
  using C = Cfg<kFP8>;
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve<C>(smem_raw, sizeof(Sched));
  Sched* s = reinterpret_cast<Sched*>(sh.extra);
  volatile int* abort_flag = sh.flags;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int G = gridDim.x;
  const int c = blockIdx.x;
  const int E = d.E, M = d.M, k = d.k, P = d.P;
  int* expert_ready = d.sync + kSyncFixed;
  int* token_cnt = expert_ready + E;
  if (tid == 0) {
    tma_prefetch_desc(&tm_w13);
    tma_prefetch_desc(&tm_wd);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_h);
  }
  const uint32_t tmem = prologue<C>(sh, warp);

  // ---------------------------------------------------------------- routing, in every CTA
  // the logits go to shared memory first (all loads in flight together), staged in the
  // stage ring, which is not in use yet (M * E * 4 <= 128 KB < ring bytes)
  float* s_logits = reinterpret_cast<float*>(sh.ring);
  const int n_logits = M * E;
  for (int i0 = tid; i0 < n_logits; i0 += kThreads * 8) {
    float v[8];
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j * kThreads < n_logits) v[j] = __ldg(d.logits + i0 + j * kThreads);
    #pragma unroll
    for (int j = 0; j < 8; ++j)
      if (i0 + j * kThreads < n_logits) s_logits[i0 + j * kThreads] = v[j];
  }
  if constexpr (kFP8) {
    // CTA t < M: max |x| of token t into the amax word
    if (c < M) {
      const uint4* xr = reinterpret_cast<const uint4*>(d.x + static_cast<size_t>(c) * d.H);
      float m = 0.f;
      for (int i = tid; i < d.H / 8; i += kThreads) {
        const uint4 u = __ldg(xr + i);
        const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&u);
        #pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float2 f = __bfloat1622float2(p[q]);
          m = fmaxf(m, fmaxf(fabsf(f.x), fabsf(f.y)));
        }
      }
      #pragma unroll
      for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      if (lane == 0) s->red[warp] = m;
    }
  }
  sched_clear(s, E, tid, kThreads);
  __syncthreads();
  if constexpr (kFP8) {
    if (c < M && tid == 0) {
      float m = 0.f;
      for (int w = 0; w < kThreads / 32; ++w) m = fmaxf(m, s->red[w]);
      if (m > 0.f) atomicMax(reinterpret_cast<unsigned*>(d.sync + kSyncAmaxX), __float_as_uint(m));
      __threadfence();
      atomicAdd(d.sync + kSyncXMax, 1);
    }
  }
  for (int t = warp; t < M; t += kThreads / 32)
    route_token_any(s_logits + static_cast<size_t>(t) * E, E, k, lane, s->ids + t * k, s->w + t * k);
  __syncthreads();
  const int fb1 = d.I / kTileRows;
  const int fb2 = (d.H / kTileRows + 1) / 2;
  const int kb1 = d.H / C::kKPerBlock;
  const int kb2 = d.I / C::kKPerBlock;
  sched_build(s, P, E, k, fb1, fb2, kb1, kb2, G, d.ws1_rows_cap, d.uniform, tid, kThreads);
  // the staged logits are dead from here on: order their generic-proxy accesses before
  // the TMA writes that reuse the ring
  fence_proxy_async_smem();
  __syncthreads();   // the schedule is complete

  // ---------------------------------------------------------------- both GEMMs
  const Ring rg = make_ring<C>(s->n_max, d.max_stages, sh.ring_bytes);
  const UnitSchedule<SmemTileFn<Sched>> src1(SmemTileFn<Sched>{s, fb1}, s->T1, s->S1, kb1);
  const UnitSchedule<SmemTileFn<Sched>> src2(SmemTileFn<Sched>{s, fb2}, s->T2, s->S2, kb2);
  GateUpHooks<kFP8> h1{&d, s, expert_ready, abort_flag};
  DownHooks<kFP8> h2{&d, s, expert_ready, token_cnt, fb1, k * fb2 * kb2, G, abort_flag};

  if (warp == 0) {
    ProducerState ps;
    run_producer<C>(d.g1, &tm_w13, &tm_x, sh, rg, src1, h1, ps, abort_flag, lane);
    if (!ps.failed) run_producer<C>(d.g2, &tm_wd, &tm_h, sh, rg, src2, h2, ps, abort_flag, lane);
    producer_quiesce<C>(sh, rg, ps, lane);
  } else if (warp == 1) {
    if (lane == 0) {
      MmaState ms;
      run_mma<C, kFP8>(d.g1, sh, rg, src1, ms, tmem, abort_flag);
      if (!ms.failed) run_mma<C, kFP8>(d.g2, sh, rg, src2, ms, tmem, abort_flag);
      mma_drain<C>(sh, ms);
    }
  } else {
    const int epi_tid = tid - 64;
    volatile int* okf = sh.flags + 2;
    bool ok = true;
    if constexpr (kFP8) {
      // x codes: once every token's max |x| is in, CTA t < M quantises token row t;
      // every CTA needs the final amax before its gate_up epilogue scales by s_x
      if (epi_tid == 0) *okf = wait_counter(d.sync + kSyncXMax, M, abort_flag) ? 1 : 0;
      named_bar_sync(1, kEpiThreads);
      ok = *okf != 0;
      if (ok && c < M) {
        const float sx = fp8_scale_from_amax(__ldcg(reinterpret_cast<const unsigned*>(d.sync + kSyncAmaxX)), d.f8);
        quant_row(d.x + static_cast<size_t>(c) * d.H, d.xq + static_cast<size_t>(c) * d.H, d.H, sx, d.f8, epi_tid);
        fence_proxy_async_global();
        __threadfence();
        named_bar_sync(1, kEpiThreads);
        if (epi_tid == 0) atomicAdd(d.sync + kSyncXq, 1);
      }
      if (!ok && epi_tid == 0) {
        report_error(d.g1.err, kErrWaitGrid);
        *abort_flag = 1;
      }
    }
    EpiState es;
    es.failed = !ok;
    if (ok) run_epilogue<C, true, kFP8>(d.g1, sh, rg, src1, h1, es, tmem, abort_flag, warp, lane);
    if constexpr (kFP8) {
      // h codes: s_h is final once every gate_up tile is done; this CTA converts the
      // valid h rows c, c + G, ...
      if (!es.failed) {
        named_bar_sync(1, kEpiThreads);
        if (epi_tid == 0) *okf = wait_counter(d.sync + kSyncGateDone, s->T1, abort_flag) ? 1 : 0;
        named_bar_sync(1, kEpiThreads);
        if (*okf == 0) {
          if (epi_tid == 0) {
            report_error(d.g1.err, kErrWaitGrid);
            *abort_flag = 1;
          }
          es.failed = true;
        }
      }
      if (!es.failed) {
        const float shs = fp8_scale_from_amax(__ldcg(reinterpret_cast<const unsigned*>(d.sync + kSyncAmaxH)), d.f8);
        for (int r = c; r < s->rows_used; r += G) {
          int lo = 0, hi = s->nact - 1;                 // active expert whose padded rows hold r
          while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (s->poff[s->act[mid]] <= r) lo = mid;
            else hi = mid - 1;
          }
          const int e = s->act[lo];
          if (r - s->poff[e] >= s->count[e]) continue;  // a pad row: never read by a stored column
          quant_row(d.g1.h + static_cast<size_t>(r) * d.I, d.hq + static_cast<size_t>(r) * d.I, d.I, shs, d.f8,
                    epi_tid);
        }
        fence_proxy_async_global();
        __threadfence();
        named_bar_sync(1, kEpiThreads);
        if (epi_tid == 0) atomicAdd(d.sync + kSyncHq, 1);
      }
    }
    if (!es.failed) run_epilogue<C, false, kFP8>(d.g2, sh, rg, src2, h2, es, tmem, abort_flag, warp, lane);
  }
  teardown<C>(tmem, warp);

  // ---------------------------------------------------------------- copies for inspection
  if (c == 0) {
    for (int p = tid; p < P; p += kThreads) {
      d.topk_ids[p] = s->ids[p];
      d.topk_w[p] = s->w[p];
    }
    sched_publish(s, P, E, d.counts, d.padded_offsets, d.padded_pairs, d.header, tid, kThreads);
    if (tid == 0) {
      if constexpr (kFP8) {
        d.last_scales[0] = fp8_scale_from_amax(__ldcg(reinterpret_cast<const unsigned*>(d.sync + kSyncAmaxX)), d.f8);
        d.last_scales[1] = fp8_scale_from_amax(__ldcg(reinterpret_cast<const unsigned*>(d.sync + kSyncAmaxH)), d.f8);
      }
    }
  }

  // ---------------------------------------------------------------- last CTA resets
  __syncthreads();
  if (tid == 0) {
    __threadfence();
    s->flag = atomicAdd(d.sync + kSyncDone, 1) == G - 1 ? 1 : 0;
  }
  __syncthreads();
  if (s->flag) {
    __threadfence();
    for (int e = tid; e < E; e += kThreads) expert_ready[e] = 0;
    for (int t = tid; t < M; t += kThreads) token_cnt[t] = 0;
    if (tid == 0) {
      for (int i = 1; i < kSyncFixed; ++i) d.sync[i] = 0;
      __threadfence();
      d.sync[kSyncDone] = 0;
    }
  }
}

}  // namespace

bool decode_supported(int M, int E, int k) { return sched_supported(M, E, k); }

size_t decode_sync_words(int E, int M_cap) { return static_cast<size_t>(kSyncFixed + E + M_cap); }

cudaError_t decode_configure() {
  cudaError_t e = cudaFuncSetAttribute(fused_decode_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       Cfg<false>::kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(fused_decode_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<true>::kSmemBytes);
}

cudaError_t launch_decode(const DecodeLaunch& l, cudaStream_t st) {
  DecodeArgs d{};
  d.logits = l.logits;
  d.x = l.x;
  d.out = l.out;
  d.M = l.M;
  d.E = l.E;
  d.k = l.k;
  d.H = l.H;
  d.I = l.I;
  d.P = l.M * l.k;
  d.ws1_rows_cap = l.ws1_rows_cap;
  d.max_stages = l.max_stages;
  d.f8 = l.f8;
  d.uniform = uniform_splits() ? 1 : 0;
  d.sync = l.sync;
  d.xq = l.xq;
  d.hq = l.hq;
  d.topk_ids = l.topk_ids;
  d.topk_w = l.topk_w;
  d.counts = l.counts;
  d.padded_offsets = l.padded_offsets;
  d.padded_pairs = l.padded_pairs;
  d.header = l.header;
  d.last_scales = l.last_scales;
  d.g1 = l.g1;
  d.g2 = l.g2;
  // the FP8 amax words live in the sync block (reset by the kernel's last CTA)
  d.g1.amax_x = d.g2.amax_x = reinterpret_cast<unsigned*>(l.sync + kSyncAmaxX);
  d.g1.amax_h = d.g2.amax_h = reinterpret_cast<unsigned*>(l.sync + kSyncAmaxH);
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = l.fp8 ? Cfg<true>::kSmemBytes : Cfg<false>::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  if (l.fp8) return cudaLaunchKernelEx(&cfg, fused_decode_kernel<true>, d, *l.tm_w13, *l.tm_wd, *l.tm_x, *l.tm_h);
  return cudaLaunchKernelEx(&cfg, fused_decode_kernel<false>, d, *l.tm_w13, *l.tm_wd, *l.tm_x, *l.tm_h);
}

}  // namespace moe
