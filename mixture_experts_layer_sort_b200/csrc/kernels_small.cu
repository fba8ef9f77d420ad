// kernels_small.cu - the two grouped GEMMs of a small batch (up to 64 tokens), which
// need neither the align kernel before them, nor the gather, nor the finalize after.
//
// At decode sizes every launch of the chain costs latency, not bandwidth
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels": fused kernels "combine routing, data movement
// and expert calculations into fewer GPU operations"). Here the forward of a small
// batch is route -> gate_up -> down (FP8: route -> quant_x -> gate_up -> quant_h ->
// down):
// - each GEMM CTA builds the batch's schedule (grouping, padded rows, tile counts and
//   split factors) in its own shared memory from the routing, as the align kernel
//   would (decode_sched.cuh); the routing stays one parallel kernel of its own;
// - gate_up reads activation rows straight from the token rows of x (or of its FP8
//   codes) with one-row TMA boxes: no gathered copy;
// - down builds its schedule before it waits for gate_up (the routing is two or more
//   launches back), so its weight loads go out as soon as its CTAs are resident; its
//   epilogue counts the K blocks added to each token and the CTA that adds a token's
//   last one converts the token's fp32 row to bf16 and re-zeroes it: no finalize
//   launch. Its last CTA records the FP8 scales of the forward and resets the amax words.
#include "decode_sched.cuh"
#include "fp8_format.cuh"
#include "gemm_pipeline.cuh"

namespace moe {

namespace {

using namespace pipe;

// gate_up: every activation row is a token row, ready once the kernel waited for its
// predecessor (done before the schedule is built).
struct SmallGateHooks {
  const Sched* s;
  int k;
  static constexpr bool kSignalTiles = false;
  static constexpr bool kTokenCompletion = false;
  __device__ __forceinline__ bool direct() const { return true; }
  __device__ __forceinline__ int direct_token(const Unit& un, int j) const {
    return s->pairs[s->off[un.t.expert] + j] / k;
  }
  __device__ __forceinline__ int dep(const Unit&) const { return 0; }
  __device__ __forceinline__ bool ready(int) const { return true; }
  __device__ __forceinline__ bool wait(int) const { return true; }
  __device__ __forceinline__ void column(const Unit&, int, float, int&, float&) const {}
  __device__ __forceinline__ void tile_done(const Unit&, int, float) {}
  __device__ __forceinline__ void down_done(const Unit&, const int*, int) {}
};

// down: the activation rows (h or its codes) are written by the previous kernel: one
// PDL wait; token rows are finished by whoever adds their last K block.
struct SmallDownHooks {
  Sched* s;
  float* acc;
  __nv_bfloat16* out;
  int* token_cnt;
  int k, H, need;
  bool waited = false;
  static constexpr bool kSignalTiles = false;
  static constexpr bool kTokenCompletion = true;
  __device__ __forceinline__ bool direct() const { return false; }
  __device__ __forceinline__ int direct_token(const Unit&, int) const { return 0; }
  __device__ __forceinline__ int dep(const Unit&) const { return 0; }
  __device__ __forceinline__ bool ready(int) const { return waited; }
  __device__ __forceinline__ bool wait(int) {
    if (!waited) {
      pdl_wait();
      pdl_trigger();
      waited = true;
    }
    return true;
  }
  __device__ __forceinline__ void column(const Unit& un, int j, float scale, int& tok, float& w) const {
    const int p = s->pairs[s->off[un.t.expert] + j];
    tok = p / k;
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
      for (int i = 0; i < nd; ++i) {
        const int t = s->done[i];
        float4* acc4 = reinterpret_cast<float4*>(acc + static_cast<size_t>(t) * H);
        uint2* out4 = reinterpret_cast<uint2*>(out + static_cast<size_t>(t) * H);
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

template <bool kGateUp, bool kFP8>
__global__ void __launch_bounds__(kThreads, 1)
    small_gemm_kernel(const __grid_constant__ SmallArgs a, const __grid_constant__ CUtensorMap tm_w,
                      const __grid_constant__ CUtensorMap tm_b) {
  using C = Cfg<kFP8>;
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve<C>(smem_raw, sizeof(Sched));
  Sched* s = reinterpret_cast<Sched*>(sh.extra);
  volatile int* abort_flag = sh.flags;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int G = gridDim.x;
  const int E = a.E, P = a.P, k = a.k;
  if (tid == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_b);
  }
  const uint32_t tmem = prologue<C>(sh, warp);
  // gate_up needs the routing (and x codes) of its predecessors; down finds the
  // routing complete already (two or more launches back) and waits later
  if constexpr (kGateUp) {
    pdl_wait();
    pdl_trigger();
  }
  sched_clear(s, E, tid, kThreads);
  for (int p = tid; p < P; p += kThreads) {
    s->ids[p] = __ldcg(a.topk_ids + p);
    if constexpr (!kGateUp) s->w[p] = __ldcg(a.topk_w + p);
  }
  __syncthreads();
  const int fb1 = a.I / kTileRows;
  const int fb2 = (a.H / kTileRows + 1) / 2;
  const int kb1 = a.H / C::kKPerBlock;
  const int kb2 = a.I / C::kKPerBlock;
  sched_build(s, P, E, k, fb1, fb2, kb1, kb2, G, a.ws1_rows_cap, a.uniform, tid, kThreads);
  __syncthreads();
  // down: everyone but the producer waits for the previous kernel here (the producer
  // issues its first weight loads first)
  if (!kGateUp && warp != 0) {
    pdl_wait();
    pdl_trigger();
  }
  const Ring rg = make_ring<C>(s->n_max, a.g.max_stages, sh.ring_bytes);
  const UnitSchedule<SmemTileFn<Sched>> src(SmemTileFn<Sched>{s, kGateUp ? fb1 : fb2}, kGateUp ? s->T1 : s->T2,
                                     kGateUp ? s->S1 : s->S2, kGateUp ? kb1 : kb2);
  SmallGateHooks hg{s, k};
  SmallDownHooks hd{s, a.g.acc, a.out, a.token_cnt, k, a.H, k * fb2 * kb2, warp != 0};

  if (warp == 0) {
    ProducerState ps;
    if constexpr (kGateUp) run_producer<C>(a.g, &tm_w, &tm_b, sh, rg, src, hg, ps, abort_flag, lane);
    else run_producer<C>(a.g, &tm_w, &tm_b, sh, rg, src, hd, ps, abort_flag, lane);
    producer_quiesce<C>(sh, rg, ps, lane);
  } else if (warp == 1) {
    if (lane == 0) {
      MmaState ms;
      run_mma<C, kFP8>(a.g, sh, rg, src, ms, tmem, abort_flag);
      mma_drain<C>(sh, ms);
    }
  } else {
    EpiState es;
    if constexpr (kGateUp) {
      run_epilogue<C, true, kFP8>(a.g, sh, rg, src, hg, es, tmem, abort_flag, warp, lane);
      if constexpr (kFP8) publish_amax(a.g.amax_h, es.lmax, lane);
    } else {
      run_epilogue<C, false, kFP8>(a.g, sh, rg, src, hd, es, tmem, abort_flag, warp, lane);
    }
  }
  teardown<C>(tmem, warp);

  if constexpr (kGateUp) {
    // the padded permutation for the FP8 h quantiser (the next kernel) and for inspection
    if (blockIdx.x == 0) sched_publish(s, P, E, a.counts, a.padded_offsets, a.padded_pairs, a.header, tid, kThreads);
  } else {
    // the last CTA: FP8 scales of the forward, amax words reset for the next one
    __syncthreads();
    if (tid == 0) {
      __threadfence();
      s->flag = atomicAdd(a.done, 1) == G - 1 ? 1 : 0;
    }
    __syncthreads();
    if (s->flag && tid == 0) {
      __threadfence();
      if constexpr (kFP8) {
        a.last_scales[0] = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
        a.last_scales[1] = fp8_scale_from_amax(__ldcg(a.amax + 1), a.f8);
        a.amax[0] = 0u;
        a.amax[1] = 0u;
      }
      *a.done = 0;
    }
  }
}

template <bool kGateUp, bool kFP8>
cudaError_t launch_one(const SmallArgs& a, const CUtensorMap& w, const CUtensorMap& b, int grid, cudaStream_t s) {
  return launch_kernel(small_gemm_kernel<kGateUp, kFP8>, dim3(grid), dim3(kThreads),
                       static_cast<size_t>(Cfg<kFP8>::kSmemBytes), s, a, w, b);
}

template <bool kGateUp, bool kFP8>
cudaError_t configure_one() {
  return cudaFuncSetAttribute(small_gemm_kernel<kGateUp, kFP8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<kFP8>::kSmemBytes);
}

}  // namespace

bool small_supported(int M, int E, int k) { return sched_supported(M, E, k) && E <= kSchedMaxExperts; }

cudaError_t small_configure() {
  cudaError_t e;
  if ((e = configure_one<true, false>()) != cudaSuccess) return e;
  if ((e = configure_one<true, true>()) != cudaSuccess) return e;
  if ((e = configure_one<false, false>()) != cudaSuccess) return e;
  return configure_one<false, true>();
}

cudaError_t launch_small_gate_up(const SmallArgs& a, const CUtensorMap& w, const CUtensorMap& x, bool fp8, int grid,
                                 cudaStream_t s) {
  return fp8 ? launch_one<true, true>(a, w, x, grid, s) : launch_one<true, false>(a, w, x, grid, s);
}

cudaError_t launch_small_down(const SmallArgs& a, const CUtensorMap& w, const CUtensorMap& h, bool fp8, int grid,
                              cudaStream_t s) {
  return fp8 ? launch_one<false, true>(a, w, h, grid, s) : launch_one<false, false>(a, w, h, grid, s);
}

}  // namespace moe
