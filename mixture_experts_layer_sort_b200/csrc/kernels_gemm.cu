// kernels_gemm.cu - the stand-alone grouped GEMMs of the MoE layer (gate_up with the
// SwiGLU epilogue, down with the routing-weight scatter-add epilogue), one launch
// each, on the tcgen05 pipeline of gemm_pipeline.cuh.
//
// Work units are the align kernel's tiles or K ranges of them (split-K), so that
// small batches still stream weights through every SM. A persistent grid of one CTA
// per SM takes its units from the balanced schedule of GlobalTiles: whole tiles
// round-robin, and the last one to two waves cut into equal K-block ranges, so that
// every CTA streams the same weight bytes. With programmatic dependent launch, the
// weight loads of the first stages go out before the kernel waits for its
// predecessor; only the activation loads wait.
//
// For wide token tiles (prefill) the same kernels run on CTA pairs: clusters of two
// CTAs, the pair being the worker of the schedule. A pair's tile covers twice the weight
// rows (gate_up: 2 x 128 features; down: 4 x 128 output rows); each CTA loads its own
// two weight tiles and half of the token tile, and the first CTA issues M = 256 MMAs
// (tcgen05 cta_group::2) that read both CTAs' shared memory and write each CTA's rows into
// its own TMEM. Per weight byte an SM then pulls half the activation bytes, which is what
// bounds these GEMMs once tiles are 128-256 tokens wide.
#include "gemm_pipeline.cuh"

namespace moe {

namespace {

using namespace pipe;

// The activation operand depends on the previous kernel of the stream: one PDL wait.
// Down with the combine folded in: token rows are finished by whoever adds their last
// K block (done / ndone: a shared-memory list of the rows a unit completed).
struct PdlHooks {
  bool waited;
  const GemmArgs* a;
  int* done;
  int* ndone;
  static constexpr bool kSignalTiles = false;
  static constexpr bool kTokenCompletion = true;
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
    const int p = __ldg(a->padded_pairs + un.t.row_start + j);
    tok = p / a->k;
    w = __ldg(a->topk_w + p) * scale;
  }
  __device__ __forceinline__ bool direct() const { return a->direct_pairs != nullptr; }
  __device__ __forceinline__ int direct_token(const Unit& un, int j) const {
    return __ldcg(a->direct_pairs + un.t.row_start + j) / a->k;
  }
  __device__ __forceinline__ void tile_done(const Unit&, int, float) {}
  __device__ __forceinline__ void down_done(const Unit& un, const int* s_tok, int epi_tid) {
    if (a->token_cnt == nullptr) return;
    __threadfence();                        // this unit's adds happen before the counts move
    named_bar_sync(1, kEpiThreads);
    if (epi_tid == 0) *ndone = 0;
    named_bar_sync(1, kEpiThreads);
    const int add = un.kb1 - un.kb0;
    const int need = a->token_need;
    for (int j = epi_tid; j < un.t.n_valid; j += kEpiThreads) {
      const int t = s_tok[j];
      if (atomicAdd(a->token_cnt + t, add) == need - add) done[atomicAdd(ndone, 1)] = t;
    }
    named_bar_sync(1, kEpiThreads);
    const int nd = *ndone;
    if (nd > 0) {
      __threadfence();
      const int H = a->H;
      for (int i = 0; i < nd; ++i) {
        const int t = done[i];
        float4* acc4 = reinterpret_cast<float4*>(a->acc + static_cast<size_t>(t) * H);
        uint2* out4 = reinterpret_cast<uint2*>(a->out + static_cast<size_t>(t) * H);
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
        if (epi_tid == 0) a->token_cnt[t] = 0;
      }
    }
    named_bar_sync(1, kEpiThreads);         // the list is reused by the next unit
  }
};

template <bool kGateUp, bool kFP8, bool kPair>
__global__ void __launch_bounds__(kThreads, 1)
    grouped_gemm_kernel(const __grid_constant__ GemmArgs a, const __grid_constant__ CUtensorMap tm_w,
                        const __grid_constant__ CUtensorMap tm_b) {
  using C = Cfg<kFP8, kGemmSmem, 512, kPair>;
  extern __shared__ uint8_t smem_raw[];
  // down: 1 KB + 4 bytes for the list of token rows a unit completes
  const Shared sh = carve<C>(smem_raw, kGateUp ? 0 : 2048);
  volatile int* abort_flag = sh.flags;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_w);
    tma_prefetch_desc(&tm_b);
  }
  const uint32_t tmem = prologue<C>(sh, warp);

  // When the previous kernel wrote the tile list, nobody reads it before waiting.
  if (a.wait_first) {
    pdl_wait();
    pdl_trigger();
  }
  const Ring rg = make_ring<C>(a.header[kHdrMaxRows], a.max_stages, sh.ring_bytes);
  const int t_off = a.hdr_tile_offset > 0 ? a.header[a.hdr_tile_offset] : 0;
  const GlobalTiles src(a.tiles + t_off, a.header[a.hdr_tiles], a.header[a.hdr_splits], a.kblocks, kPair);
  // Everyone but the producer warp waits for the previous kernel here. Otherwise the
  // tile list comes from the align kernel, at least two launches back, and is
  // complete already (see pdl_wait in sm100.cuh).
  if (warp != 0 && !a.wait_first) {
    pdl_wait();
    pdl_trigger();
  }
  PdlHooks hk{a.wait_first != 0, &a, reinterpret_cast<int*>(sh.extra), reinterpret_cast<int*>(sh.extra) + 256};

  if (warp == 0) {
    ProducerState ps;
    run_producer<C>(a, &tm_w, &tm_b, sh, rg, src, hk, ps, abort_flag, lane);
    producer_quiesce<C>(sh, rg, ps, lane);
    if constexpr (kPair) producer_tail<C>(sh, rg, ps, lane);
  } else if (warp == 1) {
    if (lane == 0) {
      // pair: the first CTA issues the MMAs of both
      if (!kPair || cluster_ctarank() == 0) {
        MmaState ms;
        run_mma<C, kFP8>(a, sh, rg, src, ms, tmem, abort_flag);
        mma_drain<C>(sh, ms);
      }
    }
  } else {
    EpiState es;
    run_epilogue<C, kGateUp, kFP8>(a, sh, rg, src, hk, es, tmem, abort_flag, warp, lane);
    if constexpr (kGateUp && kFP8) publish_amax(a.amax_h, es.lmax, lane);
  }
  if constexpr (!kGateUp) {
    if (a.token_cnt != nullptr) {
      // the last CTA: FP8 scales of the forward, amax words cleared for the next one
      __syncthreads();
      if (threadIdx.x == 64) {
        __threadfence();
        if (atomicAdd(a.cta_done, 1) == static_cast<int>(gridDim.x) - 1) {
          __threadfence();
          if constexpr (kFP8) {
            a.last_scales[0] = fp8_scale_from_amax(__ldcg(a.amax), a.f8);
            a.last_scales[1] = fp8_scale_from_amax(__ldcg(a.amax + 1), a.f8);
            a.amax[0] = 0u;
            a.amax[1] = 0u;
          }
          *a.cta_done = 0;
        }
      }
    }
  }
  teardown<C>(tmem, warp);
}

template <bool kGateUp, bool kFP8>
cudaError_t launch_one(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& b, int grid, cudaStream_t s,
                       bool pair) {
  if (!pair)
    return launch_kernel(grouped_gemm_kernel<kGateUp, kFP8, false>, dim3(grid), dim3(kThreads),
                         static_cast<size_t>(Cfg<kFP8>::kSmemBytes), s, a, w, b);
  // clusters of two CTAs, with programmatic dependent launch as for every kernel of the chain
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(grid & ~1);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg<kFP8>::kSmemBytes);
  cfg.stream = s;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  at[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 2 : 1;
  return cudaLaunchKernelEx(&cfg, grouped_gemm_kernel<kGateUp, kFP8, true>, a, w, b);
}

template <bool kGateUp, bool kFP8>
cudaError_t configure_one() {
  cudaError_t e = cudaFuncSetAttribute(grouped_gemm_kernel<kGateUp, kFP8, false>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg<kFP8>::kSmemBytes);
  if (e != cudaSuccess) return e;
  return cudaFuncSetAttribute(grouped_gemm_kernel<kGateUp, kFP8, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              Cfg<kFP8>::kSmemBytes);
}

}  // namespace

cudaError_t gemm_configure() {
  cudaError_t e;
  if ((e = configure_one<true, false>()) != cudaSuccess) return e;
  if ((e = configure_one<true, true>()) != cudaSuccess) return e;
  if ((e = configure_one<false, false>()) != cudaSuccess) return e;
  return configure_one<false, true>();
}

int gemm_pair_clusters() {
  // the bf16 and FP8 kernels take the same resources (one CTA per SM: all of its shared
  // memory and TMEM); a pair needs two such SMs of one GPC
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(2);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(Cfg<false>::kSmemBytes);
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = 2;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  int n = 0;
  if (cudaOccupancyMaxActiveClusters(&n, grouped_gemm_kernel<true, false, true>, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return 0;
  }
  return n;
}

cudaError_t launch_gemm1(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& x, bool fp8, int grid,
                         cudaStream_t s, bool pair) {
  return fp8 ? launch_one<true, true>(a, w, x, grid, s, pair) : launch_one<true, false>(a, w, x, grid, s, pair);
}

cudaError_t launch_gemm2(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& h, bool fp8, int grid,
                         cudaStream_t s, bool pair) {
  return fp8 ? launch_one<false, true>(a, w, h, grid, s, pair) : launch_one<false, false>(a, w, h, grid, s, pair);
}

}  // namespace moe
