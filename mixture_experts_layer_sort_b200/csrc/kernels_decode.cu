// kernels_decode.cu - the whole MoE layer for a decode batch (M <= 64 tokens, bf16)
// in ONE persistent, cooperative launch: routing, the grouping of (token, slot) pairs
// by expert, the gather of x into expert order, the gate_up GEMM with SwiGLU, the
// down GEMM with the routing-weight scatter-add, and the conversion of the finished
// token rows to bf16.
//
// Fused MoE kernels "combine routing, data movement and expert calculations into
// fewer GPU operations", cutting launch overhead and intermediate traffic
// (toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
// inference needs specialized kernels"); at decode sizes the separate kernels' own
// latency, not bandwidth, dominates, and this kernel removes it.
//
// How one launch replaces the chain:
// - CTA t routes token t and publishes its top-k; once all M tokens are published,
//   every CTA builds the permutation and both tile schedules itself, in shared
//   memory. The order inside an expert (ascending token, i.e. ascending pair id)
//   comes from a per-expert 64-bit token mask.
// - CTA c gathers rows c, c+G, ... of x into expert order, then bumps a counter.
// - The gate_up units start streaming weights at once; a unit's activation loads
//   wait (bounded) until all CTAs have gathered. Each finished gate_up tile bumps its
//   expert's "h ready" counter.
// - A CTA moves on to its down units as soon as it has issued its gate_up work:
//   W_down streams in while other CTAs finish gate_up; a down unit's activation
//   loads wait until every gate_up tile of its expert is done.
// - The down epilogue adds into the fp32 accumulator and counts, per token, the
//   contributions still missing; the CTA that completes a token converts its row to
//   bf16 and re-zeroes it. The last CTA to finish resets the counters.
// All CTAs must be resident at once (they wait on each other): the launch is
// cooperative, one CTA per SM. Every wait is bounded and reports through the error
// word when it gives up.
#include "gemm_pipeline.cuh"
#include "route_common.cuh"

namespace moe {

namespace {

using namespace pipe;
using C = Cfg<false>;

constexpr int kMaxTokens = 64;     // per-expert token masks are 64 bits
constexpr int kMaxPairs = 512;
constexpr int kMaxExperts = 512;

// Global sync words (zero between launches):
//   [0] CTAs that finished their gather, [1] CTAs that finished everything,
//   [2] tokens routed, [3, 3+E) gate_up tiles finished per expert,
//   [3+E, 3+E+M) down contributions per token
struct DecodeArgs {
  const float* logits;
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  int M, E, k, H, I, P;
  int ws1_rows_cap, max_stages;
  int* sync;
  __nv_bfloat16* x_perm;
  // copies of the routing for inspection (written by CTA 0)
  int* topk_ids;
  float* topk_w;
  int* counts;
  int* padded_offsets;
  int* padded_pairs;
  int* header;
  GemmArgs g1, g2;
};

// Shared-memory schedule (the pipeline's "extra" region).
struct Sched {
  int ids[kMaxPairs];
  float w[kMaxPairs];
  int count[kMaxExperts];
  int off[kMaxExperts + 1];       // compact offsets of each expert's pairs
  int poff[kMaxExperts + 1];      // padded offsets (rows of x_perm / h)
  int tmp[kMaxExperts + 1];
  int act[kMaxExperts];           // active experts, ascending
  int aidx[kMaxExperts + 1];      // index of each expert among the active ones
  unsigned mask[kMaxExperts][2];  // tokens routed to each expert
  int pairs[kMaxPairs];           // pair ids grouped by expert, ascending inside an expert
  int done[256];                  // tokens completed by the current down unit
  int ndone;
  int nact, T1, S1, T2, S2, n_max, rows_used, last_cta;
};

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}

// Units of one GEMM computed from the shared schedule: tile t = (active expert t / fb,
// row block t % fb); every expert has a single token tile (n_e <= M <= 64).
struct SmemTiles {
  const Sched* s;
  int fb, T, S, kblocks;
  // units u = blockIdx.x + i * gridDim.x of the T*S, round-robin
  __device__ __forceinline__ int count() const {
    const int n = T * S, c = static_cast<int>(blockIdx.x);
    return c < n ? (n - 1 - c) / static_cast<int>(gridDim.x) + 1 : 0;
  }
  __device__ __forceinline__ Unit unit(int i, int n_cap) const {
    const int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    const int t = u / S;
    const int ai = t / fb;
    Tile tile;
    tile.expert = s->act[ai];
    tile.fblock = t - ai * fb;
    tile.row_start = s->poff[tile.expert];
    tile.n_valid = s->count[tile.expert];
    return make_unit(tile, t, u - t * S, S, kblocks, n_cap);
  }
};

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

// gate_up: activation rows come from x_perm, complete once every CTA gathered.
struct GateUpHooks {
  const DecodeArgs* d;
  int grid;
  int* expert_ready;
  volatile int* abort_flag;
  bool gathered = false;
  static constexpr bool kSignalTiles = true;
  static constexpr bool kTokenCompletion = false;
  __device__ __forceinline__ int dep(const Unit&) const { return 0; }
  __device__ __forceinline__ bool ready(int) {
    if (gathered) return true;
    int v = 0;
    if ((threadIdx.x & 31) == 0) v = ld_acquire(d->sync) >= grid ? 1 : 0;
    v = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (v) {
      (void)ld_acquire(d->sync);     // every lane observes it before its TMA reads
      fence_proxy_async_global();
      gathered = true;
    }
    return gathered;
  }
  __device__ __forceinline__ bool wait(int dd) {
    if (ready(dd)) return true;
    const int* p = d->sync;
    const int g = grid;
    if (!spin_until([p, g]() { return ld_acquire(p) >= g; }, abort_flag)) return false;
    return ready(dd);
  }
  __device__ __forceinline__ void column(const Unit&, int, float, int&, float&) const {}
  // every epilogue thread: its h stores of the tile are visible (also to TMA reads)
  // before the expert's counter moves
  __device__ __forceinline__ void tile_done(const Unit& un, int epi_tid) {
    fence_proxy_async_global();
    __threadfence();
    named_bar_sync(1, kEpiThreads);
    if (epi_tid == 0) atomicAdd(expert_ready + un.t.expert, 1);
  }
  __device__ __forceinline__ void down_done(const Unit&, const int*, int) {}
};

// down: activation rows of expert e come from h, complete once all its gate_up
// tiles are done; tokens are converted by whoever adds their last contribution.
struct DownHooks {
  const DecodeArgs* d;
  Sched* s;
  int* expert_ready;
  int* token_cnt;
  int fb1, need;      // gate_up tiles per expert; down contributions per token
  volatile int* abort_flag;
  int last_ready = -1;
  static constexpr bool kSignalTiles = false;
  static constexpr bool kTokenCompletion = true;
  __device__ __forceinline__ int dep(const Unit& un) const { return un.t.expert; }
  __device__ __forceinline__ bool ready(int e) {
    if (e == last_ready) return true;
    int v = 0;
    if ((threadIdx.x & 31) == 0) v = ld_acquire(expert_ready + e) >= fb1 ? 1 : 0;
    v = __shfl_sync(0xFFFFFFFFu, v, 0);
    if (v) {
      (void)ld_acquire(expert_ready + e);
      fence_proxy_async_global();
      last_ready = e;
    }
    return v != 0;
  }
  __device__ __forceinline__ bool wait(int e) {
    if (ready(e)) return true;
    const int* p = expert_ready + e;
    const int f = fb1;
    if (!spin_until([p, f]() { return ld_acquire(p) >= f; }, abort_flag)) return false;
    return ready(e);
  }
  __device__ __forceinline__ void column(const Unit& un, int j, float scale, int& tok, float& w) const {
    const int p = s->pairs[s->off[un.t.expert] + j];
    tok = p / d->k;
    w = s->w[p] * scale;
  }
  __device__ __forceinline__ void tile_done(const Unit&, int) {}
  __device__ __forceinline__ void down_done(const Unit& un, const int* s_tok, int epi_tid) {
    __threadfence();                        // this unit's adds happen before the counts move
    named_bar_sync(1, kEpiThreads);
    if (epi_tid == 0) s->ndone = 0;
    named_bar_sync(1, kEpiThreads);
    for (int j = epi_tid; j < un.t.n_valid; j += kEpiThreads) {
      const int t = s_tok[j];
      if (atomicAdd(token_cnt + t, 1) == need - 1) s->done[atomicAdd(&s->ndone, 1)] = t;
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

__global__ void __launch_bounds__(kThreads, 1)
    fused_decode_kernel(const __grid_constant__ DecodeArgs d, const __grid_constant__ CUtensorMap tm_w13,
                        const __grid_constant__ CUtensorMap tm_wd, const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_h) {
  extern __shared__ uint8_t smem_raw[];
  const Shared sh = carve<C>(smem_raw, sizeof(Sched));
  Sched* s = reinterpret_cast<Sched*>(sh.extra);
  volatile int* abort_flag = sh.flags;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tid = threadIdx.x;
  const int G = gridDim.x;
  const int E = d.E, M = d.M, k = d.k, P = d.P;
  int* route_cnt = d.sync + 2;
  int* expert_ready = d.sync + 3;
  int* token_cnt = d.sync + 3 + E;
  if (tid == 0) {
    tma_prefetch_desc(&tm_w13);
    tma_prefetch_desc(&tm_wd);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_h);
  }
  const uint32_t tmem = prologue<C>(sh, warp);

  // ---------------------------------------------------------------- routing
  // CTA c routes tokens c, c+G, ... and publishes them; then everyone reads all
  for (int t = blockIdx.x; t < M; t += G) {
    if (warp == 0)
      route_token_any(d.logits + static_cast<size_t>(t) * E, E, k, lane, d.topk_ids + t * k, d.topk_w + t * k);
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int mine = blockIdx.x < M ? (M - 1 - static_cast<int>(blockIdx.x)) / G + 1 : 0;
    if (mine > 0) atomicAdd(route_cnt, mine);
  }
  for (int e = tid; e < E; e += kThreads) {
    s->count[e] = 0;
    s->mask[e][0] = 0u;
    s->mask[e][1] = 0u;
  }
  if (tid == 0) {
    const long long t0 = clock64();
    int ok = 1;
    while (ld_acquire(route_cnt) < M) {
      if (clock64() - t0 > (1ll << 31)) {
        ok = 0;
        break;
      }
      __nanosleep(32);
    }
    if (!ok) report_error(d.g1.err, kErrWaitGrid);
    s->last_cta = ok;                       // reused below as "routing complete"
  }
  __syncthreads();
  const bool routed = s->last_cta != 0;
  for (int p = tid; p < P; p += kThreads) {
    s->ids[p] = routed ? __ldcg(d.topk_ids + p) : 0;
    s->w[p] = routed ? __ldcg(d.topk_w + p) : 0.f;
  }
  __syncthreads();
  for (int p = tid; p < P; p += kThreads) {
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
    for (int e = lane; e < E; e += 32) s->tmp[e] = s->count[e] > 0 ? 1 : 0;
    __syncwarp();
    warp_exclusive_scan(s->tmp, s->aidx, E, lane);
    __syncwarp();
    for (int e = lane; e < E; e += 32)
      if (s->count[e] > 0) s->act[s->aidx[e]] = e;
    if (lane == 0) s->nact = s->aidx[E];
  }
  __syncthreads();
  // stable grouping: rank of pair (t, j) inside expert e = tokens t' < t routed to e
  for (int p = tid; p < P; p += kThreads) {
    const int e = s->ids[p];
    const int t = p / k;
    const unsigned lo = t < 32 ? (s->mask[e][0] & ((1u << t) - 1u)) : s->mask[e][0];
    const unsigned hi = t < 32 ? 0u : (s->mask[e][1] & ((1u << (t - 32)) - 1u));
    s->pairs[s->off[e] + __popc(lo) + __popc(hi)] = p;
  }
  const int fb1 = d.I / kTileRows;
  const int fb2 = (d.H / kTileRows + 1) / 2;
  const int kb1 = d.H / C::kKPerBlock;
  const int kb2 = d.I / C::kKPerBlock;
  __syncthreads();
  if (warp == 0) {
    int m = 0;
    for (int e = lane; e < E; e += 32) m = max(m, s->count[e]);
    #pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    const int A = s->nact;
    const int rows_used = s->poff[E];
    const int n_mean = A > 0 ? (P + A - 1) / A : 0;
    const int t1 = A * fb1;
    const int s1 = choose_splits_warp(t1, kb1, G, rows_used <= d.ws1_rows_cap, 2 * 16384 + n_mean * 128,
                                      n_mean * 256 * 4 * 2, lane);
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
    const int s2 = choose_splits_warp(t2, kb2, G, true, 2 * 16384 + n_mean * 128, n_mean * 128 * 4, lane);
    if (lane == 0) {
      s->T2 = t2;
      s->S2 = s2;
    }
  }
  __syncthreads();

  // copies of the grouping for inspection
  if (blockIdx.x == 0) {
    for (int e = tid; e < E; e += kThreads) {
      d.counts[e] = s->count[e];
      d.padded_offsets[e] = s->poff[e];
      for (int r = s->poff[e]; r < s->poff[e + 1]; ++r) {
        const int j = r - s->poff[e];
        d.padded_pairs[r] = j < s->count[e] ? s->pairs[s->off[e] + j] : P;
      }
    }
    if (tid == 0) {
      d.padded_offsets[E] = s->poff[E];
      d.header[kHdrRowsUsed] = s->rows_used;
    }
  }

  // ---------------------------------------------------------------- gather
  // this CTA's rows of x in expert order (pad rows are never read by a stored column)
  for (int r = blockIdx.x + warp * G; r < s->rows_used; r += G * (kThreads / 32)) {
    int lo = 0, hi = s->nact - 1;                 // active expert whose padded rows hold r
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s->poff[s->act[mid]] <= r) lo = mid;
      else hi = mid - 1;
    }
    const int e = s->act[lo];
    const int j = r - s->poff[e];
    if (j >= s->count[e]) continue;
    const int tok = s->pairs[s->off[e] + j] / k;
    const uint4* src = reinterpret_cast<const uint4*>(d.x + static_cast<size_t>(tok) * d.H);
    uint4* dst = reinterpret_cast<uint4*>(d.x_perm + static_cast<size_t>(r) * d.H);
    for (int i = lane; i < d.H / 8; i += 32) dst[i] = __ldg(src + i);
  }
  fence_proxy_async_global();
  __threadfence();
  __syncthreads();
  if (tid == 0) atomicAdd(d.sync, 1);

  // ---------------------------------------------------------------- both GEMMs
  const Ring rg = make_ring<C>(s->n_max, d.max_stages, sh.ring_bytes);
  const SmemTiles src1{s, fb1, s->T1, s->S1, kb1};
  const SmemTiles src2{s, fb2, s->T2, s->S2, kb2};
  GateUpHooks h1{&d, G, expert_ready, abort_flag};
  DownHooks h2{&d, s, expert_ready, token_cnt, fb1, k * fb2 * s->S2, abort_flag};

  if (warp == 0) {
    ProducerState ps;
    run_producer<C>(d.g1, &tm_w13, &tm_x, sh, rg, src1, h1, ps, abort_flag, lane);
    if (!ps.failed) run_producer<C>(d.g2, &tm_wd, &tm_h, sh, rg, src2, h2, ps, abort_flag, lane);
    producer_quiesce<C>(sh, rg, ps, lane);
  } else if (warp == 1) {
    if (lane == 0) {
      MmaState ms;
      run_mma<C, false>(d.g1, sh, rg, src1, ms, tmem, abort_flag);
      if (!ms.failed) run_mma<C, false>(d.g2, sh, rg, src2, ms, tmem, abort_flag);
    }
  } else {
    EpiState es;
    run_epilogue<C, true, false>(d.g1, sh, rg, src1, h1, es, tmem, abort_flag, warp, lane);
    if (!es.failed) run_epilogue<C, false, false>(d.g2, sh, rg, src2, h2, es, tmem, abort_flag, warp, lane);
  }
  teardown<C>(tmem, warp);

  // ---------------------------------------------------------------- last CTA resets
  if (tid == 0) {
    __threadfence();
    s->last_cta = atomicAdd(d.sync + 1, 1) == G - 1 ? 1 : 0;
  }
  __syncthreads();
  if (s->last_cta) {
    __threadfence();
    for (int e = tid; e < E; e += kThreads) expert_ready[e] = 0;
    for (int t = tid; t < M; t += kThreads) token_cnt[t] = 0;
    if (tid == 0) {
      d.sync[0] = 0;
      d.sync[1] = 0;
      d.sync[2] = 0;
    }
  }
}

}  // namespace

bool decode_supported(int M, int E, int k) { return M >= 1 && M <= kMaxTokens && E <= kMaxExperts && M * k <= kMaxPairs; }

size_t decode_sync_words(int E, int M_cap) { return static_cast<size_t>(3 + E + M_cap); }

cudaError_t decode_configure() {
  return cudaFuncSetAttribute(fused_decode_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmemBytes);
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
  d.sync = l.sync;
  d.x_perm = l.x_perm;
  d.topk_ids = l.topk_ids;
  d.topk_w = l.topk_w;
  d.counts = l.counts;
  d.padded_offsets = l.padded_offsets;
  d.padded_pairs = l.padded_pairs;
  d.header = l.header;
  d.g1 = l.g1;
  d.g2 = l.g2;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3(l.grid);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = C::kSmemBytes;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, fused_decode_kernel, d, *l.tm_w13, *l.tm_wd, *l.tm_x, *l.tm_h);
}

}  // namespace moe
