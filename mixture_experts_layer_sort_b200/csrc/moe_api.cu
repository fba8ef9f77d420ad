// moe_api.cu - the C ABI (include/moe_b200.h) and the host dispatcher: argument
// checks, weight storage, workspace sizing, TMA descriptor encoding and the launch
// chain of one forward pass.
//
// The forward pass is a fixed chain of precompiled kernels; the token count M is
// a runtime argument of each, and the tile list, split factors and stage-ring depth
// are computed on the device from the routing. Nothing is compiled, specialised or
// re-encoded per M (the
// pages' third change removes exactly such per-token-count recompiles:
// toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "3.
// Removing repeat compilation can reduce first-token delay"). Tensor maps of the
// weights and of the workspace are encoded once per weight load and once per
// workspace allocation; the one exception is the map over the caller's x that the
// direct-x path of the smallest bf16 batches encodes on the host per call (a host
// computation of 128 bytes, no compilation and no device work).
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>
#include <new>
#include <vector>

#include "../../include/moe_b200.h"
#include "fp8_format.cuh"
#include "moe_internal.h"
#include "sm100.cuh"

using moe::Tile;

struct moe_layer {
  int E = 0, k = 0, H = 0, I = 0, dtype = 0, device = 0, num_sms = 0;
  int pair_clusters = 0;        // CTA pairs of the grouped GEMMs resident at once
  bool loaded = false;
  // weights (library owned)
  void* w13 = nullptr;          // [E, 2I, H] gate rows then up rows of each expert (bf16 or e4m3)
  void* wd = nullptr;           // [E, H, I]
  float* wscales = nullptr;     // [E, 3] FP8 scales (device)
  int* eflags = nullptr;        // [E] precision per expert (1 = FP8), layers with a precision per expert
  CUtensorMap tm_w13{}, tm_wd{};
  // workspace, sized for M_cap tokens
  int M_cap = 0;
  long long P_cap = 0, rows_cap = 0, nblocks_cap = 0, t1_cap = 0, t2_cap = 0, ws1_rows_cap = 0;
  std::vector<void*> ws_allocs;
  int* topk_ids = nullptr;
  float* topk_w = nullptr;
  int* counts = nullptr;
  int* poff = nullptr;
  int* pairs = nullptr;
  Tile* tiles1 = nullptr;
  Tile* tiles2 = nullptr;
  int* header = nullptr;
  void* x_perm = nullptr;
  __nv_bfloat16* h = nullptr;
  uint8_t* h_q = nullptr;
  float* ws1 = nullptr;
  int* counters = nullptr;
  float* acc = nullptr;
  unsigned* amax = nullptr;     // [2] max|x|, max|h| (float bits)
  float* last_scales = nullptr; // [2]
  int* err = nullptr;
  int* sync = nullptr;          // single-launch decode: counters between its CTAs
  int* small_sync = nullptr;    // small batches: [M_cap] token K-block counts, then a CTA count
  int4* gv_records = nullptr;   // thin batches: the plan's active experts [min(E, P_cap)]
  int* chunk_buf = nullptr;     // multi-block align: [2][chunks_cap][E] chunk counts and bases
  uint8_t* xq = nullptr;        // FP8 large batches: x quantised per token [M_cap, H]
  long long chunks_cap = 0;
  CUtensorMap tm_x{}, tm_h{};
  CUtensorMap tm_xq{};          // FP8 single-launch decode: token rows of xq, one-row boxes
  uint8_t* x_perm8 = nullptr;   // precision per expert: FP8 codes of the FP8 experts' rows [rows_cap, H]
  CUtensorMap tm_x8{}, tm_hq{}; // precision per expert: maps of x_perm8 and of h_q
  // staging for moe_forward_host
  void* hx = nullptr;
  float* hl = nullptr;
  void* hout = nullptr;
  int host_cap = 0;
  // moe_forward_host replays a captured graph of copies + forward for pinned host
  // buffers, one per (M, host pointers); `graph_gen` counts the changes (weights,
  // workspace, staging, path switches) that make a captured graph stale
  struct HostGraph {
    int M;
    const void *x, *l;
    void* out;
    unsigned gen;
    cudaGraphExec_t exec;
  };
  std::vector<HostGraph> host_graphs;
  unsigned graph_gen = 0;
  cudaStream_t capture_stream = nullptr;
  // bookkeeping
  int last_M = 0, last_launches = 0;
  bool fused_decode = false;    // single-launch decode path for small batches
  int gemv_max_m = 0;           // batches of up to this many tokens take the thin-batch path
  bool last_small = false;      // the last forward took the small-batch path (no gathered x)
  bool last_pair = false;       // the last forward's grouped GEMMs ran on CTA pairs
  // per-kernel event timing
  bool profiling = false;
  struct Timed {
    int slot;
    cudaEvent_t a, b;
  };
  std::vector<Timed> pending;
  std::vector<cudaEvent_t> event_pool;
  double prof_ms[MOE_PROFILE_SLOTS] = {0};
  int prof_n[MOE_PROFILE_SLOTS] = {0};
};

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

std::mutex g_mu;
EncodeTiledFn g_encode = nullptr;
unsigned long long g_configured = 0;   // bit per device index whose kernels are configured

#define MOE_CUDA(call)                                                                           \
  do {                                                                                           \
    cudaError_t e_ = (call);                                                                     \
    if (e_ != cudaSuccess) {                                                                     \
      std::fprintf(stderr, "moe_b200: %s failed: %s (%s:%d)\n", #call, cudaGetErrorString(e_),   \
                   __FILE__, __LINE__);                                                          \
      return e_ == cudaErrorMemoryAllocation ? MOE_ERR_OOM : MOE_ERR_CUDA;                       \
    }                                                                                            \
  } while (0)

#define MOE_TRY(call)              \
  do {                             \
    int s_ = (call);               \
    if (s_ != MOE_OK) return s_;   \
  } while (0)

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int get_encoder() {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_encode) return MOE_OK;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  cudaError_t e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
  if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || fn == nullptr) return MOE_ERR_CUDA;
  g_encode = reinterpret_cast<EncodeTiledFn>(fn);
  return MOE_OK;
}

// 2-D row-major tensor [rows, inner] of 1- or 2-byte elements, box [box_rows, 128 bytes], 128B swizzle.
int encode_map(CUtensorMap* m, const void* base, bool fp8, long long inner, long long rows, int box_rows) {
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner * (fp8 ? 1 : 2))};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(fp8 ? 128 : 64), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  CUresult r = g_encode(m, fp8 ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                        const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::fprintf(stderr, "moe_b200: cuTensorMapEncodeTiled failed (%d)\n", static_cast<int>(r));
    return MOE_ERR_CUDA;
  }
  return MOE_OK;
}

int configure_device(int dev) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (dev < 64 && (g_configured >> dev) & 1ull) return MOE_OK;
  MOE_CUDA(moe::gemm_configure());
  MOE_CUDA(moe::align_configure());
  MOE_CUDA(moe::route_configure());
  MOE_CUDA(moe::decode_configure());
  MOE_CUDA(moe::small_configure());
  MOE_CUDA(moe::gemv_configure());
  if (dev < 64) g_configured |= 1ull << dev;
  return MOE_OK;
}

struct DeviceGuard {
  int prev = -1;
  bool ok = false;
  explicit DeviceGuard(int dev) {
    if (cudaGetDevice(&prev) != cudaSuccess) return;
    ok = (prev == dev) || cudaSetDevice(dev) == cudaSuccess;
  }
  ~DeviceGuard() {
    if (ok && prev >= 0) cudaSetDevice(prev);
  }
};

void free_workspace(moe_layer* L) {
  for (void* p : L->ws_allocs) cudaFree(p);
  L->ws_allocs.clear();
  L->M_cap = 0;
}

template <class T>
int ws_alloc(moe_layer* L, T** p, size_t bytes, bool zero) {
  void* q = nullptr;
  bytes = std::max<size_t>(bytes, 256);
  MOE_CUDA(cudaMalloc(&q, bytes));
  L->ws_allocs.push_back(q);
  if (zero) MOE_CUDA(cudaMemset(q, 0, bytes));
  *p = static_cast<T*>(q);
  return MOE_OK;
}

bool is_fp8(const moe_layer* L) { return L->dtype == MOE_DTYPE_FP8_E4M3 || L->dtype == MOE_DTYPE_FP8_E5M2; }
// a precision per expert (bf16 or e4m3): weights in bf16-sized slots, both kernel kinds
bool is_mixed(const moe_layer* L) { return L->dtype == MOE_DTYPE_MIXED_E4M3; }
// FP8 code format of an FP8 layer (moe::Fp8Format values)
int fp8_format(const moe_layer* L) { return L->dtype == MOE_DTYPE_FP8_E5M2 ? 1 : 0; }

int ensure_workspace(moe_layer* L, int M) {
  if (M <= L->M_cap) return MOE_OK;
  if (moe::fail_workspace_alloc()) return MOE_ERR_OOM;   // injected failure (tests): nothing allocated
  int cap = 64;
  while (cap < M) cap *= 2;
  MOE_CUDA(cudaDeviceSynchronize());   // the old workspace may still be in use
  free_workspace(L);
  ++L->graph_gen;
  const long long P = static_cast<long long>(cap) * L->k;
  const long long Emin = std::min<long long>(L->E, P);
  L->P_cap = P;
  L->rows_cap = P + Emin * (moe::kPadRows - 1);
  L->nblocks_cap = (P + moe::kTokenBlock - 1) / moe::kTokenBlock + Emin;
  L->t1_cap = L->nblocks_cap * (L->I / moe::kTileRows);
  L->t2_cap = L->nblocks_cap * (L->H / moe::kTileRows);
  const long long ws1_limit = (128ll << 20) / (8ll * L->I);
  L->ws1_rows_cap = std::min(L->rows_cap, ws1_limit);
  const size_t el = is_fp8(L) ? 1 : 2;
  MOE_TRY(ws_alloc(L, &L->topk_ids, P * 4, false));
  MOE_TRY(ws_alloc(L, &L->topk_w, P * 4, false));
  MOE_TRY(ws_alloc(L, &L->counts, (L->E + 1) * 4, true));
  MOE_TRY(ws_alloc(L, &L->poff, (L->E + 1) * 4, true));
  MOE_TRY(ws_alloc(L, &L->pairs, L->rows_cap * 4, true));
  MOE_TRY(ws_alloc(L, &L->tiles1, L->t1_cap * sizeof(Tile), false));
  MOE_TRY(ws_alloc(L, &L->tiles2, L->t2_cap * sizeof(Tile), false));
  MOE_TRY(ws_alloc(L, &L->header, moe::kHdrSlots * 4, true));
  MOE_TRY(ws_alloc(L, &L->x_perm, L->rows_cap * L->H * el, true));
  MOE_TRY(ws_alloc(L, &L->h, L->rows_cap * L->I * 2, true));
  if (is_fp8(L) || is_mixed(L)) MOE_TRY(ws_alloc(L, &L->h_q, L->rows_cap * L->I, true));
  if (is_mixed(L)) MOE_TRY(ws_alloc(L, &L->x_perm8, L->rows_cap * L->H, true));
  MOE_TRY(ws_alloc(L, &L->ws1, L->ws1_rows_cap * 2 * L->I * 4, true));
  MOE_TRY(ws_alloc(L, &L->counters, L->t1_cap * 4, true));
  MOE_TRY(ws_alloc(L, &L->acc, static_cast<size_t>(cap) * L->H * 4, true));
  MOE_TRY(ws_alloc(L, &L->amax, 2 * 4, true));
  MOE_TRY(ws_alloc(L, &L->last_scales, 2 * 4, false));
  MOE_TRY(ws_alloc(L, &L->err, 4, true));
  MOE_TRY(ws_alloc(L, &L->sync, moe::decode_sync_words(L->E, cap) * 4, true));
  MOE_TRY(ws_alloc(L, &L->small_sync, (static_cast<size_t>(cap) + 8) * 4, true));
  MOE_TRY(ws_alloc(L, &L->gv_records, moe::gemv_records_cap(L->E, P) * 16, false));
  if (is_fp8(L)) MOE_TRY(ws_alloc(L, &L->xq, static_cast<size_t>(cap) * L->H, false));
  L->chunks_cap = (P + moe::kAlignChunk - 1) / moe::kAlignChunk;
  MOE_TRY(ws_alloc(L, &L->chunk_buf, 2 * L->chunks_cap * L->E * 4, false));
  const float ones[2] = {1.f, 1.f};
  MOE_CUDA(cudaMemcpy(L->last_scales, ones, sizeof(ones), cudaMemcpyHostToDevice));
  MOE_TRY(encode_map(&L->tm_x, L->x_perm, is_fp8(L), L->H, L->rows_cap, 16));
  MOE_TRY(encode_map(&L->tm_h, is_fp8(L) ? static_cast<void*>(L->h_q) : static_cast<void*>(L->h), is_fp8(L),
                     L->I, L->rows_cap, 16));
  if (is_fp8(L)) MOE_TRY(encode_map(&L->tm_xq, L->xq, true, L->H, cap, 1));
  if (is_mixed(L)) {
    MOE_TRY(encode_map(&L->tm_x8, L->x_perm8, true, L->H, L->rows_cap, 16));
    MOE_TRY(encode_map(&L->tm_hq, L->h_q, true, L->I, L->rows_cap, 16));
  }
  L->M_cap = cap;
  return MOE_OK;
}

int encode_weight_maps(moe_layer* L) {
  ++L->graph_gen;
  // tiled storage: rows of 128 bytes, one 128-row box = one contiguous 16 KB tile
  const long long el = is_fp8(L) ? 1 : 2;
  const long long inner = 128 / el;
  MOE_TRY(encode_map(&L->tm_w13, L->w13, is_fp8(L), inner, 2ll * L->E * L->I * L->H * el / 128, moe::kTileRows));
  MOE_TRY(encode_map(&L->tm_wd, L->wd, is_fp8(L), inner, 1ll * L->E * L->H * L->I * el / 128, moe::kTileRows));
  return MOE_OK;
}

// Tile geometry of the three stored tensors: W_gate and W_up share w13 (up rows after
// gate rows). The row-major side has elements of src_el bytes (2 for a bf16 source, 1
// for FP8 codes) and is the full tensor of I_full intermediate features, of which the
// handle holds shard `shard` of I_full / I: rows [shard*I, (shard+1)*I) of W_gate and
// W_up, columns [shard*I, (shard+1)*I) of W_down. A whole tensor is shard 0 of I.
moe::TileGeom geom(const moe_layer* L, int which, long long src_el, long long I_full, int shard) {
  const long long el = is_fp8(L) ? 1 : 2;
  moe::TileGeom g{};
  g.E = L->E;
  if (which < 2) {
    g.rows = L->I;
    g.row_bytes = L->H * el;
    g.rb_total = 2 * L->I / moe::kTileRows;
    g.rb_offset = which == 0 ? 0 : L->I / moe::kTileRows;
    g.src_row_stride = L->H * src_el;
    g.src_expert_stride = I_full * L->H * src_el;
    g.src_offset = static_cast<long long>(shard) * L->I * L->H * src_el;
  } else {
    g.rows = L->H;
    g.row_bytes = L->I * el;
    g.rb_total = L->H / moe::kTileRows;
    g.rb_offset = 0;
    g.src_row_stride = I_full * src_el;
    g.src_expert_stride = L->H * I_full * src_el;
    g.src_offset = static_cast<long long>(shard) * L->I * src_el;
  }
  return g;
}

moe::TileGeom geom(const moe_layer* L, int which) {
  return geom(L, which, is_fp8(L) ? 1 : 2, L->I, 0);
}

// Weights of shard `shard` (I_full = I * shards) from bf16 sources: tiled copies, or
// per-(expert, tensor) scales and codes of the shard's own slice (FP8).
int load_bf16_sources(moe_layer* L, const void* const src[3], long long I_full, int shard, cudaStream_t st) {
  void* dst[3] = {L->w13, L->w13, L->wd};
  for (int j = 0; j < 3; ++j) {
    const moe::TileGeom g = geom(L, j, 2, I_full, shard);
    if (!is_fp8(L)) {
      MOE_CUDA(moe::launch_tile_weights(src[j], g, dst[j], st));
    } else {
      const auto* w = static_cast<const __nv_bfloat16*>(src[j]);
      MOE_CUDA(moe::launch_weight_amax(fp8_format(L), w, g, L->wscales + j, 3, st));
      MOE_CUDA(moe::launch_weight_quant_tiled(fp8_format(L), w, g, L->wscales + j, 3, static_cast<uint8_t*>(dst[j]),
                                              st));
    }
  }
  return MOE_OK;
}

cudaEvent_t pool_event(moe_layer* L) {
  if (!L->event_pool.empty()) {
    cudaEvent_t e = L->event_pool.back();
    L->event_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

// Records an event pair around one kernel launch when profiling is on.
// NVTX names of the kernel slots (the profiling slots of moe_profile_read)
const char* const kSlotNames[MOE_PROFILE_SLOTS] = {"moe route", "moe align", "moe gather", "moe gate_up GEMM",
                                                   "moe quant_h", "moe down GEMM", "moe finalize"};

struct KernelTimer {
  moe_layer* L;
  int slot;
  cudaStream_t st;
  cudaEvent_t a = nullptr;
  moe::NvtxRange range;
  KernelTimer(moe_layer* l, int s, cudaStream_t stream) : L(l), slot(s), st(stream), range(kSlotNames[s]) {
    if (L->profiling && (a = pool_event(L)) != nullptr) cudaEventRecord(a, st);
  }
  ~KernelTimer() {
    if (!a) return;
    cudaEvent_t b = pool_event(L);
    if (!b) {
      L->event_pool.push_back(a);
      return;
    }
    cudaEventRecord(b, st);
    L->pending.push_back({slot, a, b});
  }
};

int drain_profile(moe_layer* L) {
  MOE_CUDA(cudaDeviceSynchronize());
  for (auto& t : L->pending) {
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t.a, t.b) == cudaSuccess) {
      L->prof_ms[t.slot] += ms;
      L->prof_n[t.slot] += 1;
    }
    L->event_pool.push_back(t.a);
    L->event_pool.push_back(t.b);
  }
  L->pending.clear();
  return MOE_OK;
}

// Whether the chain's grouped GEMMs run on CTA pairs (M = 256 MMAs, each CTA loading half
// of a token tile): for wide token tiles (at least 96 tokens per expert on average), where
// the bytes each SM pulls per weight byte bound the GEMMs. MOE_PAIR_GEMM=0 never, =1
// whenever the shapes allow (read at every forward).
bool pair_gemm(const moe_layer* L, long long P, bool direct) {
  if (direct || L->H % 512 != 0 || L->I % 256 != 0 || L->pair_clusters < 1) return false;
  const char* e = std::getenv("MOE_PAIR_GEMM");
  if (e && e[0] == '0') return false;
  if (e && e[0] == '1') return true;
  return P >= 96ll * L->E;
}

// Whether the chain's down GEMM finishes each token row itself (the epilogue that adds
// its last K block writes `out`) instead of a finalize launch: MOE_FOLD_FINALIZE=1 (read
// at every forward). Off by default: measured on one B200, the per-unit fence and counts
// cost more than the launch they save (decode bf16 M=64 214.7 -> 224.9 us, e4m3 M=32
// 122.6 -> 135.0, prefill bf16 3998 -> 6263: with one TMEM buffer the MMAs wait for the
// longer epilogue).
bool fold_finalize() {
  const char* e = std::getenv("MOE_FOLD_FINALIZE");
  return e && e[0] == '1';
}

bool direct_x_disabled() {
  static const bool off = [] {
    const char* e = std::getenv("MOE_DISABLE_DIRECT_X");
    return e && e[0] == '1';
  }();
  return off;
}

// Whether new handles take the single-launch decode path for the batches it supports
// (MOE_FUSED_DECODE=0 or 1 overrides the default).
bool fused_decode_default() {
  static const bool on = [] {
    const char* e = std::getenv("MOE_FUSED_DECODE");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

// K blocks per expert of the down weights that the thin-batch down kernel asks into L2
// before it waits for gate_up (MOE_GEMV_PREFETCH_KB; default 0).
int gemv_prefetch_kb() {
  static const int v = [] {
    const char* e = std::getenv("MOE_GEMV_PREFETCH_KB");
    return e ? std::atoi(e) : 0;
  }();
  return v;
}

int decode_stage_cap() {
  static const int cap = [] {
    const char* e = std::getenv("MOE_MAX_STAGES_DECODE");
    return e ? std::atoi(e) : 5;
  }();
  return cap;
}

// The whole layer of a decode batch in one cooperative launch.
int forward_fused_decode(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st) {
  const bool fp8 = is_fp8(L);
  const int kper = fp8 ? 128 : 64;
  // gate_up reads token rows with one-row boxes: of the caller's x (bf16), or of the
  // codes of x the kernel writes into the workspace (FP8; map encoded with it)
  CUtensorMap tm_xd{};
  if (!fp8) MOE_TRY(encode_map(&tm_xd, x, false, L->H, M, 1));
  moe::DecodeLaunch d{};
  d.logits = logits;
  d.x = static_cast<const __nv_bfloat16*>(x);
  d.out = static_cast<__nv_bfloat16*>(out);
  d.M = M;
  d.E = L->E;
  d.k = L->k;
  d.H = L->H;
  d.I = L->I;
  d.grid = L->num_sms;
  d.ws1_rows_cap = static_cast<int>(L->ws1_rows_cap);
  d.max_stages = decode_stage_cap();
  d.fp8 = fp8;
  d.f8 = fp8_format(L);
  d.sync = L->sync;
  d.xq = L->xq;
  d.hq = L->h_q;
  d.last_scales = L->last_scales;
  d.topk_ids = L->topk_ids;
  d.topk_w = L->topk_w;
  d.counts = L->counts;
  d.padded_offsets = L->poff;
  d.padded_pairs = L->pairs;
  d.header = L->header;
  moe::GemmArgs g{};
  g.h = L->h;
  g.I = L->I;
  g.ws1 = L->ws1;
  g.tile_counters = L->counters;
  g.acc = L->acc;
  g.H = L->H;
  g.k = L->k;
  g.P = M * L->k;
  g.err = L->err;
  g.wait_budget = moe::wait_budget_cycles();
  g.w_scales = L->wscales;
  g.f8 = fp8_format(L);
  d.g1 = g;
  d.g1.kblocks = L->H / kper;
  d.g1.w_rblocks = 2 * L->I / moe::kTileRows;
  d.g1.rb_step = 1;
  d.g1.second_rb = L->I / moe::kTileRows;
  d.g2 = g;
  d.g2.kblocks = L->I / kper;
  d.g2.w_rblocks = L->H / moe::kTileRows;
  d.g2.rb_step = 2;
  d.g2.second_rb = 1;
  d.tm_w13 = &L->tm_w13;
  d.tm_wd = &L->tm_wd;
  d.tm_x = fp8 ? &L->tm_xq : &tm_xd;
  d.tm_h = &L->tm_h;
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_decode(d, st));
  }
  L->last_M = M;
  L->last_launches = 1;
  return MOE_OK;
}

// Feature slabs of the down tile order: enough that one slab of the fp32 accumulator
// (M x H x 4 bytes / slabs) stays well inside the 126 MB L2 next to the streamed
// weights and the live activations.
constexpr long long kAccSlabBytes = 64ll << 20;

int acc_slabs(int M, int H, int fblocks2) {
  static const int forced = [] {
    const char* e = std::getenv("MOE_ACC_SLABS");   // fixed slab count (1 = expert-major order)
    return e ? std::atoi(e) : 0;
  }();
  const long long bytes = static_cast<long long>(M) * H * 4;
  const long long s = forced > 0 ? forced : (bytes + kAccSlabBytes - 1) / kAccSlabBytes;
  return static_cast<int>(std::max(1ll, std::min<long long>(s, fblocks2)));
}

// Up to this many (token, slot) pairs one align block places the pairs itself (one
// chunk of 1024 pairs after another); beyond, chunks go to blocks of their own.
constexpr long long kAlignSingleBlockMaxPairs = 8192;

int forward_mixed(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st);

// Whether batches that fit the small-batch path take it (MOE_SMALL_BATCH=1; measured
// slower than the full chain, so off by default).
bool small_batch_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("MOE_SMALL_BATCH");
    return e != nullptr && e[0] == '1';
  }();
  return on;
}

// A batch of up to 64 tokens: route -> gate_up -> down (FP8: route -> quant_x ->
// gate_up -> quant_h -> down). The GEMMs build the schedule from the routing
// themselves, gate_up reads token rows directly, down finishes token rows itself.
int forward_small(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st) {
  const bool fp8 = is_fp8(L);
  const long long P = static_cast<long long>(M) * L->k;
  int launches = 0;

  moe::RouteArgs ra{};
  ra.logits = logits;
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.M = M;
  ra.E = L->E;
  ra.k = L->k;
  ra.H = L->H;
  ra.topk_ids = L->topk_ids;
  ra.topk_w = L->topk_w;
  ra.amax_x = fp8 ? L->amax : nullptr;
  ra.amax_h_reset = fp8 ? L->amax + 1 : nullptr;
  {
    KernelTimer kt(L, 0, st);
    MOE_CUDA(moe::launch_route(ra, st));
  }
  ++launches;

  // gate_up's activation rows: the caller's x rows (bf16), or their codes (FP8)
  CUtensorMap tm_xd{};
  if (fp8) {
    moe::QuantXArgs qx{};
    qx.x = static_cast<const __nv_bfloat16*>(x);
    qx.xq = L->xq;
    qx.M = M;
    qx.H = L->H;
    qx.amax_x = L->amax;
    qx.f8 = fp8_format(L);
    KernelTimer kt(L, 2, st);
    MOE_CUDA(moe::launch_quant_x(qx, st));
    ++launches;
  } else {
    MOE_TRY(encode_map(&tm_xd, x, false, L->H, M, 1));
  }

  const int kper = fp8 ? 128 : 64;
  moe::SmallArgs sa{};
  sa.topk_ids = L->topk_ids;
  sa.topk_w = L->topk_w;
  sa.out = static_cast<__nv_bfloat16*>(out);
  sa.M = M;
  sa.E = L->E;
  sa.k = L->k;
  sa.H = L->H;
  sa.I = L->I;
  sa.P = static_cast<int>(P);
  sa.ws1_rows_cap = static_cast<int>(L->ws1_rows_cap);
  sa.uniform = moe::uniform_splits() ? 1 : 0;
  sa.f8 = fp8_format(L);
  sa.token_cnt = L->small_sync;
  sa.done = L->small_sync + L->M_cap;
  sa.amax = L->amax;
  sa.last_scales = L->last_scales;
  sa.counts = L->counts;
  sa.padded_offsets = L->poff;
  sa.padded_pairs = L->pairs;
  sa.header = L->header;
  moe::GemmArgs g{};
  g.h = L->h;
  g.I = L->I;
  g.ws1 = L->ws1;
  g.tile_counters = L->counters;
  g.amax_h = L->amax + 1;
  g.amax_x = L->amax;
  g.w_scales = L->wscales;
  g.acc = L->acc;
  g.H = L->H;
  g.k = L->k;
  g.P = static_cast<int>(P);
  g.f8 = fp8_format(L);
  g.err = L->err;
  g.wait_budget = moe::wait_budget_cycles();

  moe::SmallArgs s1 = sa;
  s1.g = g;
  s1.g.kblocks = L->H / kper;
  s1.g.w_rblocks = 2 * L->I / moe::kTileRows;
  s1.g.rb_step = 1;
  s1.g.second_rb = L->I / moe::kTileRows;
  s1.g.max_stages = moe::gemm_max_stages(true);
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_small_gate_up(s1, L->tm_w13, fp8 ? L->tm_xq : tm_xd, fp8, L->num_sms, st));
  }
  ++launches;

  if (fp8) {
    moe::QuantHArgs qa{};
    qa.h = L->h;
    qa.h_q = L->h_q;
    qa.padded_pairs = L->pairs;
    qa.header = L->header;
    qa.rows_bound = static_cast<int>(P + std::min<long long>(L->E, P) * (moe::kPadRows - 1));
    qa.P = static_cast<int>(P);
    qa.I = L->I;
    qa.amax_h = L->amax + 1;
    qa.f8 = fp8_format(L);
    KernelTimer kt(L, 4, st);
    MOE_CUDA(moe::launch_quant_h(qa, st));
    ++launches;
  }

  moe::SmallArgs s2 = sa;
  s2.g = g;
  s2.g.kblocks = L->I / kper;
  s2.g.w_rblocks = L->H / moe::kTileRows;
  s2.g.rb_step = 2;
  s2.g.second_rb = 1;
  s2.g.max_stages = moe::gemm_max_stages(false);
  {
    KernelTimer kt(L, 5, st);
    MOE_CUDA(moe::launch_small_down(s2, L->tm_wd, L->tm_h, fp8, L->num_sms, st));
  }
  ++launches;
  L->last_M = M;
  L->last_launches = launches;
  L->last_small = true;
  return MOE_OK;
}

// Largest batch that new handles send to the thin-batch path (kernels_gemv.cu):
// MOE_GEMV_MAX_M overrides the built-in default. Measured on one B200 against the
// tensor-core chain, same box (decode layer E=128, H=2048, I=768): bf16 M=1 33.1 vs
// 43.1 us, M=4 63.7 vs 76.0, M=16 162 vs 152; e4m3 M=1 31.0 vs 44.7, M=8 67.9 vs 79.8;
// the E=256, H=7168 layer at M=1 131.3 vs 140.2. So: up to 8 tokens.
int gemv_max_default(int dtype, int) {
  static const int env = [] {
    const char* e = std::getenv("MOE_GEMV_MAX_M");
    return e ? std::atoi(e) : -1;
  }();
  if (env >= 0) return std::min(env, moe::kGemvMaxM);
  return dtype == MOE_DTYPE_MIXED_E4M3 ? 0 : 8;
}

bool gemv_path(const moe_layer* L, int M) {
  return M >= 1 && M <= L->gemv_max_m && !is_mixed(L) && moe::gemv_supported(M, L->E, L->k, L->H, L->I, L->num_sms, is_fp8(L));
}

// Thin batches: route + plan, then gate_up and down as streams of warp-level
// tensor-core products, three launches in all, `out` written by down.
int forward_gemv(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st) {
  const bool fp8 = is_fp8(L);
  moe::GemvArgs a{};
  a.logits = logits;
  a.x = static_cast<const __nv_bfloat16*>(x);
  a.M = M;
  a.E = L->E;
  a.k = L->k;
  a.H = L->H;
  a.I = L->I;
  a.topk_ids = L->topk_ids;
  a.topk_w = L->topk_w;
  a.counts = L->counts;
  a.padded_offsets = L->poff;
  a.padded_pairs = L->pairs;
  a.header = L->header;
  a.active = L->gv_records;
  a.amax = L->amax;
  a.xq = fp8 ? L->xq : nullptr;
  a.last_scales = L->last_scales;
  a.f8 = fp8_format(L);
  a.w13 = static_cast<const uint8_t*>(L->w13);
  a.wd = static_cast<const uint8_t*>(L->wd);
  a.w_scales = L->wscales;
  const int el = fp8 ? 1 : 2;
  a.kb1 = L->H * el / moe::kRowBytes;
  a.kb2 = L->I * el / moe::kRowBytes;
  a.et1 = static_cast<long long>(2 * L->I / moe::kTileRows) * a.kb1;
  a.et2 = static_cast<long long>(L->H / moe::kTileRows) * a.kb2;
  a.h = L->h;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.prefetch_kb = gemv_prefetch_kb();
  const int fmt = !fp8 ? 0 : (L->dtype == MOE_DTYPE_FP8_E5M2 ? 2 : 1);
  moe::gemv_down_plan(a, L->num_sms);
  {
    KernelTimer kt(L, 0, st);
    MOE_CUDA(moe::launch_gemv_plan(a, st));
  }
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_gemv_gate_up(a, fmt, st));
  }
  {
    KernelTimer kt(L, 5, st);
    MOE_CUDA(moe::launch_gemv_down(a, fmt, st));
  }
  // FP8 x codes are token rows of xq: the debug copy of x_perm lays them out like the
  // small-batch path's
  L->last_small = fp8;
  L->last_M = M;
  L->last_launches = 3;
  return MOE_OK;
}

int forward_impl(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st) {
  MOE_TRY(ensure_workspace(L, M));
  L->last_small = false;
  L->last_pair = false;
  if (is_mixed(L)) return forward_mixed(L, x, logits, M, out, st);
  // the opt-in decode paths first, then the thin-batch path, else the chain
  if (L->fused_decode && M <= L->num_sms && moe::decode_supported(M, L->E, L->k))
    return forward_fused_decode(L, x, logits, M, out, st);
  if (small_batch_enabled() && moe::small_supported(M, L->E, L->k))
    return forward_small(L, x, logits, M, out, st);
  if (gemv_path(L, M)) return forward_gemv(L, x, logits, M, out, st);
  const bool fp8 = is_fp8(L);
  const long long P = static_cast<long long>(M) * L->k;
  const int BN = moe::kTokenBlock;
  const int rows_bound = static_cast<int>(P + std::min<long long>(L->E, P) * (moe::kPadRows - 1));
  int launches = 0;

  moe::RouteArgs ra{};
  ra.logits = logits;
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.M = M;
  ra.E = L->E;
  ra.k = L->k;
  ra.H = L->H;
  ra.topk_ids = L->topk_ids;
  ra.topk_w = L->topk_w;
  ra.amax_x = fp8 ? L->amax : nullptr;
  ra.amax_h_reset = fp8 ? L->amax + 1 : nullptr;
  {
    KernelTimer kt(L, 0, st);
    MOE_CUDA(moe::launch_route(ra, st));
  }
  ++launches;

  // The smallest bf16 batches (P <= 16) skip the gather: gate_up reads each token's x row
  // itself with 1-row TMA boxes. Measured: faster at M=1, slower from M=4 on (16-row
  // boxes of gathered rows stream better than 128-byte row reads).
  const bool direct = !fp8 && P <= 16 && !direct_x_disabled();
  // CTA pairs: a tile covers two CTAs' weight row blocks (gate_up 2 x 128 features, down
  // 4 x 128), and the pairs are the workers the split-K rule counts
  const bool pair = pair_gemm(L, P, direct);

  moe::AlignArgs aa{};
  aa.topk_ids = L->topk_ids;
  aa.P = static_cast<int>(P);
  aa.E = L->E;
  aa.k = L->k;
  aa.BN = BN;
  aa.fblocks1 = L->I / (pair ? 2 * moe::kTileRows : moe::kTileRows);
  aa.fblocks2 = pair ? L->H / (4 * moe::kTileRows) : (L->H / moe::kTileRows + 1) / 2;
  const int kper = fp8 ? 128 : 64;
  aa.kblocks1 = L->H / kper;
  aa.kblocks2 = L->I / kper;
  aa.num_sms = pair ? L->pair_clusters : L->num_sms;
  const int gemm_grid = pair ? 2 * L->pair_clusters : L->num_sms;
  aa.ws1_rows_cap = static_cast<int>(L->ws1_rows_cap);
  aa.acc_slabs = acc_slabs(M, L->H, aa.fblocks2);
  aa.uniform_splits = moe::uniform_splits() ? 1 : 0;
  aa.counts = L->counts;
  aa.padded_offsets = L->poff;
  aa.padded_pairs = L->pairs;
  aa.tiles1 = L->tiles1;
  aa.tiles2 = L->tiles2;
  aa.header = L->header;
  // Large batches take the multi-block path: per-chunk counts, the plan (the align
  // block itself), then the placement of each chunk's pairs by its own block. FP8
  // large batches also quantise x once per token here, so that the gather copies bytes.
  const bool chunked = P > kAlignSingleBlockMaxPairs;
  if (chunked && fp8) {
    moe::QuantXArgs qx{};
    qx.x = static_cast<const __nv_bfloat16*>(x);
    qx.xq = L->xq;
    qx.M = M;
    qx.H = L->H;
    qx.amax_x = L->amax;
    qx.f8 = fp8_format(L);
    KernelTimer kt(L, 2, st);
    MOE_CUDA(moe::launch_quant_x(qx, st));
    ++launches;
  }
  if (chunked) {
    aa.chunks = static_cast<int>((P + moe::kAlignChunk - 1) / moe::kAlignChunk);
    aa.chunk_counts = L->chunk_buf;
    aa.chunk_base = L->chunk_buf + L->chunks_cap * L->E;
    KernelTimer kt(L, 1, st);
    MOE_CUDA(moe::launch_align_count(aa, st));
    ++launches;
  }
  {
    KernelTimer kt(L, 1, st);
    MOE_CUDA(moe::launch_align(aa, st));
  }
  ++launches;
  if (chunked) {
    KernelTimer kt(L, 1, st);
    MOE_CUDA(moe::launch_align_scatter(aa, st));
    ++launches;
  }

  CUtensorMap tm_xd{};
  if (direct) MOE_TRY(encode_map(&tm_xd, x, false, L->H, M, 1));

  moe::GatherArgs ga{};
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.padded_pairs = L->pairs;
  ga.header = L->header;
  ga.rows_bound = rows_bound;
  ga.P = static_cast<int>(P);
  ga.k = L->k;
  ga.H = L->H;
  ga.x_perm = L->x_perm;
  ga.amax_x = L->amax;
  ga.f8 = fp8_format(L);
  ga.xq = (chunked && fp8) ? L->xq : nullptr;
  if (!direct) {
    KernelTimer kt(L, 2, st);
    MOE_CUDA(moe::launch_gather(ga, fp8, st));
    ++launches;
  }

  moe::GemmArgs g{};
  g.header = L->header;
  g.h = L->h;
  g.I = L->I;
  g.ws1 = L->ws1;
  g.tile_counters = L->counters;
  g.amax_h = L->amax + 1;
  g.amax_x = L->amax;
  g.w_scales = L->wscales;
  g.acc = L->acc;
  g.H = L->H;
  g.padded_pairs = L->pairs;
  g.topk_w = L->topk_w;
  g.k = L->k;
  g.P = static_cast<int>(P);
  g.f8 = fp8_format(L);
  g.err = L->err;
  g.wait_budget = moe::wait_budget_cycles();

  moe::GemmArgs g1 = g;
  g1.tiles = L->tiles1;
  g1.hdr_tiles = moe::kHdrTiles1;
  g1.hdr_splits = moe::kHdrSplits1;
  g1.kblocks = aa.kblocks1;
  g1.w_rblocks = 2 * L->I / moe::kTileRows;
  g1.rb_step = pair ? 2 : 1;
  g1.pair_rb = pair ? 1 : 0;
  g1.second_rb = L->I / moe::kTileRows;
  g1.max_stages = moe::gemm_max_stages(true);
  g1.wait_first = direct ? 1 : 0;
  g1.direct_pairs = direct ? L->pairs : nullptr;
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_gemm1(g1, L->tm_w13, direct ? tm_xd : L->tm_x, fp8, gemm_grid, st, pair));
  }
  L->last_pair = pair;
  ++launches;

  if (fp8) {
    moe::QuantHArgs qa{};
    qa.h = L->h;
    qa.h_q = L->h_q;
    qa.padded_pairs = L->pairs;
    qa.header = L->header;
    qa.rows_bound = rows_bound;
    qa.P = static_cast<int>(P);
    qa.I = L->I;
    qa.amax_h = L->amax + 1;
    qa.f8 = fp8_format(L);
    {
      KernelTimer kt(L, 4, st);
      MOE_CUDA(moe::launch_quant_h(qa, st));
    }
    ++launches;
  }

  moe::GemmArgs g2 = g;
  g2.tiles = L->tiles2;
  g2.hdr_tiles = moe::kHdrTiles2;
  g2.hdr_splits = moe::kHdrSplits2;
  g2.kblocks = aa.kblocks2;
  g2.w_rblocks = L->H / moe::kTileRows;
  g2.rb_step = pair ? 4 : 2;
  g2.pair_rb = pair ? 2 : 0;
  g2.second_rb = 1;
  g2.max_stages = moe::gemm_max_stages(false);
  // the combine: token rows finished inside the down GEMM (counts of the K blocks each
  // token receives: k experts x tiles across H x K blocks, once per CTA of a pair), or a
  // finalize launch
  const bool fold = fold_finalize();
  if (fold) {
    g2.token_cnt = L->small_sync;
    g2.cta_done = L->small_sync + L->M_cap;
    g2.token_need = L->k * aa.fblocks2 * aa.kblocks2 * (pair ? 2 : 1);
    g2.out = static_cast<__nv_bfloat16*>(out);
    g2.amax = fp8 ? L->amax : nullptr;
    g2.last_scales = fp8 ? L->last_scales : nullptr;
  }
  {
    KernelTimer kt(L, 5, st);
    MOE_CUDA(moe::launch_gemm2(g2, L->tm_wd, L->tm_h, fp8, gemm_grid, st, pair));
  }
  ++launches;

  if (!fold) {
    moe::FinalizeArgs fa{};
    fa.acc = L->acc;
    fa.out = static_cast<__nv_bfloat16*>(out);
    fa.n = static_cast<long long>(M) * L->H;
    fa.amax = fp8 ? L->amax : nullptr;
    fa.last_scales = fp8 ? L->last_scales : nullptr;
    fa.f8 = fp8_format(L);
    {
      KernelTimer kt(L, 6, st);
      MOE_CUDA(moe::launch_finalize(fa, st));
    }
    ++launches;
  }

  L->last_M = M;
  L->last_launches = launches;
  return MOE_OK;
}

// A layer with a precision per expert (bf16 or e4m3; the per-expert FP8 choice of the
// kongchang.com page, "MoE Kernel Engineering Optimization Practices on Amazon
// SageMaker AI", section "Triton Backend Routing: A Practical Path to FP8
// Quantization"). Every expert's weights sit in a bf16-sized slot (an FP8 expert's
// codes in its first half); the align kernel lists the FP8 experts' tiles first, then
// the bf16 experts', and each GEMM runs as two launches, one per precision, over its
// own part of the list:
//   route (+ max|x|) -> align -> gather (bf16 rows or FP8 codes per row) ->
//   gate_up FP8 -> gate_up bf16 -> quant_h (FP8 experts' rows; s_h over them) ->
//   down FP8 -> down bf16 -> finalize
int forward_mixed(moe_layer* L, const void* x, const float* logits, int M, void* out, cudaStream_t st) {
  const long long P = static_cast<long long>(M) * L->k;
  const int rows_bound = static_cast<int>(P + std::min<long long>(L->E, P) * (moe::kPadRows - 1));
  const int f8 = moe::kFp8E4M3;
  int launches = 0;

  moe::RouteArgs ra{};
  ra.logits = logits;
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.M = M;
  ra.E = L->E;
  ra.k = L->k;
  ra.H = L->H;
  ra.topk_ids = L->topk_ids;
  ra.topk_w = L->topk_w;
  ra.amax_x = L->amax;
  ra.amax_h_reset = L->amax + 1;
  {
    KernelTimer kt(L, 0, st);
    MOE_CUDA(moe::launch_route(ra, st));
  }
  ++launches;

  moe::AlignArgs aa{};
  aa.topk_ids = L->topk_ids;
  aa.P = static_cast<int>(P);
  aa.E = L->E;
  aa.k = L->k;
  aa.BN = moe::kTokenBlock;
  aa.fblocks1 = L->I / moe::kTileRows;
  aa.fblocks2 = (L->H / moe::kTileRows + 1) / 2;
  aa.kblocks1 = L->H / 64;
  aa.kblocks2 = L->I / 64;
  aa.kblocks1_f8 = L->H / 128;
  aa.kblocks2_f8 = L->I / 128;
  aa.num_sms = L->num_sms;
  aa.ws1_rows_cap = static_cast<int>(L->ws1_rows_cap);
  aa.acc_slabs = 1;
  aa.uniform_splits = moe::uniform_splits() ? 1 : 0;
  aa.counts = L->counts;
  aa.padded_offsets = L->poff;
  aa.padded_pairs = L->pairs;
  aa.tiles1 = L->tiles1;
  aa.tiles2 = L->tiles2;
  aa.header = L->header;
  aa.eflags = L->eflags;
  {
    KernelTimer kt(L, 1, st);
    MOE_CUDA(moe::launch_align(aa, st));
  }
  ++launches;

  moe::GatherArgs ga{};
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.padded_pairs = L->pairs;
  ga.header = L->header;
  ga.rows_bound = rows_bound;
  ga.P = static_cast<int>(P);
  ga.k = L->k;
  ga.H = L->H;
  ga.x_perm = L->x_perm;
  ga.amax_x = L->amax;
  ga.f8 = f8;
  ga.eflags = L->eflags;
  ga.topk_ids = L->topk_ids;
  ga.x_perm8 = L->x_perm8;
  {
    KernelTimer kt(L, 2, st);
    MOE_CUDA(moe::launch_gather(ga, false, st));
  }
  ++launches;

  moe::GemmArgs g{};
  g.header = L->header;
  g.h = L->h;
  g.I = L->I;
  g.ws1 = L->ws1;
  g.tile_counters = L->counters;
  g.amax_h = L->amax + 1;
  g.amax_x = L->amax;
  g.w_scales = L->wscales;
  g.acc = L->acc;
  g.H = L->H;
  g.padded_pairs = L->pairs;
  g.topk_w = L->topk_w;
  g.k = L->k;
  g.P = static_cast<int>(P);
  g.f8 = f8;
  g.err = L->err;
  g.wait_budget = moe::wait_budget_cycles();

  // gate_up: FP8 experts, then bf16 experts (bf16-sized expert slots in both)
  moe::GemmArgs g1 = g;
  g1.tiles = L->tiles1;
  g1.w_rblocks = 2 * L->I / moe::kTileRows;
  g1.w_expert_tiles = static_cast<long long>(g1.w_rblocks) * (L->H / 64);
  g1.rb_step = 1;
  g1.second_rb = L->I / moe::kTileRows;
  g1.max_stages = moe::gemm_max_stages(true);
  moe::GemmArgs g1f = g1;
  g1f.hdr_tiles = moe::kHdrTiles1F8;
  g1f.hdr_splits = moe::kHdrSplits1F8;
  g1f.kblocks = L->H / 128;
  moe::GemmArgs g1b = g1;
  g1b.hdr_tile_offset = moe::kHdrTiles1F8;
  g1b.hdr_tiles = moe::kHdrTiles1BF;
  g1b.hdr_splits = moe::kHdrSplits1BF;
  g1b.kblocks = L->H / 64;
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_gemm1(g1f, L->tm_w13, L->tm_x8, true, L->num_sms, st));
  }
  {
    KernelTimer kt(L, 3, st);
    MOE_CUDA(moe::launch_gemm1(g1b, L->tm_w13, L->tm_x, false, L->num_sms, st));
  }
  launches += 2;

  moe::QuantHArgs qa{};
  qa.h = L->h;
  qa.h_q = L->h_q;
  qa.padded_pairs = L->pairs;
  qa.header = L->header;
  qa.rows_bound = rows_bound;
  qa.P = static_cast<int>(P);
  qa.I = L->I;
  qa.amax_h = L->amax + 1;
  qa.f8 = f8;
  qa.eflags = L->eflags;
  qa.topk_ids = L->topk_ids;
  {
    KernelTimer kt(L, 4, st);
    MOE_CUDA(moe::launch_quant_h(qa, st));
  }
  ++launches;

  moe::GemmArgs g2 = g;
  g2.tiles = L->tiles2;
  g2.w_rblocks = L->H / moe::kTileRows;
  g2.w_expert_tiles = static_cast<long long>(g2.w_rblocks) * (L->I / 64);
  g2.rb_step = 2;
  g2.second_rb = 1;
  g2.max_stages = moe::gemm_max_stages(false);
  moe::GemmArgs g2f = g2;
  g2f.hdr_tiles = moe::kHdrTiles2F8;
  g2f.hdr_splits = moe::kHdrSplits2F8;
  g2f.kblocks = L->I / 128;
  moe::GemmArgs g2b = g2;
  g2b.hdr_tile_offset = moe::kHdrTiles2F8;
  g2b.hdr_tiles = moe::kHdrTiles2BF;
  g2b.hdr_splits = moe::kHdrSplits2BF;
  g2b.kblocks = L->I / 64;
  {
    KernelTimer kt(L, 5, st);
    MOE_CUDA(moe::launch_gemm2(g2f, L->tm_wd, L->tm_hq, true, L->num_sms, st));
  }
  {
    KernelTimer kt(L, 5, st);
    MOE_CUDA(moe::launch_gemm2(g2b, L->tm_wd, L->tm_h, false, L->num_sms, st));
  }
  launches += 2;

  moe::FinalizeArgs fa{};
  fa.acc = L->acc;
  fa.out = static_cast<__nv_bfloat16*>(out);
  fa.n = static_cast<long long>(M) * L->H;
  fa.amax = L->amax;
  fa.last_scales = L->last_scales;
  fa.f8 = f8;
  {
    KernelTimer kt(L, 6, st);
    MOE_CUDA(moe::launch_finalize(fa, st));
  }
  ++launches;
  L->last_M = M;
  L->last_launches = launches;
  return MOE_OK;
}

}  // namespace

bool moe::pdl_enabled() {
  static const bool on = [] {
    const char* e = std::getenv("MOE_DISABLE_PDL");
    return !(e && e[0] == '1');
  }();
  return on;
}

long long moe::wait_budget_cycles() {
  const char* e = std::getenv("MOE_WAIT_BUDGET_CYCLES");
  return e ? std::atoll(e) : 0;
}

bool moe::fail_workspace_alloc() {
  const char* e = std::getenv("MOE_TEST_FAIL_WORKSPACE");
  return e != nullptr && e[0] == '1';
}

int moe::sm_count() {
  static int cached[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 148;
  if (dev >= 0 && dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) return 148;
  if (dev >= 0 && dev < 64) cached[dev] = n;
  return n;
}

bool moe::uniform_splits() {
  static const bool on = [] {
    const char* e = std::getenv("MOE_UNIFORM_SPLITS");
    return e && e[0] == '1';
  }();
  return on;
}

int moe::gemm_max_stages(bool gate_up) {
  static const int caps[2] = {[] {
                                const char* e = std::getenv("MOE_MAX_STAGES2");
                                return e ? std::atoi(e) : 6;   // measured best for the down GEMM
                              }(),
                              [] {
                                const char* e = std::getenv("MOE_MAX_STAGES1");
                                return e ? std::atoi(e) : 4;   // measured best for gate_up
                              }()};
  return caps[gate_up ? 1 : 0];
}

int moe_layer_view(const moe_layer* L, moe::LayerView* v) {
  if (!L || !v) return MOE_ERR_INVALID_ARG;
  v->E = L->E;
  v->k = L->k;
  v->H = L->H;
  v->I = L->I;
  v->device = L->device;
  v->num_sms = L->num_sms;
  v->fp8 = is_fp8(L);
  v->mixed = is_mixed(L);
  v->f8 = fp8_format(L);
  v->loaded = L->loaded;
  v->wscales = L->wscales;
  v->tm_w13 = L->tm_w13;
  v->tm_wd = L->tm_wd;
  return MOE_OK;
}

int moe_encode_tile_map(CUtensorMap* m, const void* base, bool fp8, long long inner, long long rows, int box_rows) {
  MOE_TRY(get_encoder());
  return encode_map(m, base, fp8, inner, rows, box_rows);
}

extern "C" {

const char* moe_status_string(int status) {
  switch (status) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument";
    case MOE_ERR_NOT_LOADED: return "weights not loaded";
    case MOE_ERR_OOM: return "device out of memory";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_UNSUPPORTED: return "unsupported device or shape";
    case MOE_ERR_DEVICE_TIMEOUT: return "device wait timed out";
    default: return "unknown status";
  }
}

int moe_create(int E, int topk, int H, int I, int dtype, moe_layer** out) {
  if (out == nullptr) return MOE_ERR_INVALID_ARG;
  *out = nullptr;
  if (E < 1 || E > 512 || topk < 1 || topk > 16 || topk > E) return MOE_ERR_INVALID_ARG;
  if (H < 128 || I < 128 || H > 16384 || I > 16384 || H % 128 || I % 128) return MOE_ERR_INVALID_ARG;
  if (dtype != MOE_DTYPE_BF16 && dtype != MOE_DTYPE_FP8_E4M3 && dtype != MOE_DTYPE_FP8_E5M2 &&
      dtype != MOE_DTYPE_MIXED_E4M3)
    return MOE_ERR_INVALID_ARG;
  int dev = 0;
  MOE_CUDA(cudaGetDevice(&dev));
  cudaDeviceProp prop;
  MOE_CUDA(cudaGetDeviceProperties(&prop, dev));
  if (prop.major != 10 || prop.minor != 0) return MOE_ERR_UNSUPPORTED;
  MOE_TRY(get_encoder());
  MOE_TRY(configure_device(dev));
  moe_layer* L = new (std::nothrow) moe_layer();
  if (!L) return MOE_ERR_OOM;
  L->E = E;
  L->k = topk;
  L->H = H;
  L->I = I;
  L->dtype = dtype;
  L->device = dev;
  L->num_sms = prop.multiProcessorCount;
  L->pair_clusters = std::min(moe::gemm_pair_clusters(), L->num_sms / 2);
  L->fused_decode = fused_decode_default();
  L->gemv_max_m = gemv_max_default(dtype, H);
  const size_t el = (dtype == MOE_DTYPE_BF16 || dtype == MOE_DTYPE_MIXED_E4M3) ? 2 : 1;
  if (cudaMalloc(&L->w13, static_cast<size_t>(E) * 2 * I * H * el) != cudaSuccess ||
      cudaMalloc(&L->wd, static_cast<size_t>(E) * H * I * el) != cudaSuccess ||
      cudaMalloc(&L->wscales, static_cast<size_t>(E) * 3 * sizeof(float)) != cudaSuccess ||
      (dtype == MOE_DTYPE_MIXED_E4M3 && cudaMalloc(&L->eflags, static_cast<size_t>(E) * sizeof(int)) != cudaSuccess)) {
    cudaFree(L->w13);
    cudaFree(L->wd);
    cudaFree(L->wscales);
    cudaFree(L->eflags);
    delete L;
    return MOE_ERR_OOM;
  }
  std::vector<float> ones(static_cast<size_t>(E) * 3, 1.f);
  cudaMemcpy(L->wscales, ones.data(), ones.size() * sizeof(float), cudaMemcpyHostToDevice);
  *out = L;
  return MOE_OK;
}

int moe_destroy(moe_layer* L) {
  if (!L) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaDeviceSynchronize();
  free_workspace(L);
  cudaFree(L->w13);
  cudaFree(L->wd);
  cudaFree(L->wscales);
  cudaFree(L->eflags);
  cudaFree(L->hx);
  cudaFree(L->hl);
  cudaFree(L->hout);
  for (auto& hg : L->host_graphs) cudaGraphExecDestroy(hg.exec);
  if (L->capture_stream) cudaStreamDestroy(L->capture_stream);
  for (auto& t : L->pending) {
    cudaEventDestroy(t.a);
    cudaEventDestroy(t.b);
  }
  for (auto e : L->event_pool) cudaEventDestroy(e);
  delete L;
  return MOE_OK;
}

int moe_load_weights(moe_layer* L, const void* w_gate, const void* w_up, const void* w_down, void* stream) {
  if (!L || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
  if (is_mixed(L)) return MOE_ERR_INVALID_ARG;   // needs the per-expert choice: moe_load_weights_mixed
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  L->loaded = false;
  const void* src[3] = {w_gate, w_up, w_down};
  MOE_TRY(load_bf16_sources(L, src, L->I, 0, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_TRY(encode_weight_maps(L));
  L->loaded = true;
  return MOE_OK;
}

int moe_load_weights_mixed(moe_layer* L, const void* w_gate, const void* w_up, const void* w_down,
                           const unsigned char* expert_fp8, void* stream) {
  if (!L || !w_gate || !w_up || !w_down || !expert_fp8) return MOE_ERR_INVALID_ARG;
  if (!is_mixed(L)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  L->loaded = false;
  std::vector<int> flags(static_cast<size_t>(L->E));
  for (int e = 0; e < L->E; ++e) flags[e] = expert_fp8[e] ? 1 : 0;
  MOE_CUDA(cudaMemcpyAsync(L->eflags, flags.data(), flags.size() * sizeof(int), cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaStreamSynchronize(st));   // `flags` is pageable host memory
  const void* src[3] = {w_gate, w_up, w_down};
  void* dst[3] = {L->w13, L->w13, L->wd};
  for (int j = 0; j < 3; ++j) {
    // bf16 experts: tiled copies into their slots
    moe::TileGeom gb = geom(L, j, 2, L->I, 0);
    gb.expert_mask = L->eflags;
    gb.mask_value = 0;
    MOE_CUDA(moe::launch_tile_weights(src[j], gb, dst[j], st));
    // FP8 experts: scale and e4m3 codes of their tensors, in the first half of a bf16-sized slot
    moe::TileGeom gf = gb;
    gf.expert_tiles = gb.rb_total * (gb.row_bytes / 128);
    gf.row_bytes = gb.row_bytes / 2;
    gf.mask_value = 1;
    const auto* w = static_cast<const __nv_bfloat16*>(src[j]);
    MOE_CUDA(moe::launch_weight_amax(moe::kFp8E4M3, w, gf, L->wscales + j, 3, st));
    MOE_CUDA(moe::launch_weight_quant_tiled(moe::kFp8E4M3, w, gf, L->wscales + j, 3, static_cast<uint8_t*>(dst[j]),
                                            st));
  }
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_TRY(encode_weight_maps(L));
  L->loaded = true;
  return MOE_OK;
}

int moe_load_weights_shard(moe_layer* L, const void* w_gate, const void* w_up, const void* w_down, int I_full,
                           int shard, int num_shards, void* stream) {
  if (!L || !w_gate || !w_up || !w_down) return MOE_ERR_INVALID_ARG;
  if (is_mixed(L)) return MOE_ERR_INVALID_ARG;
  if (num_shards < 1 || shard < 0 || shard >= num_shards) return MOE_ERR_INVALID_ARG;
  if (static_cast<long long>(L->I) * num_shards != I_full) return MOE_ERR_INVALID_ARG;
  if (!aligned16(w_gate) || !aligned16(w_up) || !aligned16(w_down)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  L->loaded = false;
  const void* src[3] = {w_gate, w_up, w_down};
  MOE_TRY(load_bf16_sources(L, src, I_full, shard, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_TRY(encode_weight_maps(L));
  L->loaded = true;
  return MOE_OK;
}

int moe_load_weights_fp8(moe_layer* L, const void* q_gate, const void* q_up, const void* q_down,
                         const float* scales_host, void* stream) {
  if (!L || !q_gate || !q_up || !q_down || !scales_host) return MOE_ERR_INVALID_ARG;
  if (!is_fp8(L)) return MOE_ERR_INVALID_ARG;
  if (!aligned16(q_gate) || !aligned16(q_up) || !aligned16(q_down)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t IH = static_cast<size_t>(L->I) * L->H;
  L->loaded = false;
  (void)IH;
  const void* src[3] = {q_gate, q_up, q_down};
  void* dst[3] = {L->w13, L->w13, L->wd};
  for (int j = 0; j < 3; ++j) MOE_CUDA(moe::launch_tile_weights(src[j], geom(L, j), dst[j], st));
  MOE_CUDA(cudaMemcpyAsync(L->wscales, scales_host, static_cast<size_t>(L->E) * 3 * sizeof(float),
                           cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaStreamSynchronize(st));
  MOE_TRY(encode_weight_maps(L));
  L->loaded = true;
  return MOE_OK;
}

int moe_reserve(moe_layer* L, int M_max, void* stream) {
  (void)stream;
  if (!L || M_max < 0) return MOE_ERR_INVALID_ARG;
  if (M_max == 0) return MOE_OK;
  DeviceGuard g(L->device);
  return ensure_workspace(L, M_max);
}

int moe_forward(moe_layer* L, const void* x, const float* logits, int M, void* out, void* stream) {
  if (!L || M < 0) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  if (M == 0) {
    L->last_launches = 0;
    L->last_M = 0;
    return MOE_OK;
  }
  if (M > (1 << 22) / L->k) return MOE_ERR_INVALID_ARG;
  if (!x || !logits || !out || !aligned16(x) || !aligned16(logits) || !aligned16(out)) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  moe::NvtxRange range("moe_forward");
  return forward_impl(L, x, logits, M, out, static_cast<cudaStream_t>(stream));
}

namespace {

bool is_pinned(const void* p) {
  cudaPointerAttributes a{};
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

// copies in, forward, copy out: enqueued on `st` (eagerly, or while capturing)
int host_chain(moe_layer* L, const void* x_host, const float* logits_host, int M, void* out_host, cudaStream_t st) {
  MOE_CUDA(cudaMemcpyAsync(L->hx, x_host, static_cast<size_t>(M) * L->H * 2, cudaMemcpyHostToDevice, st));
  MOE_CUDA(cudaMemcpyAsync(L->hl, logits_host, static_cast<size_t>(M) * L->E * 4, cudaMemcpyHostToDevice, st));
  MOE_TRY(forward_impl(L, L->hx, L->hl, M, L->hout, st));
  MOE_CUDA(cudaMemcpyAsync(out_host, L->hout, static_cast<size_t>(M) * L->H * 2, cudaMemcpyDeviceToHost, st));
  return MOE_OK;
}

// Graph of host_chain for these buffers (captured on the handle's own stream), or
// nullptr when it cannot be captured (the call then runs eagerly).
cudaGraphExec_t host_graph(moe_layer* L, const void* x_host, const float* logits_host, int M, void* out_host) {
  for (auto& hg : L->host_graphs)
    if (hg.M == M && hg.x == x_host && hg.l == logits_host && hg.out == out_host && hg.gen == L->graph_gen)
      return hg.exec;
  if (!L->capture_stream && cudaStreamCreateWithFlags(&L->capture_stream, cudaStreamNonBlocking) != cudaSuccess) {
    cudaGetLastError();
    L->capture_stream = nullptr;
    return nullptr;
  }
  cudaStream_t cs = L->capture_stream;
  if (cudaStreamBeginCapture(cs, cudaStreamCaptureModeThreadLocal) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  const int rc = host_chain(L, x_host, logits_host, M, out_host, cs);
  cudaGraph_t graph = nullptr;
  const cudaError_t e = cudaStreamEndCapture(cs, &graph);
  cudaGraphExec_t exec = nullptr;
  if (rc != MOE_OK || e != cudaSuccess || graph == nullptr ||
      cudaGraphInstantiate(&exec, graph, 0) != cudaSuccess) {
    cudaGetLastError();
    if (graph) cudaGraphDestroy(graph);
    return nullptr;
  }
  cudaGraphDestroy(graph);
  // keep at most kHostGraphs; stale generations go first, then the oldest
  constexpr size_t kHostGraphs = 16;
  for (size_t i = 0; i < L->host_graphs.size();) {
    if (L->host_graphs[i].gen != L->graph_gen) {
      cudaGraphExecDestroy(L->host_graphs[i].exec);
      L->host_graphs.erase(L->host_graphs.begin() + static_cast<long>(i));
    } else {
      ++i;
    }
  }
  if (L->host_graphs.size() >= kHostGraphs) {
    cudaGraphExecDestroy(L->host_graphs.front().exec);
    L->host_graphs.erase(L->host_graphs.begin());
  }
  L->host_graphs.push_back({M, x_host, logits_host, out_host, L->graph_gen, exec});
  return exec;
}

}  // namespace

int moe_forward_host(moe_layer* L, const void* x_host, const float* logits_host, int M, void* out_host,
                     void* stream) {
  if (!L || M < 0) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  if (M == 0) {
    L->last_launches = 0;
    return MOE_OK;
  }
  if (!x_host || !logits_host || !out_host) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (M > L->host_cap) {
    MOE_CUDA(cudaDeviceSynchronize());
    cudaFree(L->hx);
    cudaFree(L->hl);
    cudaFree(L->hout);
    L->hx = L->hout = nullptr;
    L->hl = nullptr;
    L->host_cap = 0;
    ++L->graph_gen;
    MOE_CUDA(cudaMalloc(&L->hx, static_cast<size_t>(M) * L->H * 2));
    MOE_CUDA(cudaMalloc(&L->hl, static_cast<size_t>(M) * L->E * 4));
    MOE_CUDA(cudaMalloc(&L->hout, static_cast<size_t>(M) * L->H * 2));
    L->host_cap = M;
  }
  MOE_TRY(ensure_workspace(L, M));   // (re)allocation happens here, never inside a capture
  moe::NvtxRange range("moe_forward_host");
  // Pinned buffers: one graph launch instead of three copies and five to ten kernel
  // launches from the host. Pageable buffers, profiling and the single-launch decode
  // kernel take the eager path.
  cudaGraphExec_t exec = nullptr;
  if (!L->profiling && !L->fused_decode && is_pinned(x_host) && is_pinned(logits_host) && is_pinned(out_host))
    exec = host_graph(L, x_host, logits_host, M, out_host);
  if (exec) {
    MOE_CUDA(cudaGraphLaunch(exec, st));
  } else {
    MOE_TRY(host_chain(L, x_host, logits_host, M, out_host, st));
  }
  MOE_CUDA(cudaStreamSynchronize(st));
  return MOE_OK;
}

int moe_get_device_error(moe_layer* L, int* code) {
  if (!L || !code) return MOE_ERR_INVALID_ARG;
  *code = 0;
  DeviceGuard g(L->device);
  MOE_CUDA(cudaDeviceSynchronize());
  if (L->err) {
    MOE_CUDA(cudaMemcpy(code, L->err, 4, cudaMemcpyDeviceToHost));
    if (*code != 0) MOE_CUDA(cudaMemset(L->err, 0, 4));
  }
  int na = 0;
  MOE_TRY(moe_noalloc_take_error(L->device, &na));
  if (*code == 0) *code = na;
  if (*code == 0) return MOE_OK;
  // a bounded wait that gave up, or (kErrBadTile) a tile that failed its bounds check
  return *code == moe::kErrBadTile ? MOE_ERR_CUDA : MOE_ERR_DEVICE_TIMEOUT;
}

int moe_last_launch_count(moe_layer* L) { return L ? L->last_launches : 0; }

int moe_last_gemm_pairs(moe_layer* L) { return (L && L->last_pair) ? 1 : 0; }

int moe_set_fused_decode(moe_layer* L, int enable) {
  if (!L) return MOE_ERR_INVALID_ARG;
  L->fused_decode = enable != 0;
  ++L->graph_gen;
  return MOE_OK;
}

int moe_set_gemv_max_tokens(moe_layer* L, int max_tokens) {
  if (!L || max_tokens > moe::kGemvMaxM) return MOE_ERR_INVALID_ARG;
  L->gemv_max_m = max_tokens < 0 ? gemv_max_default(L->dtype, L->H) : max_tokens;
  ++L->graph_gen;
  return MOE_OK;
}

int moe_profile_enable(moe_layer* L, int enable) {
  if (!L) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  MOE_TRY(drain_profile(L));
  for (int i = 0; i < MOE_PROFILE_SLOTS; ++i) {
    L->prof_ms[i] = 0.0;
    L->prof_n[i] = 0;
  }
  L->profiling = enable != 0;
  ++L->graph_gen;
  return MOE_OK;
}

int moe_profile_read(moe_layer* L, double* ms_sum, int* launches) {
  if (!L || !ms_sum || !launches) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  MOE_TRY(drain_profile(L));
  for (int i = 0; i < MOE_PROFILE_SLOTS; ++i) {
    ms_sum[i] = L->prof_ms[i];
    launches[i] = L->prof_n[i];
  }
  return MOE_OK;
}

int moe_debug_routing(moe_layer* L, int* topk_ids, float* topk_w, int* counts, int* padded_offsets,
                      int* padded_pairs, float* scales_host, int* tile_rows) {
  if (!L) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  MOE_CUDA(cudaDeviceSynchronize());
  if (tile_rows) *tile_rows = moe::kPadRows;
  if (L->M_cap == 0 || L->last_M == 0) return MOE_OK;
  const size_t P = static_cast<size_t>(L->last_M) * L->k;
  if (topk_ids) MOE_CUDA(cudaMemcpy(topk_ids, L->topk_ids, P * 4, cudaMemcpyDeviceToDevice));
  if (topk_w) MOE_CUDA(cudaMemcpy(topk_w, L->topk_w, P * 4, cudaMemcpyDeviceToDevice));
  if (counts) MOE_CUDA(cudaMemcpy(counts, L->counts, L->E * 4, cudaMemcpyDeviceToDevice));
  if (padded_offsets) MOE_CUDA(cudaMemcpy(padded_offsets, L->poff, (L->E + 1) * 4, cudaMemcpyDeviceToDevice));
  if (padded_pairs) {
    int rows = 0;
    MOE_CUDA(cudaMemcpy(&rows, L->header + moe::kHdrRowsUsed, 4, cudaMemcpyDeviceToHost));
    MOE_CUDA(cudaMemcpy(padded_pairs, L->pairs, static_cast<size_t>(rows) * 4, cudaMemcpyDeviceToDevice));
  }
  if (scales_host) MOE_CUDA(cudaMemcpy(scales_host, L->last_scales, 8, cudaMemcpyDeviceToHost));
  return MOE_OK;
}

int moe_debug_activations(moe_layer* L, void* x_perm_out, void* h_out) {
  if (!L) return MOE_ERR_INVALID_ARG;
  DeviceGuard g(L->device);
  MOE_CUDA(cudaDeviceSynchronize());
  if (L->M_cap == 0 || L->last_M == 0) return MOE_OK;
  int rows = 0;
  MOE_CUDA(cudaMemcpy(&rows, L->header + moe::kHdrRowsUsed, 4, cudaMemcpyDeviceToHost));
  const size_t el = is_fp8(L) ? 1 : 2;
  if (x_perm_out && L->last_small && is_fp8(L)) {
    // the small-batch path quantised x once per token and read those rows directly:
    // lay its codes out in expert order here (the gather kernel copying code rows)
    moe::GatherArgs ga{};
    ga.padded_pairs = L->pairs;
    ga.header = L->header;
    ga.rows_bound = rows;
    ga.P = L->last_M * L->k;
    ga.k = L->k;
    ga.H = L->H;
    ga.x_perm = x_perm_out;
    ga.amax_x = L->amax;
    ga.f8 = fp8_format(L);
    ga.xq = L->xq;
    MOE_CUDA(moe::launch_gather(ga, true, nullptr));
    MOE_CUDA(cudaDeviceSynchronize());
  } else if (x_perm_out) {
    MOE_CUDA(cudaMemcpy(x_perm_out, L->x_perm, static_cast<size_t>(rows) * L->H * el, cudaMemcpyDeviceToDevice));
  }
  if (h_out) MOE_CUDA(cudaMemcpy(h_out, L->h, static_cast<size_t>(rows) * L->I * 2, cudaMemcpyDeviceToDevice));
  return MOE_OK;
}

int moe_debug_weights(moe_layer* L, void* gate_out, void* up_out, void* down_out, float* scales_host) {
  if (!L) return MOE_ERR_INVALID_ARG;
  if (!L->loaded) return MOE_ERR_NOT_LOADED;
  if (is_mixed(L)) return MOE_ERR_UNSUPPORTED;
  DeviceGuard g(L->device);
  MOE_CUDA(cudaDeviceSynchronize());
  void* outs[3] = {gate_out, up_out, down_out};
  const void* srcs[3] = {L->w13, L->w13, L->wd};
  for (int j = 0; j < 3; ++j)
    if (outs[j]) MOE_CUDA(moe::launch_untile_weights(srcs[j], geom(L, j), outs[j], nullptr));
  MOE_CUDA(cudaDeviceSynchronize());
  if (scales_host && is_fp8(L))
    MOE_CUDA(cudaMemcpy(scales_host, L->wscales, static_cast<size_t>(L->E) * 3 * 4, cudaMemcpyDeviceToHost));
  return MOE_OK;
}

}  // extern "C"
