// moe_noalloc.cu - moe_forward_noalloc: the forward pass for callers that must not
// allocate device memory.
//
// moe_forward sizes its per-call scratch (permuted activations, the intermediate h,
// split-K partial sums, the fp32 combine accumulator, tile lists) on first use and
// grows it with cudaMalloc when a larger batch arrives. Some callers cannot let a
// library do that: a serving runtime that hands out all of HBM to its own pool at
// start-up and forbids later allocations, and latency-critical loops that cannot
// afford the device-wide synchronisation a cudaMalloc/cudaFree may bring. For them this entry point takes all per-call
// scratch from one fixed array in device memory, kScratchBytes large, defined at file
// scope below. Every GPU that loads the library holds that array until the process
// exits. The layer's weights are still the ones moe_load_weights stored in the
// handle; the caller passes the inputs and the output.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdio>
#include <mutex>

#include "../../include/moe_b200.h"
#include "moe_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(32) << 20;   // 32 MiB per device
constexpr int kMaxDevices = 64;
constexpr long long kSplitRowsMax = 1024;             // split-K partial-sum rows kept in the scratch

static __device__ __align__(256) unsigned char g_scratch[kScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of g_scratch on `dev` (the current device). In host code the name
// g_scratch is only a host-side stand-in, so the address is looked up once per device
// and cached; kernels are always given this looked-up address.
int scratch_address(int dev, void** out) {
  if (dev < 0 || dev >= kMaxDevices) return MOE_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_scratch);
    if (e != cudaSuccess || p == nullptr) {
      std::fprintf(stderr, "moe_forward_noalloc: cudaGetSymbolAddress failed: %s\n", cudaGetErrorString(e));
      return MOE_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return MOE_OK;
}

// The first 256 bytes of the array hold the device error word of this path (kernels
// whose bounded waits give up record a code there, first error wins). Calls never
// clear it: moe_get_device_error reads and clears it (static device memory starts
// at zero). The per-call scratch is carved from the rest.
constexpr size_t kErrWordBytes = 256;

// Bump allocator over the scratch array: 256-byte aligned pieces, no device calls.
struct Carve {
  unsigned char* base;
  size_t off = kErrWordBytes;
  template <class T>
  T* take(size_t bytes) {
    off = (off + 255) & ~size_t(255);
    T* p = reinterpret_cast<T*>(base + off);
    off += bytes;
    return p;
  }
};

#define NA_CUDA(call)                                                                              \
  do {                                                                                             \
    cudaError_t e_ = (call);                                                                       \
    if (e_ != cudaSuccess) {                                                                       \
      std::fprintf(stderr, "moe_forward_noalloc: %s failed: %s\n", #call, cudaGetErrorString(e_)); \
      return MOE_ERR_CUDA;                                                                         \
    }                                                                                              \
  } while (0)

#define NA_TRY(call)             \
  do {                           \
    int s_ = (call);             \
    if (s_ != MOE_OK) return s_; \
  } while (0)

int forward_noalloc(const moe::LayerView& v, const void* x, const float* logits, int M, void* out,
                    cudaStream_t st) {
  void* base = nullptr;
  NA_TRY(scratch_address(v.device, &base));

  const long long P = static_cast<long long>(M) * v.k;
  const int BN = moe::kTokenBlock;
  const long long Emin = std::min<long long>(v.E, P);
  const long long rows_cap = P + Emin * (moe::kPadRows - 1);
  const long long nblocks = (P + BN - 1) / BN + Emin;
  const long long t1 = nblocks * (v.I / moe::kTileRows);
  const long long t2 = nblocks * ((v.H / moe::kTileRows + 1) / 2);
  const long long ws1_rows = std::min(rows_cap, kSplitRowsMax);
  const size_t el = v.fp8 ? 1 : 2;

  Carve c{static_cast<unsigned char*>(base)};
  int* topk_ids = c.take<int>(P * 4);
  float* topk_w = c.take<float>(P * 4);
  int* counts = c.take<int>((v.E + 1) * 4);
  int* poff = c.take<int>((v.E + 1) * 4);
  int* pairs = c.take<int>(rows_cap * 4);
  moe::Tile* tiles1 = c.take<moe::Tile>(t1 * sizeof(moe::Tile));
  moe::Tile* tiles2 = c.take<moe::Tile>(t2 * sizeof(moe::Tile));
  int* header = c.take<int>(moe::kHdrSlots * 4);
  void* x_perm = c.take<unsigned char>(rows_cap * v.H * el);
  __nv_bfloat16* h = c.take<__nv_bfloat16>(rows_cap * v.I * 2);
  uint8_t* h_q = v.fp8 ? c.take<uint8_t>(rows_cap * v.I) : nullptr;
  // everything from here on must start at zero: one memset covers it
  const size_t zero_from = (c.off + 255) & ~size_t(255);
  float* ws1 = c.take<float>(ws1_rows * 2 * v.I * 4);
  int* counters = c.take<int>(t1 * 4);
  float* acc = c.take<float>(static_cast<size_t>(M) * v.H * 4);
  unsigned* amax = c.take<unsigned>(2 * 4);
  const size_t used = c.off;
  if (used > kScratchBytes) {
    std::fprintf(stderr,
                 "moe_forward_noalloc: a batch of M=%d tokens needs %zu bytes of scratch; the static "
                 "scratch holds %zu bytes (use moe_forward for larger batches)\n",
                 M, used, kScratchBytes);
    return MOE_ERR_INVALID_ARG;
  }
  NA_CUDA(cudaMemsetAsync(static_cast<unsigned char*>(base) + zero_from, 0, used - zero_from, st));

  CUtensorMap tm_x, tm_h;
  NA_TRY(moe_encode_tile_map(&tm_x, x_perm, v.fp8, v.H, rows_cap, 16));
  NA_TRY(moe_encode_tile_map(&tm_h, v.fp8 ? static_cast<void*>(h_q) : static_cast<void*>(h), v.fp8, v.I,
                             rows_cap, 16));

  const int rows_bound = static_cast<int>(rows_cap);
  const int kper = v.fp8 ? 128 : 64;

  moe::RouteArgs ra{};
  ra.logits = logits;
  ra.x = static_cast<const __nv_bfloat16*>(x);
  ra.M = M;
  ra.E = v.E;
  ra.k = v.k;
  ra.H = v.H;
  ra.topk_ids = topk_ids;
  ra.topk_w = topk_w;
  ra.amax_x = v.fp8 ? amax : nullptr;
  NA_CUDA(moe::launch_route(ra, st));

  moe::AlignArgs aa{};
  aa.topk_ids = topk_ids;
  aa.P = static_cast<int>(P);
  aa.E = v.E;
  aa.k = v.k;
  aa.BN = BN;
  aa.fblocks1 = v.I / moe::kTileRows;
  aa.fblocks2 = (v.H / moe::kTileRows + 1) / 2;
  aa.kblocks1 = v.H / kper;
  aa.kblocks2 = v.I / kper;
  aa.num_sms = v.num_sms;
  aa.ws1_rows_cap = static_cast<int>(ws1_rows);
  aa.uniform_splits = moe::uniform_splits() ? 1 : 0;
  aa.counts = counts;
  aa.padded_offsets = poff;
  aa.padded_pairs = pairs;
  aa.tiles1 = tiles1;
  aa.tiles2 = tiles2;
  aa.header = header;
  NA_CUDA(moe::launch_align(aa, st));

  moe::GatherArgs ga{};
  ga.x = static_cast<const __nv_bfloat16*>(x);
  ga.padded_pairs = pairs;
  ga.header = header;
  ga.rows_bound = rows_bound;
  ga.P = static_cast<int>(P);
  ga.k = v.k;
  ga.H = v.H;
  ga.x_perm = x_perm;
  ga.amax_x = amax;
  ga.f8 = v.f8;
  NA_CUDA(moe::launch_gather(ga, v.fp8, st));

  moe::GemmArgs g{};
  g.header = header;
  g.h = h;
  g.I = v.I;
  g.ws1 = ws1;
  g.tile_counters = counters;
  g.amax_h = amax + 1;
  g.amax_x = amax;
  g.w_scales = v.wscales;
  g.acc = acc;
  g.H = v.H;
  g.padded_pairs = pairs;
  g.topk_w = topk_w;
  g.k = v.k;
  g.P = static_cast<int>(P);
  g.f8 = v.f8;
  g.err = static_cast<int*>(base);
  g.wait_budget = moe::wait_budget_cycles();

  moe::GemmArgs g1 = g;
  g1.tiles = tiles1;
  g1.hdr_tiles = moe::kHdrTiles1;
  g1.hdr_splits = moe::kHdrSplits1;
  g1.kblocks = aa.kblocks1;
  g1.w_rblocks = 2 * v.I / moe::kTileRows;
  g1.rb_step = 1;
  g1.second_rb = v.I / moe::kTileRows;
  g1.max_stages = moe::gemm_max_stages(true);
  NA_CUDA(moe::launch_gemm1(g1, v.tm_w13, tm_x, v.fp8, v.num_sms, st));

  if (v.fp8) {
    moe::QuantHArgs qa{};
    qa.h = h;
    qa.h_q = h_q;
    qa.padded_pairs = pairs;
    qa.header = header;
    qa.rows_bound = rows_bound;
    qa.P = static_cast<int>(P);
    qa.I = v.I;
    qa.amax_h = amax + 1;
    qa.f8 = v.f8;
    NA_CUDA(moe::launch_quant_h(qa, st));
  }

  moe::GemmArgs g2 = g;
  g2.tiles = tiles2;
  g2.hdr_tiles = moe::kHdrTiles2;
  g2.hdr_splits = moe::kHdrSplits2;
  g2.kblocks = aa.kblocks2;
  g2.w_rblocks = v.H / moe::kTileRows;
  g2.rb_step = 2;
  g2.second_rb = 1;
  g2.max_stages = moe::gemm_max_stages(false);
  NA_CUDA(moe::launch_gemm2(g2, v.tm_wd, tm_h, v.fp8, v.num_sms, st));

  moe::FinalizeArgs fa{};
  fa.acc = acc;
  fa.out = static_cast<__nv_bfloat16*>(out);
  fa.n = static_cast<long long>(M) * v.H;
  fa.amax = nullptr;
  fa.last_scales = nullptr;
  fa.f8 = v.f8;
  NA_CUDA(moe::launch_finalize(fa, st));
  return MOE_OK;
}

}  // namespace

int moe_noalloc_take_error(int dev, int* code) {
  *code = 0;
  if (dev < 0 || dev >= kMaxDevices) return MOE_OK;
  void* p = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_scratch_mu);
    p = g_scratch_addr[dev];
  }
  if (p == nullptr) return MOE_OK;   // the path never ran on this device
  NA_CUDA(cudaMemcpy(code, p, sizeof(int), cudaMemcpyDeviceToHost));
  if (*code != 0) NA_CUDA(cudaMemset(p, 0, sizeof(int)));
  return MOE_OK;
}

extern "C" int moe_forward_noalloc(moe_layer* layer, const void* x, const float* router_logits, int M,
                                   void* out, void* stream) {
  moe::LayerView v;
  if (!layer || M < 0 || moe_layer_view(layer, &v) != MOE_OK) return MOE_ERR_INVALID_ARG;
  if (!v.loaded) return MOE_ERR_NOT_LOADED;
  if (v.mixed) return MOE_ERR_UNSUPPORTED;   // a precision per expert runs through moe_forward only
  if (M == 0) return MOE_OK;
  auto misaligned = [](const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) != 0; };
  if (!x || !router_logits || !out || misaligned(x) || misaligned(router_logits) || misaligned(out))
    return MOE_ERR_INVALID_ARG;
  if (M > (1 << 22) / v.k) return MOE_ERR_INVALID_ARG;
  int prev = -1;
  NA_CUDA(cudaGetDevice(&prev));
  if (prev != v.device) NA_CUDA(cudaSetDevice(v.device));
  moe::NvtxRange range("moe_forward_noalloc");
  const int status = forward_noalloc(v, x, router_logits, M, out, static_cast<cudaStream_t>(stream));
  if (prev != v.device) cudaSetDevice(prev);
  return status;
}
