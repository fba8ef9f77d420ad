// moe_internal.h - structures shared by the host dispatcher and the kernels.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>
#include <stdint.h>

namespace moe {

// An NVTX range around a host-side scope (a forward pass, one kernel launch, a weight
// load), so that a timeline tool shows the layer's steps by name. Header-only NVTX3:
// without a tool attached a push/pop costs a pointer test.
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange&) = delete;
  NvtxRange& operator=(const NvtxRange&) = delete;
};

constexpr int kPadRows = 16;        // every expert's group of rows is padded to 16 (B tile granule)
constexpr int kTileRows = 128;      // weight rows per GEMM tile (the MMA's M slot)
constexpr int kRowBytes = 128;      // bytes per K block row (one 128-byte swizzle atom)
constexpr int kMaxSplits = 16;      // largest split-K factor the scheduler picks

// Layout of the scheduler header written by the align kernel (int32 slots).
enum HeaderSlot : int {
  kHdrRowsUsed = 0,     // padded rows in use (= padded_offsets[E])
  kHdrTiles1 = 1,       // gate_up tiles
  kHdrSplits1 = 2,      // gate_up split-K factor (0 = the balanced schedule)
  kHdrTiles2 = 3,       // down tiles
  kHdrSplits2 = 4,      // down split-K factor (0 = the balanced schedule)
  kHdrTokenBlocks = 5,  // (expert, token block) pairs
  kHdrMaxRows = 6,      // widest token tile (rows of activations a stage must hold), <= BN
  // layers with a precision per expert: the tile lists hold the FP8 experts' tiles
  // first, then the bf16 experts' tiles; count and split factor of each part
  kHdrTiles1F8 = 8,
  kHdrSplits1F8 = 9,
  kHdrTiles1BF = 10,
  kHdrSplits1BF = 11,
  kHdrTiles2F8 = 12,
  kHdrSplits2F8 = 13,
  kHdrTiles2BF = 14,
  kHdrSplits2BF = 15,
  kHdrSlots = 16
};

// One output tile of a grouped GEMM: weight rows [fblock*128, +128) of expert
// `expert` times the token rows [row_start, row_start + n_valid) of the permuted
// activations (row_start is a multiple of 16; n_valid in 1..BN).
struct __align__(16) Tile {
  int expert;
  int fblock;
  int row_start;
  int n_valid;
};

struct RouteArgs {
  const float* logits;     // [M, E]
  const __nv_bfloat16* x;  // [M, H], read only for the FP8 amax
  int M, E, k, H;
  int* topk_ids;           // [M, k]
  float* topk_w;           // [M, k]
  unsigned* amax_x;        // FP8 only (else nullptr): running max |x| as float bits
  unsigned* amax_h_reset;  // when set: the max |h| word, zeroed before gate_up folds into it
};

struct AlignArgs {
  const int* topk_ids;     // [P]
  int P, E, k;
  int BN;                  // token rows per tile (kTokenBlock)
  int fblocks1, fblocks2;  // tiles across the output features: I/128 (gate_up), ceil(H/256) (down)
  int kblocks1, kblocks2;  // K blocks of gate_up (H) and down (I)
  int num_sms;
  int ws1_rows_cap;        // split-K of gate_up needs rows_used <= this
  int acc_slabs;           // down tiles ordered in this many feature slabs (<= fblocks2; 0 or 1: none)
  int uniform_splits;      // 1: one split-K factor per GEMM from a cost model; 0: balanced
  int* counts;             // [E]
  int* padded_offsets;     // [E+1]
  int* padded_pairs;       // [rows_cap]
  Tile* tiles1;
  Tile* tiles2;
  int* header;             // [kHdrSlots]
  // Multi-block path (large batches), when chunk_counts is set: pairs are taken in
  // chunks of kAlignChunk; align_count_kernel writes each chunk's per-expert counts,
  // align_kernel then sums them and writes chunk_base (the first padded row of each
  // (chunk, expert) group) instead of placing the pairs itself, and
  // align_scatter_kernel places them.
  int* chunk_counts;       // [chunks, E]
  int* chunk_base;         // [chunks, E]
  int chunks;
  // Precision per expert (nullptr: one precision for the layer): eflags[e] = 1 for an
  // FP8 expert. The tile lists then hold the FP8 experts' tiles first; kblocks1/2 are
  // the bf16 K blocks and kblocks1_f8/2_f8 the FP8 ones (128-byte rows of each).
  const int* eflags;
  int kblocks1_f8, kblocks2_f8;
};

struct GatherArgs {
  const __nv_bfloat16* x;  // [M, H]
  const int* padded_pairs;
  const int* header;
  int rows_bound;          // grid covers this many rows; rows >= rows_used exit
  int P, k, H;
  void* x_perm;            // [rows_cap, H] bf16 or FP8 codes
  const unsigned* amax_x;  // FP8 only
  int f8;                  // FP8 code format (Fp8Format)
  const uint8_t* xq;       // FP8: token rows already quantised [M, H] (copy bytes), or nullptr
  // precision per expert (nullptr: none): rows of FP8 experts get codes in x_perm8,
  // the others bf16 copies in x_perm
  const int* eflags;
  const int* topk_ids;     // [P] expert of each pair (with eflags)
  uint8_t* x_perm8;        // [rows_cap, H] FP8 codes (with eflags)
};

struct QuantXArgs {
  const __nv_bfloat16* x;  // [M, H]
  uint8_t* xq;             // [M, H] FP8 codes
  int M, H;
  const unsigned* amax_x;
  int f8;
};

struct GemmArgs {
  const Tile* tiles;
  const int* header;
  int hdr_tiles, hdr_splits;
  int kblocks;             // K blocks over the whole reduction
  int w_rblocks;           // 128-row blocks of one expert's weights (2I/128 or H/128)
  long long w_expert_tiles; // stored tiles per expert slot (0: w_rblocks * kblocks; more
                            //   when FP8 experts sit in bf16-sized slots)
  int hdr_tile_offset;     // header slot holding the index of this GEMM's first tile (0: none)
  int rb_step;             // tile row block f covers weight row blocks f*rb_step and
  int second_rb;           //   f*rb_step + second_rb (gate_up: 1 and I/128; down: 2 and 1)
  int pair_rb;             // CTA-pair kernels: the second CTA's row blocks are pair_rb further
                           //   (gate_up: rb_step 2, pair_rb 1; down: rb_step 4, pair_rb 2)
  // gate_up epilogue
  __nv_bfloat16* h;        // [rows_cap, I]
  int I;
  float* ws1;              // [ws1_rows_cap, 2I] split-K partial sums (zero between uses)
  int* tile_counters;      // [tiles1_cap] (zero between uses)
  unsigned* amax_h;        // FP8: running max |h| as float bits
  const unsigned* amax_x;  // FP8: max |x| (for s_x)
  const float* w_scales;   // FP8: [E, 3]
  // down epilogue
  float* acc;              // [M, H] fp32 accumulator (zero between uses)
  int H;
  const int* padded_pairs;
  const float* topk_w;
  int k, P;
  // down with the combine folded in (token_cnt set): the epilogue that adds a token's last
  // K block turns its row of `acc` into `out` (and clears it); the last CTA to finish
  // writes the FP8 scales of the forward and clears the amax words. No finalize launch.
  int* token_cnt;          // [M] K blocks added per token (zero between forwards)
  int token_need;          // K blocks a token receives in all (k x tiles across H x K blocks)
  int* cta_done;           // CTAs finished (zero between forwards)
  __nv_bfloat16* out;      // [M, H]
  unsigned* amax;          // FP8: [2] the forward's amax words (cleared at the end)
  float* last_scales;      // FP8: [2] s_x, s_h of the forward
  int max_stages;          // upper bound of the stage ring depth (<= the kernel's own maximum)
  int wait_first;          // 1: the previous kernel wrote the tile list (wait before reading it)
  const int* direct_pairs; // gate_up only: B rows are x rows of token pairs[row]/k (x map box = 1 row)
  int f8;                  // FP8 layers: code format of weights and activations (Fp8Format)
  int* err;
  long long wait_budget;   // SM cycles a pipeline wait may take (0: about a second)
};

struct QuantHArgs {
  const __nv_bfloat16* h;
  uint8_t* h_q;
  const int* padded_pairs;
  const int* header;
  int rows_bound, P, I;
  const unsigned* amax_h;
  int f8;                  // FP8 code format (Fp8Format)
  const int* eflags;       // precision per expert (nullptr: none): only FP8 experts' rows
  const int* topk_ids;     // [P] (with eflags)
};

struct FinalizeArgs {
  float* acc;              // [M, H]
  __nv_bfloat16* out;      // [M, H]
  long long n;             // M*H
  unsigned* amax;          // [2] reset to 0 (may be nullptr)
  float* last_scales;      // [2] s_x, s_h of this forward (may be nullptr)
  int f8;                  // FP8 code format (Fp8Format)
};

// Launch with programmatic stream serialisation (PDL) unless MOE_DISABLE_PDL=1 is set
// in the environment: the kernel may be scheduled before its predecessor in the stream
// finishes, and orders itself with griddepcontrol (see sm100.cuh).
bool pdl_enabled();
// Streaming multiprocessors of the current device (looked up once per device).
int sm_count();
// MOE_UNIFORM_SPLITS=1 replaces the balanced unit schedule by one split factor per GEMM
bool uniform_splits();
int gemm_max_stages(bool gate_up);   // ring depth cap (MOE_MAX_STAGES1/2 override, for tuning)
// Budget of the GEMMs' pipeline waits in SM cycles: 0 (the default, about a second)
// unless MOE_WAIT_BUDGET_CYCLES is set; read at every forward, so that a test can make
// a wait run out on purpose and then restore the default in the same process.
long long wait_budget_cycles();
// MOE_TEST_FAIL_WORKSPACE=1 (read at every forward): the workspace allocation reports
// an out-of-memory failure without allocating (a host-side failure injection for tests).
bool fail_workspace_alloc();
template <typename... KArgs, typename... Args>
inline cudaError_t launch_kernel(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                 Args... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = at;
  cfg.numAttrs = pdl_enabled() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, args...);
}

// Token rows per GEMM tile: the widest N of an M = 128 MMA. An expert with more
// tokens gets several token blocks.
constexpr int kTokenBlock = 256;

// Kernel launchers (each returns the cudaError_t of its launch).
cudaError_t launch_route(const RouteArgs& a, cudaStream_t s);
cudaError_t launch_align(const AlignArgs& a, cudaStream_t s);
constexpr int kAlignChunk = 1024;   // pairs per block of the multi-block align path
cudaError_t launch_align_count(const AlignArgs& a, cudaStream_t s);
cudaError_t launch_align_scatter(const AlignArgs& a, cudaStream_t s);
cudaError_t launch_gather(const GatherArgs& a, bool fp8, cudaStream_t s);
// pair: clusters of two CTAs running M = 256 MMAs (grid even; a.rb_step / a.pair_rb and the
// align kernel's tile lists set up for pairs)
cudaError_t launch_gemm1(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& x, bool fp8, int grid,
                         cudaStream_t s, bool pair = false);
cudaError_t launch_gemm2(const GemmArgs& a, const CUtensorMap& w, const CUtensorMap& h, bool fp8, int grid,
                         cudaStream_t s, bool pair = false);
cudaError_t launch_quant_h(const QuantHArgs& a, cudaStream_t s);
cudaError_t launch_quant_x(const QuantXArgs& a, cudaStream_t s);
cudaError_t launch_finalize(const FinalizeArgs& a, cudaStream_t s);
cudaError_t gemm_configure();    // opt-in dynamic shared memory sizes (current device)
// CTA pairs of the grouped GEMMs that can be resident at once on the current device (0:
// none): the pair kernels' grid is twice this, so that every pair runs in one wave.
int gemm_pair_clusters();
cudaError_t align_configure();
cudaError_t route_configure();   // shared-memory carveout of the one-row kernels

// Single-launch decode path (kernels_decode.cu): the whole layer for M <= 64 tokens
// (bf16 or FP8) in one cooperative persistent kernel.
struct DecodeLaunch {
  const float* logits;
  const __nv_bfloat16* x;
  __nv_bfloat16* out;
  int M, E, k, H, I, grid, ws1_rows_cap, max_stages;
  bool fp8;
  int f8;                  // FP8 code format (Fp8Format)
  int* sync;               // decode_sync_words(E, M_cap) ints, zero between launches
  uint8_t* xq;             // FP8: [M_cap, H] codes of x (tm_x maps it, one-row boxes)
  uint8_t* hq;             // FP8: [rows_cap, I] codes of h (tm_h maps it)
  float* last_scales;      // FP8: [2] s_x, s_h of the forward
  int* topk_ids;           // routing copies for inspection
  float* topk_w;
  int* counts;
  int* padded_offsets;
  int* padded_pairs;
  int* header;
  GemmArgs g1, g2;
  const CUtensorMap* tm_w13;
  const CUtensorMap* tm_wd;
  const CUtensorMap* tm_x;   // token rows of x (bf16) or of xq (FP8), one-row boxes
  const CUtensorMap* tm_h;   // h (bf16) or its codes (FP8), 16-row boxes
};
bool decode_supported(int M, int E, int k);
size_t decode_sync_words(int E, int M_cap);
cudaError_t decode_configure();
cudaError_t launch_decode(const DecodeLaunch& l, cudaStream_t st);

// Small batches (kernels_small.cu): the grouped GEMMs build the batch's schedule
// themselves from the routing (no align kernel), gate_up reads token rows directly (no
// gather) and down finishes token rows itself (no finalize).
struct SmallArgs {
  const int* topk_ids;     // [P] from the route kernel
  const float* topk_w;     // [P]
  __nv_bfloat16* out;      // down: [M, H]
  int M, E, k, H, I, P, ws1_rows_cap, uniform, f8;
  int* token_cnt;          // down: [M] K blocks added per token (zero between calls)
  int* done;               // down: [1] CTAs finished (zero between calls)
  unsigned* amax;          // FP8: [2] max|x|, max|h| (reset by down's last CTA)
  float* last_scales;      // FP8: [2] s_x, s_h of the forward
  int* counts;             // gate_up (CTA 0): copies of the schedule
  int* padded_offsets;
  int* padded_pairs;
  int* header;
  GemmArgs g;
};
bool small_supported(int M, int E, int k);
cudaError_t small_configure();
cudaError_t launch_small_gate_up(const SmallArgs& a, const CUtensorMap& w, const CUtensorMap& x, bool fp8, int grid,
                                 cudaStream_t s);
cudaError_t launch_small_down(const SmallArgs& a, const CUtensorMap& w, const CUtensorMap& h, bool fp8, int grid,
                              cudaStream_t s);

// Thin batches (kernels_gemv.cu): when every expert holds only a few tokens, each
// weight byte feeds one or two multiply-adds, far below the tensor cores' ridge, and
// the layer is a set of matrix-vector products that the CUDA cores finish at HBM
// speed. The forward is then route+plan -> gate_up -> down: no align, gather, split-K
// or finalize step; down writes bf16 `out` directly.
constexpr int kGemvMaxM = 16;        // largest batch of the path (token masks in the plan)
inline long long gemv_records_cap(int E, long long P) { return P < E ? P : E; }
constexpr int kHdrGemvActive = 7;    // header slot: number of active experts
struct GemvArgs {
  const float* logits;     // [M, E]
  const __nv_bfloat16* x;  // [M, H]
  int M, E, k, H, I;
  int* topk_ids;           // [P]
  float* topk_w;           // [P]
  // plan written by the route kernel: the align kernel's padded groups (counts, padded
  // offsets, padded pairs, rows used) and the active experts in ascending id order as
  // {expert, tokens, first padded row, 0}, their number in header[kHdrGemvActive]
  int* counts;
  int* padded_offsets;
  int* padded_pairs;
  int* header;
  int4* active;            // [min(E, P)] (gemv_records_cap)
  unsigned* amax;          // FP8: [2] max|x| (stored by the route kernel), max|h| (atomic max)
  uint8_t* xq;             // FP8: [M, H] codes of x (nullptr: bf16 layer)
  float* last_scales;      // FP8: [2] s_x, s_h of the forward
  int f8;                  // FP8 code format (Fp8Format)
  // weights in the tiled layout (TileGeom below)
  const uint8_t* w13;
  const uint8_t* wd;
  const float* w_scales;   // FP8: [E, 3]
  long long et1, et2;      // stored tiles per expert slot
  int kb1, kb2;            // 128-byte K blocks per row: H*b/128 (gate_up), I*b/128 (down)
  __nv_bfloat16* h;        // [P, I] h rows by pair id
  __nv_bfloat16* out;      // [M, H]
  int prefetch_kb;         // down: K blocks per expert asked into L2 before the wait (0: none)
  // down: each CTA takes a contiguous range of at most dn_units (token, 16 features)
  // units, spanning at most dn_tokens tokens (the host sizes shared memory from both)
  int dn_units, dn_tokens;
  int grid;                // CTAs of gate_up and down (two per SM)
};
// The path serves 1 <= M <= kGemvMaxM when the per-CTA staging fits shared memory
// (grid: two CTAs per SM, `sms` SMs).
bool gemv_supported(int M, int E, int k, int H, int I, int sms, bool fp8);
// Shared memory of the down kernel for a batch on `sms` SMs (fills a.grid, a.dn_units and
// a.dn_tokens).
size_t gemv_down_plan(GemvArgs& a, int sms);
cudaError_t gemv_configure();
// The three launches of the path (fmt: 0 bf16, 1 e4m3, 2 e5m2); gate_up and down run
// two CTAs per SM.
cudaError_t launch_gemv_plan(const GemvArgs& a, cudaStream_t s);
cudaError_t launch_gemv_gate_up(const GemvArgs& a, int fmt, cudaStream_t s);
cudaError_t launch_gemv_down(const GemvArgs& a, int fmt, cudaStream_t s);

// Weight preparation (load time, not on the forward path). Stored weights are
// tiled: tile (e, rb, kb) = rows [rb*128, +128) x bytes [kb*128, +128) of expert e,
// 16 KB contiguous (rows in order), tiles ordered e, then rb, then kb. This is the
// exact byte block one TMA load of a GEMM stage fetches.
struct TileGeom {
  int E;
  long long rows;       // rows of the source tensor per expert (I for gate/up, H for down)
  long long row_bytes;  // bytes of one stored row (K * element size)
  int rb_total;         // row blocks per expert in the destination (2I/128 or H/128)
  int rb_offset;        // first destination row block of this source (I/128 for up)
  long long expert_tiles;  // stored tiles per expert slot (0: rb_total * row_bytes / 128)
  const int* expert_mask;  // when set, only experts e with expert_mask[e] == mask_value
  int mask_value;
  // Row-major side (the source of a load, the destination of an un-tiling), possibly a
  // slice of a larger tensor: row r of expert e starts at byte
  // e * src_expert_stride + r * src_row_stride + src_offset. All three are multiples of 16.
  long long src_expert_stride, src_row_stride, src_offset;
};
// scales[e * stride] from the bf16 rows of g's row-major side (K = g.row_bytes elements).
cudaError_t launch_weight_amax(int f8, const __nv_bfloat16* w, const TileGeom& g, float* scales, int stride,
                               cudaStream_t s);
// bf16 source [E, rows, K] -> e4m3 codes in the tiled layout, per-expert scale scales[e*stride].
cudaError_t launch_weight_quant_tiled(int f8, const __nv_bfloat16* w, const TileGeom& g, const float* scales,
                                      int stride, uint8_t* dst, cudaStream_t s);
// row-major [E, rows, row_bytes] bytes -> tiled layout, and back.
cudaError_t launch_tile_weights(const void* src, const TileGeom& g, void* dst, cudaStream_t s);
cudaError_t launch_untile_weights(const void* src, const TileGeom& g, void* dst, cudaStream_t s);

// Read-only view of a layer handle's shape, weights and weight tensor maps, for
// entry points that live outside moe_api.cu.
struct LayerView {
  int E, k, H, I, device, num_sms;
  bool fp8, mixed, loaded;
  int f8;                  // FP8 code format (Fp8Format) when fp8
  const float* wscales;
  CUtensorMap tm_w13, tm_wd;
};

}  // namespace moe

struct moe_layer;
int moe_layer_view(const moe_layer* L, moe::LayerView* v);
// Read and clear the device error word of moe_forward_noalloc on device `dev` (the
// current device); *code = 0 when that path never ran there.
int moe_noalloc_take_error(int dev, int* code);
// 2-D tensor map [rows, inner] of bf16 (or e4m3 when fp8), 128-byte rows per box, box_rows rows.
int moe_encode_tile_map(CUtensorMap* m, const void* base, bool fp8, long long inner, long long rows, int box_rows);
