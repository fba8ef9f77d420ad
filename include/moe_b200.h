/*
 * moe_b200.h - C ABI of the B200-native (sm_100a) fused Mixture-of-Experts layer.
 *
 * The layer, per token t of a batch of M tokens:
 *   1. route:   the k largest router logits pick k experts (equal logits go to the
 *               lower expert id); their softmax weights are renormalised to sum to 1
 *               ("a token usually activates only a selected subset" of the experts;
 *               toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200",
 *               section "Why MoE inference needs specialized kernels");
 *   2. align:   (token, slot) pairs are grouped by expert and padded to tile size
 *               ("routing tokens to experts, moving data", same section);
 *   3. gate_up: h = silu(W_gate[e] x_t) * (W_up[e] x_t), a grouped GEMM with the
 *               SwiGLU activation fused into its epilogue;
 *   4. down:    out_t = sum_j w_tj * (W_down[e_j] h_(t,j)), a grouped GEMM whose
 *               epilogue applies the routing weight and scatter-adds into token
 *               order ("fuses scaling, matrix multiplication, and expert aggregation
 *               into one GPU pass", aib.vote, "AWS SageMaker MoE kernel
 *               optimizations", third paragraph).
 * The FP8 variants store weights as 8-bit floats with one fp32 scale per expert
 * tensor and quantise x and h per tensor on the fly ("FP8 tensor-quantized fused
 * MoE", toolboxkart.tech page, section "2. FP8 backend routing changes which kernel
 * path runs"), in one of the two formats the kongchang.com page names ("MoE Kernel
 * Engineering Optimization Practices on Amazon SageMaker AI", section "Triton
 * Backend Routing: A Practical Path to FP8 Quantization"): E4M3 (4 exponent and 3
 * mantissa bits, largest finite 448) or E5M2 (5 and 2, largest finite 57344).
 *
 * The token count M is a runtime argument of every call: no kernel is compiled,
 * specialised or re-encoded per M ("Removing repeat compilation can reduce
 * first-token delay", toolboxkart.tech page, section 3).
 *
 * Conventions for every entry point:
 *   - Every call returns a moe_status; nothing aborts or throws across the ABI.
 *   - Tensor pointers are DEVICE pointers on the layer's device unless a parameter
 *     says "host"; they must be 16-byte aligned, contiguous and row-major.
 *   - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).
 *   - The caller keeps ownership of every pointer it passes; the library owns the
 *     handle, its weights and its workspace, and frees them in moe_destroy.
 *   - Calls on one handle must not run concurrently from several host threads.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef struct moe_layer moe_layer;   /* opaque handle */

typedef enum {
  MOE_DTYPE_BF16 = 0,       /* bf16 weights and activations, fp32 accumulation        */
  MOE_DTYPE_FP8_E4M3 = 1,   /* e4m3 weights (per expert-tensor scale), e4m3 activations
                               (per-tensor dynamic scale), fp32 accumulation           */
  MOE_DTYPE_FP8_E5M2 = 2,   /* the same with e5m2 codes for weights and activations    */
  MOE_DTYPE_MIXED_E4M3 = 3  /* a precision per expert, bf16 or e4m3: see
                               moe_load_weights_mixed                                  */
} moe_dtype;

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = -1,    /* bad size, null or misaligned pointer, bad dtype      */
  MOE_ERR_NOT_LOADED = -2,     /* forward before moe_load_weights                      */
  MOE_ERR_OOM = -3,            /* device allocation failed                             */
  MOE_ERR_CUDA = -4,           /* a CUDA runtime or driver call failed                 */
  MOE_ERR_UNSUPPORTED = -5,    /* device is not sm_100, or the shape is not supported  */
  MOE_ERR_DEVICE_TIMEOUT = -6  /* a kernel's bounded wait expired (see device error)   */
} moe_status;

/* Create a layer with E experts, top-k routing, hidden size H and expert
 * intermediate size I, on the current CUDA device.
 * Limits (checked): 1 <= E <= 512, 1 <= topk <= min(E, 16), H and I multiples of
 * 128 with 128 <= H, I <= 16384. On success *out receives the handle. */
MOE_API int moe_create(int E, int topk, int H, int I, int dtype, moe_layer** out);

/* Release the handle, its weights and its workspace. Synchronises the device. */
MOE_API int moe_destroy(moe_layer* layer);

/* Copy bf16 expert weights into library-owned memory (device pointers):
 *   w_gate [E, I, H], w_up [E, I, H], w_down [E, H, I], each row-major bf16.
 * For an FP8 layer the library quantises them: one fp32 scale per (expert, tensor)
 * s = amax|W| / F (F = 448 for e4m3, 57344 for e5m2; s = 1 for an all-zero tensor),
 * codes = fp8(W / s) with an IEEE fp32 division, round-to-nearest-even, saturating
 * to +-F.
 * Runs on `stream` and synchronises it before returning; the caller may free the
 * sources afterwards. Calling it again replaces the weights. */
MOE_API int moe_load_weights(moe_layer* layer, const void* w_gate, const void* w_up,
                     const void* w_down, void* stream);

/* Load a layer created with MOE_DTYPE_MIXED_E4M3, choosing the precision of each
 * expert: expert_fp8 [E] (host, one byte per expert) is nonzero for an expert kept as
 * e4m3 codes, zero for one kept in bf16. Experts differ in their numerical ranges,
 * and the kongchang.com page describes deciding per expert (or per computation stage)
 * which ones run in FP8 and which keep a higher precision ("MoE Kernel Engineering
 * Optimization Practices on Amazon SageMaker AI", section "Triton Backend Routing: A
 * Practical Path to FP8 Quantization"). Sources are the bf16 tensors of
 * moe_load_weights (device pointers). An FP8 expert takes the FP8 path of an e4m3
 * layer: one scale per (expert, tensor), e4m3 codes of x with s_x over all of x, and
 * of its h rows with s_h = max|h| / 448 over the valid h rows of the FP8 experts only;
 * a bf16 expert takes the bf16 path. Each grouped GEMM then runs as two launches, one
 * per precision. Synchronises `stream`. MOE_ERR_INVALID_ARG for another dtype;
 * moe_load_weights, moe_load_weights_fp8, moe_load_weights_shard reject a mixed layer,
 * moe_forward_noalloc returns MOE_ERR_UNSUPPORTED for it and moe_debug_weights too. */
MOE_API int moe_load_weights_mixed(moe_layer* layer, const void* w_gate, const void* w_up,
                                   const void* w_down, const unsigned char* expert_fp8, void* stream);

/* Tensor parallelism over the expert intermediate dimension: load shard `shard` of
 * `num_shards` of a layer whose full intermediate size is I_full = I * num_shards (the
 * handle was created with I = I_full / num_shards). The pages run the layer at
 * eight-way tensor parallelism (toolboxkart.tech, "AWS SageMaker MoE kernel
 * optimizations H200", section "3. Removing repeat compilation can reduce first-token
 * delay"). From the FULL bf16 tensors (device pointers)
 *   w_gate [E, I_full, H], w_up [E, I_full, H], w_down [E, H, I_full]
 * the handle keeps rows [shard*I, (shard+1)*I) of every W_gate[e] and W_up[e] and the
 * matching columns [shard*I, (shard+1)*I) of every W_down[e]. SwiGLU acts on each
 * intermediate feature alone and the down projection sums over them, so the layer's
 * output is the SUM of the shards' outputs (combined by an all-reduce across the
 * ranks that hold them). Routing depends only on the logits and is the same on every
 * shard. An FP8 handle quantises its own slice: one scale per (expert, tensor) of the
 * slice, and its own per-tensor scale of h over its slice of h.
 * Synchronises `stream`. Returns MOE_ERR_INVALID_ARG when I * num_shards != I_full or
 * the shard index is out of range. */
MOE_API int moe_load_weights_shard(moe_layer* layer, const void* w_gate, const void* w_up,
                                   const void* w_down, int I_full, int shard, int num_shards,
                                   void* stream);

/* Load already-quantised weights into an FP8 layer (device pointers):
 *   q_gate [E, I, H], q_up [E, I, H], q_down [E, H, I] (uint8 codes in the layer's
 *   format, e4m3 or e5m2) and
 *   scales [E, 3] fp32 (gate, up, down scale of each expert; host pointer).
 * Weight value = decode(code) * scale. Synchronises `stream`. */
MOE_API int moe_load_weights_fp8(moe_layer* layer, const void* q_gate, const void* q_up,
                         const void* q_down, const float* scales_host, void* stream);

/* Pre-size the workspace for batches of up to M_max tokens. moe_forward grows the
 * workspace itself when a batch is larger (synchronising the device to do so), so
 * call this once before capturing moe_forward into a CUDA graph. */
MOE_API int moe_reserve(moe_layer* layer, int M_max, void* stream);

/* The layer's forward pass, asynchronous on `stream`:
 *   x             [M, H] bf16 (device)
 *   router_logits [M, E] fp32 (device)
 *   out           [M, H] bf16 (device), overwritten
 * M = 0 is a no-op. No host-device synchronisation happens inside (unless the
 * workspace must grow). Calls on one handle must be stream-ordered: the handle's
 * workspace is shared by its calls. */
MOE_API int moe_forward(moe_layer* layer, const void* x, const float* router_logits, int M,
                void* out, void* stream);

/* Host-buffer convenience: copies x_host [M,H] bf16 and logits_host [M,E] fp32 to
 * the device, runs moe_forward and copies out [M,H] bf16 back to out_host, all on
 * `stream`, and synchronises it. With pinned host buffers the copies and the
 * forward are captured once per (M, buffer addresses) into a CUDA graph that later
 * calls replay (captured again after new weights, a larger workspace or a switch of
 * the decode path); pageable buffers are copied eagerly. */
MOE_API int moe_forward_host(moe_layer* layer, const void* x_host, const float* logits_host,
                     int M, void* out_host, void* stream);

/* The forward pass for callers that cannot allocate device memory. (The pages have no
 * counterpart to this entry point; it exists for how the library is deployed.)
 * moe_forward allocates its per-call scratch on first use and grows it with cudaMalloc
 * when a larger batch arrives. A caller whose runtime owns all of HBM and forbids later
 * allocations, or a caller that cannot afford the device-wide synchronisation of
 * cudaMalloc/cudaFree inside its serving loop, uses this entry point instead: same arguments and same result as moe_forward, but every byte of
 * per-call scratch comes from one fixed 32 MiB array in device memory that the library
 * defines statically. Nothing is allocated or freed by the call.
 *   - Limit: a batch whose scratch exceeds 32 MiB is rejected with MOE_ERR_INVALID_ARG and a
 *     message on stderr (for the bf16 layer E=128, top-8, H=2048, I=768 that is a batch of
 *     more than 307 tokens; for E=256, top-8, H=7168, I=2048, more than 7); use
 *     moe_forward for those. Every GPU that loads the library holds the 32 MiB until the
 *     process exits.
 *   - Set-up: the first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress, with that device current). Make that first call before any
 *     stream capture.
 *   - Sharing: all calls on a device, from every handle, use the same array and leave
 *     their data in it; each call clears the parts that must start at zero. Two calls
 *     whose work overlaps on the GPU (different streams, or different host threads) race
 *     on the array: keep them stream-ordered.
 *   - Kernel waits are bounded as in moe_forward. A wait that gives up records its code
 *     in an error word kept at the start of the array (per device, not per handle);
 *     moe_get_device_error on any handle of that device reads and clears it.
 *   - moe_debug_routing and moe_debug_activations describe the last moe_forward call
 *     only: this path leaves the handle's workspace (and its FP8 s_x / s_h record)
 *     untouched. */
MOE_API int moe_forward_noalloc(moe_layer* layer, const void* x, const float* router_logits, int M,
                                void* out, void* stream);

/* Inverse rotary position embedding fused with per-head FP8 quantisation, for any
 * number of tokens (a run-time argument: one precompiled kernel per head size, nothing
 * compiled or specialised per token count). The pages name this kernel,
 * _fused_inv_rope_fp8_quant_per_head, as the one that was recompiled for every new
 * token count until that specialisation was removed (toolboxkart.tech, "AWS SageMaker
 * MoE kernel optimizations H200", section "3. Removing repeat compilation can reduce
 * first-token delay"; aib.vote, "AWS SageMaker MoE kernel optimizations", fourth
 * paragraph). No layer handle is needed; it runs on the current device.
 *   x         [num_tokens, num_heads, head_dim] bf16 (device), rotated by RoPE
 *   positions [num_tokens] int32 (device): the position of each token
 *   cos_sin   [max_pos, head_dim] fp32 (device): row p holds cos of the head_dim/2
 *             angles of position p, then their sin
 *   codes     [num_tokens, num_heads, head_dim] uint8 (device), written: FP8 codes
 *   scales    [num_tokens, num_heads] fp32 (device), written: one scale per vector
 * Per (token, head) vector y = x rotated back: for each pair (a', b') with the
 * angle's c, s:  a = a'c + b's,  b = b'c - a's (each product, sum and difference
 * rounded to fp32 in that order); pairs are (i, i + head_dim/2) when interleaved = 0,
 * (2i, 2i + 1) when interleaved = 1. Then scale = max|y| / F (F = 448 for
 * fp8_format = MOE_DTYPE_FP8_E4M3, 57344 for MOE_DTYPE_FP8_E5M2; 1 when y is all
 * zero) and codes = RNE(y / scale) saturated, the division in IEEE fp32.
 * A position outside [0, max_pos) gives codes 0 and scale NaN for that token (no
 * out-of-bounds read). head_dim must be 64, 128 or 256; x, cos_sin and codes 16-byte
 * aligned. num_tokens = 0 is a no-op. Asynchronous on `stream`; the caller owns every
 * buffer. Returns MOE_ERR_INVALID_ARG for a bad size, format or pointer. */
MOE_API int moe_inv_rope_fp8_quant(const void* x, const int* positions, const float* cos_sin, int max_pos,
                                   int num_tokens, int num_heads, int head_dim, int interleaved,
                                   int fp8_format, void* codes, float* scales, void* stream);

/* Select the single-launch decode path for this handle (enable = 1) or the default
 * kernel chain (enable = 0). The single-launch path runs a whole bf16 forward of up
 * to 64 tokens (M*topk <= 512, E <= 512) in one cooperative persistent kernel that
 * routes, groups, gathers and runs both grouped GEMMs with device-side dependency
 * counters ("fused MoE kernels combine routing, data movement and expert
 * calculations into fewer GPU operations": toolboxkart.tech, "AWS SageMaker MoE
 * kernel optimizations H200", section "Why MoE inference needs specialized
 * kernels"). Other batches and FP8 layers keep the chain. Same results either way. */
MOE_API int moe_set_fused_decode(moe_layer* layer, int enable);

/* Largest batch (tokens) that this handle runs on the thin-batch path, or 0 to send
 * every batch to the tensor-core kernel chain; a negative value restores the default
 * (8 tokens, where the path measured faster than the chain; 0 for MOE_DTYPE_MIXED_E4M3;
 * the environment variable MOE_GEMV_MAX_M sets the default of new handles). At decode
 * sizes an expert receives one or two tokens, so each of its weight bytes feeds one or
 * two multiply-adds: the product is a matrix-vector product bound by streaming the
 * weights, and a small batch pays mostly for launches and synchronisation around that
 * streaming (routing, data movement and combining add work around the matrix products:
 * toolboxkart.tech, "AWS SageMaker MoE kernel optimizations H200", section "Why MoE
 * inference needs specialized kernels"). The thin-batch path runs route + plan, then
 * gate_up and down as streams of warp-level tensor-core products (mma.sync on bf16
 * values, or on the e4m3 / e5m2 codes themselves) fed by cp.async: three launches, no
 * split-K, `out` written by down. Results agree with the chain within the tolerances of
 * the layer. Serves 1 <= M <= 16 with k <= 16 when the batch's activations fit one
 * block's shared memory next to a 64 KB weight ring (x: (M+1) rows of H values; h: a
 * token's k rows of I values). MOE_ERR_INVALID_ARG for a null handle or a value above
 * 16. */
MOE_API int moe_set_gemv_max_tokens(moe_layer* layer, int max_tokens);

/* Text of a status code (static storage). */
MOE_API const char* moe_status_string(int status);

/* Synchronise the device and read (then clear) the handle's device error word, or,
 * when that is clear, the error word of moe_forward_noalloc on the handle's device:
 * *code = 0 when no kernel reported an error; otherwise a code whose low byte names
 * the wait that gave up (0x01 stage full, 0x02 stage empty, 0x03 accumulator full,
 * 0x04 accumulator empty, 0x06 activation dependency, 0x07 grid) or 0x05 (a tile
 * descriptor failed its bounds check). Bounded waits never spin forever.
 * Returns MOE_OK when *code is 0, MOE_ERR_DEVICE_TIMEOUT when a wait gave up,
 * MOE_ERR_CUDA for a failed bounds check or a failed CUDA call. */
MOE_API int moe_get_device_error(moe_layer* layer, int* code);

/* Number of kernels the last moe_forward launched (0 for M = 0). */
MOE_API int moe_last_launch_count(moe_layer* layer);

/* 1 when the last moe_forward ran its grouped GEMMs on CTA pairs (clusters of two
 * CTAs issuing M = 256 tcgen05 MMAs, each CTA loading half of every token tile),
 * else 0. No counterpart in the pages: an execution detail of this library, chosen
 * per forward (wide token tiles: at least 96 tokens per expert on average, H a
 * multiple of 512 and I of 256; MOE_PAIR_GEMM=0 / 1 in the environment forces it off /
 * on where the shapes allow). 0 for a null handle. */
MOE_API int moe_last_gemm_pairs(moe_layer* layer);

/* Per-kernel timing. While enabled, every moe_forward records a CUDA event
 * before and after each kernel it launches, on the forward's stream. Kernel
 * slots: 0 route, 1 align, 2 gather, 3 gate_up GEMM, 4 h quantise (FP8 only),
 * 5 down GEMM, 6 finalise (MOE_PROFILE_SLOTS in all). Enabling clears the totals.
 * Do not enable it while capturing moe_forward into a CUDA graph. */
#define MOE_PROFILE_SLOTS 7
MOE_API int moe_profile_enable(moe_layer* layer, int enable);

/* Synchronise the device, then write per slot the summed kernel time in ms
 * (ms_sum[MOE_PROFILE_SLOTS], host) and the number of timed launches
 * (launches[MOE_PROFILE_SLOTS], host) since profiling was enabled. */
MOE_API int moe_profile_read(moe_layer* layer, double* ms_sum, int* launches);

/* Test access: copy the routing of the last forward to caller device buffers
 * (any pointer may be NULL to skip it), after synchronising the device:
 *   topk_ids [M, k] int32, topk_w [M, k] fp32, counts [E] int32,
 *   padded_offsets [E+1] int32, padded_pairs [padded_offsets[E]] int32 (pad = M*k),
 *   scales_host [2] fp32: s_x and s_h of the last FP8 forward (1 for bf16 layers).
 * `tile_rows` (host, may be NULL) receives the pad tile (rows per expert group). */
MOE_API int moe_debug_routing(moe_layer* layer, int* topk_ids, float* topk_w, int* counts,
                      int* padded_offsets, int* padded_pairs, float* scales_host,
                      int* tile_rows);

/* Test access: copy the permuted activations of the last forward (device buffer of
 * padded_offsets[E] rows of H elements: bf16, or FP8 codes for FP8 layers), and
 * the intermediate h (rows of I bf16 values) when h_out is not NULL. */
MOE_API int moe_debug_activations(moe_layer* layer, void* x_perm_out, void* h_out);

/* Test access: copy the stored weights (device buffers): FP8 layers give their codes
 * q_gate/q_up [E,I,H], q_down [E,H,I] and scales_host [E,3]; bf16 layers give the
 * bf16 copies and leave scales_host untouched. Any pointer may be NULL. */
MOE_API int moe_debug_weights(moe_layer* layer, void* gate_out, void* up_out, void* down_out,
                      float* scales_host);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
