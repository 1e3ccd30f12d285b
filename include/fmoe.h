/*
 * fmoe.h -- C ABI of the quantised MoE expert forward for B200 (sm_100a).
 *
 * One token's pass through a mixture-of-experts layer whose expert weights
 * are group-affine 4-bit or 2-bit codes resident in HBM:
 *   route   logits = W_r xn, top-k experts (k of E), softmax over the k
 *           selected logits ("What is Flash-MoE?", section "Understanding
 *           Mixture-of-Experts": 4 routed experts of 512 plus 1 shared)
 *   expert  g = W_g xn, u = W_u xn, a = silu(g) u, y = W_d a for each selected
 *           expert and the shared expert; every weight is code * scale + bias
 *           with one bf16 scale/bias per 64 inputs ("What is Flash-MoE?",
 *           sections "2. FMA-optimised dequantisation kernels" and
 *           "3. Hand-tuned Metal compute shaders": 4-bit/2-bit matrix-vector
 *           multiply, fused SwiGLU)
 *   combine h' = h + sum_k p_k y_k + sigmoid(w_sg . xn) y_shared, then the
 *           two-pass RMSNorm xn' = h' (mean(h'^2) + eps)^(-1/2) w
 *           (same section: MoE combine + residual + sigmoid gating in one
 *           pass; two-pass RMSNorm; the result feeds the next layer).
 *
 * Conventions (all entry points):
 *   - Every call returns an int status (FMOE_OK == 0 on success).  Host-side
 *     validation happens before anything is launched; on a validation error
 *     nothing is launched and no output is touched.
 *   - Pointers named d_* or documented "device" are device memory of the
 *     current CUDA device; "host" pointers are ordinary host memory.  The
 *     caller owns every buffer; no entry point allocates device memory.
 *   - Device pointers must be 16-byte aligned.
 *   - Device-side work is enqueued on the caller's stream and is
 *     asynchronous: no entry point synchronises, except the host-memory
 *     packer (it waits for its own host-to-device copies), fmoe_read_status
 *     (it waits for the device) and the expert cache (it reads each step's
 *     routing on the host, and zeroes its table at creation).
 *   - Calls may come from several host threads.  A workspace, a trace, an
 *     expert cache and the no-allocation scratch of a device serve one call
 *     at a time (or calls ordered on one stream); fmoe_set_fused and
 *     fmoe_set_tensor_cores are process-wide switches.
 *   - Faults detected on the device (an expert id outside [0, E), a NaN
 *     router logit, an exhausted wait) set bits of a sticky per-device
 *     status word; kernels never trap.  Read and clear it with
 *     fmoe_read_status().
 *   - fp32 activations, row-major: a [T][H] array holds token t's hidden
 *     vector at offset t * H.
 */
#ifndef FMOE_H_
#define FMOE_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---------------------------------------------------------------- status -- */
#define FMOE_OK 0
#define FMOE_ERR_INVALID_ARG 1   /* null pointer, bad size, misaligned pointer */
#define FMOE_ERR_UNSUPPORTED 2   /* a shape or bit width the library does not run */
#define FMOE_ERR_CUDA 3          /* a CUDA runtime call failed */
#define FMOE_ERR_DEVICE_STATUS 4 /* the device status word is non-zero */
#define FMOE_ERR_BUFFER_TOO_SMALL 5

/* bits of the device status word */
#define FMOE_STATUS_BAD_EXPERT_ID 0x1u /* an id outside [0, E) was skipped */
#define FMOE_STATUS_NAN_LOGIT 0x2u     /* a router logit was NaN (ordered below every number) */
#define FMOE_STATUS_WAIT_TIMEOUT 0x4u  /* a bounded wait gave up; results are invalid */
#define FMOE_STATUS_BAD_PACK_INPUT 0x8u /* device packer: a code out of range or a scale that cannot be pre-scaled exactly */

/* Human-readable name of a status code (static string, never NULL). */
const char* fmoe_error_string(int status);

/* Reads the calling thread's current device's status word into *status
 * (host pointer) after synchronising the device; clears it when clear != 0.
 * Returns FMOE_OK or FMOE_ERR_CUDA. */
int fmoe_read_status(uint32_t* status, int clear);

/* ----------------------------------------------------------- the layer -- */
typedef struct fmoe_layer_desc {
  int hidden;      /* H: model width; a multiple of 64 with H/64 a power of two <= 32 or a multiple of 32 */
  int inter;       /* I: expert intermediate width; same rule as H */
  int n_experts;   /* E: routed experts, 1 .. 1024 */
  int top_k;       /* k: routed experts per token, 1 .. 8, k <= E */
  int bits;        /* code width of the routed experts: 4 or 2 */
  int shared_bits; /* code width of the shared expert: 4 or 2 */
  int group;       /* inputs per scale/bias group: must be 64 */
  float eps;       /* RMSNorm epsilon (inside the square root) */
} fmoe_layer_desc;

typedef struct fmoe_layer_weights {
  fmoe_layer_desc desc;
  const void* experts;        /* device: E packed expert records, each fmoe_packed_bytes(bits, 1, H, I, 64) bytes, back to back */
  const void* shared;         /* device: one packed record of the shared expert (shared_bits) */
  const float* w_router;      /* device fp32 [E][H] */
  const float* w_shared_gate; /* device fp32 [H]: the shared expert's output is scaled by sigmoid(w_shared_gate . xn) */
  const float* norm_w;        /* device fp32 [H]: RMSNorm weight */
} fmoe_layer_weights;

/* ------------------------------------------------------------- packing -- */
/* Logical expert layout (host input of the packer, output of the unpacker):
 *   q      uint8 [3 * H * I] per expert: gate [I][H], up [I][H], down [H][I],
 *          one code (0 .. 2^bits - 1) per byte, row-major;
 *   scale, bias  uint16 bf16 bit patterns [3 * H * I / 64] per expert, one per
 *          64 consecutive inputs of a row, same matrix order, row-major.
 *   The weight of row r, input j is q * scale + bias of group j / 64.
 * Experts follow one another: expert e starts at q + e * 3 * H * I, and at
 * scale/bias + e * 3 * H * I / 64.
 *
 * Packed record (one per expert; all sections 16-byte aligned):
 *   [gate/up codes][down codes][gate/up scale-bias][down scale-bias]
 *   gate/up: I row pairs, gate row n then up row n, row by row.  A row of K
 *   inputs is split into segments of min(32, K/64) groups; within a segment
 *   4-bit codes store first the low halves (inputs 0..31) of all its groups,
 *   16 bytes each, then the high halves; 2-bit codes store each group's 16
 *   bytes in order.
 *   down: column blocks of w = 8 (4-bit) or 16 (2-bit) consecutive inputs;
 *   block nb holds, for hidden rows 0 .. H-1 in order, one 32-bit word with
 *   the codes of inputs nb*w .. nb*w + w - 1 of that row (word (nb, r) at
 *   byte 4 * (nb * H + r) of the section).
 *   Inside every 32-bit word the 8 (or 16) codes of 8 (16) consecutive
 *   inputs are permuted so that masking the word with 0x0F0F0F0F /
 *   0xF0F0F0F0 (4-bit) or 0x03030303 .. 0xC0C0C0C0 (2-bit) yields byte lanes
 *   that pair with consecutive inputs (field 2a+b, resp. 4a+b, of the word
 *   holds input 4b+a).  Scale-bias: one 32-bit word per group, bf16
 *   scale * 2^-4 (4-bit) or * 2^-6 (2-bit) in the low half, bf16 bias in the
 *   high half; gate/up row-major (row pr, group g at pr * H/64 + g), down
 *   group-major (group g, row r at g * H + r).
 * Size per expert: 3 H I bits / 8 + 3 H I / 64 * 4 bytes (7,077,888 bytes =
 * 6.75 MiB at H = 4096, I = 1024, 4-bit; 3,932,160 bytes at 2-bit). */

/* Bytes of n_experts packed records.  Returns 0 for an unsupported shape. */
size_t fmoe_packed_bytes(int bits, int n_experts, int hidden, int inter, int group);

/* Packs n_experts logical experts (host arrays, layout above) into host
 * memory h_packed (h_bytes >= fmoe_packed_bytes(...)).  Pure host code.
 * Errors: FMOE_ERR_INVALID_ARG (null, code out of range, scale that cannot be
 * pre-scaled exactly), FMOE_ERR_UNSUPPORTED (shape), FMOE_ERR_BUFFER_TOO_SMALL. */
int fmoe_pack_experts_host(const uint8_t* q, const uint16_t* scale, const uint16_t* bias, int bits,
                           int n_experts, int hidden, int inter, int group, void* h_packed,
                           size_t h_bytes);

/* Inverse of fmoe_pack_experts_host (host to host), for round-trip checks. */
int fmoe_unpack_experts_host(const void* h_packed, int bits, int n_experts, int hidden, int inter,
                             int group, uint8_t* q, uint16_t* scale, uint16_t* bias);

/* Packs on the host and copies the records into device memory d_packed
 * (d_bytes >= fmoe_packed_bytes(...)) on `stream`; returns after the copy
 * has completed.  Not for the hot path (allocates a host staging buffer). */
int fmoe_pack_experts(const uint8_t* q, const uint16_t* scale, const uint16_t* bias, int bits,
                      int n_experts, int hidden, int inter, int group, void* d_packed,
                      size_t d_bytes, cudaStream_t stream);

/* As fmoe_pack_experts, with the logical arrays already in device memory
 * (d_q, d_scale, d_bias, same layout as the host arrays; 16-byte aligned).
 * Packs on `stream` without synchronising and without a host round trip.
 * Invalid codes or scales are reported through FMOE_STATUS_BAD_PACK_INPUT in
 * the device status word (the 16-byte code chunks or scale-bias words that
 * hold them are written as zero).
 * Errors: FMOE_ERR_INVALID_ARG, FMOE_ERR_UNSUPPORTED, FMOE_ERR_BUFFER_TOO_SMALL,
 * FMOE_ERR_CUDA. */
int fmoe_pack_experts_device(const uint8_t* d_q, const uint16_t* d_scale, const uint16_t* d_bias,
                             int bits, int n_experts, int hidden, int inter, int group,
                             void* d_packed, size_t d_bytes, cudaStream_t stream);

/* Stored-format quantiser ("What is Flash-MoE?", conclusion: the offline
 * conversion of trained weights into the 4-bit / 2-bit expert files): the
 * fp32 weights d_w [n_groups][group] (device, e.g. the logical expert
 * matrices above, row-major) become codes d_q [n_groups][group] (one per
 * byte) and bf16 bit patterns d_scale, d_bias [n_groups], the inputs of
 * fmoe_pack_experts_device.  Per group: lo = min (+0 for -0), hi = max,
 * scale = bf16(fp32 (hi - lo) / (2^bits - 1)), bias = bf16(lo) (round to
 * nearest even), q = rint((w - bias) / scale) in fp32 clamped to
 * [0, 2^bits - 1] (q = 0 for scale 0).  Finite inputs only; all pointers
 * 16-byte aligned; asynchronous on `stream`.
 * Errors: FMOE_ERR_INVALID_ARG (null or misaligned), FMOE_ERR_UNSUPPORTED
 * (group != 64 or bits not 2 / 4), FMOE_ERR_CUDA. */
int fmoe_quantize_groups(const float* d_w, size_t n_groups, int group, int bits, uint8_t* d_q,
                         uint16_t* d_scale, uint16_t* d_bias, cudaStream_t stream);

/* ------------------------------------------------ host expert tier -- */
/* Routed experts held in host memory with a device cache of records
 * ("What is Flash-MoE?", section "1. SSD expert streaming": experts fetched
 * per layer from a slower tier once routing has chosen them; here the tier
 * is host memory over PCIe and the cache is explicit, least recently used
 * first, shared by all layers).  Opaque handle; host-side state only. */
typedef struct fmoe_expert_cache fmoe_expert_cache;

/* Creates a cache for n_layers layers of descriptor d:
 *   h_layer_experts[l]  host: layer l's E packed routed records, back to back
 *                       (pinned memory keeps the record copies asynchronous);
 *   d_slots             device, caller-owned: n_slots records
 *                       (d_slots_bytes >= n_slots * record bytes);
 *   d_table             device, caller-owned: n_layers * E uint64 record
 *                       addresses (written by the cache);
 *   max_tokens          largest T of a step.
 * Allocates two small pinned host buffers (table mirror, one step's ids);
 * zeroes d_table synchronously.  Errors: FMOE_ERR_INVALID_ARG,
 * FMOE_ERR_UNSUPPORTED, FMOE_ERR_BUFFER_TOO_SMALL, FMOE_ERR_CUDA. */
int fmoe_cache_create(const fmoe_layer_desc* d, int n_layers, const void* const* h_layer_experts, int n_slots,
                      void* d_slots, size_t d_slots_bytes, uint64_t* d_table, int max_tokens,
                      fmoe_expert_cache** out);
int fmoe_cache_destroy(fmoe_expert_cache* c);

/* Counters since creation: expert-steps served from the slots (an expert
 * used by several tokens of one step counts once), records copied in, and
 * their bytes. */
int fmoe_cache_stats(const fmoe_expert_cache* c, uint64_t* hits, uint64_t* misses, uint64_t* bytes_in);

/* One layer step (layer index `layer`) for T tokens, as fmoe_layer_forward
 * (or fmoe_layer_forward_logits when d_logits is given) with the routed
 * records taken from the cache (lw->experts is not read): routing on the
 * device, the step's ids copied to the host and the stream synchronised,
 * every missing record copied into a slot (the least recently used one not
 * needed by this step), the layer's table row uploaded, then the expert
 * products and the combine.  Steps of one cache must be issued in order on
 * one stream.  Errors: as fmoe_layer_forward; FMOE_ERR_BUFFER_TOO_SMALL when
 * the slots cannot hold one step's distinct experts. */
int fmoe_cache_layer_forward(fmoe_expert_cache* c, int layer, const fmoe_layer_weights* lw, const float* d_logits,
                             float* d_h, float* d_xn, int T, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* ----------------------------------------------------------- workspace -- */
/* Device workspace for T tokens of a layer with descriptor d (bytes).  The
 * workspace holds intermediates (router partial sums, logits, ids, gate
 * weights, gamma, the SwiGLU outputs a and the expert outputs y) and a few
 * counters; it must be zeroed once with fmoe_workspace_init before first use
 * and is left re-usable by every call that completes. */
size_t fmoe_workspace_bytes(const fmoe_layer_desc* d, int T);

/* Zeroes a workspace (cudaMemsetAsync on `stream`). */
int fmoe_workspace_init(void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* Offsets (bytes from the workspace start) of the intermediates that
 * fmoe_layer_forward leaves behind: which = 0 logits fp32 [T][E],
 * 1 ids int32 [T][k], 2 gate weights fp32 [T][k], 3 gamma fp32 [T],
 * 4 a fp32 [T][k+1][I], 5 y fp32 [T][k+1][H].  Returns (size_t)-1 on error. */
size_t fmoe_workspace_offset(const fmoe_layer_desc* d, int T, int which);

/* --------------------------------------------------------- entry points -- */
#define FMOE_LOGITS_GIVEN 0x1u /* route: logits are an input, skip the router product */

/* Router product and top-k (section "Understanding Mixture-of-Experts").
 *   d_xn       device fp32 [T][H] normed inputs
 *   d_w_router device fp32 [E][H]
 *   d_logits   device fp32 [T][E]: output, or input when flags has FMOE_LOGITS_GIVEN
 *   d_ids      device int32 [T][k]: selected experts, largest logit first,
 *              ties to the lower index, NaN below every number
 *   d_weights  device fp32 [T][k]: softmax of the k selected logits
 *   d_ws       device workspace of at least fmoe_workspace_bytes(d, T) bytes
 *              for a descriptor with these H, E, k (only its router part is used)
 * Errors: FMOE_ERR_INVALID_ARG, FMOE_ERR_UNSUPPORTED (k > 8, E > 1024), FMOE_ERR_CUDA. */
int fmoe_route_topk(const float* d_xn, const float* d_w_router, int T, int H, int E, int k,
                    unsigned flags, float* d_logits, int32_t* d_ids, float* d_weights, void* d_ws,
                    size_t ws_bytes, cudaStream_t stream);

/* Expert forward for T tokens: for each token t, the k experts d_ids[t][*]
 * and the shared expert, on input d_xn[t]:
 *   d_y     device fp32 [T][k+1][H]: y of each selected expert in the order of
 *           d_ids, the shared expert last (not yet weighted)
 *   d_gamma device fp32 [T]: sigmoid(w_shared_gate . xn)
 * An id outside [0, E) contributes y = 0 and sets FMOE_STATUS_BAD_EXPERT_ID.
 * Errors: FMOE_ERR_INVALID_ARG, FMOE_ERR_UNSUPPORTED, FMOE_ERR_CUDA. */
int fmoe_expert_forward(const fmoe_layer_weights* lw, const float* d_xn, int T,
                        const int32_t* d_ids, int k, float* d_y, float* d_gamma, void* d_ws,
                        size_t ws_bytes, cudaStream_t stream);

/* Combine + residual + shared gate, then RMSNorm, for T tokens:
 *   h_out[t] = h[t] + sum_j weights[t][j] y[t][j] + gamma[t] y[t][k]
 *   xn_out[t] = h_out[t] * (mean(h_out[t]^2) + eps)^(-1/2) * norm_w
 * All device fp32; y [T][k+1][H].  h_out may be h itself (in place);
 * otherwise neither output may share a byte with y, h or the other output
 * (FMOE_ERR_INVALID_ARG).  Errors: FMOE_ERR_INVALID_ARG, FMOE_ERR_CUDA. */
int fmoe_combine_residual_rmsnorm(const float* d_y, const float* d_weights, const float* d_gamma,
                                  const float* d_h, const float* d_norm_w, float eps, int T, int k,
                                  int H, float* d_h_out, float* d_xn_out, cudaStream_t stream);

/* One whole layer for T tokens, in place: reads the residual d_h [T][H] and
 * the normed input d_xn [T][H], writes h' to d_h and xn' to d_xn.  All steps
 * run on the device with no host round trip; the call is safe to capture in
 * a CUDA graph.  The intermediates stay in the workspace (see
 * fmoe_workspace_offset).  d_h and d_xn must not overlap (the same buffer
 * for both would leave xn' where h' belongs): FMOE_ERR_INVALID_ARG when
 * their T x H rows share a byte.  Errors: FMOE_ERR_INVALID_ARG,
 * FMOE_ERR_UNSUPPORTED, FMOE_ERR_CUDA. */
int fmoe_layer_forward(const fmoe_layer_weights* lw, float* d_h, float* d_xn, int T, void* d_ws,
                       size_t ws_bytes, cudaStream_t stream);

/* fmoe_layer_forward for T tokens whose state lives in host memory, for a
 * caller that feeds tokens from the host (a decode loop in plain C):
 *   hx_in   host fp32 [2][T][H]: h rows, then the normed xn rows;
 *   hx_out  host fp32 [2][T][H]: receives h' rows, then xn' rows;
 *   d_hx    device fp32 [2][T][H] (caller-owned, 16-byte aligned) that the
 *           layer runs on in place.
 * One host-to-device copy, the layer, one device-to-host copy, all on
 * `stream` (with pinned host buffers nothing blocks; hx_out is valid once
 * the stream has reached the end of the call).  hx_in and hx_out may be the
 * same buffer.  Errors: as fmoe_layer_forward (checked before any copy). */
int fmoe_layer_forward_host(const fmoe_layer_weights* lw, const float* hx_in, float* hx_out, float* d_hx,
                            int T, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* As fmoe_layer_forward, routing on given router logits d_logits [T][E]
 * (device fp32) instead of the router product. */
int fmoe_layer_forward_logits(const fmoe_layer_weights* lw, const float* d_logits, float* d_h,
                              float* d_xn, int T, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* A stack of n_layers layers (host array of weight descriptors) for T
 * tokens, in place on d_h / d_xn: layer l + 1 reads what layer l wrote --
 * the layer chain of "What is Flash-MoE?" (a2a-mcp.org), section
 * "Understanding Mixture-of-Experts": every layer's output is the next
 * layer's input.  The same results, bit for bit, as n_layers calls of
 * fmoe_layer_forward.  Up to fmoe_fused_max_tokens(1) tokens with one
 * descriptor for all layers the whole stack runs as persistent kernels
 * (cooperative launch, one CTA per SM, two tokens and up to 32 layers per
 * launch), which leave the last layer's intermediates in the workspace
 * (see fmoe_stack_forward_trace for every layer's).  If a persistent kernel
 * reports FMOE_STATUS_WAIT_TIMEOUT, re-initialise the workspace.  Errors:
 * as fmoe_layer_forward (d_h and d_xn must not overlap). */
int fmoe_stack_forward(const fmoe_layer_weights* layers, int n_layers, float* d_h, float* d_xn,
                       int T, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* Sections of one layer's record in a stack trace. */
#define FMOE_TRACE_XN_IN 0   /* fp32 [T][H]: the layer's input xn */
#define FMOE_TRACE_LOGITS 1  /* fp32 [T][E]: router logits */
#define FMOE_TRACE_IDS 2     /* int32 [T][k]: selected experts, best first */
#define FMOE_TRACE_WEIGHTS 3 /* fp32 [T][k]: their gate weights */
#define FMOE_TRACE_GAMMA 4   /* fp32 [T]: shared-expert gate */
#define FMOE_TRACE_A 5       /* fp32 [T][k+1][I]: SwiGLU outputs, shared expert last */
#define FMOE_TRACE_H_OUT 6   /* fp32 [T][H]: the layer's output h' */

/* Bytes of a trace of n_layers layers for T tokens (0 on bad arguments). */
size_t fmoe_trace_bytes(const fmoe_layer_desc* d, int T, int n_layers);

/* Byte offset of section `which` (FMOE_TRACE_*) of layer `layer`'s record
 * in a trace ((size_t)-1 on bad arguments); records follow one another,
 * sections are 256-byte aligned. */
size_t fmoe_trace_offset(const fmoe_layer_desc* d, int T, int layer, int which);

/* fmoe_stack_forward that also records, for every layer, its input xn, the
 * router logits, the selected experts and gate weights, gamma, the SwiGLU
 * outputs and its output h' into d_trace (device, 16-byte aligned, at least
 * fmoe_trace_bytes(desc, T, n_layers) bytes, caller-owned): the values the
 * launches themselves computed, for checking every layer of a persistent
 * stack launch.  All layers must share one descriptor.  Errors: as
 * fmoe_stack_forward, FMOE_ERR_INVALID_ARG for a null or misaligned trace,
 * FMOE_ERR_BUFFER_TOO_SMALL when trace_bytes is short. */
int fmoe_stack_forward_trace(const fmoe_layer_weights* layers, int n_layers, float* d_h, float* d_xn, int T,
                             void* d_ws, size_t ws_bytes, void* d_trace, size_t trace_bytes, cudaStream_t stream);

/* fmoe_stack_forward for token state in host memory (the call a plain C
 * decode loop makes once per token): hx_in / hx_out host fp32 [2][T][H]
 * (h rows, then xn rows), d_hx device fp32 [2][T][H] that the stack runs on
 * in place.  One host-to-device copy, the n_layers layers, one
 * device-to-host copy, all on `stream`; hx_in and hx_out may be the same
 * buffer.  Every layer must have the same hidden size.  Errors: as
 * fmoe_stack_forward, checked before any copy, plus
 * FMOE_ERR_BUFFER_TOO_SMALL when ws_bytes is below any layer's
 * fmoe_workspace_bytes(desc, T). */
int fmoe_stack_forward_host(const fmoe_layer_weights* layers, int n_layers, const float* hx_in, float* hx_out,
                            float* d_hx, int T, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* Chooses the implementation of the T = 1 path (and of the few-token calls
 * that run through the persistent kernel, see fmoe_fused_max_tokens): enable != 0 (the
 * default) uses the persistent fused kernel wherever its shared-memory plan
 * fits, 0 the one-kernel-per-step path.  Both compute the same layer;
 * process-wide setting, returns the previous value. */
int fmoe_set_fused(int enable);

/* Chooses the expert products of the T > 1 path for experts that receive at
 * least fmoe_tc_min_tokens() tokens in a step (and the shared expert when T
 * reaches it): enable != 0 (the default) runs them as tcgen05 tensor-core
 * matrix products on dequantised fp16 weights (inputs kept to ~22 bits as an
 * fp16 hi / lo pair), 0 as the integer-dot matrix-vector path in batches of
 * 16 tokens.  Both compute the same products within the tolerance;
 * process-wide setting, returns the previous value. */
int fmoe_set_tensor_cores(int enable);

/* Largest token count T for which fmoe_layer_forward (stack == 0) or
 * fmoe_stack_forward (stack != 0) runs the tokens through the persistent
 * kernel (when enabled, fmoe_set_fused): 4 and 8.  Tokens go two per launch
 * where the kernel has a two-token form for the code widths (4-bit routed
 * and shared experts; an odd last token, and other widths, one per launch):
 * a pair shares the router rows, the shared expert's weights and the
 * exchanges between CTAs (section "Understanding Mixture-of-Experts" of
 * "What is Flash-MoE?": the shared expert serves every token).  A token's
 * result in a pair does not depend on the other token of the pair (the work
 * is split over the CTAs by position in the pair, not by value) but is
 * rounded differently from a one-token launch.  Such calls leave, like
 * T = 1, no per-expert outputs y in the workspace; larger T take the grouped
 * path. */
int fmoe_fused_max_tokens(int stack);

/* Tokens an expert needs in a step for its products to run on the tensor
 * cores (when enabled): 3.  With the 24-bit activations of the integer-dot
 * path (two dot products per code lane), from three tokens per expert that
 * path is bound by its dot products rather than by the expert's weight
 * bytes, and the tensor-core products are faster (measured on the 64-token
 * Zipf-routed step: 0.446 against 0.490 ms at a threshold of 5). */
int fmoe_tc_min_tokens(void);

/* 1 if the persistent kernel runs layers of descriptor d at T = 1 on the
 * current device (shape and shared-memory plan fit), else 0 (also on any
 * error).  The persistent kernel leaves the gate/up outputs a in the
 * workspace but not the per-expert down outputs y: it sums them on the fly. */
int fmoe_fused_supported(const fmoe_layer_desc* d);

/* ------------------------------------------- without caller workspace -- */
/* fmoe_layer_forward for callers that cannot hand over a workspace.  The
 * Flash-MoE pages have no counterpart to this call: it exists for hosts that
 * must not reserve device memory on the path -- an engine whose device pool
 * already owns all free memory, a latency-critical loop in which an
 * allocation (with the device-wide synchronisation cudaMalloc/cudaFree can
 * imply) is not acceptable, or a plain C program with no tensor library to
 * manage a workspace.  It computes exactly what fmoe_layer_forward computes,
 * through the same kernels, and allocates nothing: its workspace is a 12 MiB
 * array in the library's device memory, one per device, set aside when the
 * library's module is loaded on that device.
 *   lw, d_h, d_xn, T, stream  as for fmoe_layer_forward.
 * Limit: fmoe_workspace_bytes(&lw->desc, T) must not exceed 12 MiB
 * (12582912 bytes), which admits up to T = 13 tokens at hidden 4096 /
 * inter 1024 / 512 experts / top-4 (from T = 3 the workspace holds the
 * tensor-core inputs, about 100 KB per token); a larger request returns
 * FMOE_ERR_BUFFER_TOO_SMALL before anything is launched.
 * First call on each device: it looks up the array's device address and
 * enqueues, on `stream`, a zeroing of the counter words at the array's start
 * (the grid-barrier and publication counters of the persistent kernel); every
 * completed call leaves them at zero again.  Make this first call on each
 * device before any stream capture begins.
 * One array per device: calls that can overlap on the device (different
 * streams, or different host threads, without ordering between them) race on
 * it and corrupt each other's results; order them, e.g. on one stream.  The
 * intermediates are not exposed.  If the device status reports
 * FMOE_STATUS_WAIT_TIMEOUT, the counters may be left non-zero and this entry
 * point must not be used again on that device in this process.
 * Errors: as fmoe_layer_forward, plus FMOE_ERR_BUFFER_TOO_SMALL above the
 * limit and FMOE_ERR_UNSUPPORTED for a device ordinal of 64 or more. */
int fmoe_layer_forward_noalloc(const fmoe_layer_weights* lw, float* d_h, float* d_xn, int T,
                               cudaStream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* FMOE_H_ */
