/*
 * moe_b200.h -- C ABI of the routed Mixture-of-Experts layer on one NVIDIA
 * B200 (sm_100a): the forward, and the backward of the bf16 layer
 * (moe_backward, at the end).
 *
 * The layer (TransformerEngine PR "DeepSeekV3Layer: full MoE transformer
 * layer", Description, DeepSeekV3MoE bullet): a sigmoid router with an
 * aux-loss-free bias and grouped top-k selection, tokens permuted into
 * expert-major order, per-expert fc1 -> SwiGLU -> fc2 as a grouped GEMM, and a
 * gate-weighted combine back to token order, with an optional shared expert.
 * Block-scaled variants: MXFP8 (same PR, Performance, MXFP8 rows) and NVFP4
 * W4A4 (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support", Modifications).
 *
 * Conventions for every call:
 *   - All pointer arguments are DEVICE pointers unless stated otherwise.  The
 *     caller allocates every buffer; no call allocates or frees memory.
 *   - Every call is asynchronous on `stream` (a cudaStream_t passed as void*;
 *     NULL is the legacy default stream) and never synchronizes the host,
 *     except moe_get_device_status.
 *   - Matrices are row-major.  "bf16" is IEEE bfloat16 stored as uint16.
 *   - Arguments are validated on the host before any launch; a bad argument
 *     returns an error code and launches nothing.  Errors found on the device
 *     (an expert index out of range, a wait that timed out) are written to a
 *     status word at the start of the workspace and read back with
 *     moe_get_device_status.  No kernel traps.
 *   - No C++ exception crosses this interface.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1,  /* null pointer, non-positive size, bad enum       */
  MOE_ERR_UNSUPPORTED = 2,  /* shape the kernels do not handle (see moe_config) */
  MOE_ERR_WORKSPACE = 3,    /* workspace smaller than the size query returned  */
  MOE_ERR_CAPACITY = 4,     /* device: expert index out of [0, E)             */
  MOE_ERR_TIMEOUT = 5,      /* device: a bounded wait gave up                  */
  MOE_ERR_CUDA = 6          /* a CUDA runtime/driver call failed              */
} moe_status;

typedef enum { MOE_BF16 = 0, MOE_MXFP8 = 1, MOE_NVFP4 = 2 } moe_dtype;

/*
 * Layer shape.  T tokens of hidden size H; E routed experts of intermediate
 * size I, in n_group contiguous groups of E/n_group; each token keeps the
 * topk_group best groups and the top_k best experts inside them; gates are
 * normalised and multiplied by routed_scaling_factor.  I_shared > 0 adds a
 * shared expert of intermediate size I_shared applied to every token with
 * weight 1.  Each expert's segment of the expert-major layout is padded to a
 * multiple of pad_multiple rows.
 *
 * Supported: 1 <= T; H, I, I_shared multiples of 128; 1 <= E <= 1024;
 * E % n_group == 0 with E/n_group >= 2 and n_group <= 32; 1 <= topk_group <=
 * n_group; 1 <= top_k <= min(32, topk_group*E/n_group); pad_multiple >= 1
 * (MXFP8, NVFP4: pad_multiple % 64 == 0; NVFP4 also needs H, I, I_shared
 * multiples of 256).
 */
typedef struct moe_config {
  int32_t T, H, I, E;
  int32_t n_group, topk_group, top_k;
  int32_t I_shared;
  float routed_scaling_factor;
  int32_t dtype;          /* moe_dtype */
  int32_t pad_multiple;
} moe_config;

/*
 * Expert weights as the grouped GEMM consumes them, written by
 * moe_prepare_weights (the caller allocates the buffers, sizes from
 * moe_prepared_weights_size).
 *   bf16, tile-major: a matrix of R rows and K columns (R % 128 == 0,
 *   K % 64 == 0) is stored as 128 x 64 tiles of 16 KB, tile (r/128, k/64) at
 *   index (r/128)*(K/64) + k/64, row-major inside the tile; element (r, k)
 *   sits at bf16 offset ((r/128)*(K/64) + k/64)*8192 + (r%128)*64 + k%64.
 *   w1, w3 hold [E*I rows, H columns] (expert e = rows e*I ..), w2 holds
 *   [E*H rows, I columns]; ws1, ws3 [I_shared, H]; ws2 [H, I_shared].
 *   MXFP8: the same tile-major layout over bytes (128 rows x 128 e4m3 codes
 *   per 16 KB tile), and *_scales hold the e8m0 scales per 32 K elements in
 *   the MMA scale layout of moe_quantize over the same rows (w1_scales for
 *   the E*I rows of w1, ...).
 *   NVFP4: the same tile-major byte layout over packed e2m1 codes (a 16 KB
 *   tile holds 128 rows x 256 elements), *_scales the e4m3 scales per 16 K
 *   elements in the MMA scale layout, and the fp32 global encode scales:
 *   w13_global [E] (W1_e and W3_e share one, as one stacked fc1 tensor),
 *   w2_global [E], ws13_global [1], ws2_global [1].  Unused otherwise.
 * Shared-expert fields are ignored when I_shared == 0.
 */
typedef struct moe_weights {
  void* w1; void* w3; void* w2;
  void* w1_scales; void* w3_scales; void* w2_scales;
  float* w13_global; float* w2_global;
  void* ws1; void* ws3; void* ws2;
  void* ws1_scales; void* ws3_scales; void* ws2_scales;
  float* ws13_global; float* ws2_global;
} moe_weights;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(moe_status s);

/*
 * Sizes.  *bytes = scratch the step calls (moe_route .. moe_combine) need in
 * `workspace`; *r_cap = rows of the expert-major buffers (row_token, the
 * permuted rows, the grouped-GEMM outputs): T*top_k + E*(pad_multiple-1)
 * rounded up to pad_multiple.  Either output pointer may be NULL.
 * A workspace holds per-call state (h, the grouped MLP's tile and chunk
 * counters, the status word): calls whose kernels may overlap on the GPU
 * (different streams) need workspaces of their own; calls in one stream may
 * share one.  Only its first 4 bytes, the status word, must be zero before
 * the first call (a call never clears it; moe_get_device_status does).
 */
moe_status moe_workspace_size(const moe_config* cfg, size_t* bytes, int32_t* r_cap);

/* Bytes of each prepared weight buffer (scale buffers are 0 for bf16). */
typedef struct moe_weight_sizes {
  size_t w13, w2, ws13, ws2;                       /* codes (w1 and w3 each w13) */
  size_t w13_scales, w2_scales, ws13_scales, ws2_scales;
  size_t w_globals, ws_globals;   /* NVFP4: w13_global and w2_global each; shared */
} moe_weight_sizes;

moe_status moe_prepared_weights_size(const moe_config* cfg, moe_weight_sizes* sizes);

/*
 * Block-scaled quantization of a row-major bf16 matrix in [rows, cols]
 * (TransformerEngine PR "DeepSeekV3Layer", Performance, "MXFP8 quantization":
 * group_quantize_mxfp8 / quantize_mxfp8_kernel_cast_only).
 *   dtype MOE_MXFP8: codes [rows, cols] e4m3 (round to nearest even,
 *   saturating at +-448), one e8m0 scale per 32 consecutive elements of a row:
 *   2^(floor(log2 amax) - 8), biased exponent clamped to [0, 254], 127 for an
 *   all-zero block.  cols % 128 == 0.
 *   Scale layout ("MMA scale layout"): for a matrix with KB = cols/32 blocks
 *   per row, the scale of (row r, block kb) is at byte
 *     ((r/128)*(KB/4) + kb/4)*512 + (r%32)*16 + ((r%128)/32)*4 + kb%4,
 *   so `scales` holds ceil(rows/128)*128*KB bytes.  global_scale unused.
 *   dtype MOE_NVFP4 (sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE support",
 *   Modifications: W4A4 NVFP4): *global_scale (device fp32, written) =
 *   2688 / amax over the whole matrix (1 when amax == 0); per 16 consecutive
 *   elements of a row, the e4m3 block scale sb = e4m3((amax16 / 6) * g) and
 *   codes e2m1(v * (g / sb)) (each step one fp32 operation, nearest-even,
 *   saturating; a zero sb gives zero codes).  codes [rows, cols/2] bytes, two
 *   e2m1 codes per byte, element 2i in the low nibble; scales in the MMA scale
 *   layout with KB = cols/16.  cols % 256 == 0.
 */
moe_status moe_quantize(int32_t dtype, const void* in, int32_t rows, int32_t cols, void* codes,
                        void* scales, float* global_scale, void* stream);

/*
 * Weight preparation (the static re-layout of expert weights for the grouped
 * GEMM kernels; the pages' counterpart is the kernel-specific weight
 * reordering and shuffling of sglang PR "Mistral Large 3 NVFP4 TRTLLM MoE
 * support", Gemini summary, "Optimized Weight Handling").
 *   which == 0: routed experts e_begin .. e_begin+e_count-1; w1, w3 point at
 *               their row-major bf16 [e_count, I, H] and w2 at [e_count, H, I];
 *               written into dst->w1/w3/w2 at those experts' place.
 *   which == 1: the shared expert (e_begin 0, e_count 1); w1, w3 [I_shared, H],
 *               w2 [H, I_shared] -> dst->ws1/ws3/ws2.
 * Can be called per expert range so a large layer never needs all its source
 * weights resident at once.  Source and destination must not overlap.
 */
moe_status moe_prepare_weights(const moe_config* cfg, int32_t which, int32_t e_begin,
                               int32_t e_count, const void* w1, const void* w3, const void* w2,
                               const moe_weights* dst, void* stream);

/*
 * Router (DeepSeekV3MoE bullet: "fused sigmoid router with aux-loss-free bias
 * and grouped top-k").
 *   x [T, H] bf16, w_router [E, H] bf16, bias [E] fp32.
 *   logits_in  [T, E] fp32 or NULL.  When given, the router GEMM is skipped
 *              and selection runs on these logits.
 *   logits_out [T, E] fp32: x . W_r^T with fp32 accumulation; required when
 *              logits_in is NULL, ignored otherwise.
 *   topk_idx [T, top_k] int32: selected experts, biased score descending,
 *              ties to the lower index.  topk_w [T, top_k] fp32: gates
 *              sigmoid(logit) / sum * routed_scaling_factor.
 */
moe_status moe_route(const moe_config* cfg, const void* x, const void* w_router,
                     const float* bias, const float* logits_in, float* logits_out,
                     int32_t* topk_idx, float* topk_w, void* workspace,
                     size_t workspace_bytes, void* stream);

/*
 * Permute into padded expert-major order (Performance, "NCCL EP local
 * permute": staging buffer to expert-major layout, zero-filled padding).
 *   topk_idx [T, top_k] int32 (values outside [0, E) set MOE_ERR_CAPACITY on
 *   the device and are skipped).
 *   counts [E] int32: rows per expert.  offsets [E+1] int32: exclusive scan of
 *   counts rounded up to pad_multiple.  row_token [r_cap] int32: token of each
 *   row, -1 for pad rows and rows past offsets[E].  token_row [T*top_k] int32:
 *   row of (t, j).  Within a segment tokens ascend.
 *   src_rows: bf16 x [T, H] (BF16) or codes from moe_quantize (MXFP8 e4m3
 *   [T, H], NVFP4 packed e2m1 [T, H/2]).  dst_rows [r_cap, same row bytes];
 *   pad rows zero.  dst_rows may be NULL: no row is copied (moe_grouped_mlp
 *   can gather the rows itself) and src_rows is then not read.
 *   src_scales / dst_scales (MXFP8, NVFP4): block scales in the MMA scale
 *   layout of moe_quantize, for T and r_cap rows; pad rows get zero scale
 *   bytes.  NULL for BF16.
 */
moe_status moe_permute(const moe_config* cfg, const int32_t* topk_idx,
                       const void* src_rows, const void* src_scales,
                       int32_t* counts, int32_t* offsets, int32_t* row_token,
                       int32_t* token_row, void* dst_rows, void* dst_scales,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * moe_permute without a workspace, for bf16 layers.  The pages have no
 * counterpart to this call; it exists for callers that cannot allocate device
 * memory: code that runs under an engine or framework that owns every device
 * allocation (a plugin handed only its input and output buffers), and code
 * that must not call cudaMalloc because cudaMalloc can synchronize the device.
 *
 * Arguments and results are those of moe_permute for a MOE_BF16 config, with
 * these differences:
 *   - dtype must be MOE_BF16 (MOE_ERR_UNSUPPORTED otherwise): the call gathers
 *     bf16 rows only;
 *   - dst_rows and src_rows are required (MOE_ERR_INVALID_ARG when NULL);
 *   - src_scales and dst_scales must be NULL (MOE_ERR_INVALID_ARG otherwise);
 *   - there is no workspace and no status word: an expert index outside
 *     [0, E) is dropped (its token_row is -1), as in moe_permute, but is not
 *     reported.
 * The histogram scratch is a fixed 1 MiB int32 array compiled into the
 * library (static __device__ storage, held on every GPU that loads the
 * library until the process exits), so ceil(T*top_k/256) * E must be at most
 * 262144; larger shapes return MOE_ERR_WORKSPACE with a message on stderr and
 * launch nothing.  The call allocates and frees nothing.
 *
 *   - The first call in each CUDA context (per device, and again after a
 *     device reset) looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture on the device.
 *   - Every call on a device shares the one array.  Nothing in it needs to
 *     start at zero (each call writes every entry before reading it), but
 *     calls whose kernels overlap on the GPU -- on different streams, or from
 *     different host threads -- race on it and give wrong results.
 */
moe_status moe_permute_noalloc(const moe_config* cfg, const int32_t* topk_idx,
                               const void* src_rows, const void* src_scales,
                               int32_t* counts, int32_t* offsets, int32_t* row_token,
                               int32_t* token_row, void* dst_rows, void* dst_scales,
                               void* stream);

/*
 * Grouped expert MLP (DeepSeekV3MoE bullet: GroupedLinear -> ScaledSwiGLU ->
 * GroupedLinear): for every expert e and its rows X_e,
 *   h = bf16(silu(X_e W1_e^T) * (X_e W3_e^T));  out = bf16(h W2_e^T),
 * and the same for the shared expert on all T tokens of x.
 *   rows [r_cap, H] (as moe_permute's dst_rows), counts/offsets from
 *   moe_permute; x [T, H] in token order (shared expert input).
 *   rows may be NULL: fc1 then reads each expert's rows straight from x,
 *   picking them by row_token [r_cap] (moe_permute's map) with 4-row TMA
 *   gathers, so no expert-major copy of x is needed (saves r_cap * H * 2
 *   bytes and the copy; on B200 the gathers stream rows more slowly than
 *   32-row boxes, so at large batch this mode is the slower one).  row_token
 *   is ignored when rows is given, and x may then be NULL if I_shared == 0.
 *   MXFP8 / NVFP4: rows and x are codes from moe_quantize, row_scales /
 *   x_scales their scales (MMA scale layout; row_scales as moe_permute's
 *   dst_scales), and h is rounded to bf16 and quantized to the same format
 *   before fc2.  NVFP4: x_global is x's global encode scale from
 *   moe_quantize; h gets one global scale per expert (and one for the shared
 *   expert) from the amax of that expert's h rows, computed on the device.
 *   out_rows [r_cap, H] bf16: fc2 output per row (rows of pads untouched).
 *   shared_out [T, H] bf16 or NULL when I_shared == 0.
 * Tensor-core kernels: tcgen05 MMA with TMEM accumulators fed by TMA.
 */
moe_status moe_grouped_mlp(const moe_config* cfg, const moe_weights* w,
                           const void* rows, const void* row_scales,
                           const void* x, const void* x_scales, const float* x_global,
                           const int32_t* counts, const int32_t* offsets,
                           const int32_t* row_token, void* out_rows, void* shared_out,
                           void* workspace, size_t workspace_bytes, void* stream);

/*
 * Combine (gate-weighted scatter-add, written as a per-token gather-reduce):
 *   y[t] = bf16( sum_{j<top_k} topk_w[t,j] * out_rows[token_row[t*top_k+j]]
 *                + shared_out[t] ), fp32 accumulation in j order.
 *   shared_out may be NULL.  y [T, H] bf16.
 */
moe_status moe_combine(const moe_config* cfg, const void* out_rows,
                       const int32_t* token_row, const float* topk_w,
                       const void* shared_out, void* y, void* stream);

/*
 * Whole layer: route -> (quantize) -> permute -> grouped MLP -> combine, with
 * every intermediate in `workspace` (size from moe_forward_workspace_size).
 * If xy_on_host != 0, x and y are HOST pointers (pinned memory recommended):
 * x is copied to the device and y back, on `stream`, inside the call.
 */
moe_status moe_forward_workspace_size(const moe_config* cfg, size_t* bytes);
moe_status moe_forward(const moe_config* cfg, const moe_weights* w,
                       const void* w_router, const float* bias,
                       const void* x, void* y, int32_t xy_on_host,
                       void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward of the bf16 layer: the gradients of a loss L with respect to the
 * layer's input, router and weights, given dy = dL/dy (TransformerEngine PR
 * "DeepSeekV3Layer", Performance, "fused grouped MLP" row: the dGLU backward,
 * the dgrad and wgrad grouped GEMMs, and the router's gradient).  With
 * y[t] = sum_j w[t,j] O[row(t,j)] + shared(x[t]), w the gates of moe_route
 * and O = h W2_e^T, h = silu(a) u, a = X W1_e^T, u = X W3_e^T:
 *   dO[row(t,j)] = w[t,j] dy[t];   dgate[t,j] = <dy[t], O[row(t,j)]>;
 *   dh = dO W2_e;  da = dh u silu'(a);  du = dh silu(a),
 *     silu'(a) = s (1 + a (1 - s)), s = sigmoid(a);
 *   dX = da W1_e + du W3_e (per expert-major row), and the same for the shared
 *     expert on x with dO = dy;
 *   gates w_j = rsf s_j / S (s = sigmoid(logit), S = sum over the selected
 *     experts): dlogit_j = rsf (g_j / S - sum_i g_i s_i / S^2) s_j (1 - s_j)
 *     for selected experts, 0 elsewhere (the selection and the bias are
 *     piecewise constant and get no gradient), g = dgate;
 *   dx[t] = sum_j dX[row(t,j)] + dx_shared[t] + (dlogits W_r)[t];
 *   dW1_e = da^T X, dW3_e = du^T X, dW2_e = dO^T h over the expert's rows;
 *   dWs1 = da_s^T x, dWs3 = du_s^T x, dWs2 = dy^T h_s;  dW_r = dlogits^T x.
 * The bf16 roundings of the forward (h, O) are read as the identity.  a, u
 * and h are recomputed from the saved rows (bf16), the intermediate gradients
 * are stored as bf16 (dO, dh, da, du, dX, and the bf16 copy of dlogits the
 * dx and dW_r contractions read), every contraction accumulates in fp32.
 * Only dtype MOE_BF16 (MOE_ERR_UNSUPPORTED otherwise).
 *
 * Transposed weight copies the dgrad contractions read, tile-major as in
 * moe_weights (element (r, k) of an R x K matrix at bf16 offset
 * ((r/128)*(K/64) + k/64)*8192 + (r%128)*64 + k%64):
 *   w2t  [E*I rows, H]: rows e*I + i hold W2_e[:, i];
 *   w13t [E*H rows, 2I]: row e*H + h holds [W1_e[:, h] | W3_e[:, h]];
 *   ws2t [I_shared rows, H]: Ws2^T (unused when I_shared == 0);
 *   wdt  [H rows, Kd]: row h holds [Ws1[:, h] | Ws3[:, h] | W_r[:, h] | 0],
 *        Kd = 2 I_shared + E rounded up to a multiple of 64.
 * Sizes in bytes from moe_backward_weights_size; written by
 * moe_prepare_backward_weights from row-major bf16 sources:
 *   which == 0: routed experts e_begin .. e_begin+e_count-1, w1 and w3
 *               [e_count, I, H], w2 [e_count, H, I] (w_router unused);
 *   which == 1: the shared expert and the router (e_begin 0, e_count 1):
 *               w1, w3 [I_shared, H], w2 [H, I_shared] (NULL when
 *               I_shared == 0), w_router [E, H].
 */
typedef struct moe_bwd_weights {
  void* w2t; void* w13t; void* ws2t; void* wdt;
} moe_bwd_weights;

typedef struct moe_bwd_weight_sizes {
  size_t w2t, w13t, ws2t, wdt;
} moe_bwd_weight_sizes;

moe_status moe_backward_weights_size(const moe_config* cfg, moe_bwd_weight_sizes* sizes);
moe_status moe_prepare_backward_weights(const moe_config* cfg, int32_t which, int32_t e_begin,
                                        int32_t e_count, const void* w1, const void* w3,
                                        const void* w2, const void* w_router,
                                        const moe_bwd_weights* dst, void* stream);

/*
 * What the forward saved, as the step calls wrote it: x [T, H] bf16; rows
 * [r_cap, H] bf16 (moe_permute's dst_rows, pad rows zero); logits [T, E]
 * (moe_route's logits_out); topk_idx, topk_w (moe_route); counts, offsets,
 * row_token, token_row (moe_permute); out_rows [r_cap, H] bf16
 * (moe_grouped_mlp).
 */
typedef struct moe_fwd_saved {
  const void* x;
  const void* rows;
  const float* logits;
  const int32_t* topk_idx;
  const float* topk_w;
  const int32_t* counts;
  const int32_t* offsets;
  const int32_t* row_token;
  const int32_t* token_row;
  const void* out_rows;
} moe_fwd_saved;

/*
 * Weight gradients, fp32 row-major: dw1, dw3 [E, I, H]; dw2 [E, H, I]; dws1,
 * dws3 [I_shared, H]; dws2 [H, I_shared]; dw_router [E, H].  Any field may be
 * NULL: that gradient is not computed.  accumulate == 0: the gradients are
 * written; accumulate != 0: they are added to the values already there (each
 * element read, summed in fp32 and written by one thread, so repeated calls
 * give the same bits), e.g. to sum micro-batches.  The routed ones need
 * pad_multiple % 64 == 0 (MOE_ERR_UNSUPPORTED otherwise): each expert's rows
 * are read in 64-row steps and the segment pads supply the zeros past its
 * last row.
 */
typedef struct moe_weight_grads {
  float* dw1; float* dw3; float* dw2;
  float* dws1; float* dws3; float* dws2;
  float* dw_router;
  int32_t accumulate;
} moe_weight_grads;

/*
 * dy [T, H] bf16 -> dx [T, H] bf16; dlogits [T, E] fp32 and dgate [T, top_k]
 * fp32 (either may be NULL); dw (NULL: no weight gradient).  w: the forward's
 * prepared weights (their W1, W3 and, for the shared expert, Ws1 and Ws3 are
 * read for the recomputation of a and u); wb: moe_prepare_backward_weights's
 * copies.  workspace: moe_backward_workspace_size bytes, its first 4 bytes
 * (the status word) zero before the first call, as for moe_workspace_size.
 */
moe_status moe_backward_workspace_size(const moe_config* cfg, size_t* bytes);
moe_status moe_backward(const moe_config* cfg, const moe_weights* w, const moe_bwd_weights* wb,
                        const moe_fwd_saved* saved, const void* dy, void* dx, float* dlogits,
                        float* dgate, const moe_weight_grads* dw, void* workspace,
                        size_t workspace_bytes, void* stream);

/*
 * Reads (and clears) the device status word at the start of `workspace`.
 * Synchronizes `stream`.  *device_status receives a moe_status value.
 */
moe_status moe_get_device_status(void* workspace, int32_t* device_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
