/*
 * moe_mxfp4.h -- C ABI of the B200 (sm_100a) MXFP4 expert-FFN MoE layer library.
 *
 * The layer is the gpt-oss-style mixture-of-experts expert block:
 *   route:   top-k of the router logits, then a softmax over those k values;
 *   permute: (token, slot) pairs grouped by expert;
 *   expert:  h = x . W_gu[e]^T + b_gu[e]  (fp32 accumulate), gate = h[2i],
 *            up = h[2i+1], a = (clamp(up, -limit, limit) + 1) * g * sigmoid(alpha g)
 *            with g = min(gate, limit);  y = a . W_d[e]^T + b_d[e];
 *   combine: out[t] = sum_j w[t,j] * y_j   (the bias sits inside the weight).
 * Expert weights are MXFP4: E2M1 codes packed two per byte (even element in the
 * low nibble) with one E8M0 scale byte per 32 consecutive elements of a row; the
 * NVFP4 variant (E4M3 scale per 16 elements plus an fp32 weight_scale_2 per
 * expert) has its own entry points, nvfp4_dequantize and moe_nvfp4_forward_ex.
 *
 * Sources, cited by page title and section:
 *   MoE-Infinity PR #152 "expert offloading Phase 2 -- MXFP4 dequant-on-copy
 *     execution", Changes: the mxfp4_dequantize op (golden rel-err 0.0) and a
 *     forward that keeps scales, bias, the [N, K//2] packed layout, the gate/up
 *     split, clamped SwiGLU and fp32 accumulation.
 *   FreeToken PR #838 "feat(gguf): serve gpt-oss gguf checkpoints on gpt_oss":
 *     review "NVFP4 down scale vs. down bias" (sum w*(s*y + b)); review
 *     "w2_bias with apply_router_weight_on_input" (biases must be absent when the
 *     router weight scales the input); "What it does" (alpha 1.702, limit 7,
 *     gate_up_bias [E, 2I], down_bias [E, H], bias before activation / before the
 *     routing weight).
 *   onnxruntime/mobius PR #719 "Add native GPT-OSS MXFP4 QMoE export", Summary and
 *     Validation: blocks [E, N, K/32, 16] (= [E, N, K/2]); E8M0 0x00..0xfe valid,
 *     0xff rejected.
 *   transformers PR #49431 "Restore GPT-OSS's router-masked expert-parallel plan":
 *     MXFP4 experts take routing data (ids + weights) rather than dispatched ids.
 *
 * Conventions for every call:
 *   - All tensor pointers are caller-owned DEVICE memory on the current CUDA
 *     device, contiguous row-major, never freed or retained by the library (the
 *     *_from_host calls take their packed bank in page-locked HOST memory instead).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  Work is
 *     enqueued on it; no call synchronises the host (except
 *     moe_get_device_error, documented below).
 *   - Return value: MOE_OK or a negative moe_status.  Argument checks happen on
 *     the host before anything is enqueued; on an argument error nothing runs and
 *     no output is touched.  No C++ exception crosses this boundary.
 *   - Problems only the device can see (an expert id outside [0, E), a 0xff
 *     scale byte) set a sticky per-device error word read by
 *     moe_get_device_error; the affected outputs are then unspecified (a 0xff
 *     scale yields NaN in dequantised values).
 */
#ifndef MOE_MXFP4_H
#define MOE_MXFP4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    MOE_OK = 0,
    MOE_ERR_INVALID_ARG = -1, /* null pointer, bad size, misalignment, bad flag mix */
    MOE_ERR_UNSUPPORTED = -2, /* valid but outside what the library implements     */
    MOE_ERR_CUDA = -3,        /* a CUDA runtime call or launch failed               */
    MOE_ERR_NO_MEMORY = -4,   /* workspace allocation failed or workspace too small */
    MOE_ERR_DEVICE = -5       /* the sticky device error word is set                */
} moe_status;

/* Device error bits reported by moe_get_device_error (ORed). */
#define MOE_DEVERR_BAD_EXPERT_ID 0x1 /* an id outside [0, E) reached the layer      */
#define MOE_DEVERR_BAD_SCALE 0x2     /* an E8M0 byte 0xff, or an E4M3 NaN byte
                                        (0x7f / 0xff), was decoded                  */
#define MOE_DEVERR_TIMEOUT 0x4       /* a bounded pipeline wait gave up              */
#define MOE_DEVERR_BAD_LOGIT 0x8     /* a token had fewer than k non-NaN router logits */
#define MOE_DEVERR_OUT_OF_BOUNDS 0x10 /* bounds-checked builds only: an index fell
                                        outside its buffer (the access was skipped) */

/* moe_mxfp4_forward_ex flags */
#define MOE_FLAG_WEIGHT_ON_INPUT 0x1u /* router weight scales each expert's input  */

/*
 * mxfp4_dequantize -- standalone dequant-on-copy of a packed MXFP4 bank to bf16
 * (MoE-Infinity PR #152, Changes: mxfp4_dequantize; golden rel-err 0.0).
 *   blocks  uint8  [E, N, K/2]  two E2M1 codes per byte, element 2m in the low
 *                                nibble of byte m, element 2m+1 in the high nibble
 *   scales  uint8  [E, N, K/32] E8M0 byte per 32 consecutive elements of a row
 *   out     bf16   [E, N, K]    out = E2M1(code) * 2^(scale - 127), exact (round
 *                                to nearest even only where the value is a bf16
 *                                subnormal or overflows: neither rounds in range);
 *                                scale 0xff gives NaN and sets MOE_DEVERR_BAD_SCALE
 * Sizes: E, N >= 1; K >= 32 and K % 32 == 0.  blocks and out must be 16-byte
 * aligned.  Errors: MOE_ERR_INVALID_ARG for null pointers, sizes or alignment.
 */
int mxfp4_dequantize(const uint8_t *blocks, const uint8_t *scales, uint16_t *out,
                     int64_t E, int64_t N, int64_t K, void *stream);

/*
 * mxfp4_dequantize_from_host / nvfp4_dequantize_from_host -- dequant-on-copy from host
 * memory (MoE-Infinity PR #152, Changes: fetched packed experts are dequantised on
 * copy).  As mxfp4_dequantize / nvfp4_dequantize, but host_blocks and host_scales are
 * page-locked HOST memory that the current device can address (cudaHostAlloc /
 * cudaMallocHost, or a cudaHostRegister'd range; mapped under unified addressing):
 * the decode kernel reads the packed codes over the host link through the device
 * mapping and writes bf16 straight into `out` (device memory), so 4.25 (MXFP4) or
 * 4.5 (NVFP4) bits per weight cross the link instead of 16.  scale2 (NVFP4) is device
 * memory or NULL.  Both host buffers must hold the whole bank; MOE_ERR_INVALID_ARG
 * when the first or last byte of either is not such host memory, or for the sizes
 * and alignment rules of the device-memory calls.  The host memory must stay
 * allocated and unmodified until the stream has run the call.
 */
int mxfp4_dequantize_from_host(const uint8_t *host_blocks, const uint8_t *host_scales, uint16_t *out,
                               int64_t E, int64_t N, int64_t K, void *stream);
int nvfp4_dequantize_from_host(const uint8_t *host_blocks, const uint8_t *host_scales,
                               const float *scale2, uint16_t *out, int64_t E, int64_t N, int64_t K,
                               void *stream);

/*
 * moe_route -- top-k routing (transformers PR #49431: the MXFP4 experts consume
 * routing ids and weights).  For each token t:
 *   ids[t, 0..k)     the k largest logits in decreasing order, ties to the lower
 *                    expert index;
 *   weights[t, j]    exp(l_j - l_max) / sum over the k chosen of exp(l_i - l_max).
 *   router_logits fp32 [T, E]; ids int32 [T, k]; weights fp32 [T, k].
 * Sizes: T >= 1, 1 <= E <= 256, 1 <= k <= min(E, 8).  NaN logits are never chosen:
 * a token with fewer than k non-NaN logits gets id -1 and weight 0 in its remaining
 * slots (the softmax runs over the chosen logits only) and MOE_DEVERR_BAD_LOGIT is
 * raised; the forward calls then drop those slots (and raise
 * MOE_DEVERR_BAD_EXPERT_ID).
 */
int moe_route(const float *router_logits, int64_t T, int64_t E, int k, int32_t *ids,
              float *weights, void *stream);

/*
 * moe_router_route -- the router linear layer fused with moe_route (FreeToken PR #838:
 * the gpt-oss router is the linear module mlp.router, with a bias):
 *   logits[t, e] = x[t] . w_router[e] + b_router[e]   (bf16 operands, fp32 accumulate
 *                                                       on the tensor cores)
 *   ids, weights  = moe_route of those fp32 logits (same selection rule and softmax)
 *   x         bf16 [T, H];  w_router bf16 [E, H];  b_router fp32 [E] or NULL (= zero)
 *   logits    fp32 [T, E] or NULL: when given, receives the logits the routing used
 *   ids int32 [T, k]; weights fp32 [T, k]
 * Sizes: T >= 1; H >= 64 and H % 64 == 0; 1 <= E <= 256; 1 <= k <= min(E, 8).  x and
 * w_router must be 16-byte aligned.  Errors: MOE_ERR_INVALID_ARG for null pointers,
 * sizes or alignment; MOE_ERR_UNSUPPORTED for E > 256.
 */
int moe_router_route(const uint16_t *x, const uint16_t *w_router, const float *b_router, int64_t T,
                     int64_t H, int64_t E, int k, float *logits, int32_t *ids, float *weights,
                     void *stream);

/*
 * moe_mxfp4_forward -- the expert layer, weights on the output
 * (FreeToken PR #838: sum w*(y + b); bias before the routing weight):
 *   x               bf16  [T, H]
 *   ids, weights    int32 / fp32 [T, k]  (e.g. from moe_route)
 *   gate_up_blocks  uint8 [E, 2I, H/2], gate_up_scales uint8 [E, 2I, H/32]
 *   gate_up_bias    fp32  [E, 2I] or NULL (= zero)
 *   down_blocks     uint8 [E, H, I/2],  down_scales uint8 [E, H, I/32]
 *   down_bias       fp32  [E, H]  or NULL (= zero)
 *   alpha, limit    clamped SwiGLU constants (gpt-oss: 1.702, 7.0)
 *   out             bf16  [T, H], must not alias any input
 * Gate/up rows are interleaved: row 2i of the gate_up bank is gate i, row 2i+1 is
 * up i.  Sizes: T, E >= 1; 1 <= k <= min(E, 8); H % 64 == 0; I % 64 == 0.
 * The workspace (moe_mxfp4_workspace_size bytes) is allocated and freed
 * stream-ordered from the device's default memory pool.
 */
int moe_mxfp4_forward(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                      const int32_t *ids, const float *weights,
                      const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                      const float *gate_up_bias, const uint8_t *down_blocks,
                      const uint8_t *down_scales, const float *down_bias, float alpha,
                      float limit, uint16_t *out, void *stream);

/*
 * moe_mxfp4_forward_ex -- as moe_mxfp4_forward, with flags and a caller workspace.
 *   flags            0 or MOE_FLAG_WEIGHT_ON_INPUT.  With the router weight on the
 *                    input each expert sees bf16(w[t,j] * x[t]) and the outputs
 *                    are summed unweighted; both biases must then be NULL
 *                    (FreeToken PR #838 review: per-expert biases need the router
 *                    weight on the output) or MOE_ERR_INVALID_ARG is returned.
 *   workspace        device memory of at least workspace_bytes, 256-byte aligned,
 *                    or NULL to let the call allocate it stream-ordered.
 *   workspace_bytes  >= moe_mxfp4_workspace_size(T, H, I, E, k) when workspace is
 *                    given, else MOE_ERR_NO_MEMORY.
 * The workspace must not be used by other work on the GPU while the call runs.
 */
int moe_mxfp4_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                         const int32_t *ids, const float *weights,
                         const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                         const float *gate_up_bias, const uint8_t *down_blocks,
                         const uint8_t *down_scales, const float *down_bias, float alpha,
                         float limit, uint16_t *out, uint32_t flags, void *workspace,
                         size_t workspace_bytes, void *stream);

/* Bytes of workspace moe_mxfp4_forward_ex (and moe_nvfp4_forward_ex) needs for
 * these sizes (0 on bad sizes). */
size_t moe_mxfp4_workspace_size(int64_t T, int64_t H, int64_t I, int64_t E, int k);

/*
 * moe_token_tile_rows -- the token-tile height (rows of one expert per tile of the
 * grouped GEMMs) that moe_mxfp4_forward_ex (nvfp4 = 0) or moe_nvfp4_forward_ex
 * (nvfp4 != 0) uses for these sizes on the current device, or MOE_ERR_INVALID_ARG
 * for sizes the forward refuses.  Host-only; enqueues nothing.
 */
int moe_token_tile_rows(int64_t T, int64_t H, int64_t I, int64_t E, int k, int nvfp4);

/*
 * moe_permute -- the layer's grouping of (token, slot) pairs by expert, on its own
 * (FreeToken PR #838, "What it does": expert-ordered prefill views; the gather of
 * [T, k, 2I] rows its review names).  Pair p = t*k + j is routed to ids[p]:
 *   ids           int32 [T, k]
 *   counts        int32 [E]      pairs per expert
 *   offsets       int32 [E + 1]  exclusive scan of counts; offsets[E] = valid pairs
 *   tile_offsets  int32 [E + 1]  the same scan over ceil(counts[e] / tile_rows)
 *   sorted_pairs  int32 [T*k]    row r (expert order) holds its pair p; inside one
 *                                expert the rows follow ascending p (stable); rows
 *                                past offsets[E] are left untouched
 *   pair_rows     int32 [T*k] or NULL: the inverse, the row of pair p (-1 when the
 *                                pair was dropped)
 * Ids outside [0, E) drop their pair and raise MOE_DEVERR_BAD_EXPERT_ID.  Sizes:
 * T >= 1; 1 <= k <= 8; 1 <= E <= 256; tile_rows >= 1; T*k < 2^31.  Errors:
 * MOE_ERR_INVALID_ARG for null pointers or sizes.
 */
int moe_permute(const int32_t *ids, int64_t T, int k, int64_t E, int tile_rows, int32_t *counts,
                int32_t *offsets, int32_t *tile_offsets, int32_t *sorted_pairs, int32_t *pair_rows,
                void *stream);

/*
 * NVFP4 expert banks: the packed E2M1 codes of the MXFP4 layout with one E4M3 scale
 * byte per 16 consecutive elements of a row (OCP OFP8 v1.0 E4M3: bias 7, 3 mantissa
 * bits, subnormals m/8 * 2^-6, 0x7f / 0xff NaN, no infinities) and one fp32
 * weight_scale_2 per expert and projection.  FreeToken PR #838, review item "NVFP4
 * down scale vs. down bias": the fp32 scale multiplies the expert's matrix product
 * before its bias, out = sum_j w_j * (s * y_j + b).
 */

/*
 * nvfp4_dequantize -- standalone dequant of a packed NVFP4 bank to bf16.
 *   blocks  uint8 [E, N, K/2]   E2M1 codes, element 2m in the low nibble of byte m
 *   scales  uint8 [E, N, K/16]  E4M3 byte per 16 consecutive elements of a row
 *   scale2  fp32  [E] or NULL   weight_scale_2 per expert (NULL = 1)
 *   out     bf16  [E, N, K]     E2M1(code) * E4M3(scale) * scale2, rounded once to
 *                               nearest even from the exact product (exact when
 *                               scale2 is NULL or a power of two in range); NaN as
 *                               0x7fc0; a NaN scale byte sets MOE_DEVERR_BAD_SCALE
 * Sizes: E, N >= 1; K >= 16 and K % 16 == 0.  blocks and out must be 16-byte
 * aligned, scale2 4-byte aligned.  Errors: MOE_ERR_INVALID_ARG for null pointers,
 * sizes or alignment.
 */
int nvfp4_dequantize(const uint8_t *blocks, const uint8_t *scales, const float *scale2,
                     uint16_t *out, int64_t E, int64_t N, int64_t K, void *stream);

/*
 * moe_nvfp4_forward_ex -- the expert layer of moe_mxfp4_forward_ex over NVFP4 banks:
 *   gate_up_scales  uint8 [E, 2I, H/16] E4M3;  gate_up_scale2 fp32 [E, 2] (gate, up)
 *                   or NULL (= 1): h[2i] = s_gate * (W x)[2i] + b[2i],
 *                   h[2i+1] = s_up * (W x)[2i+1] + b[2i+1]
 *   down_scales     uint8 [E, H, I/16] E4M3;   down_scale2 fp32 [E] or NULL (= 1):
 *                   y = s_down * (W_d a) + b_d, out = sum_j w_j * y_j
 * Every other argument, size rule, flag, workspace rule and error as
 * moe_mxfp4_forward_ex; the workspace size is moe_mxfp4_workspace_size.  scale2
 * arrays must be 4-byte aligned.  NaN scale bytes set MOE_DEVERR_BAD_SCALE.
 */
int moe_nvfp4_forward_ex(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E, int k,
                         const int32_t *ids, const float *weights,
                         const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                         const float *gate_up_scale2, const float *gate_up_bias,
                         const uint8_t *down_blocks, const uint8_t *down_scales,
                         const float *down_scale2, const float *down_bias, float alpha,
                         float limit, uint16_t *out, uint32_t flags, void *workspace,
                         size_t workspace_bytes, void *stream);

/*
 * Expert parallelism (transformers PR #49431 "Restore GPT-OSS's router-masked
 * expert-parallel plan": with the experts spread over ranks, each rank's MXFP4
 * experts consume the routing data restricted to the experts it owns).  A rank that
 * owns experts [base, base + E_local) of the layer runs the layer in four calls
 * around two exchanges:
 *   moe_permute          its tokens' pairs in expert order (= owner order when
 *                        experts are split into contiguous ranges), pair_rows given
 *   moe_gather_pairs     the rows to ship: x rows, expert ids, routing weights
 *   (exchange)           rows offsets[base_r] .. offsets[base_r + E_r] go to rank r
 *   moe_mxfp4_expert_rows  the received rows through the rank's own experts -> fp32
 *   (exchange back)      each row returns to the rank it came from, in the same order
 *   moe_combine_pairs    the returned rows summed per token in slot order
 * On one rank the four calls give moe_mxfp4_forward_ex's output bit for bit.
 */

/*
 * moe_gather_pairs -- the expert-ordered rows of a permutation as a self-contained
 * batch.  For r < offsets[E] (read on the device), p = sorted_pairs[r]:
 *   x_rows[r] = x[p / k]   bf16 [T*k, H] (rows past offsets[E] untouched)
 *   row_ids[r] = ids[p]    int32 [T*k]
 *   row_weights[r] = weights[p]   fp32 [T*k]
 * x [T, H] bf16, ids / weights [T, k]; sorted_pairs and offsets as moe_permute wrote
 * them.  Sizes: T >= 1; 1 <= k <= 8; 1 <= E <= 256; H % 8 == 0; x and x_rows 16-byte
 * aligned.  Errors: MOE_ERR_INVALID_ARG.
 */
int moe_gather_pairs(const uint16_t *x, int64_t T, int64_t H, int k, const int32_t *ids, const float *weights,
                     const int32_t *sorted_pairs, const int32_t *offsets, int64_t E, uint16_t *x_rows,
                     int32_t *row_ids, float *row_weights, void *stream);

/*
 * moe_mxfp4_expert_rows -- R independent rows through the experts of a bank slice:
 * row r goes to expert row_ids[r] - expert_base of gate_up_* / down_* (banks of E
 * experts, laid out as for moe_mxfp4_forward_ex) and
 *   y_rows[r] = row_weights[r] * (W_d a + b_d)      (flags 0: weight on the output)
 *   y_rows[r] = W_d a                               (MOE_FLAG_WEIGHT_ON_INPUT: the
 *                                                    expert input is bf16(w * x))
 * with a the clamped SwiGLU of W_gu x + b_gu, i.e. one slot of moe_mxfp4_forward_ex
 * before the combine, in fp32 [R, H] (16-byte aligned).  Rows whose id falls outside
 * [expert_base, expert_base + E) are left unwritten and raise
 * MOE_DEVERR_BAD_EXPERT_ID.  workspace: NULL (allocated stream-ordered) or at least
 * moe_mxfp4_workspace_size(R, H, I, E, 1) bytes.  Every other rule and error as
 * moe_mxfp4_forward_ex; expert_base must lie in [0, 2^31).
 */
int moe_mxfp4_expert_rows(const uint16_t *x_rows, int64_t R, int64_t H, int64_t I, int64_t E, int64_t expert_base,
                          const int32_t *row_ids, const float *row_weights, const uint8_t *gate_up_blocks,
                          const uint8_t *gate_up_scales, const float *gate_up_bias,
                          const uint8_t *down_blocks, const uint8_t *down_scales, const float *down_bias,
                          float alpha, float limit, float *y_rows, uint32_t flags, void *workspace,
                          size_t workspace_bytes, void *stream);

/*
 * moe_combine_pairs -- out[t] = sum over j < k of y_rows[pair_rows[t*k + j]] in slot
 * order, in fp32, rounded once to bf16; slots whose pair_rows entry is -1 contribute
 * nothing (FreeToken PR #838 review: the result is sum w*(y + b), the weight already
 * inside each row).  y_rows fp32 [rows, H] (16-byte aligned), pair_rows int32
 * [T*k] (moe_permute's inverse), out bf16 [T, H].  Sizes: T >= 1; 1 <= k <= 8;
 * H % 4 == 0.  Errors: MOE_ERR_INVALID_ARG.
 */
int moe_combine_pairs(const float *y_rows, const int32_t *pair_rows, int64_t T, int k, int64_t H, uint16_t *out,
                      void *stream);

/* Static English text for a moe_status value. */
const char *moe_status_string(int status);

/*
 * moe_get_device_error -- synchronise `stream`, then return the sticky device
 * error bits (MOE_DEVERR_*) of the current device, clearing them.  Returns a
 * negative moe_status if the synchronisation itself fails.  Meant for tests and
 * diagnostics, not for the hot path.
 */
int moe_get_device_error(void *stream);

/*
 * moe_mxfp4_forward_noalloc -- the layer of moe_mxfp4_forward_ex, for callers that
 * cannot allocate device memory.  No counterpart in the paper.
 *
 * Some callers cannot call cudaMalloc or the stream-ordered allocator: a plugin
 * handed only its input and output buffers by a host framework that owns all
 * device memory, a serving loop that must never allocate after start-up (an
 * allocation can block, fail under a fixed memory budget, or synchronise the
 * device), or a process whose device memory is partitioned up front.  This call
 * allocates nothing: its scratch is one file-scope device array of
 * MOE_NOALLOC_SCRATCH_BYTES (32 MiB) that every GPU loading this library keeps
 * until the process exits.
 *   Arguments, flags and errors are those of moe_mxfp4_forward_ex without the
 *   workspace.  Sizes whose moe_mxfp4_workspace_size exceeds
 *   MOE_NOALLOC_SCRATCH_BYTES are refused with MOE_ERR_NO_MEMORY before anything
 *   is enqueued (for H = I = 2880 and k = 4 that is about 340 tokens).
 *   The first call on a device looks up the array's device address on that
 *   device (cudaGetSymbolAddress, with the device current); make that first call
 *   before any stream capture.  Later calls on the device reuse the address while
 *   the device's context stays the same; after the context is destroyed and made
 *   again (cudaDeviceReset) the next call looks it up anew, so make that call
 *   outside stream capture too.
 *   Every call on a device shares the one array, which keeps the previous call's
 *   contents; the layer writes every scratch byte before it reads it, so nothing
 *   needs clearing.  Calls whose work overlaps on the GPU (different streams
 *   without ordering between them) race on the array: order them.
 */
#define MOE_NOALLOC_SCRATCH_BYTES (32u * 1024u * 1024u)
int moe_mxfp4_forward_noalloc(const uint16_t *x, int64_t T, int64_t H, int64_t I, int64_t E,
                              int k, const int32_t *ids, const float *weights,
                              const uint8_t *gate_up_blocks, const uint8_t *gate_up_scales,
                              const float *gate_up_bias, const uint8_t *down_blocks,
                              const uint8_t *down_scales, const float *down_bias, float alpha,
                              float limit, uint16_t *out, uint32_t flags, void *stream);

/*
 * Instrumentation (not part of the layer's math).  Kernel launches made by the
 * calls above are counted per stage; while timing is enabled each launch is also
 * bracketed by a pair of CUDA events recorded on the call's stream.
 *   moe_profile_enable(on)        on != 0 starts event timing of every stage, 0
 *                                 stops it.
 *   moe_profile_enable_stages(mask) times only the stages whose bit (1 << stage)
 *                                 is set (0 stops timing); bits past
 *                                 MOE_PROFILE_STAGES give MOE_ERR_INVALID_ARG.
 *                                 An event pair sits between a stage's kernel and
 *                                 its neighbours in the stream, so timing a stage
 *                                 keeps that kernel from overlapping their tails
 *                                 (programmatic dependent launch); untimed
 *                                 stages keep it.
 *   moe_profile_read(ms, launches) waits for every recorded event, writes the
 *                                 summed kernel milliseconds and the launch counts
 *                                 per stage (arrays of MOE_PROFILE_STAGES entries,
 *                                 either may be NULL) since the previous read, and
 *                                 resets both.  Host-side state, one per process;
 *                                 not thread-safe.
 */
#define MOE_PROFILE_STAGES 7
enum {
    MOE_STAGE_ROUTE = 0,   /* moe_route                                   */
    MOE_STAGE_PERMUTE = 1, /* pair histogram / scan / stable scatter      */
    MOE_STAGE_GATHER = 2,  /* expert-ordered copy of the inputs           */
    MOE_STAGE_GATE_UP = 3, /* gate_up grouped GEMM + bias + clamped SwiGLU */
    MOE_STAGE_DOWN = 4,    /* down grouped GEMM + bias + routing weight   */
    MOE_STAGE_COMBINE = 5, /* per-token sum of the k expert rows          */
    MOE_STAGE_DEQUANT = 6  /* mxfp4_ / nvfp4_dequantize (+ _from_host)   */
};
int moe_profile_enable(int on);
int moe_profile_enable_stages(uint32_t stage_mask);
int moe_profile_read(double *ms, int64_t *launches);

#ifdef __cplusplus
}
#endif

#endif /* MOE_MXFP4_H */
