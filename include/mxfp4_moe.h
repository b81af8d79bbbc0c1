/*
 * mxfp4_moe.h -- C ABI of the MXFP4 mixture-of-experts expert block on NVIDIA B200 (sm_100a).
 *
 * What it computes
 * ----------------
 * The expert block of a GPT-OSS-style MoE layer whose expert weights stay packed as MXFP4,
 * forward and input-gradient backward, for adapter (LoRA) training where the quantized base
 * is frozen.  Sources:
 *   - "Add MXFP4 training support via a dequantize-on-the-fly fallback" (huggingface/
 *     transformers #47464), section "What this does": top-k router plus a GptOssExperts-style
 *     expert loop over weights dequantized on the fly, packed storage never modified; section
 *     "Relation to the backward triton kernels": gradients must reach the inputs through the
 *     expert math, the frozen base never needs a weight gradient.
 *   - "Integrate finegrained kernels: SOTA performance and per-module quantization"
 *     (huggingface/transformers #49658), commit on the gate|up row interleave (gate j at row
 *     2j, up j at row 2j+1; the GLU splits with stride 2) and commit on the per-expert bias
 *     operand (bias indexed by the tile's expert id, on the same output-row axis as the
 *     weight, fused in both GEMMs; the host keeps only the routing-weighted reduce).
 *   - OCP Microscaling Formats (MX) v1.0: E2M1 elements, UE8M0 scales (2^(s-127), 255 = NaN),
 *     32 elements per scale.
 *
 * Notation: T tokens, H hidden size, I intermediate size, E experts, k experts per token,
 * A = T*k (token, slot) assignments.  Forward per token t with selected experts e_j, j < k:
 *     w_t       = softmax over the k largest logits (largest first, ties -> lower index)
 *     h_{t,j}   = x_t W_gu[e_j]^T + b_gu[e_j]                       (2I, interleaved g/u)
 *     a_{t,j}   = (min(max(u,-L),L) + 1) * min(g,L) * sigmoid(alpha*min(g,L))   (I)
 *     y_{t,j}   = a_{t,j} W_d[e_j]^T + b_d[e_j]                      (H)
 *     out_t     = sum_j w_{t,j} y_{t,j}
 * Backward (given dY = dL/d out): dX = dL/dx, d_topk_w[t,j] = <dY_t, y_{t,j}>, and
 * d_logits = softmax-over-k Jacobian applied to d_topk_w (zero for unselected experts).
 * No weight gradient.
 *
 * Conventions for every entry point
 * ---------------------------------
 *  - All tensor pointers are DEVICE pointers owned by the caller, row-major, densely packed,
 *    at least 16-byte aligned.  "bf16" buffers are uint16_t bit patterns.  The library never
 *    allocates or frees device memory and never synchronizes the stream, except
 *    mxfp4_moe_check and mxfp4_moe_profile_end (mxfp4_moe_forward_static works on a static
 *    device array that exists while the library is loaded).
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default stream).  Work is
 *    enqueued on it and the call returns; results are valid once the stream reaches them.
 *  - Return value: 0 on success, a negative MXFP4_MOE_ERR_* code otherwise.  Argument errors
 *    are detected before anything is enqueued.  Faults detected on the device (a bounded wait
 *    that expired, an index out of range) are written to an error word inside the workspace
 *    and reported by mxfp4_moe_check.
 *  - The current CUDA device must be an sm_100 part (B200); otherwise
 *    MXFP4_MOE_ERR_UNSUPPORTED_DEVICE.
 *  - Shapes: H and I multiples of 32 (one MX block), 1 <= k <= E <= 256, T >= 1, A = T*k < 2^31.
 */
#ifndef MXFP4_MOE_H_
#define MXFP4_MOE_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MXFP4_MOE_API __attribute__((visibility("default")))
#else
#define MXFP4_MOE_API
#endif

#define MXFP4_MOE_OK 0
#define MXFP4_MOE_ERR_INVALID_ARG (-1)         /* null pointer, bad shape, misaligned pointer */
#define MXFP4_MOE_ERR_WORKSPACE_TOO_SMALL (-2)  /* ws_bytes below mxfp4_moe_workspace_size  */
#define MXFP4_MOE_ERR_UNSUPPORTED_DEVICE (-3)   /* current device is not sm_100           */
#define MXFP4_MOE_ERR_CUDA (-4)                 /* a CUDA runtime call or launch failed    */
#define MXFP4_MOE_ERR_DEVICE_TIMEOUT (-5)       /* a bounded device-side wait expired      */
#define MXFP4_MOE_ERR_DEVICE_BOUNDS (-6)        /* a device-side index check failed        */

/* Problem shape and GLU constants (GPT-OSS: glu_alpha = 1.702, glu_limit = 7).
 * Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", section "What this does" (the GptOssExperts expert loop and its activation).
 * gate_up_format selects the operands of the forward's gate_up GEMM:
 *   MXFP4_MOE_GATE_UP_BF16 (0, what a zero-initialised struct gives): the weights dequantized
 *     to bf16 on the fly against the bf16 token rows;
 *   MXFP4_MOE_GATE_UP_BLOCK_SCALED (1): the weights' E2M1 codes and UE8M0 scales as stored
 *     against the token rows split into two E4M3 parts with a UE8M0 scale per 32 elements, on
 *     the block-scaled tensor-core MMA ("Integrate finegrained kernels: SOTA performance and
 *     per-module quantization", the commits on the activation format and input recipe).
 * Any other value is INVALID_ARG.  The backward is the same for both. */
#define MXFP4_MOE_GATE_UP_BF16 0
#define MXFP4_MOE_GATE_UP_BLOCK_SCALED 1
typedef struct {
  int32_t T, H, I, E, k;
  float glu_alpha;
  float glu_limit;
  int32_t gate_up_format;
} mxfp4_moe_dims;

/* Frozen expert weights in the packed MXFP4 layout (read only, never modified).
 * Source: "Integrate finegrained kernels: SOTA performance and per-module quantization", the loader commit (`_blocks` / `_scales` tensors) and the gate|up row
 * interleave commit; OCP Microscaling Formats (MX) v1.0 for the E2M1 / UE8M0 encodings.
 *   gu_blocks  uint8 [E][2I][H/2]  gate_up rows, interleaved: row 2j = gate j, row 2j+1 = up j.
 *                                  Byte i of a row holds element 2i (low nibble) and 2i+1
 *                                  (high nibble), E2M1 codes.
 *   gu_scales  uint8 [E][2I][H/32] UE8M0 scale of each 32-element block of a row.
 *   gu_bias    bf16  [E][2I]       interleaved like the rows.
 *   dn_blocks  uint8 [E][H][I/2]   down rows, same packing along I.
 *   dn_scales  uint8 [E][H][I/32]
 *   dn_bias    bf16  [E][H]
 * Stacked [gate; up] checkpoints must be interleaved first (mxfp4_moe_interleave_gate_up
 * does it); the bytes do not tell the two orders apart. */
typedef struct {
  const uint8_t* gu_blocks;
  const uint8_t* gu_scales;
  const uint16_t* gu_bias;
  const uint8_t* dn_blocks;
  const uint8_t* dn_scales;
  const uint16_t* dn_bias;
} mxfp4_moe_weights;

/* Bytes of device workspace that mxfp4_moe_forward / mxfp4_moe_backward_input need for `d`
 * (no counterpart in the pages: the caller-owned memory of this interface).
 * The forward leaves its saved state in the workspace (routing, permutation, the GLU output and
 * its two derivative factors per (assignment, feature)); the backward reads it and uses the
 * rest as scratch.
 * Errors: INVALID_ARG (null pointers, bad shape). */
MXFP4_MOE_API int mxfp4_moe_workspace_size(const mxfp4_moe_dims* d, size_t* bytes);

/* Bytes of the transposed weight copy made by mxfp4_moe_transpose_weights (no counterpart in
 * the pages). */
MXFP4_MOE_API int mxfp4_moe_transposed_weights_size(const mxfp4_moe_dims* d, size_t* bytes);

/* One-time layout step for the backward (no counterpart in the pages; like "Integrate finegrained kernels: SOTA performance and per-module quantization"'s one-time
 * post-load layout conversions).  Weights are frozen, so it is done once per set of
 * weights, not per step).  The input-gradient GEMMs contract over the OUTPUT axis of the
 * stored weights (dact = dy W_d, dx = dh W_gu), where the 32-element scale blocks run across
 * the contraction.  This call writes the same E2M1 codes and UE8M0 scale bytes, transposed:
 *   [0, E*I*H/2)           dn_blocks_t uint8 [E][I][H/2]   element (i, h) = W_d[e][h][i]
 *   then E*(2I)*H/2 bytes  gu_blocks_t uint8 [E][H][2I/2]  element (h, n) = W_gu[e][n][h]
 *   then E*(I/32)*H bytes  dn_scales_t uint8 [E][I/32][H]  = dn_scales[e][h][i/32]
 *   then E*(H/32)*2I bytes gu_scales_t uint8 [E][H/32][2I] = gu_scales[e][n][h/32]
 * (each region starts 256-byte aligned).  Values are not re-quantized; the copy is still
 * packed MXFP4 (4.25 bits per weight).
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL (wt_bytes too small), UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_transpose_weights(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w, void* wt,
                                size_t wt_bytes, void* stream);

/* Forward.  Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", section "What this does" (top-k router + expert loop over weights
 * dequantized on the fly); "Integrate finegrained kernels: SOTA performance and per-module quantization", commits on the gate|up interleave and the per-expert bias.
 *   x        bf16  [T][H]   activations
 *   logits   fp32  [T][E]   router logits (the router linear stays with the caller)
 *   y        bf16  [T][H]   output: sum_j w_{t,j} y_{t,j}
 *   topk_idx int32 [T][k]   output, may be NULL: selected experts, largest logit first
 *   topk_w   fp32  [T][k]   output, may be NULL: softmax over the selected logits
 *   ws, ws_bytes            workspace (>= mxfp4_moe_workspace_size); keep it unmodified until
 *                           mxfp4_moe_backward_input has been enqueued if a backward follows.
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_forward(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w, const uint16_t* x,
                      const float* logits, uint16_t* y, int32_t* topk_idx, float* topk_w,
                      void* ws, size_t ws_bytes, void* stream);

/* Forward for callers that cannot allocate device memory (no counterpart in the source pages:
 * a deployment form of mxfp4_moe_forward, not part of the method).
 * Who needs it: code that runs the layer where it holds no device allocator -- an
 * inference-engine plugin whose enqueue step receives only input and output pointers, a
 * process whose device memory belongs to another framework's pool, or a latency-critical
 * serving loop that cannot pay for cudaMalloc's implicit device synchronization.
 * What it does: exactly mxfp4_moe_forward, with the workspace taken from a fixed array of
 * MXFP4_MOE_STATIC_SCRATCH_BYTES (64 MiB) that the library holds in device memory.  The array
 * exists in every CUDA context that loads the library's module holding it: under the CUDA 12
 * default of lazy module loading, on each device where this entry point has run; with
 * CUDA_MODULE_LOADING=EAGER, on every device the library is used on.  It stays until the
 * process exits (or the context is destroyed).  Arguments mean what they mean for
 * mxfp4_moe_forward; the caller still provides x, logits, y and the optional topk_idx /
 * topk_w.  No cudaMalloc, cudaFree or other allocating call is made.
 * Set-up: the first call in a context looks up the array's device address
 * (cudaGetSymbolAddress) with that device current and caches it together with the context
 * handle, so make that first call before any stream capture.  A cudaDeviceReset (or any other
 * teardown of the context) reloads the module, possibly at another address; the next call
 * notices the new context and looks the address up again, so after a reset the first call
 * must again come before any capture.
 * Sharing: every call uses the same array and leaves its contents there for the next call; the
 * call clears what must start at zero.  Calls that overlap on the GPU (other streams, other
 * host threads) race on the array and must be serialized by the caller.  The saved state it
 * leaves is not usable by mxfp4_moe_backward_input.  Device-side faults (an expired bounded
 * wait, an index check) are recorded in the array's error word: read them with
 * mxfp4_moe_forward_static_check.
 * Errors: WORKSPACE_TOO_SMALL when mxfp4_moe_workspace_size(d) exceeds
 * MXFP4_MOE_STATIC_SCRATCH_BYTES (at H = I = 2880, k = 4 that is above 480 tokens);
 * otherwise as mxfp4_moe_forward. */
#define MXFP4_MOE_STATIC_SCRATCH_BYTES (64ull << 20)
MXFP4_MOE_API int mxfp4_moe_forward_static(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w,
                                           const uint16_t* x, const float* logits, uint16_t* y,
                                           int32_t* topk_idx, float* topk_w, void* stream);

/* Companion of mxfp4_moe_forward_static (no counterpart in the source pages): synchronizes
 * `stream`, then reads and clears the error word of the static array in the current context,
 * like mxfp4_moe_check does for a workspace.  Returns 0, DEVICE_TIMEOUT or DEVICE_BOUNDS (from
 * the device, with the tag in *where, which may be NULL), CUDA if the stream reported an error,
 * UNSUPPORTED_DEVICE on a device other than sm_100.  Allocates nothing. */
MXFP4_MOE_API int mxfp4_moe_forward_static_check(void* stream, int32_t* where);

/* Input-gradient backward through the frozen quantized weights (no weight gradient).
 * Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", sections "Why (the silent-gradient trap)" and "Relation to the backward
 * triton kernels" (gradients must reach the inputs through the expert math).
 *   wt       the transposed copy from mxfp4_moe_transpose_weights for the same weights
 *   dy       bf16 [T][H]  upstream gradient dL/d(out)
 *   ws       the workspace the matching mxfp4_moe_forward used (its saved state is read; the
 *            scratch part is overwritten)
 *   dx       bf16 [T][H]  output dL/dx
 *   d_topk_w fp32 [T][k]  output dL/d(topk_w), slot order of the forward's topk_idx
 *   d_logits fp32 [T][E]  output, may be NULL: dL/d(logits) through the softmax over k
 * Errors: INVALID_ARG, WORKSPACE_TOO_SMALL, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_backward_input(const mxfp4_moe_dims* d, const mxfp4_moe_weights* w,
                             const void* wt, size_t wt_bytes, const uint16_t* dy, void* ws,
                             size_t ws_bytes, uint16_t* dx, float* d_topk_w, float* d_logits,
                             void* stream);

/* Layout helper: stacked gate_up rows to the interleaved order the block expects.
 * "Integrate finegrained kernels: SOTA performance and per-module quantization", commit on the
 * gate|up row interleave: GPT-OSS ships gate_up with gate j at row 2j and up j at row 2j+1,
 * checkpoints stored with the halves stacked ([all gates; all ups]) must be converted by the
 * caller, and the bytes cannot be inspected to tell which order a tensor is in.
 *   stacked_blocks uint8 [E][2I][H/2], stacked_scales uint8 [E][2I][H/32], stacked_bias bf16
 *   [E][2I] with row j = gate j and row I + j = up j; the outputs (same shapes, caller-owned,
 *   not overlapping the inputs) receive row 2j = gate j and row 2j + 1 = up j.  Bytes are
 *   copied unchanged (no re-quantization).  Uses d->E, d->H, d->I only.  Packed pointers must
 *   be 16-byte aligned.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_interleave_gate_up(const mxfp4_moe_dims* d, const uint8_t* stacked_blocks,
                                 const uint8_t* stacked_scales, const uint16_t* stacked_bias,
                                 uint8_t* blocks, uint8_t* scales, uint16_t* bias, void* stream);

/* Grouped matmul over expert-sorted rows with MXFP4 weights dequantized on the fly: the
 * product the block's GEMMs are built on, without their epilogues ("Integrate finegrained
 * kernels: SOTA performance and per-module quantization", the experts' grouped GEMM over
 * expert-sorted rows; "Add MXFP4 training support via a dequantize-on-the-fly fallback",
 * section "What this does": weights dequantized on the fly, packed storage never modified).
 * For every expert e and row r in [off[e], off[e+1]):
 *     out[r][n] = bf16( sum_k x[r][k] * W_e[n][k] )   (fp32 accumulation)
 *   off     int32 [E+1] DEVICE, off[0] = 0, non-decreasing, off[E] = A
 *   x       bf16  [A][K]
 *   transposed == 0: blocks uint8 [E][N][K/2], scales uint8 [E][N][K/32] (the stored layout:
 *                    W_e[n][k] = E2M1(code) * 2^(s[e][n][k/32] - 127))
 *   transposed == 1: blocks uint8 [E][N][K/2], scales uint8 [E][N/32][K] (the layout
 *                    mxfp4_moe_transpose_weights writes: W_e[n][k] uses s[e][n/32][k])
 *   out     bf16  [A][N]
 *   err_word  device int32[4] or NULL: a device-side fault (an expired bounded wait) is
 *             recorded there; read it with mxfp4_moe_check.
 * N and K multiples of 32, 1 <= E <= 256.  Used to test the fused dequantizer bit for bit
 * (one-hot rows of x pick single weights), and usable as a grouped expert projection.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_grouped_matmul(int32_t E, int32_t N, int32_t K, int32_t A,
                                           const int32_t* off, const uint16_t* x,
                                           const uint8_t* blocks, const uint8_t* scales,
                                           int32_t transposed, uint16_t* out, int32_t* err_word,
                                           void* stream);

/* The residual stream between stacked blocks, the caller's side of the block boundary, in one
 * kernel.  Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", section
 * "What this does" (decoder layers around the MoE block, trained with gradient
 * checkpointing: residual stream and router linear); the fusion has no counterpart there.
 *   x_out[t][h]  = bf16(x[t][h] + y[t][h])          fp32 sum rounded once (round to nearest
 *                                                   even); only when y is not NULL
 *   logits[t][e] = sum_h xs[t][h] * w_r[h][e] + b_r[e]   fp32 accumulation of the bf16
 *                                                   products, xs = x_out (y given) or x
 *                                                   (y NULL); only when logits is not NULL
 *   x, y, x_out  bf16 [T][H] DEVICE, 16-byte aligned; x_out NULL exactly when y is NULL
 *   w_r          bf16 [H][E] DEVICE, 16-byte aligned (the router linear), required with logits
 *   b_r          bf16 [E] DEVICE or NULL (no bias)
 *   logits       fp32 [T][E] DEVICE or NULL
 * T >= 0, H a multiple of 32, 1 <= E <= 256; at least one of y and logits.  x_out must not
 * overlap x or y.  Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_residual_router(int32_t T, int32_t H, int32_t E, const uint16_t* x,
                                            const uint16_t* y, const uint16_t* w_r,
                                            const uint16_t* b_r, uint16_t* x_out,
                                            float* logits, void* stream);

/* The residual stream's gradient through one stacked block, in one kernel.  Source: "Add
 * MXFP4 training support via a dequantize-on-the-fly fallback", section "What this does"
 * (the backward of gradient-checkpointed decoder layers); the fusion has no counterpart there.
 *   g_out[t][h] = bf16(g[t][h] + dx[t][h] + sum_e d_logits[t][e] * w_r[h][e])
 * in fp32 (fused multiply-adds over e in ascending order, then g + dx + that sum), rounded
 * once.
 *   g, dx, g_out  bf16 [T][H] DEVICE, 16-byte aligned; g_out may be g itself
 *   d_logits      fp32 [T][E] DEVICE (mxfp4_moe_backward_input's router gradient)
 *   w_r           bf16 [H][E] DEVICE, 16-byte aligned
 * T >= 0, H a multiple of 32, 1 <= E <= 256.  Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_grad_chain(int32_t T, int32_t H, int32_t E, const uint16_t* g,
                                       const uint16_t* dx, const float* d_logits,
                                       const uint16_t* w_r, uint16_t* g_out, void* stream);

/* Standalone dequantization (diagnostics and tests): rows of packed MXFP4 -> bf16.
 * Source: "Add MXFP4 training support via a dequantize-on-the-fly fallback", section "What this does" (`_dequantize_weights`); OCP MX v1.0.
 *   blocks uint8 [rows][K/2], scales uint8 [rows][K/32], out bf16 [rows][K]; K multiple of 32.
 * out = bf16(E2M1(code) * 2^(s-127)), exact (the product is always representable in bf16 or
 * overflows to inf); s = 255 gives NaN.
 * Errors: INVALID_ARG, UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_dequantize(const uint8_t* blocks, const uint8_t* scales, int64_t rows, int64_t K,
                         uint16_t* out, void* stream);

/* (No counterpart in the pages: failure detection of this library.)
 * Synchronize `stream`, then read and clear the device error word in `ws` (a workspace used by
 * forward/backward).  Returns 0, DEVICE_TIMEOUT or DEVICE_BOUNDS (from the device), or CUDA
 * if the stream reported an error.  `where` (may be NULL) receives the device-side tag. */
MXFP4_MOE_API int mxfp4_moe_check(void* ws, void* stream, int32_t* where);

/* Self-test of failure detection (a diagnostic with no counterpart in the pages).  Enqueues one
 * small kernel on `stream` whose two device-side waits are on barriers that nothing ever
 * completes.  The first wait runs out after the library's one-second limit: it records
 * MXFP4_MOE_ERR_DEVICE_TIMEOUT with tag 0xF00 in the error word at the start of `ws` and
 * raises the kernel's abort flag; the second wait (started half a second later) must leave
 * through that flag and sets the 32-bit word at byte offset 8 of `ws` to 1; the kernel then
 * frees its tensor memory and returns.  Nothing faults and the CUDA context stays usable.
 *   ws: device memory, at least 16 bytes, 16-byte aligned, the first 16 bytes zero (a fresh
 *       workspace qualifies); the caller owns it.
 * Returns OK once enqueued; the outcome is read with mxfp4_moe_check(ws, ...), which then
 * returns DEVICE_TIMEOUT with *where == 0xF00.  Takes about one second of device time.
 * Errors: INVALID_ARG (null, short or misaligned ws), UNSUPPORTED_DEVICE, CUDA. */
MXFP4_MOE_API int mxfp4_moe_selftest_wait_timeout(void* ws, size_t ws_bytes, void* stream);

/* Per-kernel timing (diagnostics; no counterpart in the pages).  Between mxfp4_moe_profile_begin() and
 * mxfp4_moe_profile_end(), the library records a CUDA event pair on the launching stream around
 * every kernel it enqueues (host-side bookkeeping only; results are unchanged).
 * mxfp4_moe_profile_end synchronizes those events and fills up to `max` entries of `out` with
 * one line per kernel name: launches and summed device time in milliseconds; `*n` receives the
 * number of distinct kernels.  Not thread-safe: profile from one host thread.
 * Errors: INVALID_ARG (null out/n), CUDA. */
typedef struct {
  char name[48];
  int32_t launches;
  double total_ms;
} mxfp4_moe_kernel_time;
MXFP4_MOE_API int mxfp4_moe_profile_begin(void);
MXFP4_MOE_API int mxfp4_moe_profile_end(mxfp4_moe_kernel_time* out, int32_t max, int32_t* n);

/* Static description of a return code (no counterpart in the pages). */
MXFP4_MOE_API const char* mxfp4_moe_strerror(int code);

/* How this library was built (no counterpart in the pages): bit 0 set for the debug build
 * (libmxfp4_moe_debug.so, compiled with MXFP4_MOE_DEBUG=1), whose kernels check the indices
 * they read from the workspace (perm, inv, the expert offsets) and record
 * MXFP4_MOE_ERR_DEVICE_BOUNDS with a tag in the error word instead of making an access
 * through a bad index.  The release build returns 0 and carries no such checks.  Never fails. */
#define MXFP4_MOE_BUILD_DEBUG 1
MXFP4_MOE_API int mxfp4_moe_build_flags(void);

#ifdef __cplusplus
}
#endif

#endif /* MXFP4_MOE_H_ */
