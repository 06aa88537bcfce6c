/*
 * dynconv.h -- C ABI of the B200 (sm_100a) dynamic-convolution library.
 *
 * The library computes the per-sample kernel-mixture convolution:
 *
 *   alpha_b = sigmoid(FC(GAP(x_b)))  or  softmax(FC(GAP(x_b)) / tau)
 *   W_b     = sum_i alpha_{b,i} W_i                 (n static experts W_i)
 *   y_b     = conv2d(x_b, W_b) + sum_i alpha_{b,i} bias_i
 *
 * Sources: the kernel as a sum of n static kernels, each weighted by an
 * attention computed from the input, is the definition in "KernelWarehouse: Rethinking the Design of
 * Dynamic Convolution" (abstract); one specialised kernel per example is
 * "CondConv: Conditionally Parameterized Convolutions for Efficient Inference"
 * (abstract); the temperature on the kernel attention is from "FMDConv: Fast
 * multi-attention dynamic convolution via speed-accuracy trade-off" (abstract).
 * The router's exact form (global average pool -> one linear layer -> sigmoid
 * or temperature softmax), the bias mixing, the NHWC layout and the bf16
 * storage are readings taken where those pages are silent.
 *
 * Conventions shared by every entry point:
 *  - All tensor pointers are DEVICE pointers owned by the caller; the library
 *    never frees them and keeps no reference after the call's work completes.
 *  - Calls only enqueue work on `stream` (a cudaStream_t passed as void*;
 *    NULL is the legacy default stream) and return; results are valid once the
 *    stream reaches that point.
 *  - No call allocates device memory. Scratch, where a variant needs it, is a
 *    caller-provided workspace (see dynconv_workspace_size).
 *  - Return value: DYNCONV_OK (0) or a negative status below. Argument errors
 *    are detected on the host before anything is launched. No C++ exception
 *    crosses this interface. There is no CPU fallback: without a usable
 *    sm_100 device the calls fail with DYNCONV_ERR_CUDA.
 *
 * Layouts (row-major, last index fastest):
 *   x        [B][H][W][C_in]                    dtype (fp32 or bf16), NHWC
 *   experts  [n][C_out][KH][KW][C_in/groups]    dtype
 *   Wr       [n][C_in] fp32,  br [n] fp32       router weights / bias
 *   bias     [n][C_out] fp32, or NULL for none  per-expert output bias
 *   alpha    [B][n] fp32                        routing weights
 *   y        [B][H_out][W_out][C_out]           dtype, NHWC
 * with H_out = (H + 2*pad - KH)/stride + 1, W_out likewise.
 */
#ifndef DYNCONV_H
#define DYNCONV_H

#include <stddef.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- status codes ---------------------------------------------------- */
#define DYNCONV_OK               0
#define DYNCONV_ERR_INVALID_ARG (-1)  /* NULL pointer, non-positive size, tau <= 0 with softmax,
                                         groups not dividing the channels, bad enum value */
#define DYNCONV_ERR_UNSUPPORTED (-2)  /* a shape or variant that no kernel here handles */
#define DYNCONV_ERR_MISALIGNED  (-3)  /* a pointer not 16-byte aligned (vector loads / TMA) */
#define DYNCONV_ERR_CUDA        (-4)  /* a CUDA runtime or driver error (no device, launch failure) */
#define DYNCONV_ERR_TIMEOUT     (-5)  /* a kernel's bounded wait expired (see dynconv_device_status) */
#define DYNCONV_ERR_WORKSPACE   (-6)  /* the forced variant needs a larger workspace */

/* ---- enums -------------------------------------------------------------- */
typedef enum { DYNCONV_F32 = 0, DYNCONV_BF16 = 1 } dynconv_dtype;
typedef enum { DYNCONV_SIGMOID = 0, DYNCONV_SOFTMAX = 1 } dynconv_mode;

/* Which forward kernel runs.
 *  AUTO    - chosen by a host cost model from the descriptor (and the workspace
 *            the caller passed);
 *  FUSED   - input-side mixing inside the tensor-core convolution: every CTA
 *            mixes its sample's weight tile from the experts on CUDA cores
 *            into a bf16 shared-memory operand of tcgen05 MMAs (bf16 only);
 *  OUTSIDE - output-side mixing: y_b = sum_i alpha_{b,i} (x_b conv W_i) + b_b as
 *            one K-stacked tensor-core GEMM over (expert, tap, channel) with the
 *            operand alpha_{b,i} W_i (bf16 only; n times the conv work);
 *  PREMIX  - W_b for all samples is mixed first into the workspace (bf16),
 *            on CUDA cores when n <= 8 (a store-bound stream of at most 8
 *            multiply-adds per weight) and by a tcgen05 GEMM over the experts
 *            when n > 8; then a tensor-core convolution TMA-loads it
 *            (bf16 only; needs dynconv_workspace_size bytes);
 *  DIRECT  - CUDA-core direct convolution, fp32 accumulation, any shape
 *            (the fp32 path; also bf16 shapes the tensor-core kernels reject);
 *  DEPTHWISE - CUDA-core depthwise kernel (groups == C_in == C_out). */
typedef enum {
  DYNCONV_VARIANT_AUTO = 0,
  DYNCONV_VARIANT_FUSED = 1,
  DYNCONV_VARIANT_OUTSIDE = 2,
  DYNCONV_VARIANT_PREMIX = 3,
  DYNCONV_VARIANT_DIRECT = 4,
  DYNCONV_VARIANT_DEPTHWISE = 5
} dynconv_variant;

/* Layer descriptor. groups must divide C_in and C_out; the depthwise kernel
 * takes groups == C_in == C_out. `variant` forces a kernel (AUTO: cost model). */
typedef struct {
  int B, C_in, H, W, C_out, KH, KW, stride, pad, groups, n;
  int dtype;    /* dynconv_dtype */
  int variant;  /* dynconv_variant */
} dynconv_desc;

/* ---- routing ------------------------------------------------------------
 * alpha[b][i] for every sample b of x (steps: global average pool over the
 * H*W unpadded pixels, one linear layer z = Wr g + br, then sigmoid(z), or
 * softmax(z / tau) over the n experts).
 *   desc   uses B, C_in, H, W, n, dtype;
 *   x      device, [B][H][W][C_in] of desc->dtype, 16-byte aligned, and
 *          C_in * sizeof(dtype) a multiple of 16;
 *   Wr     device fp32 [n][C_in];  br device fp32 [n] or NULL (zero bias);
 *   mode   dynconv_mode; tau > 0 required for SOFTMAX, ignored for SIGMOID;
 *   alpha  device fp32 [B][n], written.
 * Deterministic: the reduction order is fixed. Errors: INVALID_ARG,
 * MISALIGNED, UNSUPPORTED (n > 1024 or C_in > 16384), CUDA. */
int dynconv_route(const dynconv_desc* desc, const void* x, const float* Wr, const float* br,
                  int mode, float tau, float* alpha, void* stream);

/* ---- forward -------------------------------------------------------------
 * y_b = conv2d(x_b, sum_i alpha[b][i] W_i) + sum_i alpha[b][i] bias_i for every b.
 *   x, experts, y  device, layouts above, desc->dtype, 16-byte aligned;
 *   alpha          device fp32 [B][n] (typically written by dynconv_route on
 *                  the same stream);
 *   bias           device fp32 [n][C_out] or NULL;
 *   workspace      device scratch of workspace_bytes bytes, or NULL/0. Only the
 *                  PREMIX variant uses it; AUTO never picks PREMIX unless the
 *                  workspace is large enough. It holds every sample's mixed
 *                  kernel and, after them, the mixing GEMM's tile counter
 *                  (zeroed on the stream by each call); its contents need not
 *                  be preserved between calls, and two calls in flight at once
 *                  need two workspaces.
 *                  (The counters with which the streamed mixing publishes each
 *                  K slice live in library-owned device memory, one slot per
 *                  stream, zero between launches; after a bounded wait expired
 *                  they are re-zeroed when dynconv_device_status reports it.)
 * Precision: bf16 in, fp32 accumulate, the mixed kernel rounded once to bf16
 * (tensor-core variants), y rounded once to bf16. fp32 layers accumulate and
 * mix in fp32.
 * Errors: INVALID_ARG, UNSUPPORTED (forced variant cannot take the shape),
 * MISALIGNED, WORKSPACE (forced PREMIX with too small a workspace), CUDA. */
int dynconv_forward(const dynconv_desc* desc, const void* x, const void* experts,
                    const float* alpha, const float* bias, void* y, void* workspace,
                    size_t workspace_bytes, void* stream);

/* ---- FMDConv channel attentions ----------------------------------------------
 * FMDConv combines the kernel attention with an input attention and an output
 * attention (FMDConv: Fast multi-attention dynamic convolution via
 * speed-accuracy trade-off, abstract). The page gives no formula; the reading
 * taken: per-sample, per-channel factors in (0, 1), computed like the kernel
 * attention from the average pool g_b of the layer input,
 *   a_in[b][c]  = sigmoid(Wi[c][:] . g_b + bi[c])   (c < C_in),
 *   a_out[b][o] = sigmoid(Wo[o][:] . g_b + bo[o])   (o < C_out),
 * and applied as y_b = a_out_b * (conv2d(a_in_b * x_b, W_b) + sum_i alpha_bi bias_i),
 * each factor multiplying one channel of every pixel.
 *
 * dynconv_route_channels: a_in and/or a_out (either pair Wi/a_in or Wo/a_out
 * may be NULL, not both): Wi fp32 [C_in][C_in], bi fp32 [C_in] or NULL,
 * a_in fp32 [B][C_in]; Wo fp32 [C_out][C_in], bo [C_out] or NULL, a_out fp32
 * [B][C_out]; x as dynconv_route. Deterministic.
 * Errors: INVALID_ARG, UNSUPPORTED (C_in or C_out > 1024), MISALIGNED, CUDA.
 *
 * dynconv_forward_attn: dynconv_forward with a_in [B][C_in] and a_out
 * [B][C_out] (device fp32, either NULL = all ones). The output factor is taken
 * in every variant's epilogue. The input factor is folded into the mixed
 * kernel (W_b[o][kh][kw][c] * a_in[b][c], the same by linearity); variants that
 * take it: PREMIX with the CUDA-core mixer (n <= 8), DEPTHWISE, DIRECT. With
 * a_in and variant AUTO the choice falls back to those; a forced FUSED or
 * OUTSIDE variant with a_in returns UNSUPPORTED.
 * Errors as dynconv_forward. */
int dynconv_route_channels(const dynconv_desc* desc, const void* x, const float* Wi,
                           const float* bi, float* a_in, const float* Wo, const float* bo,
                           float* a_out, void* stream);
int dynconv_forward_attn(const dynconv_desc* desc, const void* x, const void* experts,
                         const float* alpha, const float* bias, const float* a_in,
                         const float* a_out, void* y, void* workspace, size_t workspace_bytes,
                         void* stream);

/* ---- routing pooled in the previous layer (chained layers) -----------------
 * When layer L+1's input is layer L's output, the average pool of L+1's
 * routing step can be taken in L's epilogue, where the output is already in
 * registers: dynconv_forward_pooled writes, besides y, partial channel sums of
 * y as stored, and dynconv_route_pooled finishes L+1's routing from them
 * without reading its input again. (The pages give the attentions as
 * input-dependent, KernelWarehouse, abstract; the average pool is the reading
 * taken for the routing step, see dynconv_route.)
 *
 * dynconv_pool_parts: the number P >= 1 of partial sums per (sample, channel)
 * that dynconv_forward_pooled writes for this descriptor and workspace size
 * (the same inputs dynconv_select_variant takes), or a negative status. Pure
 * host function.
 *
 * dynconv_forward_pooled: as dynconv_forward, and
 *   ysum  device fp32 [B][P][C_out]: ysum[b][p][c] is the sum, over the p-th of
 *         P fixed disjoint subsets of the output pixels (together all of them),
 *         of y[b][h][w][c] as stored (after rounding to desc->dtype); every
 *         element is written. Deterministic.
 *   The tensor-core variants add the sums in their epilogue; the CUDA-core
 *   variants (DIRECT, DEPTHWISE) add them in a second pass over y.
 * Errors as dynconv_forward; INVALID_ARG if ysum is NULL.
 *
 * dynconv_route_pooled: alpha for the layer described by `desc` (desc->C_in =
 * the previous layer's C_out; desc->H, desc->W = its output size), from `parts`
 * partial sums per channel: g[b][c] = (sum over p, in order, of
 * ysum[b][p][c]) / (H*W); then the linear layer and activation exactly as
 * dynconv_route (same Wr, br, mode, tau, alpha). Deterministic.
 * Errors: INVALID_ARG (NULL pointers, parts < 1, bad mode or tau),
 * UNSUPPORTED (n > 1024 or C_in > 16384), CUDA. */
int dynconv_pool_parts(const dynconv_desc* desc, size_t workspace_bytes);
int dynconv_forward_pooled(const dynconv_desc* desc, const void* x, const void* experts,
                           const float* alpha, const float* bias, void* y, float* ysum,
                           void* workspace, size_t workspace_bytes, void* stream);
int dynconv_route_pooled(const dynconv_desc* desc, const float* ysum, int parts, const float* Wr,
                         const float* br, int mode, float tau, float* alpha, void* stream);

/* ---- forward without caller-provided scratch ----------------------------
 * The pages describe no such entry point; it has no counterpart in the method.
 *
 * For callers that cannot allocate device memory where they call the layer:
 * for example a plugin or callback run by a host framework that owns all
 * device memory and hands out no workspace, or code that must not call
 * cudaMalloc after start-up (cudaMalloc synchronises the device and can fail
 * once memory is committed). It computes exactly what dynconv_forward with the
 * PREMIX variant computes, bit for bit: the same mixer PREMIX selects (CUDA
 * cores for n <= 8, the tcgen05 mixing GEMM above), then the tensor-core
 * convolution; but its scratch is a fixed array that the library itself
 * defines in device memory: DYNCONV_NOALLOC_MAX_BYTES bytes, reserved on every
 * GPU on which the library's kernels are loaded, for the life of the process.
 *
 *   desc, x, experts, alpha, bias, y, stream: as for dynconv_forward (bf16,
 *   dense, stride 1, "same" padding; desc->variant is ignored).
 * Limit: the shape must fit, dynconv_workspace_size(desc) <= DYNCONV_NOALLOC_MAX_BYTES;
 * larger shapes are rejected with DYNCONV_ERR_WORKSPACE before anything runs
 * (for example B=64, 128->128 channels, 3x3 needs 18.9 MB and fits; B=256,
 * 256->256, 3x3 needs 302 MB and does not).
 * Set-up: this entry point's first call on a device, made with that device
 * current, looks up the array's device address (and, like every entry point's
 * first call, queries the device); make that first call before any stream
 * capture.
 * Shared state: every call uses the same array, which keeps the last call's
 * contents. Nothing has to start at zero (the mixing kernel writes every
 * element the convolution reads), but two calls whose kernels overlap on the
 * GPU (different streams or host threads without ordering) race on the array:
 * order them (same stream, or events).
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * Errors: INVALID_ARG, UNSUPPORTED, WORKSPACE, MISALIGNED, CUDA. */
#define DYNCONV_NOALLOC_MAX_BYTES (32u * 1024u * 1024u)
int dynconv_forward_noalloc(const dynconv_desc* desc, const void* x, const void* experts,
                            const float* alpha, const float* bias, void* y, void* stream);

/* Bytes of workspace the PREMIX variant needs for this descriptor (0 if it
 * cannot run this shape). Pure host function. */
size_t dynconv_workspace_size(const dynconv_desc* desc);

/* The variant AUTO resolves to for this descriptor and workspace size
 * (a dynconv_variant value), or a negative status. Pure host function. */
int dynconv_select_variant(const dynconv_desc* desc, size_t workspace_bytes);

/* ---- status and diagnostics ------------------------------------------------ */

/* Static, human-readable text for a status code (never NULL). */
const char* dynconv_status_string(int status);

/* Text of the last CUDA error this thread saw inside the library (static
 * storage, overwritten by the next error), or "" if none. */
const char* dynconv_last_error(void);

/* Synchronise `stream`, then read and clear this device's error word, which
 * kernels set when a bounded wait on a barrier expires (they then skip the
 * rest of their work and exit cleanly, leaving y unspecified). Returns
 * DYNCONV_OK, DYNCONV_ERR_TIMEOUT, or DYNCONV_ERR_CUDA. */
int dynconv_device_status(void* stream);

/* Number of kernel launches the library has issued in this process. */
unsigned long long dynconv_launch_count(void);

/* Test hook. key 1: bounded-wait limit in microseconds for subsequent launches
 * (0 restores the default of 500000). key 2: when nonzero, the next forward
 * launch of a tensor-core variant withholds one producer arrival, so that its
 * consumer's bounded wait must expire and report DYNCONV_ERR_TIMEOUT.
 * key 3: tensor-core descriptor base-offset mode for shifted activation views
 * (0, the default and the correct choice on B200: left zero; 1: the swizzle
 * phase (address >> 7) & 7 is written into the descriptor, which gives wrong
 * results). Only for re-verifying that choice on a device.
 * key 4: CTAs per sample of the routing kernel's cluster (1..8; 0 restores
 * the automatic choice), for tuning measurements.
 * key 5: 1 (default) launches the forward kernels with a programmatic
 * stream-serialization edge (they may start while the previous kernel on the
 * stream finishes, and wait for it before reading memory); 0 launches them
 * plainly. For measurements.
 * key 6: 1 runs PREMIX with n <= 8 as one persistent cooperative kernel that
 * streams the mixing into the convolution (per-K-slice counters); 0 (default)
 * runs it as two kernels (mixing, then convolution). The counters live in a
 * few fixed slots per device, one per stream for the life of the process;
 * calls on further streams run the two-kernel form.
 * key 7: which kernel mixes the per-sample kernels of the two-kernel PREMIX
 * form: 0 (default) the CUDA-core mixer when n <= 8, else the tensor-core
 * GEMM with M = samples; 1 always that GEMM (and never the streamed kernel of
 * key 6); 2 the CUDA-core mixer only (forward returns
 * DYNCONV_ERR_UNSUPPORTED when n > 8); 3 the transposed GEMM (M = weights,
 * N = samples) for batches of at most 256. The tensor-core mixers take no
 * input attention.
 * key 8: which kernel runs DEPTHWISE: 0 (default) the pipelined kernel
 * (persistent CTAs, resident expert slabs, TMA-fed ring of input tiles) when
 * the shape fits it, else the per-tile kernel; 1 always the per-tile kernel;
 * 2 / 3 the pipelined kernel with 2 / 4 output columns per thread.
 * key 9: the convolution of PREMIX: 1 (default) the persistent kernel (one
 * CTA per SM, two TMEM accumulators, the epilogue of one unit overlapping the
 * next unit's MMAs) where it pays (three or more units per CTA, or at most
 * four K steps per unit), no pooled sums are asked for and the shape fits it;
 * 2 the persistent kernel whenever it fits; 0 always one CTA per unit.
 * key 10: PREMIX with n > 8 when every sample's mixed kernel together is much
 * larger than the L2: 0 (default) mixes every sample's kernel first, then
 * convolves; 1 mixes and convolves one group (of samples, or of 128-channel
 * tiles) at a time through two workspace slots, the mixing of the next group
 * on an internal stream overlapping the convolution of the current one; 2
 * does the same in sequence on the caller's stream through one slot (each
 * group's mixed kernels read back from L2). A value of 4096 or more turns
 * form 1 on for every size, and a value of -4096 or less form 2, with groups
 * of about |value| bytes (for tests of ragged groups and for tuning).
 * key 11: the backward's mixing gradient: 1 (default) the tensor-core kernel
 * (per-sample weight gradients as bf16 hi / lo planes, one pass for the
 * expert and attention gradients) when it applies; 0 the CUDA-core kernel.
 * key 12: the epilogue of the tensor-core mixing GEMM: 0 (default) stages
 * each tile through shared memory and writes whole rows; 1 stores each
 * thread's 32 mixed weights straight from registers (two 32-byte stores) when
 * the kernel size is a multiple of 16 and the workspace 32-byte aligned
 * (measured slower on B200). For measurements.
 * key 13: the address of a device buffer of 64-bit words (0, the default:
 * off). While it is set, the routing kernel (CTA rank r of sample b at
 * [(b * ranks + r) * 8]), the pipelined depthwise kernel and the CUDA-core
 * mixing kernel (at [(4096 + block) * 8]) record their phase times (the
 * layouts are described at the kernels), and each CTA of
 * the PREMIX, FUSED and OUTSIDE tensor-core convolutions writes 8 words at
 * [block * 8]: its SM cycle
 * counter at entry, past the grid wait, when the first operands are in
 * shared memory, after the MMA issue of the (one-CTA-per-unit kernel: only;
 * persistent kernel: first) unit, when the accumulator is complete
 * (persistent kernel: after the last unit's MMA issue) and when every
 * epilogue is done; its SM id; and the global timer at entry. The buffer
 * must hold 8 words per CTA of every such launch made meanwhile. For
 * measurements.
 * key 14: output rows per unit of the persistent PREMIX convolution: 0
 * (default) as planned; 1..256 that many (capped at the layer's height)
 * when such a unit fits, else the convolution falls back to one CTA per
 * unit. For measurements.
 * key 18: how the tensor-core mixing GEMM of a one-pass PREMIX forward hands
 * out its tiles: from a counter in the workspace (zeroed on the stream before
 * the launch), each CTA taking the next tile, so that CTAs whose expert tiles
 * arrive faster take more -- 1 (default) when the expert bank is larger than
 * half the L2, 2 always, 0 never (statically: tile c + j * grid to CTA c).
 * Same results either way.
 * Returns DYNCONV_OK or DYNCONV_ERR_INVALID_ARG. */
int dynconv_test_hook(int key, long long value);

#ifdef __cplusplus
}
#endif
#endif /* DYNCONV_H */
