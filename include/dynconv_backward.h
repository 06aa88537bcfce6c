/*
 * Backward pass of the per-sample kernel-mixture convolution (sm_100a).
 *
 * The per-example kernels and their mixture are learned (CondConv:
 * Conditionally Parameterized Convolutions for Efficient Inference, abstract;
 * KernelWarehouse: Rethinking the Design of Dynamic Convolution, abstract), so
 * a training step needs the gradients of the forward definition in
 * dynconv.h. Given dy = dL/dy of a scalar loss L, with
 * g[b][c] = GAP(x_b)[c], z = Wr g + br, alpha = act(z),
 * W_b = sum_i alpha[b][i] W_i, b_b = sum_i alpha[b][i] bias_i:
 *
 *   dW_b[co][kh][kw][ci] = sum over output pixels of dy * (the input element the
 *                          forward multiplied with W_b[co][kh][kw][ci])
 *   db_b[co]             = sum over output pixels of dy[b][.][.][co]
 *   dexperts_i           = sum_b alpha[b][i] dW_b         dbias_i = sum_b alpha[b][i] db_b
 *   dalpha[b][i]         = <dW_b, W_i> + <db_b, bias_i>
 *   dz                   = dalpha * alpha * (1 - alpha)                      (sigmoid)
 *                          alpha * (dalpha - sum_j alpha_j dalpha_j) / tau   (softmax of z/tau)
 *   dWr[i][c] = sum_b dz[b][i] g[b][c]    dbr[i] = sum_b dz[b][i]    dg[b][c] = sum_i dz[b][i] Wr[i][c]
 *   dx[b][h][w][ci]      = the convolution's input gradient with W_b
 *                          + dg[b][ci] / (H*W)  on every pixel
 *
 * Three calls, in this order for a full step (each enqueues on `stream` and
 * returns at once; nothing is allocated):
 *   dynconv_backward_weight  dexperts, dbias, dalpha
 *   dynconv_route_backward   dWr, dbr, dg          (needs dalpha)
 *   dynconv_backward_data    dx                    (needs dg)
 * A layer with attentions from elsewhere (not this router) skips the middle
 * call and passes dg = NULL.
 *
 * Layouts are those of dynconv.h: x NHWC [B][H][W][C_in] and dy NHWC
 * [B][H_out][W_out][C_out] in desc->dtype; experts [n][C_out][KH][KW][C_in/groups]
 * in desc->dtype; alpha, bias, Wr as in dynconv.h (fp32). Every gradient is
 * fp32 and in the layout of the value it belongs to, except dx, which is in
 * desc->dtype, rounded once: dg/(H*W) is added to the convolution's input
 * gradient in fp32 before the rounding, on the forward kernels (through their
 * epilogue's per-channel term) and on the generic kernel alike. Outputs are
 * overwritten, not accumulated.
 * All results are deterministic (no floating-point atomics).
 *
 * Ownership: the caller allocates every buffer (device memory) and the
 * workspace; the library keeps no pointer after the call's kernels finish.
 * Errors: negative dynconv status codes; nothing is launched when a call
 * returns INVALID_ARG, UNSUPPORTED, MISALIGNED or WORKSPACE. A bounded wait
 * that expires inside a kernel is reported by dynconv_device_status.
 */
#ifndef DYNCONV_BACKWARD_H
#define DYNCONV_BACKWARD_H

#include "dynconv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* Bytes of device workspace that the three backward calls need for this
 * descriptor (one buffer serves all three, in turn; 0 on an invalid
 * descriptor). Pure host function. */
size_t dynconv_backward_workspace_size(const dynconv_desc* desc);

/* Gradients of the experts, their biases and the attentions.
 *   x        input of the forward, desc->dtype, NHWC
 *   dy       dL/dy, desc->dtype, NHWC [B][H_out][W_out][C_out]
 *   experts  the n kernels, desc->dtype
 *   alpha    fp32 [B][n], the attentions the forward used
 *   bias     fp32 [n][C_out] or NULL (no bias: dbias must be NULL, and
 *            dalpha has no bias term)
 *   dexperts fp32 [n][C_out][KH][KW][C_in/groups]  (out)
 *   dbias    fp32 [n][C_out] or NULL               (out)
 *   dalpha   fp32 [B][n]                           (out)
 *   workspace, workspace_bytes: at least dynconv_backward_workspace_size(desc)
 *            bytes, 256-byte aligned; contents need not be preserved.
 * The per-sample gradients dW_b are computed by the tcgen05 weight-gradient
 * kernel when desc->variant is AUTO or a tensor-core variant and the shape
 * allows it (bf16, groups 1, stride 1, C_in and C_out multiples of 8,
 * W_out <= 128); else, for a bf16 depthwise layer (groups = C_in = C_out,
 * stride 1, square 3x3, 5x5 or 7x7, C_in a multiple of 8), by the depthwise
 * CUDA-core kernel (desc->variant DEPTHWISE forces it); else by the generic
 * CUDA-core kernel (desc->variant DIRECT forces it). A forced variant on a
 * shape its kernel does not take returns UNSUPPORTED.
 * Errors: INVALID_ARG (NULL pointer, bias/dbias mismatch, bad descriptor),
 * UNSUPPORTED, MISALIGNED (x, dy or workspace not 16-byte aligned on the
 * tensor-core path), WORKSPACE, CUDA. */
int dynconv_backward_weight(const dynconv_desc* desc, const void* x, const void* dy,
                            const void* experts, const float* alpha, const float* bias,
                            float* dexperts, float* dbias, float* dalpha, void* workspace,
                            size_t workspace_bytes, void* stream);

/* Gradients of the router (the linear layer on the average pool) and of the
 * pooled vector.
 *   x        input of the forward (its average pool g is taken again here)
 *   Wr       fp32 [n][C_in]
 *   alpha    fp32 [B][n], dalpha fp32 [B][n] (from dynconv_backward_weight)
 *   mode, tau: as in dynconv_route
 *   dWr fp32 [n][C_in], dbr fp32 [n], dg fp32 [B][C_in]  (out; dbr may be NULL)
 *   workspace, workspace_bytes: as for dynconv_backward_weight (the same
 *            buffer serves all three calls); may be NULL, the channel sums of
 *            x then run with less parallelism.
 * dg is also used as scratch for the channel sums of x.
 * Errors: INVALID_ARG (NULL pointers, bad mode or tau), UNSUPPORTED
 * (n > 1024), CUDA. */
int dynconv_route_backward(const dynconv_desc* desc, const void* x, const float* Wr,
                           const float* alpha, const float* dalpha, int mode, float tau,
                           float* dWr, float* dbr, float* dg, void* workspace,
                           size_t workspace_bytes, void* stream);

/* Gradient of the layer's input.
 *   dy, experts, alpha: as for dynconv_backward_weight
 *   dg       fp32 [B][C_in] from dynconv_route_backward, or NULL (attentions
 *            that do not depend on x)
 *   dx       desc->dtype NHWC [B][H][W][C_in]  (out)
 * With stride 1 and KH - 1 - pad = KW - 1 - pad >= 0, the input gradient is a
 * convolution of dy with every expert transposed (input and output channels
 * swapped within each group) and flipped in both spatial axes, padding
 * KH - 1 - pad, mixed with the same attentions: it runs on the forward
 * kernels (desc->variant chooses among them as in dynconv_forward, for that
 * transposed shape), after a kernel writes the transposed experts into the
 * workspace. Other shapes run a CUDA-core kernel. dg/(H*W) is then added in
 * place.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA, and those of
 * dynconv_forward for the transposed shape; an error of that forward call (a
 * forced variant that cannot take the transposed shape) comes after the
 * transposition kernel has run: dx is then not written. */
int dynconv_backward_data(const dynconv_desc* desc, const void* dy, const void* experts,
                          const float* alpha, const float* dg, void* dx, void* workspace,
                          size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DYNCONV_BACKWARD_H */
