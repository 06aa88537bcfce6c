/*
 * Kernel cells shared through a warehouse (sm_100a).
 *
 * KernelWarehouse: Rethinking the Design of Dynamic Convolution (abstract)
 * redefines the kernel, its assembly and the attention function so that the
 * number of mixed parts can exceed 100, sharing parameters within a layer and
 * across neighbouring layers; the page gives no formula. Reading taken here:
 *
 *   the layer's kernel, flattened in the layout [C_out][KH][KW][C_in/groups]
 *   (|W| elements), is split into m = `cells` contiguous cells of s = |W| / m
 *   elements; a warehouse holds n cells E[n][s] (desc->n = n; one warehouse
 *   may serve every layer whose cell size is s); each kernel cell j of sample
 *   b is its own attention-weighted mixture
 *       W_b[j*s + e] = sum_i alpha[b][j][i] * E[i][e];
 *   the attentions come from the same router as dynconv_route, with m*n
 *   outputs, the activation taken per cell (softmax over the n values of a
 *   cell with temperature tau, or an elementwise sigmoid);
 *   y_b = conv2d(x_b, W_b) + bias (bias static, [C_out], not mixed; or none).
 *
 * With m = 1 this is dynconv_route + dynconv_forward with the warehouse as the
 * n experts and no bias. Forward only: no backward for cells.
 *
 * Layouts as in dynconv.h; warehouse [n][s] in desc->dtype; alpha fp32
 * [B][m][n]; Wr fp32 [m*n][C_in], br fp32 [m*n] or NULL; bias fp32 [C_out] or
 * NULL. All pointers are device pointers owned by the caller; calls enqueue on
 * `stream` and return; nothing is allocated. Errors are the dynconv status
 * codes; nothing is launched when a call returns INVALID_ARG, UNSUPPORTED,
 * MISALIGNED or WORKSPACE.
 */
#ifndef DYNCONV_CELLS_H
#define DYNCONV_CELLS_H

#include "dynconv.h"

#ifdef __cplusplus
extern "C" {
#endif

/* alpha[B][m][n] for m = cells, n = desc->n: the average pool (fp32, pixel
 * slices summed into the workspace, then added in order), the linear layer
 * (eight outputs per warp at a time, fixed-order sums) and the activation per
 * cell (softmax: the cell's maximum subtracted), two cells per CTA.
 *   workspace, workspace_bytes: at least dynconv_cells_workspace_size(desc,
 *   cells) bytes, 256-byte aligned (the same buffer as the forward call's).
 * Errors: INVALID_ARG (NULL pointers, cells < 1, bad mode or tau),
 * UNSUPPORTED (m*n > 4096 or C_in > 16384), WORKSPACE, MISALIGNED, CUDA. */
int dynconv_route_cells(const dynconv_desc* desc, int cells, const void* x, const float* Wr,
                        const float* br, int mode, float tau, float* alpha, void* workspace,
                        size_t workspace_bytes, void* stream);

/* Workspace bytes of dynconv_route_cells and dynconv_forward_cells for this
 * descriptor and cell count (one buffer serves both; 0 if the shape is not
 * taken). Pure host function. */
size_t dynconv_cells_workspace_size(const dynconv_desc* desc, int cells);

/* y for the layer in `desc` (desc->n = warehouse cells n <= 1024) with the
 * kernel assembled from `cells` cells. A CUDA-core kernel writes every
 * sample's W_b (rounded once to desc->dtype) into the workspace; the
 * convolution then runs on the forward kernels (dynconv_forward) with the B
 * per-sample kernels as B experts and one-hot attentions, which reproduces
 * each W_b exactly, in chunks of at most 64 samples: the PREMIX variant where
 * the shape allows it, else DEPTHWISE, else DIRECT (desc->variant is ignored).
 * Requires |W| % cells == 0 and s a multiple of 16 bytes' worth of elements
 * (8 for bf16, 4 for fp32), 16-byte aligned warehouse.
 * Errors: INVALID_ARG, UNSUPPORTED, MISALIGNED, WORKSPACE, CUDA. */
int dynconv_forward_cells(const dynconv_desc* desc, int cells, const void* x,
                          const void* warehouse, const float* alpha, const float* bias, void* y,
                          void* workspace, size_t workspace_bytes, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* DYNCONV_CELLS_H */
