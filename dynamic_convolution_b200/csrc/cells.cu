// Host side of the warehouse-cell entry points declared in
// include/dynconv_cells.h: argument checks, workspace layout, launches of the
// cell kernels, and the convolution through the forward entry point with the
// per-sample kernels as experts under one-hot attentions. A translation unit
// of its own (device state and error reporting through internal.h).
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>

#include "dynconv.h"
#include "dynconv_cells.h"
#include "internal.h"

#include "cells_kernels.cuh"

namespace {

constexpr int kChunk = 64;      // samples per convolution call (one-hot attentions kChunk^2)
constexpr int kMixSamples = 8;  // samples per CTA of the cell mixing

int out_size(int in, int k, int stride, int pad) { return (in + 2 * pad - k) / stride + 1; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
size_t elem_bytes(const dynconv_desc* d) { return d->dtype == DYNCONV_F32 ? 4 : 2; }
long long wsize_of(const dynconv_desc* d) {
  return 1LL * d->C_out * d->KH * d->KW * (d->C_in / d->groups);
}

// The forward call for one chunk of bc samples: bc experts (the chunk's
// kernels) under one-hot attentions.
dynconv_desc chunk_desc(const dynconv_desc* d, int bc, int variant) {
  dynconv_desc c = *d;
  c.B = bc;
  c.n = bc;
  c.variant = variant;
  return c;
}

bool depthwise_shape(const dynconv_desc* d) {
  return d->dtype == DYNCONV_BF16 && d->groups == d->C_in && d->C_in == d->C_out &&
         d->stride == 1 && d->KH == d->KW && (d->KH == 3 || d->KH == 5 || d->KH == 7) &&
         d->C_in % 8 == 0;
}

// PREMIX when the forward takes it for every chunk size used, else
// DEPTHWISE for depthwise shapes, else DIRECT.
int conv_variant(const dynconv_desc* d) {
  const int bc = std::min(d->B, kChunk), bt = d->B % kChunk;
  dynconv_desc c = chunk_desc(d, bc, DYNCONV_VARIANT_PREMIX);
  bool premix = dynconv_workspace_size(&c) != 0;
  if (premix && bt != 0 && bt != bc) {
    c = chunk_desc(d, bt, DYNCONV_VARIANT_PREMIX);
    premix = dynconv_workspace_size(&c) != 0;
  }
  if (premix) return DYNCONV_VARIANT_PREMIX;
  return depthwise_shape(d) ? DYNCONV_VARIANT_DEPTHWISE : DYNCONV_VARIANT_DIRECT;
}

// Pixel slices of the routing's average pool: about four CTAs per SM in all
// (for at most 160 SMs), at least 32 pixels per slice.
int pool_slices(int B, int HW) {
  const int want = std::max(1, (4 * 160 + B - 1) / std::max(B, 1));
  return std::max(1, std::min(want, HW / 32));
}
size_t pool_bytes(const dynconv_desc* d) {
  return align256(4ull * d->B * d->C_in * pool_slices(d->B, d->H * d->W));
}

struct CellsLayout {
  size_t wb = 0, ident = 0, ident_tail = 0, bias_rows = 0, conv = 0, total = 0;
};

bool cells_shape_ok(const dynconv_desc* d, int cells) {
  const long long ws = wsize_of(d);
  if (cells < 1 || ws % cells != 0) return false;
  const long long s = ws / cells;
  const int vec = d->dtype == DYNCONV_F32 ? 4 : 8;
  return s % vec == 0 && d->n <= 1024;
}

CellsLayout cells_layout(const dynconv_desc* d, int cells) {
  CellsLayout L;
  const int bc = std::min(d->B, kChunk);
  L.wb = 0;
  L.ident = align256(L.wb + static_cast<size_t>(d->B) * wsize_of(d) * elem_bytes(d));
  L.ident_tail = align256(L.ident + 4ull * bc * bc);
  L.bias_rows = align256(L.ident_tail + 4ull * bc * bc);
  L.conv = align256(L.bias_rows + 4ull * bc * d->C_out);
  size_t conv = 0;
  if (conv_variant(d) == DYNCONV_VARIANT_PREMIX) {
    dynconv_desc c = chunk_desc(d, bc, DYNCONV_VARIANT_PREMIX);
    conv = dynconv_workspace_size(&c);
  }
  L.total = std::max(align256(L.conv + conv), pool_bytes(d));
  (void)cells;
  return L;
}

template <typename T>
int launch_mix(const dcc::CmParams& p, int vec, size_t smem, cudaStream_t s) {
  const dim3 grid(static_cast<unsigned>((p.s / vec + dcc::kCellThreads - 1) / dcc::kCellThreads),
                  p.m, (p.B + kMixSamples - 1) / kMixSamples);
  auto kern = dcc::cells_mix_kernel<T, kMixSamples>;
  if (smem > 48 * 1024) {
    cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(kern), smem);
    if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(cells_mix)");
  }
  kern<<<grid, dcc::kCellThreads, smem, s>>>(p);
  return dc_lib::launched("cells_mix_kernel");
}

}  // namespace

extern "C" {

int dynconv_route_cells(const dynconv_desc* desc, int cells, const void* x, const float* Wr,
                        const float* br, int mode, float tau, float* alpha, void* workspace,
                        size_t workspace_bytes, void* stream) {
  int rc = dc_lib::validate(desc);
  if (rc) return rc;
  if (!x || !Wr || !alpha || cells < 1) return DYNCONV_ERR_INVALID_ARG;
  if (mode != DYNCONV_SIGMOID && mode != DYNCONV_SOFTMAX) return DYNCONV_ERR_INVALID_ARG;
  if (mode == DYNCONV_SOFTMAX && !(tau > 0.f)) return DYNCONV_ERR_INVALID_ARG;
  if (1LL * cells * desc->n > 4096 || desc->C_in > 16384) return DYNCONV_ERR_UNSUPPORTED;
  if (desc->B == 0) return DYNCONV_OK;
  const int HW = desc->H * desc->W;
  const int S = pool_slices(desc->B, HW);
  if (!workspace || workspace_bytes < pool_bytes(desc)) return DYNCONV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNCONV_ERR_MISALIGNED;
  dc_lib::DeviceInfo di;
  rc = dc_lib::device_info(&di);
  if (rc) return rc;
  const size_t smem = sizeof(float) * (static_cast<size_t>(desc->C_in) +
                                       static_cast<size_t>(dcc::kCellsPerCta) * desc->n);
  if (smem > static_cast<size_t>(di.max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  float* part = static_cast<float*>(workspace);
  const int Ps = (HW + S - 1) / S;
  if (desc->dtype == DYNCONV_F32)
    dcc::cells_pool_kernel<float><<<dim3(S, desc->B), dcc::kCellThreads, 0, s>>>(
        desc->C_in, HW, Ps, static_cast<const float*>(x), part);
  else
    dcc::cells_pool_kernel<__nv_bfloat16><<<dim3(S, desc->B), dcc::kCellThreads, 0, s>>>(
        desc->C_in, HW, Ps, static_cast<const __nv_bfloat16*>(x), part);
  rc = dc_lib::launched("cells_pool_kernel");
  if (rc) return rc;
  if (smem > 48 * 1024) {
    cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(dcc::route_cells_kernel), smem);
    if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(route_cells)");
  }
  dcc::route_cells_kernel<<<dim3((cells + dcc::kCellsPerCta - 1) / dcc::kCellsPerCta, desc->B),
                            dcc::kCellThreads, smem, s>>>(desc->C_in, HW, S, cells, desc->n, mode,
                                                          tau, part, Wr, br, alpha);
  return dc_lib::launched("route_cells_kernel");
}

size_t dynconv_cells_workspace_size(const dynconv_desc* desc, int cells) {
  if (dc_lib::validate(desc) != DYNCONV_OK || !cells_shape_ok(desc, cells)) return 0;
  return cells_layout(desc, cells).total;
}

int dynconv_forward_cells(const dynconv_desc* desc, int cells, const void* x,
                          const void* warehouse, const float* alpha, const float* bias, void* y,
                          void* workspace, size_t workspace_bytes, void* stream) {
  int rc = dc_lib::validate(desc);
  if (rc) return rc;
  if (!x || !warehouse || !alpha || !y || cells < 1) return DYNCONV_ERR_INVALID_ARG;
  if (!cells_shape_ok(desc, cells)) return DYNCONV_ERR_UNSUPPORTED;
  if (desc->B == 0) return DYNCONV_OK;
  if (!aligned16(warehouse)) return DYNCONV_ERR_MISALIGNED;
  const CellsLayout L = cells_layout(desc, cells);
  if (!workspace || workspace_bytes < L.total) return DYNCONV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNCONV_ERR_MISALIGNED;
  const int variant = conv_variant(desc);
  if (variant == DYNCONV_VARIANT_PREMIX && (!aligned16(x) || !aligned16(y)))
    return DYNCONV_ERR_MISALIGNED;
  dc_lib::DeviceInfo di;
  rc = dc_lib::device_info(&di);
  if (rc) return rc;
  const size_t mix_smem = sizeof(float) * kMixSamples * static_cast<size_t>(desc->n);  // [n][SB]
  if (mix_smem > static_cast<size_t>(di.max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* wsb = static_cast<char*>(workspace);
  const long long ws = wsize_of(desc);

  // 1. every sample's kernel from the warehouse cells
  dcc::CmParams p{};
  p.B = desc->B; p.m = cells; p.n = desc->n; p.s = ws / cells; p.wsize = ws;
  p.E = warehouse; p.alpha = alpha; p.Wb = wsb + L.wb;
  rc = desc->dtype == DYNCONV_F32 ? launch_mix<float>(p, 4, mix_smem, s)
                                  : launch_mix<__nv_bfloat16>(p, 8, mix_smem, s);
  if (rc) return rc;
  // 2. one-hot attentions (full chunk and tail) and per-sample bias rows
  const int bc = std::min(desc->B, kChunk), bt = desc->B % kChunk;
  float* ident = reinterpret_cast<float*>(wsb + L.ident);
  float* ident_tail = reinterpret_cast<float*>(wsb + L.ident_tail);
  float* bias_rows = reinterpret_cast<float*>(wsb + L.bias_rows);
  const int t1 = std::max(bc * bc, bias ? bc * desc->C_out : 0);
  dcc::onehot_kernel<<<(t1 + dcc::kCellThreads - 1) / dcc::kCellThreads, dcc::kCellThreads, 0, s>>>(
      bc, ident, bias, desc->C_out, bc, bias_rows);
  rc = dc_lib::launched("onehot_kernel");
  if (rc) return rc;
  if (bt != 0 && bt != bc) {
    dcc::onehot_kernel<<<(bt * bt + dcc::kCellThreads - 1) / dcc::kCellThreads, dcc::kCellThreads,
                         0, s>>>(bt, ident_tail, nullptr, desc->C_out, 0, nullptr);
    rc = dc_lib::launched("onehot_kernel");
    if (rc) return rc;
  }
  // 3. the convolution, chunk by chunk, through the forward entry point
  const int Ho = out_size(desc->H, desc->KH, desc->stride, desc->pad);
  const int Wo = out_size(desc->W, desc->KW, desc->stride, desc->pad);
  const size_t xs = static_cast<size_t>(desc->H) * desc->W * desc->C_in * elem_bytes(desc);
  const size_t ys = static_cast<size_t>(Ho) * Wo * desc->C_out * elem_bytes(desc);
  const size_t wbs = static_cast<size_t>(ws) * elem_bytes(desc);
  for (int b0 = 0; b0 < desc->B; b0 += kChunk) {
    const int n_here = std::min(kChunk, desc->B - b0);
    const dynconv_desc c = chunk_desc(desc, n_here, variant);
    rc = dynconv_forward(&c, static_cast<const char*>(x) + b0 * xs, wsb + L.wb + b0 * wbs,
                         n_here == bc ? ident : ident_tail, bias ? bias_rows : nullptr,
                         static_cast<char*>(y) + b0 * ys,
                         workspace_bytes > L.conv ? wsb + L.conv : nullptr,
                         workspace_bytes - L.conv, stream);
    if (rc) return rc;
  }
  return DYNCONV_OK;
}

}  // extern "C"
