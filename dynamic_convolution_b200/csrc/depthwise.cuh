// CUDA-core depthwise dynamic convolution (groups == C_in == C_out), bf16 in /
// out, fp32 mixing and accumulation, stride 1, square K in {3, 5, 7}.
//
// y_b[c] = sum_{kh,kw} x_b[oh+kh-p, ow+kw-p, c] * W_b[c,kh,kw] + b_b[c] with
// W_b = sum_i alpha_{b,i} W_i (the linear kernel mixture of KernelWarehouse,
// abstract; per-example kernels of CondConv, abstract).
//
// The layer is memory-bound with an ALU floor close to the HBM floor, so the
// kernel is built to touch each input byte once from HBM and keep the FMA pipe
// fed:
//  * one CTA per (sample, block of kRows output rows, 32-channel chunk, column
//    block); the zero-padded input window (rows + halo) is staged in shared
//    memory with 16-byte vector loads, so padding costs no branches later;
//  * the CTA mixes its 32 channels' K*K weights and biases once (fp32);
//  * each thread owns one channel pair (bf16x2) and one output column, keeps
//    its 2*K*K weights in registers, and walks down the kRows output rows with
//    a K-row register window (K new values per row);
//  * consecutive threads take consecutive channel pairs, so shared-memory reads
//    are conflict-free and the NHWC stores coalesce.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kDwChunk = 32;       // channels per CTA
constexpr int kDwPairs = kDwChunk / 2;
constexpr int kDwRows = 7;         // output rows per CTA
constexpr int kDwMaxCols = 32;     // output columns per CTA

struct DwParams {
  int B, C, H, W, pad, n, Ho, Wo;
  int tile_cols;                   // output columns per CTA (<= kDwMaxCols)
  const __nv_bfloat16* x;
  const __nv_bfloat16* experts;    // [n][C][K][K][1]
  const float* alpha;
  const float* bias;               // may be null
  __nv_bfloat16* y;
};

template <int K>
__global__ void __launch_bounds__(kDwPairs * kDwMaxCols) depthwise_kernel(DwParams p) {
  constexpr int KK = K * K;
  constexpr int TR = kDwRows + K - 1;             // staged input rows
  const int TC = p.tile_cols + K - 1;             // staged input columns
  const int b = blockIdx.z;
  const int c0 = blockIdx.y * kDwChunk;
  const int nrow_blocks = (p.Ho + kDwRows - 1) / kDwRows;
  const int oh0 = (blockIdx.x % nrow_blocks) * kDwRows;
  const int ow0 = (blockIdx.x / nrow_blocks) * p.tile_cols;
  const int t = threadIdx.x;
  const int nthreads = blockDim.x;

  extern __shared__ __align__(16) unsigned char dw_smem[];
  float* w_s = reinterpret_cast<float*>(dw_smem);              // [kDwChunk][KK]
  float* bias_s = w_s + kDwChunk * KK;                          // [kDwChunk]
  float* alpha_s = bias_s + kDwChunk;                           // [n]
  uint32_t* tile = reinterpret_cast<uint32_t*>(alpha_s + ((p.n + 3) & ~3));  // [TR][TC][kDwPairs]

  for (int i = t; i < p.n; i += nthreads) alpha_s[i] = p.alpha[static_cast<size_t>(b) * p.n + i];

  // stage the zero-padded input window: 4 x 16-byte vectors per pixel (32 channels)
  const __nv_bfloat16* xb = p.x + static_cast<size_t>(b) * p.H * p.W * p.C;
  const int nvec = TR * TC * (kDwChunk / 8);
  for (int v = t; v < nvec; v += nthreads) {
    const int q = v & 3;
    const int pix = v >> 2;
    const int r = pix / TC, cc = pix % TC;
    const int ih = oh0 + r - p.pad, iw = ow0 + cc - p.pad;
    const int ch = c0 + q * 8;
    uint4 val = make_uint4(0u, 0u, 0u, 0u);
    if (ih >= 0 && ih < p.H && iw >= 0 && iw < p.W && ch < p.C)
      val = ld_nc_v4(xb + (static_cast<size_t>(ih) * p.W + iw) * p.C + ch);
    *reinterpret_cast<uint4*>(tile + (static_cast<size_t>(r) * TC + cc) * kDwPairs + q * 4) = val;
  }
  __syncthreads();

  // mix this chunk's kernels and biases (fp32)
  for (int e = t; e < kDwChunk * KK; e += nthreads) {
    const int cl = e / KK, k = e % KK;
    const int c = c0 + cl;
    float s = 0.f;
    if (c < p.C)
      for (int i = 0; i < p.n; ++i)
        s = fmaf(alpha_s[i],
                 __bfloat162float(p.experts[(static_cast<size_t>(i) * p.C + c) * KK + k]), s);
    w_s[e] = s;
  }
  for (int cl = t; cl < kDwChunk; cl += nthreads) {
    float s = 0.f;
    const int c = c0 + cl;
    if (p.bias && c < p.C)
      for (int i = 0; i < p.n; ++i) s = fmaf(alpha_s[i], p.bias[static_cast<size_t>(i) * p.C + c], s);
    bias_s[cl] = s;
  }
  __syncthreads();

  const int cp = t % kDwPairs;     // channel pair within the chunk
  const int col = t / kDwPairs;    // output column within the tile
  const int c = c0 + 2 * cp;
  const int ow = ow0 + col;
  if (col >= p.tile_cols || ow >= p.Wo || c >= p.C) return;

  float w0[KK], w1[KK];
#pragma unroll
  for (int k = 0; k < KK; ++k) {
    w0[k] = w_s[(2 * cp) * KK + k];
    w1[k] = w_s[(2 * cp + 1) * KK + k];
  }
  const float bias0 = bias_s[2 * cp], bias1 = bias_s[2 * cp + 1];

  // K-row register window of the input columns col .. col+K-1
  float win0[K][K], win1[K][K];
#pragma unroll
  for (int r = 0; r < K - 1; ++r)
#pragma unroll
    for (int kw = 0; kw < K; ++kw) {
      const uint32_t v = tile[(static_cast<size_t>(r) * TC + col + kw) * kDwPairs + cp];
      win0[r + 1][kw] = bf16lo_to_f32(v);
      win1[r + 1][kw] = bf16hi_to_f32(v);
    }

  __nv_bfloat16* yb = p.y + static_cast<size_t>(b) * p.Ho * p.Wo * p.C;
#pragma unroll
  for (int orow = 0; orow < kDwRows; ++orow) {
    // slide: drop the top row, load input row orow+K-1
#pragma unroll
    for (int r = 0; r < K - 1; ++r)
#pragma unroll
      for (int kw = 0; kw < K; ++kw) {
        win0[r][kw] = win0[r + 1][kw];
        win1[r][kw] = win1[r + 1][kw];
      }
#pragma unroll
    for (int kw = 0; kw < K; ++kw) {
      const uint32_t v =
          tile[(static_cast<size_t>(orow + K - 1) * TC + col + kw) * kDwPairs + cp];
      win0[K - 1][kw] = bf16lo_to_f32(v);
      win1[K - 1][kw] = bf16hi_to_f32(v);
    }
    // two partial sums per channel for more independent FMA chains
    float a0 = bias0, a1 = bias1, e0 = 0.f, e1 = 0.f;
#pragma unroll
    for (int kh = 0; kh < K; ++kh)
#pragma unroll
      for (int kw = 0; kw < K; ++kw) {
        if (kh & 1) {
          e0 = fmaf(win0[kh][kw], w0[kh * K + kw], e0);
          e1 = fmaf(win1[kh][kw], w1[kh * K + kw], e1);
        } else {
          a0 = fmaf(win0[kh][kw], w0[kh * K + kw], a0);
          a1 = fmaf(win1[kh][kw], w1[kh * K + kw], a1);
        }
      }
    const int oh = oh0 + orow;
    if (oh < p.Ho)
      *reinterpret_cast<uint32_t*>(yb + (static_cast<size_t>(oh) * p.Wo + ow) * p.C + c) =
          pack_bf16x2(a0 + e0, a1 + e1);
  }
}

}  // namespace dc
