// CUDA-core direct convolution with the per-sample mixed kernel, fp32
// accumulation. Any kernel size, stride, padding and group count. This is the
// fp32 path and the path for bf16 shapes the tensor-core kernels do not take.
//
// y_b = conv2d(x_b, sum_i alpha_{b,i} W_i) + sum_i alpha_{b,i} bias_i: the mixed
// kernel, a weighted sum of n static kernels (KernelWarehouse, abstract),
// applied per example (CondConv, abstract); cross-correlation with zero
// padding is the reading taken.
//
// One CTA per (pixel block, output-channel block, sample). The CTA first mixes
// its slab of W_b (fp32) and the mixed bias into shared memory, then each
// thread produces (pixel, channel) outputs; consecutive threads take
// consecutive output channels so the NHWC stores coalesce.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kDirectThreads = 256;
constexpr int kDirectPix = 64;  // output pixels per CTA

struct DirectParams {
  int B, Cin, H, W, Cout, KH, KW, stride, pad, groups, n, Ho, Wo;
  int cob;  // output channels per CTA
  const void* x;
  const void* experts;
  const float* alpha;
  const float* bias;  // may be null
  void* y;
  const float* a_in;   // [B][Cin] input channel attention, or null
  const float* a_out;  // [B][Cout] output channel attention, or null
  const float* chan_add;  // [B][Cout] or null: chan_scale * chan_add joins the mixed bias
  float chan_scale;
};

template <typename T>
__global__ void __launch_bounds__(kDirectThreads) direct_conv_kernel(DirectParams p) {
  extern __shared__ float dsm[];
  const int b = blockIdx.z;
  const int co0 = blockIdx.y * p.cob;
  const int cob = min(p.cob, p.Cout - co0);
  const int pix0 = blockIdx.x * kDirectPix;
  const int Cg = p.Cin / p.groups;
  const int Coutg = p.Cout / p.groups;
  const int taps = p.KH * p.KW;
  const int wrow = taps * Cg;  // weights per output channel

  grid_dependency_wait();  // alpha (and possibly x) come from earlier kernels
  // the next kernel on the stream (a routing kernel of the next layer) may
  // be scheduled while this one runs: it waits for this grid's completion
  // before it reads anything this grid writes
  grid_launch_dependents();
  float* alpha_s = dsm;                     // [n]
  float* bias_s = alpha_s + p.n;            // [cob]
  float* w_s = bias_s + p.cob;              // [cob][KH][KW][Cg]

  for (int i = threadIdx.x; i < p.n; i += kDirectThreads)
    alpha_s[i] = p.alpha[static_cast<size_t>(b) * p.n + i];
  __syncthreads();

  const T* E = static_cast<const T*>(p.experts);
  const size_t wsize = static_cast<size_t>(p.Cout) * wrow;
  for (int e = threadIdx.x; e < cob * wrow; e += kDirectThreads) {
    const size_t off = static_cast<size_t>(co0) * wrow + e;
    float s = 0.f;
    for (int i = 0; i < p.n; ++i) s = fmaf(alpha_s[i], to_f32<T>(E[i * wsize + off]), s);
    if (p.a_in != nullptr) {  // input attention of channel (group of co) * Cg + ci
      const int cl = e / wrow, ci = e % Cg;
      s *= p.a_in[static_cast<size_t>(b) * p.Cin + ((co0 + cl) / Coutg) * Cg + ci];
    }
    w_s[e] = s;
  }
  for (int c = threadIdx.x; c < cob; c += kDirectThreads) {
    float s = 0.f;
    if (p.bias)
      for (int i = 0; i < p.n; ++i)
        s = fmaf(alpha_s[i], p.bias[static_cast<size_t>(i) * p.Cout + co0 + c], s);
    if (p.chan_add)
      s = fmaf(p.chan_add[static_cast<size_t>(b) * p.Cout + co0 + c], p.chan_scale, s);
    bias_s[c] = s;
  }
  __syncthreads();

  const T* xb = static_cast<const T*>(p.x) + static_cast<size_t>(b) * p.H * p.W * p.Cin;
  T* yb = static_cast<T*>(p.y) + static_cast<size_t>(b) * p.Ho * p.Wo * p.Cout;
  const int npix = p.Ho * p.Wo;
  for (int idx = threadIdx.x; idx < kDirectPix * cob; idx += kDirectThreads) {
    const int pix = pix0 + idx / cob;
    const int cl = idx % cob;
    if (pix >= npix) break;
    const int co = co0 + cl;
    const int oh = pix / p.Wo, ow = pix % p.Wo;
    const int cin0 = (co / Coutg) * Cg;
    const float* wr = w_s + static_cast<size_t>(cl) * wrow;
    float acc = bias_s[cl];
    for (int kh = 0; kh < p.KH; ++kh) {
      const int ih = oh * p.stride + kh - p.pad;
      if (ih < 0 || ih >= p.H) continue;
      for (int kw = 0; kw < p.KW; ++kw) {
        const int iw = ow * p.stride + kw - p.pad;
        if (iw < 0 || iw >= p.W) continue;
        const T* xp = xb + (static_cast<size_t>(ih) * p.W + iw) * p.Cin + cin0;
        const float* wp = wr + (kh * p.KW + kw) * Cg;
        for (int ci = 0; ci < Cg; ++ci) acc = fmaf(to_f32<T>(xp[ci]), wp[ci], acc);
      }
    }
    if (p.a_out != nullptr) acc *= p.a_out[static_cast<size_t>(b) * p.Cout + co];
    yb[static_cast<size_t>(pix) * p.Cout + co] = from_f32<T>(acc);
  }
}

}  // namespace dc
