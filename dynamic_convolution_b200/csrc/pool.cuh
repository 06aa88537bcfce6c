// Routing pooled in the previous layer, for chained layers (the output of one
// dynamic-convolution layer is the input of the next).
//
// The tensor-core convolution can add, in its epilogue, the channel sums of
// the outputs it stores (one partial per row block); the routing of the next
// layer then needs only those partial sums: g = (sum of partials) / (H*W),
// followed by the linear layer and the activation of the routing step (the
// attentions are input-dependent, KernelWarehouse, abstract; CondConv,
// abstract; FMDConv, abstract for the temperature). This removes the second
// full read of the activation tensor that the routing kernel would otherwise
// make.
//
//  * pool_sum_kernel: the same partial sums in a separate pass over y, for the
//    CUDA-core forward kernels (one partial per sample).
//  * route_pooled_kernel: one CTA per sample; partials added in order, the
//    linear layer with warp-shuffle dot products, the activation in one warp.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kPoolThreads = 256;

// ysum[b][0][c] = sum over the H*W pixels of y[b][.][.][c], pixels in order,
// four interleaved accumulators added in a fixed order at the end.
template <typename T>
__global__ void __launch_bounds__(kPoolThreads) pool_sum_kernel(const T* y, int HW, int C,
                                                                float* ysum) {
  grid_dependency_wait();  // y comes from the forward kernel before
  const int b = blockIdx.x;
  const T* yb = y + static_cast<size_t>(b) * HW * C;
  for (int c = threadIdx.x; c < C; c += kPoolThreads) {
    float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
    int px = 0;
    for (; px + 3 < HW; px += 4) {
      a0 += to_f32<T>(yb[static_cast<size_t>(px) * C + c]);
      a1 += to_f32<T>(yb[static_cast<size_t>(px + 1) * C + c]);
      a2 += to_f32<T>(yb[static_cast<size_t>(px + 2) * C + c]);
      a3 += to_f32<T>(yb[static_cast<size_t>(px + 3) * C + c]);
    }
    for (; px < HW; ++px) a0 += to_f32<T>(yb[static_cast<size_t>(px) * C + c]);
    ysum[static_cast<size_t>(b) * C + c] = (a0 + a1) + (a2 + a3);
  }
}

struct RoutePooledParams {
  int B, C, HW, n, parts;
  int mode;  // 0 sigmoid, 1 softmax
  float tau;
  const float* ysum;  // [B][parts][C]
  const float* Wr;    // [n][C]
  const float* br;    // [n] or null
  float* alpha;       // [B][n]
};

__global__ void __launch_bounds__(kPoolThreads) route_pooled_kernel(RoutePooledParams p) {
  extern __shared__ float rp_smem[];
  float* g = rp_smem;      // [C]
  float* z = g + p.C;      // [n]
  grid_launch_dependents();
  grid_dependency_wait();  // ysum comes from the previous layer's forward
  const int b = blockIdx.x, t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const float inv_hw = 1.0f / static_cast<float>(p.HW);
  const float* yb = p.ysum + static_cast<size_t>(b) * p.parts * p.C;
  for (int c = t; c < p.C; c += kPoolThreads) {
    float s = 0.f;
    for (int q = 0; q < p.parts; ++q) s += yb[static_cast<size_t>(q) * p.C + c];
    g[c] = s * inv_hw;
  }
  __syncthreads();
  for (int i = warp; i < p.n; i += kPoolThreads / 32) {
    const float* wr = p.Wr + static_cast<size_t>(i) * p.C;
    float s = 0.f;
    for (int c = lane; c < p.C; c += 32) s = fmaf(wr[c], g[c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) z[i] = s + (p.br ? p.br[i] : 0.f);
  }
  __syncthreads();
  float* out = p.alpha + static_cast<size_t>(b) * p.n;
  if (p.mode == 0) {
    for (int i = t; i < p.n; i += kPoolThreads) out[i] = 1.0f / (1.0f + expf(-z[i]));
  } else if (warp == 0) {
    float m = -INFINITY;
    for (int i = lane; i < p.n; i += 32) m = fmaxf(m, z[i] / p.tau);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    float s = 0.f;
    for (int i = lane; i < p.n; i += 32) s += expf(z[i] / p.tau - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    const float inv = 1.0f / s;
    for (int i = lane; i < p.n; i += 32) out[i] = expf(z[i] / p.tau - m) * inv;
  }
}

}  // namespace dc
