// Kernels of the warehouse-cell path: the per-cell routing and the cell
// mixing. Kernel cells shared through a warehouse (KernelWarehouse, abstract)
// in the reading stated in include/dynconv_cells.h: cell j of sample b's
// kernel is sum_i alpha[b][j][i] * E[i], its attentions a per-cell softmax (or
// sigmoid) of one linear layer on the average pool.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace dcc {

using dc::from_f32;
using dc::to_f32;

constexpr int kCellThreads = 256;

// alpha[b][j][i] for one sample per CTA: (1) the average pool g[c] of x_b
// (thread = (channel c, pixel lane l), lanes summed in order), (2) the
// logits z[k] = br[k] + sum_c Wr[k][c] g[c] (one warp per logit, a fixed
// xor-shuffle tree over the lanes), (3) per cell j (one thread per cell) the
// sigmoid of each logit, or the softmax of the cell's n logits divided by tau
// with the cell's maximum subtracted.
template <typename T>
__global__ void __launch_bounds__(kCellThreads)
    route_cells_kernel(int C, int HW, int m, int n, int mode, float tau, const T* __restrict__ x,
                       const float* __restrict__ Wr, const float* __restrict__ br,
                       float* __restrict__ alpha) {
  extern __shared__ float rc_s[];
  float* g = rc_s;                 // [C]
  float* z = rc_s + C;             // [m * n]
  float* lanes = z + m * n;        // [kCellThreads]
  const int b = blockIdx.x, t = threadIdx.x;
  const T* xb = x + static_cast<size_t>(b) * HW * C;
  const float inv_hw = 1.f / static_cast<float>(HW);
  for (int c0 = 0; c0 < C; c0 += kCellThreads) {
    const int nc = min(kCellThreads, C - c0);
    const int nl = kCellThreads / nc;   // pixel lanes
    const int c = c0 + t % nc, l = t / nc;
    float s = 0.f;
    if (l < nl) {
#pragma unroll 8
      for (int p = l; p < HW; p += nl) s += to_f32(xb[static_cast<size_t>(p) * C + c]);
    }
    lanes[t] = s;
    __syncthreads();
    if (t < nc) {
      float tot = 0.f;
      for (int k = 0; k < nl; ++k) tot += lanes[k * nc + t];
      g[c0 + t] = tot * inv_hw;
    }
    __syncthreads();
  }
  const int warp = t >> 5, lane = t & 31;
  for (int k = warp; k < m * n; k += kCellThreads / 32) {
    const float* w = Wr + static_cast<size_t>(k) * C;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s = fmaf(w[c], g[c], s);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) s += __shfl_xor_sync(0xffffffffu, s, off);
    if (lane == 0) z[k] = s + (br ? br[k] : 0.f);
  }
  __syncthreads();
  for (int j = t; j < m; j += kCellThreads) {
    const float* zj = z + static_cast<size_t>(j) * n;
    float* aj = alpha + (static_cast<size_t>(b) * m + j) * n;
    if (mode == 0) {
      for (int i = 0; i < n; ++i) aj[i] = 1.f / (1.f + expf(-zj[i]));
    } else {
      float mx = zj[0];
      for (int i = 1; i < n; ++i) mx = fmaxf(mx, zj[i]);
      float den = 0.f;
      for (int i = 0; i < n; ++i) den += expf((zj[i] - mx) / tau);
      const float inv = 1.f / den;
      for (int i = 0; i < n; ++i) aj[i] = expf((zj[i] - mx) / tau) * inv;
    }
  }
}

struct CmParams {
  int B, m, n;
  long long s;         // elements per cell (a multiple of VEC)
  long long wsize;     // m * s
  const void* E;       // warehouse [n][s]
  const float* alpha;  // [B][m][n]
  void* Wb;            // [B][wsize]
};

// W_b[b][j*s + e] = sum_i alpha[b][j][i] * E[i][e]. CTA = (VEC*256 elements of
// a cell, cell j, SB samples); thread = VEC consecutive elements: per expert
// one 16-byte load of the warehouse and VEC * SB multiply-adds, the SB
// samples' attentions of cell j staged in shared memory; rounded once.
template <typename T, int SB>
__global__ void __launch_bounds__(kCellThreads) cells_mix_kernel(CmParams p) {
  constexpr int VEC = 16 / static_cast<int>(sizeof(T));
  extern __shared__ float cm_a[];  // [SB][n]
  const int j = blockIdx.y, b0 = blockIdx.z * SB;
  for (int e = threadIdx.x; e < SB * p.n; e += kCellThreads) {
    const int u = e / p.n, i = e - u * p.n;
    cm_a[e] = b0 + u < p.B ? p.alpha[(static_cast<size_t>(b0 + u) * p.m + j) * p.n + i] : 0.f;
  }
  __syncthreads();
  const long long e0 = (static_cast<long long>(blockIdx.x) * kCellThreads + threadIdx.x) * VEC;
  if (e0 >= p.s) return;
  const T* E = static_cast<const T*>(p.E);
  float acc[SB][VEC];
#pragma unroll
  for (int u = 0; u < SB; ++u)
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[u][k] = 0.f;
#pragma unroll 2
  for (int i = 0; i < p.n; ++i) {
    alignas(16) T ev[VEC];
    *reinterpret_cast<uint4*>(ev) =
        *reinterpret_cast<const uint4*>(E + static_cast<size_t>(i) * p.s + e0);
#pragma unroll
    for (int u = 0; u < SB; ++u) {
      const float a = cm_a[u * p.n + i];
#pragma unroll
      for (int k = 0; k < VEC; ++k) acc[u][k] = fmaf(a, to_f32(ev[k]), acc[u][k]);
    }
  }
#pragma unroll
  for (int u = 0; u < SB; ++u) {
    if (b0 + u >= p.B) break;
    alignas(16) T o[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) o[k] = from_f32<T>(acc[u][k]);
    *reinterpret_cast<uint4*>(static_cast<T*>(p.Wb) + static_cast<size_t>(b0 + u) * p.wsize +
                              static_cast<size_t>(j) * p.s + e0) =
        *reinterpret_cast<const uint4*>(o);
  }
}

// Identity [r][r] (fp32) followed by `rows` copies of bias[C] (when bias is
// given): the one-hot attentions and per-sample bias rows that hand the
// per-sample kernels to the forward entry point.
__global__ void __launch_bounds__(kCellThreads)
    onehot_kernel(int r, float* __restrict__ ident, const float* __restrict__ bias, int C,
                  int rows, float* __restrict__ bias_rows) {
  const int t = blockIdx.x * kCellThreads + threadIdx.x;
  if (t < r * r) ident[t] = (t / r == t % r) ? 1.f : 0.f;
  if (bias && t < rows * C) bias_rows[t] = bias[t % C];
}

}  // namespace dcc
