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

// The average pool in pixel slices: CTA (slice, sample) sums x_b over its
// pixels into part[b][slice][c] (thread = (channel c, pixel lane l), lanes
// added in order).
template <typename T>
__global__ void __launch_bounds__(kCellThreads)
    cells_pool_kernel(int C, int HW, int Ps, const T* __restrict__ x, float* __restrict__ part) {
  __shared__ float lanes[kCellThreads];
  const int slice = blockIdx.x, nslices = gridDim.x, b = blockIdx.y, t = threadIdx.x;
  const int p0 = slice * Ps, p1 = min(HW, p0 + Ps);
  const T* xb = x + static_cast<size_t>(b) * HW * C;
  for (int c0 = 0; c0 < C; c0 += kCellThreads) {
    const int nc = min(kCellThreads, C - c0);
    const int nl = kCellThreads / nc;
    const int c = c0 + t % nc, l = t / nc;
    float s = 0.f;
    if (l < nl) {
#pragma unroll 8
      for (int p = p0 + l; p < p1; p += nl) s += to_f32(xb[static_cast<size_t>(p) * C + c]);
    }
    __syncthreads();
    lanes[t] = s;
    __syncthreads();
    if (t < nc) {
      float tot = 0.f;
      for (int k = 0; k < nl; ++k) tot += lanes[k * nc + t];
      part[(static_cast<size_t>(b) * nslices + slice) * C + c0 + t] = tot;
    }
  }
}

// alpha[b][j][i] for the cells j of one group and one sample per CTA (grid:
// cell groups, samples): g[c] = (slice sums in order) / HW in shared memory;
// logits z[k] = br[k] + sum_c Wr[k][c] g[c] of the group's cells, eight
// logits per warp at a time (lanes over c, a fixed xor-shuffle tree each);
// then per cell (one warp each) the sigmoid of each logit, or the softmax of
// the cell's n logits divided by tau, the cell's maximum subtracted (maximum
// and sum by fixed shuffle trees).
constexpr int kCellsPerCta = 2;

__global__ void __launch_bounds__(kCellThreads)
    route_cells_kernel(int C, int HW, int nslices, int m, int n, int mode, float tau,
                       const float* __restrict__ part, const float* __restrict__ Wr,
                       const float* __restrict__ br, float* __restrict__ alpha) {
  extern __shared__ float rc_s[];
  float* g = rc_s;                 // [C]
  float* z = rc_s + C;             // [kCellsPerCta * n]
  const int b = blockIdx.y, j0 = blockIdx.x * kCellsPerCta, t = threadIdx.x;
  const int nj = min(kCellsPerCta, m - j0);
  const float inv_hw = 1.f / static_cast<float>(HW);
  for (int c = t; c < C; c += kCellThreads) {
    float s = 0.f;
    for (int k = 0; k < nslices; ++k) s += part[(static_cast<size_t>(b) * nslices + k) * C + c];
    g[c] = s * inv_hw;
  }
  __syncthreads();
  const int warp = t >> 5, lane = t & 31, nwarps = kCellThreads / 32;
  const int nk = nj * n, k0 = j0 * n;
  for (int kb = warp * 8; kb < nk; kb += nwarps * 8) {
    float acc[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) acc[u] = 0.f;
    for (int c = lane; c < C; c += 32) {
      const float gc = g[c];
#pragma unroll
      for (int u = 0; u < 8; ++u)
        if (kb + u < nk) acc[u] = fmaf(Wr[static_cast<size_t>(k0 + kb + u) * C + c], gc, acc[u]);
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      float v = acc[u];
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
      if (lane == 0 && kb + u < nk) z[kb + u] = v + (br ? br[k0 + kb + u] : 0.f);
    }
  }
  __syncthreads();
  for (int jj = warp; jj < nj; jj += nwarps) {
    const float* zj = z + static_cast<size_t>(jj) * n;
    float* aj = alpha + (static_cast<size_t>(b) * m + j0 + jj) * n;
    if (mode == 0) {
      for (int i = lane; i < n; i += 32) aj[i] = 1.f / (1.f + expf(-zj[i]));
    } else {
      float mx = -INFINITY;
      for (int i = lane; i < n; i += 32) mx = fmaxf(mx, zj[i]);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
      float den = 0.f;
      for (int i = lane; i < n; i += 32) den += expf((zj[i] - mx) / tau);
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xffffffffu, den, off);
      const float inv = 1.f / den;
      for (int i = lane; i < n; i += 32) aj[i] = expf((zj[i] - mx) / tau) * inv;
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
// a cell, cell j, SB samples); thread = VEC consecutive elements: the SB
// samples' attentions of cell j are staged in shared memory; per expert one
// 16-byte load of the warehouse (four experts' loads in flight), then VEC * SB
// multiply-adds as packed fp32 pairs; rounded once.
template <typename T, int SB>
__global__ void __launch_bounds__(kCellThreads) cells_mix_kernel(CmParams p) {
  constexpr int VEC = 16 / static_cast<int>(sizeof(T));
  constexpr int PAIRS = VEC / 2;
  extern __shared__ float cm_a[];  // [n][SB]
  const int j = blockIdx.y, b0 = blockIdx.z * SB;
  for (int e = threadIdx.x; e < SB * p.n; e += kCellThreads) {
    const int i = e / SB, u = e - i * SB;
    cm_a[e] = b0 + u < p.B ? p.alpha[(static_cast<size_t>(b0 + u) * p.m + j) * p.n + i] : 0.f;
  }
  __syncthreads();
  const long long e0 = (static_cast<long long>(blockIdx.x) * kCellThreads + threadIdx.x) * VEC;
  if (e0 >= p.s) return;
  const T* E = static_cast<const T*>(p.E) + e0;
  uint64_t acc[SB][PAIRS];
#pragma unroll
  for (int u = 0; u < SB; ++u)
#pragma unroll
    for (int q = 0; q < PAIRS; ++q) acc[u][q] = 0ull;
  int i = 0;
  for (; i + 4 <= p.n; i += 4) {
    uint4 raw[4];
#pragma unroll
    for (int r = 0; r < 4; ++r)
      raw[r] = *reinterpret_cast<const uint4*>(E + static_cast<size_t>(i + r) * p.s);
#pragma unroll
    for (int r = 0; r < 4; ++r) {
      uint64_t ev[PAIRS];
      const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw[r]);
      if constexpr (sizeof(T) == 2) {
#pragma unroll
        for (int q = 0; q < PAIRS; ++q) ev[q] = dc::bf16x2_to_f32x2(w[q]);
      } else {
#pragma unroll
        for (int q = 0; q < PAIRS; ++q) ev[q] = (static_cast<uint64_t>(w[2 * q + 1]) << 32) | w[2 * q];
      }
      const float* ai = cm_a + (i + r) * SB;
#pragma unroll
      for (int u = 0; u < SB; ++u) {
        const uint64_t a2 = dc::pack_f32x2(ai[u], ai[u]);
#pragma unroll
        for (int q = 0; q < PAIRS; ++q) acc[u][q] = dc::ffma2(a2, ev[q], acc[u][q]);
      }
    }
  }
  for (; i < p.n; ++i) {
    const uint4 raw = *reinterpret_cast<const uint4*>(E + static_cast<size_t>(i) * p.s);
    uint64_t ev[PAIRS];
    const uint32_t* w = reinterpret_cast<const uint32_t*>(&raw);
    if constexpr (sizeof(T) == 2) {
#pragma unroll
      for (int q = 0; q < PAIRS; ++q) ev[q] = dc::bf16x2_to_f32x2(w[q]);
    } else {
#pragma unroll
      for (int q = 0; q < PAIRS; ++q) ev[q] = (static_cast<uint64_t>(w[2 * q + 1]) << 32) | w[2 * q];
    }
    const float* ai = cm_a + i * SB;
#pragma unroll
    for (int u = 0; u < SB; ++u) {
      const uint64_t a2 = dc::pack_f32x2(ai[u], ai[u]);
#pragma unroll
      for (int q = 0; q < PAIRS; ++q) acc[u][q] = dc::ffma2(a2, ev[q], acc[u][q]);
    }
  }
#pragma unroll
  for (int u = 0; u < SB; ++u) {
    if (b0 + u >= p.B) break;
    alignas(16) T o[VEC];
#pragma unroll
    for (int q = 0; q < PAIRS; ++q) {
      o[2 * q] = from_f32<T>(__uint_as_float(static_cast<uint32_t>(acc[u][q])));
      o[2 * q + 1] = from_f32<T>(__uint_as_float(static_cast<uint32_t>(acc[u][q] >> 32)));
    }
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
