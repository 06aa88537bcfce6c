// Routing kernel: alpha_b = act(Wr * GAP(x_b) + br).
//
// The routing weights are "input-dependent attentions" over n static kernels
// (KernelWarehouse: Rethinking the Design of Dynamic Convolution, abstract),
// one vector per example (CondConv, abstract), with a temperature on the
// softmax (FMDConv, abstract: temperature-degraded kernel attention). The
// global-average-pool -> single linear layer -> sigmoid / softmax(z/tau) form
// is the reading taken where the pages give no formula.
//
// Design: one thread-block cluster per sample. Each CTA of the cluster streams
// a contiguous slice of the sample's pixels with 16-byte NHWC vector loads and
// keeps per-channel fp32 partial sums; the partials are combined in a fixed
// order inside the CTA and then, through distributed shared memory, by the
// cluster's rank-0 CTA, which also runs the FC (warp-shuffle dot products) and
// the activation (warp-shuffle max / sum for the softmax). No global scratch,
// no atomics, deterministic.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace dc {

constexpr int kRouteThreads = 256;

struct RouteParams {
  int B, C, HW, n;
  int mode;       // 0 sigmoid, 1 softmax
  float tau;
  const void* x;
  const float* Wr;
  const float* br;  // may be null
  float* alpha;
};

// VEC channels per load: 16 bytes when the channel count allows it, else 1.
template <typename T, int VEC>
__device__ __forceinline__ void load_vec(const T* p, float (&v)[VEC]) {
  if constexpr (VEC * sizeof(T) == 16) {
    const uint4 u = ld_nc_v4(p);
    if constexpr (sizeof(T) == 2) {
      v[0] = bf16lo_to_f32(u.x); v[1] = bf16hi_to_f32(u.x);
      v[2] = bf16lo_to_f32(u.y); v[3] = bf16hi_to_f32(u.y);
      v[4] = bf16lo_to_f32(u.z); v[5] = bf16hi_to_f32(u.z);
      v[6] = bf16lo_to_f32(u.w); v[7] = bf16hi_to_f32(u.w);
    } else {
      v[0] = __uint_as_float(u.x); v[1] = __uint_as_float(u.y);
      v[2] = __uint_as_float(u.z); v[3] = __uint_as_float(u.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < VEC; ++j) v[j] = to_f32<T>(p[j]);
  }
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kRouteThreads) route_kernel(RouteParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int nsplit = static_cast<int>(cluster.num_blocks());
  const int b = blockIdx.y;
  const int t = threadIdx.x;

  extern __shared__ float route_smem[];
  const int C = p.C;
  const int nv = C / VEC;                                  // vectors per pixel
  const int tpp = nv < kRouteThreads ? nv : kRouteThreads;  // threads per pixel
  const int lanes_p = kRouteThreads / tpp;                  // pixels in flight per step
  float* partial = route_smem;                              // [lanes_p][C]
  float* csum = partial + static_cast<size_t>(lanes_p) * C;  // [C], this CTA's slice sum
  float* g = csum + C;                                      // [C], rank 0: the pooled vector
  float* z = g + C;                                         // [n], rank 0: logits

  // ---- this CTA's pixel slice, per-channel partial sums in registers
  const int p_begin = static_cast<int>((static_cast<long long>(p.HW) * rank) / nsplit);
  const int p_end = static_cast<int>((static_cast<long long>(p.HW) * (rank + 1)) / nsplit);
  const T* xb = static_cast<const T*>(p.x) + static_cast<size_t>(b) * p.HW * C;
  const int pl = t / tpp;
  if (pl < lanes_p) {
    for (int v = t % tpp; v < nv; v += tpp) {
      float acc[VEC];
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
      int px = p_begin + pl;
      // four loads in flight per thread
      for (; px + 3 * lanes_p < p_end; px += 4 * lanes_p) {
        float v0[VEC], v1[VEC], v2[VEC], v3[VEC];
        load_vec<T, VEC>(xb + static_cast<size_t>(px) * C + v * VEC, v0);
        load_vec<T, VEC>(xb + static_cast<size_t>(px + lanes_p) * C + v * VEC, v1);
        load_vec<T, VEC>(xb + static_cast<size_t>(px + 2 * lanes_p) * C + v * VEC, v2);
        load_vec<T, VEC>(xb + static_cast<size_t>(px + 3 * lanes_p) * C + v * VEC, v3);
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc[j] += (v0[j] + v1[j]) + (v2[j] + v3[j]);
      }
      for (; px < p_end; px += lanes_p) {
        float v0[VEC];
        load_vec<T, VEC>(xb + static_cast<size_t>(px) * C + v * VEC, v0);
#pragma unroll
        for (int j = 0; j < VEC; ++j) acc[j] += v0[j];
      }
#pragma unroll
      for (int j = 0; j < VEC; ++j) partial[static_cast<size_t>(pl) * C + v * VEC + j] = acc[j];
    }
  }
  __syncthreads();
  for (int c = t; c < C; c += kRouteThreads) {
    float s = 0.f;
    for (int l = 0; l < lanes_p; ++l) s += partial[static_cast<size_t>(l) * C + c];
    csum[c] = s;
  }
  cluster.sync();

  // ---- rank 0: combine the cluster's slices in rank order, then FC + activation
  if (rank == 0) {
    const float inv_hw = 1.0f / static_cast<float>(p.HW);
    for (int c = t; c < C; c += kRouteThreads) {
      float s = 0.f;
      for (int r = 0; r < nsplit; ++r) s += cluster.map_shared_rank(csum, r)[c];
      g[c] = s * inv_hw;
    }
  }
  cluster.sync();  // peers' shared memory must outlive rank 0's reads
  if (rank != 0) return;

  __syncthreads();
  const int warp = t >> 5, lane = t & 31;
  for (int i = warp; i < p.n; i += kRouteThreads / 32) {
    const float* wr = p.Wr + static_cast<size_t>(i) * C;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s = fmaf(wr[c], g[c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) z[i] = s + (p.br ? p.br[i] : 0.f);
  }
  __syncthreads();

  float* out = p.alpha + static_cast<size_t>(b) * p.n;
  if (p.mode == 0) {
    for (int i = t; i < p.n; i += kRouteThreads) out[i] = 1.0f / (1.0f + expf(-z[i]));
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
