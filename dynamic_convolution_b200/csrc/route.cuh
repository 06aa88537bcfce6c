// Routing kernel: alpha_b = act(Wr * GAP(x_b) + br).
//
// The routing weights are "input-dependent attentions" over n static kernels
// (KernelWarehouse: Rethinking the Design of Dynamic Convolution, abstract),
// one vector per example (CondConv, abstract), with a temperature on the
// softmax (FMDConv, abstract: temperature-degraded kernel attention). The
// global-average-pool -> single linear layer -> sigmoid / softmax(z/tau) form
// is the reading taken where the pages give no formula.
//
// Design: one thread-block cluster per sample, built around the latency
// chain rather than bandwidth (the whole input is ~10 MB):
//  * every thread issues its 16-byte NHWC loads in batches of 16 before it
//    adds any of them, so the cluster has the sample's bytes in flight at once;
//  * the rank-0 CTA prefetches the router weights Wr and br into shared
//    memory while those loads are in flight;
//  * each CTA reduces its per-thread partial sums in a fixed order, then PUSHES
//    its per-channel sums into rank 0's shared memory with remote stores
//    (distributed shared memory) -- one cluster barrier, no remote loads;
//  * rank 0 adds the slices in rank order, runs the FC from shared memory
//    (warp-shuffle dot products) and the activation (warp-shuffle max / sum
//    for the softmax).
// No global scratch, no atomics, deterministic.
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
// Raw loads and the conversion to fp32 are separate so that a batch of loads
// is issued before the first one is used.
template <typename T, int VEC>
union RawVec {
  uint4 u;   // 16-byte path
  T s[VEC];  // scalar path
};

template <typename T, int VEC>
__device__ __forceinline__ void load_raw(const T* p, RawVec<T, VEC>& r) {
  if constexpr (VEC * sizeof(T) == 16) {
    r.u = ld_nc_v4(p);
  } else {
#pragma unroll
    for (int j = 0; j < VEC; ++j) r.s[j] = p[j];
  }
}

template <typename T, int VEC>
__device__ __forceinline__ void add_raw(const RawVec<T, VEC>& r, float (&acc)[VEC]) {
  if constexpr (VEC * sizeof(T) == 16) {
    const uint4 u = r.u;
    if constexpr (sizeof(T) == 2) {
      acc[0] += bf16lo_to_f32(u.x); acc[1] += bf16hi_to_f32(u.x);
      acc[2] += bf16lo_to_f32(u.y); acc[3] += bf16hi_to_f32(u.y);
      acc[4] += bf16lo_to_f32(u.z); acc[5] += bf16hi_to_f32(u.z);
      acc[6] += bf16lo_to_f32(u.w); acc[7] += bf16hi_to_f32(u.w);
    } else {
      acc[0] += __uint_as_float(u.x); acc[1] += __uint_as_float(u.y);
      acc[2] += __uint_as_float(u.z); acc[3] += __uint_as_float(u.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] += to_f32<T>(r.s[j]);
  }
}

// Shared-memory floats the kernel needs (the host sizes the launch with it).
__host__ __device__ inline size_t route_smem_floats(int C, int n, int VEC, int nsplit) {
  const int nv = C / VEC;
  const int tpp = nv < kRouteThreads ? nv : kRouteThreads;
  const int lanes_p = kRouteThreads / tpp;
  const size_t wr = static_cast<size_t>(n) * C <= 8192 ? static_cast<size_t>(n) * C : 0;
  return static_cast<size_t>(lanes_p) * C + static_cast<size_t>(nsplit) * C + C + wr + 2 * n;
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(RouteParams p) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int nsplit = static_cast<int>(cluster.num_blocks());
  const int b = blockIdx.y;
  const int t = threadIdx.x;
  // the forward kernel may be scheduled as soon as every routing CTA runs; it
  // waits for this grid's completion before it reads alpha
  grid_launch_dependents();

  extern __shared__ float route_smem[];
  const int C = p.C;
  const int nv = C / VEC;                                  // vectors per pixel
  const int tpp = nv < kRouteThreads ? nv : kRouteThreads;  // threads per pixel
  const int lanes_p = kRouteThreads / tpp;                  // pixels in flight per step
  const bool wr_in_smem = static_cast<size_t>(p.n) * C <= 8192;
  float* partial = route_smem;                                  // [lanes_p][C]
  float* sums = partial + static_cast<size_t>(lanes_p) * C;     // [nsplit][C], rank 0 only
  float* g = sums + static_cast<size_t>(nsplit) * C;            // [C]
  float* wr_s = g + C;                                          // [n][C] if it fits
  float* br_s = wr_s + (wr_in_smem ? static_cast<size_t>(p.n) * C : 0);  // [n]
  float* z = br_s + p.n;                                        // [n]

  // ---- this CTA's pixel slice: all loads first, then the adds
  const int p_begin = static_cast<int>((static_cast<long long>(p.HW) * rank) / nsplit);
  const int p_end = static_cast<int>((static_cast<long long>(p.HW) * (rank + 1)) / nsplit);
  const T* xb = static_cast<const T*>(p.x) + static_cast<size_t>(b) * p.HW * C;
  const int pl = t / tpp;
  if (pl < lanes_p) {
    for (int v = t % tpp; v < nv; v += tpp) {
      float acc[VEC];
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
      // batches of 16 loads issued back to back, then added in a fixed order
      for (int px = p_begin + pl; px < p_end; px += 16 * lanes_p) {
        RawVec<T, VEC> raw[16];
#pragma unroll
        for (int uu = 0; uu < 16; ++uu) {
          const int pp = px + uu * lanes_p;
          if (pp < p_end) load_raw<T, VEC>(xb + static_cast<size_t>(pp) * C + v * VEC, raw[uu]);
        }
#pragma unroll
        for (int uu = 0; uu < 16; ++uu)
          if (px + uu * lanes_p < p_end) add_raw<T, VEC>(raw[uu], acc);
      }
#pragma unroll
      for (int j = 0; j < VEC; ++j) partial[static_cast<size_t>(pl) * C + v * VEC + j] = acc[j];
    }
  }
  // rank 0: router weights into shared memory while the loads are in flight
  if (rank == 0) {
    if (wr_in_smem)
      for (int e = t; e < p.n * C; e += kRouteThreads) wr_s[e] = p.Wr[e];
    for (int i = t; i < p.n; i += kRouteThreads) br_s[i] = p.br ? p.br[i] : 0.f;
  }
  __syncthreads();
  // fixed-order reduction over the pixel lanes, pushed into rank 0's slot for this rank
  float* dst = cluster.map_shared_rank(sums, 0) + static_cast<size_t>(rank) * C;
  for (int c = t; c < C; c += kRouteThreads) {
    float s = 0.f;
    for (int l = 0; l < lanes_p; ++l) s += partial[static_cast<size_t>(l) * C + c];
    dst[c] = s;
  }
  cluster.sync();  // remote stores visible to rank 0; peers may exit after this
  if (rank != 0) return;

  const float inv_hw = 1.0f / static_cast<float>(p.HW);
  for (int c = t; c < C; c += kRouteThreads) {
    float s = 0.f;
    for (int r = 0; r < nsplit; ++r) s += sums[static_cast<size_t>(r) * C + c];
    g[c] = s * inv_hw;
  }
  __syncthreads();
  const int warp = t >> 5, lane = t & 31;
  for (int i = warp; i < p.n; i += kRouteThreads / 32) {
    const float* wr = wr_in_smem ? wr_s + static_cast<size_t>(i) * C : p.Wr + static_cast<size_t>(i) * C;
    float s = 0.f;
    for (int c = lane; c < C; c += 32) s = fmaf(wr[c], g[c], s);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) z[i] = s + br_s[i];
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
