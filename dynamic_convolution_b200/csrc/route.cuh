// Routing kernel: alpha_b = act(Wr * GAP(x_b) + br).
//
// The routing weights are attentions over n static kernels computed from the input
// (KernelWarehouse: Rethinking the Design of Dynamic Convolution, abstract),
// one vector per example (CondConv, abstract), with a temperature on the
// softmax (FMDConv, abstract: temperature-degraded kernel attention). The
// global-average-pool -> single linear layer -> sigmoid / softmax(z/tau) form
// is the reading taken where the pages give no formula.
//
// Design: one thread-block cluster per sample, each CTA a contiguous slice of
// the sample's pixels, built around the latency chain (the whole input is a
// few MB):
//  * the slice is contiguous in NHWC, so one thread moves it into shared
//    memory with a few bulk copies (cp.async.bulk, up to four in flight),
//    together with the router weights Wr when they fit: the bytes in flight
//    are not limited by per-thread load queues;
//  * the threads add the staged pixels in a fixed order;
//  * the linear layer is split over the ranks: each CTA multiplies its own
//    channel sums by Wr and PUSHES its n partial logits into rank 0's shared
//    memory (distributed shared memory); after the one cluster barrier rank 0
//    adds nsplit x n numbers, scales by 1/HW, adds br and applies the
//    activation.
// When Wr does not fit in shared memory the CTAs push per-channel sums to
// rank 0; after the barrier every rank reads them back (DSMEM, rank order),
// computes the logits of every nsplit-th expert from Wr rows in global
// memory and pushes them to rank 0, which after a second cluster barrier adds
// br and applies the activation. When a pixel's
// channels are not a multiple of 16 bytes the threads load the pixels
// themselves (no bulk copy). No global scratch, no atomics, deterministic.
#pragma once

#include <cooperative_groups.h>

#include "common.cuh"

namespace dc {

constexpr int kRouteThreads = 256;
constexpr int kRoutePieceBytes = 24 * 1024;  // largest bulk piece
constexpr int kRouteRing = 4;                // bulk pieces in flight per CTA
constexpr int kRouteWrSmemBytes = 32 * 1024;  // largest Wr staged in shared memory
constexpr int kErrWaitRoute = 0x107;

struct RouteParams {
  int B, C, HW, n;
  int mode;       // 0 sigmoid, 1 softmax
  float tau;
  const void* x;
  const float* Wr;
  const float* br;  // may be null
  float* alpha;
  int nsplit;       // CTAs per sample (the cluster size)
  int piece_px;     // pixels per bulk piece (bulk path)
  int wr_smem;      // 1: Wr staged in shared memory, partial logits per rank
  int* err;
  long long wait_ns;
  unsigned long long* stamps;  // optional [grid][8] phase stamps for measurements, or null
};

// Shared-memory carve-up, in bytes; the host sizes the launch with `total`.
struct RouteSmem {
  size_t ring, wr, partial, g, recv, brs, z, bars, flag, total;
};

__host__ __device__ inline RouteSmem route_smem(int C, int n, int VEC, int elem_bytes,
                                                int nsplit, int piece_px, int wr_smem,
                                                bool bulk) {
  const int nv = C / VEC;
  const int tpp = nv < kRouteThreads ? nv : kRouteThreads;
  const int lanes_p = kRouteThreads / tpp;
  RouteSmem s{};
  size_t off = 0;
  auto take = [&](size_t bytes, size_t align) {
    off = (off + align - 1) / align * align;
    const size_t at = off;
    off += bytes;
    return at;
  };
  const size_t piece = static_cast<size_t>(piece_px) * C * elem_bytes;
  s.ring = take(bulk ? kRouteRing * piece : 0, 128);
  s.wr = take(wr_smem ? static_cast<size_t>(n) * C * 4 : 0, 128);
  s.partial = take(static_cast<size_t>(lanes_p) * C * 4, 16);
  s.g = take(static_cast<size_t>(C) * 4, 16);
  s.recv = take(static_cast<size_t>(nsplit) * (wr_smem ? n : C) * 4, 16);
  s.brs = take(static_cast<size_t>(n) * 4, 16);
  s.z = take(static_cast<size_t>(n) * 4, 16);
  s.bars = take((kRouteRing + 1) * 8, 8);
  s.flag = take(4, 4);
  s.total = off;
  return s;
}

template <typename T, int VEC>
__device__ __forceinline__ void add_vec(const void* src, float (&acc)[VEC]) {
  if constexpr (VEC * sizeof(T) == 16) {
    const uint4 u = *reinterpret_cast<const uint4*>(src);
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
    const T* v = static_cast<const T*>(src);
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] += to_f32<T>(v[j]);
  }
}

template <typename T, int VEC>
__global__ void __launch_bounds__(kRouteThreads, 2) route_kernel(RouteParams p) {
  namespace cg = cooperative_groups;
  constexpr bool kBulk = VEC * sizeof(T) == 16;
  cg::cluster_group cluster = cg::this_cluster();
  const int rank = static_cast<int>(cluster.block_rank());
  const int nsplit = p.nsplit;
  const int b = blockIdx.y;
  const int t = threadIdx.x;
  // the forward kernel may be scheduled as soon as every routing CTA runs; it
  // waits for this grid's completion before it reads alpha
  grid_launch_dependents();
  // launched with a programmatic edge: the set-up below reads no global
  // memory; x, Wr, br and alpha are touched only after the wait

  extern __shared__ __align__(128) unsigned char route_raw[];
  const int C = p.C;
  const RouteSmem L = route_smem(C, p.n, VEC, static_cast<int>(sizeof(T)), nsplit, p.piece_px,
                                 p.wr_smem, kBulk && p.piece_px > 0);
  float* wr_s = reinterpret_cast<float*>(route_raw + L.wr);
  float* partial = reinterpret_cast<float*>(route_raw + L.partial);  // [lanes_p][C]
  float* g = reinterpret_cast<float*>(route_raw + L.g);              // [C]
  float* recv = reinterpret_cast<float*>(route_raw + L.recv);        // rank 0: [nsplit][n or C]
  float* brs = reinterpret_cast<float*>(route_raw + L.brs);          // [n]
  float* z = reinterpret_cast<float*>(route_raw + L.z);              // [n]
  const uint32_t ring = smem_u32(route_raw + L.ring);
  const uint32_t bar0 = smem_u32(route_raw + L.bars);
  const uint32_t wrbar = bar0 + 8u * kRouteRing;  // after the ring's barriers
  volatile int* abort_flag = reinterpret_cast<volatile int*>(route_raw + L.flag);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  const int nv = C / VEC;                                  // vectors per pixel
  const int tpp = nv < kRouteThreads ? nv : kRouteThreads;  // threads per pixel
  const int lanes_p = kRouteThreads / tpp;                  // pixels in flight per step
  const int pl = t / tpp;
  const size_t row_bytes = static_cast<size_t>(C) * sizeof(T);

  // ---- this CTA's pixel slice
  const int p_begin = static_cast<int>((static_cast<long long>(p.HW) * rank) / nsplit);
  const int p_end = static_cast<int>((static_cast<long long>(p.HW) * (rank + 1)) / nsplit);
  const int npx = p_end - p_begin;
  const unsigned char* src =
      static_cast<const unsigned char*>(p.x) + (static_cast<size_t>(b) * p.HW + p_begin) * row_bytes;
  const int piece_px = p.piece_px;
  const int npieces = (kBulk && piece_px > 0) ? (npx + piece_px - 1) / piece_px : 0;
  const size_t piece_bytes = static_cast<size_t>(piece_px) * row_bytes;
  int issued = 0;  // pieces issued (thread 0 only)
  auto issue = [&](int k) {
    ++issued;
    const int px = min(piece_px, npx - k * piece_px);
    const uint32_t bytes = static_cast<uint32_t>(px * row_bytes);
    const int slot = k % kRouteRing;
    mbar_arrive_expect_tx(bar0 + 8u * slot, bytes);
    bulk_load(ring + static_cast<uint32_t>(slot * piece_bytes), src + k * piece_bytes, bytes,
              bar0 + 8u * slot);
  };

  if (t == 0) {
    for (int r = 0; r < kRouteRing; ++r) mbar_init(bar0 + 8u * r, 1);
    mbar_init(wrbar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  // phase stamps (measurement hook): [0] entry, [1] past the grid wait, [2]
  // slice summed, [3] past the cluster barrier, [5] end, [6] SM id, [7]
  // global timer at entry
  unsigned long long* stp =
      (p.stamps != nullptr && t == 0) ? p.stamps + (static_cast<size_t>(b) * nsplit + rank) * 8 : nullptr;
  if (stp) {
    stp[0] = clock64();
    stp[7] = globaltimer_ns();
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    stp[6] = smid;
  }
  grid_dependency_wait();
  if (stp) stp[1] = clock64();
  if (t == 0) {
    if (p.wr_smem) {
      const uint32_t wb = static_cast<uint32_t>(p.n) * C * 4u;
      mbar_arrive_expect_tx(wrbar, wb);
      bulk_load(smem_u32(wr_s), p.Wr, wb, wrbar);
    }
    for (int k = 0; k < npieces && k < kRouteRing; ++k) issue(k);
  }
  __syncthreads();

  // ---- per-thread channel sums over the slice, fixed order
  if (npieces > 0) {
    // bulk path: one channel vector per thread (nv <= 256), pieces consumed in order
    const int v = t % tpp;
    const bool active = pl < lanes_p;
    float acc[VEC];
#pragma unroll
    for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
    for (int k = 0; k < npieces; ++k) {
      const bool ok = wait_bounded(bar0 + 8u * (k % kRouteRing),
                                   static_cast<uint32_t>(k / kRouteRing) & 1u, ctl,
                                   kErrWaitRoute);
      if (ok && active) {
        const int pk = min(piece_px, npx - k * piece_px);
        const unsigned char* base = route_raw + L.ring + (k % kRouteRing) * piece_bytes;
        for (int px = pl; px < pk; px += lanes_p)
          add_vec<T, VEC>(base + px * row_bytes + v * (VEC * sizeof(T)), acc);
      }
      __syncthreads();  // every reader is done with this slot
      if (t == 0 && k + kRouteRing < npieces && ok) issue(k + kRouteRing);
    }
    if (active) {
#pragma unroll
      for (int j = 0; j < VEC; ++j) partial[static_cast<size_t>(pl) * C + v * VEC + j] = acc[j];
    }
  } else {
    // register path: rows that are not 16-byte multiples, or very wide rows
    const T* xb = reinterpret_cast<const T*>(src);
    for (int v = t % tpp; v < nv && pl < lanes_p; v += tpp) {
      float acc[VEC];
#pragma unroll
      for (int j = 0; j < VEC; ++j) acc[j] = 0.f;
      for (int px = pl; px < npx; px += lanes_p)
        add_vec<T, VEC>(xb + static_cast<size_t>(px) * C + v * VEC, acc);
#pragma unroll
      for (int j = 0; j < VEC; ++j) partial[static_cast<size_t>(pl) * C + v * VEC + j] = acc[j];
    }
  }
  if (stp) stp[2] = clock64();
  if (rank == 0)  // read now: its latency overlaps the reductions below
    for (int i = t; i < p.n; i += kRouteThreads) brs[i] = p.br ? p.br[i] : 0.f;
  __syncthreads();
  for (int c = t; c < C; c += kRouteThreads) {
    float s = 0.f;
    for (int l = 0; l < lanes_p; ++l) s += partial[static_cast<size_t>(l) * C + c];
    g[c] = s;
  }
  __syncthreads();

  const int warp = t >> 5, lane = t & 31;
  if (p.wr_smem) {
    // partial logits of this slice, pushed into rank 0's slot for this rank
    const bool ok = wait_bounded(wrbar, 0, ctl, kErrWaitRoute);
    float* dst = cluster.map_shared_rank(recv, 0) + static_cast<size_t>(rank) * p.n;
    for (int i = warp; i < p.n; i += kRouteThreads / 32) {
      float s = 0.f;
      if (ok)
        for (int c = lane; c < C; c += 32) s = fmaf(wr_s[static_cast<size_t>(i) * C + c], g[c], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) dst[i] = s;
    }
  } else {
    float* dst = cluster.map_shared_rank(recv, 0) + static_cast<size_t>(rank) * C;
    for (int c = t; c < C; c += kRouteThreads) dst[c] = g[c];
  }
  cluster.sync();  // remote stores visible to rank 0; with Wr staged, peers may exit after this
  if (stp) {
    stp[3] = clock64();
    stp[5] = stp[3];
  }
  if (*abort_flag && t == 0) {
    // a bounded wait gave up: let the copies still in flight land before exit
    for (int k = (issued > kRouteRing ? issued - kRouteRing : 0); k < issued; ++k)
      wait_drain(bar0 + 8u * (k % kRouteRing), static_cast<uint32_t>(k / kRouteRing) & 1u,
                 p.wait_ns, p.err);
    if (p.wr_smem) wait_drain(wrbar, 0, p.wait_ns, p.err);
  }
  const float inv_hw = 1.0f / static_cast<float>(p.HW);
  if (!p.wr_smem) {
    // Wr too large to stage: the linear layer is split over the ranks by
    // expert. Every rank adds the ranks' channel sums held by rank 0 (DSMEM
    // reads, rank order) into the mean, computes the logits of experts
    // rank, rank + nsplit, ... (one warp per expert, Wr rows read from L2) and
    // pushes them into rank 0's z; every rank reaches both cluster barriers.
    const float* r0 = cluster.map_shared_rank(recv, 0);
    for (int c = t; c < C; c += kRouteThreads) {
      float s = 0.f;
      for (int r = 0; r < nsplit; ++r) s += r0[static_cast<size_t>(r) * C + c];
      g[c] = s * inv_hw;
    }
    __syncthreads();
    float* zdst = cluster.map_shared_rank(z, 0);
    for (int i = rank + warp * nsplit; i < p.n; i += (kRouteThreads / 32) * nsplit) {
      const float* wr = p.Wr + static_cast<size_t>(i) * C;
      float s = 0.f;
      for (int c = lane; c < C; c += 32) s = fmaf(wr[c], g[c], s);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) zdst[i] = s;
    }
    cluster.sync();  // logits at rank 0; nobody reads rank 0's channel sums any more
    if (rank != 0) return;
    for (int i = t; i < p.n; i += kRouteThreads) z[i] += brs[i];
    __syncthreads();
  } else if (rank != 0) {
    return;
  }
  float* out = p.alpha + static_cast<size_t>(b) * p.n;
  if (p.wr_smem && p.n <= 32) {
    // warp 0 alone: lane i sums expert i's partial logits, then the activation
    if (warp == 0) {
      float zi = -INFINITY;
      if (lane < p.n) {
        float s = 0.f;
        for (int r = 0; r < nsplit; ++r) s += recv[static_cast<size_t>(r) * p.n + lane];
        zi = s * inv_hw + brs[lane];
      }
      if (p.mode == 0) {
        if (lane < p.n) out[lane] = 1.0f / (1.0f + expf(-zi));
      } else {
        const float zt = lane < p.n ? zi / p.tau : -INFINITY;
        float m = zt;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
        const float e = lane < p.n ? expf(zt - m) : 0.f;
        float s = e;
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (lane < p.n) out[lane] = e * (1.0f / s);
      }
      if (stp) stp[5] = clock64();
    }
    return;
  }
  if (p.wr_smem) {
    for (int i = t; i < p.n; i += kRouteThreads) {
      float s = 0.f;
      for (int r = 0; r < nsplit; ++r) s += recv[static_cast<size_t>(r) * p.n + i];
      z[i] = s * inv_hw + brs[i];
    }
  }
  __syncthreads();

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
