// CUDA-core kernels of the layer's backward pass: channel sums, the generic
// per-sample weight gradient, the mixture's gradients (experts, biases,
// attentions), the router's gradients, the expert transposition that turns
// the input gradient into a forward convolution, the generic input gradient,
// and the pooled vector's share of the input gradient.
//
// The gradients are those of the forward definition (chain rule): the
// per-example kernel is a weighted sum of n learned static kernels
// (KernelWarehouse, abstract; CondConv, abstract), with the attentions from a
// softmax with temperature or a sigmoid of a linear layer on the average pool
// (FMDConv, abstract, for the temperature). Every sum over samples runs in
// sample order inside one thread, and every other reduction in a fixed tree:
// results do not depend on scheduling.
#pragma once

#include <cooperative_groups.h>
#include <cstdint>
#include <cuda_bf16.h>

#include "common.cuh"

namespace dcb {

using dc::from_f32;
using dc::to_f32;

constexpr int kBwThreads = 256;

// 16-byte asynchronous copy global -> shared (cp.async, L2 only); with
// valid == false nothing is read and the 16 bytes are zero-filled (src must
// still be a mapped address).
__device__ __forceinline__ void cp_async_16(uint32_t dst, const void* src, bool valid) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(valid ? 16 : 0)
               : "memory");
}
// Wait for every cp.async this thread issued.
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.commit_group;\n\tcp.async.wait_group 0;" ::: "memory");
}

// ------------------------------------------------------------ channel sums

// Channel sums in two passes. chansum_kernel: CTA (slice, sample) sums the
// pixels [slice * P_s, (slice + 1) * P_s) of v[b][p][c] (v is [B][P][C]) into
// part[b][slice][c]: thread t takes the VEC channels of vector t % cv (cv =
// C / VEC vectors per pixel) and every L-th pixel of the slice (L = 256 / cv
// pixel lanes), four 16-byte loads in flight; the L lane sums are added in
// lane order. chansum_finish_kernel adds the slices in order. VEC = 1 is the
// unvectorised form (any C, any alignment).
// CLUSTER: the slices of a sample form one thread-block cluster (at most 8);
// each CTA keeps its slice's sums in shared memory and, after a cluster
// barrier, rank 0 adds the ranks' sums in rank order (the finishing pass's
// order, so the same bits) and writes out[b][c]; no second kernel.
template <typename T, int VEC, bool CLUSTER = false>
__global__ void __launch_bounds__(kBwThreads) chansum_kernel(const T* __restrict__ v, int P, int C,
                                                             int Ps, float* __restrict__ part) {
  extern __shared__ float cs_part[];  // [L][C], then (CLUSTER) this slice's sums [C]
  float* mine = cs_part + kBwThreads * VEC;
  const int b = blockIdx.y, slice = blockIdx.x;
  const int nslices = gridDim.x;
  const int p_begin = slice * Ps, p_end = min(P, p_begin + Ps);
  const int cv = C / VEC;
  const T* vb = v + static_cast<size_t>(b) * P * C;
  for (int v0 = 0; v0 < cv; v0 += kBwThreads) {
    const int nvec = min(kBwThreads, cv - v0);
    const int L = kBwThreads / nvec;
    const int t = threadIdx.x;
    const int vi = v0 + t % nvec, lane_p = t / nvec;
    float acc[VEC];
#pragma unroll
    for (int k = 0; k < VEC; ++k) acc[k] = 0.f;
    if (lane_p < L) {
      int p = p_begin + lane_p;
      for (; p + 3 * L < p_end; p += 4 * L) {
        alignas(16) T q[4][VEC];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const T* src = vb + static_cast<size_t>(p + u * L) * C + static_cast<size_t>(vi) * VEC;
          if constexpr (VEC * sizeof(T) == 16)
            *reinterpret_cast<uint4*>(q[u]) = *reinterpret_cast<const uint4*>(src);
          else
#pragma unroll
            for (int k = 0; k < VEC; ++k) q[u][k] = src[k];
        }
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int k = 0; k < VEC; ++k) acc[k] += to_f32(q[u][k]);
      }
      for (; p < p_end; p += L) {
        const T* src = vb + static_cast<size_t>(p) * C + static_cast<size_t>(vi) * VEC;
#pragma unroll
        for (int k = 0; k < VEC; ++k) acc[k] += to_f32(src[k]);
      }
    }
    __syncthreads();
    if (lane_p < L)
#pragma unroll
      for (int k = 0; k < VEC; ++k) cs_part[lane_p * (nvec * VEC) + (t % nvec) * VEC + k] = acc[k];
    __syncthreads();
    for (int e = t; e < nvec * VEC; e += kBwThreads) {
      float s = 0.f;
      for (int l = 0; l < L; ++l) s += cs_part[l * (nvec * VEC) + e];
      if constexpr (CLUSTER)
        mine[static_cast<size_t>(v0) * VEC + e] = s;
      else
        part[(static_cast<size_t>(b) * nslices + slice) * C + static_cast<size_t>(v0) * VEC + e] = s;
    }
    if constexpr (CLUSTER) __syncthreads();  // cs_part is reused by the next chunk
  }
  if constexpr (CLUSTER) {
    namespace cg = cooperative_groups;
    cg::cluster_group cluster = cg::this_cluster();
    cluster.sync();  // every slice's sums are in its shared memory
    if (cluster.block_rank() == 0) {
      for (int c = threadIdx.x; c < C; c += kBwThreads) {
        float s = 0.f;
        for (int r = 0; r < nslices; ++r) s += cluster.map_shared_rank(mine, r)[c];
        part[static_cast<size_t>(b) * C + c] = s;
      }
    }
    cluster.sync();  // no CTA leaves while rank 0 reads its shared memory
  }
}

// out[b][c] = sum over slices, in order, of part[b][slice][c].
__global__ void __launch_bounds__(kBwThreads)
    chansum_finish_kernel(int B, int C, int nslices, const float* __restrict__ part,
                          float* __restrict__ out) {
  const long long e = static_cast<long long>(blockIdx.x) * kBwThreads + threadIdx.x;
  if (e >= 1LL * B * C) return;
  const long long b = e / C;
  const int c = static_cast<int>(e - b * C);
  float s = 0.f;
#pragma unroll 4
  for (int k = 0; k < nslices; ++k) s += part[(b * nslices + k) * C + c];
  out[e] = s;
}

// ------------------------------------------- per-sample weight gradient

struct WgdParams {
  int B, Cin, H, W, Cout, KH, KW, stride, pad, groups, Ho, Wo;
  long long wsize;  // Cout * KH * KW * Cin/groups
  const void* x;
  const void* dy;
  float* dW;        // [B][wsize]
};

// dW[b][co][kh][kw][ci] = sum over output pixels (oh, ow) of
// dy[b][oh][ow][co] * x[b][oh*s+kh-p][ow*s+kw-p][g(co)*Cg+ci] (zero outside the
// image). One thread per weight element of one sample, threads ordered input
// channel fastest, then output channel, then tap: in a dense layer a warp's x
// loads are contiguous and its dy loads one broadcast; in a depthwise layer
// (one input channel per output channel) both are contiguous runs of channels.
template <typename T>
__global__ void __launch_bounds__(kBwThreads) wgrad_direct_kernel(WgdParams p) {
  const long long o = static_cast<long long>(blockIdx.x) * kBwThreads + threadIdx.x;
  const int b = blockIdx.y;
  if (o >= p.wsize) return;
  const int Cg = p.Cin / p.groups, Coutg = p.Cout / p.groups;
  const int cil = static_cast<int>(o % Cg);
  const long long t = o / Cg;
  const int co = static_cast<int>(t % p.Cout);
  const int tap = static_cast<int>(t / p.Cout);
  const int kh = tap / p.KW, kw = tap - kh * p.KW;
  const int ci = (co / Coutg) * Cg + cil;
  const T* xb = static_cast<const T*>(p.x) + static_cast<size_t>(b) * p.H * p.W * p.Cin + ci;
  const T* dyb = static_cast<const T*>(p.dy) + static_cast<size_t>(b) * p.Ho * p.Wo * p.Cout + co;
  float acc = 0.f;
  for (int oh = 0; oh < p.Ho; ++oh) {
    const int ih = oh * p.stride + kh - p.pad;
    if (ih < 0 || ih >= p.H) continue;
    for (int ow = 0; ow < p.Wo; ++ow) {
      const int iw = ow * p.stride + kw - p.pad;
      if (iw < 0 || iw >= p.W) continue;
      acc = fmaf(to_f32(dyb[(static_cast<size_t>(oh) * p.Wo + ow) * p.Cout]),
                 to_f32(xb[(static_cast<size_t>(ih) * p.W + iw) * p.Cin]), acc);
    }
  }
  p.dW[static_cast<size_t>(b) * p.wsize + (static_cast<size_t>(co) * p.KH * p.KW + tap) * Cg +
       cil] = acc;
}

// Depthwise per-sample weight gradient (groups = C_in = C_out, stride 1,
// square K x K, bf16): dW[b][c][kh][kw] = sum over output pixels of
// dy[b][oh][ow][c] * x[b][oh+kh-p][ow+kw-p][c]. CTA = (32 channels, sample);
// bands of output rows are staged in shared memory (x with its K-1 halo rows
// and columns, zero outside the image, and dy), 16-byte loads. Thread = (lane:
// channel, threadIdx.y: kh): it slides a K-wide register window of x along each
// output row, so each output pixel costs two shared loads and K multiply-adds.
constexpr int kDwgChunk = 32;

struct DwgParams {
  int B, C, H, W, Ho, Wo, pad, band;
  const __nv_bfloat16* x;
  const __nv_bfloat16* dy;
  float* dW;  // [B][C][K][K]
};

template <int K>
__global__ void __launch_bounds__(32 * K) wgrad_dw_kernel(DwgParams p) {
  extern __shared__ __align__(16) unsigned char dwg_smem[];
  const int Wp = p.Wo + K - 1;
  __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(dwg_smem);
  __nv_bfloat16* ds = xs + static_cast<size_t>(p.band + K - 1) * Wp * kDwgChunk;
  const int lane = threadIdx.x, kh = threadIdx.y;
  const int tid = kh * 32 + lane;
  const int c0 = blockIdx.x * kDwgChunk, b = blockIdx.y;
  float acc[K];
#pragma unroll
  for (int k = 0; k < K; ++k) acc[k] = 0.f;
  for (int oh0 = 0; oh0 < p.Ho; oh0 += p.band) {
    const int R = min(p.band, p.Ho - oh0);
    __syncthreads();  // the previous band's readers are done
    const int xrows = R + K - 1;
    // asynchronous 16-byte copies (all in flight at once), zero-filled outside
    // the image and past the last channel
    for (int e = tid; e < xrows * Wp * 4; e += 32 * K) {
      const int v = e & 3, pix = e >> 2;
      const int r = pix / Wp, col = pix - r * Wp;
      const int ih = oh0 + r - p.pad, iw = col - p.pad, c = c0 + v * 8;
      const bool ok = ih >= 0 && ih < p.H && iw >= 0 && iw < p.W && c < p.C;
      const __nv_bfloat16* src =
          ok ? p.x + ((static_cast<size_t>(b) * p.H + ih) * p.W + iw) * p.C + c : p.x;
      cp_async_16(dc::smem_u32(xs + static_cast<size_t>(pix) * kDwgChunk + v * 8), src, ok);
    }
    for (int e = tid; e < R * p.Wo * 4; e += 32 * K) {
      const int v = e & 3, pix = e >> 2;
      const int r = pix / p.Wo, ow = pix - r * p.Wo, c = c0 + v * 8;
      const bool ok = c < p.C;
      const __nv_bfloat16* src =
          ok ? p.dy + ((static_cast<size_t>(b) * p.Ho + oh0 + r) * p.Wo + ow) * p.C + c : p.dy;
      cp_async_16(dc::smem_u32(ds + static_cast<size_t>(pix) * kDwgChunk + v * 8), src, ok);
    }
    cp_async_wait_all();
    __syncthreads();
    for (int r = 0; r < R; ++r) {
      // x row r + kh of the band, halo column q holds input column q - pad
      const __nv_bfloat16* xr = xs + static_cast<size_t>(r + kh) * Wp * kDwgChunk + lane;
      const __nv_bfloat16* dr = ds + static_cast<size_t>(r) * p.Wo * kDwgChunk + lane;
      // ring of K values: halo column q sits at index q % K
      float win[K];
#pragma unroll
      for (int k = 0; k < K - 1; ++k) win[k] = __bfloat162float(xr[k * kDwgChunk]);
      for (int ow0 = 0; ow0 < p.Wo; ow0 += K) {
#pragma unroll
        for (int j = 0; j < K; ++j) {
          const int ow = ow0 + j;
          if (ow < p.Wo) {
            win[(j + K - 1) % K] = __bfloat162float(xr[(ow + K - 1) * kDwgChunk]);
            const float d = __bfloat162float(dr[ow * kDwgChunk]);
#pragma unroll
            for (int k = 0; k < K; ++k) acc[k] = fmaf(d, win[(j + k) % K], acc[k]);
          }
        }
      }
    }
  }
  const int c = c0 + lane;
  if (c < p.C)
#pragma unroll
    for (int kw = 0; kw < K; ++kw)
      p.dW[((static_cast<size_t>(b) * p.C + c) * K + kh) * K + kw] = acc[kw];
}

// ------------------------------------------------ the mixture's gradients

constexpr int kMgMaxExperts = 8;     // experts per CTA at most (grid.y walks the rest)
constexpr int kMgChunk = 4 * kBwThreads;  // weights per CTA: four per thread
constexpr int kMgSampleBlock = 32;   // samples per partial-sum round

struct MgParams {
  int B, n;
  long long wsize;
  int chunks;            // ceil(wsize / kMgChunk)
  int vec;               // wsize % 4 == 0 and 16-byte aligned dW, dexperts
  const float* dW;       // [B][wsize] per-sample weight gradients
  const void* experts;   // [n][wsize], T
  const float* alpha;    // [B][n]
  float* dexperts;       // [n][wsize], or with bsplit > 1 partials [bsplit][n][wsize]
  float* part;           // [chunks][B][n]: sum over this chunk of dW[b][w] * E[i][w]
  int bsplit;            // sample groups (grid.z), each of bs samples
  int bs;
};

// dexperts[i][w] = sum_b alpha[b][i] dW[b][w] for the CTA's 1024 weights and
// NE experts (fewer in the last group), over the CTA's group of samples, and
// the chunk's share of dalpha[b][i] = <dW_b, E_i>. Each thread holds four
// weights: per sample one 16-byte load of dW (eight samples' loads in flight),
// four multiply-adds per expert into dexperts and four into the dot product.
// The dot products of SU samples x NE experts (32 values per lane) are summed
// over the warp by a transpose through shared memory: lane l writes its values
// as row l of a 32 x 33 tile, lane j adds column j in row order. The warps'
// sums meet in shared memory and are added in warp order.
template <typename T, int NE>
__global__ void __launch_bounds__(kBwThreads) mixgrad_kernel(MgParams p) {
  constexpr int SU = (32 / NE) < 8 ? (32 / NE) : 8;  // samples per reduction
  extern __shared__ float mg_smem[];
  float* alpha_s = mg_smem;                                          // [B][NE]
  float* red = alpha_s + static_cast<size_t>(p.B) * NE;              // [8][32][NE]
  float* tiles = red + (kBwThreads / 32) * kMgSampleBlock * NE;      // [8][32][33]
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* tl = tiles + warp * (32 * 33);
  const int chunk = blockIdx.x;
  const int i0 = blockIdx.y * NE;
  const int ne = min(NE, p.n - i0);
  for (int e = threadIdx.x; e < p.B * NE; e += kBwThreads) {
    const int b = e / NE, i = e - b * NE;
    alpha_s[e] = i < ne ? p.alpha[static_cast<size_t>(b) * p.n + i0 + i] : 0.f;
  }
  const long long w = static_cast<long long>(chunk) * kMgChunk + threadIdx.x * 4;
  const T* E = static_cast<const T*>(p.experts);
  float ev[NE][4];
#pragma unroll
  for (int i = 0; i < NE; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k)
      ev[i][k] = (i < ne && w + k < p.wsize)
                     ? to_f32(E[static_cast<size_t>(i0 + i) * p.wsize + w + k])
                     : 0.f;
  float dex[NE][4];
#pragma unroll
  for (int i = 0; i < NE; ++i)
#pragma unroll
    for (int k = 0; k < 4; ++k) dex[i][k] = 0.f;
  __syncthreads();

  const int b_begin = blockIdx.z * p.bs, b_end = min(p.B, b_begin + p.bs);
  for (int b0 = b_begin; b0 < b_end; b0 += kMgSampleBlock) {
    const int nbb = min(kMgSampleBlock, b_end - b0);
    for (int bb0 = 0; bb0 < nbb; bb0 += 8) {
      // eight samples' loads in flight before the math
      float v[8][4];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const float* src = p.dW + static_cast<size_t>(b0 + bb0 + u) * p.wsize + w;
        if (bb0 + u >= nbb || w >= p.wsize) {
#pragma unroll
          for (int k = 0; k < 4; ++k) v[u][k] = 0.f;
        } else if (p.vec) {
          const float4 q = *reinterpret_cast<const float4*>(src);
          v[u][0] = q.x; v[u][1] = q.y; v[u][2] = q.z; v[u][3] = q.w;
        } else {
#pragma unroll
          for (int k = 0; k < 4; ++k) v[u][k] = w + k < p.wsize ? src[k] : 0.f;
        }
      }
#pragma unroll
      for (int h = 0; h < 8; h += SU) {
#pragma unroll
        for (int u = 0; u < SU; ++u) {
          // samples past the group have v = 0 and alpha rows that are not read
          const int bq = min(b0 + bb0 + h + u, p.B - 1);
          const float* ab = alpha_s + static_cast<size_t>(bq) * NE;
#pragma unroll
          for (int i = 0; i < NE; ++i) {
            const float a = ab[i];
            float d = 0.f;
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              dex[i][k] = fmaf(a, v[h + u][k], dex[i][k]);
              d = fmaf(v[h + u][k], ev[i][k], d);
            }
            tl[lane * 33 + u * NE + i] = d;
          }
        }
        __syncwarp();
        if (lane < SU * NE) {
          float sum = 0.f;
#pragma unroll 8
          for (int l = 0; l < 32; ++l) sum += tl[l * 33 + lane];
          const int bb = bb0 + h + lane / NE;
          if (bb < nbb) red[(warp * kMgSampleBlock + bb) * NE + lane % NE] = sum;
        }
        __syncwarp();
      }
    }
    __syncthreads();
    for (int e = threadIdx.x; e < nbb * ne; e += kBwThreads) {
      const int bb = e / ne, i = e - bb * ne;
      float s = 0.f;
      for (int wp = 0; wp < kBwThreads / 32; ++wp) s += red[(wp * kMgSampleBlock + bb) * NE + i];
      p.part[(static_cast<size_t>(chunk) * p.B + b0 + bb) * p.n + i0 + i] = s;
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < NE; ++i) {
    if (i < ne) {
      float* dst = p.dexperts + (static_cast<size_t>(blockIdx.z) * p.n + i0 + i) * p.wsize + w;
      if (p.vec && w < p.wsize) {
        *reinterpret_cast<float4*>(dst) = make_float4(dex[i][0], dex[i][1], dex[i][2], dex[i][3]);
      } else {
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (w + k < p.wsize) dst[k] = dex[i][k];
      }
    }
  }
}

// dexperts[e] = sum over sample groups, in order, of part[g][e] (e over
// n * wsize), four elements per thread.
__global__ void __launch_bounds__(kBwThreads)
    dexperts_finish_kernel(long long total, int groups, const float* __restrict__ part,
                           float* __restrict__ dexperts) {
  for (long long e = (static_cast<long long>(blockIdx.x) * kBwThreads + threadIdx.x) * 4; e < total;
       e += static_cast<long long>(gridDim.x) * kBwThreads * 4) {
    float s[4] = {0.f, 0.f, 0.f, 0.f};
    for (int g = 0; g < groups; ++g)
#pragma unroll
      for (int k = 0; k < 4; ++k)
        if (e + k < total) s[k] += part[static_cast<size_t>(g) * total + e + k];
#pragma unroll
    for (int k = 0; k < 4; ++k)
      if (e + k < total) dexperts[e + k] = s[k];
  }
}

// dalpha[b][i] = sum over chunks of part[chunk][b][i]
//              + sum_co db[b][co] * bias[i][co]    (bias may be NULL).
// One CTA per sample. With n < 256 the chunks and the output channels are
// split into S = 256 / n interleaved slices (thread t: expert t % n, slice
// t / n), each summed in order by one thread; the slice sums are then added
// in slice order.
__global__ void __launch_bounds__(kBwThreads)
    dalpha_finish_kernel(int B, int n, int Cout, int chunks, const float* __restrict__ part,
                         const float* __restrict__ db, const float* __restrict__ bias,
                         float* __restrict__ dalpha) {
  __shared__ float slice_sum[kBwThreads];
  const int b = blockIdx.x;
  const int S = n < kBwThreads ? kBwThreads / n : 1;
  for (int i0 = 0; i0 < n; i0 += kBwThreads) {
    const int i = i0 + (S > 1 ? static_cast<int>(threadIdx.x) % n : static_cast<int>(threadIdx.x));
    const int sl = S > 1 ? static_cast<int>(threadIdx.x) / n : 0;
    float s = 0.f;
    if (i < n && sl < S) {
#pragma unroll 8
      for (int c = sl; c < chunks; c += S) s += part[(static_cast<size_t>(c) * B + b) * n + i];
      if (bias) {
        // this slice's share of <db_b, bias_i>
        float t = 0.f;
#pragma unroll 8
        for (int co = sl; co < Cout; co += S)
          t = fmaf(db[static_cast<size_t>(b) * Cout + co], bias[static_cast<size_t>(i) * Cout + co], t);
        s += t;
      }
    }
    slice_sum[threadIdx.x] = s;
    __syncthreads();
    if (sl == 0 && i < n) {
      float tot = 0.f;
      for (int k = 0; k < S; ++k) tot += slice_sum[k * (S > 1 ? n : 0) + threadIdx.x];
      dalpha[static_cast<size_t>(b) * n + i] = tot;
    }
    __syncthreads();
  }
}

// dbias[i][co] = sum_b alpha[b][i] * db[b][co]. CTA = (32 channels, up to 8
// experts); thread (lane: channel, y: one of 8 interleaved sample slices)
// sums its slice for each expert; the slices are added in order.
__global__ void __launch_bounds__(256)
    dbias_kernel(int B, int n, int Cout, const float* __restrict__ alpha,
                 const float* __restrict__ db, float* __restrict__ dbias) {
  __shared__ float red[8][8][33];  // [slice][expert][channel]
  const int co = blockIdx.x * 32 + threadIdx.x;
  const int i0 = blockIdx.y * 8, ne = min(8, n - i0);
  float acc[8];
#pragma unroll
  for (int k = 0; k < 8; ++k) acc[k] = 0.f;
  if (co < Cout)
    for (int b = threadIdx.y; b < B; b += 8) {
      const float d = db[static_cast<size_t>(b) * Cout + co];
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (k < ne) acc[k] = fmaf(alpha[static_cast<size_t>(b) * n + i0 + k], d, acc[k]);
    }
#pragma unroll
  for (int k = 0; k < 8; ++k) red[threadIdx.y][k][threadIdx.x] = acc[k];
  __syncthreads();
  if (threadIdx.y < ne && co < Cout) {
    const int k = threadIdx.y;
    float s = 0.f;
#pragma unroll
    for (int sl = 0; sl < 8; ++sl) s += red[sl][k][threadIdx.x];
    dbias[static_cast<size_t>(i0 + k) * Cout + co] = s;
  }
}

// ------------------------------------------------------ router gradients

// dz[b][i] from the attention's gradient through the activation:
// sigmoid: dalpha * alpha * (1 - alpha); softmax of z/tau:
// alpha_i * (dalpha_i - sum_j alpha_j dalpha_j) / tau, the sum over j in order.
__device__ __forceinline__ float dz_of(const float* a, const float* da, int n, int i, int mode,
                                       float tau) {
  if (mode == 0) return da[i] * a[i] * (1.f - a[i]);
  float dot = 0.f;
  for (int j = 0; j < n; ++j) dot = fmaf(a[j], da[j], dot);
  return a[i] * (da[i] - dot) / tau;
}

// Router parameters: dWr[i][c] = sum_b dz[b][i] * gsum[b][c] / HW and
// dbr[i] = sum_b dz[b][i]. Grid (ceil(C / (256 / slices)), n): the CTA first
// takes dz[b][i] for every sample into shared memory (one thread per sample);
// then `slices` (1, 2, 4 or 8) groups of its threads each sum a contiguous
// part of the samples for 256 / slices consecutive channels (coalesced rows
// of gsum), and the first group adds the partial sums in group order -- a
// fixed order, with `slices` chains per channel instead of one over the batch.
constexpr int kRbpMaxSlices = 8;
__global__ void __launch_bounds__(kBwThreads)
    route_bwd_param_kernel(int B, int C, int n, int slices, float inv_hw, int mode, float tau,
                           const float* __restrict__ alpha, const float* __restrict__ dalpha,
                           const float* __restrict__ gsum, float* __restrict__ dWr,
                           float* __restrict__ dbr) {
  extern __shared__ float dz_s[];  // [B], then the partial sums [slices][256 / slices]
  float* part = dz_s + ((B + 3) & ~3);
  const int i = blockIdx.y;
  for (int b = threadIdx.x; b < B; b += kBwThreads)
    dz_s[b] = dz_of(alpha + static_cast<size_t>(b) * n, dalpha + static_cast<size_t>(b) * n, n,
                    i, mode, tau);
  __syncthreads();
  const int cpc = kBwThreads / slices;  // channels per CTA
  const int lane = threadIdx.x % cpc, q = threadIdx.x / cpc;
  const int c = blockIdx.x * cpc + lane;
  const int per = (B + slices - 1) / slices;
  const int b0 = q * per, b1 = min(B, b0 + per);
  float s = 0.f;
  if (c < C) {
#pragma unroll 8
    for (int b = b0; b < b1; ++b) s = fmaf(dz_s[b], gsum[static_cast<size_t>(b) * C + c], s);
  }
  part[threadIdx.x] = s;  // = part[q * cpc + lane]
  __syncthreads();
  if (q == 0 && c < C) {
    float t = 0.f;
    for (int k = 0; k < slices; ++k) t += part[k * cpc + lane];
    dWr[static_cast<size_t>(i) * C + c] = t * inv_hw;
  }
  if (dbr && blockIdx.x == 0 && threadIdx.x == 0) {
    float t = 0.f;
    for (int b = 0; b < B; ++b) t += dz_s[b];
    dbr[i] = t;
  }
}

// The pooled vector's gradient: dg[b][c] = sum_i dz[b][i] * Wr[i][c]. Grid
// (ceil(C / 256), B); dz of the sample goes to shared memory first (the
// softmax's sum over j by a fixed tree).
__global__ void __launch_bounds__(kBwThreads)
    route_bwd_dg_kernel(int C, int n, int mode, float tau, const float* __restrict__ alpha,
                        const float* __restrict__ dalpha, const float* __restrict__ Wr,
                        float* __restrict__ dg) {
  extern __shared__ float rd_s[];  // dz [n] then the tree [256]
  float* dz = rd_s;
  float* tree = rd_s + n;
  const int b = blockIdx.y;
  const float* a = alpha + static_cast<size_t>(b) * n;
  const float* da = dalpha + static_cast<size_t>(b) * n;
  float dot = 0.f;
  if (mode == 1) {
    float s = 0.f;
    for (int j = threadIdx.x; j < n; j += kBwThreads) s = fmaf(a[j], da[j], s);
    tree[threadIdx.x] = s;
    __syncthreads();
    for (int off = kBwThreads / 2; off > 0; off >>= 1) {
      if (threadIdx.x < off) tree[threadIdx.x] += tree[threadIdx.x + off];
      __syncthreads();
    }
    dot = tree[0];
  }
  for (int i = threadIdx.x; i < n; i += kBwThreads)
    dz[i] = mode == 0 ? da[i] * a[i] * (1.f - a[i]) : a[i] * (da[i] - dot) / tau;
  __syncthreads();
  const int c = blockIdx.x * kBwThreads + threadIdx.x;
  if (c < C) {
    float s = 0.f;
    for (int i = 0; i < n; ++i) s = fmaf(dz[i], Wr[static_cast<size_t>(i) * C + c], s);
    dg[static_cast<size_t>(b) * C + c] = s;
  }
}

// ------------------------------------------------------- input gradient

// Et[i][ci][kh][kw][col] = E[i][g*Coutg + col][KH-1-kh][KW-1-kw][ci - g*Cg],
// g = ci / Cg: every expert with input and output channels swapped within
// its group and flipped in both spatial axes, so that the input gradient of
// the convolution is a forward convolution of dy with the same attentions.
// One thread per output element (grid-stride), writes contiguous.
template <typename T>
__global__ void __launch_bounds__(kBwThreads)
    transpose_experts_kernel(int n, int Cin, int Cout, int KH, int KW, int groups,
                             const T* __restrict__ E, T* __restrict__ Et) {
  const int Cg = Cin / groups, Coutg = Cout / groups;
  const long long total = 1LL * n * Cin * KH * KW * Coutg;
  for (long long o = static_cast<long long>(blockIdx.x) * kBwThreads + threadIdx.x; o < total;
       o += static_cast<long long>(gridDim.x) * kBwThreads) {
    long long t = o;
    const int col = static_cast<int>(t % Coutg);
    t /= Coutg;
    const int kw = static_cast<int>(t % KW);
    t /= KW;
    const int kh = static_cast<int>(t % KH);
    t /= KH;
    const int ci = static_cast<int>(t % Cin);
    const long long i = t / Cin;
    const int g = ci / Cg;
    const int co = g * Coutg + col;
    const size_t src = ((((static_cast<size_t>(i) * Cout + co) * KH + (KH - 1 - kh)) * KW +
                         (KW - 1 - kw)) * Cg) + (ci - g * Cg);
    Et[o] = E[src];
  }
}

struct DgdParams {
  int B, Cin, H, W, Cout, KH, KW, stride, pad, groups, Ho, Wo, n;
  const void* dy;
  const void* experts;
  const float* alpha;
  const float* dg;   // [B][Cin] or NULL
  float inv_hw;
  void* dx;
};

// Generic input gradient (any stride, padding, groups): one thread per
// element of dx, summing dy * W_b over the (output pixel, tap) pairs that
// read it, W_b mixed on the fly from the experts; plus dg/(H*W); rounded once.
template <typename T>
__global__ void __launch_bounds__(kBwThreads) dgrad_direct_kernel(DgdParams p) {
  const long long total = 1LL * p.B * p.H * p.W * p.Cin;
  const long long o = static_cast<long long>(blockIdx.x) * kBwThreads + threadIdx.x;
  if (o >= total) return;
  const int ci = static_cast<int>(o % p.Cin);
  long long t = o / p.Cin;
  const int iw = static_cast<int>(t % p.W);
  t /= p.W;
  const int ih = static_cast<int>(t % p.H);
  const int b = static_cast<int>(t / p.H);
  const int Cg = p.Cin / p.groups, Coutg = p.Cout / p.groups;
  const int g = ci / Cg, cil = ci - g * Cg;
  const T* E = static_cast<const T*>(p.experts);
  const T* dyb = static_cast<const T*>(p.dy) + static_cast<size_t>(b) * p.Ho * p.Wo * p.Cout;
  const float* ab = p.alpha + static_cast<size_t>(b) * p.n;
  const size_t wsize = static_cast<size_t>(p.Cout) * p.KH * p.KW * Cg;
  float acc = 0.f;
  for (int kh = 0; kh < p.KH; ++kh) {
    const int th = ih + p.pad - kh;
    if (th < 0 || th % p.stride) continue;
    const int oh = th / p.stride;
    if (oh >= p.Ho) continue;
    for (int kw = 0; kw < p.KW; ++kw) {
      const int tw = iw + p.pad - kw;
      if (tw < 0 || tw % p.stride) continue;
      const int ow = tw / p.stride;
      if (ow >= p.Wo) continue;
      for (int col = 0; col < Coutg; ++col) {
        const int co = g * Coutg + col;
        const size_t widx = ((static_cast<size_t>(co) * p.KH + kh) * p.KW + kw) * Cg + cil;
        float wv = 0.f;
        for (int i = 0; i < p.n; ++i) wv = fmaf(ab[i], to_f32(E[i * wsize + widx]), wv);
        acc = fmaf(to_f32(dyb[(static_cast<size_t>(oh) * p.Wo + ow) * p.Cout + co]), wv, acc);
      }
    }
  }
  if (p.dg) acc += p.dg[static_cast<size_t>(b) * p.Cin + ci] * p.inv_hw;
  static_cast<T*>(p.dx)[o] = from_f32<T>(acc);
}

// Et = every expert transposed within its group and flipped in both spatial
// axes, as transpose_experts_kernel, through 32 x 32 tiles of shared memory
// so that both the reads (input channels contiguous) and the writes (output
// channels contiguous) are coalesced. Grid (tiles of the group's [Coutg][Cg]
// matrix, taps * groups, n); block (32, 8).
template <typename T>
__global__ void __launch_bounds__(256)
    transpose_experts_tiled_kernel(int Cin, int Cout, int KH, int KW, int groups,
                                   const T* __restrict__ E, T* __restrict__ Et) {
  __shared__ T tile[32][33];
  const int Cg = Cin / groups, Coutg = Cout / groups;
  const int tiles_c = (Cg + 31) / 32;
  const int cil0 = (blockIdx.x % tiles_c) * 32, col0 = (blockIdx.x / tiles_c) * 32;
  const int taps = KH * KW;
  const int tap = blockIdx.y % taps, g = blockIdx.y / taps;
  const int kh = tap / KW, kw = tap - kh * KW;
  const int tap_src = (KH - 1 - kh) * KW + (KW - 1 - kw);
  const size_t i = blockIdx.z;
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int col = col0 + r, cil = cil0 + threadIdx.x;
    T v = from_f32<T>(0.f);
    if (col < Coutg && cil < Cg)
      v = E[((i * Cout + g * Coutg + col) * taps + tap_src) * Cg + cil];
    tile[r][threadIdx.x] = v;
  }
  __syncthreads();
  for (int r = threadIdx.y; r < 32; r += 8) {
    const int cil = cil0 + r, col = col0 + threadIdx.x;
    if (col < Coutg && cil < Cg)
      Et[((i * Cin + g * Cg + cil) * taps + tap) * Coutg + col] = tile[threadIdx.x][r];
  }
}

// The same flipped transposition for bf16 with both channel counts of a
// group multiples of 8, in 64 x 64 tiles moved as 16-byte chunks: a CTA reads
// 64 output-channel rows of 128 contiguous bytes, stages them in shared
// memory (row pitch 66 elements, so the column gathers spread over the
// banks) and writes 64 input-channel rows of 128 contiguous bytes. Grid
// (tiles of the group's [Coutg][Cg] matrix, taps * groups, n); 256 threads.
__global__ void __launch_bounds__(256)
    transpose_experts_v8_kernel(int Cin, int Cout, int KH, int KW, int groups,
                                const __nv_bfloat16* __restrict__ E, __nv_bfloat16* __restrict__ Et) {
  constexpr int kPitch = 66;  // elements per staged row
  __shared__ __align__(16) unsigned short tile[64 * kPitch];
  const int Cg = Cin / groups, Coutg = Cout / groups;
  const int tiles_c = (Cg + 63) / 64;
  const int cil0 = (blockIdx.x % tiles_c) * 64, col0 = (blockIdx.x / tiles_c) * 64;
  const int taps = KH * KW;
  const int tap = blockIdx.y % taps, g = blockIdx.y / taps;
  const int kh = tap / KW, kw = tap - kh * KW;
  const int tap_src = (KH - 1 - kh) * KW + (KW - 1 - kw);
  const size_t i = blockIdx.z;
  for (int u = threadIdx.x; u < 512; u += 256) {
    const int r = u >> 3, c8 = (u & 7) * 8;  // output-channel row, input-channel offset
    const int col = col0 + r, cil = cil0 + c8;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (col < Coutg && cil < Cg)
      v = *reinterpret_cast<const uint4*>(E + ((i * Cout + g * Coutg + col) * taps + tap_src) * Cg + cil);
    uint32_t* dst = reinterpret_cast<uint32_t*>(tile + r * kPitch + c8);
    dst[0] = v.x; dst[1] = v.y; dst[2] = v.z; dst[3] = v.w;
  }
  __syncthreads();
  for (int u = threadIdx.x; u < 512; u += 256) {
    const int r = u >> 3, c8 = (u & 7) * 8;  // input-channel row, output-channel offset
    const int cil = cil0 + r, col = col0 + c8;
    uint32_t w[4];
#pragma unroll
    for (int j = 0; j < 4; ++j)
      w[j] = static_cast<uint32_t>(tile[(c8 + 2 * j) * kPitch + r]) |
             (static_cast<uint32_t>(tile[(c8 + 2 * j + 1) * kPitch + r]) << 16);
    if (col < Coutg && cil < Cg)
      *reinterpret_cast<uint4*>(Et + ((i * Cin + g * Cg + cil) * taps + tap) * Coutg + col) =
          make_uint4(w[0], w[1], w[2], w[3]);
  }
}

}  // namespace dcb
