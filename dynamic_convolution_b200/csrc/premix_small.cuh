// Kernel mixing on CUDA cores for few experts (n <= 8):
//     W[b][w] = sum_i alpha[b][i] * E[i][w]
// for every sample b and weight element w -- the per-example "linear mixture
// of n static kernels weighted with their input-dependent attentions"
// (KernelWarehouse, abstract; CondConv, abstract: one kernel per example).
//
// With n <= 8 the mixing costs at most 4 FMAs per output byte, so it is a
// store-bound stream, not a GEMM: a thread takes 8 consecutive weights (one
// 16-byte load per expert, widened to fp32 once) and a block of samples, and
// writes one 16-byte store per sample; the 32 lanes of a warp cover 512
// contiguous bytes of one sample's kernel. fp32 accumulation in expert order
// i = 0, 1, ..., one rounding to bf16 per weight.
//
// Compared with the tensor-core mixing GEMM it has no set-up chain (no TMEM,
// no barriers, no operand build), so the first stores leave one load
// round-trip after the routing weights are available.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kPsThreads = 256;
constexpr int kPsMaxExperts = 8;

struct PsParams {
  int B, n;
  int sblock;           // samples per thread (1..16)
  int sblocks;          // ceil(B / sblock)
  long long wsize;      // weight elements per expert (multiple of 8)
  long long chunks;     // wsize / 8
  long long items;      // chunks * sblocks
  const __nv_bfloat16* experts;  // [n][wsize]
  const float* alpha;            // [B][n]
  __nv_bfloat16* out;            // [B][wsize]
};

// NMAX: the expert count rounded up to 2, 4 or 8 (fewer registers for fewer experts)
template <int NMAX>
__global__ void __launch_bounds__(kPsThreads) premix_small_kernel(PsParams p) {
  extern __shared__ float ps_alpha[];  // [B][n]
  // the convolution may be scheduled as soon as every CTA of this grid runs
  grid_launch_dependents();
  grid_dependency_wait();  // alpha comes from the routing kernel
  const int na = p.B * p.n;
  for (int e = threadIdx.x; e < na; e += kPsThreads) ps_alpha[e] = p.alpha[e];
  __syncthreads();

  const long long stride = static_cast<long long>(gridDim.x) * kPsThreads;
  for (long long it = static_cast<long long>(blockIdx.x) * kPsThreads + threadIdx.x; it < p.items;
       it += stride) {
    const long long sb = it / p.chunks;
    const long long ch = it - sb * p.chunks;
    // the 8 weights of every expert, widened to packed fp32 pairs
    uint4 raw[NMAX];
#pragma unroll
    for (int i = 0; i < NMAX; ++i)
      if (i < p.n) raw[i] = ld_nc_v4(p.experts + static_cast<size_t>(i) * p.wsize + ch * 8);
    uint64_t ef[NMAX][4];
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
      if (i < p.n) {
        ef[i][0] = bf16x2_to_f32x2(raw[i].x);
        ef[i][1] = bf16x2_to_f32x2(raw[i].y);
        ef[i][2] = bf16x2_to_f32x2(raw[i].z);
        ef[i][3] = bf16x2_to_f32x2(raw[i].w);
      }
    }
    const int b0 = static_cast<int>(sb) * p.sblock;
    const int b1 = min(p.B, b0 + p.sblock);
#pragma unroll 2
    for (int b = b0; b < b1; ++b) {
      const float* ab = ps_alpha + b * p.n;
      uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
      for (int i = 0; i < NMAX; ++i) {
        if (i < p.n) {
          const float a = ab[i];
          const uint64_t a2 = pack_f32x2(a, a);
#pragma unroll
          for (int q = 0; q < 4; ++q) acc[q] = ffma2(a2, ef[i][q], acc[q]);
        }
      }
      uint4 o;
      o.x = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[0])),
                        __uint_as_float(static_cast<uint32_t>(acc[0] >> 32)));
      o.y = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[1])),
                        __uint_as_float(static_cast<uint32_t>(acc[1] >> 32)));
      o.z = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[2])),
                        __uint_as_float(static_cast<uint32_t>(acc[2] >> 32)));
      o.w = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[3])),
                        __uint_as_float(static_cast<uint32_t>(acc[3] >> 32)));
      *reinterpret_cast<uint4*>(p.out + static_cast<size_t>(b) * p.wsize + ch * 8) = o;
    }
  }
}

// Host-side plan: as many samples per thread (up to 16) as keep at least one
// CTA's worth of items per SM, so that the grid runs in a single wave (fewer
// samples per thread when the kernel is small). Returns false when the shape
// is outside this kernel.
inline bool plan_premix_small(int B, int n, long long wsize, int sms, PsParams* p,
                              unsigned* grid) {
  if (n < 1 || n > kPsMaxExperts || B < 1 || wsize % 8 != 0) return false;
  if (static_cast<long long>(B) * n * 4 > 16384) return false;
  const long long chunks = wsize / 8;
  const long long target = static_cast<long long>(sms) * kPsThreads;
  int sblock = 16;
  while (sblock > 1 && chunks * ((B + sblock - 1) / sblock) < target) sblock >>= 1;
  p->B = B;
  p->n = n;
  p->sblock = sblock;
  p->sblocks = (B + sblock - 1) / sblock;
  p->wsize = wsize;
  p->chunks = chunks;
  p->items = chunks * p->sblocks;
  const long long ctas = (p->items + kPsThreads - 1) / kPsThreads;
  *grid = static_cast<unsigned>(std::min<long long>(ctas, static_cast<long long>(sms) * 8));
  return true;
}


// ---------------------------------------------------------------------------
// The same mixing in K-slice order with per-slice publication, for a hand-off
// to the convolution that does not wait for the whole kernel: a slice is one
// tap of one 64-channel chunk of every sample's kernel (what the convolution
// consumes in one K step). Slices [0, fa) are cut into small items (few
// samples each) so that they are complete after about one load round-trip;
// the rest use larger items. After each round of 256 consecutive items a CTA
// adds the number of items it finished to each touched slice's counter
// (stores, proxy fence, CTA barrier, one cumulative fence, atomics). The
// consumer resets the counters after its last CTA finished.
struct PoParams {
  int B, n, Cin, Cout, taps, k_steps;
  long long wsize;
  int fa;                      // slices in tier A
  int sbA, nsbA, ipsA;         // samples per item, sample blocks, items per slice
  int sbB, nsbB, ipsB;
  long long nA, nB;            // items of tier A, tier B
  const __nv_bfloat16* experts;
  const float* alpha;
  __nv_bfloat16* out;
  unsigned int* counters;      // [k_steps], zero at launch
};

template <int NMAX>
__device__ __forceinline__ void mix_item(const PoParams& p, const float* alpha_s, int k, int local,
                                         int sblock) {
  const int jc = local & 7;  // 16-byte chunk of the 64-channel slice
  const int rest = local >> 3;
  const int co = rest % p.Cout;
  const int sb = rest / p.Cout;
  const int cc = k / p.taps, tap = k - cc * p.taps;
  const int ch0 = cc * 64 + jc * 8;
  if (ch0 >= p.Cin) return;
  const long long off = (static_cast<long long>(co) * p.taps + tap) * p.Cin + ch0;
  uint4 raw[NMAX];
#pragma unroll
  for (int i = 0; i < NMAX; ++i)
    if (i < p.n) raw[i] = ld_nc_v4(p.experts + i * p.wsize + off);
  uint64_t ef[NMAX][4];
#pragma unroll
  for (int i = 0; i < NMAX; ++i) {
    if (i < p.n) {
      ef[i][0] = bf16x2_to_f32x2(raw[i].x);
      ef[i][1] = bf16x2_to_f32x2(raw[i].y);
      ef[i][2] = bf16x2_to_f32x2(raw[i].z);
      ef[i][3] = bf16x2_to_f32x2(raw[i].w);
    }
  }
  const int b0 = sb * sblock;
  const int b1 = min(p.B, b0 + sblock);
#pragma unroll 2
  for (int b = b0; b < b1; ++b) {
    const float* ab = alpha_s + b * p.n;
    uint64_t acc[4] = {0ull, 0ull, 0ull, 0ull};
#pragma unroll
    for (int i = 0; i < NMAX; ++i) {
      if (i < p.n) {
        const uint64_t a2 = pack_f32x2(ab[i], ab[i]);
#pragma unroll
        for (int q = 0; q < 4; ++q) acc[q] = ffma2(a2, ef[i][q], acc[q]);
      }
    }
    uint4 o;
    o.x = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[0])),
                      __uint_as_float(static_cast<uint32_t>(acc[0] >> 32)));
    o.y = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[1])),
                      __uint_as_float(static_cast<uint32_t>(acc[1] >> 32)));
    o.z = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[2])),
                      __uint_as_float(static_cast<uint32_t>(acc[2] >> 32)));
    o.w = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[3])),
                      __uint_as_float(static_cast<uint32_t>(acc[3] >> 32)));
    *reinterpret_cast<uint4*>(p.out + static_cast<long long>(b) * p.wsize + off) = o;
  }
}

template <int NMAX>
__global__ void __launch_bounds__(kPsThreads) premix_ordered_kernel(PoParams p) {
  extern __shared__ float po_alpha[];  // [B][n]
  // the convolution may be scheduled as soon as every CTA of this grid runs;
  // it reads nothing before it has acquired the counter of slice 0
  grid_launch_dependents();
  grid_dependency_wait();  // alpha comes from the routing kernel
  const int na = p.B * p.n;
  for (int e = threadIdx.x; e < na; e += kPsThreads) po_alpha[e] = p.alpha[e];
  __syncthreads();
  const int tm = threadIdx.x;
  const long long stride = static_cast<long long>(gridDim.x) * kPsThreads;
  for (int tier = 0; tier < 2; ++tier) {
    const long long n_items = tier == 0 ? p.nA : p.nB;
    const int ips = tier == 0 ? p.ipsA : p.ipsB;
    const int sblock = tier == 0 ? p.sbA : p.sbB;
    const int k0 = tier == 0 ? 0 : p.fa;
    for (long long rb = static_cast<long long>(blockIdx.x) * kPsThreads; rb < n_items; rb += stride) {
      const long long it = rb + tm;
      if (it < n_items) {
        const int kk = static_cast<int>(it / ips);
        mix_item<NMAX>(p, po_alpha, k0 + kk, static_cast<int>(it - static_cast<long long>(kk) * ips),
                       sblock);
      }
      asm volatile("fence.proxy.async.global;" ::: "memory");  // read next by TMA
      __syncthreads();
      if (tm == 0) {
        __threadfence();  // cumulative over the CTA's stores ordered by the barrier
        const long long hi = min(rb + kPsThreads, n_items);
        for (long long kk = rb / ips; kk * ips < hi; ++kk) {
          const long long s0 = max(rb, kk * ips);
          const long long s1 = min(hi, (kk + 1) * ips);
          atomicAdd(p.counters + k0 + kk, static_cast<unsigned int>(s1 - s0));
        }
      }
    }
  }
}

// Host-side plan of the slice-ordered mixing. Returns false when the shape is
// outside it.
inline bool plan_premix_ordered(int B, int n, int Cin, int Cout, int taps, int k_steps, int sms,
                                PoParams* p, unsigned* grid) {
  if (n < 1 || n > kPsMaxExperts || B < 1 || Cin % 8 != 0) return false;
  if (static_cast<long long>(B) * n * 4 > 16384) return false;
  p->B = B; p->n = n; p->Cin = Cin; p->Cout = Cout; p->taps = taps; p->k_steps = k_steps;
  p->wsize = 1LL * Cout * taps * Cin;
  p->fa = std::min(k_steps, 2);
  const long long threads = 1LL * sms * kPsThreads;
  // tier A: the fewest samples per item that still fit its slices in one round
  int sb = 1;
  while (sb < 16 && 1LL * p->fa * ((B + sb - 1) / sb) * Cout * 8 > threads) sb <<= 1;
  p->sbA = std::min(sb, B);
  p->nsbA = (B + p->sbA - 1) / p->sbA;
  p->ipsA = p->nsbA * Cout * 8;
  p->nA = 1LL * p->fa * p->ipsA;
  p->sbB = std::min(16, B);
  p->nsbB = (B + p->sbB - 1) / p->sbB;
  p->ipsB = p->nsbB * Cout * 8;
  p->nB = 1LL * (k_steps - p->fa) * p->ipsB;
  *grid = static_cast<unsigned>(sms);
  return true;
}

}  // namespace dc
