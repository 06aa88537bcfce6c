// Kernel mixing on CUDA cores for few experts (n <= 8):
//     W[b][w] = sum_i alpha[b][i] * E[i][w]
// for every sample b and weight element w -- each example's kernel is n static
// kernels summed with weights that depend on the input (KernelWarehouse,
// abstract; CondConv, abstract: one kernel per example).
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
  const float* a_in;             // [B][Cin] input channel attention, or null
  int Cin;                       // input channels (with a_in: weight w has channel w % Cin)
  unsigned long long* stamps;    // optional [grid][8] phase stamps for measurements, or null
};

// NMAX: the expert count rounded up to 2, 4 or 8 (fewer registers for fewer experts)
template <int NMAX>
__global__ void __launch_bounds__(kPsThreads) premix_small_kernel(PsParams p) {
  extern __shared__ float ps_alpha[];  // [B][n], then [B][Cin] when a_in is given
  float* ps_ain = ps_alpha + p.B * p.n;
  // phase stamps (measurement hook): [0] entry, [1] past the grid wait,
  // [5] end, [6] SM id, [7] global timer at entry
  unsigned long long* stp =
      (p.stamps != nullptr && threadIdx.x == 0) ? p.stamps + blockIdx.x * 8 : nullptr;
  if (stp) {
    stp[0] = clock64();
    stp[7] = globaltimer_ns();
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    stp[6] = smid;
  }
  grid_dependency_wait();  // alpha comes from the routing kernel
  if (stp) stp[1] = clock64();
  // The convolution may be scheduled once every CTA of this grid is past its
  // wait: everything launched before this kernel (the writer of x included)
  // has then completed, so the convolution may load x before its own wait.
  grid_launch_dependents();
  const int na = p.B * p.n;
  for (int e = threadIdx.x; e < na; e += kPsThreads) ps_alpha[e] = p.alpha[e];
  if (p.a_in != nullptr)
    for (int e = threadIdx.x; e < p.B * p.Cin; e += kPsThreads) ps_ain[e] = p.a_in[e];
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
    // with input attention: the 8 weights are 8 consecutive input channels of
    // one (output channel, tap); the factor of channel c scales W_b[., ., c]
    // (linearity: the same as scaling input channel c of x)
    const int cin0 = p.a_in != nullptr ? static_cast<int>((ch * 8) % p.Cin) : 0;
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
      if (p.a_in != nullptr) {
        const float* ai = ps_ain + b * p.Cin + cin0;
#pragma unroll
        for (int q = 0; q < 4; ++q)
          acc[q] = pack_f32x2(__uint_as_float(static_cast<uint32_t>(acc[q])) * ai[2 * q],
                              __uint_as_float(static_cast<uint32_t>(acc[q] >> 32)) * ai[2 * q + 1]);
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
  if (stp) stp[5] = clock64();
}

// Host-side plan: as many samples per thread (up to 16) as keep at least one
// CTA's worth of items per SM, so that the grid runs in a single wave (fewer
// samples per thread when the kernel is small). Returns false when the shape
// is outside this kernel.
inline bool plan_premix_small(int B, int n, long long wsize, int sms, PsParams* p,
                              unsigned* grid) {
  if (n < 1 || n > kPsMaxExperts || B < 1 || wsize % 8 != 0) return false;
  if (static_cast<long long>(B) * n * 4 > 16384) return false;
  p->a_in = nullptr;
  p->Cin = 0;
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

}  // namespace dc
