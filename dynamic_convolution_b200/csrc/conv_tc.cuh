// Tensor-core (tcgen05) implicit-GEMM dynamic convolution, bf16 in / out,
// fp32 accumulation in tensor memory.
//
// Per work unit (sample b, block of R image rows, block of 128 output
// channels) the kernel computes
//     D[co][pix] = sum_k A[co][k] * Bop[pix][k]
// with k running over (tap kh,kw ; input-channel chunk of 64). The GEMM is
// "swapped": M = output channels (128 per tile), N = the R*W pixels of the
// unit, so the per-sample kernel is the A operand and the pixel count only has
// to be a multiple of 16 (an image row block maps onto N exactly).
//
//  * Bop tiles are the activations of tap (kh,kw): one 4-D TMA box
//    {64 channels, W, R, 1} of x at (c, kw-pad, h0+kh-pad, b). Zero padding is
//    the TMA's out-of-bounds fill, so the halo costs nothing.
//  * A tiles (128 x 64 bf16, K-major, 128-byte swizzle) depend on the variant:
//      FUSED    A = sum_i alpha_{b,i} E_i[co-tile][tap][c-chunk], mixed by 8
//               warps on CUDA cores from 16-byte expert loads (L2-resident),
//               rounded once to bf16: "a linear mixture of n static kernels
//               weighted with their input-dependent attentions"
//               (KernelWarehouse, abstract), one kernel per example (CondConv,
//               abstract);
//      OUTSIDE  k also runs over the experts and A = alpha_{b,i} E_i: the sum
//               over experts happens in the accumulator, i.e.
//               y = sum_i alpha_i (x conv W_i), the same result by linearity;
//      PREMIX   A = W_b tile, TMA-loaded from a workspace where a separate
//               tensor-core kernel stored every sample's mixed kernel.
//  * One thread issues tcgen05.mma (M=128, N<=256 per instruction, K=16) into
//    TMEM and commits each stage back to its "empty" barrier.
//  * The epilogue (8 warps) reads TMEM lane = output channel, adds the mixed
//    bias sum_i alpha_i bias_i, rounds to bf16, transposes through shared
//    memory and writes 16-byte NHWC segments.
// Every barrier wait is bounded; on expiry the CTA raises an abort flag,
// records an error word, drains its in-flight TMA / MMA work, frees TMEM and
// exits.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kTcThreads = 384;      // 12 warps
constexpr int kTcMixWarp0 = 4;       // warps 4..11 mix (FUSED/OUTSIDE) and run the epilogue
constexpr int kTcMixThreads = 256;
constexpr int kTcATileBytes = 128 * 128;  // 128 rows x 64 bf16

enum TcVariant { kFused = 1, kOutside = 2, kPremix = 3 };

struct TcParams {
  int B, H, W, Cin, Cout, KH, KW, pad, n;
  int R;              // image rows per unit
  int tiles_h;        // ceil(H / R)
  int m_tiles;        // ceil(Cout / 128)
  int n_valid;        // R * W
  int n_mma0, n_mma1; // MMA N of the two column chunks (n_mma1 may be 0)
  int kc;             // 64-channel chunks per tap: ceil(Cin / 64)
  int k_steps;        // pipeline steps per unit
  int stages;
  int b_tile_bytes;   // bytes of one activation stage (1024-aligned)
  uint32_t tmem_cols;
  const __nv_bfloat16* experts;
  const float* alpha;
  const float* bias;  // may be null
  __nv_bfloat16* y;
  int* err;
  long long wait_ns;
  int inject_skip;    // test hook: withhold the first mixer arrival
};

template <int VARIANT>
__global__ void __launch_bounds__(kTcThreads, 1)
    tc_conv_kernel(const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap, TcParams p) {
  extern __shared__ __align__(1024) unsigned char tc_smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // ---- unit decode: consecutive CTAs share a sample
  int u = blockIdx.x;
  const int mt = u % p.m_tiles;
  u /= p.m_tiles;
  const int th = u % p.tiles_h;
  const int b = u / p.tiles_h;
  const int m0 = mt * 128;
  const int h0 = th * p.R;

  // ---- shared-memory carve-up (1024-aligned tiles first)
  const uint32_t raw = smem_u32(tc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = tc_smem_raw + (base - raw);
  const int S = p.stages;
  const uint32_t a_base = base;
  const uint32_t b_base = a_base + S * kTcATileBytes;
  const uint32_t bar_base = b_base + S * p.b_tile_bytes;
  // barriers: fullA[S], fullB[S], empty[S], accum, drain
  auto fullA = [&](int s) { return bar_base + 8u * s; };
  auto fullB = [&](int s) { return bar_base + 8u * (S + s); };
  auto empty = [&](int s) { return bar_base + 8u * (2 * S + s); };
  const uint32_t accum_bar = bar_base + 8u * (3 * S);
  const uint32_t drain_bar = accum_bar + 8u;
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (3 * S + 2);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* alpha_s = reinterpret_cast<float*>(misc + 16);

  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(fullA(s), VARIANT == kPremix ? 1 : kTcMixThreads / 32);
      mbar_init(fullB(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    if (VARIANT == kPremix) tma_prefetch_desc(&wmap);
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), p.tmem_cols);
    tmem_relinquish();
  }
  for (int i = threadIdx.x; i < p.n; i += kTcThreads)
    alpha_s[i] = p.alpha[static_cast<size_t>(b) * p.n + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int taps = p.KH * p.KW;
  const int steps_per_expert = taps * p.kc;  // OUTSIDE: k = expert * steps_per_expert + kk

  if (warp == 0) {
    // ======================= TMA producer =======================
    if (lane == 0) {
      int issued = 0;
      for (int k = 0; k < p.k_steps; ++k) {
        const int s = k % S;
        const uint32_t ph = static_cast<uint32_t>(k / S) & 1u;
        if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
        const int kk = (VARIANT == kOutside) ? k % steps_per_expert : k;
        const int tap = kk / p.kc, cc = kk % p.kc;
        const int kh = tap / p.KW, kw = tap % p.KW;
        mbar_arrive_expect_tx(fullB(s), 64u * 2u * p.W * p.R);
        tma_load_4d(b_base + s * p.b_tile_bytes, &xmap, fullB(s), cc * 64, kw - p.pad,
                    h0 + kh - p.pad, b);
        if (VARIANT == kPremix) {
          mbar_arrive_expect_tx(fullA(s), kTcATileBytes);
          tma_load_3d(a_base + s * kTcATileBytes, &wmap, fullA(s), cc * 64, tap,
                      b * p.Cout + m0);
        }
        ++issued;
      }
      // drain: every load issued must land before the CTA may exit
      for (int j = (issued > S ? issued - S : 0); j < issued; ++j) {
        const int s = j % S;
        const uint32_t ph = static_cast<uint32_t>(j / S) & 1u;
        wait_drain(fullB(s), ph, p.wait_ns, p.err);
        if (VARIANT == kPremix) wait_drain(fullA(s), ph, p.wait_ns, p.err);
      }
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    if (lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(128, p.n_mma0);
      const uint32_t idesc1 = idesc_bf16_f32(128, p.n_mma1 > 0 ? p.n_mma1 : 16);
      bool ok = true;
      int k = 0;
      for (; k < p.k_steps; ++k) {
        const int s = k % S;
        const uint32_t ph = static_cast<uint32_t>(k / S) & 1u;
        if (!wait_bounded(fullA(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
        if (!wait_bounded(fullB(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_s = a_base + s * kTcATileBytes;
        const uint32_t b_s = b_base + s * p.b_tile_bytes;
#pragma unroll
        for (int q = 0; q < 4; ++q) {  // 4 x K=16 per 64-wide stage
          const uint64_t ad = smem_desc_sw128(a_s + q * 32);
          const uint32_t acc = (k > 0 || q > 0) ? 1u : 0u;
          tc_mma_f16(tmem_base, ad, smem_desc_sw128(b_s + q * 32), idesc0, acc);
          if (p.n_mma1 > 0)
            tc_mma_f16(tmem_base + p.n_mma0, ad,
                       smem_desc_sw128(b_s + p.n_mma0 * 128 + q * 32), idesc1, acc);
        }
        tc_commit(empty(s));
      }
      if (ok) {
        tc_commit(accum_bar);
      } else {
        // drain whatever MMAs were issued before giving up
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else if (warp >= kTcMixWarp0) {
    const int mt_id = threadIdx.x - kTcMixWarp0 * 32;  // 0..255
    // ======================= mixers (FUSED / OUTSIDE) =======================
    if (VARIANT != kPremix) {
      const size_t wsize = static_cast<size_t>(p.Cout) * taps * p.Cin;  // one expert
      bool ok = true;
      for (int k = 0; k < p.k_steps && ok; ++k) {
        const int s = k % S;
        const uint32_t ph = static_cast<uint32_t>(k / S) & 1u;
        if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitMixer)) { ok = false; break; }
        const int kk = (VARIANT == kOutside) ? k % steps_per_expert : k;
        const int tap = kk / p.kc, cc = kk % p.kc;
        const uint32_t a_s = a_base + s * kTcATileBytes;
        // this thread's four 16-byte chunks: rows r0 + 32u (u = 0..3), chunk j
        const int j = mt_id & 7;
        const int r0 = mt_id >> 3;
        const int ci = cc * 64 + j * 8;
        float acc[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
          for (int e = 0; e < 8; ++e) acc[u][e] = 0.f;
        const __nv_bfloat16* src[4];
        bool live[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int co = m0 + r0 + 32 * u;
          live[u] = co < p.Cout && ci < p.Cin;
          src[u] = p.experts + (static_cast<size_t>(live[u] ? co : 0) * taps + tap) * p.Cin +
                   (live[u] ? ci : 0);
        }
        if (VARIANT == kFused) {
          // two experts x four chunks = eight 16-byte loads in flight per thread
          for (int i = 0; i < p.n; i += 2) {
            const bool two = i + 1 < p.n;
            uint4 v0[4], v1[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              v0[u] = live[u] ? ld_nc_v4(src[u] + i * wsize) : make_uint4(0u, 0u, 0u, 0u);
              v1[u] = (live[u] && two) ? ld_nc_v4(src[u] + (i + 1) * wsize)
                                       : make_uint4(0u, 0u, 0u, 0u);
            }
            const float a0 = alpha_s[i];
            const float a1 = two ? alpha_s[i + 1] : 0.f;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              const uint32_t w0[4] = {v0[u].x, v0[u].y, v0[u].z, v0[u].w};
              const uint32_t w1[4] = {v1[u].x, v1[u].y, v1[u].z, v1[u].w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                acc[u][2 * e] = fmaf(a0, bf16lo_to_f32(w0[e]), acc[u][2 * e]);
                acc[u][2 * e + 1] = fmaf(a0, bf16hi_to_f32(w0[e]), acc[u][2 * e + 1]);
                acc[u][2 * e] = fmaf(a1, bf16lo_to_f32(w1[e]), acc[u][2 * e]);
                acc[u][2 * e + 1] = fmaf(a1, bf16hi_to_f32(w1[e]), acc[u][2 * e + 1]);
              }
            }
          }
        } else {  // OUTSIDE: A = alpha_i * W_i for this step's expert i
          const int i = k / steps_per_expert;
          const float a = alpha_s[i];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint4 v = live[u] ? ld_nc_v4(src[u] + i * wsize) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              acc[u][2 * e] = a * bf16lo_to_f32(w[e]);
              acc[u][2 * e + 1] = a * bf16hi_to_f32(w[e]);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = r0 + 32 * u;
          const uint4 packed =
              make_uint4(pack_bf16x2(acc[u][0], acc[u][1]), pack_bf16x2(acc[u][2], acc[u][3]),
                         pack_bf16x2(acc[u][4], acc[u][5]), pack_bf16x2(acc[u][6], acc[u][7]));
          // K-major, 128-byte swizzle: 16-byte chunk j of row r lands at chunk j ^ (r % 8)
          st_shared_v4(a_s + r * 128 + ((j ^ (r & 7)) << 4), packed);
        }
        fence_proxy_async_smem();
        __syncwarp();
        const bool withhold = (p.inject_skip != 0) && k == 0 && blockIdx.x == 0;
        if (lane == 0 && !withhold) mbar_arrive(fullA(s));
      }
    }

    // ======================= epilogue =======================
    const int q = warp & 3;                      // TMEM lane quarter
    const int half = (warp - kTcMixWarp0) >> 2;  // column half
    const int co = m0 + 32 * q + lane;
    float bb = 0.f;
    if (p.bias != nullptr && co < p.Cout)
      for (int i = 0; i < p.n; ++i) bb = fmaf(alpha_s[i], p.bias[static_cast<size_t>(i) * p.Cout + co], bb);
    if (wait_bounded(accum_bar, 0, ctl, kErrWaitEpilogue)) {
      tc_fence_after();
      // per-warp 32 px x 32 co bf16 staging tile in the (now idle) A stage buffers
      const uint32_t stage = a_base + (warp - kTcMixWarp0) * 2048;
      const int n_pad = p.n_mma0 + p.n_mma1;
      const int nchunks = (n_pad + 31) / 32;
      for (int ch = half; ch < nchunks; ch += 2) {
        uint32_t r[32];
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ch * 32, r);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(r[j]) + bb);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + j * 64 + lane * 2),
                       "h"(*reinterpret_cast<const unsigned short*>(&h))
                       : "memory");
        }
        __syncwarp();
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int jj = it * 8 + (lane >> 2);   // pixel within the chunk
          const int part = lane & 3;             // 16-byte part of the 64-byte row
          const int pix = ch * 32 + jj;
          const int rr = pix / p.W, ww = pix % p.W;
          const int oh = h0 + rr;
          const int c8 = m0 + 32 * q + part * 8;
          if (pix < p.n_valid && oh < p.H && c8 < p.Cout) {
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stage + jj * 64 + part * 16));
            __nv_bfloat16* dst =
                p.y + ((static_cast<size_t>(b) * p.H + oh) * p.W + ww) * p.Cout + c8;
            *reinterpret_cast<uint4*>(dst) = v;
          }
        }
        __syncwarp();
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace dc
