// PREMIX with the kernel mixing streamed into the convolution: one persistent
// cooperative kernel, one CTA per SM, for few experts (n <= 8).
//
//   W_b = sum_i alpha[b][i] E_i for every sample b (n static kernels summed
//   with weights that depend on the input, KernelWarehouse, abstract; one
//   kernel per example, CondConv, abstract),
//   then y_b = conv(x_b, W_b) + sum_i alpha[b][i] bias_i.
//
// The convolution consumes W_b one K step (one tap of one 64-channel chunk)
// at a time, so the mixing is published per K step ("slice") instead of per
// kernel launch:
//  * warps 4..11 first mix: the items of all slices (8 weights x a block of
//    samples each, as the few-expert CUDA-core mixer) are dealt out to the
//    grid in slice order; after each round a CTA adds the number of items it
//    finished to each slice's counter in the workspace (release);
//  * warp 2 loads the W_b tile of step k by TMA once slice k's counter shows
//    all its items (acquire), warp 0 loads the activation tiles, warp 1 issues
//    tcgen05.mma exactly as the convolution kernel does;
//  * warps 4..11 then run the epilogue of the CTA's units.
// Slice 0 is ready after one round of mixing; the later slices are written
// while the MMAs of the earlier ones run, so the 2*B*|W| bytes of mixed
// kernels are hidden behind the tensor-core work instead of preceding it.
//
// The slice counters live in a state slot owned by the library (one per
// stream, never in caller memory): every launch finds them at zero and the
// last CTA to finish zeroes them again, so the targets are this launch's item
// counts whatever shape ran before. All CTAs are co-resident (cooperative
// launch); every wait is bounded.
#pragma once

#include "conv_tc.cuh"

namespace dc {

constexpr int kMcThreads = 384;
constexpr int kMcMixer0 = 4;            // first mixer / epilogue warp
constexpr int kMcMaxExperts = 8;
constexpr int kMcStateWords = 1024;     // 4 KB of state per slot
constexpr int kMcSlots = 64;            // state slots (one per stream in use)
constexpr int kMcSliceWord0 = 64;       // slice counters start here
constexpr int kMcMaxSlices = kMcStateWords - kMcSliceWord0;
constexpr int kMcEpiStage = 8 * 2048;   // epilogue staging: 2 KB per warp

struct MixParams {
  TcParams cv;              // geometry, experts/alpha/bias/y, error word, wait limit
  __nv_bfloat16* wb;        // [B][wsize] mixed kernels
  unsigned int* state;      // slot: [1] finished CTAs, [64 + k] slice k (all zero between launches)
  long long wsize;          // Cout * taps * Cin
  int sblock, nsb;          // samples per item, sample blocks
  int ips;                  // items per slice: nsb * Cout * 8
  long long total_items;    // k_steps * ips
  int units;                // (sample, row block, channel tile)
  int alpha_off;            // shared-memory offsets from the 1024-aligned base
  int stage_off;
  int bar_off;
};

__device__ __forceinline__ unsigned int ld_acquire_u32(const unsigned int* p) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

template <int NMAX>
__global__ void __launch_bounds__(kMcThreads, 1)
    mixconv_kernel(const __grid_constant__ CUtensorMap xmap,
                   const __grid_constant__ CUtensorMap wmap, MixParams mp) {
  extern __shared__ __align__(1024) unsigned char mc_smem_raw[];
  const TcParams& p = mp.cv;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(mc_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = mc_smem_raw + (base - raw);
  const int SA = p.sa, SB = p.sb;
  const uint32_t a_base = base;
  const uint32_t b_base = a_base + SA * kTcATileBytes;
  const uint32_t stage_base = base + mp.stage_off;
  float* alpha_s = reinterpret_cast<float*>(base_ptr + mp.alpha_off);
  const uint32_t bar_base = base + mp.bar_off;
  auto fullA = [&](int s) { return bar_base + 8u * s; };
  auto emptyA = [&](int s) { return bar_base + 8u * (SA + s); };
  auto fullB = [&](int s) { return bar_base + 8u * (2 * SA + s); };
  auto emptyB = [&](int s) { return bar_base + 8u * (2 * SA + SB + s); };
  const uint32_t afull = bar_base + 8u * (2 * SA + 2 * SB);
  const uint32_t aempty = afull + 8u;
  const uint32_t drain_bar = afull + 16u;
  unsigned char* misc = base_ptr + mp.bar_off + 8 * (2 * SA + 2 * SB + 3);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  volatile int* last_s = reinterpret_cast<volatile int*>(misc + 8);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  // ---- set-up that reads no global memory (overlaps the previous kernel)
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < SA; ++s) {
      mbar_init(fullA(s), 1);
      mbar_init(emptyA(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(fullB(s), 1);
      mbar_init(emptyB(s), 1);
    }
    mbar_init(afull, 1);
    mbar_init(aempty, 8);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&wmap);
  }
  grid_dependency_wait();  // alpha from the routing kernel; x, experts before it
  const int na = p.B * p.n;
  for (int e = threadIdx.x; e < na; e += kMcThreads) alpha_s[e] = p.alpha[e];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int taps = p.KH * p.KW;
  const int my_units = mp.units > static_cast<int>(blockIdx.x)
                           ? (mp.units - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                           : 0;
  auto decode = [&](int j, int& b, int& m0, int& h0) {
    int u = blockIdx.x + j * gridDim.x;
    const int mt = u % p.m_tiles;
    u /= p.m_tiles;
    const int th = u % p.tiles_h;
    b = u / p.tiles_h;
    m0 = mt * 128;
    h0 = th * p.R;
  };

  if (warp == 0) {
    if (lane == 0) {  // ======== activations
      const uint32_t bytes = 64u * 2u * p.Wp * p.b_box_rows;
      int issued = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int j = 0; j < my_units && ok; ++j) {
        int b, m0, h0;
        decode(j, b, m0, h0);
        for (int cc = 0; cc < p.kc; ++cc) {
          if (!wait_bounded(emptyB(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(fullB(s), bytes);
          tma_load_4d(b_base + s * p.b_tile_bytes, &xmap, fullB(s), cc * 64, -p.pad, h0 - p.pad, b);
          ++issued;
          if (++s == SB) { s = 0; ph ^= 1u; }
        }
      }
      for (int i = (issued > SB ? issued - SB : 0); i < issued; ++i)
        wait_drain(fullB(i % SB), static_cast<uint32_t>(i / SB) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 2) {
    if (lane == 0) {  // ======== mixed kernels, slice by slice
      const unsigned int* slices = mp.state + kMcSliceWord0;
      int issued = 0, s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int ready = 0;  // slices [0, ready) seen complete
      for (int j = 0; j < my_units && ok; ++j) {
        int b, m0, h0;
        decode(j, b, m0, h0);
        int cc = 0, tap = 0;
        for (int k = 0; k < p.k_steps; ++k) {
          if (k >= ready) {
            const uint64_t t0 = globaltimer_ns();
            for (uint32_t it = 0;; ++it) {
              const unsigned int v = ld_acquire_u32(slices + k);
              if (v >= static_cast<unsigned int>(mp.ips)) break;
              if (*abort_flag) { ok = false; break; }
              __nanosleep(64);
              if ((it & 15u) == 15u &&
                  static_cast<long long>(globaltimer_ns() - t0) > p.wait_ns) {
                *abort_flag = 1;
                atomicCAS(p.err, 0, kErrWaitGrid);
                ok = false;
                break;
              }
            }
            if (!ok) break;
            ready = k + 1;
            // order the TMA (async proxy) reads after the acquire above
            asm volatile("fence.proxy.async.global;" ::: "memory");
          }
          if (!wait_bounded(emptyA(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(fullA(s), kTcATileBytes);
          tma_load_3d(a_base + s * kTcATileBytes, &wmap, fullA(s), cc * 64, tap, b * p.Cout + m0);
          ++issued;
          if (++tap == p.spc) { tap = 0; ++cc; }
          if (++s == SA) { s = 0; ph ^= 1u; }
        }
      }
      for (int i = (issued > SA ? issued - SA : 0); i < issued; ++i)
        wait_drain(fullA(i % SA), static_cast<uint32_t>(i / SA) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {  // ======== MMA issuer (counters only; see conv_tc.cuh)
      const uint32_t idesc0 = idesc_bf16_f32(128, p.n_mma0);
      const uint32_t idesc1 = idesc_bf16_f32(128, p.n_mma1 > 0 ? p.n_mma1 : 16);
      const uint64_t a_desc0 = smem_desc_sw128(a_base);
      const uint64_t b_desc0 = smem_desc_sw128(b_base);
      const uint64_t b_n1 = static_cast<uint64_t>(p.n_mma0) * 8u;
      const uint64_t b_stage = static_cast<uint64_t>(p.b_tile_bytes) >> 4;
      const uint64_t row_skip = static_cast<uint64_t>(p.Wp - p.KW + 1) * 8u;
      const bool two = p.n_mma1 > 0;
      uint32_t s = 0, ph = 0, sbi = 0, phb = 0;
      bool ok = true;
      for (int j = 0; j < my_units && ok; ++j) {
        if (j > 0 && !wait_bounded(aempty, static_cast<uint32_t>((j - 1) & 1), ctl, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        int t = 0, tap = 0, kw = 0;
        uint64_t tap_off = 0;
        for (int k = 0; k < p.k_steps; ++k) {
          if (t == 0 && !wait_bounded(fullB(sbi), phb, ctl, kErrWaitMma)) { ok = false; break; }
          if (!wait_bounded(fullA(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          const uint64_t ad = a_desc0 + s * (kTcATileBytes >> 4);
          const uint64_t bd = b_desc0 + sbi * b_stage + tap_off;
          const uint32_t acc0 = k > 0 ? 1u : 0u;
          tc_mma_f16(tmem_base, ad, bd, idesc0, acc0);
          if (two) tc_mma_f16(tmem_base + p.n_mma0, ad, bd + b_n1, idesc1, acc0);
#pragma unroll
          for (int q = 1; q < 4; ++q) {
            tc_mma_f16(tmem_base, ad + 2 * q, bd + 2 * q, idesc0, 1u);
            if (two) tc_mma_f16(tmem_base + p.n_mma0, ad + 2 * q, bd + b_n1 + 2 * q, idesc1, 1u);
          }
          tc_commit(emptyA(s));
          if (++tap == taps) {
            tap = 0; kw = 0; tap_off = 0;
          } else if (++kw == p.KW) {
            kw = 0; tap_off += row_skip;
          } else {
            tap_off += 8u;
          }
          if (++t == p.spc) {
            t = 0;
            tc_commit(emptyB(sbi));
            if (++sbi == static_cast<uint32_t>(SB)) { sbi = 0; phb ^= 1u; }
          }
          if (++s == static_cast<uint32_t>(SA)) { s = 0; ph ^= 1u; }
        }
        if (ok) tc_commit(afull);
      }
      if (!ok) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else if (warp >= kMcMixer0) {
    const int tm = threadIdx.x - kMcMixer0 * 32;  // 0..255
    // ======== mixing: rounds of 256 consecutive items per CTA, slice-major
    {
      const long long stride = static_cast<long long>(gridDim.x) * 256;
      for (long long rb = static_cast<long long>(blockIdx.x) * 256; rb < mp.total_items;
           rb += stride) {
        const long long it = rb + tm;
        if (it < mp.total_items && !*abort_flag) {
          const int k = static_cast<int>(it / mp.ips);
          const int local = static_cast<int>(it - static_cast<long long>(k) * mp.ips);
          const int jc = local & 7;                // 16-byte chunk of the 64-channel slice
          const int rest = local >> 3;
          const int co = rest % p.Cout;
          const int sb = rest / p.Cout;
          const int cc = k / taps, tap = k - cc * taps;
          const int ch0 = cc * 64 + jc * 8;
          if (ch0 < p.Cin) {
            const long long off = (static_cast<long long>(co) * taps + tap) * p.Cin + ch0;
            uint4 raw[NMAX];
#pragma unroll
            for (int i = 0; i < NMAX; ++i)
              if (i < p.n) raw[i] = ld_nc_v4(p.experts + i * mp.wsize + off);
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
            const int b0 = sb * mp.sblock;
            const int b1 = min(p.B, b0 + mp.sblock);
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
              *reinterpret_cast<uint4*>(mp.wb + static_cast<long long>(b) * mp.wsize + off) = o;
            }
          }
        }
        // publish: every writer makes its stores visible (to the async proxy too)
        // before one thread adds this round's item counts to the slice counters
        asm volatile("fence.proxy.async.global;" ::: "memory");
        __threadfence();
        asm volatile("bar.sync 1, 256;" ::: "memory");
        if (tm == 0) {
          const long long lo = rb;
          const long long hi = min(rb + 256, mp.total_items);
          for (long long k = lo / mp.ips; k * mp.ips < hi; ++k) {
            const long long s0 = max(lo, k * mp.ips);
            const long long s1 = min(hi, (k + 1) * mp.ips);
            atomicAdd(mp.state + kMcSliceWord0 + k, static_cast<unsigned int>(s1 - s0));
          }
        }
      }
    }

    // ======== epilogue of this CTA's units
    const int q = warp & 3;                    // TMEM lane quarter
    const int half = (warp - kMcMixer0) >> 2;  // column half
    const uint32_t stage = stage_base + (warp - kMcMixer0) * 2048;
    const int n_pad = p.n_mma0 + p.n_mma1;
    const int nchunks = (n_pad + 31) / 32;
    const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
    const int part = lane & 3;
    for (int j = 0; j < my_units; ++j) {
      int b, m0, h0;
      decode(j, b, m0, h0);
      const int co = m0 + 32 * q + lane;
      float bb = 0.f;
      if (p.bias != nullptr && co < p.Cout)
        for (int i = 0; i < p.n; ++i)
          bb = fmaf(alpha_s[b * p.n + i], p.bias[static_cast<size_t>(i) * p.Cout + co], bb);
      const int c8 = m0 + 32 * q + part * 8;
      const bool c_ok = c8 < p.Cout;
      __nv_bfloat16* ybase = p.y + static_cast<size_t>(b) * p.H * p.W * p.Cout + c8;
      if (!wait_bounded(afull, static_cast<uint32_t>(j & 1), ctl, kErrWaitEpilogue)) break;
      tc_fence_after();
      auto process = [&](const uint32_t (&r)[32], int ch) {
#pragma unroll
        for (int jj = 0; jj < 32; jj += 2) {
          const uint32_t w = pack_bf16x2(__uint_as_float(r[jj]) + bb, __uint_as_float(r[jj + 1]) + bb);
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + jj * 64 + lane * 2),
                       "h"(static_cast<unsigned short>(w & 0xFFFFu))
                       : "memory");
          asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + (jj + 1) * 64 + lane * 2),
                       "h"(static_cast<unsigned short>(w >> 16))
                       : "memory");
        }
        __syncwarp();
        int pix = ch * 32 + (lane >> 2);
        int rr = pix / p.Wp;
        int cw = pix - rr * p.Wp;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int oh = h0 + rr;
          if (c_ok && pix < p.n_virt && cw < p.W && oh < p.H) {
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stage + (it * 8 + (lane >> 2)) * 64 + part * 16));
            *reinterpret_cast<uint4*>(ybase + (static_cast<size_t>(oh) * p.W + cw) * p.Cout) = v;
          }
          pix += 8;
          cw += 8;
          while (cw >= p.Wp) { cw -= p.Wp; ++rr; }
        }
        __syncwarp();
      };
      uint32_t ra[32], rb[32];
      int ch = half;
      if (ch < nchunks) tmem_ld_32x32b_x32(trow + ch * 32, ra);
      while (ch < nchunks) {
        tmem_ld_wait(ra);
        if (ch + 2 < nchunks) tmem_ld_32x32b_x32(trow + (ch + 2) * 32, rb);
        process(ra, ch);
        ch += 2;
        if (ch >= nchunks) break;
        tmem_ld_wait(rb);
        if (ch + 2 < nchunks) tmem_ld_32x32b_x32(trow + (ch + 2) * 32, ra);
        process(rb, ch);
        ch += 2;
      }
      // this warp is done reading the accumulator of unit j
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(aempty);
    }
  }

  // ---- teardown; the last CTA to finish zeroes the slot for the next launch
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
  if (threadIdx.x == 0) {
    int last = 0;
    if (!*abort_flag) {
      __threadfence();
      last = atomicAdd(mp.state + 1, 1u) == gridDim.x - 1;
    }
    *last_s = last;
  }
  __syncthreads();
  if (*last_s) {
    __threadfence();  // every CTA's counter updates happened before its arrival
    for (int k = threadIdx.x; k < p.k_steps; k += kMcThreads) mp.state[kMcSliceWord0 + k] = 0u;
    if (threadIdx.x == 0) mp.state[1] = 0u;
  }
}

}  // namespace dc
