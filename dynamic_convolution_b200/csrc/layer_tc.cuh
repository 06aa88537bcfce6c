// Fused PREMIX forward: one persistent, cooperative kernel (one CTA per SM)
// that first mixes every sample's kernel with tensor cores into the workspace
// and then runs the tensor-core convolution from it:
//
//   phase 1  W[b][w] = sum_i alpha[b][i] E[i][w]  (the GEMM of premix.cuh:
//            M = samples, N = 256 weights, K = experts; alpha split in bf16
//            hi + lo; experts an MN-major operand as stored)
//   grid barrier (all CTAs; bounded wait)
//   phase 2  y = conv(x, W_b) + b_b  (the swapped implicit GEMM of conv_tc.cuh:
//            M = 128 output channels, N = pixels of R rows on the padded-width
//            grid, K = (tap, 64-channel chunk)), units distributed round-robin
//            over the CTAs, TMEM handed from one unit to the next through an
//            accumulator-empty barrier.
//
// Compared with two kernels this removes a launch, the second kernel's
// set-up (TMEM allocation, barrier initialisation, tensor-map fetch), and the
// gap between them; "a linear mixture of n static kernels weighted with their
// input-dependent attentions" (KernelWarehouse, abstract) per example
// (CondConv, abstract) is computed once per sample and consumed from L2.
#pragma once

#include "common.cuh"
#include "conv_tc.cuh"
#include "premix.cuh"

namespace dc {

constexpr int kFusedThreads = 384;
constexpr int kFusedEpiStage = 8 * 2048;  // conv epilogue staging: 8 warps x 32 px x 32 co bf16
constexpr int kFusedPmStage = 32 * 128 * 2;  // mixing epilogue staging per warp: 32 samples x 128 bf16

struct FusedParams {
  PmParams pm;
  TcParams cv;
  unsigned int* grid_bar;  // {count, generation} in the workspace (see fused_grid_barrier)
  int units;               // conv units (sample, row block, 128-channel tile)
  int region_bytes;        // shared bytes both phases may use (1024-aligned)
};

// Grid-wide barrier on two words {count, generation} in the workspace. The
// last CTA to arrive resets the count and advances the generation, so the
// words are left ready for the next launch (the host zeroes them once, on a
// workspace's first use). Waiters poll with a short sleep between probes so
// that 148 spinning threads do not starve the arrivals on the same L2 line.
// Returns false if this CTA gave up (bounded wait) or had aborted already.
__device__ __forceinline__ bool fused_grid_barrier(unsigned int* words, const WaitCtl& ctl) {
  __threadfence();  // release this thread's global writes
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned int* count = words;
    unsigned int* gen = words + 1;
    unsigned int g;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(g) : "l"(gen) : "memory");
    __threadfence();
    const unsigned int old = atomicAdd(count, 1u);
    if (old == gridDim.x - 1) {
      atomicExch(count, 0u);
      __threadfence();
      asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(gen), "r"(g + 1u) : "memory");
    } else {
      const uint64_t t0 = globaltimer_ns();
      for (uint32_t it = 0;; ++it) {
        unsigned int v;
        asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(gen) : "memory");
        if (v != g) break;
        __nanosleep(64);
        if ((it & 15u) == 0 && static_cast<long long>(globaltimer_ns() - t0) > ctl.limit_ns) {
          *ctl.abort_flag = 1;
          atomicCAS(ctl.err, 0, kErrWaitGrid);
          break;
        }
      }
    }
  }
  __syncthreads();
  return *ctl.abort_flag == 0;
}

__global__ void __launch_bounds__(kFusedThreads, 1)
    premix_conv_kernel(const __grid_constant__ CUtensorMap emap,
                       const __grid_constant__ CUtensorMap xmap,
                       const __grid_constant__ CUtensorMap wmap, FusedParams fp) {
  extern __shared__ __align__(1024) unsigned char fz_smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const PmParams& pm = fp.pm;
  const TcParams& p = fp.cv;

  const uint32_t raw = smem_u32(fz_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = fz_smem_raw + (base - raw);

  // ---- activation stages: a region of their own, so that the first unit's
  // tiles can be loaded while the mixing phase runs
  const int SA = p.sa, SB = p.sb;
  const uint32_t b_base = base;
  const uint32_t r_base = b_base + SB * p.b_tile_bytes;   // region shared by both phases
  // ---- phase-1 layout (premix)
  const int S = pm.stages;
  const int kcols = (pm.nk + 63) / 64;
  const uint32_t pa_base = r_base;                        // A operands (alpha hi/lo)
  const uint32_t pe_base = pa_base + pm.a_bytes;          // expert stages
  const uint32_t pst_base = pe_base + S * pm.stage_bytes; // epilogue staging (4 warps)
  float* alpha_s = reinterpret_cast<float*>(base_ptr + (pst_base - base) + 4 * kFusedPmStage);
  // ---- phase-2 layout (convolution)
  const uint32_t a_base = r_base;
  const uint32_t cst_base = a_base + SA * kTcATileBytes;
  // ---- barriers and misc after the region
  const uint32_t bar_base = r_base + fp.region_bytes;
  auto full = [&](int s) { return bar_base + 8u * s; };
  auto empty = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * S + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * S + 2 + a); };
  const uint32_t cbar = bar_base + 8u * (2 * S + 4);
  auto fullA = [&](int s) { return cbar + 8u * s; };
  auto emptyA = [&](int s) { return cbar + 8u * (SA + s); };
  auto fullB = [&](int s) { return cbar + 8u * (2 * SA + s); };
  auto emptyB = [&](int s) { return cbar + 8u * (2 * SA + SB + s); };
  const uint32_t afull = cbar + 8u * (2 * SA + 2 * SB);
  const uint32_t aempty = afull + 8u;
  const uint32_t drain_bar = aempty + 8u;
  unsigned char* misc = base_ptr + (drain_bar + 8u - base);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 4);
    }
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
    tma_prefetch_desc(&emap);
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&wmap);
    // x is an input of this kernel (written before it started): the first
    // unit's activation tiles can be fetched now, during the mixing phase
    if (static_cast<int>(blockIdx.x) < fp.units) {
      int u = blockIdx.x;
      u /= p.m_tiles;
      const int th = u % p.tiles_h;
      const int b0 = u / p.tiles_h;
      const int pre = p.kc < SB ? p.kc : SB;
      for (int cc = 0; cc < pre; ++cc) {
        mbar_arrive_expect_tx(fullB(cc), 64u * 2u * p.Wp * p.b_box_rows);
        tma_load_4d(b_base + cc * p.b_tile_bytes, &xmap, fullB(cc), cc * 64, -p.pad, th * p.R - p.pad, b0);
      }
    }
  }
  grid_dependency_wait();  // alpha comes from the routing kernel

  // =========================== phase 1: mixing GEMM ===========================
  const int na = pm.B * pm.n;
  for (int e = threadIdx.x; e < na; e += kFusedThreads) alpha_s[e] = pm.alpha[e];
  for (int e = threadIdx.x; e < pm.a_bytes / 16; e += kFusedThreads)
    st_shared_v4(pa_base + e * 16, make_uint4(0u, 0u, 0u, 0u));
  __syncthreads();
  for (int e = threadIdx.x; e < na; e += kFusedThreads) {
    const int m = e / pm.n, k = e - m * pm.n;
    const int mt = m >> 7, r = m & 127;
    const float a = alpha_s[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(a);
    const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
    const uint32_t off = static_cast<uint32_t>(k >> 6) * 16384u + r * 128u +
                         ((((k & 63) >> 3) ^ (r & 7)) << 4) + (k & 7) * 2;
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(pa_base + (mt * 2 + 0) * kcols * 16384u + off),
                 "h"(*reinterpret_cast<const unsigned short*>(&hi)) : "memory");
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(pa_base + (mt * 2 + 1) * kcols * 16384u + off),
                 "h"(*reinterpret_cast<const unsigned short*>(&lo)) : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  {
    const long long my_tiles =
        pm.tiles > blockIdx.x ? (pm.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
    const long long ntile0 = blockIdx.x / pm.m_tiles;
    const int mt0 = blockIdx.x % pm.m_tiles;
    const long long dn = gridDim.x / pm.m_tiles;
    const int dm = gridDim.x % pm.m_tiles;
    if (warp == 0) {
      if (lane == 0) {
        long long issued = 0;
        long long ntile = ntile0;
        int mt = mt0, s = 0;
        uint32_t ph = 0;
        for (long long j = 0; j < my_tiles; ++j) {
          if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
          mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(pm.stage_bytes));
          const uint32_t dst = pe_base + s * pm.stage_bytes;
#pragma unroll
          for (int a = 0; a < 4; ++a)
            tma_load_2d(dst + a * pm.nk * 128, &emap, full(s), static_cast<int>(ntile * kPmN + a * 64), 0);
          ++issued;
          ntile += dn;
          mt += dm;
          if (mt >= pm.m_tiles) { mt -= pm.m_tiles; ++ntile; }
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        for (long long j = (issued > S ? issued - S : 0); j < issued; ++j)
          wait_drain(full(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1), pm.wait_ns, pm.err);
      }
    } else if (warp == 1) {
      if (lane == 0) {
        const uint32_t idesc = idesc_bf16_f32(128, kPmN) | (1u << 16);  // B is MN-major
        const uint64_t e_desc0 = smem_desc_mn_sw128(pe_base, static_cast<uint32_t>(pm.nk) * 128u);
        const uint64_t a_desc0 = smem_desc_sw128(pa_base);
        const uint64_t a_half = static_cast<uint64_t>(kcols) * (16384 >> 4);
        const uint64_t stage = static_cast<uint64_t>(pm.stage_bytes) >> 4;
        const int ksteps = pm.nk / 16;
        int mt = mt0, s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (long long j = 0; j < my_tiles && ok; ++j) {
          const int ab = static_cast<int>(j & 1);
          if (!wait_bounded(full(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
          if (!wait_bounded(tempty(ab), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          const uint64_t bd = e_desc0 + s * stage;
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(mt) * 2 * a_half;
          const uint32_t d = tmem_base + ab * kPmN;
          for (int kk = 0; kk < ksteps; ++kk) {
            const uint64_t aoff = static_cast<uint64_t>(kk >> 2) * (16384 >> 4) + (kk & 3) * 2;
            tc_mma_f16(d, ad + aoff, bd + kk * (2048 >> 4), idesc, kk > 0 ? 1u : 0u);
            tc_mma_f16(d, ad + a_half + aoff, bd + kk * (2048 >> 4), idesc, 1u);
          }
          tc_commit(empty(s));
          tc_commit(tfull(ab));
          mt += dm;
          if (mt >= pm.m_tiles) mt -= pm.m_tiles;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        // every MMA of this phase must finish before TMEM is reused
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, pm.wait_ns, pm.err);
      }
    } else if (warp >= 2 && warp < 6) {
      // the 256 weights of a tile in two halves of 128 through an 8 KB staging
      // block per warp (XOR-swizzled 16-byte chunks: conflict-light writes and
      // reads); each store instruction writes 2 samples x 256 contiguous bytes
      const int q = warp & 3;
      const uint32_t stg = pst_base + (warp - 2) * kFusedPmStage;
      long long ntile = ntile0;
      int mt = mt0;
      for (long long j = 0; j < my_tiles; ++j) {
        const int ab = static_cast<int>(j & 1);
        if (!wait_bounded(tfull(ab), static_cast<uint32_t>((j >> 1) & 1), ctl, kErrWaitEpilogue)) break;
        tc_fence_after();
        const bool live = mt * 128 + 32 * q < pm.B;
        const int nrows = live ? min(32, pm.B - (mt * 128 + 32 * q)) : 0;
#pragma unroll 1
        for (int hh = 0; hh < 2; ++hh) {
#pragma unroll 1
          for (int ch = 0; ch < (live ? 4 : 0); ++ch) {
            uint32_t r[32];
            tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * kPmN +
                                   (hh * 4 + ch) * 32, r);
            tmem_ld_wait();
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              const int c = ch * 4 + v;  // 16-byte chunk of this sample's 256-byte half row
              st_shared_v4(stg + lane * 256 + ((c ^ (lane & 15)) << 4), o);
            }
          }
          if (hh == 1) {  // the accumulator buffer is free once both halves are read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(tempty(ab));
          }
          __syncwarp();
          const long long w = ntile * kPmN + hh * 128 + (lane & 15) * 8;
          const bool wok = w < pm.wsize;
#pragma unroll 4
          for (int sr = (lane >> 4); sr < nrows; sr += 2) {
            const int b = mt * 128 + 32 * q + sr;
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stg + sr * 256 + (((lane & 15) ^ (sr & 15)) << 4)));
            if (wok) *reinterpret_cast<uint4*>(pm.out + static_cast<size_t>(b) * pm.wsize + w) = v;
          }
          __syncwarp();
        }
        ntile += dn;
        mt += dm;
        if (mt >= pm.m_tiles) { mt -= pm.m_tiles; ++ntile; }
      }
      // the mixed kernels are read next by TMA (async proxy) in other CTAs
      asm volatile("fence.proxy.async.global;" ::: "memory");
    }
  }

  tc_fence_before();
  const bool go = fused_grid_barrier(fp.grid_bar, ctl);
  tc_fence_after();

  // =========================== phase 2: convolution ===========================
  const int taps = p.KH * p.KW;
  const int my_units = fp.units > static_cast<int>(blockIdx.x)
                           ? (fp.units - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
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
  if (go) {
    if (warp == 0) {
      if (lane == 0) {  // activations
        const uint32_t bytes = 64u * 2u * p.Wp * p.b_box_rows;
        const int pre = my_units > 0 ? (p.kc < SB ? p.kc : SB) : 0;  // issued during set-up
        int issued = pre, s = pre % SB;
        uint32_t ph = static_cast<uint32_t>(pre / SB) & 1u;
        bool ok = true;
        for (int j = 0; j < my_units && ok; ++j) {
          int b, m0, h0;
          decode(j, b, m0, h0);
          for (int cc = (j == 0 ? pre : 0); cc < p.kc; ++cc) {
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
      if (lane == 0) {  // mixed kernels
        // order the TMA reads below after the barrier that published them
        asm volatile("fence.proxy.async.global;" ::: "memory");
        int issued = 0, s = 0;
        uint32_t ph = 0;
        bool ok = true;
        for (int j = 0; j < my_units && ok; ++j) {
          int b, m0, h0;
          decode(j, b, m0, h0);
          int cc = 0, tap = 0;
          for (int k = 0; k < p.k_steps; ++k) {
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
      if (lane == 0) {  // MMA issuer (counters only; see conv_tc.cuh)
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
          wait_drain(drain_bar, 1, p.wait_ns, p.err);
        }
      }
    } else if (warp >= 4) {
      const int q = warp & 3;
      const int half = (warp - 4) >> 2;
      const uint32_t stage = cst_base + (warp - 4) * 2048;
      const int n_pad = p.n_mma0 + p.n_mma1;
      const int nchunks = (n_pad + 31) / 32;
      for (int j = 0; j < my_units; ++j) {
        int b, m0, h0;
        decode(j, b, m0, h0);
        const int co = m0 + 32 * q + lane;
        float bb = 0.f;
        if (p.bias != nullptr && co < p.Cout)
          for (int i = 0; i < p.n; ++i)
            bb = fmaf(p.alpha[static_cast<size_t>(b) * p.n + i], p.bias[static_cast<size_t>(i) * p.Cout + co], bb);
        if (!wait_bounded(afull, static_cast<uint32_t>(j & 1), ctl, kErrWaitEpilogue)) break;
        tc_fence_after();
        for (int ch = half; ch < nchunks; ch += 2) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ch * 32, r);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 32; ++jj) {
            const __nv_bfloat16 h = __float2bfloat16_rn(__uint_as_float(r[jj]) + bb);
            asm volatile("st.shared.b16 [%0], %1;" ::"r"(stage + jj * 64 + lane * 2),
                         "h"(*reinterpret_cast<const unsigned short*>(&h))
                         : "memory");
          }
          __syncwarp();
#pragma unroll
          for (int it = 0; it < 4; ++it) {
            const int jj = it * 8 + (lane >> 2);
            const int part = lane & 3;
            const int pix = ch * 32 + jj;
            const int rr = pix / p.Wp, cw = pix % p.Wp;
            const int oh = h0 + rr;
            const int c8 = m0 + 32 * q + part * 8;
            if (pix < p.n_virt && cw < p.W && oh < p.H && c8 < p.Cout) {
              uint4 v;
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                           : "r"(stage + jj * 64 + part * 16));
              __nv_bfloat16* dst =
                  p.y + ((static_cast<size_t>(b) * p.H + oh) * p.W + cw) * p.Cout + c8;
              *reinterpret_cast<uint4*>(dst) = v;
            }
          }
          __syncwarp();
        }
        // this warp is done reading the accumulator of unit j
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(aempty);
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dc
