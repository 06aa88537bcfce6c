// Tensor-core gradients of the kernel mixture. With the per-sample weight
// gradients dW_b (the kernel is a weighted sum of static kernels,
// KernelWarehouse, abstract; one kernel per example, CondConv, abstract):
//     dexperts[i][w] = sum_b alpha[b][i] * dW[b][w]
//     dalpha[b][i]   = sum_w dW[b][w] * E[i][w]      (+ <db_b, bias_i>, added later)
// Both contract the same dW tile, so one pass over dW serves both GEMMs:
//  * dW arrives as two bf16 planes, hi = bf16(v) and lo = bf16(v - hi)
//    (~16 bits of v); a stage holds [128 samples][128 weights] of each plane
//    (two 64-weight atoms, rows = samples, 128-byte swizzle), zero-filled by
//    TMA past the batch;
//  * dexperts: M = 128 weights, N = 2 x experts, K = samples. The dW tile is
//    an MN-major A operand as stored; B = alpha split as hi (rows 0..nk-1) and
//    lo (rows nk..2nk-1) of one K-major operand built once per CTA, so one
//    MMA per dW plane and K step gives dW * alpha_hi and dW * alpha_lo side
//    by side; the epilogue adds the two column blocks;
//  * dalpha: M = 128 samples, N = experts, K = weights. The SAME dW tile is a
//    K-major A operand; B = the experts' tile, K-major, bf16 exact.
//    Products hi*E + lo*E, accumulated in TMEM over all tiles of the CTA.
// Persistent CTAs walk the 128-weight tiles (both sample halves per tile);
// each tile's dexperts is complete when its last half is in (no partials) and
// leaves through a double-buffered accumulator; each CTA's dalpha sums leave
// once at the end as one partial [CTA][B][n], summed in CTA order afterwards.
// Warp 0 issues TMA, warp 1 the MMAs, warps 2..5 read TMEM. Every wait is
// bounded.
#pragma once

#include "common.cuh"

namespace dcb {

constexpr int kMtThreads = 192;
constexpr int kMtTile = 128;  // weights per tile

struct MtParams {
  int B, n, nk;       // samples (<= 256), experts (<= 64), experts padded to 16, 32 or 64
  int halves;         // ceil(B / 128)
  int stages;
  long long wsize;
  long long tiles;    // wsize / 128
  int plane_bytes;    // one plane's tile: 2 atoms x 128 rows x 128 B = 32 KB
  int e_bytes;        // experts' tile: 2 atoms x nk rows x 128 B
  int stage_bytes;    // hi + lo + experts
  int b_bytes;        // alpha operand: (halves * 2) atoms x 2*nk rows x 128 B
  const float* alpha;  // [B][n]
  float* dexperts;     // [n][wsize]
  float* part;         // [gridDim.x][B][n]
  int* err;
  long long wait_ns;
};

__global__ void __launch_bounds__(kMtThreads, 1)
    mixgrad_tc_kernel(const __grid_constant__ CUtensorMap himap,
                      const __grid_constant__ CUtensorMap lomap,
                      const __grid_constant__ CUtensorMap emap, MtParams p) {
  using namespace dc;
  extern __shared__ __align__(1024) unsigned char mt_smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(mt_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = mt_smem_raw + (base - raw);
  const int S = p.stages;
  const uint32_t al_base = base;                  // [K atom][2nk rows (hi, lo) x 128 B]
  const uint32_t st_base = al_base + p.b_bytes;   // [stage][hi | lo | experts]
  const uint32_t bar_base = st_base + S * p.stage_bytes;
  auto full = [&](int s) { return bar_base + 8u * s; };
  auto empty = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * S + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * S + 2 + a); };
  const uint32_t adone = bar_base + 8u * (2 * S + 4);
  const uint32_t drain_bar = adone + 8u;
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * S + 6);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};
  // TMEM columns: two dexperts accumulators of 2 nk columns (hi | lo) at 0
  // and 2 nk, then the dalpha halves (nk columns each) from 4 nk
  const uint32_t dex_cols = 2u * p.nk;
  const uint32_t da_base = 2u * dex_cols;
  const uint32_t kCols = da_base + 2u * p.nk <= 256u ? 256u : 512u;

  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), kCols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), 4);
    }
    mbar_init(adone, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&himap);
    tma_prefetch_desc(&lomap);
    tma_prefetch_desc(&emap);
  }
  // alpha as the dexperts GEMM's B operand: K-major, row = expert (hi rows
  // 0..nk-1, lo rows nk..2nk-1), K = sample, 64 samples per 128-byte row
  // (atom), zero outside [B) x [n)
  for (int e = threadIdx.x; e < p.b_bytes / 16; e += kMtThreads)
    st_shared_v4(al_base + e * 16, make_uint4(0u, 0u, 0u, 0u));
  __syncthreads();
  for (int e = threadIdx.x; e < p.B * p.n; e += kMtThreads) {
    const int b = e / p.n, i = e - b * p.n;
    const float a = p.alpha[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(a);
    const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
    const uint32_t atom = static_cast<uint32_t>(b >> 6) * 2u * p.nk * 128u;
    const int rl = i + p.nk;  // the lo row
    const uint32_t off_hi = atom + i * 128u + ((((b & 63) >> 3) ^ (i & 7)) << 4) + (b & 7) * 2;
    const uint32_t off_lo = atom + rl * 128u + ((((b & 63) >> 3) ^ (rl & 7)) << 4) + (b & 7) * 2;
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(al_base + off_hi),
                 "h"(*reinterpret_cast<const unsigned short*>(&hi)) : "memory");
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(al_base + off_lo),
                 "h"(*reinterpret_cast<const unsigned short*>(&lo)) : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long my_tiles =
      p.tiles > blockIdx.x ? (p.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const uint32_t atom_bytes = 128u * 128u;  // one plane atom: 128 samples x 128 B

  if (warp == 0) {
    // ================================ TMA ================================
    if (lane == 0) {
      long long issued = 0;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long long j = 0; j < my_tiles && ok; ++j) {
        const long long t = blockIdx.x + j * gridDim.x;
        for (int h = 0; h < p.halves; ++h) {
          if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(2 * p.plane_bytes + p.e_bytes));
          const uint32_t dst = st_base + s * p.stage_bytes;
          for (int a = 0; a < 2; ++a) {
            const int w0 = static_cast<int>(t * kMtTile + a * 64);
            tma_load_2d(dst + a * atom_bytes, &himap, full(s), w0, h * 128);
            tma_load_2d(dst + p.plane_bytes + a * atom_bytes, &lomap, full(s), w0, h * 128);
            tma_load_2d(dst + 2 * p.plane_bytes + a * p.nk * 128, &emap, full(s), w0, 0);
          }
          ++issued;
          if (++s == S) { s = 0; ph ^= 1u; }
        }
      }
      for (long long k = (issued > S ? issued - S : 0); k < issued; ++k)
        wait_drain(full(static_cast<int>(k % S)), static_cast<uint32_t>((k / S) & 1), p.wait_ns,
                   p.err);
    }
  } else if (warp == 1) {
    // ================================ MMA ================================
    if (lane == 0) {
      // dexperts: A (dW) MN-major, B (alpha) K-major; dalpha: both K-major
      const uint32_t idesc_dex = idesc_bf16_f32(128, 2 * p.nk) | (1u << 15);
      const uint32_t idesc_da = idesc_bf16_f32(128, p.nk);
      const uint64_t al = smem_desc_sw128(al_base);
      const uint64_t al_kcol = static_cast<uint64_t>(2 * p.nk) * (128 >> 4);  // next 64 samples
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long long j = 0; j < my_tiles && ok; ++j) {
        const int ab = static_cast<int>(j & 1);
        if (!wait_bounded(tempty(ab), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, ctl, kErrWaitMma)) {
          ok = false;
          break;
        }
        const uint32_t d_dex = tmem_base + ab * dex_cols;
        for (int h = 0; h < p.halves; ++h) {
          if (!wait_bounded(full(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = st_base + s * p.stage_bytes;
          // dexperts: K = the half's 128 samples in 8 steps of 16 rows (+2048 B)
          const uint64_t dh_mn = smem_desc_mn_sw128_lbo(st, atom_bytes);
          const uint64_t dl_mn = smem_desc_mn_sw128_lbo(st + p.plane_bytes, atom_bytes);
          for (int kk = 0; kk < 8; ++kk) {
            const int ks = h * 8 + kk;  // 16-sample step in the batch
            const uint64_t boff = static_cast<uint64_t>(ks >> 2) * al_kcol + (ks & 3) * 2;
            const uint64_t aoff = static_cast<uint64_t>(kk) * (2048 >> 4);
            tc_mma_f16(d_dex, dh_mn + aoff, al + boff, idesc_dex, (h > 0 || kk > 0) ? 1u : 0u);
            tc_mma_f16(d_dex, dl_mn + aoff, al + boff, idesc_dex, 1u);
          }
          // dalpha of this half: K = the tile's 128 weights, two 64-weight atoms
          const uint32_t d_da = tmem_base + da_base + h * p.nk;
          for (int kk = 0; kk < 8; ++kk) {
            const int a = kk >> 2;
            const uint64_t koff = (kk & 3) * 2;
            const uint64_t dh_k = smem_desc_sw128(st + a * atom_bytes) + koff;
            const uint64_t dl_k = smem_desc_sw128(st + p.plane_bytes + a * atom_bytes) + koff;
            const uint64_t e_k = smem_desc_sw128(st + 2 * p.plane_bytes + a * p.nk * 128) + koff;
            tc_mma_f16(d_da, dh_k, e_k, idesc_da, (j > 0 || kk > 0) ? 1u : 0u);
            tc_mma_f16(d_da, dl_k, e_k, idesc_da, 1u);
          }
          tc_commit(empty(s));
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull(ab));
      }
      if (ok) {
        tc_commit(adone);
      } else {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else {
    // ============================= epilogue =============================
    // warp w reads TMEM lanes 32*(w%4) .. +31: weights of the tile (dexperts)
    // or samples of a half (dalpha)
    const int q = warp & 3;
    bool ok = true;
    for (long long j = 0; j < my_tiles; ++j) {
      const long long t = blockIdx.x + j * gridDim.x;
      const int ab = static_cast<int>(j & 1);
      if (!wait_bounded(tfull(ab), static_cast<uint32_t>((j >> 1) & 1), ctl, kErrWaitEpilogue)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // columns 0..nk-1: dW * alpha_hi, nk..2nk-1: dW * alpha_lo; 32 experts
      // per pass
      const uint32_t ta = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * dex_cols;
      float* dst = p.dexperts + t * kMtTile + 32 * q + lane;
      for (int e0 = 0; e0 < p.nk; e0 += 32) {
        uint32_t r[32], r2[32];
        tmem_ld_32x32b_x32(ta + e0, r);
        tmem_ld_32x32b_x32(ta + p.nk + e0, r2);
        tmem_ld_wait(r);
        tmem_ld_wait(r2);
        if (e0 + 32 >= p.nk) {
          // every read of this accumulator is complete: release it
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(tempty(ab));
        }
#pragma unroll
        for (int i = 0; i < 32; ++i)
          if (e0 + i < p.n && i < p.nk)
            dst[static_cast<size_t>(e0 + i) * p.wsize] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
      }
    }
    if (ok && my_tiles > 0 && wait_bounded(adone, 0, ctl, kErrWaitEpilogue)) {
      tc_fence_after();
      for (int h = 0; h < p.halves; ++h) {
        for (int e0 = 0; e0 < p.nk; e0 += 32) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(
              tmem_base + (static_cast<uint32_t>(32 * q) << 16) + da_base + h * p.nk + e0, r);
          tmem_ld_wait(r);
          const int b = h * 128 + 32 * q + lane;
          if (b < p.B) {
            float* dst = p.part + (static_cast<size_t>(blockIdx.x) * p.B + b) * p.n + e0;
#pragma unroll
            for (int i = 0; i < 32; ++i)
              if (e0 + i < p.n && i < p.nk) dst[i] = __uint_as_float(r[i]);
          }
        }
      }
    } else if (my_tiles == 0) {
      // no tile: this CTA's partial is zero
      for (int h = 0; h < p.halves; ++h) {
        const int b = h * 128 + 32 * q + lane;
        if (b < p.B)
          for (int i = 0; i < p.n; ++i)
            p.part[(static_cast<size_t>(blockIdx.x) * p.B + b) * p.n + i] = 0.f;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, kCols);
  }
}

}  // namespace dcb
