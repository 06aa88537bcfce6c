// Tensor-core per-sample weight gradient:
//   dW_b[co][kh][kw][ci] = sum over output pixels (oh, ow) of
//                          dy[b][oh][ow][co] * x[b][oh+kh-p][ow+kw-p][ci]
// (stride 1, groups 1, zero outside the image) -- the gradient of the
// convolution with the per-example kernel (CondConv, abstract), which the
// mixture's gradients then combine (KernelWarehouse, abstract: the kernel is a
// weighted sum of static kernels, so each expert's gradient is the
// attention-weighted sum of the per-sample gradients).
//
// One sample's gradient is a GEMM with M = output channels, N = (tap, input
// channel), K = output pixels. Both operands come straight from the NHWC
// tensors as MN-major tiles, no transposition:
//  * A = dy: a TMA box {64 channels, W_out, BH rows, 1} lands as BH*W_out
//    rows of 128 bytes (one per output pixel) in the 128-byte swizzle; two
//    such 64-channel atoms (LBO apart) make M = 128.
//  * B = x shifted by one tap: the same box shape at (ci0, kw-p, oh0+kh-p, b),
//    zero-filled by TMA outside the image. Each of up to four atoms is one
//    (tap, 64-channel block) pair, so one MMA has N = 64 * atoms <= 256.
//  * K rows: a K tile is BH whole output rows (BH*W_out <= 128 pixels); rows
//    past it up to the next multiple of 16 stay zero (written once at start,
//    never by TMA), so every MMA step covers 16 rows.
//  * D (fp32) in TMEM, double-buffered (2 x 256 columns) so that the store of
//    one unit overlaps the MMAs of the next.
// A unit of work is (sample, 128 output channels, group of <= 4 atoms);
// persistent CTAs walk the units. Warp 0 issues TMA, warp 1 the MMAs, warps
// 2..5 move D to the fp32 dW buffer [B][C_out][KH][KW][C_in]. Every wait is
// bounded; on expiry the kernel records the error, drains and exits.
#pragma once

#include "common.cuh"

namespace dcb {

constexpr int kWgThreads = 192;
constexpr int kWgMaxAtoms = 4;
constexpr int kWgStageBytes = 32 * 32 * 4;  // one warp's 32 rows x 32 fp32

// Shared-memory matrix descriptor of an MN-major operand in the 128-byte
// swizzle: rows of 64 bf16 along M (or N), one row per K index; 64-element
// atoms `lbo` bytes apart (leading byte offset), 8-row K groups 1024 bytes
// apart (stride byte offset); fixed version 1 in bits 46-47, swizzle mode 2.
__device__ __forceinline__ uint64_t smem_desc_mn_sw128_lbo(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>(1024u >> 4) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

struct WgParams {
  int B, Cin, Cout, Ho, Wo, KH, KW, pad;
  int BH;           // output rows per K tile
  int ktiles;       // K tiles per sample, ceil(Ho / BH)
  int ksteps;       // 16-row MMA steps per K tile
  int atom_bytes;   // bytes of one 64-column atom of a stage (ksteps * 16 rows * 128 B)
  int box_bytes;    // bytes TMA writes into one atom (BH * Wo rows * 128 B)
  int cblk;         // ceil(Cin / 64)
  int natoms;       // KH * KW * cblk
  int agroups;      // ceil(natoms / 4)
  int co_tiles;     // ceil(Cout / 128)
  int stages;
  long long units;  // B * co_tiles * agroups
  float* dW;        // fp32 [B][Cout][KH][KW][Cin] -- or, with hilo, two bf16 planes there
  int hilo;         // 1: dW as bf16 hi = bf16(v) and lo = bf16(v - hi), planes [B][wsize] each
  int* err;
  long long wait_ns;
};

__global__ void __launch_bounds__(kWgThreads, 1)
    wgrad_tc_kernel(const __grid_constant__ CUtensorMap dymap,
                    const __grid_constant__ CUtensorMap xmap, WgParams p) {
  using namespace dc;
  extern __shared__ __align__(1024) unsigned char wg_smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(wg_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = wg_smem_raw + (base - raw);
  const int S = p.stages;
  const uint32_t ab_bytes = static_cast<uint32_t>(p.atom_bytes);
  const uint32_t stage_bytes = (2 + kWgMaxAtoms) * ab_bytes;
  const uint32_t stg_base = base + S * stage_bytes;  // epilogue staging: 4 warps x 4 KB
  const uint32_t bar_base = stg_base + 4 * kWgStageBytes;
  auto full = [&](int s) { return bar_base + 8u * s; };
  auto empty = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * S + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * S + 4);
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * S + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  // every stage starts zero: the rows past a K tile stay zero for good
  for (uint32_t o = threadIdx.x * 16u; o < S * stage_bytes; o += kWgThreads * 16u)
    st_shared_v4(base + o, make_uint4(0u, 0u, 0u, 0u));
  fence_proxy_async_smem();
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
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
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&dymap);
    tma_prefetch_desc(&xmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const long long my_units =
      p.units > blockIdx.x ? (p.units - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const int taps = p.KH * p.KW;

  if (warp == 0) {
    if (lane == 0) {
      long long issued = 0;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long long j = 0; j < my_units && ok; ++j) {
        const long long u = blockIdx.x + j * gridDim.x;
        const int ag = static_cast<int>(u % p.agroups);
        const long long t = u / p.agroups;
        const int cot = static_cast<int>(t % p.co_tiles);
        const int b = static_cast<int>(t / p.co_tiles);
        const int nat = min(kWgMaxAtoms, p.natoms - ag * kWgMaxAtoms);
        const int co0 = cot * 128;
        const bool hi_half = co0 + 64 < p.Cout;  // rows 64..127 of A exist
        const uint32_t bytes =
            static_cast<uint32_t>((1 + (hi_half ? 1 : 0) + nat) * p.box_bytes);
        for (int kt = 0; kt < p.ktiles; ++kt) {
          if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(full(s), bytes);
          const uint32_t dst = base + s * stage_bytes;
          const int oh0 = kt * p.BH;
          tma_load_4d(dst, &dymap, full(s), co0, 0, oh0, b);
          if (hi_half) tma_load_4d(dst + ab_bytes, &dymap, full(s), co0 + 64, 0, oh0, b);
          for (int a = 0; a < nat; ++a) {
            const int atom = ag * kWgMaxAtoms + a;
            const int tap = atom / p.cblk, cb = atom - tap * p.cblk;
            const int kh = tap / p.KW, kw = tap - kh * p.KW;
            tma_load_4d(dst + (2 + a) * ab_bytes, &xmap, full(s), cb * 64, kw - p.pad,
                        oh0 + kh - p.pad, b);
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
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long long j = 0; j < my_units && ok; ++j) {
        const long long u = blockIdx.x + j * gridDim.x;
        const int ag = static_cast<int>(u % p.agroups);
        const int nat = min(kWgMaxAtoms, p.natoms - ag * kWgMaxAtoms);
        // A and B both MN-major (bits 15 and 16), N = 64 per atom
        const uint32_t idesc =
            idesc_bf16_f32(128, static_cast<uint32_t>(64 * nat)) | (1u << 15) | (1u << 16);
        const int ab = static_cast<int>(j & 1);
        if (!wait_bounded(tempty(ab), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, ctl, kErrWaitMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d = tmem_base + ab * 256;
        for (int kt = 0; kt < p.ktiles; ++kt) {
          if (!wait_bounded(full(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
          tc_fence_after();
          const uint32_t st = base + s * stage_bytes;
          const uint64_t a_desc = smem_desc_mn_sw128_lbo(st, ab_bytes);
          const uint64_t b_desc = smem_desc_mn_sw128_lbo(st + 2 * ab_bytes, ab_bytes);
          for (int kk = 0; kk < p.ksteps; ++kk)
            // 16 K rows = two 8-row groups of 1024 bytes
            tc_mma_f16(d, a_desc + kk * (2048 >> 4), b_desc + kk * (2048 >> 4), idesc,
                       (kt > 0 || kk > 0) ? 1u : 0u);
          tc_commit(empty(s));
          if (++s == S) { s = 0; ph ^= 1u; }
        }
        if (!ok) break;
        tc_commit(tfull(ab));
      }
      if (!ok) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else {
    // warps 2..5: warp w reads TMEM lanes 32*(w%4) .. +31, output channels
    // co0 + 32*(w%4) + lane. Each 32 x 32 fp32 block goes through shared
    // memory (16-byte slots XOR-ed with the row, conflict-free both ways) so
    // that every store instruction writes four whole 128-byte rows of dW.
    const int q = warp & 3;
    const uint32_t stg = stg_base + (warp - 2) * kWgStageBytes;
    for (long long j = 0; j < my_units; ++j) {
      const long long u = blockIdx.x + j * gridDim.x;
      const int ag = static_cast<int>(u % p.agroups);
      const long long t = u / p.agroups;
      const int cot = static_cast<int>(t % p.co_tiles);
      const int b = static_cast<int>(t / p.co_tiles);
      const int nat = min(kWgMaxAtoms, p.natoms - ag * kWgMaxAtoms);
      const int ab = static_cast<int>(j & 1);
      if (!wait_bounded(tfull(ab), static_cast<uint32_t>((j >> 1) & 1), ctl, kErrWaitEpilogue)) break;
      tc_fence_after();
      for (int a = 0; a < nat; ++a) {
        const int atom = ag * kWgMaxAtoms + a;
        const int tap = atom / p.cblk, cb = atom - tap * p.cblk;
#pragma unroll 1
        for (int h = 0; h < 2; ++h) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * 256 +
                                 a * 64 + h * 32,
                             r);
          tmem_ld_wait(r);
          if (p.hilo) {
            // hi / lo planes: each lane (row) stages its 32 values twice as
            // 64 bf16 bytes (16-byte chunks XOR-ed with the row's low bits);
            // every store instruction then writes 8 whole 64-byte row pieces
            const long long wsize = static_cast<long long>(p.Cout) * taps * p.Cin;
            __nv_bfloat16* hi_plane = reinterpret_cast<__nv_bfloat16*>(p.dW);
            __nv_bfloat16* lo_plane = hi_plane + static_cast<size_t>(p.B) * wsize;
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint32_t hw[4], lw[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const float f0 = __uint_as_float(r[8 * v + 2 * e]);
                const float f1 = __uint_as_float(r[8 * v + 2 * e + 1]);
                hw[e] = pack_bf16x2(f0, f1);
                lw[e] = pack_bf16x2(f0 - bf16lo_to_f32(hw[e]), f1 - bf16hi_to_f32(hw[e]));
              }
              const uint32_t slot = ((v ^ (lane & 3)) << 4);
              st_shared_v4(stg + lane * 64 + slot, make_uint4(hw[0], hw[1], hw[2], hw[3]));
              st_shared_v4(stg + 2048 + lane * 64 + slot, make_uint4(lw[0], lw[1], lw[2], lw[3]));
            }
            __syncwarp();
            const int ci = cb * 64 + h * 32 + 8 * (lane & 3);
#pragma unroll
            for (int it = 0; it < 4; ++it) {
              const int row = 8 * it + (lane >> 2);
              const uint32_t off = row * 64 + (((lane & 3) ^ (row & 3)) << 4);
              uint4 vh, vl;
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(vh.x), "=r"(vh.y), "=r"(vh.z), "=r"(vh.w)
                           : "r"(stg + off));
              asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                           : "=r"(vl.x), "=r"(vl.y), "=r"(vl.z), "=r"(vl.w)
                           : "r"(stg + 2048 + off));
              const int co_r = cot * 128 + 32 * q + row;
              if (co_r < p.Cout && ci < p.Cin) {
                const size_t e = (static_cast<size_t>(b) * p.Cout + co_r) * taps * p.Cin +
                                 static_cast<size_t>(tap) * p.Cin + ci;
                *reinterpret_cast<uint4*>(hi_plane + e) = vh;
                *reinterpret_cast<uint4*>(lo_plane + e) = vl;
              }
            }
            __syncwarp();
            continue;
          }
#pragma unroll
          for (int v = 0; v < 8; ++v)
            st_shared_v4(stg + lane * 128 + ((v ^ (lane & 7)) << 4),
                         make_uint4(r[4 * v], r[4 * v + 1], r[4 * v + 2], r[4 * v + 3]));
          __syncwarp();
          const int ci = cb * 64 + h * 32 + 4 * (lane & 7);
#pragma unroll
          for (int it = 0; it < 8; ++it) {
            const int row = 4 * it + (lane >> 3);
            uint4 v;
            asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                         : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                         : "r"(stg + row * 128 + (((lane & 7) ^ (row & 7)) << 4)));
            const int co_r = cot * 128 + 32 * q + row;
            if (co_r < p.Cout && ci < p.Cin)
              *reinterpret_cast<uint4*>(
                  p.dW + ((static_cast<size_t>(b) * p.Cout + co_r) * taps + tap) * p.Cin + ci) = v;
          }
          __syncwarp();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(ab));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

}  // namespace dcb
