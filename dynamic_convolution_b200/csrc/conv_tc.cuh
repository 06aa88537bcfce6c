// Tensor-core (tcgen05) implicit-GEMM dynamic convolution, bf16 in / out,
// fp32 accumulation in tensor memory. Stride 1, "same" padding.
//
// Per work unit (sample b, block of R output rows, block of 128 output
// channels) the kernel computes
//     D[co][p] = sum_{tap, c} A_tap[co][c] * X[p + s_tap][c]
// The GEMM is "swapped": M = output channels (128 per tile), N = pixels, so
// the per-sample kernel is the A operand and the pixel count only has to be a
// multiple of 16.
//
// Activations: the unit's input rows plus the KH-1 halo rows, at the padded
// width Wp = W + KW - 1, are loaded ONCE per 64-channel chunk with one 4-D TMA
// box {64 channels, Wp, R+KH-1, 1} at (c, -pad, h0-pad, b); out-of-bounds
// reads are the zero padding. Output pixels are computed on the same padded
// grid (p = r*Wp + c; columns c >= W are discarded), so tap (kh, kw) reads the
// tile at a constant row shift s_tap = kh*Wp + kw: every tap is the same smem
// tile at another descriptor start address. The 128-byte swizzle is applied
// on absolute shared-memory address bits by both the TMA and the tensor core,
// so a view may start at any 128-byte row with the descriptor's base offset
// left at 0 (checked on B200 against the oracle). Each activation byte
// crosses L2 once per unit instead of once per tap.
//
// The weight operand A (128 x 64 bf16 per step, K-major, 128-byte swizzle)
// depends on the variant:
//   FUSED    A = sum_i alpha_{b,i} E_i[co-tile][tap][c-chunk], mixed by 8 warps
//            on CUDA cores from expert tiles that one thread TMA-loads into a
//            ring in shared memory (the same swizzled layout as A, so the mix
//            is elementwise) and rounded once to bf16:
//            the kernel is a weighted sum of n static kernels with weights
//            that depend on the input (KernelWarehouse, abstract), one
//            kernel per example (CondConv, abstract);
//   OUTSIDE  the step also runs over the experts and A = alpha_{b,i} E_i (one
//            TMA-loaded expert tile per step, scaled and rounded): the
//            sum over experts happens in the accumulator,
//            y = sum_i alpha_i (x conv W_i) -- the same result by linearity;
//   PREMIX   A = W_b tile, TMA-loaded from a workspace where the premix kernel
//            stored every sample's mixed kernel.
// One thread issues tcgen05.mma (M=128, N<=256 per instruction, K=16) and
// commits each stage back to its "empty" barrier. The epilogue reads TMEM
// lane = output channel with 16x256b loads, adds the mixed bias
// sum_i alpha_i bias_i, rounds to bf16, transposes 8x8 blocks into shared
// memory with stmatrix and writes 16-byte NHWC segments.
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
// The epilogue stages 12 x 2 KB in the idle A stages; the pooled channel
// sums (3 x 128 floats) follow them (the A stages hold at least 32 KB).
constexpr int kTcPoolOff = 12 * 2048;

enum TcVariant { kFused = 1, kOutside = 2, kPremix = 3 };

struct TcParams {
  int B, H, W, Cin, Cout, KH, KW, pad, n;
  int R;              // output rows per unit
  int tiles_h;        // ceil(H / R)
  int m_tiles;        // ceil(Cout / 128)
  int Wp;             // padded width W + KW - 1
  int n_virt;         // R * Wp pixels on the padded grid
  int n_mma0, n_mma1; // MMA N of the two column chunks (n_mma1 may be 0)
  int kc;             // 64-channel chunks: ceil(Cin / 64)
  int spc;            // A steps per chunk: taps (FUSED, PREMIX) or n * taps (OUTSIDE)
  int k_steps;        // kc * spc
  int sa, sb;         // A and B pipeline stages
  int b_tile_bytes;   // bytes of one activation stage (1024-aligned)
  int b_box_rows;     // R + KH - 1
  uint32_t tmem_cols;
  int desc_base_mode; // 0 (correct on B200); 1 writes (address >> 7) & 7 as base offset
  const __nv_bfloat16* experts;
  const float* alpha;
  const float* bias;  // may be null
  __nv_bfloat16* y;
  int* err;
  long long wait_ns;
  int inject_skip;    // test hook: withhold the first mixer arrival of CTA 0
  float* ysum;        // optional [B][tiles_h][Cout]: per-unit channel sums of y as stored
  const float* a_out; // optional [B][Cout] output channel attention (FMDConv)
  const float* chan_add;  // optional [B][Cout]: chan_scale * chan_add[b][co] joins the mixed
  float chan_scale;       // bias before the single rounding of y
  int co_base;            // persistent kernel: channel offset of this launch in y and the biases
  int ld_c;               // persistent kernel: channel stride of y and bias rows (0: Cout)
  int x_early;            // PREMIX: first x boxes may load before the grid wait (after a mixer)
  int se;                 // FUSED / OUTSIDE: expert-tile stages (16 KB each)
  unsigned long long* stamps;  // optional [grid][8] phase stamps for measurements, or null
};

// Phase stamps of one CTA (measurement hook): slot i of this CTA's 8 holds the
// SM cycle counter (slots 0..5), the SM id (6) and the global timer at entry
// (7, nanoseconds, to align CTAs of different SMs).
__device__ __forceinline__ void tc_stamp(const TcParams& p, int i) {
  if (p.stamps != nullptr) {
    p.stamps[static_cast<size_t>(blockIdx.x) * 8 + i] = clock64();
    if (i == 0) p.stamps[static_cast<size_t>(blockIdx.x) * 8 + 7] = globaltimer_ns();
  }
}

// ---- epilogue building blocks (both kernels)
// A warp owns one TMEM lane quarter (32 output channels) and walks its
// 32-pixel chunks. A chunk is loaded as two 16x256b.x4 loads (lanes 0..15 and
// 16..31 of the quarter): thread t then holds, per half h and 8-pixel group
// j, channels 16h + t/4 (e = 0) and 16h + 8 + t/4 (e = 1) at pixels 8j + 2(t%4)
// and +1 -- exactly the fragment of an 8x8 (channels x pixels) b16 matrix, so
// one stmatrix.trans per four matrices writes the chunk pixel-major into the
// warp's 2 KB staging tile: 64-byte pixel rows, 16-byte chunk c (channels
// 8c .. 8c+7) of local pixel p at position c ^ ((p >> 1) & 3), conflict-free
// for the matrix stores and for the 16-byte read-back.
__device__ __forceinline__ void epi_load_chunk(uint32_t trow, int col, uint32_t (&r)[32]) {
  tmem_ld_16x256b_x4(trow + static_cast<uint32_t>(col), r);
  tmem_ld_16x256b_x4(trow + (16u << 16) + static_cast<uint32_t>(col), r + 16);
}

__device__ __forceinline__ uint32_t epi_slot(uint32_t stage, int pix, int chunk) {
  return stage + pix * 64 + ((chunk ^ ((pix >> 1) & 3)) << 4);
}

// y = (accumulator + bias) * scale, rounded once to bf16, staged transposed.
// bias[h][e] and scale[h][e] belong to channel 16h + 8e + lane/4 of the quarter
// (SCALED false: no output attention, scale 1).
template <bool SCALED>
__device__ __forceinline__ void epi_stage_chunk(const uint32_t (&r)[32], const float (&bias)[2][2],
                                                const float (&scale)[2][2], uint32_t stage,
                                                int lane) {
  const int m = lane >> 3, rr = lane & 7;  // this thread addresses row rr of matrix m
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint32_t P[4][2];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const uint32_t* v = r + 16 * h + 4 * j;
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        float a = __uint_as_float(v[2 * e]) + bias[h][e];
        float b = __uint_as_float(v[2 * e + 1]) + bias[h][e];
        if (SCALED) {
          a *= scale[h][e];
          b *= scale[h][e];
        }
        P[j][e] = pack_bf16x2(a, b);
      }
    }
#pragma unroll
    for (int s2 = 0; s2 < 2; ++s2) {
      // matrices (e, j) = (0, 2s2), (1, 2s2), (0, 2s2+1), (1, 2s2+1)
      const int pix = 8 * (2 * s2 + (m >> 1)) + rr;
      stmatrix_x4_trans(epi_slot(stage, pix, 2 * h + (m & 1)), P[2 * s2][0], P[2 * s2][1],
                        P[2 * s2 + 1][0], P[2 * s2 + 1][1]);
    }
  }
}

__device__ __forceinline__ uint64_t tc_desc(uint32_t saddr, int base_mode) {
  uint64_t d = smem_desc_sw128(saddr);
  if (base_mode) d |= static_cast<uint64_t>((saddr >> 7) & 7u) << 49;
  return d;
}

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
  const int SA = p.sa, SB = p.sb;
  const int SE = VARIANT == kPremix ? 0 : p.se;  // expert-tile stages (FUSED, OUTSIDE)
  const uint32_t a_base = base;
  const uint32_t e_base = a_base + SA * kTcATileBytes;
  const uint32_t b_base = e_base + SE * kTcATileBytes;
  const uint32_t bar_base = b_base + SB * p.b_tile_bytes;
  auto fullA = [&](int s) { return bar_base + 8u * s; };
  auto emptyA = [&](int s) { return bar_base + 8u * (SA + s); };
  auto fullB = [&](int s) { return bar_base + 8u * (2 * SA + s); };
  auto emptyB = [&](int s) { return bar_base + 8u * (2 * SA + SB + s); };
  const uint32_t accum_bar = bar_base + 8u * (2 * SA + 2 * SB);
  const uint32_t drain_bar = accum_bar + 8u;
  auto fullE = [&](int s) { return bar_base + 8u * (2 * SA + 2 * SB + 2 + s); };
  auto emptyE = [&](int s) { return bar_base + 8u * (2 * SA + 2 * SB + 2 + SE + s); };
  const uint32_t bias_bar = bar_base + 8u * (2 * SA + 2 * SB + 2 + 2 * SE);
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * SA + 2 * SB + 3 + 2 * SE);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  float* alpha_s = reinterpret_cast<float*>(misc + 16);
  // the tile's 128 mixed biases and output attentions, made by warp 3 while
  // the MMAs run
  float* bias_s = reinterpret_cast<float*>(misc + 16 + ((4 * p.n + 15) & ~15));
  float* scale_s = bias_s + 128;

  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  // Everything above this line is set-up that reads no global memory; with a
  // programmatic launch edge it overlaps the tail of the previous kernel.
  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), p.tmem_cols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    tc_stamp(p, 0);  // entry
    for (int s = 0; s < SA; ++s) {
      mbar_init(fullA(s), VARIANT == kPremix ? 1 : kTcMixThreads / 32);
      mbar_init(emptyA(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(fullB(s), 1);
      mbar_init(emptyB(s), 1);
    }
    mbar_init(accum_bar, 1);
    mbar_init(drain_bar, 1);
    mbar_init(bias_bar, 1);
    for (int s = 0; s < SE; ++s) {
      mbar_init(fullE(s), 1);
      mbar_init(emptyE(s), kTcMixThreads / 32);
    }
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&wmap);
  }
  __syncwarp();
  // The first activation boxes need nothing but the barriers. After one of
  // this library's mixing kernels (p.x_early: they signal their dependents
  // only once every CTA is past its own wait, so whatever wrote x has
  // completed) they are issued before this kernel's wait, overlapping the
  // mixing kernel's tail; otherwise right after it.
  const int pre_b = p.kc < SB ? p.kc : SB;
  if (threadIdx.x == 32 && p.x_early) {
    for (int cc = 0; cc < pre_b; ++cc) {
      mbar_arrive_expect_tx(fullB(cc), 64u * 2u * p.Wp * p.b_box_rows);
      tma_load_4d(b_base + cc * p.b_tile_bytes, &xmap, fullB(cc), cc * 64, -p.pad, h0 - p.pad, b);
    }
  }
  grid_dependency_wait();
  // the next kernel on the stream (a routing kernel of the next layer) may
  // be scheduled while this one runs: it waits for this grid's completion
  // before it reads anything this grid writes
  grid_launch_dependents();
  if (threadIdx.x == 32) {
    tc_stamp(p, 1);  // past the grid wait
    for (int cc = 0; cc < (p.x_early ? 0 : pre_b); ++cc) {
      mbar_arrive_expect_tx(fullB(cc), 64u * 2u * p.Wp * p.b_box_rows);
      tma_load_4d(b_base + cc * p.b_tile_bytes, &xmap, fullB(cc), cc * 64, -p.pad, h0 - p.pad, b);
    }
    if (VARIANT == kPremix) {
      const int pre_a = p.k_steps < SA ? p.k_steps : SA;
      for (int k = 0; k < pre_a; ++k) {
        mbar_arrive_expect_tx(fullA(k), kTcATileBytes);
        tma_load_3d(a_base + k * kTcATileBytes, &wmap, fullA(k), (k / p.spc) * 64, k % p.spc,
                    b * p.Cout + m0);
      }
    }
  }
  if (VARIANT != kPremix)  // PREMIX needs alpha only for the bias, in the epilogue
    for (int i = threadIdx.x; i < p.n; i += kTcThreads)
      alpha_s[i] = p.alpha[static_cast<size_t>(b) * p.n + i];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int taps = p.KH * p.KW;

  if (warp == 0) {
    // ======================= activation producer (TMA) =======================
    if (lane == 0) {
      const int pre_b = p.kc < SB ? p.kc : SB;  // issued during set-up
      int issued = pre_b;
      const uint32_t bytes = 64u * 2u * p.Wp * p.b_box_rows;
      for (int cc = pre_b; cc < p.kc; ++cc) {
        const int s = cc % SB;
        const uint32_t ph = static_cast<uint32_t>(cc / SB) & 1u;
        if (!wait_bounded(emptyB(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
        mbar_arrive_expect_tx(fullB(s), bytes);
        tma_load_4d(b_base + s * p.b_tile_bytes, &xmap, fullB(s), cc * 64, -p.pad, h0 - p.pad, b);
        ++issued;
      }
      for (int j = (issued > SB ? issued - SB : 0); j < issued; ++j)
        wait_drain(fullB(j % SB), static_cast<uint32_t>(j / SB) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 2) {
    // ============ expert-tile producer (FUSED, OUTSIDE): TMA, consumption order ============
    if constexpr (VARIANT != kPremix) {
      if (lane == 0) {
      const int ne = VARIANT == kFused ? p.n : 1;
      int issued = 0;
      bool ok = true;
      for (int k = 0; k < p.k_steps && ok; ++k) {
        const int cc = k / p.spc, t = k % p.spc;
        const int tap = VARIANT == kFused ? t : t % taps;
        for (int j = 0; j < ne; ++j, ++issued) {
          const int i = VARIANT == kFused ? j : t / taps;  // expert
          const int s = issued % SE;
          const uint32_t ph = static_cast<uint32_t>(issued / SE) & 1u;
          if (!wait_bounded(emptyE(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(fullE(s), kTcATileBytes);
          tma_load_3d(e_base + s * kTcATileBytes, &wmap, fullE(s), cc * 64, tap, i * p.Cout + m0);
        }
      }
      for (int j = (issued > SE ? issued - SE : 0); j < issued; ++j)
        wait_drain(fullE(j % SE), static_cast<uint32_t>(j / SE) & 1u, p.wait_ns, p.err);
      }
    }
    // ======================= weight producer (PREMIX) =======================
    if (VARIANT == kPremix && lane == 0) {
      const int pre_a = p.k_steps < SA ? p.k_steps : SA;  // issued during set-up
      int issued = pre_a;
      for (int k = pre_a; k < p.k_steps; ++k) {
        const int s = k % SA;
        const uint32_t ph = static_cast<uint32_t>(k / SA) & 1u;
        if (!wait_bounded(emptyA(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
        const int cc = k / p.spc, tap = k % p.spc;
        mbar_arrive_expect_tx(fullA(s), kTcATileBytes);
        tma_load_3d(a_base + s * kTcATileBytes, &wmap, fullA(s), cc * 64, tap, b * p.Cout + m0);
        ++issued;
      }
      for (int j = (issued > SA ? issued - SA : 0); j < issued; ++j)
        wait_drain(fullA(j % SA), static_cast<uint32_t>(j / SA) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 1) {
    // ======================= MMA issuer =======================
    // The tensor pipe accepts the next MMA only about when it starts the
    // previous one, so anything this single thread does between two steps
    // leaves the pipe idle. The loop therefore carries all indices as counters
    // and builds descriptors by adding offsets to precomputed ones (no
    // divisions, no tables): start-address fields count 16-byte units.
    if (lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(128, p.n_mma0);
      const uint32_t idesc1 = idesc_bf16_f32(128, p.n_mma1 > 0 ? p.n_mma1 : 16);
      const uint64_t a_desc0 = tc_desc(a_base, 0);
      const uint64_t b_desc0 = tc_desc(b_base, p.desc_base_mode);
      const uint64_t b_n1 = static_cast<uint64_t>(p.n_mma0) * 8u;  // n_mma0 rows of 128 B
      const uint64_t b_stage = static_cast<uint64_t>(p.b_tile_bytes) >> 4;
      const uint64_t row_skip = static_cast<uint64_t>(p.Wp - p.KW + 1) * 8u;
      const bool two = p.n_mma1 > 0;
      uint32_t s = 0, ph = 0, sbi = 0, phb = 0;
      int t = 0, tap = 0, kw = 0;
      uint64_t tap_off = 0;  // s_tap * 128 bytes, in 16-byte units
      // The operands of step k+1 are waited for before the last two MMAs of
      // step k are issued, so that the barrier probes and the fence overlap
      // MMAs already queued in the tensor pipe.
      bool ok = p.k_steps > 0 && wait_bounded(fullB(0), 0, ctl, kErrWaitMma) &&
                wait_bounded(fullA(0), 0, ctl, kErrWaitMma);
      if (ok) tc_fence_after();
      tc_stamp(p, 2);  // first operands in shared memory
      for (int k = 0; k < p.k_steps && ok; ++k) {
        const uint64_t ad = a_desc0 + s * (kTcATileBytes >> 4);
        const uint64_t bd = b_desc0 + sbi * b_stage + tap_off;
        const uint32_t acc0 = k > 0 ? 1u : 0u;
        tc_mma_f16(tmem_base, ad, bd, idesc0, acc0);
        if (two) tc_mma_f16(tmem_base + p.n_mma0, ad, bd + b_n1, idesc1, acc0);
#pragma unroll
        for (int q = 1; q < 3; ++q) {  // K=16 sub-steps: +32 bytes in both operands
          tc_mma_f16(tmem_base, ad + 2 * q, bd + 2 * q, idesc0, 1u);
          if (two) tc_mma_f16(tmem_base + p.n_mma0, ad + 2 * q, bd + b_n1 + 2 * q, idesc1, 1u);
        }
        // advance the tap (kw fastest), the step within the chunk, the stages
        const uint32_t s_cur = s, sbi_cur = sbi;
        bool chunk_end = false;
        if (++tap == taps) {
          tap = 0; kw = 0; tap_off = 0;
        } else if (++kw == p.KW) {
          kw = 0; tap_off += row_skip;
        } else {
          tap_off += 8u;
        }
        if (++t == p.spc) {
          t = 0;
          chunk_end = true;
          if (++sbi == static_cast<uint32_t>(SB)) { sbi = 0; phb ^= 1u; }
        }
        if (++s == static_cast<uint32_t>(SA)) { s = 0; ph ^= 1u; }
        // operands of the next step
        // (with a single activation stage the next chunk's box can only land
        // after this chunk's MMAs release the stage: wait for it after the commit)
        const bool b_now = chunk_end && SB > 1;
        if (k + 1 < p.k_steps) {
          if (b_now && !wait_bounded(fullB(sbi), phb, ctl, kErrWaitMma)) ok = false;
          if (ok && !wait_bounded(fullA(s), ph, ctl, kErrWaitMma)) ok = false;
          if (ok) tc_fence_after();
        }
        tc_mma_f16(tmem_base, ad + 6, bd + 6, idesc0, 1u);
        if (two) tc_mma_f16(tmem_base + p.n_mma0, ad + 6, bd + b_n1 + 6, idesc1, 1u);
        tc_commit(emptyA(s_cur));
        if (chunk_end) tc_commit(emptyB(sbi_cur));
        if (ok && chunk_end && SB == 1 && k + 1 < p.k_steps) {
          if (!wait_bounded(fullB(sbi), phb, ctl, kErrWaitMma)) ok = false;
          else tc_fence_after();
        }
      }
      tc_stamp(p, 3);  // last MMA issued
      if (ok) {
        tc_commit(accum_bar);
      } else {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else if (warp >= kTcMixWarp0) {
    const int mt_id = threadIdx.x - kTcMixWarp0 * 32;  // 0..255
    // ======================= mixers (FUSED / OUTSIDE) =======================
    // The expert tiles arrive by TMA in the same 128-byte-swizzled K-major
    // layout as the A tile, so the mix is elementwise over shared memory:
    // thread t takes the 16-byte chunks t, t + 256, t + 512, t + 768 of every
    // tile (conflict-free), accumulates alpha_i * E_i in fp32 in expert order
    // (FUSED: the step's n experts; OUTSIDE: the step's one expert) and
    // rounds once to bf16 into the A stage.
    if constexpr (VARIANT != kPremix) {
      const int ne = VARIANT == kFused ? p.n : 1;
      int consumed = 0;
      bool ok = true;
      for (int k = 0; k < p.k_steps && ok; ++k) {
        const int s = k % SA;
        const uint32_t ph = static_cast<uint32_t>(k / SA) & 1u;
        if (!wait_bounded(emptyA(s), ph ^ 1u, ctl, kErrWaitMixer)) break;
        const int t = k % p.spc;
        uint64_t acc[4][4];
#pragma unroll
        for (int uu = 0; uu < 4; ++uu)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[uu][e] = 0ull;
        for (int j = 0; j < ne; ++j, ++consumed) {
          const int es = consumed % SE;
          const uint32_t eph = static_cast<uint32_t>(consumed / SE) & 1u;
          if (!wait_bounded(fullE(es), eph, ctl, kErrWaitMixer)) { ok = false; break; }
          const float a = alpha_s[VARIANT == kFused ? j : t / taps];
          const uint64_t a2 = pack_f32x2(a, a);
          const uint32_t src = e_base + es * kTcATileBytes + mt_id * 16;
          uint4 v[4];
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) v[uu] = ld_shared_v4(src + uu * 4096);
          __syncwarp();
          if (lane == 0) mbar_arrive(emptyE(es));  // this warp is done reading the slot
#pragma unroll
          for (int uu = 0; uu < 4; ++uu) {
            acc[uu][0] = ffma2(a2, bf16x2_to_f32x2(v[uu].x), acc[uu][0]);
            acc[uu][1] = ffma2(a2, bf16x2_to_f32x2(v[uu].y), acc[uu][1]);
            acc[uu][2] = ffma2(a2, bf16x2_to_f32x2(v[uu].z), acc[uu][2]);
            acc[uu][3] = ffma2(a2, bf16x2_to_f32x2(v[uu].w), acc[uu][3]);
          }
        }
        if (!ok) break;
        const uint32_t dst = a_base + s * kTcATileBytes + mt_id * 16;
#pragma unroll
        for (int uu = 0; uu < 4; ++uu) {
          uint4 o;
          o.x = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[uu][0])),
                            __uint_as_float(static_cast<uint32_t>(acc[uu][0] >> 32)));
          o.y = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[uu][1])),
                            __uint_as_float(static_cast<uint32_t>(acc[uu][1] >> 32)));
          o.z = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[uu][2])),
                            __uint_as_float(static_cast<uint32_t>(acc[uu][2] >> 32)));
          o.w = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(acc[uu][3])),
                            __uint_as_float(static_cast<uint32_t>(acc[uu][3] >> 32)));
          st_shared_v4(dst + uu * 4096, o);
        }
        fence_proxy_async_smem();
        __syncwarp();
        const bool withhold = (p.inject_skip != 0) && k == 0 && blockIdx.x == 0;
        if (lane == 0 && !withhold) mbar_arrive(fullA(s));
      }
    }
  }

  if (warp == 3) {
    // ---- the tile's mixed biases sum_i alpha_i bias_i[co] (+ the per-channel
    // term) and output attentions, one channel per lane and pass, while the
    // MMAs run; published through bias_bar
    const float* ab = VARIANT == kPremix ? p.alpha + static_cast<size_t>(b) * p.n : alpha_s;
    for (int c = lane; c < 128; c += 32) {
      const int co = m0 + c;
      float acc = 0.f;
      if (p.bias != nullptr && co < p.Cout)
        for (int i = 0; i < p.n; ++i)
          acc = fmaf(ab[i], p.bias[static_cast<size_t>(i) * p.Cout + co], acc);
      if (p.chan_add != nullptr && co < p.Cout)
        acc = fmaf(p.chan_add[static_cast<size_t>(b) * p.Cout + co], p.chan_scale, acc);
      bias_s[c] = acc;
      // output attention: y = a_out * (conv + mixed bias), channel by channel
      scale_s[c] = (p.a_out != nullptr && co < p.Cout) ? p.a_out[static_cast<size_t>(b) * p.Cout + co]
                                                       : 1.f;
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(bias_bar);
  }

  // ======================= epilogue (all 12 warps) =======================
  // Warps 0..2 join once their lane 0 is done with its producer / MMA role,
  // warp 3 once the biases are made. Warp w reads TMEM lane quarter w % 4
  // (output channels 32*(w%4) ..) and every third 32-pixel chunk from w / 4.
  __syncwarp();
  {
    const int q = warp & 3;   // TMEM lane quarter
    const int grp = warp >> 2;  // chunk phase 0..2
    if (wait_bounded(accum_bar, 0, ctl, kErrWaitEpilogue) &&
        wait_bounded(bias_bar, 0, ctl, kErrWaitEpilogue)) {
      // the mixed bias (and output attention) of this thread's four channels
      // 32q + 16h + 8e + lane/4 of the tile
      float bb[2][2], so[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          bb[h][e] = bias_s[32 * q + 16 * h + 8 * e + (lane >> 2)];
          so[h][e] = scale_s[32 * q + 16 * h + 8 * e + (lane >> 2)];
        }
      tc_fence_after();
      if (threadIdx.x == 96) tc_stamp(p, 4);  // accumulator complete
      // Per warp: chunks of 32 pixels x 32 output channels. The next chunk's
      // TMEM load is in flight while this one is rounded, transposed through a
      // 2 KB staging tile in the (now idle) A stage buffers, and written as
      // 16-byte NHWC segments. Pixel coordinates on the padded grid advance
      // incrementally (one division per chunk).
      const uint32_t stage = a_base + warp * 2048;
      const int n_pad = p.n_mma0 + p.n_mma1;
      const int nchunks = (n_pad + 31) / 32;
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16);
      const int part = lane & 3;  // 16-byte part of a pixel's 64-byte row
      const int c8 = m0 + 32 * q + part * 8;
      const bool c_ok = c8 < p.Cout;
      __nv_bfloat16* ybase = p.y + static_cast<size_t>(b) * p.H * p.W * p.Cout + c8;
      // optional pooling for the next layer's routing: this thread's 8 output
      // channels summed over the pixels it stores, in a fixed order
      const bool pool = p.ysum != nullptr;
      float ps[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) ps[e] = 0.f;
      auto process = [&](const uint32_t (&r)[32], int ch) {
        if (p.a_out != nullptr) epi_stage_chunk<true>(r, bb, so, stage, lane);
        else epi_stage_chunk<false>(r, bb, so, stage, lane);
        __syncwarp();
        int pix = ch * 32 + (lane >> 2);
        int rr = pix / p.Wp;
        int cw = pix - rr * p.Wp;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int oh = h0 + rr;
          if (c_ok && pix < p.n_virt && cw < p.W && oh < p.H) {
            const uint4 v = ld_shared_v4(epi_slot(stage, it * 8 + (lane >> 2), part));
            *reinterpret_cast<uint4*>(ybase + (static_cast<size_t>(oh) * p.W + cw) * p.Cout) = v;
            if (pool) {
              const uint32_t w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                ps[2 * e] += bf16lo_to_f32(w4[e]);
                ps[2 * e + 1] += bf16hi_to_f32(w4[e]);
              }
            }
          }
          pix += 8;
          cw += 8;
          while (cw >= p.Wp) { cw -= p.Wp; ++rr; }
        }
        __syncwarp();
      };
      uint32_t ra[32], rb[32];
      int ch = grp;
      if (ch < nchunks) epi_load_chunk(trow, ch * 32, ra);
      while (ch < nchunks) {
        tmem_ld_wait(ra);
        if (ch + 3 < nchunks) epi_load_chunk(trow, (ch + 3) * 32, rb);
        process(ra, ch);
        ch += 3;
        if (ch >= nchunks) break;
        tmem_ld_wait(rb);
        if (ch + 3 < nchunks) epi_load_chunk(trow, (ch + 3) * 32, ra);
        process(rb, ch);
        ch += 3;
      }
      if (pool) {
        // lanes with the same 16-byte part hold the same channels: fixed tree,
        // then each (chunk phase, quarter) leaves 32 channel sums in shared memory
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          ps[e] += __shfl_xor_sync(0xffffffffu, ps[e], 4);
          ps[e] += __shfl_xor_sync(0xffffffffu, ps[e], 8);
          ps[e] += __shfl_xor_sync(0xffffffffu, ps[e], 16);
        }
        if (lane < 4) {
          float* dst = reinterpret_cast<float*>(base_ptr + kTcPoolOff) + grp * 128 + 32 * q + lane * 8;
#pragma unroll
          for (int e = 0; e < 8; ++e) dst[e] = ps[e];
        }
      }
    }
  }

  // ---- teardown
  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_stamp(p, 5);  // epilogue done
    if (p.stamps != nullptr) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      p.stamps[static_cast<size_t>(blockIdx.x) * 8 + 6] = smid;
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
  if (p.ysum != nullptr && threadIdx.x < 128 && m0 + static_cast<int>(threadIdx.x) < p.Cout &&
      !*abort_flag) {
    const float* src = reinterpret_cast<const float*>(base_ptr + kTcPoolOff);
    const float t = src[threadIdx.x] + src[128 + threadIdx.x] + src[256 + threadIdx.x];
    p.ysum[(static_cast<size_t>(b) * p.tiles_h + th) * p.Cout + m0 + threadIdx.x] = t;
  }
}

}  // namespace dc

namespace dc {

// ---------------------------------------------------------------------------
// Persistent form of the PREMIX convolution: one CTA per SM walks the units
// (sample, row block, 128-channel tile) blockIdx.x, +gridDim.x, ... with two
// TMEM accumulators, so that the epilogue of one unit (TMEM -> bias, rounding
// -> shared-memory transpose -> NHWC stores) runs while the MMAs of the next
// unit accumulate into the other buffer, and the TMA producers load the next
// unit's activations and mixed-kernel tiles meanwhile. Roles: warp 0 loads
// activation boxes, warp 2 loads mixed-kernel tiles, warp 1 issues the MMAs,
// warps 4..11 run the epilogue (two warps per TMEM lane quarter, alternate
// 32-pixel chunks). A launch may cover a slice of the output channels
// (co_base, with ld_c the full channel count) when the mixed kernels of one
// 128-channel group at a time are in the workspace.
// Same arithmetic, rounding and outputs as tc_conv_kernel
// with VARIANT = kPremix; the pooled channel sums of the chained-block forward
// are not produced here (that call runs tc_conv_kernel).
// ---------------------------------------------------------------------------

constexpr int kTpEpiWarp0 = 4;
constexpr int kTpEpiWarps = 8;
constexpr int kTpStageBytes = kTpEpiWarps * 2048;  // epilogue transpose tiles

__global__ void __launch_bounds__(kTcThreads, 1)
    tc_conv_persist_kernel(const __grid_constant__ CUtensorMap xmap,
                           const __grid_constant__ CUtensorMap wmap, TcParams p) {
  extern __shared__ __align__(1024) unsigned char tp_smem_raw[];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  const uint32_t raw = smem_u32(tp_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = tp_smem_raw + (base - raw);
  const int SA = p.sa, SB = p.sb;
  const uint32_t a_base = base;
  const uint32_t b_base = a_base + SA * kTcATileBytes;
  const uint32_t epi_base = b_base + SB * p.b_tile_bytes;  // 8 x 2 KB
  const uint32_t bar_base = epi_base + kTpStageBytes;
  auto fullA = [&](int s) { return bar_base + 8u * s; };
  auto emptyA = [&](int s) { return bar_base + 8u * (SA + s); };
  auto fullB = [&](int s) { return bar_base + 8u * (2 * SA + s); };
  auto emptyB = [&](int s) { return bar_base + 8u * (2 * SA + SB + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * SA + 2 * SB + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * SA + 2 * SB + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * SA + 2 * SB + 4);
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * SA + 2 * SB + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};

  const int units = p.B * p.tiles_h * p.m_tiles;
  const int my_units = static_cast<int>(blockIdx.x) < units
                           ? (units - static_cast<int>(blockIdx.x) + gridDim.x - 1) / gridDim.x
                           : 0;
  auto decode = [&](int i, int& b, int& h0, int& m0, int& th) {
    int u = static_cast<int>(blockIdx.x) + i * static_cast<int>(gridDim.x);
    const int mt = u % p.m_tiles;
    u /= p.m_tiles;
    th = u % p.tiles_h;
    b = u / p.tiles_h;
    m0 = mt * 128;
    h0 = th * p.R;
  };

  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), p.tmem_cols);
    tmem_relinquish();
  }
  if (threadIdx.x == 32) {
    tc_stamp(p, 0);  // entry
    for (int s = 0; s < SA; ++s) {
      mbar_init(fullA(s), 1);
      mbar_init(emptyA(s), 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(fullB(s), 1);
      mbar_init(emptyB(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), kTpEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&wmap);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The mixing kernel this convolution follows signals its dependents only
  // once all of its CTAs are past their own wait, so whatever wrote x has
  // completed: the first activation boxes are loaded before this kernel's
  // wait, overlapping the mixing kernel's tail. The mixed kernels are read
  // only after the wait. (p.x_early is 0 when the previous kernel on the
  // stream is not such a mixing kernel.)
  const int pre_x = (p.x_early && my_units > 0) ? (p.kc < SB ? p.kc : SB) : 0;
  if (warp == 0 && lane == 0 && pre_x > 0) {
    int b, h0, m0, th;
    decode(0, b, h0, m0, th);
    for (int cc = 0; cc < pre_x; ++cc) {
      mbar_arrive_expect_tx(fullB(cc), 64u * 2u * p.Wp * p.b_box_rows);
      tma_load_4d(b_base + cc * p.b_tile_bytes, &xmap, fullB(cc), cc * 64, -p.pad, h0 - p.pad, b);
    }
  }
  grid_dependency_wait();
  // the next kernel on the stream (a routing kernel of the next layer) may
  // be scheduled while this one runs: it waits for this grid's completion
  // before it reads anything this grid writes
  grid_launch_dependents();
  if (threadIdx.x == 32) tc_stamp(p, 1);  // past the grid wait
  const int taps = p.KH * p.KW;
  const uint32_t acc_cols = p.tmem_cols >> 1;

  if (warp == 0) {
    // ==================== activation producer (TMA) ====================
    if (lane == 0) {
      const uint32_t bytes = 64u * 2u * p.Wp * p.b_box_rows;
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < my_units && ok; ++i) {
        int b, h0, m0, th;
        decode(i, b, h0, m0, th);
        for (int cc = 0; cc < p.kc; ++cc, ++issued) {
          if (issued < pre_x) continue;  // loaded before the wait
          const int s = issued % SB;
          const uint32_t ph = static_cast<uint32_t>(issued / SB) & 1u;
          if (!wait_bounded(emptyB(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(fullB(s), bytes);
          tma_load_4d(b_base + s * p.b_tile_bytes, &xmap, fullB(s), cc * 64, -p.pad, h0 - p.pad, b);
        }
      }
      for (int j = (issued > SB ? issued - SB : 0); j < issued; ++j)
        wait_drain(fullB(j % SB), static_cast<uint32_t>(j / SB) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 2) {
    // ==================== mixed-kernel producer (TMA) ====================
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < my_units && ok; ++i) {
        int b, h0, m0, th;
        decode(i, b, h0, m0, th);
        int cc = 0, tap = 0;
        for (int k = 0; k < p.k_steps; ++k, ++issued) {
          const int s = issued % SA;
          const uint32_t ph = static_cast<uint32_t>(issued / SA) & 1u;
          if (!wait_bounded(emptyA(s), ph ^ 1u, ctl, kErrWaitProducer)) { ok = false; break; }
          mbar_arrive_expect_tx(fullA(s), kTcATileBytes);
          tma_load_3d(a_base + s * kTcATileBytes, &wmap, fullA(s), cc * 64, tap, b * p.Cout + m0);
          if (++tap == p.spc) { tap = 0; ++cc; }
        }
      }
      for (int j = (issued > SA ? issued - SA : 0); j < issued; ++j)
        wait_drain(fullA(j % SA), static_cast<uint32_t>(j / SA) & 1u, p.wait_ns, p.err);
    }
  } else if (warp == 1) {
    // ============================ MMA issuer ============================
    if (lane == 0) {
      const uint32_t idesc0 = idesc_bf16_f32(128, p.n_mma0);
      const uint64_t a_desc0 = tc_desc(a_base, 0);
      const uint64_t b_desc0 = tc_desc(b_base, p.desc_base_mode);
      const uint64_t b_stage = static_cast<uint64_t>(p.b_tile_bytes) >> 4;
      const uint64_t row_skip = static_cast<uint64_t>(p.Wp - p.KW + 1) * 8u;
      uint32_t s = 0, ph = 0, sbi = 0, phb = 0;
      bool ok = true;
      for (int i = 0; i < my_units && ok; ++i) {
        const int ab = i & 1;
        const uint32_t d = tmem_base + ab * acc_cols;
        if (!wait_bounded(tempty(ab), (static_cast<uint32_t>(i >> 1) & 1u) ^ 1u, ctl, kErrWaitMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        int t = 0, tap = 0, kw = 0;
        uint64_t tap_off = 0;
        if (!wait_bounded(fullB(sbi), phb, ctl, kErrWaitMma) ||
            !wait_bounded(fullA(s), ph, ctl, kErrWaitMma)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (i == 0) tc_stamp(p, 2);  // first operands of the first unit
        for (int k = 0; k < p.k_steps && ok; ++k) {
          const uint64_t ad = a_desc0 + s * (kTcATileBytes >> 4);
          const uint64_t bd = b_desc0 + sbi * b_stage + tap_off;
          tc_mma_f16(d, ad, bd, idesc0, k > 0 ? 1u : 0u);
#pragma unroll
          for (int q = 1; q < 3; ++q) tc_mma_f16(d, ad + 2 * q, bd + 2 * q, idesc0, 1u);
          const uint32_t s_cur = s, sbi_cur = sbi;
          bool chunk_end = false;
          if (++tap == taps) {
            tap = 0; kw = 0; tap_off = 0;
          } else if (++kw == p.KW) {
            kw = 0; tap_off += row_skip;
          } else {
            tap_off += 8u;
          }
          if (++t == p.spc) {
            t = 0;
            chunk_end = true;
            if (++sbi == static_cast<uint32_t>(SB)) { sbi = 0; phb ^= 1u; }
          }
          if (++s == static_cast<uint32_t>(SA)) { s = 0; ph ^= 1u; }
          if (k + 1 < p.k_steps) {
            if (chunk_end && !wait_bounded(fullB(sbi), phb, ctl, kErrWaitMma)) ok = false;
            if (ok && !wait_bounded(fullA(s), ph, ctl, kErrWaitMma)) ok = false;
            if (ok) tc_fence_after();
          }
          tc_mma_f16(d, ad + 6, bd + 6, idesc0, 1u);
          tc_commit(emptyA(s_cur));
          if (chunk_end) tc_commit(emptyB(sbi_cur));
        }
        if (ok) tc_commit(tfull(ab));
        if (i == 0) tc_stamp(p, 3);       // first unit's MMAs issued
        if (i == my_units - 1) tc_stamp(p, 4);  // last unit's MMAs issued
      }
      if (!ok) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else if (warp >= kTpEpiWarp0) {
    // ============================= epilogue =============================
    const int q = warp & 3;                    // TMEM lane quarter
    const int grp = (warp - kTpEpiWarp0) >> 2;  // chunk phase 0..1
    const uint32_t stage = epi_base + (warp - kTpEpiWarp0) * 2048;
    const int part = lane & 3;
    const int nchunks = (p.n_mma0 + 31) / 32;
    const int ldc = p.ld_c > 0 ? p.ld_c : p.Cout;  // channel stride of y and bias rows
    const int cb = p.co_base;                       // channel offset of this launch
    for (int i = 0; i < my_units; ++i) {
      const int ab = i & 1;
      int b, h0, m0, th;
      decode(i, b, h0, m0, th);
      // the mixed bias (and output attention) of this thread's four channels
      // 32q + 16h + 8e + lane/4 of the tile (cb + co in y and the biases)
      float bb[2][2], so[2][2];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int e2 = 0; e2 < 2; ++e2) {
          const int co = m0 + 32 * q + 16 * h + 8 * e2 + (lane >> 2);
          float acc = 0.f;
          if (p.bias != nullptr && co < p.Cout) {
            const float* al = p.alpha + static_cast<size_t>(b) * p.n;
            for (int e = 0; e < p.n; ++e)
              acc = fmaf(al[e], p.bias[static_cast<size_t>(e) * ldc + cb + co], acc);
          }
          if (p.chan_add != nullptr && co < p.Cout)
            acc = fmaf(p.chan_add[static_cast<size_t>(b) * ldc + cb + co], p.chan_scale, acc);
          bb[h][e2] = acc;
          so[h][e2] = (p.a_out != nullptr && co < p.Cout)
                          ? p.a_out[static_cast<size_t>(b) * ldc + cb + co] : 1.f;
        }
      if (!wait_bounded(tfull(ab), static_cast<uint32_t>(i >> 1) & 1u, ctl, kErrWaitEpilogue)) break;
      tc_fence_after();
      const uint32_t trow = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * acc_cols;
      const int c8 = m0 + 32 * q + part * 8;
      const bool c_ok = c8 < p.Cout;
      __nv_bfloat16* ybase = p.y + static_cast<size_t>(b) * p.H * p.W * ldc + cb + c8;
      auto process = [&](const uint32_t (&r)[32], int ch) {
        if (p.a_out != nullptr) epi_stage_chunk<true>(r, bb, so, stage, lane);
        else epi_stage_chunk<false>(r, bb, so, stage, lane);
        __syncwarp();
        int pix = ch * 32 + (lane >> 2);
        int rr = pix / p.Wp;
        int cw = pix - rr * p.Wp;
#pragma unroll
        for (int it = 0; it < 4; ++it) {
          const int oh = h0 + rr;
          if (c_ok && pix < p.n_virt && cw < p.W && oh < p.H) {
            const uint4 v = ld_shared_v4(epi_slot(stage, it * 8 + (lane >> 2), part));
            *reinterpret_cast<uint4*>(ybase + (static_cast<size_t>(oh) * p.W + cw) * ldc) = v;
          }
          pix += 8;
          cw += 8;
          while (cw >= p.Wp) { cw -= p.Wp; ++rr; }
        }
        __syncwarp();
      };
      uint32_t ra[32], rb[32];
      int ch = grp;
      if (ch < nchunks) epi_load_chunk(trow, ch * 32, ra);
      while (ch < nchunks) {
        tmem_ld_wait(ra);
        if (ch + 2 < nchunks) epi_load_chunk(trow, (ch + 2) * 32, rb);
        process(ra, ch);
        ch += 2;
        if (ch >= nchunks) break;
        tmem_ld_wait(rb);
        if (ch + 2 < nchunks) epi_load_chunk(trow, (ch + 2) * 32, ra);
        process(rb, ch);
        ch += 2;
      }
      // this warp's reads of the accumulator are complete: release it
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(ab));
    }
  }

  tc_fence_before();
  __syncthreads();
  if (threadIdx.x == 0) {
    tc_stamp(p, 5);  // every unit's epilogue done
    if (p.stamps != nullptr) {
      uint32_t smid;
      asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
      p.stamps[static_cast<size_t>(blockIdx.x) * 8 + 6] = smid;
    }
  }
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, p.tmem_cols);
  }
}

}  // namespace dc
