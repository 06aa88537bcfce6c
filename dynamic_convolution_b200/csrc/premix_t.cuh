// Tensor-core kernel mixing for a few samples (the groups of the grouped
// PREMIX pipeline, and any batch of at most 256):
//     W[s][w] = sum_i alpha[s][i] * E[i][w]
// -- per-example kernels that are weighted sums of n static kernels
// (KernelWarehouse, abstract; CondConv, abstract) -- as the GEMM
//     D[w][s] = sum_i E[i][w] * alpha[s][i],   M = 128 weights, N = samples, K = experts,
// i.e. transposed with respect to premix_kernel (M = samples there). With
// few samples that orientation leaves most of the 128 accumulator rows empty
// and one epilogue warp in four storing; here every TMEM lane is a weight,
// all four epilogue warps work, and one tcgen05.ld brings 32 samples.
//  * A = the experts as stored (E[i][w], w contiguous): an MN-major operand,
//    two TMA boxes {64 weights, K experts} per tile in the 128-byte swizzle.
//  * B = alpha, split into bf16 hi + lo (two MMAs per K step, ~16 bits of
//    alpha), K-major, built once per CTA.
//  * D (fp32) in TMEM, up to 8 accumulators of N columns: the MMAs run up to
//    8 tiles ahead of the epilogue, so the latency of one tile's MMA
//    completion and TMEM read overlaps the others'.
//  * Epilogue, 8 warps (two per TMEM lane quarter, alternate 16-sample
//    column groups): lane = weight w, 16 samples per load; neighbouring lanes
//    swap one value (shuffle) so that each lane stores two adjacent weights
//    of one sample (even lanes sample s, odd lanes sample s+1): every store
//    instruction writes two 64-byte runs.
// Persistent: one CTA per SM walks the 128-weight tiles.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kPtThreads = 320;  // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kPtEpiWarps = 8;
constexpr int kPtMaxAcc = 8;     // TMEM accumulators (tiles in flight between MMA and epilogue)
constexpr int kPtM = 128;        // weights per tile

struct PtParams {
  int S, n, nk;          // samples (<= 256), experts, experts padded to 16
  int npad;              // samples padded to 32 (MMA N)
  int nacc;              // TMEM accumulators of npad columns (<= kPtMaxAcc, nacc * npad <= 512)
  int stages;
  long long wsize;       // weights to mix per sample (this launch's slice)
  long long tiles;       // ceil(wsize / 128)
  int a_bytes;           // one expert stage: 2 atoms x nk rows x 128 B
  int b_bytes;           // alpha operand, one of hi / lo: kcols x npad x 128 B
  const float* alpha;    // [S][n]
  __nv_bfloat16* out;    // [S][wsize]
  int* err;
  long long wait_ns;
};

__global__ void __launch_bounds__(kPtThreads, 1)
    premix_t_kernel(const __grid_constant__ CUtensorMap emap, PtParams p) {
  extern __shared__ __align__(1024) unsigned char pt_smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(pt_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = pt_smem_raw + (base - raw);
  const int S = p.stages;
  const uint32_t b_base = base;                          // [hi/lo][kcol][npad rows x 128 B]
  const uint32_t e_base = b_base + 2 * p.b_bytes;        // [stage][2 atoms][nk rows x 128 B]
  const uint32_t bar_base = e_base + S * p.a_bytes;
  auto full = [&](int s) { return bar_base + 8u * s; };
  auto empty = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * S + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * S + kPtMaxAcc + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * S + 2 * kPtMaxAcc);
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * S + 2 * kPtMaxAcc + 1);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};
  uint32_t tcols = 32;
  while (tcols < static_cast<uint32_t>(p.nacc * p.npad)) tcols <<= 1;
  const int NA = p.nacc;

  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), tcols);
    tmem_relinquish();
  }
  grid_dependency_wait();  // alpha comes from the routing kernel
  grid_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < NA; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), kPtEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&emap);
  }
  // B operands: alpha hi / lo, K-major in the 128-byte swizzle (row = sample,
  // 64 experts per 128-byte row, 8-row groups 1024 bytes apart), zero outside
  // [S) x [n)
  for (int e = threadIdx.x; e < 2 * p.b_bytes / 16; e += kPtThreads)
    st_shared_v4(b_base + e * 16, make_uint4(0u, 0u, 0u, 0u));
  __syncthreads();
  for (int e = threadIdx.x; e < p.S * p.n; e += kPtThreads) {
    const int r = e / p.n, k = e - r * p.n;  // sample row, expert
    const float a = p.alpha[e];
    const __nv_bfloat16 hi = __float2bfloat16_rn(a);
    const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
    const uint32_t off = static_cast<uint32_t>(k >> 6) * p.npad * 128u + r * 128u +
                         ((((k & 63) >> 3) ^ (r & 7)) << 4) + (k & 7) * 2;
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(b_base + off),
                 "h"(*reinterpret_cast<const unsigned short*>(&hi)) : "memory");
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(b_base + p.b_bytes + off),
                 "h"(*reinterpret_cast<const unsigned short*>(&lo)) : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const long long my_tiles =
      p.tiles > blockIdx.x ? (p.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;

  if (warp == 0) {
    if (lane == 0) {
      long long issued = 0;
      int s = 0;
      uint32_t ph = 0;
      for (long long j = 0; j < my_tiles; ++j) {
        const long long t = blockIdx.x + j * gridDim.x;
        if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
        mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(p.a_bytes));
        const uint32_t dst = e_base + s * p.a_bytes;
        tma_load_2d(dst, &emap, full(s), static_cast<int>(t * kPtM), 0);
        tma_load_2d(dst + p.nk * 128, &emap, full(s), static_cast<int>(t * kPtM + 64), 0);
        ++issued;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      for (long long j = (issued > S ? issued - S : 0); j < issued; ++j)
        wait_drain(full(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1), p.wait_ns,
                   p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // A (experts) MN-major, B (alpha) K-major
      const uint32_t idesc = idesc_bf16_f32(kPtM, p.npad) | (1u << 15);
      const uint64_t a_desc0 = smem_desc_mn_sw128(e_base, static_cast<uint32_t>(p.nk) * 128u);
      const uint64_t b_desc0 = smem_desc_sw128(b_base);
      const uint64_t b_half = static_cast<uint64_t>(p.b_bytes) >> 4;  // hi -> lo
      const uint64_t b_kcol = static_cast<uint64_t>(p.npad) * (128 >> 4);
      const uint64_t stage = static_cast<uint64_t>(p.a_bytes) >> 4;
      const int ksteps = p.nk / 16;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long long j = 0; j < my_tiles; ++j) {
        const int ab = static_cast<int>(j % NA);
        const uint32_t aph = static_cast<uint32_t>((j / NA) & 1);
        if (!wait_bounded(full(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
        if (!wait_bounded(tempty(ab), aph ^ 1u, ctl, kErrWaitMma)) { ok = false; break; }
        tc_fence_after();
        const uint64_t ad = a_desc0 + s * stage;
        const uint32_t d = tmem_base + ab * p.npad;
        for (int kk = 0; kk < ksteps; ++kk) {
          // K step kk: 16 expert rows of A = +2048 bytes; 16 experts of B =
          // +32 bytes within a 64-wide column, then the next column
          const uint64_t boff = static_cast<uint64_t>(kk >> 2) * b_kcol + (kk & 3) * 2;
          tc_mma_f16(d, ad + kk * (2048 >> 4), b_desc0 + boff, idesc, kk > 0 ? 1u : 0u);
          tc_mma_f16(d, ad + kk * (2048 >> 4), b_desc0 + b_half + boff, idesc, 1u);
        }
        tc_commit(empty(s));
        tc_commit(tfull(ab));
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      if (!ok) {
        tc_commit(drain_bar);
        wait_drain(drain_bar, 0, p.wait_ns, p.err);
      }
    }
  } else if (warp < 2 + kPtEpiWarps) {
    // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 = weights of the tile;
    // the two warps of a lane quarter take alternate 16-sample column groups
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const int ngroups = (p.S + 15) / 16;
    const bool odd = lane & 1;
    for (long long j = 0; j < my_tiles; ++j) {
      const long long t = blockIdx.x + j * gridDim.x;
      const int ab = static_cast<int>(j % NA);
      if (!wait_bounded(tfull(ab), static_cast<uint32_t>((j / NA) & 1), ctl, kErrWaitEpilogue)) break;
      tc_fence_after();
      const long long w = t * kPtM + 32 * q + lane;    // this lane's weight
      const long long wp = w & ~1LL;                   // the pair a lane stores
      const bool wok = wp < p.wsize;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * p.npad;
      for (int g = half; g < ngroups; g += 2) {
        uint32_t r[16];
        tmem_ld_32x32b_x16(taddr + g * 16, r);
        tmem_ld_wait16(r);
#pragma unroll
        for (int v = 0; v < 16; v += 2) {
          // even lanes keep sample v, odd lanes sample v+1; each sends the
          // other sample's value to its neighbour
          const float mine_v = __uint_as_float(r[v]), mine_v1 = __uint_as_float(r[v + 1]);
          const float other = __shfl_xor_sync(0xffffffffu, odd ? mine_v : mine_v1, 1);
          const int sidx = g * 16 + v + (odd ? 1 : 0);
          const uint32_t packed = odd ? pack_bf16x2(other, mine_v1) : pack_bf16x2(mine_v, other);
          if (wok && sidx < p.S)
            *reinterpret_cast<uint32_t*>(p.out + static_cast<size_t>(sidx) * p.wsize + wp) = packed;
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
    tmem_dealloc(tmem_base, tcols);
  }
}

// Host-side plan of one premix_t launch: 0, -2 (tensor map), -3 (shape).
// `estride`: elements from one expert to the next.
struct PremixTLaunch {
  PtParams p;
  CUtensorMap emap;
  unsigned grid = 0;
  size_t smem = 0;
};

template <typename EncodeFn>
inline int plan_premix_t(const __nv_bfloat16* experts, long long estride, const float* alpha,
                         __nv_bfloat16* out, int S, int n, long long wsize, int* err,
                         long long wait_ns, int ctas, EncodeFn encode, PremixTLaunch* out_l) {
  if (S < 1 || S > 256 || n < 1 || n > 256 || wsize % 2 != 0 || wsize < 1) return -3;
  PtParams& p = out_l->p;
  p = PtParams{};
  p.S = S;
  p.n = n;
  p.nk = (n + 15) / 16 * 16;
  p.npad = (S + 31) / 32 * 32;  // whole 32-column loads stay inside one accumulator
  p.wsize = wsize;
  p.tiles = (wsize + kPtM - 1) / kPtM;
  p.a_bytes = 2 * p.nk * 128;
  p.b_bytes = ((p.nk + 63) / 64) * p.npad * 128;
  p.nacc = std::max(2, std::min(kPtMaxAcc, 512 / p.npad));
  const int budget = 200 * 1024 - 2 * p.b_bytes;
  p.stages = std::min(6, budget / p.a_bytes);
  if (p.stages < 2) return -3;
  p.alpha = alpha;
  p.out = out;
  p.err = err;
  p.wait_ns = wait_ns;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(wsize), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(estride) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(p.nk)};
  const cuuint32_t es[2] = {1u, 1u};
  if (encode(&out_l->emap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(experts),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return -2;
  // at least 120 KB, so that two CTAs never share an SM's TMEM
  out_l->smem = std::max<size_t>(120 * 1024, 1024 + 2 * static_cast<size_t>(p.b_bytes) +
                                                 static_cast<size_t>(p.stages) * p.a_bytes +
                                                 8 * (2 * p.stages + 2 * kPtMaxAcc + 1) + 16);
  out_l->grid = static_cast<unsigned>(std::min<long long>(p.tiles, ctas));
  return 0;
}

}  // namespace dc
