// Tensor-core kernel mixing: W[b][w] = sum_i alpha[b][i] * E[i][w] for every
// sample b and every weight element w -- n static kernels summed with weights
// that depend on the input (KernelWarehouse,
// abstract), done for all samples at once so that every expert byte is read
// from HBM once per pass instead of once per sample.
//
// As a GEMM: M = samples (128 per tile), N = weight elements (256 per tile),
// K = experts (padded to a multiple of 16).
//  * A = alpha, converted once per CTA into two bf16 operands, alpha_hi =
//    bf16(alpha) and alpha_lo = bf16(alpha - alpha_hi), K-major with the
//    128-byte swizzle; two MMAs per K step (hi and lo) keep ~16 bits of alpha.
//  * B = the experts exactly as they are stored, E[i][w] with w contiguous:
//    an MN-major operand. TMA boxes {64 weights, K experts} land as 128-byte
//    rows per expert with the 128-byte swizzle; 64-weight atoms sit
//    LBO = K*128 bytes apart, 8-expert groups SBO = 1024 bytes apart.
//  * D (fp32) lives in TMEM, double-buffered (2 x 256 columns) so the
//    epilogue of one tile overlaps the MMAs of the next. Eight epilogue warps,
//    two per TMEM lane quarter (32 samples), each taking one 128-column half
//    of the tile, two 32-column TMEM loads in flight: each rounds to bf16,
//    stages its 32 x 128 block in shared memory (XOR-swizzled 16-byte
//    chunks), and writes it back as whole 256-byte row segments (two samples
//    per store instruction). (A second form stores each lane's 64 contiguous
//    bytes straight from registers; measured slower, it stays for
//    measurements.)
// Persistent: one CTA per SM walks the (weight-tile, sample-tile) space,
// either statically (tile c + j * grid for CTA c, every role counting along)
// or taking the next tile from a global counter, so that CTAs whose expert
// reads arrive faster take more tiles; then the producer publishes each
// tile's index in a 16-entry ring in shared memory (tagged with its sequence
// number) for the MMA and epilogue warps, and an end entry closes the
// sequence.
#pragma once

#include "common.cuh"

namespace dc {

constexpr int kPmThreads = 320;   // warp 0 TMA, warp 1 MMA, warps 2..9 epilogue
constexpr int kPmEpiWarps = 8;    // two per TMEM lane quarter, one 128-column half each
constexpr int kPmN = 256;         // weights per tile
constexpr int kPmHalf = kPmN / 2; // columns of one epilogue warp
constexpr int kPmStageBytes = 32 * kPmHalf * 2;  // one warp's 32 samples x 128 bf16
constexpr int kPmMaxStages = 4;   // expert stages in flight (8 measured slower on the deep 3x3 layer)

__host__ __device__ inline int pm_nk(int n) { return (n + 15) / 16 * 16; }
__host__ __device__ inline int pm_kcols(int n) { return (pm_nk(n) + 63) / 64; }

inline bool premix_shape_ok(int B, int n, int Cout, int taps, int Cin) {
  if (n > 256 || B <= 0) return false;
  const long long wsize = 1LL * Cout * taps * Cin;
  if (wsize % 8 != 0) return false;
  const int m_tiles = (B + 127) / 128;
  const long long a_bytes = 2LL * m_tiles * pm_kcols(n) * 16384;
  const long long stage = 1LL * pm_nk(n) * 512;
  const long long alpha_bytes = 4LL * B * n;  // alpha staged in shared memory
  return a_bytes <= 65536 && alpha_bytes <= 16384 &&
         a_bytes + 2 * stage + kPmEpiWarps * kPmStageBytes + alpha_bytes <= 200 * 1024;
}

struct PmParams {
  int B, n, nk, m_tiles, stages;
  long long wsize;       // weight elements per expert
  long long tiles;       // n_tiles * m_tiles
  int a_bytes;           // bytes of all A operands
  int stage_bytes;       // bytes of one expert stage
  int direct_store;      // 1: epilogue stores from registers (wsize % 16 == 0, out 32-byte aligned)
  int stg_bytes;         // one epilogue warp's staging tile: 32 samples x (128 / rep) bf16
  int rep;               // 1, 2 or 4: copies of the batch in the 128 A rows (B <= 128 / rep), each
                         // copy's epilogue warps storing 256 / rep of the tile's columns
  const float* alpha;
  __nv_bfloat16* out;    // [B][wsize]
  int* err;
  long long wait_ns;
  unsigned int* tile_ctr;  // zeroed counter: tiles taken dynamically (null: statically)
};

constexpr int kPmRing = 16;  // tile-index ring entries (more than stages + 3 in flight)

__device__ __forceinline__ uint64_t smem_desc_mn_sw128(uint32_t saddr, uint32_t lbo) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;  // between 64-element MN atoms
  d |= static_cast<uint64_t>(1024u >> 4) << 32;             // between 8-row K groups
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(2u) << 61;
  return d;
}

// REP = p.rep, a template parameter so that the epilogue's column split,
// chunk count and store pattern are compile-time constants (the epilogue is
// the kernel's bound when the expert bank is L2-resident).
template <int REP>
__global__ void __launch_bounds__(kPmThreads, 1)
    premix_kernel(const __grid_constant__ CUtensorMap emap, PmParams p) {
  extern __shared__ __align__(1024) unsigned char pm_smem_raw[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t raw = smem_u32(pm_smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* base_ptr = pm_smem_raw + (base - raw);
  const int S = p.stages;
  const int kcols = (p.nk + 63) / 64;
  const uint32_t a_base = base;                         // [m_tile][hi/lo][kcol][128 rows x 128 B]
  const uint32_t e_base = a_base + p.a_bytes;           // [stage][4 atoms][nk rows x 128 B]
  const uint32_t st_base = e_base + S * p.stage_bytes;  // epilogue staging: 8 warps x 8 KB
  const uint32_t bar_base = st_base + (p.direct_store ? 0u : kPmEpiWarps * p.stg_bytes);
  auto full = [&](int s) { return bar_base + 8u * s; };
  auto empty = [&](int s) { return bar_base + 8u * (S + s); };
  auto tfull = [&](int a) { return bar_base + 8u * (2 * S + a); };
  auto tempty = [&](int a) { return bar_base + 8u * (2 * S + 2 + a); };
  const uint32_t drain_bar = bar_base + 8u * (2 * S + 4);
  unsigned char* misc = base_ptr + (bar_base - base) + 8u * (2 * S + 5);
  volatile uint32_t* tmem_slot = reinterpret_cast<volatile uint32_t*>(misc);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(misc + 4);
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};
  // ring entry of sequence number j: (j << 32) | (tile + 1), 0 in the low half = end
  volatile unsigned long long* ring = reinterpret_cast<volatile unsigned long long*>(
      misc + 16 + ((4 * p.B * p.n + 15) & ~15));

  if (warp == 0) {
    tmem_alloc(smem_u32(const_cast<uint32_t*>(tmem_slot)), 512);
    tmem_relinquish();
  }
  grid_dependency_wait();  // alpha comes from the routing kernel
  // The convolution may be scheduled once every CTA of this grid is past its
  // wait: everything launched before this kernel has then completed, so the
  // convolution may load x (not the mixed kernels) before its own wait.
  grid_launch_dependents();
  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull(a), 1);
      mbar_init(tempty(a), kPmEpiWarps);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    for (int i = 0; i < kPmRing; ++i) ring[i] = ~0ull;  // no sequence number matches
    fence_mbar_init();
    tma_prefetch_desc(&emap);
  }
  // A operands: alpha split into bf16 hi + lo, zero outside [B) x [n).
  // Stage alpha in shared memory first (all loads in flight at once), then
  // build both operands from it.
  float* alpha_s = reinterpret_cast<float*>(misc + 16);
  const int na = p.B * p.n;
  for (int e = threadIdx.x; e < na; e += kPmThreads) alpha_s[e] = p.alpha[e];
  __syncthreads();
  // zero both operands with 16-byte stores, then place the B*n live values
  for (int e = threadIdx.x; e < p.a_bytes / 16; e += kPmThreads)
    st_shared_v4(a_base + e * 16, make_uint4(0u, 0u, 0u, 0u));
  __syncthreads();
  constexpr int spr = 128 / REP;  // A rows per copy of the batch
  for (int e = threadIdx.x; e < na * REP; e += kPmThreads) {
    const int g = e / na, e1 = e - g * na;   // copy, (sample, expert)
    const int m = e1 / p.n, k = e1 - m * p.n;  // sample row, expert
    const int mt = m >> 7, r = (m & 127) + g * spr;
    const float a = alpha_s[e1];
    const __nv_bfloat16 hi = __float2bfloat16_rn(a);
    const __nv_bfloat16 lo = __float2bfloat16_rn(a - __bfloat162float(hi));
    const uint32_t off = static_cast<uint32_t>(k >> 6) * 16384u + r * 128u +
                         ((((k & 63) >> 3) ^ (r & 7)) << 4) + (k & 7) * 2;
    const uint32_t hi_addr = a_base + (mt * 2 + 0) * kcols * 16384u + off;
    const uint32_t lo_addr = a_base + (mt * 2 + 1) * kcols * 16384u + off;
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(hi_addr),
                 "h"(*reinterpret_cast<const unsigned short*>(&hi)) : "memory");
    asm volatile("st.shared.b16 [%0], %1;" ::"r"(lo_addr),
                 "h"(*reinterpret_cast<const unsigned short*>(&lo)) : "memory");
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // Static hand-out: tile j of this CTA is t = blockIdx.x + j * gridDim.x,
  // walked with incremental counters by every role (no END entry needed).
  const bool dyn = p.tile_ctr != nullptr;
  const long long my_tiles =
      p.tiles > blockIdx.x ? (p.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x : 0;
  const long long ntile0 = blockIdx.x / p.m_tiles;
  const int mt0 = blockIdx.x % p.m_tiles;
  const long long dn = gridDim.x / p.m_tiles;
  const int dm = gridDim.x % p.m_tiles;
  // Tile t is (weight tile t / m_tiles, sample tile t % m_tiles). The
  // epilogue finds tile j's ring entry once the producer has written it (before
  // that tile's loads, long before its accumulator is complete): a bounded
  // poll on the entry's sequence tag.
  auto ring_tile = [&](long long j, long long& t) -> bool {
    const unsigned long long want = static_cast<unsigned long long>(j) << 32;
    unsigned long long e = ring[j & (kPmRing - 1)];
    if ((e & ~0xFFFFFFFFull) != want) {
      const uint64_t t0 = globaltimer_ns();
      while (((e = ring[j & (kPmRing - 1)]) & ~0xFFFFFFFFull) != want) {
        if (*abort_flag) return false;
        if (static_cast<long long>(globaltimer_ns() - t0) > p.wait_ns) {
          *abort_flag = 1;
          atomicCAS(p.err, 0, kErrWaitEpilogue);
          return false;
        }
      }
    }
    t = static_cast<long long>(e & 0xFFFFFFFFull) - 1;
    return true;
  };

  if (warp == 0) {
    if (lane == 0) {
      long long issued = 0;
      int s = 0;
      uint32_t ph = 0;
      bool ended = false;
      long long ntile_s = ntile0;
      int mt_s = mt0;
      for (long long j = 0;; ++j) {
        if (!dyn && j >= my_tiles) break;
        if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitProducer)) break;
        long long ntile = ntile_s;
        if (dyn) {
          // a tile is claimed only once a stage is free to load it
          long long t = static_cast<long long>(atomicAdd(p.tile_ctr, 1u));
          if (t >= p.tiles) t = -1;  // end of this CTA's sequence
          ring[j & (kPmRing - 1)] = (static_cast<unsigned long long>(j) << 32) |
                                    static_cast<unsigned long long>(t + 1);
          if (t < 0) {
            mbar_arrive(full(s));  // publishes the end entry
            ended = true;
            break;
          }
          ntile = p.m_tiles == 1 ? t : static_cast<long long>(static_cast<uint32_t>(t) /
                                                            static_cast<uint32_t>(p.m_tiles));
        } else {
          ntile_s += dn;
          mt_s += dm;
          if (mt_s >= p.m_tiles) { mt_s -= p.m_tiles; ++ntile_s; }
        }
        mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(p.stage_bytes));
        const uint32_t dst = e_base + s * p.stage_bytes;
#pragma unroll
        for (int a = 0; a < 4; ++a)
          tma_load_2d(dst + a * p.nk * 128, &emap, full(s),
                      static_cast<int>(ntile * kPmN + a * 64), 0);
        ++issued;
        if (++s == S) { s = 0; ph ^= 1u; }
      }
      // every load in flight lands before the CTA exits; the end entry reused
      // the stage of load issued - S (consumed: its empty barrier had fired),
      // and its arrive moved that barrier one phase on, so that load is not
      // waited for again
      for (long long j = (issued > S ? issued - S : 0) + (ended && issued >= S ? 1 : 0); j < issued;
           ++j)
        wait_drain(full(static_cast<int>(j % S)), static_cast<uint32_t>((j / S) & 1), p.wait_ns,
                   p.err);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, kPmN) | (1u << 16);  // B is MN-major
      const uint32_t lbo = static_cast<uint32_t>(p.nk) * 128u;
      const uint64_t e_desc0 = smem_desc_mn_sw128(e_base, lbo);
      const uint64_t a_desc0 = smem_desc_sw128(a_base);
      const uint64_t a_half = static_cast<uint64_t>(kcols) * (16384 >> 4);  // hi -> lo
      const uint64_t stage = static_cast<uint64_t>(p.stage_bytes) >> 4;
      const int ksteps = p.nk / 16;
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      int mt_s = mt0;
      for (long long j = 0;; ++j) {
        if (!dyn && j >= my_tiles) break;
        const int ab = static_cast<int>(j & 1);
        if (!wait_bounded(full(s), ph, ctl, kErrWaitMma)) { ok = false; break; }
        // (dynamic: the entry was written before the arrive that completed full(s))
        const unsigned long long e = dyn ? ring[j & (kPmRing - 1)] : 1ull;
        if (!wait_bounded(tempty(ab), static_cast<uint32_t>((j >> 1) & 1) ^ 1u, ctl, kErrWaitMma)) { ok = false; break; }
        if ((e & 0xFFFFFFFFull) == 0) {
          mbar_arrive(tfull(ab));  // end: the epilogue reads the end entry
          break;
        }
        int mt = mt_s;
        if (dyn) {
          const uint32_t tt = static_cast<uint32_t>(e) - 1u;  // 32-bit tile index (tiles < 2^31)
          mt = p.m_tiles == 1 ? 0 : static_cast<int>(tt % static_cast<uint32_t>(p.m_tiles));
        } else {
          mt_s += dm;
          if (mt_s >= p.m_tiles) mt_s -= p.m_tiles;
        }
        tc_fence_after();
        const uint64_t bd = e_desc0 + s * stage;
        const uint64_t ad = a_desc0 + static_cast<uint64_t>(mt) * 2 * a_half;
        const uint32_t d = tmem_base + ab * kPmN;
        for (int kk = 0; kk < ksteps; ++kk) {
          // K step kk: 16 expert rows = +2048 bytes of B; A advances 32 bytes within a
          // 64-wide column, then jumps to the next 16 KB column
          const uint64_t aoff = static_cast<uint64_t>(kk >> 2) * (16384 >> 4) + (kk & 3) * 2;
          tc_mma_f16(d, ad + aoff, bd + kk * (2048 >> 4), idesc, kk > 0 ? 1u : 0u);
          tc_mma_f16(d, ad + a_half + aoff, bd + kk * (2048 >> 4), idesc, 1u);
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
  } else if (warp < 2 + kPmEpiWarps) {
    // Epilogue: warp w reads TMEM lanes 32*(w%4) .. +31 (= 32 samples of the
    // tile) and the columns of its half, 32 at a time with the next load in
    // flight.
    const int q = warp & 3;
    const int half = (warp - 2) >> 2;
    const uint32_t stg = st_base + (warp - 2) * p.stg_bytes;
    long long ntile_s = ntile0;
    int mt_s = mt0;
    for (long long j = 0;; ++j) {
      if (!dyn && j >= my_tiles) break;
      const int ab = static_cast<int>(j & 1);
      if (!wait_bounded(tfull(ab), static_cast<uint32_t>((j >> 1) & 1), ctl, kErrWaitEpilogue)) break;
      long long ntile = ntile_s;
      int mt = mt_s;
      if (dyn) {
        long long t;
        if (!ring_tile(j, t) || t < 0) break;
        const uint32_t tt = static_cast<uint32_t>(t);
        ntile = p.m_tiles == 1 ? static_cast<long long>(tt)
                               : static_cast<long long>(tt / static_cast<uint32_t>(p.m_tiles));
        mt = static_cast<int>(tt - static_cast<uint32_t>(ntile) * static_cast<uint32_t>(p.m_tiles));
      } else {
        ntile_s += dn;
        mt_s += dm;
        if (mt_s >= p.m_tiles) { mt_s -= p.m_tiles; ++ntile_s; }
      }
      tc_fence_after();
      // TMEM lanes 32q .. 32q+31 hold samples row0 .. row0+31 of copy g; copy
      // g's warps store columns [g, g+1) * 256 / rep of the tile, this half
      // of them (cw columns). A warp whose samples are all past the batch
      // only releases the buffer.
      const int g = (32 * q) / spr;
      const int row0 = mt * 128 + 32 * q - g * spr;
      constexpr int cw = kPmHalf / REP;
      const int col0 = g * (kPmN / REP) + half * cw;
      const bool live = row0 < p.B;
      const long long w0 = ntile * kPmN + (REP == 1 ? half * kPmHalf : col0);
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(32 * q) << 16) + ab * kPmN +
                             (REP == 1 ? half * kPmHalf : col0);
      if (live) {
        uint32_t ra[32], rb[32];
        if (p.direct_store) {
          // each lane (one sample) writes 64 contiguous bytes per chunk as two
          // 32-byte stores straight from registers
          const int b = row0 + lane;
          __nv_bfloat16* dst = p.out + static_cast<size_t>(b < p.B ? b : 0) * p.wsize + w0;
          auto emit = [&](const uint32_t (&r)[32], int ch) {
            uint32_t o[16];
#pragma unroll
            for (int v = 0; v < 16; ++v)
              o[v] = pack_bf16x2(__uint_as_float(r[2 * v]), __uint_as_float(r[2 * v + 1]));
#pragma unroll
            for (int h = 0; h < 2; ++h)
              if (b < p.B && w0 + ch * 32 + h * 16 < p.wsize)
                st_global_v8(dst + ch * 32 + h * 16, o + 8 * h);
          };
          tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll 1
          for (int ch = 0; ch < kPmHalf / 32; ch += 2) {
            tmem_ld_wait(ra);
            tmem_ld_32x32b_x32(taddr + (ch + 1) * 32, rb);
            emit(ra, ch);
            tmem_ld_wait(rb);
            if (ch + 2 < kPmHalf / 32) tmem_ld_32x32b_x32(taddr + (ch + 2) * 32, ra);
            emit(rb, ch + 1);
          }
        } else {
          // staged: row `lane` of the 32 x (2 cw)-byte block, 16-byte chunk c
          // at position c ^ (lane % (cw / 8)): 32 lanes fill the bank groups evenly
          constexpr int cpr = cw / 8;  // 16-byte chunks per row
          auto stage_chunk = [&](const uint32_t (&r)[32], int ch) {
#pragma unroll
            for (int v = 0; v < 4; ++v) {
              uint4 o;
              o.x = pack_bf16x2(__uint_as_float(r[8 * v + 0]), __uint_as_float(r[8 * v + 1]));
              o.y = pack_bf16x2(__uint_as_float(r[8 * v + 2]), __uint_as_float(r[8 * v + 3]));
              o.z = pack_bf16x2(__uint_as_float(r[8 * v + 4]), __uint_as_float(r[8 * v + 5]));
              o.w = pack_bf16x2(__uint_as_float(r[8 * v + 6]), __uint_as_float(r[8 * v + 7]));
              const int c = ch * 4 + v;  // 16-byte chunk of this sample's segment
              st_shared_v4(stg + lane * (2 * cw) + ((c ^ (lane & (cpr - 1))) << 4), o);
            }
          };
          constexpr int nch = cw / 32;
          tmem_ld_32x32b_x32(taddr, ra);
#pragma unroll 1
          for (int ch = 0; ch < nch; ch += 2) {
            tmem_ld_wait(ra);
            if (ch + 1 < nch) tmem_ld_32x32b_x32(taddr + (ch + 1) * 32, rb);
            stage_chunk(ra, ch);
            if (ch + 1 >= nch) break;
            tmem_ld_wait(rb);
            if (ch + 2 < nch) tmem_ld_32x32b_x32(taddr + (ch + 2) * 32, ra);
            stage_chunk(rb, ch + 1);
          }
        }
      }
      // the TMEM buffer is free once every lane's loads completed
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty(ab));
      if (live && !p.direct_store) {
        // 32 / cpr samples per store instruction, cpr lanes of 16 bytes each
        // covering one sample's 2 cw-byte segment (cw = 128: lanes 0..15 row
        // sr, 16..31 row sr + 1)
        constexpr int cpr = cw / 8;
        const int part = lane & (cpr - 1);
        constexpr int rstep = 32 / cpr;
        const long long w = w0 + part * 8;
        const bool wok = w < p.wsize;
        const int nrows = min(32, p.B - row0);
#pragma unroll 4
        for (int sr = lane / cpr; sr < 32; sr += rstep) {
          uint4 v;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                       : "r"(stg + sr * (2 * cw) + ((part ^ (sr & (cpr - 1))) << 4)));
          if (wok && sr < nrows)
            *reinterpret_cast<uint4*>(p.out + static_cast<size_t>(row0 + sr) * p.wsize + w) = v;
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// The kernel instantiation for a plan's copy count (PmParams::rep).
inline void (*premix_kernel_for(int rep))(const CUtensorMap, PmParams) {
  return rep == 4 ? premix_kernel<4> : rep == 2 ? premix_kernel<2> : premix_kernel<1>;
}

// Host-side plan of one premix launch.
struct PremixLaunch {
  PmParams p;
  CUtensorMap emap;
  unsigned grid = 0;
  size_t smem = 0;
};

// Fills `out`. Returns 0, -2 (tensor map), -3 (shape).
template <typename EncodeFn>
inline int plan_premix(const __nv_bfloat16* experts, const float* alpha, __nv_bfloat16* out_ws,
                       int B, int n, long long wsize, int* err, long long wait_ns, int sms,
                       EncodeFn encode, PremixLaunch* out, long long estride = 0,
                       bool allow_direct = true, unsigned int* tile_ctr = nullptr) {
  // estride: elements from one expert to the next (default wsize); a larger
  // stride mixes a contiguous slice of wsize elements of every expert
  PmParams& p = out->p;
  p = PmParams{};
  p.B = B;
  p.n = n;
  p.nk = pm_nk(n);
  p.m_tiles = (B + 127) / 128;
  p.wsize = wsize;
  const long long n_tiles = (wsize + kPmN - 1) / kPmN;
  p.tiles = n_tiles * p.m_tiles;
  p.a_bytes = 2 * p.m_tiles * pm_kcols(n) * 16384;
  p.stage_bytes = p.nk * 512;
  p.direct_store =
      (allow_direct && wsize % 16 == 0 && (reinterpret_cast<uintptr_t>(out_ws) & 31u) == 0) ? 1 : 0;
  // small batches: copies of the batch fill the 128 accumulator rows, so that
  // every epilogue warp has samples to store (each copy a share of the columns)
  p.rep = (p.direct_store || p.m_tiles != 1) ? 1 : B <= 32 ? 4 : B <= 64 ? 2 : 1;
  p.stg_bytes = kPmStageBytes / p.rep;
  const int staging = p.direct_store ? 0 : kPmEpiWarps * p.stg_bytes;
  const int budget = 200 * 1024 - p.a_bytes - staging - 4 * B * n - 16 - 8 * kPmRing;
  p.stages = std::min(kPmMaxStages, budget / p.stage_bytes);
  if (p.stages < 2 || p.tiles >= (1LL << 31)) return -3;
  p.alpha = alpha;
  p.out = out_ws;
  p.err = err;
  p.wait_ns = wait_ns;
  p.tile_ctr = tile_ctr;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(wsize), static_cast<cuuint64_t>(n)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(estride > 0 ? estride : wsize) * 2};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(p.nk)};
  const cuuint32_t es[2] = {1u, 1u};
  if (encode(&out->emap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16*>(experts),
             dims, strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return -2;
  // at least 120 KB so that two CTAs never share an SM (each holds all 512 TMEM columns)
  out->smem = std::max<size_t>(120 * 1024, 1024 + static_cast<size_t>(p.a_bytes) +
                                               static_cast<size_t>(p.stages) * p.stage_bytes +
                                               staging + 8 * (2 * p.stages + 5) + 16 +
                                               ((4 * static_cast<size_t>(B) * n + 15) & ~15) +
                                               8 * kPmRing);
  out->grid = static_cast<unsigned>(std::min<long long>(p.tiles, sms));
  return 0;
}

}  // namespace dc
