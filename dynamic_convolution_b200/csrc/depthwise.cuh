// CUDA-core depthwise dynamic convolution (groups == C_in == C_out), bf16 in /
// out, fp32 mixing and accumulation, stride 1, square K in {3, 5, 7}.
//
// y_b[c] = sum_{kh,kw} x_b[oh+kh-p, ow+kw-p, c] * W_b[c,kh,kw] + b_b[c] with
// W_b = sum_i alpha_{b,i} W_i (the linear kernel mixture of KernelWarehouse,
// abstract; per-example kernels of CondConv, abstract).
//
// The layer is memory-bound with an FMA floor close to the HBM floor, so the
// kernel touches each input byte once from HBM and keeps the FMA pipe fed:
//  * one CTA per (sample, 32-channel chunk, block of up to kDwMaxRows output
//    rows, block of output columns); the zero-padded input window is staged
//    in shared memory by ONE 4-D TMA box {32 channels, cols+K-1, rows+K-1, 1}
//    whose out-of-bounds fill is the zero padding;
//  * while the box is in flight the CTA mixes its 32 channels' K*K weights
//    and biases (fp32), with every expert load of a thread issued at once;
//  * each thread owns one channel pair (bf16x2) and two adjacent output
//    columns, keeps its 2*K*K weights in registers and walks down the output
//    rows with a circular K-row window over K+1 input columns (K+1 new values
//    per row for two outputs, six independent accumulation chains visited
//    in rotation, so the packed-FMA latency never stalls a warp);
//  * the channel pair is computed with the packed fp32 instructions of sm_100
//    (fma.rn.f32x2: two independent fp32 FMAs, each rounded as a scalar FMA),
//    which halves the instruction count of this issue-bound loop.
//  * consecutive threads take consecutive channel pairs: shared-memory reads
//    are conflict-free and the NHWC stores coalesce.
#pragma once

#include <type_traits>

#include "common.cuh"

namespace dc {

constexpr int kDwChunk = 32;       // channels per CTA
constexpr int kDwPairs = kDwChunk / 2;
constexpr int kDwMaxRows = 28;     // output rows per CTA (at most)
constexpr int kDwColsPerThread = 2;
constexpr int kDwMaxColThreads = 16;  // column threads per CTA -> up to 32 output columns
constexpr int kDwThreads = kDwPairs * kDwMaxColThreads;

struct DwParams {
  int B, C, H, W, pad, n, Ho, Wo;
  int rows;                        // output rows per CTA
  int cols;                        // output columns per CTA (<= kDwColsPerThread * kDwMaxColThreads)
  int col_threads;                 // ceil(cols / kDwColsPerThread)
  const __nv_bfloat16* experts;    // [n][C][K][K][1]
  const float* alpha;
  const float* bias;               // may be null
  __nv_bfloat16* y;
  int* err;
  long long wait_ns;
  const float* a_in;               // [B][C] input channel attention, or null
  const float* a_out;              // [B][C] output channel attention, or null
  const float* chan_add;           // [B][C] or null: chan_scale * chan_add joins the mixed bias
  float chan_scale;
};

template <int K>
__global__ void __launch_bounds__(kDwThreads, K <= 5 ? 2 : 1)
    depthwise_kernel(const __grid_constant__ CUtensorMap xmap, DwParams p) {
  constexpr int KK = K * K;
  const int TC = ((p.cols + 1) & ~1) + K - 1;      // staged input columns (even column count + halo)
  const int TR = p.rows + K - 1;                  // staged input rows
  const int b = blockIdx.z;
  const int c0 = blockIdx.y * kDwChunk;
  const int nrow_blocks = (p.Ho + p.rows - 1) / p.rows;
  const int oh0 = (blockIdx.x % nrow_blocks) * p.rows;
  const int ow0 = (blockIdx.x / nrow_blocks) * p.cols;
  const int t = threadIdx.x;

  extern __shared__ __align__(128) unsigned char dw_smem_raw[];
  // tile first (TMA destination, 128-byte aligned), then the small arrays
  unsigned char* dw_smem = dw_smem_raw + ((128u - (smem_u32(dw_smem_raw) & 127u)) & 127u);
  uint32_t* tile = reinterpret_cast<uint32_t*>(dw_smem);                // [TR][TC][kDwPairs]
  const size_t tile_bytes = static_cast<size_t>(TR) * TC * kDwChunk * 2;
  float* w_s = reinterpret_cast<float*>(dw_smem + ((tile_bytes + 127) & ~size_t(127)));  // [32][KK]
  float* bias_s = w_s + kDwChunk * KK;                                  // [32]
  float* alpha_s = bias_s + kDwChunk;                                   // [n]
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const uint32_t bar_a = smem_u32(&bar);
  const WaitCtl ctl{const_cast<volatile int*>(&abort_flag), p.err, p.wait_ns};

  grid_dependency_wait();  // alpha (and possibly x) come from earlier kernels
  // the next kernel on the stream (a routing kernel of the next layer) may
  // be scheduled while this one runs: it waits for this grid's completion
  // before it reads anything this grid writes
  grid_launch_dependents();
  if (t == 0) {
    abort_flag = 0;
    mbar_init(bar_a, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(bar_a, static_cast<uint32_t>(tile_bytes));
    tma_load_4d(smem_u32(tile), &xmap, bar_a, c0, ow0 - p.pad, oh0 - p.pad, b);
  }
  for (int i = t; i < p.n; i += kDwThreads) alpha_s[i] = p.alpha[static_cast<size_t>(b) * p.n + i];
  __syncthreads();

  // mix this chunk's kernels and biases (fp32). The loads are the latency
  // chain of the prologue, so each thread issues the expert values of up to
  // four weight elements (x 8 experts) before it adds any of them.
  {
    constexpr int kE = 4;
    const size_t es = static_cast<size_t>(p.C) * KK;
    for (int e0 = t; e0 < kDwChunk * KK; e0 += kE * kDwThreads) {
      float s[kE];
      const __nv_bfloat16* src[kE];
      bool live[kE];
#pragma unroll
      for (int u = 0; u < kE; ++u) {
        const int e = e0 + u * kDwThreads;
        const int cl = e / KK, k = e - cl * KK;
        live[u] = e < kDwChunk * KK && c0 + cl < p.C;
        src[u] = p.experts + static_cast<size_t>(live[u] ? c0 + cl : 0) * KK + (live[u] ? k : 0);
        s[u] = 0.f;
      }
      for (int i = 0; i < p.n; i += 8) {
        __nv_bfloat16 v[kE][8];
#pragma unroll
        for (int u = 0; u < kE; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            v[u][q] = (live[u] && i + q < p.n) ? src[u][(i + q) * es] : __float2bfloat16_rn(0.f);
#pragma unroll
        for (int u = 0; u < kE; ++u)
#pragma unroll
          for (int q = 0; q < 8; ++q)
            if (i + q < p.n) s[u] = fmaf(alpha_s[i + q], __bfloat162float(v[u][q]), s[u]);
      }
#pragma unroll
      for (int u = 0; u < kE; ++u)
        if (e0 + u * kDwThreads < kDwChunk * KK) w_s[e0 + u * kDwThreads] = s[u];
    }
  }
  if (t < kDwChunk) {
    const int c = c0 + t;
    float s = 0.f;
    if (p.bias && c < p.C) {
      for (int i = 0; i < p.n; i += 8) {
        float v[8];
#pragma unroll
        for (int q = 0; q < 8; ++q) v[q] = i + q < p.n ? p.bias[static_cast<size_t>(i + q) * p.C + c] : 0.f;
#pragma unroll
        for (int q = 0; q < 8; ++q) if (i + q < p.n) s = fmaf(alpha_s[i + q], v[q], s);
      }
    }
    if (p.chan_add && c < p.C) s = fmaf(p.chan_add[static_cast<size_t>(b) * p.C + c], p.chan_scale, s);
    bias_s[t] = s;
  }
  __syncthreads();
  const bool tile_ok = wait_bounded(bar_a, 0, ctl, kErrWaitEpilogue);

  const int cp = t % kDwPairs;     // channel pair within the chunk
  const int ct = t / kDwPairs;     // column-pair thread
  const int c = c0 + 2 * cp;
  if (!tile_ok || ct >= p.col_threads || c >= p.C) return;

  // weights of the channel pair, packed (lo = channel c, hi = channel c+1);
  // input attention scales the channel's kernel (depthwise: one input channel)
  const float ai0 = p.a_in ? p.a_in[static_cast<size_t>(b) * p.C + c] : 1.f;
  const float ai1 = p.a_in ? p.a_in[static_cast<size_t>(b) * p.C + c + 1] : 1.f;
  uint64_t w2[KK];
#pragma unroll
  for (int k = 0; k < KK; ++k)
    w2[k] = pack_f32x2(w_s[(2 * cp) * KK + k] * ai0, w_s[(2 * cp + 1) * KK + k] * ai1);
  const uint64_t bias2 = pack_f32x2(bias_s[2 * cp], bias_s[2 * cp + 1]);
  // output attention: y = a_out * (conv + mixed bias)
  const float ao0 = p.a_out ? p.a_out[static_cast<size_t>(b) * p.C + c] : 1.f;
  const float ao1 = p.a_out ? p.a_out[static_cast<size_t>(b) * p.C + c + 1] : 1.f;
  __nv_bfloat16* yb = p.y + static_cast<size_t>(b) * p.Ho * p.Wo * p.C;

  // this thread's two adjacent output columns
  const int col = 2 * ct;
  const int ow = ow0 + col;
  const uint32_t* tcol = tile + static_cast<size_t>(col) * kDwPairs + cp;
  const size_t row_stride = static_cast<size_t>(TC) * kDwPairs;
  // circular K-row window over the K+1 input columns col .. col+K: input row r
  // lives in slot r % K. Rows are walked in groups of K with the group body
  // unrolled, so every slot index is a compile-time constant and the window
  // never moves between registers.
  uint64_t win[K][K + 1];
#pragma unroll
  for (int r = 0; r < K - 1; ++r)
#pragma unroll
    for (int kw = 0; kw <= K; ++kw) win[r][kw] = bf16x2_to_f32x2(tcol[r * row_stride + kw * kDwPairs]);
#pragma unroll 1
  for (int g = 0; g < p.rows; g += K) {
#pragma unroll
    for (int j = 0; j < K; ++j) {
      const int orow = g + j;
      if (orow >= p.rows) break;
      const int in_row = orow + K - 1;
#pragma unroll
      for (int kw = 0; kw <= K; ++kw)
        win[(j + K - 1) % K][kw] = bf16x2_to_f32x2(tcol[in_row * row_stride + kw * kDwPairs]);
      // six independent chains (kernel row mod 3, two columns), visited in
      // rotation so that consecutive FMAs never depend on each other
      uint64_t acc[3][2] = {{bias2, bias2}, {0ull, 0ull}, {0ull, 0ull}};
#pragma unroll
      for (int kw = 0; kw < K; ++kw)
#pragma unroll
        for (int kh = 0; kh < K; ++kh) {
          const uint64_t w = w2[kh * K + kw];
          acc[kh % 3][0] = ffma2(win[(j + kh) % K][kw], w, acc[kh % 3][0]);
          acc[kh % 3][1] = ffma2(win[(j + kh) % K][kw + 1], w, acc[kh % 3][1]);
        }
      uint64_t s0 = fadd2(fadd2(acc[0][0], acc[1][0]), acc[2][0]);
      uint64_t s1 = fadd2(fadd2(acc[0][1], acc[1][1]), acc[2][1]);
      if (p.a_out) {
        s0 = pack_f32x2(__uint_as_float(static_cast<uint32_t>(s0)) * ao0,
                        __uint_as_float(static_cast<uint32_t>(s0 >> 32)) * ao1);
        s1 = pack_f32x2(__uint_as_float(static_cast<uint32_t>(s1)) * ao0,
                        __uint_as_float(static_cast<uint32_t>(s1 >> 32)) * ao1);
      }
      const int oh = oh0 + orow;
      if (oh < p.Ho) {
        __nv_bfloat16* dst = yb + (static_cast<size_t>(oh) * p.Wo + ow) * p.C + c;
        if (col < p.cols && ow < p.Wo)
          *reinterpret_cast<uint32_t*>(dst) = pack_bf16x2(__uint_as_float(static_cast<uint32_t>(s0)),
                                                          __uint_as_float(static_cast<uint32_t>(s0 >> 32)));
        if (col + 1 < p.cols && ow + 1 < p.Wo)
          *reinterpret_cast<uint32_t*>(dst + p.C) =
              pack_bf16x2(__uint_as_float(static_cast<uint32_t>(s1)),
                          __uint_as_float(static_cast<uint32_t>(s1 >> 32)));
      }
    }
  }
}

}  // namespace dc

namespace dc {

// ---------------------------------------------------------------------------
// Pipelined depthwise kernel (the default when the expert slab fits).
//
// The same layer arithmetic as depthwise_kernel above, organised so that HBM
// and the FMA pipe stay busy together:
//  * persistent CTAs, one per SM; CTA i owns the channel chunk i % nchunks for
//    its whole life and walks the tiles (sample, row band, column band) of that
//    chunk with stride = the number of CTAs sharing the chunk;
//  * the chunk's expert slabs [n][CC][K*K] (and bias slabs) are copied into
//    shared memory once per CTA by bulk copies and stay resident;
//  * a producer warp keeps S tiles in flight: per tile one 4-D TMA box of the
//    zero-padded input window {CC channels, CB+K-1 columns, RB+K-1 rows}, plus
//    the sample's attentions (and channel factors) stored by its lanes;
//  * the compute warps first mix the tile's kernels together (CC*K*K weights,
//    CC biases, fp32, from the resident slabs) into the stage, then each thread
//    takes NC (2 or 4) adjacent output columns of ONE channel pair and walks
//    the input rows of the band: for every input row it loads K+NC-1 packed
//    pairs and adds them into the K output rows (x NC columns) that use that
//    input row (vertical accumulators, packed fp32x2 FMAs: NC*K*K per row for
//    K+NC-1 loads);
//    an output row is stored when its last input row is in. The rows are
//    walked in groups of K with every accumulator slot a compile-time
//    register; only the first and the last groups carry the band-edge tests.
//    Consecutive threads take consecutive channel pairs of one column pair,
//    so with 32 or 64 pairs per chunk a warp's loads are conflict-free.
// Every wait is bounded (mbarriers only, no named barriers); on expiry the
// CTA raises its abort flag, the producer drains its in-flight copies, and
// all warps leave.
// ---------------------------------------------------------------------------

template <int K, int NC>
struct DwpShape;
// Most compute threads per CTA and the register cap that fits them (plus the
// producer warp) in one SM's 64 K registers -- registers are granted to warps
// in groups of four, so the cap is 64 K / (32 * warps rounded up to 4),
// rounded down to 8: the K*K packed weights and the K x NC open output rows
// stay in registers for the whole tile. NC = output columns per thread.
template <>
struct DwpShape<3, 2> { static constexpr int kComp = 736; static constexpr int kRegs = 80; };
template <>
struct DwpShape<5, 2> { static constexpr int kComp = 480; static constexpr int kRegs = 128; };
template <>
struct DwpShape<7, 2> { static constexpr int kComp = 352; static constexpr int kRegs = 168; };
template <>
struct DwpShape<3, 4> { static constexpr int kComp = 608; static constexpr int kRegs = 96; };
template <>
struct DwpShape<5, 4> { static constexpr int kComp = 352; static constexpr int kRegs = 168; };
template <>
struct DwpShape<7, 4> { static constexpr int kComp = 224; static constexpr int kRegs = 255; };

constexpr int kDwpMaxStages = 4;
constexpr int kErrWaitDwp = 0x108;

struct DwpParams {
  int B, C, H, W, pad, n, Ho, Wo;
  int CC;           // channels per chunk (multiple of 8)
  int CB;           // output columns per tile
  int nc;           // output columns per compute thread (2 or 4)
  int ncomp;        // compute threads (a multiple of 32; the producer warp follows)
  int RB;           // output rows per tile
  int nchunks, bands, cbands;
  int S;            // stages in flight
  int stage_bytes;  // one stage: box | misc (128-aligned)
  int box_bytes;    // (RB+K-1) * (CB rounded up to nc, + K-1) * CC * 2
  int misc_off;     // alpha[n] | a_in[CC] | a_out[CC] | chan_add[CC], from the stage base
  int w_off;        // two mixed-kernel buffers, each [K*K][CC] weights + [CC] biases (fp32)
  int e_off;        // resident expert slabs [n][CC][K*K] bf16
  int eb_off;       // resident bias slabs [n][CC] fp32
  int bar_off;
  const __nv_bfloat16* experts;  // [n][C][K][K]
  const float* alpha;            // [B][n]
  const float* bias;             // [n][C] or null
  __nv_bfloat16* y;
  const float* a_in;             // [B][C] or null
  const float* a_out;            // [B][C] or null
  const float* chan_add;         // [B][C] or null
  float chan_scale;
  int* err;
  long long wait_ns;
  unsigned long long* stamps;  // optional [grid][8] phase stamps for measurements, or null
};

// CCPT: the channel pairs per chunk when known at compile time (the stride
// between staged columns, so every window load has an immediate offset), or
// 0 for any chunk width. NC: output columns per compute thread.
template <int K, int CCPT, int NC>
__global__ void __maxnreg__((DwpShape<K, NC>::kRegs))
    depthwise_pipe_kernel(const __grid_constant__ CUtensorMap xmap, DwpParams p) {
  constexpr int KK = K * K;
  const int NCOMP = p.ncomp;
  const int NWARP_C = NCOMP >> 5;
  extern __shared__ __align__(128) unsigned char dwp_raw[];
  unsigned char* sm = dwp_raw + ((128u - (smem_u32(dwp_raw) & 127u)) & 127u);
  const int t = threadIdx.x;
  const int warp = t >> 5, lane = t & 31;
  const int CCp = CCPT > 0 ? CCPT : (p.CC >> 1);
  const int TC = (p.CB + NC - 1) / NC * NC + K - 1;  // staged columns: tile width + halo

  // This CTA's chunk and a contiguous run of the chunk's tiles, so that
  // consecutive tiles are the row bands of one sample and share its kernels.
  const int chunk = blockIdx.x % p.nchunks;
  const int local = blockIdx.x / p.nchunks;
  const int sharers = (gridDim.x - chunk + p.nchunks - 1) / p.nchunks;
  const int c0 = chunk * p.CC;
  const int cc_valid = min(p.CC, p.C - c0);
  const int tiles = p.B * p.bands * p.cbands;
  const int t_begin = static_cast<int>(static_cast<long long>(local) * tiles / sharers);
  const int t_end = static_cast<int>(static_cast<long long>(local + 1) * tiles / sharers);
  const int my_tiles = local < sharers ? t_end - t_begin : 0;

  const uint32_t bar0 = smem_u32(sm + p.bar_off);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kDwpMaxStages + s); };
  auto mixed = [&](int g) { return bar0 + 8u * (2 * kDwpMaxStages + g); };  // 2 buffers
  const uint32_t ebar = bar0 + 8u * (2 * kDwpMaxStages + 2);
  volatile int* abort_flag =
      reinterpret_cast<volatile int*>(sm + p.bar_off + 8 * (2 * kDwpMaxStages + 3));
  const WaitCtl ctl{abort_flag, p.err, p.wait_ns};
  const __nv_bfloat16* ebuf = reinterpret_cast<const __nv_bfloat16*>(sm + p.e_off);
  const float* ebias = reinterpret_cast<const float*>(sm + p.eb_off);

  if (t == 0) {
    for (int s = 0; s < kDwpMaxStages; ++s) {
      mbar_init(full(s), 33);        // producer lane 0's expect-tx arrive + 32 lane arrives
      mbar_init(empty(s), NWARP_C);  // one arrive per compute warp
    }
    mbar_init(mixed(0), NWARP_C);
    mbar_init(mixed(1), NWARP_C);
    mbar_init(ebar, 1);
    *abort_flag = 0;
    fence_mbar_init();
    tma_prefetch_desc(&xmap);
  }
  __syncthreads();
  grid_dependency_wait();  // alpha (and x) come from earlier kernels
  // the next kernel on the stream (a routing kernel of the next layer) may
  // be scheduled while this one runs: it waits for this grid's completion
  // before it reads anything this grid writes
  grid_launch_dependents();
  // phase stamps (measurement hook): [0] entry after set-up, [1] slabs in,
  // [5] end, [6] SM id, [7] global timer at entry
  if (p.stamps != nullptr && t == 0) {
    unsigned long long* stp = p.stamps + blockIdx.x * 8;
    stp[0] = clock64();
    stp[7] = globaltimer_ns();
    uint32_t smid;
    asm volatile("mov.u32 %0, %%smid;" : "=r"(smid));
    stp[6] = smid;
  }

  auto tile_coords = [&](int k, int& b, int& oh0, int& ow0) {
    int u = t_begin + k;
    const int cb = u % p.cbands;
    u /= p.cbands;
    const int band = u % p.bands;
    b = u / p.bands;
    oh0 = band * p.RB;
    ow0 = cb * p.CB;
  };

  if (warp == NWARP_C) {
    // =============================== producer ===============================
    if (my_tiles > 0 && lane == 0) {
      const uint32_t eb = static_cast<uint32_t>(cc_valid) * KK * 2;
      const uint32_t bb = p.bias ? static_cast<uint32_t>(cc_valid) * 4 : 0u;
      mbar_arrive_expect_tx(ebar, static_cast<uint32_t>(p.n) * (eb + bb));
      for (int i = 0; i < p.n; ++i) {
        bulk_load(smem_u32(sm + p.e_off) + static_cast<uint32_t>(i) * p.CC * KK * 2,
                  p.experts + (static_cast<size_t>(i) * p.C + c0) * KK, eb, ebar);
        if (p.bias)
          bulk_load(smem_u32(sm + p.eb_off) + static_cast<uint32_t>(i) * p.CC * 4,
                    p.bias + static_cast<size_t>(i) * p.C + c0, bb, ebar);
      }
    }
    int issued = 0;
    for (int k = 0; k < my_tiles; ++k) {
      const int s = k % p.S;
      const uint32_t ph = static_cast<uint32_t>(k / p.S) & 1u;
      if (!wait_bounded(empty(s), ph ^ 1u, ctl, kErrWaitDwp)) break;
      int b, oh0, ow0;
      tile_coords(k, b, oh0, ow0);
      unsigned char* st = sm + static_cast<size_t>(s) * p.stage_bytes;
      float* misc = reinterpret_cast<float*>(st + p.misc_off);
      for (int j = lane; j < p.n; j += 32) misc[j] = p.alpha[static_cast<size_t>(b) * p.n + j];
      float* fin = misc + p.n;
      for (int c = lane; c < cc_valid; c += 32) {
        const size_t o = static_cast<size_t>(b) * p.C + c0 + c;
        fin[c] = p.a_in ? p.a_in[o] : 1.f;
        fin[p.CC + c] = p.a_out ? p.a_out[o] : 1.f;
        fin[2 * p.CC + c] = p.chan_add ? p.chan_add[o] * p.chan_scale : 0.f;
      }
      if (lane == 0) {
        mbar_arrive_expect_tx(full(s), static_cast<uint32_t>(p.box_bytes));
        tma_load_4d(smem_u32(st), &xmap, full(s), c0, ow0 - p.pad, oh0 - p.pad, b);
      }
      __syncwarp();
      mbar_arrive(full(s));
      ++issued;
    }
    if (lane == 0) {
      // leave no copy in flight: the last S issued tiles (the compute warps
      // consumed the rest), and the resident slabs
      for (int j = (issued > p.S ? issued - p.S : 0); j < issued; ++j)
        wait_drain(full(j % p.S), static_cast<uint32_t>(j / p.S) & 1u, p.wait_ns, p.err);
      if (my_tiles > 0) wait_drain(ebar, 0, p.wait_ns, p.err);
    }
    return;
  }

  // ================================ compute ================================
  if (my_tiles == 0) return;
  if (!wait_bounded(ebar, 0, ctl, kErrWaitDwp)) return;
  if (p.stamps != nullptr && t == 0) p.stamps[blockIdx.x * 8 + 1] = clock64();
  const int cgrp = t / CCp, pair = t - (t / CCp) * CCp;
  const int col = NC * cgrp;  // this thread's output columns col .. col + NC - 1 in the tile
  const int w_floats = (KK + 1) * p.CC;
  // this thread's mixing items it = t, t + NCOMP, ...: (tap, channel) walked
  // incrementally (tap KK = the bias)
  const int d_tap = NCOMP / p.CC, d_c = NCOMP - (NCOMP / p.CC) * p.CC;
  int prev_b = -1, gen = -1;
  uint64_t w2[KK];
  uint64_t bias2 = 0;
  float ao0 = 1.f, ao1 = 1.f;
  for (int k = 0; k < my_tiles; ++k) {
    const int s = k % p.S;
    const uint32_t ph = static_cast<uint32_t>(k / p.S) & 1u;
    if (!wait_bounded(full(s), ph, ctl, kErrWaitDwp)) return;
    int b, oh0, ow0;
    tile_coords(k, b, oh0, ow0);
    unsigned char* st = sm + static_cast<size_t>(s) * p.stage_bytes;
    const float* misc = reinterpret_cast<const float*>(st + p.misc_off);
    const float* fin = misc + p.n;

    if (b != prev_b) {
      // ---- a new sample: mix its kernels (fp32, expert by expert) into the
      // next of the two buffers; the previous sample's buffer may still be
      // read by a slower warp until it has passed this sample's barrier
      prev_b = b;
      ++gen;
      float* wb = reinterpret_cast<float*>(sm + p.w_off) + (gen & 1) * w_floats;  // [KK][CC] | [CC]
      int tap = t / p.CC, c = t - (t / p.CC) * p.CC;
      for (int it = t; it < w_floats; it += NCOMP) {
        if (c < cc_valid) {
          float sacc = 0.f;
          if (tap < KK) {
            const __nv_bfloat16* e = ebuf + c * KK + tap;
            for (int j = 0; j < p.n; ++j, e += p.CC * KK)
              sacc = fmaf(misc[j], __bfloat162float(*e), sacc);
            wb[it] = sacc * fin[c];  // input attention folded (depthwise: one channel)
          } else {
            if (p.bias)
              for (int j = 0; j < p.n; ++j) sacc = fmaf(misc[j], ebias[j * p.CC + c], sacc);
            wb[it] = sacc + fin[2 * p.CC + c];
          }
        }
        tap += d_tap;
        c += d_c;
        if (c >= p.CC) { c -= p.CC; ++tap; }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(mixed(gen & 1));
      if (!wait_bounded(mixed(gen & 1), static_cast<uint32_t>(gen >> 1) & 1u, ctl, kErrWaitDwp))
        return;
      // the sample's weights stay in registers for all its tiles
#pragma unroll
      for (int q = 0; q < KK; ++q) w2[q] = *reinterpret_cast<const uint64_t*>(wb + q * p.CC + 2 * pair);
      bias2 = *reinterpret_cast<const uint64_t*>(wb + KK * p.CC + 2 * pair);
      ao0 = fin[p.CC + 2 * pair];
      ao1 = fin[p.CC + 2 * pair + 1];
    }

    const int ow = ow0 + col;
    const int c = c0 + 2 * pair;
    const bool active = col < p.CB && ow < p.Wo && c < p.C;
    if (active) {
      const bool scale_out = p.a_out != nullptr;
      const int ncv = min(NC, min(p.CB - col, p.Wo - ow));  // columns of this thread in the image
      const uint32_t* xw = reinterpret_cast<const uint32_t*>(st) + col * CCp + pair;
      const int row_words = TC * CCp;
      const size_t ystride = static_cast<size_t>(p.Wo) * p.C;  // one output row
      // output row o of the tile goes to ydst0 + o * ystride (rows past Ho are skipped)
      __nv_bfloat16* ydst0 =
          p.y + (static_cast<size_t>(b) * p.Ho * p.Wo + static_cast<size_t>(oh0) * p.Wo + ow) * p.C + c;
      const int rows_out = min(p.RB, p.Ho - oh0);  // rows of this band inside the image
      const int rows_in = p.RB + K - 1;
      uint64_t acc[K][NC];  // open output rows, slot o % K
      auto store_row = [&](const uint64_t (&a)[NC], int o) {
        if (o < rows_out) {
          __nv_bfloat16* dst = ydst0 + static_cast<size_t>(o) * ystride;
#pragma unroll
          for (int q = 0; q < NC; ++q) {
            float l = __uint_as_float(static_cast<uint32_t>(a[q]));
            float h = __uint_as_float(static_cast<uint32_t>(a[q] >> 32));
            if (scale_out) { l *= ao0; h *= ao1; }
            if (q == 0 || q < ncv) *reinterpret_cast<uint32_t*>(dst + q * p.C) = pack_bf16x2(l, h);
          }
        }
      };
      // One group of K input rows starting at ir0 (a multiple of K): input
      // row ir feeds output rows o = ir - kh, opens row ir (kh = 0: the
      // accumulator starts from the bias) and completes row ir - (K-1). Every
      // loop is fully unrolled, so each accumulator slot is a fixed register.
      // The band edges (o < 0, o >= RB, ir >= rows_in) are compile-time for
      // the HEAD group (ir0 = 0, RB >= K) and the TAIL group (ir0 = RB, RB a
      // multiple of K); MID groups have none; GENERIC tests them at run time.
      enum { MID = 0, HEAD = 1, TAIL = 2, GENERIC = 3 };
      auto group = [&](int ir0, auto kind_tag) {
        constexpr int KIND = decltype(kind_tag)::value;
        const uint32_t* xr = xw + ir0 * row_words;
#pragma unroll
        for (int j = 0; j < K; ++j, xr += row_words) {
          const int ir = ir0 + j;
          if (KIND == TAIL && j >= K - 1) continue;              // ir >= RB + K - 1
          if (KIND == GENERIC && ir >= rows_in) continue;
          uint64_t xv[K + NC - 1];
#pragma unroll
          for (int kw = 0; kw < K + NC - 1; ++kw) xv[kw] = bf16x2_to_f32x2(xr[kw * CCp]);
          // the K open rows this input row feeds (kh = 0 opens row ir from
          // the bias, kh = K-1 completes row ir - K + 1); for small windows the
          // products run kw-outer so that the K x NC accumulator chains
          // interleave
          bool live[K];
          uint64_t a[K][NC];
#pragma unroll
          for (int kh = 0; kh < K; ++kh) {
            const int o = ir - kh;
            if (KIND == MID) live[kh] = true;
            else if (KIND == HEAD) live[kh] = j >= kh;   // o >= 0; o < K <= RB
            else if (KIND == TAIL) live[kh] = j < kh;    // o < RB; o >= RB - K + 1 >= 0
            else live[kh] = o >= 0 && o < p.RB;
#pragma unroll
            for (int q = 0; q < NC; ++q) a[kh][q] = kh == 0 ? bias2 : acc[(j - kh + K) % K][q];
          }
          if constexpr (K * NC <= 10) {
#pragma unroll
            for (int kw = 0; kw < K; ++kw)
#pragma unroll
              for (int kh = 0; kh < K; ++kh)
                if (live[kh])
#pragma unroll
                  for (int q = 0; q < NC; ++q)
                    a[kh][q] = ffma2(xv[kw + q], w2[kh * K + kw], a[kh][q]);
          } else {  // larger windows: row by row (fewer live registers)
#pragma unroll
            for (int kh = 0; kh < K; ++kh)
              if (live[kh])
#pragma unroll
                for (int kw = 0; kw < K; ++kw)
#pragma unroll
                  for (int q = 0; q < NC; ++q)
                    a[kh][q] = ffma2(xv[kw + q], w2[kh * K + kw], a[kh][q]);
          }
          if (live[K - 1]) store_row(a[K - 1], ir - (K - 1));
#pragma unroll
          for (int kh = 0; kh < K - 1; ++kh)
            if (live[kh])
#pragma unroll
              for (int q = 0; q < NC; ++q) acc[(j - kh + K) % K][q] = a[kh][q];  // slot o % K
        }
      };
      using KMid = std::integral_constant<int, MID>;
      using KHead = std::integral_constant<int, HEAD>;
      using KTail = std::integral_constant<int, TAIL>;
      using KGen = std::integral_constant<int, GENERIC>;
      if (p.RB >= K && p.RB % K == 0) {
        group(0, KHead{});
#pragma unroll 1
        for (int ir0 = K; ir0 < p.RB; ir0 += K) group(ir0, KMid{});
        group(p.RB, KTail{});
      } else {
#pragma unroll 1
        for (int ir0 = 0; ir0 < rows_in; ir0 += K) group(ir0, KGen{});
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(empty(s));
  }
  if (p.stamps != nullptr && t == 0) p.stamps[blockIdx.x * 8 + 5] = clock64();
}

}  // namespace dc
