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
