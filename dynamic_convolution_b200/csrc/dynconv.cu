// Host side of the C ABI declared in include/dynconv.h: argument validation,
// variant selection, tensor-map encoding and kernel launches. Device code lives
// in the *.cuh files included below (one translation unit, sm_100a only).
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <utility>
#include <vector>

#include "dynconv.h"
#include "internal.h"

#include "common.cuh"
#include "conv_tc.cuh"
#include "depthwise.cuh"
#include "direct.cuh"
#include "premix.cuh"
#include "premix_small.cuh"
#include "premix_t.cuh"
#include "mixconv.cuh"
#include "route.cuh"
#include "pool.cuh"

namespace {

// One error word per device (module globals are instantiated per device).
__device__ int g_device_err;

// Scratch of dynconv_forward_noalloc: a fixed array in device memory, one per
// device that loads this module. In host code its name is only a stand-in, not
// a device address: dynconv_forward_noalloc looks the address up on its first
// call on each device and keeps it in g_noalloc_ptr.
static __device__ __align__(256) unsigned char g_noalloc_scratch[DYNCONV_NOALLOC_MAX_BYTES];
// State slots of the streamed mixing (slice counters), zero between launches.
static __device__ __align__(256) unsigned int g_mix_state[dc::kMcSlots][dc::kMcStateWords];

constexpr long long kDefaultWaitNs = 500LL * 1000 * 1000;  // 0.5 s
constexpr int kMaxDevices = 64;

struct DeviceState {
  bool ready = false;
  int* err = nullptr;  // device address of g_device_err on this device
  int sms = 0;
  int max_smem_optin = 0;
  int cc_major = 0, cc_minor = 0;
  long long l2_bytes = 0;
};

std::mutex g_mu;
DeviceState g_dev[kMaxDevices];
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
std::atomic<unsigned long long> g_launches{0};
std::atomic<long long> g_wait_ns{kDefaultWaitNs};
std::atomic<int> g_inject_skip{0};
std::atomic<int> g_route_split{0};  // 0: automatic
std::atomic<int> g_use_pdl{1};      // programmatic launch edges on forward kernels
std::atomic<int> g_stream_mix{0};   // PREMIX with n <= 8: mixing streamed into the convolution
std::atomic<int> g_premix_mixer{0};  // 0 automatic, 1 tensor-core GEMM, 2 CUDA cores (n <= 8),
                                     // 3 the transposed tensor-core GEMM (B <= 256)
std::atomic<int> g_dw_kernel{0};     // 0 pipelined depthwise kernel when it fits, 1 the per-tile one,
                                     // 2 / 3 the pipelined one with 2 / 4 columns per thread
constexpr int kDwpDefaultNc = 2;     // columns per thread of the pipelined depthwise kernel
constexpr int kTransposedMixMax = 0;   // batches up to this mix with the transposed GEMM by default
                                     // (none: the M = samples GEMM with eight epilogue warps
                                     // measured faster even at 32 samples)
std::atomic<int> g_conv_persist{1};  // PREMIX convolution: 1 persistent kernel when it fits, 0 one CTA per unit
std::atomic<int> g_group_mix{0};     // PREMIX, n > 8, large B*|W|: 0 one pass, 1 grouped mixing
                                     // pipeline (concurrent), 2 grouped in sequence
std::atomic<int> g_premix_direct{0}; // premix epilogue: 1 stores from registers when aligned, 0 staged
std::atomic<int> g_mixgrad_tc{1};    // backward: 1 tensor-core mixing gradient when it fits, 0 CUDA cores
std::atomic<long long> g_group_bytes{40LL << 20};  // target bytes of one group's mixed kernels
std::atomic<unsigned long long> g_conv_stamps{0};  // device buffer for the kernels' phase stamps
std::atomic<int> g_persist_rows{0};  // persistent convolution: output rows per unit (0: planned)
std::atomic<int> g_premix_dyn{1};    // mixing GEMM (one pass) tiles from a counter: 1 when the
                                     // experts exceed half the L2, 2 always, 0 never (static)
std::atomic<long long> g_group_min{64LL << 20};    // below this B*|W| the one-pass form is used
thread_local char g_last_err[256] = "";

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);
EncodeTiledFn g_encode = nullptr;

int cuda_fail(cudaError_t e, const char* what) {
  std::snprintf(g_last_err, sizeof(g_last_err), "%s: %s", what, cudaGetErrorString(e));
  return DYNCONV_ERR_CUDA;
}

// Current device's state; initialises it on first use (error-word address, limits).
int device_state(DeviceState** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return cuda_fail(cudaErrorInvalidDevice, "device index");
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState& st = g_dev[dev];
  if (!st.ready) {
    cudaDeviceProp prop;
    e = cudaGetDeviceProperties(&prop, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDeviceProperties");
    if (prop.major != 10) {
      std::snprintf(g_last_err, sizeof(g_last_err),
                    "device %d is sm_%d%d; this library is built for sm_100a only", dev,
                    prop.major, prop.minor);
      return DYNCONV_ERR_CUDA;
    }
    st.sms = prop.multiProcessorCount;
    st.max_smem_optin = static_cast<int>(prop.sharedMemPerBlockOptin);
    st.l2_bytes = prop.l2CacheSize;
    st.cc_major = prop.major;
    st.cc_minor = prop.minor;
    void* addr = nullptr;
    e = cudaGetSymbolAddress(&addr, g_device_err);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(error word)");
    st.err = static_cast<int*>(addr);
    if (!g_encode) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      e = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q);
      if (e != cudaSuccess || q != cudaDriverEntryPointSuccess || !fn)
        return cuda_fail(e == cudaSuccess ? cudaErrorSymbolNotFound : e,
                         "cuTensorMapEncodeTiled entry point");
      g_encode = reinterpret_cast<EncodeTiledFn>(fn);
    }
    st.ready = true;
  }
  *out = &st;
  return DYNCONV_OK;
}

// cudaFuncSetAttribute once per (device, kernel, size): keeps launches cheap
// and keeps the call out of stream captures after the first launch.
std::mutex g_smem_mu;
std::map<std::pair<int, const void*>, size_t> g_smem_set;

template <typename K>
cudaError_t ensure_smem(K kern, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(dev, reinterpret_cast<const void*>(kern));
  std::lock_guard<std::mutex> lk(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) g_smem_set[key] = bytes;
  return e;
}

// Launch with a programmatic stream-serialization edge: the kernel may start
// while the previous kernel on the stream finishes; it calls
// griddepcontrol.wait before reading any global memory.
template <typename Kern, typename... Args>
cudaError_t launch_pdl(Kern kern, dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_use_pdl.load() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kern, args...);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

int out_size(int in, int k, int stride, int pad) { return (in + 2 * pad - k) / stride + 1; }

int validate_desc(const dynconv_desc* d) {
  if (!d) return DYNCONV_ERR_INVALID_ARG;
  if (d->B < 0 || d->C_in <= 0 || d->H <= 0 || d->W <= 0 || d->C_out <= 0 || d->KH <= 0 ||
      d->KW <= 0 || d->stride <= 0 || d->pad < 0 || d->groups <= 0 || d->n <= 0)
    return DYNCONV_ERR_INVALID_ARG;
  if (d->dtype != DYNCONV_F32 && d->dtype != DYNCONV_BF16) return DYNCONV_ERR_INVALID_ARG;
  if (d->variant < DYNCONV_VARIANT_AUTO || d->variant > DYNCONV_VARIANT_DEPTHWISE)
    return DYNCONV_ERR_INVALID_ARG;
  if (d->C_in % d->groups != 0 || d->C_out % d->groups != 0) return DYNCONV_ERR_INVALID_ARG;
  if (out_size(d->H, d->KH, d->stride, d->pad) <= 0 || out_size(d->W, d->KW, d->stride, d->pad) <= 0)
    return DYNCONV_ERR_INVALID_ARG;
  // 32-bit index arithmetic inside the kernels
  const long long xe = 1LL * d->B * d->H * d->W * d->C_in;
  const long long ye = 1LL * d->B * out_size(d->H, d->KH, d->stride, d->pad) *
                       out_size(d->W, d->KW, d->stride, d->pad) * d->C_out;
  if (xe >= (1LL << 40) || ye >= (1LL << 40)) return DYNCONV_ERR_UNSUPPORTED;
  return DYNCONV_OK;
}

size_t elem_bytes(const dynconv_desc* d) { return d->dtype == DYNCONV_F32 ? 4 : 2; }

// ------------------------------------------------------------------ planning

struct TcPlan {
  dc::TcParams p;
  int grid = 0;
  size_t smem = 0;
  double cost = 0;  // estimated SM cycles of the longest SM
};

bool tc_shape_ok(const dynconv_desc* d) {
  return d->dtype == DYNCONV_BF16 && d->groups == 1 && d->stride == 1 && d->C_in % 8 == 0 &&
         d->C_out % 8 == 0 && d->W + d->KW - 1 <= 256 && d->KH <= 32 && d->n <= 1024 &&
         out_size(d->H, d->KH, 1, d->pad) == d->H && out_size(d->W, d->KW, 1, d->pad) == d->W;
}

// Descriptor base-offset mode for shifted activation views (see conv_tc.cuh).
// 0 is correct on B200: the swizzle is applied on absolute address bits.
int g_desc_base_mode = 0;

// Build the tensor-core plan for one variant, or return false.
//
// Cost model (SM clock cycles of the busiest SM): per A step the MMA takes
// 2*N_pad cycles (M=128, K=64 at 4096 MAC/clk); producing A costs its L2
// bytes at ~20 B/clk per SM (the measured share of L2 bandwidth when every
// SM streams), n*16 KB for FUSED and 16 KB otherwise; the activation tile costs
// its bytes once per chunk; units run in waves over the SMs.
bool tc_plan(const dynconv_desc* d, int variant, int sms, int max_smem, TcPlan* out) {
  if (!tc_shape_ok(d)) return false;
  const int taps = d->KH * d->KW;
  const int kc = (d->C_in + 63) / 64;
  const int m_tiles = (d->C_out + 127) / 128;
  const int spc = variant == DYNCONV_VARIANT_OUTSIDE ? taps * d->n : taps;
  const int k_steps = kc * spc;
  const int Wp = d->W + d->KW - 1;
  if (Wp > 256) return false;
  const int s_tap_max = (d->KH - 1) * Wp + (d->KW - 1);
  bool found = false;
  TcPlan best;
  for (int R = 1; R <= d->H; ++R) {
    const int n_virt = R * Wp;
    const int n_pad = (n_virt + 15) / 16 * 16;
    if (n_pad > 512) break;
    const int box_rows = R + d->KH - 1;
    if (box_rows > 256) break;
    int n0 = n_pad, n1 = 0;
    if (n_pad > 256) { n0 = 256; n1 = n_pad - 256; }
    const int rows = std::max(box_rows * Wp, s_tap_max + n_pad);
    const int b_tile = (rows * 128 + 1023) / 1024 * 1024;
    const size_t fixed = 1024 /*align slack*/ + 8 * 64 /*barriers*/ + 16 + 4 * d->n + 64 +
                         1024 /*the tile's biases and output attentions*/;
    const size_t T = dc::kTcATileBytes;
    int sb = kc > 1 ? 2 : 1;
    int sa = 0, se = 0;
    if (variant == DYNCONV_VARIANT_PREMIX) {
      if (fixed + sb * static_cast<size_t>(b_tile) + 2 * T > static_cast<size_t>(max_smem)) continue;
      sa = static_cast<int>((max_smem - fixed - sb * static_cast<size_t>(b_tile)) / T);
      sa = std::min(sa, 8);
    } else {
      // two A stages and a ring of expert tiles (ideally two K steps' worth,
      // at least two tiles); one activation stage when two leave too few
      const int ne = variant == DYNCONV_VARIANT_FUSED ? d->n : 1;
      const int want = std::min(16, std::max(4, 2 * ne));
      for (int tsb = sb; tsb >= 1 && se < want; --tsb) {
        const long long room = static_cast<long long>(max_smem) - static_cast<long long>(fixed) -
                               tsb * static_cast<long long>(b_tile) - 2 * static_cast<long long>(T);
        const int fit = room > 0 ? static_cast<int>(std::min<long long>(room / T, want)) : 0;
        if (fit > se) { se = fit; sb = tsb; }
      }
      if (se < 2) continue;
      sa = 2;
    }
    const int tiles_h = (d->H + R - 1) / R;
    const long long units = 1LL * d->B * tiles_h * m_tiles;
    const long long waves = (units + sms - 1) / sms;
    const double mma = 2.0 * n_pad;
    // operand bytes per K step: PREMIX one mixed-kernel tile (~20 B/clk from
    // HBM or L2), FUSED n expert tiles and OUTSIDE one (L2-resident, TMA)
    const double a_bytes = variant == DYNCONV_VARIANT_FUSED ? 16384.0 * d->n : 16384.0;
    const double a_cost = a_bytes / (variant == DYNCONV_VARIANT_PREMIX ? 20.0 : 40.0);
    const double b_cost = static_cast<double>(box_rows) * Wp * 128.0 / 20.0;
    const double t_unit = k_steps * std::max(mma, a_cost) + kc * b_cost / 4.0 + 40.0 * n_pad + 3000.0;
    const double cost = waves * t_unit;
    if (!found || cost < best.cost) {
      found = true;
      best.cost = cost;
      best.grid = static_cast<int>(units);
      best.smem = fixed + sb * static_cast<size_t>(b_tile) + (sa + se) * T;
      dc::TcParams& p = best.p;
      std::memset(&p, 0, sizeof(p));
      p.B = d->B; p.H = d->H; p.W = d->W; p.Cin = d->C_in; p.Cout = d->C_out;
      p.KH = d->KH; p.KW = d->KW; p.pad = d->pad; p.n = d->n;
      p.R = R; p.tiles_h = tiles_h; p.m_tiles = m_tiles; p.Wp = Wp; p.n_virt = n_virt;
      p.n_mma0 = n0; p.n_mma1 = n1; p.kc = kc; p.spc = spc; p.k_steps = k_steps;
      p.sa = sa; p.sb = sb; p.se = se; p.b_tile_bytes = b_tile; p.b_box_rows = box_rows;
      p.desc_base_mode = g_desc_base_mode;
      uint32_t cols = 32;
      while (cols < static_cast<uint32_t>(n_pad)) cols <<= 1;
      p.tmem_cols = cols;
    }
  }
  if (!found || best.grid <= 0 || best.grid > (1 << 30)) return false;
  *out = best;
  return true;
}

// Plan of the persistent PREMIX convolution (tc_conv_persist_kernel): two
// TMEM accumulators of up to 256 columns each, so row blocks of at most 256
// padded pixels; one CTA per SM. Cost (cycles of the busiest CTA): its units
// times the slowest of MMA issue (2 * N_pad per K step), operand bytes
// (16 KB per step at ~20 B/clk from L2), the epilogue (~4 cycles per padded
// pixel column) and the unit's HBM bytes at its share of the bandwidth
// (~23 B/clk per SM); plus one epilogue and a fixed set-up.
bool tc_plan_persist(const dynconv_desc* d, int sms, int max_smem, TcPlan* out) {
  if (!tc_shape_ok(d)) return false;
  const int taps = d->KH * d->KW;
  const int kc = (d->C_in + 63) / 64;
  const int m_tiles = (d->C_out + 127) / 128;
  const int k_steps = kc * taps;
  const int Wp = d->W + d->KW - 1;
  if (Wp > 256) return false;
  const int s_tap_max = (d->KH - 1) * Wp + (d->KW - 1);
  bool found = false;
  TcPlan best;
  const int want_rows = g_persist_rows.load();
  for (int R = 1; R <= d->H; ++R) {
    const int n_virt = R * Wp;
    const int n_pad = (n_virt + 15) / 16 * 16;
    if (n_pad > 256) break;
    if (want_rows > 0 && R != std::min(want_rows, d->H)) continue;
    const int box_rows = R + d->KH - 1;
    if (box_rows > 256) break;
    const int rows = std::max(box_rows * Wp, s_tap_max + n_pad);
    const int b_tile = (rows * 128 + 1023) / 1024 * 1024;
    const size_t fixed = 1024 + dc::kTpStageBytes + 8 * 64 + 16;
    const int sb = kc > 1 ? 2 : 1;
    if (fixed + sb * static_cast<size_t>(b_tile) + 2 * dc::kTcATileBytes > static_cast<size_t>(max_smem))
      continue;
    int sa = static_cast<int>((max_smem - fixed - sb * static_cast<size_t>(b_tile)) / dc::kTcATileBytes);
    sa = std::min(sa, std::max(2, std::min(8, k_steps + 2)));
    const int tiles_h = (d->H + R - 1) / R;
    const long long units = 1LL * d->B * tiles_h * m_tiles;
    const long long grid = std::min<long long>(units, sms);
    const long long per_cta = (units + grid - 1) / grid;
    const double mma = k_steps * std::max(2.0 * n_pad, 16384.0 / 20.0);
    const double epi = 4.0 * n_pad;
    const double bytes = 2.0 * (static_cast<double>(kc) * 64 * Wp * box_rows + 128.0 * R * d->W) +
                         16384.0 * k_steps;
    const double t_unit = std::max({mma, epi, bytes / 23.0});
    const double cost = per_cta * t_unit + epi + 3000.0;
    if (!found || cost < best.cost) {
      found = true;
      best.cost = cost;
      best.grid = static_cast<int>(grid);
      best.smem = fixed + sb * static_cast<size_t>(b_tile) + sa * static_cast<size_t>(dc::kTcATileBytes);
      dc::TcParams& p = best.p;
      std::memset(&p, 0, sizeof(p));
      p.B = d->B; p.H = d->H; p.W = d->W; p.Cin = d->C_in; p.Cout = d->C_out;
      p.KH = d->KH; p.KW = d->KW; p.pad = d->pad; p.n = d->n;
      p.R = R; p.tiles_h = tiles_h; p.m_tiles = m_tiles; p.Wp = Wp; p.n_virt = n_virt;
      p.n_mma0 = n_pad; p.n_mma1 = 0; p.kc = kc; p.spc = taps; p.k_steps = k_steps;
      p.sa = sa; p.sb = sb; p.b_tile_bytes = b_tile; p.b_box_rows = box_rows;
      p.desc_base_mode = g_desc_base_mode;
      uint32_t cols = 32;
      while (cols < static_cast<uint32_t>(n_pad)) cols <<= 1;
      p.tmem_cols = 2 * cols;
    }
  }
  if (!found || best.grid <= 0) return false;
  *out = best;
  return true;
}

bool depthwise_ok(const dynconv_desc* d) {
  return d->dtype == DYNCONV_BF16 && d->groups == d->C_in && d->C_in == d->C_out &&
         d->stride == 1 && d->KH == d->KW && (d->KH == 3 || d->KH == 5 || d->KH == 7) &&
         d->C_in % 8 == 0 && d->n <= 4096 && out_size(d->H, d->KH, 1, d->pad) >= 1 &&
         out_size(d->W, d->KW, 1, d->pad) >= 1;
}

// Plan of the pipelined depthwise kernel (depthwise_pipe_kernel) with `nc`
// output columns per thread: chunk width CC and tile width CB so that the
// CC/2 x ceil(CB/nc) compute threads fill the kernel's most threads with the
// least waste (idle threads, channels past C, columns past W_out); then the
// tallest row band RB for which three stages, the resident expert and bias
// slabs and the barriers fit in shared memory (two stages when three do not
// fit). False when the shape does not fit.
bool dwp_plan(const dynconv_desc* d, int sms, int max_smem, bool has_bias, int nc,
              dc::DwpParams* p, int* grid, size_t* smem_out) {
  const int K = d->KH, KK = K * K;
  int ncomp = 0;
  if (nc == 2)
    ncomp = K == 3 ? dc::DwpShape<3, 2>::kComp : K == 5 ? dc::DwpShape<5, 2>::kComp
                                                        : dc::DwpShape<7, 2>::kComp;
  else if (nc == 4)
    ncomp = K == 3 ? dc::DwpShape<3, 4>::kComp : K == 5 ? dc::DwpShape<5, 4>::kComp
                                                        : dc::DwpShape<7, 4>::kComp;
  else
    return false;
  const int Ho = out_size(d->H, K, 1, d->pad), Wo = out_size(d->W, K, 1, d->pad);
  const int C = d->C_in;
  auto a128 = [](size_t v) { return (v + 127) / 128 * 128; };
  const size_t bars = 8 * (3 * dc::kDwpMaxStages + 1) + 16;
  // Shared bytes of a chunk width: the resident slabs, the two mixed-kernel
  // buffers, one stage's attentions; and the band plan of a (CC, CB): the
  // tallest band for which S = 3 stages fit (S = 2 when that band would be
  // shorter than min(Ho, 8)), balanced over the bands, then rounded up to a
  // multiple of K when that still fits (every band-edge test of the kernel
  // is then resolved at compile time).
  struct Slabs { size_t e, eb, w, misc; };
  auto slabs_of = [&](int CC) {
    return Slabs{a128(static_cast<size_t>(d->n) * CC * KK * 2),
                 has_bias ? a128(static_cast<size_t>(d->n) * CC * 4) : 0,
                 2 * a128(static_cast<size_t>(KK + 1) * CC * 4),
                 a128(static_cast<size_t>(d->n + 3 * CC) * 4)};
  };
  auto band_plan = [&](int CC, int CB, int* S, int* RB, int* bands) {
    const Slabs sl = slabs_of(CC);
    const size_t fixed = 128 + sl.w + sl.e + sl.eb + bars;
    const size_t TC = static_cast<size_t>((CB + nc - 1) / nc * nc + K - 1);
    if (fixed >= static_cast<size_t>(max_smem)) return false;
    for (int st : {3, 2}) {
      const size_t per = (static_cast<size_t>(max_smem) - fixed) / st;
      if (per <= sl.misc) continue;
      const long long rows = static_cast<long long>((per - sl.misc) / 128 * 128 / (TC * CC * 2));
      const long long rb = std::min<long long>({rows - (K - 1), Ho, 256 - (K - 1)});
      if (rb <= 0 || (rb < std::min(Ho, 8) && st == 3)) continue;
      int nb = static_cast<int>((Ho + rb - 1) / rb);
      int r = (Ho + nb - 1) / nb;
      const int rk = (r + K - 1) / K * K;
      if (rk <= rb) {
        r = rk;
        nb = (Ho + r - 1) / r;
      }
      *S = st;
      *RB = r;
      *bands = nb;
      return true;
    }
    return false;
  };
  double best = -1;
  int bCC = 0, bCB = 0;
  for (int CC = 8; CC <= std::min(256, (C + 7) / 8 * 8); CC += 8) {
    const int nch = (C + CC - 1) / CC;
    for (int CB = 1; CB <= std::min(Wo, 256 - (K - 1) - (nc - 1)); ++CB) {
      const int thr = CC / 2 * ((CB + nc - 1) / nc);  // one thread per channel pair and column group
      if (thr > ncomp) break;
      int S = 0, RB = 0, bands = 0;
      if (!band_plan(CC, CB, &S, &RB, &bands)) continue;
      const int cbands = (Wo + CB - 1) / CB;
      const int warps = (thr + 31) / 32;
      // useful work: channels past C, columns past W_out (the tile width
      // rounded up to nc), rows past H_out and the idle lanes of the last
      // warp are waste; the halo columns and rows are staged for every tile
      // (a mild preference for wide and tall tiles); a warp of 32 consecutive
      // pairs of one column group reads without bank conflicts, other chunk
      // widths with some; fewer than 8 compute warps hide latency less well
      const double eff =
          static_cast<double>(C) / (nch * CC) * Wo /
          (static_cast<double>(cbands) * ((CB + nc - 1) / nc * nc)) * Ho /
          (static_cast<double>(bands) * RB) * thr / (32.0 * warps) *
          (1.0 - 0.25 * (K - 1) / (CB + K - 1.0)) * (1.0 - 0.25 * (K - 1) / (RB + K - 1.0)) *
          ((CC / 2) % 32 == 0 ? 1.0 : 0.85) * std::min(1.0, warps / 8.0);
      if (eff > best + 1e-9) { best = eff; bCC = CC; bCB = CB; }
    }
  }
  if (bCC == 0) return false;
  const int CC = bCC, CB = bCB;
  int S = 0, RB = 0, bands = 0;
  if (!band_plan(CC, CB, &S, &RB, &bands)) return false;
  const Slabs sl = slabs_of(CC);
  const size_t e_bytes = sl.e, eb_bytes = sl.eb, w_bytes = sl.w, misc_bytes = sl.misc;
  const int TC = (CB + nc - 1) / nc * nc + K - 1;  // staged columns
  std::memset(p, 0, sizeof(*p));
  p->B = d->B; p->C = C; p->H = d->H; p->W = d->W; p->pad = d->pad; p->n = d->n;
  p->Ho = Ho; p->Wo = Wo; p->CC = CC; p->CB = CB; p->RB = RB;
  p->nc = nc;
  p->ncomp = (CC / 2 * ((CB + nc - 1) / nc) + 31) / 32 * 32;
  p->nchunks = (C + CC - 1) / CC;
  p->bands = bands;
  p->cbands = (Wo + CB - 1) / CB;
  p->S = S;
  p->box_bytes = (RB + K - 1) * TC * CC * 2;
  p->misc_off = static_cast<int>(a128(static_cast<size_t>(p->box_bytes)));
  p->stage_bytes = p->misc_off + static_cast<int>(misc_bytes);
  p->w_off = S * p->stage_bytes;
  p->e_off = p->w_off + static_cast<int>(w_bytes);
  p->eb_off = p->e_off + static_cast<int>(e_bytes);
  p->bar_off = p->eb_off + static_cast<int>(eb_bytes);
  const long long tiles_per_chunk = 1LL * d->B * p->bands * p->cbands;
  const long long g = std::min<long long>(std::max(sms, p->nchunks), p->nchunks * tiles_per_chunk);
  if (g <= 0 || g > (1 << 30)) return false;
  *grid = static_cast<int>(g);
  *smem_out = 128 + static_cast<size_t>(p->bar_off) + bars;
  return *smem_out <= static_cast<size_t>(max_smem);
}

// Workspace of PREMIX: the mixed kernels of every sample (256-byte aligned).
size_t premix_wb_bytes(const dynconv_desc* d) {
  return (static_cast<size_t>(d->B) * d->C_out * d->KH * d->KW * d->C_in * 2 + 255) & ~size_t(255);
}
// The mixed kernels, then 256 bytes for the mixing GEMM's tile counter.
constexpr size_t kPmCtrBytes = 256;
size_t premix_workspace(const dynconv_desc* d) {
  if (!tc_shape_ok(d)) return 0;
  if (!dc::premix_shape_ok(d->B, d->n, d->C_out, d->KH * d->KW, d->C_in)) return 0;
  return premix_wb_bytes(d) + kPmCtrBytes;
}

// Cost-model choice among the kernels that can run this descriptor.
int select_variant(const dynconv_desc* d, size_t ws_bytes, int sms, int max_smem) {
  if (d->dtype == DYNCONV_F32) return DYNCONV_VARIANT_DIRECT;
  if (d->groups != 1) return depthwise_ok(d) ? DYNCONV_VARIANT_DEPTHWISE : DYNCONV_VARIANT_DIRECT;
  if (!tc_shape_ok(d)) return DYNCONV_VARIANT_DIRECT;
  int best = DYNCONV_VARIANT_DIRECT;
  double best_cost = 0;
  for (int v : {DYNCONV_VARIANT_FUSED, DYNCONV_VARIANT_OUTSIDE, DYNCONV_VARIANT_PREMIX}) {
    TcPlan pl;
    if (!tc_plan(d, v, sms, max_smem, &pl)) continue;
    double cost = pl.cost;
    if (v == DYNCONV_VARIANT_PREMIX) {
      const size_t need = premix_workspace(d);
      if (need == 0 || ws_bytes < need) continue;
      // mixing GEMM: expert read + workspace write, bandwidth-bound (~23 B/clk/SM of HBM)
      const double bytes = 2.0 * d->n * d->C_out * d->KH * d->KW * d->C_in + static_cast<double>(need);
      cost += bytes / (23.0 * sms) + 3000.0;
    }
    if (best == DYNCONV_VARIANT_DIRECT || cost < best_cost) {
      best = v;
      best_cost = cost;
    }
  }
  return best;
}

// ------------------------------------------------------------------ launches

int check_launch(const char* what) {
  g_launches.fetch_add(1, std::memory_order_relaxed);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return cuda_fail(e, what);
  return DYNCONV_OK;
}

// Activations as a 4-D tensor {C_in, W, H, B}; one box = one 64-channel chunk
// of box_rows input rows at the padded width Wp (zero fill outside the image).
int encode_x_map(CUtensorMap* map, const void* x, const dynconv_desc* d, int Wp, int box_rows) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d->C_in), static_cast<cuuint64_t>(d->W),
                              static_cast<cuuint64_t>(d->H), static_cast<cuuint64_t>(d->B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d->C_in) * 2,
                                 static_cast<cuuint64_t>(d->W) * d->C_in * 2,
                                 static_cast<cuuint64_t>(d->H) * d->W * d->C_in * 2};
  const cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(Wp), static_cast<cuuint32_t>(box_rows), 1u};
  const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(x) failed: %d",
                  static_cast<int>(r));
    return DYNCONV_ERR_CUDA;
  }
  return DYNCONV_OK;
}

// Mixed kernels in the workspace, viewed as [B*C_out rows][taps][C_in], box {64, 1, 128}.
int encode_w_map(CUtensorMap* map, const void* w, const dynconv_desc* d) {
  const int taps = d->KH * d->KW;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(d->C_in), static_cast<cuuint64_t>(taps),
                              static_cast<cuuint64_t>(d->B) * d->C_out};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(d->C_in) * 2,
                                 static_cast<cuuint64_t>(taps) * d->C_in * 2};
  const cuuint32_t box[3] = {64u, 1u, 128u};
  const cuuint32_t es[3] = {1u, 1u, 1u};
  CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(w), dims,
                        strides, box, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
                        CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                        CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(w) failed: %d",
                  static_cast<int>(r));
    return DYNCONV_ERR_CUDA;
  }
  return DYNCONV_OK;
}

template <int V>
int launch_tc(const TcPlan& plan, const CUtensorMap& xmap, const CUtensorMap& wmap,
              cudaStream_t stream) {
  cudaError_t e = ensure_smem(dc::tc_conv_kernel<V>, plan.smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc_conv)");
  e = launch_pdl(dc::tc_conv_kernel<V>, dim3(plan.grid), dim3(dc::kTcThreads), plan.smem, stream,
                 xmap, wmap, plan.p);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_fail(e, "tc_conv_kernel launch");
  }
  return check_launch("tc_conv_kernel");
}


// The PREMIX convolution on mixed kernels already in the workspace: the
// persistent kernel when its plan exists, no pooled sums are asked for and it
// pays -- a CTA gets three or more units, or a unit has at most four K steps
// (its epilogue, not its MMAs, is then the unit's cost). With one or two
// MMA-bound units per CTA the persistent kernel issues as many MMAs per CTA as
// one CTA per (larger) unit does, while the epilogue of the first unit runs
// beside the MMA-issuing thread of the second and delays it; measured on the
// 3x3 layer (B=64, 128 channels, 28x28): 30.1 us against 26.4 us per forward.
// Else one CTA per unit.
int launch_premix_conv(const dynconv_desc* d, const TcPlan& plan, const DeviceState* st,
                       const void* x, const CUtensorMap& xmap, const CUtensorMap& wmap,
                       cudaStream_t stream) {
  TcPlan pp;
  const bool have = g_conv_persist.load() && plan.p.ysum == nullptr &&
                    tc_plan_persist(d, st->sms, st->max_smem_optin, &pp);
  const int units = have ? pp.p.B * pp.p.tiles_h * pp.p.m_tiles : 0;
  const bool pays = have && ((units + pp.grid - 1) / pp.grid >= 3 || pp.p.k_steps <= 4);
  if (pays || (have && g_conv_persist.load() == 2)) {
    const dc::TcParams& q = plan.p;
    pp.p.experts = q.experts; pp.p.alpha = q.alpha; pp.p.bias = q.bias; pp.p.y = q.y;
    pp.p.err = q.err; pp.p.wait_ns = q.wait_ns; pp.p.a_out = q.a_out;
    pp.p.chan_add = q.chan_add; pp.p.chan_scale = q.chan_scale; pp.p.stamps = q.stamps;
    // launched right after one of this library's mixing kernels (they signal
    // dependents only past their own wait), with a programmatic edge
    pp.p.x_early = g_use_pdl.load() ? 1 : 0;
    CUtensorMap pxmap;
    int rc = encode_x_map(&pxmap, x, d, pp.p.Wp, pp.p.b_box_rows);
    if (rc) return rc;
    cudaError_t e = ensure_smem(dc::tc_conv_persist_kernel, pp.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc_conv_persist)");
    e = launch_pdl(dc::tc_conv_persist_kernel, dim3(pp.grid), dim3(dc::kTcThreads), pp.smem,
                   stream, pxmap, wmap, pp.p);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      return cuda_fail(e, "tc_conv_persist_kernel launch");
    }
    return check_launch("tc_conv_persist_kernel");
  }
  TcPlan np = plan;
  np.p.x_early = g_use_pdl.load() ? 1 : 0;  // right after one of this library's mixing kernels
  return launch_tc<dc::kPremix>(np, xmap, wmap, stream);
}

// ------------------------------------------------------------ grouped PREMIX
// When every sample's mixed kernel together (B*|W| bf16) is far larger than
// the L2 and the mixing runs on the tensor-core GEMM (n > 8), the mixed
// kernels are made and consumed one group at a time through two workspace
// slots: the mixing GEMM of group g+1 runs on an internal stream while the
// persistent convolution consumes group g on the caller's stream, so a
// group's mixed kernels are read back while they are still in L2 instead of
// making a round trip through HBM. A group is either a run of samples (the
// experts, read once per group, stay in L2) or, when all samples' kernels for
// a run of 128-channel tiles fit, a run of output-channel tiles (every expert
// byte is read once in total). Event edges order the two streams; a stream
// capture records them as graph edges.
constexpr size_t kGroupExpertL2 = 48u << 20;  // sample groups: the experts must stay in L2
constexpr int kGroupTransposedMax = 64;       // groups of at most this many samples mix with premix_t

struct GroupPlan {
  int kind = 0;     // 0 none, 1 runs of samples, 2 runs of 128-channel tiles
  int groups = 0;
  int per = 0;      // samples (kind 1) or channels (kind 2) per group
  size_t slot = 0;  // bytes of one slot (256-aligned)
};

GroupPlan group_plan(const dynconv_desc* d) {
  GroupPlan g;
  if (d->n <= dc::kPsMaxExperts || !tc_shape_ok(d)) return g;
  const size_t taps_cin = static_cast<size_t>(d->KH) * d->KW * d->C_in;
  const size_t wsize = d->C_out * taps_cin;
  const size_t group_bytes = static_cast<size_t>(g_group_bytes.load());
  if (static_cast<size_t>(d->B) * wsize * 2 < static_cast<size_t>(g_group_min.load())) return g;
  const int m_tiles = (d->C_out + 127) / 128;
  const size_t per_tile = static_cast<size_t>(d->B) * 128 * taps_cin * 2;
  if (m_tiles >= 2 && per_tile <= group_bytes &&
      dc::premix_shape_ok(d->B, d->n, 128, d->KH * d->KW, d->C_in)) {
    const int mg = static_cast<int>(std::min<size_t>(m_tiles - 1, group_bytes / per_tile));
    g.kind = 2;
    g.per = mg * 128;
    g.groups = (d->C_out + g.per - 1) / g.per;
    g.slot = (static_cast<size_t>(d->B) * g.per * taps_cin * 2 + 255) & ~size_t(255);
    return g;
  }
  if (static_cast<size_t>(d->n) * wsize * 2 > kGroupExpertL2) return g;
  const int bg = static_cast<int>(std::max<size_t>(1, group_bytes / (wsize * 2)));
  if (bg >= d->B) return g;
  g.groups = (d->B + bg - 1) / bg;
  g.per = (d->B + g.groups - 1) / g.groups;  // balanced runs of samples
  if (!dc::premix_shape_ok(g.per, d->n, d->C_out, d->KH * d->KW, d->C_in)) return GroupPlan{};
  g.kind = 1;
  g.slot = (static_cast<size_t>(bg) * wsize * 2 + 255) & ~size_t(255);
  return g;
}

// The internal stream and events of one (device, caller stream), created on
// first use and kept for the life of the process.
struct AuxStream {
  cudaStream_t aux = nullptr;
  cudaEvent_t start = nullptr, mixed[2] = {nullptr, nullptr}, used[2] = {nullptr, nullptr};
};
std::mutex g_aux_mu;
std::map<std::pair<int, void*>, AuxStream> g_aux;

int aux_stream(cudaStream_t caller, AuxStream** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  std::lock_guard<std::mutex> lk(g_aux_mu);
  const auto key = std::make_pair(dev, static_cast<void*>(caller));
  auto it = g_aux.find(key);
  if (it != g_aux.end()) {
    *out = &it->second;
    return DYNCONV_OK;
  }
  AuxStream a;
  int prio = 0;
  if (caller != nullptr && cudaStreamGetPriority(caller, &prio) != cudaSuccess) prio = 0;
  e = cudaStreamCreateWithPriority(&a.aux, cudaStreamNonBlocking, prio);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamCreateWithPriority (internal stream)");
  cudaEvent_t* evs[5] = {&a.start, &a.mixed[0], &a.mixed[1], &a.used[0], &a.used[1]};
  for (cudaEvent_t* ev : evs) {
    e = cudaEventCreateWithFlags(ev, cudaEventDisableTiming);
    if (e != cudaSuccess) return cuda_fail(e, "cudaEventCreateWithFlags (internal event)");
  }
  auto ins = g_aux.emplace(key, a);
  *out = &ins.first->second;
  return DYNCONV_OK;
}

// PREMIX through the grouped pipeline (see group_plan). DYNCONV_ERR_UNSUPPORTED
// when a group's convolution has no persistent plan (nothing launched then).
int run_grouped(const dynconv_desc* d, const GroupPlan& gp, const DeviceState* st, const void* x,
                const void* experts, const float* alpha, const float* bias, void* y, void* ws,
                const float* a_out, const float* chan_add, float chan_scale, cudaStream_t stream) {
  const size_t taps_cin = static_cast<size_t>(d->KH) * d->KW * d->C_in;
  const size_t wsize = d->C_out * taps_cin;
  // every group's convolution must have a persistent plan before anything runs
  std::vector<TcPlan> plans(gp.groups);
  std::vector<dynconv_desc> subs(gp.groups);
  for (int g = 0; g < gp.groups; ++g) {
    dynconv_desc s = *d;
    if (gp.kind == 1) s.B = std::min(gp.per, d->B - g * gp.per);
    else s.C_out = std::min(gp.per, d->C_out - g * gp.per);
    subs[g] = s;
    // a group's convolution gets at most half of the SMs: the next group's
    // mixing runs on the others meanwhile
    if (!tc_plan_persist(&s, std::max(1, st->sms / 2), st->max_smem_optin, &plans[g]))
      return DYNCONV_ERR_UNSUPPORTED;
  }
  AuxStream* ax = nullptr;
  int rc = aux_stream(stream, &ax);
  if (rc) return rc;
  cudaError_t e = cudaEventRecord(ax->start, stream);
  if (e == cudaSuccess) e = cudaStreamWaitEvent(ax->aux, ax->start, 0);
  if (e != cudaSuccess) return cuda_fail(e, "grouped mixing: stream edge");
  const __nv_bfloat16* E = static_cast<const __nv_bfloat16*>(experts);
  for (int g = 0; g < gp.groups; ++g) {
    const int slot = g & 1;
    void* wsl = static_cast<char*>(ws) + slot * gp.slot;
    const dynconv_desc& s = subs[g];
    const size_t b0 = gp.kind == 1 ? static_cast<size_t>(g) * gp.per : 0;
    const size_t c0 = gp.kind == 2 ? static_cast<size_t>(g) * gp.per : 0;
    // ---- mixing of group g on the internal stream, once its slot is free
    if (g >= 2) {
      e = cudaStreamWaitEvent(ax->aux, ax->used[slot], 0);
      if (e != cudaSuccess) return cuda_fail(e, "grouped mixing: slot edge");
    }
    const long long wg = static_cast<long long>(s.C_out) * static_cast<long long>(taps_cin);
    // later groups share the GPU with the previous group's convolution
    const int mix_sms = g == 0 ? st->sms : std::max(16, st->sms - plans[g - 1].grid);
    if (s.B <= kGroupTransposedMax) {
      // few samples: M = weights, N = samples (every epilogue warp busy)
      dc::PremixTLaunch pl;
      rc = dc::plan_premix_t(E + c0 * taps_cin, static_cast<long long>(wsize), alpha + b0 * d->n,
                             static_cast<__nv_bfloat16*>(wsl), s.B, d->n, wg, st->err,
                             g_wait_ns.load(), mix_sms, g_encode, &pl);
      if (rc == -2) {
        std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(grouped premix) failed");
        return DYNCONV_ERR_CUDA;
      }
      if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
      e = ensure_smem(dc::premix_t_kernel, pl.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix_t)");
      dc::premix_t_kernel<<<pl.grid, dc::kPtThreads, pl.smem, ax->aux>>>(pl.emap, pl.p);
      rc = check_launch("premix_t_kernel (grouped)");
    } else {
      dc::PremixLaunch pl;
      rc = dc::plan_premix(E + c0 * taps_cin, alpha + b0 * d->n, static_cast<__nv_bfloat16*>(wsl),
                           s.B, d->n, wg, st->err, g_wait_ns.load(), mix_sms, g_encode, &pl,
                           static_cast<long long>(wsize), g_premix_direct.load() != 0);
      if (rc == -2) {
        std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(grouped premix) failed");
        return DYNCONV_ERR_CUDA;
      }
      if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
      const auto pk = dc::premix_kernel_for(pl.p.rep);
      e = ensure_smem(pk, pl.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix)");
      pk<<<pl.grid, dc::kPmThreads, pl.smem, ax->aux>>>(pl.emap, pl.p);
      rc = check_launch("premix_kernel (grouped)");
    }
    if (rc) return rc;
    e = cudaEventRecord(ax->mixed[slot], ax->aux);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(stream, ax->mixed[slot], 0);
    if (e != cudaSuccess) return cuda_fail(e, "grouped mixing: mixed edge");
    // ---- convolution of group g on the caller's stream
    TcPlan& pp = plans[g];
    const size_t xoff = b0 * d->H * d->W * d->C_in;
    const size_t yoff = b0 * d->H * d->W * d->C_out;
    pp.p.experts = E;
    pp.p.alpha = alpha + b0 * d->n;
    pp.p.bias = bias;
    pp.p.y = static_cast<__nv_bfloat16*>(y) + yoff;
    pp.p.err = st->err;
    pp.p.wait_ns = g_wait_ns.load();
    pp.p.a_out = a_out ? a_out + b0 * d->C_out : nullptr;
    pp.p.chan_add = chan_add ? chan_add + b0 * d->C_out : nullptr;
    pp.p.chan_scale = chan_scale;
    pp.p.co_base = static_cast<int>(c0);
    pp.p.ld_c = d->C_out;
    CUtensorMap xmap, wmap;
    rc = encode_x_map(&xmap, static_cast<const __nv_bfloat16*>(x) + xoff, &s, pp.p.Wp,
                      pp.p.b_box_rows);
    if (rc) return rc;
    rc = encode_w_map(&wmap, wsl, &s);
    if (rc) return rc;
    e = ensure_smem(dc::tc_conv_persist_kernel, pp.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc_conv_persist)");
    e = launch_pdl(dc::tc_conv_persist_kernel, dim3(pp.grid), dim3(dc::kTcThreads), pp.smem,
                   stream, xmap, wmap, pp.p);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      return cuda_fail(e, "tc_conv_persist_kernel launch (grouped)");
    }
    rc = check_launch("tc_conv_persist_kernel (grouped)");
    if (rc) return rc;
    e = cudaEventRecord(ax->used[slot], stream);
    if (e != cudaSuccess) return cuda_fail(e, "grouped mixing: slot release");
  }
  return DYNCONV_OK;
}

// The grouped PREMIX form in sequence on the caller's stream: for each group
// the mixing kernel (all SMs) writes the group's mixed kernels into one
// workspace slot, then the convolution (all SMs) reads them back -- from L2,
// since the slot (tens of MB) is far smaller than the L2 and was just
// written. No internal stream: every launch carries a programmatic edge, and
// the convolution never signals its dependents early, so the next group's
// mixing reads and overwrites the slot only once the convolution has
// completed.
int run_grouped_seq(const dynconv_desc* d, const GroupPlan& gp, const DeviceState* st,
                    const void* x, const void* experts, const float* alpha, const float* bias,
                    void* y, void* ws, const float* a_out, const float* chan_add,
                    float chan_scale, cudaStream_t stream) {
  const size_t taps_cin = static_cast<size_t>(d->KH) * d->KW * d->C_in;
  const size_t wsize = d->C_out * taps_cin;
  std::vector<TcPlan> plans(gp.groups);
  std::vector<dynconv_desc> subs(gp.groups);
  for (int g = 0; g < gp.groups; ++g) {
    dynconv_desc s = *d;
    if (gp.kind == 1) s.B = std::min(gp.per, d->B - g * gp.per);
    else s.C_out = std::min(gp.per, d->C_out - g * gp.per);
    subs[g] = s;
    // channel groups write into y at a channel offset: only the persistent
    // kernel takes one
    const bool ok = gp.kind == 2 ? tc_plan_persist(&s, st->sms, st->max_smem_optin, &plans[g])
                                 : tc_plan(&s, DYNCONV_VARIANT_PREMIX, st->sms, st->max_smem_optin,
                                           &plans[g]);
    if (!ok) return DYNCONV_ERR_UNSUPPORTED;
  }
  const __nv_bfloat16* E = static_cast<const __nv_bfloat16*>(experts);
  int rc = DYNCONV_OK;
  for (int g = 0; g < gp.groups; ++g) {
    const dynconv_desc& s = subs[g];
    const size_t b0 = gp.kind == 1 ? static_cast<size_t>(g) * gp.per : 0;
    const size_t c0 = gp.kind == 2 ? static_cast<size_t>(g) * gp.per : 0;
    const long long wg = static_cast<long long>(s.C_out) * static_cast<long long>(taps_cin);
    cudaError_t e;
    if (g_premix_mixer.load() == 3 && s.B <= 256) {
      dc::PremixTLaunch pl;
      rc = dc::plan_premix_t(E + c0 * taps_cin, static_cast<long long>(wsize), alpha + b0 * d->n,
                             static_cast<__nv_bfloat16*>(ws), s.B, d->n, wg, st->err,
                             g_wait_ns.load(), st->sms, g_encode, &pl);
      if (rc == -2) {
        std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(grouped premix) failed");
        return DYNCONV_ERR_CUDA;
      }
      if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
      e = ensure_smem(dc::premix_t_kernel, pl.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix_t)");
      e = launch_pdl(dc::premix_t_kernel, dim3(pl.grid), dim3(dc::kPtThreads), pl.smem, stream,
                     pl.emap, pl.p);
      if (e != cudaSuccess) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cuda_fail(e, "premix_t_kernel launch (grouped)");
      }
      rc = check_launch("premix_t_kernel (grouped)");
    } else {
      dc::PremixLaunch pl;
      rc = dc::plan_premix(E + c0 * taps_cin, alpha + b0 * d->n, static_cast<__nv_bfloat16*>(ws),
                           s.B, d->n, wg, st->err, g_wait_ns.load(), st->sms, g_encode, &pl,
                           static_cast<long long>(wsize), g_premix_direct.load() != 0);
      if (rc == -2) {
        std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(grouped premix) failed");
        return DYNCONV_ERR_CUDA;
      }
      if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
      const auto pk = dc::premix_kernel_for(pl.p.rep);
      e = ensure_smem(pk, pl.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix)");
      e = launch_pdl(pk, dim3(pl.grid), dim3(dc::kPmThreads), pl.smem, stream,
                     pl.emap, pl.p);
      if (e != cudaSuccess) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cuda_fail(e, "premix_kernel launch (grouped)");
      }
      rc = check_launch("premix_kernel (grouped)");
    }
    if (rc) return rc;
    TcPlan& pp = plans[g];
    const size_t xoff = b0 * d->H * d->W * d->C_in;
    const size_t yoff = b0 * d->H * d->W * d->C_out;
    pp.p.experts = E;
    pp.p.alpha = alpha + b0 * d->n;
    pp.p.bias = bias;
    pp.p.y = static_cast<__nv_bfloat16*>(y) + yoff;
    pp.p.err = st->err;
    pp.p.wait_ns = g_wait_ns.load();
    pp.p.a_out = a_out ? a_out + b0 * d->C_out : nullptr;
    pp.p.chan_add = chan_add ? chan_add + b0 * d->C_out : nullptr;
    pp.p.chan_scale = chan_scale;
    CUtensorMap xmap, wmap;
    rc = encode_x_map(&xmap, static_cast<const __nv_bfloat16*>(x) + xoff, &s, pp.p.Wp,
                      pp.p.b_box_rows);
    if (rc) return rc;
    rc = encode_w_map(&wmap, ws, &s);
    if (rc) return rc;
    if (gp.kind == 1) {
      rc = launch_premix_conv(&s, pp, st, static_cast<const __nv_bfloat16*>(x) + xoff, xmap, wmap,
                              stream);
    } else {
      pp.p.co_base = static_cast<int>(c0);
      pp.p.ld_c = d->C_out;
      pp.p.x_early = g_use_pdl.load() ? 1 : 0;
      e = ensure_smem(dc::tc_conv_persist_kernel, pp.smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(tc_conv_persist)");
      e = launch_pdl(dc::tc_conv_persist_kernel, dim3(pp.grid), dim3(dc::kTcThreads), pp.smem,
                     stream, xmap, wmap, pp.p);
      if (e != cudaSuccess) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cuda_fail(e, "tc_conv_persist_kernel launch (grouped)");
      }
      rc = check_launch("tc_conv_persist_kernel (grouped)");
    }
    if (rc) return rc;
  }
  return DYNCONV_OK;
}

// State slot of the streamed mixing for (device, stream): launches on one
// stream are ordered, so they may share a slot; every stream gets a slot of
// its own, kept for the life of the process. When all kMcSlots slots of the
// device belong to other streams, a slot is never taken from one of them (its
// kernel may still be running on those counters): the call returns
// DYNCONV_ERR_UNSUPPORTED and the caller runs the two-kernel PREMIX form.
std::mutex g_slot_mu;
std::map<std::pair<int, void*>, int> g_slot_of;
bool g_slots_dirty[64] = {};  // per device: a bounded wait expired, zero all slots

int mix_state_slot(void* stream, unsigned int** out, cudaStream_t s) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  void* base = nullptr;
  e = cudaGetSymbolAddress(&base, g_mix_state);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(mixing state)");
  std::lock_guard<std::mutex> lk(g_slot_mu);
  if (dev >= 0 && dev < 64 && g_slots_dirty[dev]) {
    e = cudaMemsetAsync(base, 0, sizeof(g_mix_state), s);
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(mixing state)");
    g_slots_dirty[dev] = false;
  }
  const auto key = std::make_pair(dev, stream);
  auto it = g_slot_of.find(key);
  int slot = -1;
  if (it != g_slot_of.end()) {
    slot = it->second;
  } else {
    bool used[dc::kMcSlots] = {};
    for (auto jt = g_slot_of.begin(); jt != g_slot_of.end(); ++jt)
      if (jt->first.first == dev) used[jt->second] = true;
    for (int i = 0; i < dc::kMcSlots && slot < 0; ++i)
      if (!used[i]) slot = i;
    if (slot < 0) return DYNCONV_ERR_UNSUPPORTED;  // every slot belongs to another stream
    g_slot_of[key] = slot;
  }
  *out = static_cast<unsigned int*>(base) + static_cast<size_t>(slot) * dc::kMcStateWords;
  return DYNCONV_OK;
}

// PREMIX with the mixing streamed into the convolution (one persistent
// cooperative kernel, n <= 8). Returns DYNCONV_ERR_UNSUPPORTED (and launches
// nothing) when the shape is outside it.
int run_mixconv(const dynconv_desc* d, const TcPlan& plan_in, const DeviceState* st,
                const void* experts, const float* alpha, const float* bias, void* y, void* ws,
                const CUtensorMap& xmap, const CUtensorMap& wmap, cudaStream_t stream) {
  if (d->n > dc::kMcMaxExperts || plan_in.p.k_steps > dc::kMcMaxSlices) return DYNCONV_ERR_UNSUPPORTED;
  if (static_cast<size_t>(d->B) * d->n * 4 > 16384 || d->C_in % 8 != 0) return DYNCONV_ERR_UNSUPPORTED;
  if (!aligned16(experts)) return DYNCONV_ERR_UNSUPPORTED;
  dc::MixParams mp{};
  mp.cv = plan_in.p;
  mp.wsize = static_cast<long long>(d->C_out) * d->KH * d->KW * d->C_in;
  // items: 8 weights x up to 16 samples; fewer samples per item when a whole
  // grid of mixer threads would otherwise get less than one item
  const long long threads = static_cast<long long>(st->sms) * 256;
  int sblock = 16;
  while (sblock > 1 &&
         1LL * mp.cv.k_steps * ((d->B + sblock - 1) / sblock) * d->C_out * 8 < threads)
    sblock >>= 1;
  sblock = std::min(sblock, d->B);
  mp.sblock = sblock;
  mp.nsb = (d->B + sblock - 1) / sblock;
  mp.ips = mp.nsb * d->C_out * 8;
  mp.total_items = 1LL * mp.cv.k_steps * mp.ips;
  mp.units = plan_in.grid;
  // shared memory from the 1024-aligned base: A stages | B stages | epilogue
  // staging | alpha | barriers
  const size_t b_bytes = static_cast<size_t>(mp.cv.sb) * mp.cv.b_tile_bytes;
  const size_t alpha_bytes = (static_cast<size_t>(d->B) * d->n * 4 + 15) & ~size_t(15);
  size_t total = 0;
  int sa = 8;
  for (; sa >= 2; --sa) {
    const size_t bar_off = static_cast<size_t>(sa) * dc::kTcATileBytes + b_bytes + dc::kMcEpiStage + alpha_bytes;
    total = 1024 + bar_off + 8 * (2 * sa + 2 * mp.cv.sb + 3) + 16;
    if (total <= static_cast<size_t>(st->max_smem_optin)) break;
  }
  if (sa < 2) return DYNCONV_ERR_UNSUPPORTED;
  mp.cv.sa = sa;
  mp.stage_off = static_cast<int>(static_cast<size_t>(sa) * dc::kTcATileBytes + b_bytes);
  mp.alpha_off = mp.stage_off + dc::kMcEpiStage;
  mp.bar_off = static_cast<int>(mp.alpha_off + alpha_bytes);
  mp.cv.experts = static_cast<const __nv_bfloat16*>(experts);
  mp.cv.alpha = alpha;
  mp.cv.bias = bias;
  mp.cv.y = static_cast<__nv_bfloat16*>(y);
  mp.cv.err = st->err;
  mp.cv.wait_ns = g_wait_ns.load();
  mp.wb = static_cast<__nv_bfloat16*>(ws);
  int rc = mix_state_slot(static_cast<void*>(stream), &mp.state, stream);
  if (rc) return rc;  // UNSUPPORTED when no slot is free: the two-kernel form runs
  cudaError_t e = cudaSuccess;
  auto kern = d->n <= 2 ? dc::mixconv_kernel<2>
              : d->n <= 4 ? dc::mixconv_kernel<4> : dc::mixconv_kernel<8>;
  e = ensure_smem(kern, total);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(mixconv)");
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(st->sms);
  cfg.blockDim = dim3(dc::kMcThreads);
  cfg.dynamicSmemBytes = total;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_use_pdl.load() ? 2 : 1;
  e = cudaLaunchKernelEx(&cfg, kern, xmap, wmap, mp);
  if (e != cudaSuccess && cfg.numAttrs == 2) {
    // a cooperative launch that does not take the programmatic edge: plain order
    (void)cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, kern, xmap, wmap, mp);
  }
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_fail(e, "mixconv_kernel launch");
  }
  return check_launch("mixconv_kernel");
}

int run_tc(const dynconv_desc* d, int variant, const DeviceState* st, const void* x,
           const void* experts, const float* alpha, const float* bias, void* y, void* ws,
           size_t ws_bytes, cudaStream_t stream, float* ysum = nullptr,
           const float* a_in = nullptr, const float* a_out = nullptr,
           const float* chan_add = nullptr, float chan_scale = 0.f) {
  // input attention is folded into the mixed kernel: only the PREMIX variant
  // with the CUDA-core mixer takes it
  if (a_in != nullptr && variant != DYNCONV_VARIANT_PREMIX) return DYNCONV_ERR_UNSUPPORTED;
  TcPlan plan;
  if (!tc_plan(d, variant, st->sms, st->max_smem_optin, &plan)) return DYNCONV_ERR_UNSUPPORTED;
  plan.p.ysum = ysum;
  plan.p.a_out = a_out;
  plan.p.chan_add = chan_add;
  plan.p.chan_scale = chan_scale;
  plan.p.experts = static_cast<const __nv_bfloat16*>(experts);
  plan.p.alpha = alpha;
  plan.p.bias = bias;
  plan.p.y = static_cast<__nv_bfloat16*>(y);
  plan.p.err = st->err;
  plan.p.wait_ns = g_wait_ns.load();
  plan.p.inject_skip = g_inject_skip.exchange(0);
  plan.p.stamps = reinterpret_cast<unsigned long long*>(g_conv_stamps.load());
  CUtensorMap xmap, wmap;
  std::memset(&wmap, 0, sizeof(wmap));
  int rc = encode_x_map(&xmap, x, d, plan.p.Wp, plan.p.b_box_rows);
  if (rc) return rc;
  if (variant == DYNCONV_VARIANT_FUSED || variant == DYNCONV_VARIANT_OUTSIDE) {
    // the experts as n "samples" of the mixed-kernel layout: tiles {64 ci, 1 tap, 128 co}
    if (!aligned16(experts)) return DYNCONV_ERR_MISALIGNED;
    dynconv_desc de = *d;
    de.B = d->n;
    rc = encode_w_map(&wmap, experts, &de);
    if (rc) return rc;
    return variant == DYNCONV_VARIANT_FUSED ? launch_tc<dc::kFused>(plan, xmap, wmap, stream)
                                            : launch_tc<dc::kOutside>(plan, xmap, wmap, stream);
  }
  // PREMIX: mix every sample's kernel into the workspace, then convolve from it
  const size_t need = premix_workspace(d);
  if (need == 0) return DYNCONV_ERR_UNSUPPORTED;
  if (!ws || ws_bytes < need) return DYNCONV_ERR_WORKSPACE;
  if (!aligned16(ws)) return DYNCONV_ERR_MISALIGNED;
  plan.p.inject_skip = 0;
  if (g_stream_mix.load() && g_premix_mixer.load() != 1 && d->n <= dc::kMcMaxExperts &&
      ysum == nullptr && a_in == nullptr && a_out == nullptr && chan_add == nullptr) {
    rc = encode_w_map(&wmap, ws, d);
    if (rc) return rc;
    rc = run_mixconv(d, plan, st, experts, alpha, bias, y, ws, xmap, wmap, stream);
    if (rc != DYNCONV_ERR_UNSUPPORTED) return rc;
  }
  // large B*|W| with the tensor-core mixer: the grouped pipeline through L2
  if (g_group_mix.load() && ysum == nullptr && a_in == nullptr && g_premix_mixer.load() != 2) {
    const GroupPlan gp = group_plan(d);
    const bool seq = g_group_mix.load() == 2;
    if (gp.kind != 0 && ws_bytes >= (seq ? 1 : 2) * gp.slot &&
        (reinterpret_cast<uintptr_t>(ws) & 255u) == 0) {
      rc = seq ? run_grouped_seq(d, gp, st, x, experts, alpha, bias, y, ws, a_out, chan_add,
                                 chan_scale, stream)
               : run_grouped(d, gp, st, x, experts, alpha, bias, y, ws, a_out, chan_add,
                             chan_scale, stream);
      if (rc != DYNCONV_ERR_UNSUPPORTED) return rc;
    }
  }
  // few experts: the store-bound CUDA-core mixer (no set-up chain)
  if (g_premix_mixer.load() != 1) {
    dc::PsParams ps;
    unsigned grid = 0;
    if (dc::plan_premix_small(d->B, d->n,
                              static_cast<long long>(d->C_out) * d->KH * d->KW * d->C_in, st->sms,
                              &ps, &grid) &&
        aligned16(experts)) {
      ps.experts = static_cast<const __nv_bfloat16*>(experts);
      ps.alpha = alpha;
      ps.out = static_cast<__nv_bfloat16*>(ws);
      ps.a_in = a_in;
      ps.Cin = d->C_in;
      ps.stamps = g_conv_stamps.load() ? reinterpret_cast<unsigned long long*>(g_conv_stamps.load()) +
                                             4096 * 8 : nullptr;  // after the convolution's
      size_t smem = sizeof(float) * static_cast<size_t>(d->B) * d->n;
      if (a_in != nullptr) smem += sizeof(float) * static_cast<size_t>(d->B) * d->C_in;
      if (smem > static_cast<size_t>(st->max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
      auto kern = d->n <= 2 ? dc::premix_small_kernel<2>
                  : d->n <= 4 ? dc::premix_small_kernel<4> : dc::premix_small_kernel<8>;
      cudaError_t e = cudaSuccess;
      if (smem > 48 * 1024) e = ensure_smem(kern, smem);
      if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix_small)");
      e = launch_pdl(kern, dim3(grid), dim3(dc::kPsThreads), smem, stream, ps);
      if (e != cudaSuccess) {
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cuda_fail(e, "premix_small_kernel launch");
      }
      rc = check_launch("premix_small_kernel");
      if (rc) return rc;
      rc = encode_w_map(&wmap, ws, d);
      if (rc) return rc;
      return launch_premix_conv(d, plan, st, x, xmap, wmap, stream);
    }
    if (g_premix_mixer.load() == 2) return DYNCONV_ERR_UNSUPPORTED;
  }
  if (a_in != nullptr) return DYNCONV_ERR_UNSUPPORTED;  // the GEMM mixer does not take it
  const long long wsize_all = static_cast<long long>(d->C_out) * d->KH * d->KW * d->C_in;
  const int mixer = g_premix_mixer.load();
  if ((mixer == 3 && d->B <= 256) || (mixer == 0 && d->B <= kTransposedMixMax)) {
    // the transposed mixing GEMM (M = weights, N = samples) over the whole batch
    dc::PremixTLaunch tl;
    rc = dc::plan_premix_t(static_cast<const __nv_bfloat16*>(experts), wsize_all, alpha,
                           static_cast<__nv_bfloat16*>(ws), d->B, d->n, wsize_all, st->err,
                           g_wait_ns.load(), st->sms, g_encode, &tl);
    if (rc == -2) {
      std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(premix_t) failed");
      return DYNCONV_ERR_CUDA;
    }
    if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
    cudaError_t e = ensure_smem(dc::premix_t_kernel, tl.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix_t)");
    e = launch_pdl(dc::premix_t_kernel, dim3(tl.grid), dim3(dc::kPtThreads), tl.smem, stream,
                   tl.emap, tl.p);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      return cuda_fail(e, "premix_t_kernel launch");
    }
    rc = check_launch("premix_t_kernel");
    if (rc) return rc;
    rc = encode_w_map(&wmap, ws, d);
    if (rc) return rc;
    return launch_premix_conv(d, plan, st, x, xmap, wmap, stream);
  }
  dc::PremixLaunch pl;
  // tile counter after the mixed kernels, zeroed on the stream before the launch
  // (when the expert bank streams from HBM, the CTAs' expert reads arrive at
  // uneven rates; from L2 they do not, and the counter's memset would only
  // cost the launch its programmatic overlap with the routing kernel)
  const double expert_bytes = 2.0 * d->n * d->C_out * d->KH * d->KW * d->C_in;
  const int dyn = g_premix_dyn.load();
  unsigned int* tile_ctr =
      (dyn == 2 || (dyn == 1 && expert_bytes > 0.5 * st->l2_bytes))
          ? reinterpret_cast<unsigned int*>(static_cast<char*>(ws) + premix_wb_bytes(d))
          : nullptr;
  rc = dc::plan_premix(static_cast<const __nv_bfloat16*>(experts), alpha,
                       static_cast<__nv_bfloat16*>(ws), d->B, d->n,
                       static_cast<long long>(d->C_out) * d->KH * d->KW * d->C_in, st->err,
                       g_wait_ns.load(), st->sms, g_encode, &pl, 0, g_premix_direct.load() != 0,
                       tile_ctr);
  if (rc == -2) {
    std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(premix) failed");
    return DYNCONV_ERR_CUDA;
  }
  if (rc != 0) return DYNCONV_ERR_UNSUPPORTED;
  {
    const auto pk = dc::premix_kernel_for(pl.p.rep);
    cudaError_t e = ensure_smem(pk, pl.smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(premix)");
    if (tile_ctr != nullptr) {
      e = cudaMemsetAsync(tile_ctr, 0, sizeof(unsigned int), stream);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(premix tile counter)");
    }
    e = launch_pdl(pk, dim3(pl.grid), dim3(dc::kPmThreads), pl.smem, stream,
                   pl.emap, pl.p);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      return cuda_fail(e, "premix_kernel launch");
    }
    rc = check_launch("premix_kernel");
    if (rc) return rc;
  }
  rc = encode_w_map(&wmap, ws, d);
  if (rc) return rc;
  return launch_premix_conv(d, plan, st, x, xmap, wmap, stream);
}

}  // namespace

// ====================================================================== C ABI

extern "C" {

const char* dynconv_status_string(int status) {
  switch (status) {
    case DYNCONV_OK: return "ok";
    case DYNCONV_ERR_INVALID_ARG: return "invalid argument";
    case DYNCONV_ERR_UNSUPPORTED: return "unsupported shape or variant";
    case DYNCONV_ERR_MISALIGNED: return "pointer not 16-byte aligned";
    case DYNCONV_ERR_CUDA: return "CUDA error";
    case DYNCONV_ERR_TIMEOUT: return "a kernel's bounded wait expired";
    case DYNCONV_ERR_WORKSPACE: return "workspace too small for the requested variant";
    default: return "unknown status";
  }
}

const char* dynconv_last_error(void) { return g_last_err; }

unsigned long long dynconv_launch_count(void) { return g_launches.load(); }

int dynconv_test_hook(int key, long long value) {
  if (key == 1) {
    if (value < 0) return DYNCONV_ERR_INVALID_ARG;
    g_wait_ns.store(value == 0 ? kDefaultWaitNs : value * 1000LL);
    return DYNCONV_OK;
  }
  if (key == 2) {
    g_inject_skip.store(value != 0 ? 1 : 0);
    return DYNCONV_OK;
  }
  if (key == 4) {
    if (value < 0 || value > 8) return DYNCONV_ERR_INVALID_ARG;
    g_route_split.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 5) {
    if (value != 0 && value != 1) return DYNCONV_ERR_INVALID_ARG;
    g_use_pdl.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 6) {
    if (value != 0 && value != 1) return DYNCONV_ERR_INVALID_ARG;
    g_stream_mix.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 7) {
    if (value < 0 || value > 3) return DYNCONV_ERR_INVALID_ARG;
    g_premix_mixer.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 3) {
    if (value != 0 && value != 1) return DYNCONV_ERR_INVALID_ARG;
    g_desc_base_mode = static_cast<int>(value);
    return DYNCONV_OK;
  }
  if (key == 8) {
    if (value < 0 || value > 3) return DYNCONV_ERR_INVALID_ARG;
    g_dw_kernel.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 9) {
    if (value < 0 || value > 2) return DYNCONV_ERR_INVALID_ARG;
    g_conv_persist.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 11) {
    if (value != 0 && value != 1) return DYNCONV_ERR_INVALID_ARG;
    g_mixgrad_tc.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 13) {
    // a device buffer of at least grid * 8 64-bit words (0: off)
    g_conv_stamps.store(static_cast<unsigned long long>(value));
    return DYNCONV_OK;
  }
  if (key == 18) {
    if (value < 0 || value > 2) return DYNCONV_ERR_INVALID_ARG;
    g_premix_dyn.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 14) {
    if (value < 0 || value > 256) return DYNCONV_ERR_INVALID_ARG;
    g_persist_rows.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 12) {
    if (value != 0 && value != 1) return DYNCONV_ERR_INVALID_ARG;
    g_premix_direct.store(static_cast<int>(value));
    return DYNCONV_OK;
  }
  if (key == 10) {
    // 0 off, 1 concurrent groups, 2 sequential groups; >= 4096: concurrent
    // groups of about that many bytes at every size; a negative value <= -4096:
    // sequential groups of about -value bytes at every size
    if (value > 2 && value < 4096) return DYNCONV_ERR_INVALID_ARG;
    if (value < 0 && value > -4096) return DYNCONV_ERR_INVALID_ARG;
    const long long bytes = value >= 4096 ? value : value <= -4096 ? -value : 0;
    g_group_mix.store(value == 0 ? 0 : (value == 2 || value <= -4096) ? 2 : 1);
    g_group_bytes.store(bytes ? bytes : (40LL << 20));
    g_group_min.store(bytes ? 0 : (64LL << 20));
    return DYNCONV_OK;
  }
  return DYNCONV_ERR_INVALID_ARG;
}

size_t dynconv_workspace_size(const dynconv_desc* desc) {
  if (validate_desc(desc) != DYNCONV_OK) return 0;
  return premix_workspace(desc);
}

int dynconv_select_variant(const dynconv_desc* desc, size_t workspace_bytes) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (desc->variant != DYNCONV_VARIANT_AUTO) return desc->variant;
  // 148 SMs and 227 KB of opt-in shared memory per CTA: the B200 figures, so
  // that the choice is available without a device.
  return select_variant(desc, workspace_bytes, 148, 232448);
}

int dynconv_route(const dynconv_desc* desc, const void* x, const float* Wr, const float* br,
                  int mode, float tau, float* alpha, void* stream) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!x || !Wr || !alpha) return DYNCONV_ERR_INVALID_ARG;
  if (mode != DYNCONV_SIGMOID && mode != DYNCONV_SOFTMAX) return DYNCONV_ERR_INVALID_ARG;
  if (mode == DYNCONV_SOFTMAX && !(tau > 0.f)) return DYNCONV_ERR_INVALID_ARG;
  if (desc->n > 1024 || desc->C_in > 16384) return DYNCONV_ERR_UNSUPPORTED;
  if (desc->B == 0) return DYNCONV_OK;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc) return rc;

  const int C = desc->C_in;
  const size_t eb = elem_bytes(desc);
  const bool vec = aligned16(x) && (C * eb) % 16 == 0;
  const int VEC = vec ? static_cast<int>(16 / eb) : 1;
  const int HW = desc->H * desc->W;
  // about two CTAs per SM in one wave, at most 8 per sample (portable cluster)
  int nsplit = (2 * st->sms) / std::max(desc->B, 1);
  if (g_route_split.load() > 0) nsplit = g_route_split.load();
  nsplit = std::max(1, std::min({nsplit, 8, HW}));
  // bulk staging of each CTA's contiguous pixel slice when a pixel row is a
  // 16-byte multiple and one channel vector per thread covers it; pieces of at
  // most 48 KB, balanced
  const size_t row_bytes = static_cast<size_t>(C) * eb;
  int piece_px = 0;
  if (vec && C / VEC <= dc::kRouteThreads) {
    const int slice_px = (HW + nsplit - 1) / nsplit;
    int per = static_cast<int>(std::max<size_t>(1, dc::kRoutePieceBytes / row_bytes));
    per = std::min(per, slice_px);
    const int pieces = (slice_px + per - 1) / per;
    piece_px = (slice_px + pieces - 1) / pieces;
  }
  const size_t wr_bytes = static_cast<size_t>(desc->n) * C * 4;
  const int wr_smem = (wr_bytes <= dc::kRouteWrSmemBytes && wr_bytes % 16 == 0 && aligned16(Wr)) ? 1 : 0;
  size_t smem = dc::route_smem(C, desc->n, VEC, static_cast<int>(eb), nsplit, piece_px, wr_smem,
                               piece_px > 0).total;
  // very wide rows without staged Wr: fewer ranks (rank 0 receives nsplit x C sums)
  while (smem > static_cast<size_t>(st->max_smem_optin) && nsplit > 1) {
    --nsplit;
    smem = dc::route_smem(C, desc->n, VEC, static_cast<int>(eb), nsplit, piece_px, wr_smem,
                          piece_px > 0).total;
  }
  if (smem > static_cast<size_t>(st->max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;

  dc::RouteParams p{desc->B, C, HW, desc->n, mode, tau, x, Wr, br, alpha,
                    nsplit, piece_px, wr_smem, st->err, g_wait_ns.load(),
                    reinterpret_cast<unsigned long long*>(g_conv_stamps.load())};
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nsplit, desc->B, 1);
  cfg.blockDim = dim3(dc::kRouteThreads, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = nsplit;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = g_use_pdl.load() ? 2 : 1;

  cudaError_t e;
  auto launch = [&](auto kern) {
    if (smem > 48 * 1024) {
      cudaError_t ea = ensure_smem(kern, smem);
      if (ea != cudaSuccess) return ea;
    }
    return cudaLaunchKernelEx(&cfg, kern, p);
  };
  if (desc->dtype == DYNCONV_BF16)
    e = vec ? launch(dc::route_kernel<__nv_bfloat16, 8>) : launch(dc::route_kernel<__nv_bfloat16, 1>);
  else
    e = vec ? launch(dc::route_kernel<float, 4>) : launch(dc::route_kernel<float, 1>);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_fail(e, "route_kernel launch");
  }
  return check_launch("route_kernel");
}

}  // extern "C"

namespace {

// The channel sums of y in a second pass (one partial per sample), for the
// CUDA-core forward kernels.
int pool_pass(const dynconv_desc* d, const void* y, float* ysum, cudaStream_t s) {
  const int Ho = out_size(d->H, d->KH, d->stride, d->pad);
  const int Wo = out_size(d->W, d->KW, d->stride, d->pad);
  cudaError_t e;
  if (d->dtype == DYNCONV_F32)
    e = launch_pdl(dc::pool_sum_kernel<float>, dim3(d->B), dim3(dc::kPoolThreads), 0, s,
                   static_cast<const float*>(y), Ho * Wo, d->C_out, ysum);
  else
    e = launch_pdl(dc::pool_sum_kernel<__nv_bfloat16>, dim3(d->B), dim3(dc::kPoolThreads), 0, s,
                   static_cast<const __nv_bfloat16*>(y), Ho * Wo, d->C_out, ysum);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_fail(e, "pool_sum_kernel launch");
  }
  return check_launch("pool_sum_kernel");
}

// The pipelined depthwise kernel; DYNCONV_ERR_UNSUPPORTED (nothing launched)
// when the shape does not fit its plan.
int run_depthwise_pipe(const dynconv_desc* d, const DeviceState* st, const void* x,
                       const void* experts, const float* alpha, const float* bias, void* y,
                       const float* a_in, const float* a_out, const float* chan_add,
                       float chan_scale, cudaStream_t s) {
  dc::DwpParams p;
  int grid = 0;
  size_t smem = 0;
  const int hook = g_dw_kernel.load();
  const int nc = hook == 3 ? 4 : hook == 2 ? 2 : kDwpDefaultNc;
  if (!dwp_plan(d, st->sms, st->max_smem_optin, bias != nullptr, nc, &p, &grid, &smem))
    return DYNCONV_ERR_UNSUPPORTED;
  const int K = d->KH;
  p.experts = static_cast<const __nv_bfloat16*>(experts);
  p.alpha = alpha;
  p.bias = bias;
  p.y = static_cast<__nv_bfloat16*>(y);
  p.a_in = a_in;
  p.a_out = a_out;
  p.chan_add = chan_add;
  p.chan_scale = chan_scale;
  p.err = st->err;
  p.wait_ns = g_wait_ns.load();
  p.stamps = reinterpret_cast<unsigned long long*>(g_conv_stamps.load());
  CUtensorMap xmap;
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(d->C_in), static_cast<cuuint64_t>(d->W),
                              static_cast<cuuint64_t>(d->H), static_cast<cuuint64_t>(d->B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(d->C_in) * 2,
                                 static_cast<cuuint64_t>(d->W) * d->C_in * 2,
                                 static_cast<cuuint64_t>(d->H) * d->W * d->C_in * 2};
  const cuuint32_t box[4] = {static_cast<cuuint32_t>(p.CC),
                             static_cast<cuuint32_t>((p.CB + nc - 1) / nc * nc + K - 1),
                             static_cast<cuuint32_t>(p.RB + K - 1), 1u};
  const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  if (g_encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides,
               box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
    std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(depthwise pipe) failed");
    return DYNCONV_ERR_CUDA;
  }
  auto go = [&](auto kern, int threads) -> int {
    cudaFuncAttributes fa;
    cudaError_t e = cudaFuncGetAttributes(&fa, kern);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncGetAttributes(depthwise pipe)");
    if (fa.maxThreadsPerBlock < threads) return DYNCONV_ERR_UNSUPPORTED;  // the per-tile kernel runs
    e = ensure_smem(kern, smem);
    if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(depthwise pipe)");
    e = launch_pdl(kern, dim3(grid), dim3(threads), smem, s, xmap, p);
    if (e != cudaSuccess) {
      g_launches.fetch_add(1, std::memory_order_relaxed);
      char what[160];
      std::snprintf(what, sizeof(what),
                    "depthwise_pipe_kernel launch (grid %d, %d threads, %zu B shared, %d regs)",
                    grid, threads, smem, fa.numRegs);
      return cuda_fail(e, what);
    }
    return check_launch("depthwise_pipe_kernel");
  };
  // 32 channel pairs per chunk: the window's column stride is a compile-time constant
  const bool c32 = p.CC == 64;
  const int threads = p.ncomp + 32;
#define DC_DWP_GO(KV, NCV) \
  return c32 ? go(dc::depthwise_pipe_kernel<KV, 32, NCV>, threads) \
             : go(dc::depthwise_pipe_kernel<KV, 0, NCV>, threads)
  if (nc == 4) {
    if (K == 3) DC_DWP_GO(3, 4);
    if (K == 5) DC_DWP_GO(5, 4);
    DC_DWP_GO(7, 4);
  }
  if (K == 3) DC_DWP_GO(3, 2);
  if (K == 5) DC_DWP_GO(5, 2);
  DC_DWP_GO(7, 2);
#undef DC_DWP_GO
}

int resolve_variant(const dynconv_desc* desc, size_t ws_bytes, const DeviceState* st) {
  int variant = desc->variant;
  if (variant == DYNCONV_VARIANT_AUTO)
    variant = select_variant(desc, ws_bytes, st->sms, st->max_smem_optin);
  return variant;
}

int forward_impl(const dynconv_desc* desc, const void* x, const void* experts,
                 const float* alpha, const float* bias, void* y, void* workspace,
                 size_t workspace_bytes, void* stream, float* ysum,
                 const float* a_in = nullptr, const float* a_out = nullptr,
                 const float* chan_add = nullptr, float chan_scale = 0.f) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!x || !experts || !alpha || !y) return DYNCONV_ERR_INVALID_ARG;
  if (desc->B == 0) return DYNCONV_OK;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  int variant = resolve_variant(desc, workspace ? workspace_bytes : 0, st);
  if (a_in != nullptr && desc->variant == DYNCONV_VARIANT_AUTO &&
      (variant == DYNCONV_VARIANT_FUSED || variant == DYNCONV_VARIANT_OUTSIDE ||
       (variant == DYNCONV_VARIANT_PREMIX && desc->n > dc::kPsMaxExperts))) {
    // input attention needs the CUDA-core mixer (PREMIX, n <= 8) or a CUDA-core kernel
    const bool premix_ok = desc->n <= dc::kPsMaxExperts && workspace != nullptr &&
                           premix_workspace(desc) != 0 && workspace_bytes >= premix_workspace(desc);
    variant = premix_ok ? DYNCONV_VARIANT_PREMIX : DYNCONV_VARIANT_DIRECT;
  }

  switch (variant) {
    case DYNCONV_VARIANT_FUSED:
    case DYNCONV_VARIANT_OUTSIDE:
    case DYNCONV_VARIANT_PREMIX: {
      if (!tc_shape_ok(desc)) return DYNCONV_ERR_UNSUPPORTED;
      if (!aligned16(x) || !aligned16(experts) || !aligned16(y)) return DYNCONV_ERR_MISALIGNED;
      return run_tc(desc, variant, st, x, experts, alpha, bias, y, workspace, workspace_bytes, s,
                    ysum, a_in, a_out, chan_add, chan_scale);
    }
    case DYNCONV_VARIANT_DEPTHWISE: {
      if (!depthwise_ok(desc)) return DYNCONV_ERR_UNSUPPORTED;
      if (!aligned16(x) || !aligned16(y)) return DYNCONV_ERR_MISALIGNED;
      if (g_dw_kernel.load() != 1 && aligned16(experts) && (bias == nullptr || aligned16(bias))) {
        rc = run_depthwise_pipe(desc, st, x, experts, alpha, bias, y, a_in, a_out, chan_add,
                                chan_scale, s);
        if (rc != DYNCONV_ERR_UNSUPPORTED) {
          if (rc || ysum == nullptr) return rc;
          return pool_pass(desc, y, ysum, s);
        }
      }
      dc::DwParams p{};
      const int K = desc->KH;
      p.B = desc->B; p.C = desc->C_in; p.H = desc->H; p.W = desc->W; p.pad = desc->pad;
      p.n = desc->n;
      p.Ho = out_size(desc->H, K, 1, desc->pad);
      p.Wo = out_size(desc->W, K, 1, desc->pad);
      p.rows = std::min(p.Ho, dc::kDwMaxRows);
      p.cols = std::min(p.Wo, dc::kDwColsPerThread * dc::kDwMaxColThreads);
      p.col_threads = (p.cols + dc::kDwColsPerThread - 1) / dc::kDwColsPerThread;
      p.experts = static_cast<const __nv_bfloat16*>(experts);
      p.alpha = alpha;
      p.bias = bias;
      p.y = static_cast<__nv_bfloat16*>(y);
      p.err = st->err;
      p.wait_ns = g_wait_ns.load();
      p.a_in = a_in;
      p.a_out = a_out;
      p.chan_add = chan_add;
      p.chan_scale = chan_scale;
      const int TC = ((p.cols + 1) & ~1) + K - 1, TR = p.rows + K - 1;
      const size_t tile_bytes = static_cast<size_t>(TR) * TC * dc::kDwChunk * 2;
      const size_t smem = 128 + ((tile_bytes + 127) & ~size_t(127)) +
                          sizeof(float) * (dc::kDwChunk * K * K + dc::kDwChunk + p.n);
      if (smem > static_cast<size_t>(st->max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
      // activations {C, W, H, B}; one box = 32 channels of the zero-padded window
      CUtensorMap xmap;
      const cuuint64_t dims[4] = {static_cast<cuuint64_t>(desc->C_in), static_cast<cuuint64_t>(desc->W),
                                  static_cast<cuuint64_t>(desc->H), static_cast<cuuint64_t>(desc->B)};
      const cuuint64_t strides[3] = {static_cast<cuuint64_t>(desc->C_in) * 2,
                                     static_cast<cuuint64_t>(desc->W) * desc->C_in * 2,
                                     static_cast<cuuint64_t>(desc->H) * desc->W * desc->C_in * 2};
      const cuuint32_t box[4] = {static_cast<cuuint32_t>(dc::kDwChunk), static_cast<cuuint32_t>(TC),
                                 static_cast<cuuint32_t>(TR), 1u};
      const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
      if (g_encode(&xmap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(x), dims, strides,
                   box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS) {
        std::snprintf(g_last_err, sizeof(g_last_err), "cuTensorMapEncodeTiled(depthwise) failed");
        return DYNCONV_ERR_CUDA;
      }
      const int row_blocks = (p.Ho + p.rows - 1) / p.rows;
      const int col_blocks = (p.Wo + p.cols - 1) / p.cols;
      dim3 grid(row_blocks * col_blocks, (desc->C_in + dc::kDwChunk - 1) / dc::kDwChunk, desc->B);
      auto go = [&](auto kern) -> int {
        cudaError_t e = ensure_smem(kern, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(depthwise)");
        e = launch_pdl(kern, grid, dim3(dc::kDwThreads), smem, s, xmap, p);
        if (e != cudaSuccess) {
          g_launches.fetch_add(1, std::memory_order_relaxed);
          return cuda_fail(e, "depthwise_kernel launch");
        }
        return check_launch("depthwise_kernel");
      };
      rc = K == 3 ? go(dc::depthwise_kernel<3>)
           : K == 5 ? go(dc::depthwise_kernel<5>) : go(dc::depthwise_kernel<7>);
      if (rc || ysum == nullptr) return rc;
      return pool_pass(desc, y, ysum, s);
    }
    case DYNCONV_VARIANT_DIRECT: {
      const int Cg = desc->C_in / desc->groups;
      const long long wrow = 1LL * desc->KH * desc->KW * Cg;
      const long long budget = (st->max_smem_optin - 4LL * desc->n - 1024) / 4;
      long long cob = std::min<long long>(desc->C_out, 64);
      while (cob > 1 && cob * (wrow + 1) > budget) cob /= 2;
      if (cob * (wrow + 1) > budget) return DYNCONV_ERR_UNSUPPORTED;
      dc::DirectParams p{};
      p.B = desc->B; p.Cin = desc->C_in; p.H = desc->H; p.W = desc->W; p.Cout = desc->C_out;
      p.KH = desc->KH; p.KW = desc->KW; p.stride = desc->stride; p.pad = desc->pad;
      p.groups = desc->groups; p.n = desc->n;
      p.Ho = out_size(desc->H, desc->KH, desc->stride, desc->pad);
      p.Wo = out_size(desc->W, desc->KW, desc->stride, desc->pad);
      p.cob = static_cast<int>(cob);
      p.x = x; p.experts = experts; p.alpha = alpha; p.bias = bias; p.y = y;
      p.a_in = a_in; p.a_out = a_out;
      p.chan_add = chan_add; p.chan_scale = chan_scale;
      const size_t smem = sizeof(float) * (desc->n + cob + cob * wrow);
      dim3 grid((p.Ho * p.Wo + dc::kDirectPix - 1) / dc::kDirectPix,
                static_cast<unsigned>((desc->C_out + cob - 1) / cob), desc->B);
      auto go = [&](auto kern) -> int {
        cudaError_t e = ensure_smem(kern, smem);
        if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(direct)");
        e = launch_pdl(kern, grid, dim3(dc::kDirectThreads), smem, s, p);
        if (e != cudaSuccess) {
          g_launches.fetch_add(1, std::memory_order_relaxed);
          return cuda_fail(e, "direct_conv_kernel launch");
        }
        return check_launch("direct_conv_kernel");
      };
      rc = desc->dtype == DYNCONV_F32 ? go(dc::direct_conv_kernel<float>)
                                      : go(dc::direct_conv_kernel<__nv_bfloat16>);
      if (rc || ysum == nullptr) return rc;
      return pool_pass(desc, y, ysum, s);
    }
    default:
      return DYNCONV_ERR_INVALID_ARG;
  }
}

}  // namespace

extern "C" {

int dynconv_forward(const dynconv_desc* desc, const void* x, const void* experts,
                    const float* alpha, const float* bias, void* y, void* workspace,
                    size_t workspace_bytes, void* stream) {
  return forward_impl(desc, x, experts, alpha, bias, y, workspace, workspace_bytes, stream,
                      nullptr);
}

int dynconv_forward_attn(const dynconv_desc* desc, const void* x, const void* experts,
                         const float* alpha, const float* bias, const float* a_in,
                         const float* a_out, void* y, void* workspace, size_t workspace_bytes,
                         void* stream) {
  return forward_impl(desc, x, experts, alpha, bias, y, workspace, workspace_bytes, stream,
                      nullptr, a_in, a_out);
}

int dynconv_route_channels(const dynconv_desc* desc, const void* x, const float* Wi,
                           const float* bi, float* a_in, const float* Wo, const float* bo,
                           float* a_out, void* stream) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!x || (!Wi && !Wo) || (Wi && !a_in) || (Wo && !a_out)) return DYNCONV_ERR_INVALID_ARG;
  // each attention is the routing computation with one output per channel
  // and the sigmoid activation
  if (Wi) {
    dynconv_desc di = *desc;
    di.n = desc->C_in;
    rc = dynconv_route(&di, x, Wi, bi, DYNCONV_SIGMOID, 1.0f, a_in, stream);
    if (rc) return rc;
  }
  if (Wo) {
    dynconv_desc dout = *desc;
    dout.n = desc->C_out;
    rc = dynconv_route(&dout, x, Wo, bo, DYNCONV_SIGMOID, 1.0f, a_out, stream);
    if (rc) return rc;
  }
  return DYNCONV_OK;
}

int dynconv_forward_pooled(const dynconv_desc* desc, const void* x, const void* experts,
                           const float* alpha, const float* bias, void* y, float* ysum,
                           void* workspace, size_t workspace_bytes, void* stream) {
  if (!ysum) return DYNCONV_ERR_INVALID_ARG;
  return forward_impl(desc, x, experts, alpha, bias, y, workspace, workspace_bytes, stream, ysum);
}

int dynconv_pool_parts(const dynconv_desc* desc, size_t workspace_bytes) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  int sms = 148, max_smem = 232448;
  DeviceState* st = nullptr;
  if (device_state(&st) == DYNCONV_OK) {
    sms = st->sms;
    max_smem = st->max_smem_optin;
  }
  int variant = desc->variant;
  if (variant == DYNCONV_VARIANT_AUTO) variant = select_variant(desc, workspace_bytes, sms, max_smem);
  if (variant == DYNCONV_VARIANT_FUSED || variant == DYNCONV_VARIANT_OUTSIDE ||
      variant == DYNCONV_VARIANT_PREMIX) {
    TcPlan plan;
    if (!tc_plan(desc, variant, sms, max_smem, &plan)) return DYNCONV_ERR_UNSUPPORTED;
    return plan.p.tiles_h;
  }
  return 1;
}

int dynconv_route_pooled(const dynconv_desc* desc, const float* ysum, int parts, const float* Wr,
                         const float* br, int mode, float tau, float* alpha, void* stream) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!ysum || !Wr || !alpha || parts < 1) return DYNCONV_ERR_INVALID_ARG;
  if (mode != DYNCONV_SIGMOID && mode != DYNCONV_SOFTMAX) return DYNCONV_ERR_INVALID_ARG;
  if (mode == DYNCONV_SOFTMAX && !(tau > 0.f)) return DYNCONV_ERR_INVALID_ARG;
  if (desc->n > 1024 || desc->C_in > 16384) return DYNCONV_ERR_UNSUPPORTED;
  if (desc->B == 0) return DYNCONV_OK;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc) return rc;
  dc::RoutePooledParams p{desc->B, desc->C_in, desc->H * desc->W, desc->n, parts, mode, tau,
                          ysum, Wr, br, alpha};
  const size_t smem = sizeof(float) * (static_cast<size_t>(desc->C_in) + desc->n);
  if (smem > static_cast<size_t>(st->max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
  cudaError_t e = cudaSuccess;
  if (smem > 48 * 1024) e = ensure_smem(dc::route_pooled_kernel, smem);
  if (e != cudaSuccess) return cuda_fail(e, "cudaFuncSetAttribute(route_pooled)");
  e = launch_pdl(dc::route_pooled_kernel, dim3(desc->B), dim3(dc::kPoolThreads), smem,
                 static_cast<cudaStream_t>(stream), p);
  if (e != cudaSuccess) {
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cuda_fail(e, "route_pooled_kernel launch");
  }
  return check_launch("route_pooled_kernel");
}

int dynconv_forward_noalloc(const dynconv_desc* desc, const void* x, const void* experts,
                            const float* alpha, const float* bias, void* y, void* stream) {
  int rc = validate_desc(desc);
  if (rc) return rc;
  if (!x || !experts || !alpha || !y) return DYNCONV_ERR_INVALID_ARG;
  if (desc->B == 0) return DYNCONV_OK;
  dynconv_desc d = *desc;
  d.variant = DYNCONV_VARIANT_PREMIX;
  if (!tc_shape_ok(&d)) return DYNCONV_ERR_UNSUPPORTED;
  const size_t need = premix_workspace(&d);
  if (need == 0) return DYNCONV_ERR_UNSUPPORTED;
  if (need > DYNCONV_NOALLOC_MAX_BYTES) {
    std::snprintf(g_last_err, sizeof(g_last_err),
                  "shape needs %zu bytes of scratch; the built-in array holds %u", need,
                  DYNCONV_NOALLOC_MAX_BYTES);
    return DYNCONV_ERR_WORKSPACE;
  }
  if (!aligned16(x) || !aligned16(experts) || !aligned16(y)) return DYNCONV_ERR_MISALIGNED;
  DeviceState* st = nullptr;
  rc = device_state(&st);
  if (rc) return rc;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  void* scratch = nullptr;
  {
    // first call on this device (which is current): look the array's address up
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
      e = cudaGetSymbolAddress(&g_noalloc_ptr[dev], g_noalloc_scratch);
      if (e != cudaSuccess) {
        g_noalloc_ptr[dev] = nullptr;
        return cuda_fail(e, "cudaGetSymbolAddress(no-alloc scratch)");
      }
    }
    scratch = g_noalloc_ptr[dev];
  }
  return run_tc(&d, DYNCONV_VARIANT_PREMIX, st, x, experts, alpha, bias, y, scratch,
                DYNCONV_NOALLOC_MAX_BYTES, static_cast<cudaStream_t>(stream));
}

int dynconv_device_status(void* stream) {
  DeviceState* st = nullptr;
  int rc = device_state(&st);
  if (rc) return rc;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int word = 0;
  e = cudaMemcpyFromSymbol(&word, g_device_err, sizeof(int));
  if (e != cudaSuccess) return cuda_fail(e, "read error word");
  if (word != 0) {
    {
      int dev = 0;
      if (cudaGetDevice(&dev) == cudaSuccess && dev >= 0 && dev < 64) {
        std::lock_guard<std::mutex> lk(g_slot_mu);
        g_slots_dirty[dev] = true;
      }
    }
    const int zero = 0;
    e = cudaMemcpyToSymbol(g_device_err, &zero, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "clear error word");
    std::snprintf(g_last_err, sizeof(g_last_err), "device error word 0x%x", word);
    return DYNCONV_ERR_TIMEOUT;
  }
  return DYNCONV_OK;
}

}  // extern "C"

// ============================================== helpers for the other units

namespace dc_lib {

int device_info(DeviceInfo* out) {
  DeviceState* st = nullptr;
  const int rc = device_state(&st);
  if (rc) return rc;
  out->err = st->err;
  out->sms = st->sms;
  out->max_smem_optin = st->max_smem_optin;
  out->wait_ns = g_wait_ns.load();
  out->encode_tiled = reinterpret_cast<void*>(g_encode);
  return DYNCONV_OK;
}

int fail(int status, const char* msg) {
  std::snprintf(g_last_err, sizeof(g_last_err), "%s", msg);
  return status;
}

int cuda_error(cudaError_t e, const char* what) { return cuda_fail(e, what); }

int launched(const char* what) { return check_launch(what); }

int validate(const dynconv_desc* desc) { return validate_desc(desc); }

bool mixgrad_tc_enabled() { return g_mixgrad_tc.load() != 0; }

int forward_add(const dynconv_desc* desc, const void* x, const void* experts, const float* alpha,
                const float* bias, void* y, void* workspace, size_t workspace_bytes, void* stream,
                const float* chan_add, float chan_scale) {
  return forward_impl(desc, x, experts, alpha, bias, y, workspace, workspace_bytes, stream,
                      nullptr, nullptr, nullptr, chan_add, chan_scale);
}

cudaError_t set_smem(const void* kernel, size_t bytes) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const auto key = std::make_pair(dev, kernel);
  std::lock_guard<std::mutex> lk(g_smem_mu);
  auto it = g_smem_set.find(key);
  if (it != g_smem_set.end() && it->second >= bytes) return cudaSuccess;
  e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(bytes));
  if (e == cudaSuccess) g_smem_set[key] = bytes;
  return e;
}

}  // namespace dc_lib
