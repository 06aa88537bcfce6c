// Host side of the backward entry points declared in include/dynconv_backward.h:
// argument checks, workspace layout, tensor maps and launches. A translation
// unit of its own (the forward unit, dynconv.cu, shares device state and
// error reporting through internal.h); the input gradient reuses the forward
// entry point on the transposed problem.
#include <cuda.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <cstdint>
#include <cstdio>

#include "dynconv.h"
#include "dynconv_backward.h"
#include "internal.h"

#include "backward_kernels.cuh"
#include "backward_wgrad_tc.cuh"
#include "backward_mixgrad_tc.cuh"

namespace {

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

int out_size(int in, int k, int stride, int pad) { return (in + 2 * pad - k) / stride + 1; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }
size_t elem_bytes(const dynconv_desc* d) { return d->dtype == DYNCONV_F32 ? 4 : 2; }
long long wsize_of(const dynconv_desc* d) {
  return 1LL * d->C_out * d->KH * d->KW * (d->C_in / d->groups);
}

// ------------------------------------------------------- workspace layout

// Slices of the channel sums are sized for at most this many SMs (the
// workspace size is a pure host function).
constexpr int kMaxSms = 160;

int chansum_slices(int B, int P, int sms);

struct WeightLayout {
  size_t dW = 0, db = 0, part = 0, cs = 0, dex = 0, total = 0;
  int chunks = 0;
  int bsplit = 1;  // sample groups of the mixing gradient (partial dexperts when > 1)
};

// Sample groups for the mixing gradient: about two CTAs per SM in all, at
// least 8 samples per group.
int mix_bsplit(const dynconv_desc* d, int chunks) {
  const int ne = d->n > 4 ? 8 : d->n > 2 ? 4 : d->n;
  const long long ctas = 1LL * chunks * ((d->n + ne - 1) / ne);
  const long long want = (2LL * kMaxSms + ctas - 1) / ctas;
  return static_cast<int>(std::max<long long>(1, std::min<long long>(want, d->B / 8)));
}

WeightLayout weight_layout(const dynconv_desc* d) {
  WeightLayout L;
  const long long ws = wsize_of(d);
  L.chunks = static_cast<int>((ws + dcb::kMgChunk - 1) / dcb::kMgChunk);
  L.dW = 0;
  L.db = align256(L.dW + 4ull * d->B * ws);
  L.part = align256(L.db + 4ull * d->B * d->C_out);
  L.cs = align256(L.part + 4ull * L.chunks * d->B * d->n);
  const int Ho = out_size(d->H, d->KH, d->stride, d->pad), Wo = out_size(d->W, d->KW, d->stride, d->pad);
  L.dex = align256(L.cs + 4ull * d->B * d->C_out * chansum_slices(d->B, Ho * Wo, kMaxSms));
  L.bsplit = mix_bsplit(d, L.chunks);
  L.total = align256(L.dex + (L.bsplit > 1 ? 4ull * L.bsplit * d->n * ws : 0));
  return L;
}

// The input gradient as a forward convolution: stride 1 and one padding
// value that stays non-negative after the flip (square kernels).
bool transposed_ok(const dynconv_desc* d) {
  return d->stride == 1 && d->KH == d->KW && d->KH - 1 - d->pad >= 0;
}

dynconv_desc transposed_desc(const dynconv_desc* d) {
  dynconv_desc t = *d;
  t.C_in = d->C_out;
  t.C_out = d->C_in;
  t.H = out_size(d->H, d->KH, 1, d->pad);
  t.W = out_size(d->W, d->KW, 1, d->pad);
  t.pad = d->KH - 1 - d->pad;
  return t;
}

size_t data_workspace(const dynconv_desc* d) {
  if (!transposed_ok(d)) return 0;
  const dynconv_desc t = transposed_desc(d);
  return align256(static_cast<size_t>(d->n) * wsize_of(d) * elem_bytes(d)) +
         dynconv_workspace_size(&t);
}

// ------------------------------------------------- tensor-core weight gradient

bool wgrad_tc_shape_ok(const dynconv_desc* d) {
  const int Wo = out_size(d->W, d->KW, 1, d->pad);
  return d->dtype == DYNCONV_BF16 && d->groups == 1 && d->stride == 1 && d->C_in % 8 == 0 &&
         d->C_out % 8 == 0 && Wo <= 128;
}

int encode_4d(EncodeTiledFn enc, CUtensorMap* map, const void* base, int C, int W, int H, int B,
              int box_w, int box_h) {
  const cuuint64_t dims[4] = {static_cast<cuuint64_t>(C), static_cast<cuuint64_t>(W),
                              static_cast<cuuint64_t>(H), static_cast<cuuint64_t>(B)};
  const cuuint64_t strides[3] = {static_cast<cuuint64_t>(C) * 2,
                                 static_cast<cuuint64_t>(W) * C * 2,
                                 static_cast<cuuint64_t>(H) * W * C * 2};
  const cuuint32_t box[4] = {64u, static_cast<cuuint32_t>(box_w), static_cast<cuuint32_t>(box_h),
                             1u};
  const cuuint32_t es[4] = {1u, 1u, 1u, 1u};
  if (enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void*>(base), dims, strides, box,
          es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
    return dc_lib::fail(DYNCONV_ERR_UNSUPPORTED,
                        "cuTensorMapEncodeTiled (weight gradient) refused the shape");
  return DYNCONV_OK;
}

int run_wgrad_tc(const dynconv_desc* d, const dc_lib::DeviceInfo& di, const void* x,
                 const void* dy, float* dW, cudaStream_t s, bool hilo = false) {
  const int Ho = out_size(d->H, d->KH, 1, d->pad), Wo = out_size(d->W, d->KW, 1, d->pad);
  dcb::WgParams p{};
  p.B = d->B; p.Cin = d->C_in; p.Cout = d->C_out; p.Ho = Ho; p.Wo = Wo;
  p.KH = d->KH; p.KW = d->KW; p.pad = d->pad;
  // K tiles of whole output rows, at most 128 pixels, balanced
  int tiles = (Ho * Wo + 127) / 128;
  int BH = (Ho + tiles - 1) / tiles;
  while (BH * Wo > 128) {
    ++tiles;
    BH = (Ho + tiles - 1) / tiles;
  }
  p.BH = BH;
  p.ktiles = (Ho + BH - 1) / BH;
  p.ksteps = (BH * Wo + 15) / 16;
  p.atom_bytes = p.ksteps * 16 * 128;
  p.box_bytes = BH * Wo * 128;
  p.cblk = (d->C_in + 63) / 64;
  p.natoms = d->KH * d->KW * p.cblk;
  p.agroups = (p.natoms + dcb::kWgMaxAtoms - 1) / dcb::kWgMaxAtoms;
  p.co_tiles = (d->C_out + 127) / 128;
  p.units = 1LL * d->B * p.co_tiles * p.agroups;
  const int stage_bytes = (2 + dcb::kWgMaxAtoms) * p.atom_bytes;
  p.stages = std::min(4, (210 * 1024 - 4 * dcb::kWgStageBytes) / stage_bytes);
  if (p.stages < 2) return dc_lib::fail(DYNCONV_ERR_UNSUPPORTED, "weight-gradient tile too large");
  p.dW = dW;
  p.hilo = hilo ? 1 : 0;
  p.err = di.err;
  p.wait_ns = di.wait_ns;
  auto enc = reinterpret_cast<EncodeTiledFn>(di.encode_tiled);
  CUtensorMap dymap, xmap;
  int rc = encode_4d(enc, &dymap, dy, d->C_out, Wo, Ho, d->B, Wo, BH);
  if (rc) return rc;
  rc = encode_4d(enc, &xmap, x, d->C_in, d->W, d->H, d->B, Wo, BH);
  if (rc) return rc;
  // at least 120 KB, so that two CTAs never share an SM (each holds all 512 TMEM columns)
  const size_t smem = std::max<size_t>(
      120 * 1024, 1024 + static_cast<size_t>(p.stages) * stage_bytes + 4 * dcb::kWgStageBytes +
                      8 * (2 * p.stages + 5) + 16);
  if (smem > static_cast<size_t>(di.max_smem_optin))
    return dc_lib::fail(DYNCONV_ERR_UNSUPPORTED, "weight-gradient shared memory");
  cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(dcb::wgrad_tc_kernel), smem);
  if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(wgrad_tc)");
  const unsigned grid = static_cast<unsigned>(std::min<long long>(p.units, di.sms));
  dcb::wgrad_tc_kernel<<<grid, dcb::kWgThreads, smem, s>>>(dymap, xmap, p);
  return dc_lib::launched("wgrad_tc_kernel");
}

int run_wgrad_direct(const dynconv_desc* d, const void* x, const void* dy, float* dW,
                     cudaStream_t s) {
  dcb::WgdParams p{};
  p.B = d->B; p.Cin = d->C_in; p.H = d->H; p.W = d->W; p.Cout = d->C_out;
  p.KH = d->KH; p.KW = d->KW; p.stride = d->stride; p.pad = d->pad; p.groups = d->groups;
  p.Ho = out_size(d->H, d->KH, d->stride, d->pad);
  p.Wo = out_size(d->W, d->KW, d->stride, d->pad);
  p.wsize = wsize_of(d);
  p.x = x; p.dy = dy; p.dW = dW;
  const dim3 grid(static_cast<unsigned>((p.wsize + dcb::kBwThreads - 1) / dcb::kBwThreads), d->B);
  if (d->dtype == DYNCONV_F32)
    dcb::wgrad_direct_kernel<float><<<grid, dcb::kBwThreads, 0, s>>>(p);
  else
    dcb::wgrad_direct_kernel<__nv_bfloat16><<<grid, dcb::kBwThreads, 0, s>>>(p);
  return dc_lib::launched("wgrad_direct_kernel");
}

bool wgrad_dw_ok(const dynconv_desc* d) {
  return d->dtype == DYNCONV_BF16 && d->groups == d->C_in && d->C_in == d->C_out &&
         d->stride == 1 && d->KH == d->KW && (d->KH == 3 || d->KH == 5 || d->KH == 7) &&
         d->C_in % 8 == 0;
}

// Bands of output rows small enough for ~3 CTAs per SM (at most 80 KB), or
// 0 when even one row does not fit.
int wgrad_dw_band(const dynconv_desc* d, int max_smem, size_t* smem_out) {
  const int K = d->KH;
  const int Ho = out_size(d->H, K, 1, d->pad), Wo = out_size(d->W, K, 1, d->pad);
  const int Wp = Wo + K - 1;
  auto bytes = [&](int band) {
    return static_cast<size_t>((band + K - 1) * Wp + band * Wo) * dcb::kDwgChunk * 2;
  };
  int band = Ho;
  while (band > 1 && bytes(band) > 80 * 1024) band = (band + 1) / 2;
  if (bytes(band) > static_cast<size_t>(max_smem)) return 0;
  *smem_out = bytes(band);
  return band;
}

int run_wgrad_dw(const dynconv_desc* d, int band, size_t smem, const void* x, const void* dy,
                 float* dW, cudaStream_t s) {
  dcb::DwgParams p{};
  p.B = d->B; p.C = d->C_in; p.H = d->H; p.W = d->W; p.pad = d->pad; p.band = band;
  p.Ho = out_size(d->H, d->KH, 1, d->pad);
  p.Wo = out_size(d->W, d->KW, 1, d->pad);
  p.x = static_cast<const __nv_bfloat16*>(x);
  p.dy = static_cast<const __nv_bfloat16*>(dy);
  p.dW = dW;
  const dim3 grid((d->C_in + dcb::kDwgChunk - 1) / dcb::kDwgChunk, d->B);
  auto go = [&](auto kern, int K) -> int {
    if (smem > 48 * 1024) {
      cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(kern), smem);
      if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(wgrad_dw)");
    }
    kern<<<grid, dim3(32, K), smem, s>>>(p);
    return dc_lib::launched("wgrad_dw_kernel");
  };
  return d->KH == 3 ? go(dcb::wgrad_dw_kernel<3>, 3)
         : d->KH == 5 ? go(dcb::wgrad_dw_kernel<5>, 5) : go(dcb::wgrad_dw_kernel<7>, 7);
}

// Pixel slices per sample for the channel sums: about four CTAs per SM in
// all, at least 32 pixels per slice.
int chansum_slices(int B, int P, int sms) {
  const int want = std::max(1, (4 * sms + B - 1) / std::max(B, 1));
  return std::max(1, std::min(want, P / 32));
}

// out[b][c] = sum over pixels of v; `scratch` holds B * slices * C floats.
int run_chansum(const dynconv_desc* d, int sms, const void* v, int P, int C, float* scratch,
                float* out, cudaStream_t s) {
  const bool bf = d->dtype == DYNCONV_BF16;
  const int vec = bf ? 8 : 4;
  const bool vok = C % vec == 0 && aligned16(v);
  const size_t smem = sizeof(float) * dcb::kBwThreads * (vok ? vec : 1);
  int slices = scratch ? chansum_slices(d->B, P, sms) : 1;
  // up to 8 slices: one cluster per sample adds them in shared memory (no
  // finishing kernel, no scratch); more go through the scratch and a second pass
  const size_t smem_cl = smem + sizeof(float) * static_cast<size_t>(C);
  const bool cluster = slices > 1 && slices <= 16 && smem_cl <= 48 * 1024;
  if (cluster) slices = std::min(slices, 8);
  if (slices == 1) scratch = out;  // one slice: the partial is the sum
  const int Ps = (P + slices - 1) / slices;
  const dim3 grid(slices, d->B);
  if (cluster) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(dcb::kBwThreads, 1, 1);
    cfg.dynamicSmemBytes = smem_cl;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = slices;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e;
    if (bf)
      e = vok ? cudaLaunchKernelEx(&cfg, dcb::chansum_kernel<__nv_bfloat16, 8, true>,
                                   static_cast<const __nv_bfloat16*>(v), P, C, Ps, out)
              : cudaLaunchKernelEx(&cfg, dcb::chansum_kernel<__nv_bfloat16, 1, true>,
                                   static_cast<const __nv_bfloat16*>(v), P, C, Ps, out);
    else
      e = vok ? cudaLaunchKernelEx(&cfg, dcb::chansum_kernel<float, 4, true>,
                                   static_cast<const float*>(v), P, C, Ps, out)
              : cudaLaunchKernelEx(&cfg, dcb::chansum_kernel<float, 1, true>,
                                   static_cast<const float*>(v), P, C, Ps, out);
    if (e != cudaSuccess) return dc_lib::cuda_error(e, "chansum_kernel (cluster) launch");
    return dc_lib::launched("chansum_kernel");
  }
  if (bf) {
    if (vok)
      dcb::chansum_kernel<__nv_bfloat16, 8><<<grid, dcb::kBwThreads, smem, s>>>(
          static_cast<const __nv_bfloat16*>(v), P, C, Ps, scratch);
    else
      dcb::chansum_kernel<__nv_bfloat16, 1><<<grid, dcb::kBwThreads, smem, s>>>(
          static_cast<const __nv_bfloat16*>(v), P, C, Ps, scratch);
  } else {
    if (vok)
      dcb::chansum_kernel<float, 4><<<grid, dcb::kBwThreads, smem, s>>>(
          static_cast<const float*>(v), P, C, Ps, scratch);
    else
      dcb::chansum_kernel<float, 1><<<grid, dcb::kBwThreads, smem, s>>>(
          static_cast<const float*>(v), P, C, Ps, scratch);
  }
  int rc = dc_lib::launched("chansum_kernel");
  if (rc || slices == 1) return rc;
  const long long total = 1LL * d->B * C;
  dcb::chansum_finish_kernel<<<static_cast<unsigned>((total + dcb::kBwThreads - 1) / dcb::kBwThreads),
                               dcb::kBwThreads, 0, s>>>(d->B, C, slices, scratch, out);
  return dc_lib::launched("chansum_finish_kernel");
}

// The tensor-core mixing gradient applies to dW from the tcgen05 weight
// gradient (written as bf16 hi / lo planes) with at most 256 samples, 32
// experts and kernels of a multiple of 128 weights.
bool mixgrad_tc_ok(const dynconv_desc* d) {
  return dc_lib::mixgrad_tc_enabled() && d->dtype == DYNCONV_BF16 && d->B >= 1 && d->B <= 256 &&
         d->n <= 64 && wsize_of(d) % dcb::kMtTile == 0;
}

// dexperts (complete) and one dalpha partial per CTA; returns the number of
// partials in `part` through *nparts.
int run_mixgrad_tc(const dynconv_desc* d, const dc_lib::DeviceInfo& di, const void* planes,
                   const void* experts, const float* alpha, float* dexperts, float* part,
                   int max_parts, int* nparts, cudaStream_t s) {
  const long long ws = wsize_of(d);
  dcb::MtParams p{};
  p.B = d->B; p.n = d->n; p.nk = d->n <= 16 ? 16 : d->n <= 32 ? 32 : 64;
  p.halves = (d->B + 127) / 128;
  p.wsize = ws;
  p.tiles = ws / dcb::kMtTile;
  p.plane_bytes = 2 * 128 * 128;
  p.e_bytes = 2 * p.nk * 128;
  p.stage_bytes = 2 * p.plane_bytes + p.e_bytes;
  p.b_bytes = p.halves * 2 * 2 * p.nk * 128;
  const size_t fixed = 1024 + static_cast<size_t>(p.b_bytes) + 8 * 32 + 16;
  p.stages = static_cast<int>(std::min<size_t>(3, (di.max_smem_optin - fixed) / p.stage_bytes));
  if (p.stages < 2) return DYNCONV_ERR_UNSUPPORTED;
  p.alpha = alpha;
  p.dexperts = dexperts;
  p.part = part;
  p.err = di.err;
  p.wait_ns = di.wait_ns;
  auto enc = reinterpret_cast<EncodeTiledFn>(di.encode_tiled);
  auto map2d = [&](CUtensorMap* m, const void* base, long long inner, int rows, int box_rows) {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(inner), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(inner) * 2};
    const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
    const cuuint32_t es[2] = {1u, 1u};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
               es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  CUtensorMap himap, lomap, emap;
  const __nv_bfloat16* hi = static_cast<const __nv_bfloat16*>(planes);
  const __nv_bfloat16* lo = hi + static_cast<size_t>(d->B) * ws;
  if (!map2d(&himap, hi, ws, d->B, 128) || !map2d(&lomap, lo, ws, d->B, 128) ||
      !map2d(&emap, experts, ws, d->n, p.nk))
    return dc_lib::fail(DYNCONV_ERR_UNSUPPORTED, "cuTensorMapEncodeTiled (mixing gradient)");
  const size_t smem = fixed + static_cast<size_t>(p.stages) * p.stage_bytes;
  cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(dcb::mixgrad_tc_kernel), smem);
  if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(mixgrad_tc)");
  const int grid = static_cast<int>(std::min<long long>({p.tiles, static_cast<long long>(di.sms),
                                                         static_cast<long long>(max_parts)}));
  dcb::mixgrad_tc_kernel<<<grid, dcb::kMtThreads, smem, s>>>(himap, lomap, emap, p);
  *nparts = grid;
  return dc_lib::launched("mixgrad_tc_kernel");
}

template <typename T>
int launch_mixgrad(const dcb::MgParams& p, int ne, size_t smem, cudaStream_t s) {
  const dim3 grid(p.chunks, (p.n + ne - 1) / ne, p.bsplit);
  auto go = [&](auto kern) -> int {
    if (smem > 48 * 1024) {
      cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(kern), smem);
      if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(mixgrad)");
    }
    kern<<<grid, dcb::kBwThreads, smem, s>>>(p);
    return dc_lib::launched("mixgrad_kernel");
  };
  switch (ne) {
    case 1: return go(dcb::mixgrad_kernel<T, 1>);
    case 2: return go(dcb::mixgrad_kernel<T, 2>);
    case 4: return go(dcb::mixgrad_kernel<T, 4>);
    default: return go(dcb::mixgrad_kernel<T, 8>);
  }
}

}  // namespace

extern "C" {

size_t dynconv_backward_workspace_size(const dynconv_desc* desc) {
  if (dc_lib::validate(desc) != DYNCONV_OK) return 0;
  const size_t route = align256(4ull * desc->B * desc->C_in *
                                chansum_slices(desc->B, desc->H * desc->W, kMaxSms));
  return std::max({weight_layout(desc).total, data_workspace(desc), route});
}

int dynconv_backward_weight(const dynconv_desc* desc, const void* x, const void* dy,
                            const void* experts, const float* alpha, const float* bias,
                            float* dexperts, float* dbias, float* dalpha, void* workspace,
                            size_t workspace_bytes, void* stream) {
  int rc = dc_lib::validate(desc);
  if (rc) return rc;
  if (!x || !dy || !experts || !alpha || !dexperts || !dalpha) return DYNCONV_ERR_INVALID_ARG;
  if ((bias == nullptr) != (dbias == nullptr)) return DYNCONV_ERR_INVALID_ARG;
  const dynconv_desc* d = desc;
  const bool tc_ok = wgrad_tc_shape_ok(d);
  bool use_tc;
  switch (d->variant) {
    case DYNCONV_VARIANT_AUTO: use_tc = tc_ok; break;
    case DYNCONV_VARIANT_FUSED:
    case DYNCONV_VARIANT_OUTSIDE:
    case DYNCONV_VARIANT_PREMIX:
      if (!tc_ok) return DYNCONV_ERR_UNSUPPORTED;
      use_tc = true;
      break;
    default: use_tc = false; break;
  }
  if (use_tc && (!aligned16(x) || !aligned16(dy))) {
    if (d->variant != DYNCONV_VARIANT_AUTO) return DYNCONV_ERR_MISALIGNED;
    use_tc = false;
  }
  const WeightLayout L = weight_layout(d);
  const long long ws = wsize_of(d);
  if (d->B == 0) {
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    cudaError_t e = cudaMemsetAsync(dexperts, 0, 4ull * d->n * ws, s);
    if (e == cudaSuccess && dbias) e = cudaMemsetAsync(dbias, 0, 4ull * d->n * d->C_out, s);
    return e == cudaSuccess ? DYNCONV_OK : dc_lib::cuda_error(e, "cudaMemsetAsync");
  }
  if (!workspace || workspace_bytes < L.total) return DYNCONV_ERR_WORKSPACE;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNCONV_ERR_MISALIGNED;
  dc_lib::DeviceInfo di;
  rc = dc_lib::device_info(&di);
  if (rc) return rc;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  char* wsb = static_cast<char*>(workspace);
  float* dW = reinterpret_cast<float*>(wsb + L.dW);
  float* db = reinterpret_cast<float*>(wsb + L.db);
  float* part = reinterpret_cast<float*>(wsb + L.part);

  // experts per CTA of the mixing gradient: every sample's dW is read
  // ceil(n / ne) times; its shared memory is checked before anything runs
  const int ne = d->n > 4 ? 8 : d->n > 2 ? 4 : d->n;
  const size_t mg_smem = sizeof(float) * (static_cast<size_t>(d->B) * ne +
                                          (dcb::kBwThreads / 32) * dcb::kMgSampleBlock * ne +
                                          (dcb::kBwThreads / 32) * 32 * 33);
  if (mg_smem > static_cast<size_t>(di.max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;

  // 1. per-sample weight gradients (as bf16 hi / lo planes when the
  // tensor-core mixing gradient reads them)
  const bool mg_tc = use_tc && mixgrad_tc_ok(d) && aligned16(experts);
  if (use_tc) {
    rc = run_wgrad_tc(d, di, x, dy, dW, s, mg_tc);
    if (rc == DYNCONV_ERR_UNSUPPORTED && d->variant == DYNCONV_VARIANT_AUTO) use_tc = false;
    else if (rc) return rc;
  }
  if (!use_tc) {
    size_t dw_smem = 0;
    const int band = (wgrad_dw_ok(d) && aligned16(x) && aligned16(dy) &&
                      d->variant != DYNCONV_VARIANT_DIRECT)
                         ? wgrad_dw_band(d, di.max_smem_optin, &dw_smem)
                         : 0;
    if (d->variant == DYNCONV_VARIANT_DEPTHWISE && band == 0) return DYNCONV_ERR_UNSUPPORTED;
    rc = band > 0 ? run_wgrad_dw(d, band, dw_smem, x, dy, dW, s)
                  : run_wgrad_direct(d, x, dy, dW, s);
    if (rc) return rc;
  }
  // 2. per-sample bias gradients: channel sums of dy
  const int Ho = out_size(d->H, d->KH, d->stride, d->pad);
  const int Wo = out_size(d->W, d->KW, d->stride, d->pad);
  rc = run_chansum(d, std::min(di.sms, kMaxSms), dy, Ho * Wo, d->C_out,
                   reinterpret_cast<float*>(wsb + L.cs), db, s);
  if (rc) return rc;
  // 3. the experts' gradients and the chunks' shares of dalpha
  int nparts = L.chunks;
  if (use_tc && mg_tc) {
    rc = run_mixgrad_tc(d, di, dW, experts, alpha, dexperts, part, L.chunks, &nparts, s);
    if (rc) return rc;
  } else {
  dcb::MgParams mp{};
  mp.B = d->B; mp.n = d->n; mp.wsize = ws; mp.chunks = L.chunks;
  mp.vec = (ws % 4 == 0 && aligned16(dexperts)) ? 1 : 0;
  mp.dW = dW; mp.experts = experts; mp.alpha = alpha; mp.part = part;
  mp.bsplit = L.bsplit;
  mp.bs = (d->B + L.bsplit - 1) / L.bsplit;
  mp.dexperts = L.bsplit > 1 ? reinterpret_cast<float*>(wsb + L.dex) : dexperts;
  if (L.bsplit > 1) mp.vec = ws % 4 == 0 ? 1 : 0;
  rc = d->dtype == DYNCONV_F32 ? launch_mixgrad<float>(mp, ne, mg_smem, s)
                               : launch_mixgrad<__nv_bfloat16>(mp, ne, mg_smem, s);
  if (rc) return rc;
  if (L.bsplit > 1) {
    const long long total = 1LL * d->n * ws;
    const unsigned g = static_cast<unsigned>(
        std::min<long long>((total / 4 + dcb::kBwThreads) / dcb::kBwThreads, 16LL * di.sms));
    dcb::dexperts_finish_kernel<<<g, dcb::kBwThreads, 0, s>>>(total, L.bsplit, mp.dexperts,
                                                              dexperts);
    rc = dc_lib::launched("dexperts_finish_kernel");
    if (rc) return rc;
  }
  }
  // 4. dalpha = sum of the partial shares + <db_b, bias_i>
  dcb::dalpha_finish_kernel<<<d->B, dcb::kBwThreads, 0, s>>>(d->B, d->n, d->C_out, nparts, part,
                                                             db, bias, dalpha);
  rc = dc_lib::launched("dalpha_finish_kernel");
  if (rc) return rc;
  // 5. dbias
  if (dbias) {
    dcb::dbias_kernel<<<dim3((d->C_out + 31) / 32, (d->n + 7) / 8), dim3(32, 8), 0, s>>>(
        d->B, d->n, d->C_out, alpha, db, dbias);
    rc = dc_lib::launched("dbias_kernel");
  }
  return rc;
}

int dynconv_route_backward(const dynconv_desc* desc, const void* x, const float* Wr,
                           const float* alpha, const float* dalpha, int mode, float tau,
                           float* dWr, float* dbr, float* dg, void* workspace,
                           size_t workspace_bytes, void* stream) {
  int rc = dc_lib::validate(desc);
  if (rc) return rc;
  if (!x || !Wr || !alpha || !dalpha || !dWr || !dg) return DYNCONV_ERR_INVALID_ARG;
  if (mode != DYNCONV_SIGMOID && mode != DYNCONV_SOFTMAX) return DYNCONV_ERR_INVALID_ARG;
  if (mode == DYNCONV_SOFTMAX && !(tau > 0.f)) return DYNCONV_ERR_INVALID_ARG;
  if (desc->n > 1024) return DYNCONV_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int C = desc->C_in, n = desc->n, B = desc->B;
  if (B == 0) {
    cudaError_t e = cudaMemsetAsync(dWr, 0, 4ull * n * C, s);
    if (e == cudaSuccess && dbr) e = cudaMemsetAsync(dbr, 0, 4ull * n, s);
    return e == cudaSuccess ? DYNCONV_OK : dc_lib::cuda_error(e, "cudaMemsetAsync");
  }
  dc_lib::DeviceInfo di;
  rc = dc_lib::device_info(&di);
  if (rc) return rc;
  const size_t smem_param = sizeof(float) * ((static_cast<size_t>(B) + 3) / 4 * 4 + dcb::kBwThreads);
  const size_t smem_dg = sizeof(float) * (static_cast<size_t>(n) + dcb::kBwThreads);
  if (smem_param > static_cast<size_t>(di.max_smem_optin)) return DYNCONV_ERR_UNSUPPORTED;
  // the channel sums of x go to dg first (scratch), then dg is overwritten;
  // their pixel slices use the workspace when it has room
  const int sms = std::min(di.sms, kMaxSms);
  const size_t cs_bytes =
      4ull * B * C * chansum_slices(B, desc->H * desc->W, sms);
  float* cs = (workspace && workspace_bytes >= cs_bytes &&
               (reinterpret_cast<uintptr_t>(workspace) & 15u) == 0)
                  ? static_cast<float*>(workspace)
                  : nullptr;
  rc = run_chansum(desc, sms, x, desc->H * desc->W, C, cs, dg, s);
  if (rc) return rc;
  if (smem_param > 48 * 1024) {
    cudaError_t e = dc_lib::set_smem(reinterpret_cast<const void*>(dcb::route_bwd_param_kernel),
                                     smem_param);
    if (e != cudaSuccess) return dc_lib::cuda_error(e, "cudaFuncSetAttribute(route_bwd_param)");
  }
  const float inv_hw = 1.f / static_cast<float>(desc->H * desc->W);
  // the most sample slices (shorter chains) that keep the grid within one CTA per SM
  int slices = dcb::kRbpMaxSlices;
  while (slices > 1 &&
         static_cast<long long>((C + dcb::kBwThreads / slices - 1) / (dcb::kBwThreads / slices)) * n >
             sms)
    slices >>= 1;
  const int cpc = dcb::kBwThreads / slices;
  dcb::route_bwd_param_kernel<<<dim3((C + cpc - 1) / cpc, n), dcb::kBwThreads, smem_param, s>>>(
      B, C, n, slices, inv_hw, mode, tau, alpha, dalpha, dg, dWr, dbr);
  rc = dc_lib::launched("route_bwd_param_kernel");
  if (rc) return rc;
  dcb::route_bwd_dg_kernel<<<dim3((C + dcb::kBwThreads - 1) / dcb::kBwThreads, B),
                             dcb::kBwThreads, smem_dg, s>>>(C, n, mode, tau, alpha, dalpha, Wr,
                                                            dg);
  return dc_lib::launched("route_bwd_dg_kernel");
}

int dynconv_backward_data(const dynconv_desc* desc, const void* dy, const void* experts,
                          const float* alpha, const float* dg, void* dx, void* workspace,
                          size_t workspace_bytes, void* stream) {
  int rc = dc_lib::validate(desc);
  if (rc) return rc;
  if (!dy || !experts || !alpha || !dx) return DYNCONV_ERR_INVALID_ARG;
  if (desc->B == 0) return DYNCONV_OK;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const dynconv_desc* d = desc;
  const float inv_hw = 1.f / static_cast<float>(d->H * d->W);
  if (transposed_ok(d)) {
    const size_t et_bytes = align256(static_cast<size_t>(d->n) * wsize_of(d) * elem_bytes(d));
    if (!workspace || workspace_bytes < et_bytes) return DYNCONV_ERR_WORKSPACE;
    if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return DYNCONV_ERR_MISALIGNED;
    const dynconv_desc t = transposed_desc(d);
    // refuse what the forward would refuse before anything runs
    const int v = dynconv_select_variant(&t, workspace_bytes - et_bytes);
    if (v < 0) return v;
    dc_lib::DeviceInfo di;
    rc = dc_lib::device_info(&di);
    if (rc) return rc;
    const int Cg = d->C_in / d->groups, Coutg = d->C_out / d->groups;
    const int taps_groups = d->KH * d->KW * d->groups;
    if (d->dtype == DYNCONV_BF16 && Cg % 8 == 0 && Coutg % 8 == 0 && taps_groups <= 65535 &&
        d->n <= 65535 && (reinterpret_cast<uintptr_t>(experts) & 15u) == 0) {
      // 64 x 64 tiles moved as 16-byte chunks
      const dim3 grid(((Cg + 63) / 64) * ((Coutg + 63) / 64), taps_groups, d->n);
      dcb::transpose_experts_v8_kernel<<<grid, 256, 0, s>>>(
          d->C_in, d->C_out, d->KH, d->KW, d->groups, static_cast<const __nv_bfloat16*>(experts),
          reinterpret_cast<__nv_bfloat16*>(workspace));
    } else if (Cg >= 8 && Coutg >= 8 && taps_groups <= 65535 && d->n <= 65535) {
      // 32 x 32 tiles of each group's [Coutg][Cg] matrix per (tap, group, expert)
      const dim3 grid(((Cg + 31) / 32) * ((Coutg + 31) / 32), taps_groups, d->n), block(32, 8);
      if (d->dtype == DYNCONV_F32)
        dcb::transpose_experts_tiled_kernel<float><<<grid, block, 0, s>>>(
            d->C_in, d->C_out, d->KH, d->KW, d->groups, static_cast<const float*>(experts),
            reinterpret_cast<float*>(workspace));
      else
        dcb::transpose_experts_tiled_kernel<__nv_bfloat16><<<grid, block, 0, s>>>(
            d->C_in, d->C_out, d->KH, d->KW, d->groups,
            static_cast<const __nv_bfloat16*>(experts),
            reinterpret_cast<__nv_bfloat16*>(workspace));
    } else {
      const long long total = 1LL * d->n * wsize_of(d);
      const unsigned grid = static_cast<unsigned>(
          std::min<long long>((total + dcb::kBwThreads - 1) / dcb::kBwThreads, 8LL * di.sms));
      if (d->dtype == DYNCONV_F32)
        dcb::transpose_experts_kernel<float><<<grid, dcb::kBwThreads, 0, s>>>(
            d->n, d->C_in, d->C_out, d->KH, d->KW, d->groups, static_cast<const float*>(experts),
            reinterpret_cast<float*>(workspace));
      else
        dcb::transpose_experts_kernel<__nv_bfloat16><<<grid, dcb::kBwThreads, 0, s>>>(
            d->n, d->C_in, d->C_out, d->KH, d->KW, d->groups,
            static_cast<const __nv_bfloat16*>(experts),
            reinterpret_cast<__nv_bfloat16*>(workspace));
    }
    rc = dc_lib::launched("transpose_experts_kernel");
    if (rc) return rc;
    char* rest = static_cast<char*>(workspace) + et_bytes;
    // dx = (transposed convolution of dy) + dg / (H W), added before the
    // convolution's single rounding of dx
    return dc_lib::forward_add(&t, dy, workspace, alpha, nullptr, dx,
                               workspace_bytes > et_bytes ? rest : nullptr,
                               workspace_bytes - et_bytes, stream, dg, inv_hw);
  }
  dcb::DgdParams p{};
  p.B = d->B; p.Cin = d->C_in; p.H = d->H; p.W = d->W; p.Cout = d->C_out;
  p.KH = d->KH; p.KW = d->KW; p.stride = d->stride; p.pad = d->pad; p.groups = d->groups;
  p.Ho = out_size(d->H, d->KH, d->stride, d->pad);
  p.Wo = out_size(d->W, d->KW, d->stride, d->pad);
  p.n = d->n;
  p.dy = dy; p.experts = experts; p.alpha = alpha; p.dg = dg; p.inv_hw = inv_hw; p.dx = dx;
  const long long n_dx = 1LL * d->B * d->H * d->W * d->C_in;
  const unsigned grid = static_cast<unsigned>((n_dx + dcb::kBwThreads - 1) / dcb::kBwThreads);
  if (d->dtype == DYNCONV_F32)
    dcb::dgrad_direct_kernel<float><<<grid, dcb::kBwThreads, 0, s>>>(p);
  else
    dcb::dgrad_direct_kernel<__nv_bfloat16><<<grid, dcb::kBwThreads, 0, s>>>(p);
  return dc_lib::launched("dgrad_direct_kernel");
}

}  // extern "C"
