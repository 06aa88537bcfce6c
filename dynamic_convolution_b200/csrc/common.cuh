// Shared device helpers: bounded barrier waits with a CTA-wide abort flag and a
// per-device error word, and small numeric helpers.
#pragma once

#include <cstdint>
#include <cuda_bf16.h>

#include "ptx.cuh"

namespace dc {

// Error word values (nonzero = a bounded wait expired; the low byte says where).
enum : int {
  kErrNone = 0,
  kErrWaitProducer = 0x101,
  kErrWaitMma = 0x102,
  kErrWaitMixer = 0x103,
  kErrWaitEpilogue = 0x104,
  kErrWaitDrain = 0x105,
  kErrWaitGrid = 0x106,
};

struct WaitCtl {
  volatile int* abort_flag;  // shared memory, CTA-wide
  int* err;                  // global, per device
  long long limit_ns;
};

// Wait for `parity`'s phase of `bar` to complete. Gives up (returns false) when
// another thread of the CTA has aborted, or after ctl.limit_ns, in which case it
// raises the CTA's abort flag and records `code` in the device error word.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, const WaitCtl& ctl,
                                             int code) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 31u) == 0) {
      if (*ctl.abort_flag) return false;
      if (static_cast<long long>(globaltimer_ns() - t0) > ctl.limit_ns) {
        *ctl.abort_flag = 1;
        atomicCAS(ctl.err, 0, code);
        return false;
      }
    }
  }
}

// Drain wait used on the exit path: bounded, never raises the abort flag again.
__device__ __forceinline__ void wait_drain(uint32_t bar, uint32_t parity, long long limit_ns,
                                           int* err) {
  if (mbar_try_wait(bar, parity)) return;
  const uint64_t t0 = globaltimer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity)) return;
    if (static_cast<long long>(globaltimer_ns() - t0) > limit_ns) {
      atomicCAS(err, 0, kErrWaitDrain);
      return;
    }
  }
}

template <typename T>
__device__ __forceinline__ float to_f32(T v);
template <>
__device__ __forceinline__ float to_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}

template <typename T>
__device__ __forceinline__ T from_f32(float v);
template <>
__device__ __forceinline__ float from_f32<float>(float v) {
  return v;
}
template <>
__device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

}  // namespace dc
