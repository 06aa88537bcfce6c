// Library-internal entry points shared by the translation units of
// libdynconv.so (the forward unit, dynconv.cu, defines them). Hidden
// visibility: they are not part of the C ABI and are not exported.
#pragma once

#include <cuda_runtime.h>

#include "dynconv.h"

#define DC_HIDDEN __attribute__((visibility("hidden")))

namespace dc_lib {

struct DeviceInfo {
  int* err;             // device error word that bounded waits write
  int sms;              // multiprocessors
  int max_smem_optin;   // opt-in shared memory per block, bytes
  long long wait_ns;    // limit of every bounded wait
  void* encode_tiled;   // the driver's cuTensorMapEncodeTiled
};

// The current device's state (queried once per device). DYNCONV_OK or a
// negative status with the message set.
DC_HIDDEN int device_info(DeviceInfo* out);
// Sets the calling thread's last-error text and returns `status`.
DC_HIDDEN int fail(int status, const char* msg);
// DYNCONV_ERR_CUDA with "what: <CUDA error string>" as the message.
DC_HIDDEN int cuda_error(cudaError_t e, const char* what);
// Counts one kernel launch and checks cudaGetLastError.
DC_HIDDEN int launched(const char* what);
// cudaFuncSetAttribute(MaxDynamicSharedMemorySize) once per (device, kernel, size).
DC_HIDDEN cudaError_t set_smem(const void* kernel, size_t bytes);
// The descriptor checks every entry point makes (DYNCONV_OK or INVALID_ARG /
// UNSUPPORTED).
DC_HIDDEN int validate(const dynconv_desc* desc);
// Test hook 11: whether the backward may run the tensor-core mixing gradient.
DC_HIDDEN bool mixgrad_tc_enabled();
// dynconv_forward with one more per-(sample, output channel) term:
// chan_scale * chan_add[b][co] is added to the mixed bias, so that it joins
// the convolution before the single rounding of y (chan_add may be null).
DC_HIDDEN int forward_add(const dynconv_desc* desc, const void* x, const void* experts,
                          const float* alpha, const float* bias, void* y, void* workspace,
                          size_t workspace_bytes, void* stream, const float* chan_add,
                          float chan_scale);

}  // namespace dc_lib
