// Shared device/host helpers of the GradLev scan library (CUDA, sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "gradlev.h"

namespace gradlev {

// ---------------------------------------------------------------- dtype I/O
__device__ __forceinline__ float to_f32(float v) { return v; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 v) { return __bfloat162float(v); }

template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// Device status word at the start of every workspace (see gradlev_device_status).
struct DeviceStatus {
  unsigned int code;    // 0 = ok, else a gradlev_status value
  unsigned int where;   // kernel-specific location of the failed wait
  unsigned int pad[2];
};

// Launch accounting for gradlev_last_launch_count(): every entry point resets the
// count, every kernel launch adds one.
void count_launch();
void reset_launch_count();

}  // namespace gradlev
