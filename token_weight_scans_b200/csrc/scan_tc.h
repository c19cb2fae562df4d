// Host-side interface of the tensor-core (tcgen05) GradLev scan kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace gradlev {
namespace tc {

struct TcFwdParams {
  int B, H, T, din, dout;   // din == 128, dout % 128 == 0
  const float* eta;         // [B,H,T]
  const float* alpha;       // [B,H,T]
  const float* W0;          // [H,dout,din] float32
  __nv_bfloat16* y;         // [B,H,T,dout]
  DeviceStatus* status;     // device status word (workspace head)
  uint64_t timeout_ns;      // bound of every wait inside the kernel
  int inject;               // test hook: 1 = withhold one completion signal
};

bool fwd_shape_ok(int din, int dout);
cudaError_t launch_fwd(const TcFwdParams& p, const void* x, const void* g, cudaStream_t st);
size_t fwd_smem_bytes();

}  // namespace tc
}  // namespace gradlev
