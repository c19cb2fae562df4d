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
  __nv_bfloat16* y;         // [B,H,T,dout], or null (state checkpoints only)
  __nv_bfloat16* ckpt;      // [B*H][n_chunks][dout][din] chunk-start states, or null
  DeviceStatus* status;     // device status word (workspace head)
  uint64_t timeout_ns;      // bound of every wait inside the kernel
  int inject;               // test hook: 1 = withhold one completion signal
};

// The reverse scan of one 128-row slice [n0, n0+128) of d_out: the rows of the
// state and adjoint evolve independently, so a d_out = 256 problem is two
// slice problems whose dx, d_eta and d_alpha add up (accumulate = 1 on the
// second slice) and whose dg and dW0 rows are disjoint.
struct TcBwdParams {
  int B, H, T, din, dout;   // din == 128, dout in {128, 256}
  int n0;                   // first d_out row of this slice
  int accumulate;           // add dx, d_eta, d_alpha onto the values already there
  const float* eta;
  const float* alpha;
  const float* W0;          // [H,128,128] float32
  __nv_bfloat16* dx;        // [B,H,T,128]
  __nv_bfloat16* dg;        // [B,H,T,128]
  float* d_eta;             // [B,H,T]
  float* d_alpha;           // [B,H,T]
  float* dW0_part;          // [B*H][128][128] float32 per-scan partials
  DeviceStatus* status;
  uint64_t timeout_ns;
};

constexpr int kChunk = 64;  // tokens per chunk of the tensor-core kernels

bool fwd_shape_ok(int din, int dout);
bool bwd_shape_ok(int din, int dout);
// bytes of the bf16 chunk-start state checkpoints the tensor-core kernels exchange
size_t ckpt_bytes(int B, int H, int T, int din, int dout);
cudaError_t launch_fwd(const TcFwdParams& p, const void* x, const void* g, cudaStream_t st);
cudaError_t launch_bwd(const TcBwdParams& p, const void* x, const void* g, const void* dy,
                       const void* ckpt, cudaStream_t st);
size_t fwd_smem_bytes();

}  // namespace tc
}  // namespace gradlev
