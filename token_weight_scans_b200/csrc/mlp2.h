// Host-side interface of the two-layer reconstruction kernels (mlp2.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "common.cuh"

namespace gradlev {
namespace mlp2 {

struct TqueryArgs {
  int B, H, T, dx, dh, dy;
  int control;        // 1: the persistent W2 in the reconstruction (no S2 term)
  const void* x;      // [B,H,T,dx]  dtype
  const void* h;      // [B,H,T,dh]  tanh of the first layer's output
  const void* g2hat;  // [B,H,T,dy]  the second layer's given costates (drive S2)
  const void* y;      // [B,H,T,dy]  the second layer's output
  const void* v;      // [B,H,T,dy]  targets
  const float* eta;   // [B,H,T]
  const float* alpha; // [B,H,T]
  const float* W2;    // [H,dy,dh]
  void* g2til;        // [B,H,T,dy]  out: y - v
  void* g1til;        // [B,H,T,dh]  out: (1 - h^2) (.) ((W2 + S2_t)^T g2til)
  float* dW1;         // [B,H,dh,dx] out: sum_t g1til_t x_t^T
};

bool shape_ok(int dx, int dh, int dy);
cudaError_t launch_tanh(const void* a, void* h, size_t elems, bool bf16, cudaStream_t st);
cudaError_t launch_tquery(const TqueryArgs& a, bool bf16, cudaStream_t st);
// out = y - v over `elems` elements (a multiple of 4)
cudaError_t launch_sub(const void* y, const void* v, void* out, size_t elems, bool bf16,
                       cudaStream_t st);
// dW1[bh] = sum_t g1[bh][t] x[bh][t]^T, [dh][dx] fp32 per (b,h); shape_ok() limits apply
cudaError_t launch_outer_sum(const void* g1, const void* x, float* dW1, int BH, int T, int dh,
                             int dx, bool bf16, cudaStream_t st);
// The same sum on the tensor cores for bf16 with dh = dx = 128 (TMA tiles, tcgen05 MMAs,
// bounded waits reported through `status`).
bool outer_tc_ok(int dh, int dx);
cudaError_t launch_outer_tc(const void* g1, const void* x, float* dW1, int BH, int T,
                            DeviceStatus* status, cudaStream_t st);

}  // namespace mlp2
}  // namespace gradlev
