// Host-side interface of the consistency-step kernels (consistency.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gradlev {
namespace consistency {

struct ResidualArgs {
  size_t ntok;       // B * H * T
  int dout;          // multiple of 4
  const void* y;     // [ntok][dout] dtype
  const void* ghat;  // [ntok][dout]
  const void* v;     // [ntok][dout]
  void* gtil;        // [ntok][dout] out: y - v
  void* dv;          // [ntok][dout] out: -(y - v), or null
  float* loss_tok;   // [ntok] out: 0.5 ||y - v||^2
  float* loss_c;     // [ntok] out: ||ghat - (y - v)||^2
};

cudaError_t launch_residual(const ResidualArgs& a, bool bf16, cudaStream_t st);
// dghat += 2 lam (ghat - gtil) over `elems` elements (a multiple of 4)
cudaError_t launch_finish(void* dghat, const void* ghat, const void* gtil, float lam,
                          size_t elems, bool bf16, cudaStream_t st);

}  // namespace consistency
}  // namespace gradlev
