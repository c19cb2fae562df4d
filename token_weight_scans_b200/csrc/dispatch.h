// Internal dispatch shared by the C entry points (gradlev_abi.cu, gradlev_noalloc.cu).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "gradlev.h"

namespace gradlev {

constexpr size_t kStatusBytes = 256;  // device status word + alignment pad

// Which kernel family serves a shape: the tcgen05 kernels for bf16 with
// d_in = d_out = 128, the CUDA-core kernels otherwise.
bool use_tc(int din, int dout, gradlev_dtype dt);

// Bytes of the reverse scan's scratch: status word, per-scan dW0 partials and,
// when `own_states`, the chunk-start states of a forward state sweep.
size_t bwd_scratch_bytes(int B, int H, int T, int din, int dout, gradlev_dtype dt,
                         bool own_states);

// The carried state of a split sequence, all [B,H,d_out,d_in] fp32 and optional:
// S0 the start deviation (null = 0), ST the end deviation (forward output), LamT the
// adjoint flowing in at the end (null = 0), dS0 the adjoint at the first token
// (reverse output).
struct StateIO {
  const float* S0 = nullptr;
  float* ST = nullptr;
  const float* LamT = nullptr;
  float* dS0 = nullptr;
};

// Launch the reverse scan with its scratch at `ws` (bwd_scratch_bytes(.., ckpt == NULL)
// bytes, 256-byte aligned). Shapes and pointers must already be validated. io.S0 is read
// only when ckpt is null (the forward sweep that recomputes the states starts from it).
// clear_status = false keeps what earlier launches of the same call wrote into the
// status word at the start of `ws`.
gradlev_status bwd_run(int B, int H, int T, int din, int dout, gradlev_dtype dt, const void* x,
                       const void* g, const float* eta, const float* alpha, const float* W0,
                       const void* dy, void* dx, void* dg, float* d_eta, float* d_alpha,
                       float* dW0, const void* ckpt, char* ws, cudaStream_t st,
                       const StateIO& io = StateIO{}, bool clear_status = true);

}  // namespace gradlev
