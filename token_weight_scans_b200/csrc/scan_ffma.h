// Host-side interface of the CUDA-core (FFMA) GradLev scan kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

namespace gradlev {
namespace ffma {

struct FwdArgs {
  int B, H, T, din, dout;
  const void* x;      // [B,H,T,din] float or bf16
  const void* g;      // [B,H,T,dout]
  const float* eta;   // [B,H,T]
  const float* alpha; // [B,H,T]
  const float* W0;    // [H,dout,din]
  void* y;            // [B,H,T,dout] or null (state sweep only)
  float* ckpt;        // [B*H][n_chunks][dout][din] or null
  const float* S0 = nullptr;  // [B*H][dout][din] carried start state, or null (zero)
  float* ST = nullptr;        // [B*H][dout][din] receives the state after the last token, or null
};

struct BwdArgs {
  int B, H, T, din, dout;
  const void* x;
  const void* g;
  const float* eta;
  const float* alpha;
  const float* W0;
  const void* dy;     // [B,H,T,dout]
  void* dx;           // [B,H,T,din]
  void* dg;           // [B,H,T,dout]
  float* d_eta;       // [B,H,T]
  float* d_alpha;     // [B,H,T]
  float* dW0;         // [H,dout,din]
  const float* ckpt;  // chunk-start states written by the forward sweep
  float* dW0_part;    // [B*H][dout][din] scratch
  const float* LamT = nullptr;  // [B*H][dout][din] adjoint flowing in at the end, or null (zero)
  float* dS0 = nullptr;         // [B*H][dout][din] receives the adjoint at the first token, or null
};

bool shape_ok(int din, int dout);
size_t ckpt_bytes(int B, int H, int T, int din, int dout);
size_t dW0_part_bytes(int B, int H, int din, int dout);
cudaError_t launch_fwd(const FwdArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_bwd(const BwdArgs& a, bool bf16, cudaStream_t st);
// dW0[h] = sum over b of part[b][h] (fixed order); used by both kernel families
cudaError_t launch_reduce_dW0(const float* part, float* dW0, int B, int H, int dd,
                              cudaStream_t st);

}  // namespace ffma
}  // namespace gradlev
