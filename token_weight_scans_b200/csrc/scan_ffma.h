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
  const float* S0 = nullptr;  // [B*H][nseg][dout][din] start state of each segment, or null (zero)
  float* ST = nullptr;        // [B*H][dout][din] receives the state after the last token, or null
                              // (written by the last segment)
  // Segments: nseg CTAs per scan walk chunks [seg * seg_chunks, (seg + 1) * seg_chunks).
  int nseg = 1;
  int seg_chunks = 1 << 30;
  int summary = 0;            // 1: state carry only, from zero (y and ckpt must be null)
  float* Sloc = nullptr;      // summary: [B*H][nseg][dout][din] each segment's local end state
  float* segL = nullptr;      // summary: [B*H][nseg] log2 of the product of alpha over the segment
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
  const float* LamT = nullptr;  // [B*H][nseg][dout][din] adjoint at each segment's end, or null (zero)
  float* dS0 = nullptr;         // [B*H][dout][din] receives the adjoint at the first token, or null
                                // (written by the first segment)
  // Segments, walked backwards: dW0_part is then [B][nseg][H][dout][din].
  int nseg = 1;
  int seg_chunks = 1 << 30;
  int summary = 0;              // 1: adjoint carry only, from zero at the segment's end
  float* Lloc = nullptr;        // summary: [B*H][nseg][dout][din] each segment's local adjoint
  float* segL = nullptr;        // summary: [B*H][nseg] log2 of the product of alpha over the segment
};

bool shape_ok(int din, int dout);
size_t ckpt_bytes(int B, int H, int T, int din, int dout);
size_t dW0_part_bytes(int B, int H, int din, int dout);
// Chunks of the CUDA-core kernels (tokens per chunk).
constexpr int kChunk = 32;
cudaError_t launch_fwd(const FwdArgs& a, bool bf16, cudaStream_t st);
cudaError_t launch_bwd(const BwdArgs& a, bool bf16, cudaStream_t st);
// dW0[h] = sum over b of part[b][h] (fixed order); used by both kernel families
cudaError_t launch_reduce_dW0(const float* part, float* dW0, int B, int H, int dd,
                              cudaStream_t st);

}  // namespace ffma
}  // namespace gradlev
