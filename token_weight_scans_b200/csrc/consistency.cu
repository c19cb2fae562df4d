// The elementwise steps around the scans in one GradLev training step of the
// adapted layer (Cognaptus, "Parallelize the Training, Keep the Learning
// Serial", section "The predictor is constrained by the learner it is supposed
// to reproduce").
//
// The forward scan runs on the predicted costates ghat and gives y. For the
// synthetic test's inner loss 0.5 ||y - v||^2, the costates that the trajectory
// implies are gtil_t = y_t - v_t. The training loss
//   L = sum_t 0.5 ||gtil_t||^2 + lam ||ghat_t - gtil_t||^2   (gtil the target)
// needs two more steps:
//   residual: gtil, the per-token losses, and dv = -gtil. gtil is also the
//             reverse scan's dy, since it is the token loss's output gradient;
//   finish:   d ghat = dg (from the reverse scan) + 2 lam (ghat - gtil).
// Both read each operand once, and both are HBM-bound.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "consistency.h"

namespace gradlev {
namespace consistency {

constexpr int kWarps = 8;  // tokens per CTA of the residual kernel

__device__ __forceinline__ void load4v(const float* p, float (&o)[4]) {
  const float4 v = *reinterpret_cast<const float4*>(p);
  o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
}
__device__ __forceinline__ void load4v(const __nv_bfloat16* p, float (&o)[4]) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  o[0] = __uint_as_float(u.x << 16); o[1] = __uint_as_float(u.x & 0xffff0000u);
  o[2] = __uint_as_float(u.y << 16); o[3] = __uint_as_float(u.y & 0xffff0000u);
}
__device__ __forceinline__ void store4v(float* p, const float (&o)[4]) {
  *reinterpret_cast<float4*>(p) = make_float4(o[0], o[1], o[2], o[3]);
}
__device__ __forceinline__ void store4v(__nv_bfloat16* p, const float (&o)[4]) {
  const __nv_bfloat162 a = __floats2bfloat162_rn(o[0], o[1]);
  const __nv_bfloat162 b = __floats2bfloat162_rn(o[2], o[3]);
  uint2 u;
  u.x = *reinterpret_cast<const uint32_t*>(&a);
  u.y = *reinterpret_cast<const uint32_t*>(&b);
  *reinterpret_cast<uint2*>(p) = u;
}

// One warp per token; d_out % 4 == 0 (4 elements per lane per step, coalesced).
template <typename Tio>
__global__ void __launch_bounds__(kWarps * 32) residual_kernel(ResidualArgs a) {
  const int lane = threadIdx.x & 31;
  const size_t tok = (size_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tok >= a.ntok) return;  // warp-uniform
  const size_t row = tok * a.dout;
  const Tio* y = static_cast<const Tio*>(a.y) + row;
  const Tio* gh = static_cast<const Tio*>(a.ghat) + row;
  const Tio* v = static_cast<const Tio*>(a.v) + row;
  Tio* gt = static_cast<Tio*>(a.gtil) + row;
  Tio* dv = a.dv ? static_cast<Tio*>(a.dv) + row : nullptr;
  float st = 0.f, sc = 0.f;
  for (int e = 4 * lane; e < a.dout; e += 128) {
    float yy[4], gg[4], vv[4], g4[4], m4[4];
    load4v(y + e, yy);
    load4v(gh + e, gg);
    load4v(v + e, vv);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      g4[i] = yy[i] - vv[i];
      const float r = gg[i] - g4[i];
      st = fmaf(g4[i], g4[i], st);
      sc = fmaf(r, r, sc);
      m4[i] = -g4[i];
    }
    store4v(gt + e, g4);
    if (dv) store4v(dv + e, m4);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    st += __shfl_xor_sync(0xffffffffu, st, o);
    sc += __shfl_xor_sync(0xffffffffu, sc, o);
  }
  if (lane == 0) {
    a.loss_tok[tok] = 0.5f * st;
    a.loss_c[tok] = sc;
  }
}

// dghat += 2 lam (ghat - gtil), 4 elements per thread (n4 = elements / 4).
template <typename Tio>
__global__ void finish_kernel(void* dghat, const void* ghat, const void* gtil, float two_lam,
                              size_t n4) {
  Tio* dg = static_cast<Tio*>(dghat);
  const Tio* gh = static_cast<const Tio*>(ghat);
  const Tio* gt = static_cast<const Tio*>(gtil);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n4;
       i += (size_t)gridDim.x * blockDim.x) {
    float d[4], a[4], b[4];
    load4v(dg + 4 * i, d);
    load4v(gh + 4 * i, a);
    load4v(gt + 4 * i, b);
#pragma unroll
    for (int k = 0; k < 4; ++k) d[k] = fmaf(two_lam, a[k] - b[k], d[k]);
    store4v(dg + 4 * i, d);
  }
}

cudaError_t launch_residual(const ResidualArgs& a, bool bf16, cudaStream_t st) {
  const size_t grid = (a.ntok + kWarps - 1) / kWarps;
  if (bf16)
    residual_kernel<__nv_bfloat16><<<(unsigned)grid, kWarps * 32, 0, st>>>(a);
  else
    residual_kernel<float><<<(unsigned)grid, kWarps * 32, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_finish(void* dghat, const void* ghat, const void* gtil, float lam,
                          size_t elems, bool bf16, cudaStream_t st) {
  const size_t n4 = elems / 4;
  const size_t want = (n4 + 255) / 256;
  const unsigned grid = (unsigned)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  if (bf16)
    finish_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(dghat, ghat, gtil, 2.f * lam, n4);
  else
    finish_kernel<float><<<grid, 256, 0, st>>>(dghat, ghat, gtil, 2.f * lam, n4);
  count_launch();
  return cudaGetLastError();
}

}  // namespace consistency
}  // namespace gradlev
