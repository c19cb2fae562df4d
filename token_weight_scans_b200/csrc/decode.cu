// Deployment decode: the token-by-token forward pass, costate and update of the
// adapted layer, with its deviation carried between calls.
//
// GradLev abstract: at deployment the auxiliary predictor is discarded and the
// model updates itself by token-by-token forward and backward passes (Cognaptus,
// "Parallelize the Training, Keep the Learning Serial", opening section: a
// forward pass, a backward pass and a weight update per token). For one adapted
// linear layer with the inner loss 0.5 ||W x_t - v_t||^2 of the pages' synthetic
// test, a token is
//
//   y_t = (W0 + S) x_t,   g_t = y_t - v_t,   S <- alpha_t S - eta_t g_t x_t^T.
//
// Within a token the rows of S are independent: y_t[n] needs row n of W0 + S
// and x_t, and the update of row n needs g_t[n] and x_t. So a warp owns kRows
// rows, keeps them (S and W0, fp32) in registers across all T tokens of the
// call, one float4 per lane per 128 columns, and forms y_t[n] with a butterfly
// reduction. Every lane ends the butterfly with the same sum, since each step
// adds the same two values. HBM traffic is the minimum: S read once and written
// once per call, W0 read once (shared through L2 by the batch rows), and the
// per-token vectors.

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "common.cuh"
#include "gradlev.h"

namespace gradlev {
namespace decode {

constexpr int kWarps = 4;                     // warps per CTA
constexpr int kRows = 4;                      // rows of S per warp
constexpr int kRowsPerCta = kWarps * kRows;
constexpr int kMaxDin = 256;                  // two float4 per lane

struct DecodeArgs {
  int B, H, T, din, dout;
  const void* x;       // [B,H,T,din]
  const void* v;       // [B,H,T,dout]
  const float* eta;    // [B,H,T]
  const float* alpha;  // [B,H,T]
  const float* W0;     // [H,dout,din]
  float* S;            // [B,H,dout,din], in and out
  void* y;             // [B,H,T,dout]
  void* g;             // [B,H,T,dout] or null
};

__device__ __forceinline__ float4 load4(const float* p) {
  return *reinterpret_cast<const float4*>(p);
}
__device__ __forceinline__ float4 load4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

template <typename Tio, int NK4>
// 8 CTAs per SM (at most 64 registers) for d_in <= 128, so that the B8 H16 d128 grid of
// 1024 CTAs runs in one wave on 148 SMs; a second wave doubles the time of a call.
__global__ void __launch_bounds__(kWarps * 32, NK4 == 1 ? 8 : 4) decode_kernel(DecodeArgs a) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tiles = (a.dout + kRowsPerCta - 1) / kRowsPerCta;
  const int bh = blockIdx.x / tiles, tile = blockIdx.x - bh * tiles;
  const int h = bh % a.H;
  const int nb = tile * kRowsPerCta + warp * kRows;  // first row of this warp
  const int din = a.din;
  float4 s[kRows][NK4], w[kRows][NK4];
  bool kok[NK4];
#pragma unroll
  for (int i = 0; i < NK4; ++i) kok[i] = 4 * (lane + 32 * i) < din;
  const float4 zero = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int n = nb + r;
    const bool rok = n < a.dout;
#pragma unroll
    for (int i = 0; i < NK4; ++i) {
      const size_t k = 4 * (size_t)(lane + 32 * i);
      const bool ok = rok && kok[i];
      s[r][i] = ok ? load4(a.S + ((size_t)bh * a.dout + n) * din + k) : zero;
      w[r][i] = ok ? load4(a.W0 + ((size_t)h * a.dout + n) * din + k) : zero;
    }
  }
  const Tio* xg = static_cast<const Tio*>(a.x);
  const Tio* vg = static_cast<const Tio*>(a.v);
  Tio* yg = static_cast<Tio*>(a.y);
  Tio* gg = static_cast<Tio*>(a.g);
  const size_t tok0 = (size_t)bh * a.T;
  for (int t = 0; t < a.T; ++t) {
    const size_t tok = tok0 + t;
    float4 xv[NK4];
#pragma unroll
    for (int i = 0; i < NK4; ++i)
      xv[i] = kok[i] ? load4(xg + tok * din + 4 * (lane + 32 * i)) : zero;
    const float et = a.eta[tok], al = a.alpha[tok];
#pragma unroll
    for (int r = 0; r < kRows; ++r) {
      const int n = nb + r;
      if (n >= a.dout) break;  // warp-uniform
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < NK4; ++i) {
        p = fmaf(w[r][i].x + s[r][i].x, xv[i].x, p);
        p = fmaf(w[r][i].y + s[r][i].y, xv[i].y, p);
        p = fmaf(w[r][i].z + s[r][i].z, xv[i].z, p);
        p = fmaf(w[r][i].w + s[r][i].w, xv[i].w, p);
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) p += __shfl_xor_sync(0xffffffffu, p, o);
      const float gv = p - to_f32(vg[tok * a.dout + n]);
      if (lane == r) {  // the warp's rows are written by different lanes
        yg[tok * a.dout + n] = from_f32<Tio>(p);
        if (gg) gg[tok * a.dout + n] = from_f32<Tio>(gv);
      }
      const float c = et * gv;
#pragma unroll
      for (int i = 0; i < NK4; ++i) {
        s[r][i].x = fmaf(-c, xv[i].x, al * s[r][i].x);
        s[r][i].y = fmaf(-c, xv[i].y, al * s[r][i].y);
        s[r][i].z = fmaf(-c, xv[i].z, al * s[r][i].z);
        s[r][i].w = fmaf(-c, xv[i].w, al * s[r][i].w);
      }
    }
  }
#pragma unroll
  for (int r = 0; r < kRows; ++r) {
    const int n = nb + r;
    if (n >= a.dout) break;
#pragma unroll
    for (int i = 0; i < NK4; ++i)
      if (kok[i])
        *reinterpret_cast<float4*>(a.S + ((size_t)bh * a.dout + n) * din + 4 * (lane + 32 * i)) =
            s[r][i];
  }
}

template <typename Tio>
static cudaError_t launch_t(const DecodeArgs& a, cudaStream_t st) {
  const int tiles = (a.dout + kRowsPerCta - 1) / kRowsPerCta;
  const int grid = a.B * a.H * tiles;
  if (a.din <= 128)
    decode_kernel<Tio, 1><<<grid, kWarps * 32, 0, st>>>(a);
  else
    decode_kernel<Tio, 2><<<grid, kWarps * 32, 0, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

static bool aligned(const void* p, size_t n) { return ((uintptr_t)p % n) == 0; }

}  // namespace decode
}  // namespace gradlev

using namespace gradlev;

extern "C" {

gradlev_status gradlev_decode_step(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                   const void* x, const void* v, const float* eta,
                                   const float* alpha, const float* W0, float* S, void* y,
                                   void* g, void* stream) {
  using namespace gradlev::decode;
  reset_launch_count();
  if (B <= 0 || H <= 0 || T <= 0 || d_in <= 0 || d_out <= 0) return GRADLEV_ERR_INVALID_ARG;
  if (dt != GRADLEV_F32 && dt != GRADLEV_BF16) return GRADLEV_ERR_INVALID_ARG;
  if (d_in % 4 != 0 || d_in > kMaxDin) return GRADLEV_ERR_UNSUPPORTED;
  const long long tiles = (d_out + kRowsPerCta - 1) / kRowsPerCta;
  if ((long long)B * H * tiles >= (1LL << 31) || (long long)B * H * T >= (1LL << 31))
    return GRADLEV_ERR_UNSUPPORTED;
  if (!x || !v || !eta || !alpha || !W0 || !S || !y) return GRADLEV_ERR_INVALID_ARG;
  const size_t es = dt == GRADLEV_BF16 ? 2 : 4;
  if (!aligned(x, 4 * es) || !aligned(v, es) || !aligned(y, es) || (g && !aligned(g, es)) ||
      !aligned(eta, 4) || !aligned(alpha, 4) || !aligned(W0, 16) || !aligned(S, 16))
    return GRADLEV_ERR_INVALID_ARG;
  DecodeArgs a{B, H, T, d_in, d_out, x, v, eta, alpha, W0, S, y, g};
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const cudaError_t e =
      dt == GRADLEV_BF16 ? launch_t<__nv_bfloat16>(a, st) : launch_t<float>(a, st);
  return e == cudaSuccess ? GRADLEV_OK : GRADLEV_ERR_CUDA;
}

}  // extern "C"
