// The two-layer adapted MLP of the synthetic test (Cognaptus, "Parallelize the
// Training, Keep the Learning Serial", section "The synthetic test checks the
// mechanism, not model quality"): the parts of its parallel reconstruction that
// are not a forward scan.
//
// Both layers' forwards are the library's scans driven by the given costates:
//   a = scan(x; g1hat, W1),  h = tanh(a),  y = scan(h; g2hat, W2).
// The costates the trajectory implies are then reconstructed by backpropagating
// each token's loss 0.5 ||y_t - v_t||^2 through that token's adapted weights:
//   g2til_t = y_t - v_t,
//   g1til_t = (1 - h_t^2) (.) q_t,   q_t = (W2 + S2_t)^T g2til_t,
//   dW1     = sum_t g1til_t x_t^T    (the first matrix's gradient),
// where S2_t = sum_{j<t} (prod_{r=j+1}^{t-1} alpha_r) (-eta_j) g2hat_j h_j^T is
// the second layer's deviation. The control of the same section (the persistent
// W2 in place of the adapted one) drops the S2 term.
//
// q_t is a scan read "transposed": the second layer's state is queried from the
// output side. One CTA per (b, h) walks chunks of FC tokens with S2 in shared
// memory, as the CUDA-core forward does. Within a chunk
//   q_t = W2^T u_t + D[t][-1] S2_in^T u_t + sum_{j<t} (u_t . g2hat_j)(-eta_j) D[t][j] h_j,
// with D[t][j] = prod_{r=j+1}^{t-1} alpha_r (direct products, so alpha = 0 and 1 are
// exact). The chunk-to-chunk carry is the same formula at t = FC. dW1 accumulates in
// registers over the whole walk.

#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "common.cuh"
#include "mlp2.h"

namespace gradlev {
namespace mlp2 {

constexpr int FC = 32;       // tokens per chunk
constexpr int FT = 256;      // threads per CTA
constexpr int LDD = FC + 2;  // row stride of the decay table
constexpr int LDC = FC + 1;  // row stride of the FC x FC table

struct Layout {
  int LDH, LDY, LDX;
  size_t S2, Hc, Gc, Uc, Xc, G1c, P, Dt, et, al, total;  // offsets in floats
};

__host__ __device__ inline Layout layout(int dx, int dh, int dy) {
  Layout L;
  L.LDH = dh + 4;
  L.LDY = dy + 4;
  L.LDX = dx + 4;
  size_t o = 0;
  L.S2 = o;  o += (size_t)dy * L.LDH;
  L.Hc = o;  o += (size_t)FC * L.LDH;
  L.Gc = o;  o += (size_t)FC * L.LDY;
  L.Uc = o;  o += (size_t)FC * L.LDY;
  L.Xc = o;  o += (size_t)FC * L.LDX;
  L.G1c = o; o += (size_t)FC * L.LDH;
  L.P = o;   o += (size_t)FC * LDC;
  L.Dt = o;  o += (size_t)(FC + 1) * LDD;
  L.et = o;  o += FC;
  L.al = o;  o += FC;
  L.total = o;
  return L;
}

bool shape_ok(int dx, int dh, int dy) {
  if (dx % 4 || dh % 8 || dy % 8 || dx < 4 || dh < 8 || dy < 8) return false;
  if ((long)dh * dx > 2L * 8 * 4 * FT) return false;  // dW1 fits the registers (2 items)
  return layout(dx, dh, dy).total * sizeof(float) <= 227 * 1024;
}

template <typename Tio>
__device__ __forceinline__ void load_rows(float* dst, int ld, const Tio* src, int n_valid,
                                          int width, int tid) {
  for (int e = tid; e < FC * width; e += FT) {
    const int i = e / width, k = e - i * width;
    dst[i * ld + k] = (i < n_valid) ? to_f32(src[(size_t)i * width + k]) : 0.f;
  }
}

template <typename Tio>
__global__ void __launch_bounds__(FT, 1) tquery_kernel(TqueryArgs a) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  const int dx = a.dx, dh = a.dh, dy = a.dy, tid = threadIdx.x;
  const Layout L = layout(dx, dh, dy);
  float* S2 = sm + L.S2;
  float* Hc = sm + L.Hc;
  float* Gc = sm + L.Gc;
  float* Uc = sm + L.Uc;
  float* Xc = sm + L.Xc;
  float* G1c = sm + L.G1c;
  float* P = sm + L.P;
  float* Dt = sm + L.Dt;
  float* et = sm + L.et;
  float* al = sm + L.al;
  const int LDH = L.LDH, LDY = L.LDY, LDX = L.LDX;

  const int bh = blockIdx.x, hd = bh % a.H;
  const size_t tok0 = (size_t)bh * a.T;
  const int nch = (a.T + FC - 1) / FC;
  const Tio* xg = static_cast<const Tio*>(a.x);
  const Tio* hg = static_cast<const Tio*>(a.h);
  const Tio* gg = static_cast<const Tio*>(a.g2hat);
  const Tio* yg = static_cast<const Tio*>(a.y);
  const Tio* vg = static_cast<const Tio*>(a.v);
  Tio* g2o = static_cast<Tio*>(a.g2til);
  Tio* g1o = static_cast<Tio*>(a.g1til);
  const float* W2 = a.W2 + (size_t)hd * dy * dh;

  for (int e = tid; e < dy * dh; e += FT) {
    const int n = e / dh, k = e - n * dh;
    S2[n * LDH + k] = 0.f;
  }
  const int NKX4 = dx / 4, NBH = dh / 8, NKH = dh / 4, NBY = dy / 8;
  float4 dw[2][8];
#pragma unroll
  for (int it = 0; it < 2; ++it)
#pragma unroll
    for (int r = 0; r < 8; ++r) dw[it][r] = make_float4(0.f, 0.f, 0.f, 0.f);

  for (int c = 0; c < nch; ++c) {
    const int t0 = c * FC;
    const int nt = min(FC, a.T - t0);
    __syncthreads();
    load_rows(Hc, LDH, hg + (tok0 + t0) * dh, nt, dh, tid);
    load_rows(Gc, LDY, gg + (tok0 + t0) * dy, nt, dy, tid);
    load_rows(Xc, LDX, xg + (tok0 + t0) * dx, nt, dx, tid);
    for (int e = tid; e < FC * dy; e += FT) {  // u = y - v, written out as g2til
      const int i = e / dy, n = e - i * dy;
      float u = 0.f;
      if (i < nt) {
        const size_t o = (tok0 + t0 + i) * dy + n;
        u = to_f32(yg[o]) - to_f32(vg[o]);
        g2o[o] = from_f32<Tio>(u);
      }
      Uc[i * LDY + n] = u;
    }
    if (tid < FC) {
      et[tid] = tid < nt ? a.eta[tok0 + t0 + tid] : 0.f;
      al[tid] = tid < nt ? a.alpha[tok0 + t0 + tid] : 1.f;
    }
    __syncthreads();
    // decay table D[i][j+1] = prod_{r=j+1}^{i-1} al[r], i in [0, FC], j in [-1, FC-1]
    if (tid <= FC) {
      const int jp = tid;
      float pr = 1.f;
      for (int i = 0; i <= FC; ++i) {
        if (i < jp) {
          Dt[i * LDD + jp] = 0.f;
        } else {
          Dt[i * LDD + jp] = pr;
          if (i < FC) pr *= al[i];
        }
      }
    }
    __syncthreads();
    // P[i][j] = (u_i . g2hat_j) (-eta_j) D[i][j] for j < i
    for (int e = tid; e < FC * FC; e += FT) {
      const int i = e / FC, j = e - i * FC;
      float v = 0.f;
      if (j < i && !a.control) {
        float acc = 0.f;
        for (int n = 0; n < dy; n += 4) {
          const float4 uu = *reinterpret_cast<const float4*>(&Uc[i * LDY + n]);
          const float4 gv = *reinterpret_cast<const float4*>(&Gc[j * LDY + n]);
          acc += uu.x * gv.x + uu.y * gv.y + uu.z * gv.z + uu.w * gv.w;
        }
        v = acc * (-et[j]) * Dt[i * LDD + j + 1];
      }
      P[i * LDC + j] = v;
    }
    __syncthreads();
    // q_i = W2^T u_i + D[i][-1] S2_in^T u_i + sum_j P_ij h_j; g1til_i = (1 - h_i^2) q_i.
    // Thread tile: 4 tokens x 4 hidden units k = kg + NKH * r.
    for (int tile = tid; tile < (FC / 4) * NKH; tile += FT) {
      const int ig = tile / NKH, kg = tile - ig * NKH;
      float aw[4][4], as[4][4], ap[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) aw[q][r] = as[q][r] = ap[q][r] = 0.f;
      for (int n = 0; n < dy; ++n) {
        float uq[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) uq[q] = Uc[(ig * 4 + q) * LDY + n];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int k = kg + NKH * r;
          const float w = __ldg(&W2[(size_t)n * dh + k]);
          const float sv = S2[n * LDH + k];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            aw[q][r] = fmaf(uq[q], w, aw[q][r]);
            as[q][r] = fmaf(uq[q], sv, as[q][r]);
          }
        }
      }
      if (!a.control) {
        for (int j = 0; j < FC; ++j) {
          float hv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) hv[r] = Hc[j * LDH + kg + NKH * r];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float pv = P[(ig * 4 + q) * LDC + j];
#pragma unroll
            for (int r = 0; r < 4; ++r) ap[q][r] = fmaf(pv, hv[r], ap[q][r]);
          }
        }
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int i = ig * 4 + q;
        const float gam = a.control ? 0.f : Dt[i * LDD];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int k = kg + NKH * r;
          const float hk = Hc[i * LDH + k];
          const float g1 = (1.f - hk * hk) * (aw[q][r] + gam * as[q][r] + ap[q][r]);
          G1c[i * LDH + k] = i < nt ? g1 : 0.f;
          if (i < nt) g1o[(tok0 + t0 + i) * dh + k] = from_f32<Tio>(g1);
        }
      }
    }
    __syncthreads();
    // dW1 += sum_i g1til_i x_i^T (registers) and the carry
    // S2 <- D[FC][-1] S2 + sum_j (-eta_j D[FC][j]) g2hat_j h_j^T
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int item = tid + it * FT;
      if (item < NBH * NKX4) {
        const int nb = item / NKX4, k4 = item - nb * NKX4;
        for (int i = 0; i < nt; ++i) {
          const float4 xv = *reinterpret_cast<const float4*>(&Xc[i * LDX + 4 * k4]);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const float gv = G1c[i * LDH + nb * 8 + r];
            dw[it][r].x = fmaf(gv, xv.x, dw[it][r].x);
            dw[it][r].y = fmaf(gv, xv.y, dw[it][r].y);
            dw[it][r].z = fmaf(gv, xv.z, dw[it][r].z);
            dw[it][r].w = fmaf(gv, xv.w, dw[it][r].w);
          }
        }
      }
    }
    const float gC = Dt[FC * LDD];
    for (int item = tid; item < NBY * (dh / 4); item += FT) {
      const int nb = item / (dh / 4), k4 = item - nb * (dh / 4);
      float4 acc[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const float4 s = *reinterpret_cast<const float4*>(&S2[(nb * 8 + r) * LDH + 4 * k4]);
        acc[r] = make_float4(gC * s.x, gC * s.y, gC * s.z, gC * s.w);
      }
      for (int j = 0; j < nt; ++j) {
        const float w = -et[j] * Dt[FC * LDD + j + 1];
        const float4 hv = *reinterpret_cast<const float4*>(&Hc[j * LDH + 4 * k4]);
#pragma unroll
        for (int r = 0; r < 8; ++r) {
          const float c2 = w * Gc[j * LDY + nb * 8 + r];
          acc[r].x = fmaf(c2, hv.x, acc[r].x);
          acc[r].y = fmaf(c2, hv.y, acc[r].y);
          acc[r].z = fmaf(c2, hv.z, acc[r].z);
          acc[r].w = fmaf(c2, hv.w, acc[r].w);
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) *reinterpret_cast<float4*>(&S2[(nb * 8 + r) * LDH + 4 * k4]) = acc[r];
    }
  }
  float* dst = a.dW1 + (size_t)bh * dh * dx;
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int item = tid + it * FT;
    if (item < NBH * NKX4) {
      const int nb = item / NKX4, k4 = item - nb * NKX4;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        *reinterpret_cast<float4*>(&dst[(size_t)(nb * 8 + r) * dx + 4 * k4]) = dw[it][r];
    }
  }
}

// 16-byte vectors of the I/O type: 8 bf16 or 4 float per lane-load.
__device__ __forceinline__ float vget(uint32_t w, int hi) {
  return __uint_as_float(hi ? (w & 0xffff0000u) : (w << 16));
}
__device__ __forceinline__ uint32_t vpack(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

template <typename Tio, typename F>
__device__ __forceinline__ uint4 vmap(uint4 u, F f) {
  if constexpr (sizeof(Tio) == 2) {
    u.x = vpack(f(vget(u.x, 0)), f(vget(u.x, 1)));
    u.y = vpack(f(vget(u.y, 0)), f(vget(u.y, 1)));
    u.z = vpack(f(vget(u.z, 0)), f(vget(u.z, 1)));
    u.w = vpack(f(vget(u.w, 0)), f(vget(u.w, 1)));
  } else {
    u.x = __float_as_uint(f(__uint_as_float(u.x)));
    u.y = __float_as_uint(f(__uint_as_float(u.y)));
    u.z = __float_as_uint(f(__uint_as_float(u.z)));
    u.w = __float_as_uint(f(__uint_as_float(u.w)));
  }
  return u;
}

// h = tanh(a): 16-byte vectors, then a scalar tail
template <typename Tio>
__global__ void tanh_kernel(const Tio* __restrict__ a, Tio* __restrict__ h, size_t n) {
  constexpr int V = 16 / sizeof(Tio);
  const size_t nv = n / V, stride = (size_t)gridDim.x * blockDim.x;
  const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (size_t i = t; i < nv; i += stride)
    reinterpret_cast<uint4*>(h)[i] =
        vmap<Tio>(reinterpret_cast<const uint4*>(a)[i], [](float x) { return tanhf(x); });
  for (size_t i = nv * V + t; i < n; i += stride) h[i] = from_f32<Tio>(tanhf(to_f32(a[i])));
}

cudaError_t launch_tanh(const void* a, void* h, size_t elems, bool bf16, cudaStream_t st) {
  const size_t want = (elems / (bf16 ? 8 : 4) + 255) / 256;
  const unsigned grid = (unsigned)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  if (bf16)
    tanh_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(a),
                                                    static_cast<__nv_bfloat16*>(h), elems);
  else
    tanh_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(a), static_cast<float*>(h),
                                            elems);
  count_launch();
  return cudaGetLastError();
}

// out = y - v: 16-byte vectors, then a scalar tail
template <typename Tio>
__global__ void sub_kernel(const Tio* __restrict__ y, const Tio* __restrict__ v,
                           Tio* __restrict__ out, size_t n) {
  constexpr int V = 16 / sizeof(Tio);
  const size_t nv = n / V, stride = (size_t)gridDim.x * blockDim.x;
  const size_t t = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  for (size_t i = t; i < nv; i += stride) {
    const uint4 a = reinterpret_cast<const uint4*>(y)[i];
    const uint4 b = reinterpret_cast<const uint4*>(v)[i];
    uint4 r;
    if constexpr (sizeof(Tio) == 2) {
      r.x = vpack(vget(a.x, 0) - vget(b.x, 0), vget(a.x, 1) - vget(b.x, 1));
      r.y = vpack(vget(a.y, 0) - vget(b.y, 0), vget(a.y, 1) - vget(b.y, 1));
      r.z = vpack(vget(a.z, 0) - vget(b.z, 0), vget(a.z, 1) - vget(b.z, 1));
      r.w = vpack(vget(a.w, 0) - vget(b.w, 0), vget(a.w, 1) - vget(b.w, 1));
    } else {
      r.x = __float_as_uint(__uint_as_float(a.x) - __uint_as_float(b.x));
      r.y = __float_as_uint(__uint_as_float(a.y) - __uint_as_float(b.y));
      r.z = __float_as_uint(__uint_as_float(a.z) - __uint_as_float(b.z));
      r.w = __float_as_uint(__uint_as_float(a.w) - __uint_as_float(b.w));
    }
    reinterpret_cast<uint4*>(out)[i] = r;
  }
  for (size_t i = nv * V + t; i < n; i += stride)
    out[i] = from_f32<Tio>(to_f32(y[i]) - to_f32(v[i]));
}

// dW1 = sum_t g1_t x_t^T for one (b,h) per CTA: chunks of FC tokens are staged in
// shared memory and every thread accumulates up to two 8 x 4 blocks in registers.
template <typename Tio>
__global__ void __launch_bounds__(FT, 1) outer_sum_kernel(const Tio* __restrict__ g1,
                                                          const Tio* __restrict__ x,
                                                          float* __restrict__ dW1, int T, int dh,
                                                          int dx) {
  extern __shared__ float4 smem4[];
  float* Gs = reinterpret_cast<float*>(smem4);      // [FC][dh + 4]
  const int LDH = dh + 4, LDX = dx + 4;
  float* Xs = Gs + (size_t)FC * LDH;                // [FC][dx + 4]
  const int tid = threadIdx.x, bh = blockIdx.x;
  const size_t tok0 = (size_t)bh * T;
  const int NKX4 = dx / 4, NBH = dh / 8;
  float4 dw[2][8];
#pragma unroll
  for (int it = 0; it < 2; ++it)
#pragma unroll
    for (int r = 0; r < 8; ++r) dw[it][r] = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int t0 = 0; t0 < T; t0 += FC) {
    const int nt = min(FC, T - t0);
    __syncthreads();
    load_rows(Gs, LDH, g1 + (tok0 + t0) * dh, nt, dh, tid);
    load_rows(Xs, LDX, x + (tok0 + t0) * dx, nt, dx, tid);
    __syncthreads();
#pragma unroll
    for (int it = 0; it < 2; ++it) {
      const int item = tid + it * FT;
      if (item < NBH * NKX4) {
        const int nb = item / NKX4, k4 = item - nb * NKX4;
        for (int i = 0; i < nt; ++i) {
          const float4 xv = *reinterpret_cast<const float4*>(&Xs[i * LDX + 4 * k4]);
#pragma unroll
          for (int r = 0; r < 8; ++r) {
            const float gv = Gs[i * LDH + nb * 8 + r];
            dw[it][r].x = fmaf(gv, xv.x, dw[it][r].x);
            dw[it][r].y = fmaf(gv, xv.y, dw[it][r].y);
            dw[it][r].z = fmaf(gv, xv.z, dw[it][r].z);
            dw[it][r].w = fmaf(gv, xv.w, dw[it][r].w);
          }
        }
      }
    }
  }
  float* dst = dW1 + (size_t)bh * dh * dx;
#pragma unroll
  for (int it = 0; it < 2; ++it) {
    const int item = tid + it * FT;
    if (item < NBH * NKX4) {
      const int nb = item / NKX4, k4 = item - nb * NKX4;
#pragma unroll
      for (int r = 0; r < 8; ++r)
        *reinterpret_cast<float4*>(&dst[(size_t)(nb * 8 + r) * dx + 4 * k4]) = dw[it][r];
    }
  }
}

cudaError_t launch_sub(const void* y, const void* v, void* out, size_t elems, bool bf16,
                       cudaStream_t st) {
  const size_t want = (elems / (bf16 ? 8 : 4) + 255) / 256;
  const unsigned grid = (unsigned)(want < 148 * 16 ? (want > 0 ? want : 1) : 148 * 16);
  if (bf16)
    sub_kernel<__nv_bfloat16><<<grid, 256, 0, st>>>(static_cast<const __nv_bfloat16*>(y),
                                                   static_cast<const __nv_bfloat16*>(v),
                                                   static_cast<__nv_bfloat16*>(out), elems);
  else
    sub_kernel<float><<<grid, 256, 0, st>>>(static_cast<const float*>(y),
                                           static_cast<const float*>(v),
                                           static_cast<float*>(out), elems);
  count_launch();
  return cudaGetLastError();
}

template <typename Tio>
static cudaError_t launch_outer_sum_t(const void* g1, const void* x, float* dW1, int BH, int T,
                                      int dh, int dx, cudaStream_t st) {
  const size_t smem = sizeof(float) * (size_t)FC * ((dh + 4) + (dx + 4));
  cudaError_t e = cudaFuncSetAttribute(outer_sum_kernel<Tio>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  outer_sum_kernel<Tio><<<BH, FT, smem, st>>>(static_cast<const Tio*>(g1),
                                              static_cast<const Tio*>(x), dW1, T, dh, dx);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_outer_sum(const void* g1, const void* x, float* dW1, int BH, int T, int dh,
                             int dx, bool bf16, cudaStream_t st) {
  return bf16 ? launch_outer_sum_t<__nv_bfloat16>(g1, x, dW1, BH, T, dh, dx, st)
              : launch_outer_sum_t<float>(g1, x, dW1, BH, T, dh, dx, st);
}

template <typename Tio>
static cudaError_t launch_tquery_t(const TqueryArgs& a, cudaStream_t st) {
  const size_t smem = layout(a.dx, a.dh, a.dy).total * sizeof(float);
  cudaError_t e = cudaFuncSetAttribute(tquery_kernel<Tio>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  tquery_kernel<Tio><<<a.B * a.H, FT, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_tquery(const TqueryArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_tquery_t<__nv_bfloat16>(a, st) : launch_tquery_t<float>(a, st);
}

}  // namespace mlp2
}  // namespace gradlev
