// CUDA-core (FFMA) chunkwise GradLev scans: the float32 path of the library.
//
// Per (b, h) scan one CTA walks the sequence in chunks of FC = 32 tokens (or, when
// few long scans cannot fill the GPU, one CTA per segment of it: a summary pass from
// a zero start, the segment combine, then the main pass from the combined start
// state) and keeps the d_out x d_in float32 state in shared memory. Within a chunk the
// recurrence S_{t+1} = alpha_t S_t - eta_t g_t x_t^T (Cognaptus, "Parallelize
// the Training, Keep the Learning Serial", section "Once the gradient signals
// are known, the weight trajectory becomes parallelizable") is unrolled into
// its discounted-sum form, so every token of the chunk is evaluated in
// parallel from the chunk-start state:
//
//   S_{c0+i} = D[i][-1] S_in + sum_{j<i} D[i][j] (-eta_j) g_j x_j^T,
//   D[i][j]  = prod_{r=j+1}^{i-1} alpha_r          (chunk-local indices)
//
// and the chunk-to-chunk carry is the same formula at i = FC. The decay
// products D are formed by direct multiplication (no logarithms), so alpha = 0
// and alpha = 1 are exact.
//
// The reverse scan (GradLev abstract: exact scans for reverse
// backpropagation) walks the chunks backwards carrying the state adjoint
// Lam_t = alpha_t Lam_{t+1} + u_t x_t^T in shared memory, with the chunk-start
// states S_in read back from checkpoints written by a forward sweep.
// d_alpha_t = <Lam_{t+1}, S_t> is evaluated exactly per chunk as the four
// cross terms of (chunk-end adjoint + intra-chunk adjoint) x (chunk-start state
// + intra-chunk state), which avoids any division by alpha.

#include <cuda_bf16.h>

#include <atomic>
#include <cuda_runtime.h>

#include <type_traits>

#include "common.cuh"
#include "scan_ffma.h"

namespace gradlev {
namespace ffma {

constexpr int FC = kChunk;  // tokens per chunk
constexpr int FT = 256;   // threads per CTA
constexpr int LDD = FC + 2;  // row stride of the decay table
constexpr int LDC = FC + 1;  // row stride of FC x FC tables
static_assert(FC == 32 && FT == 256, "the warp-level passes map a chunk's tokens to lanes, 8 warps");

__device__ __forceinline__ float dot4(float4 a, float4 b) {
  return a.x * b.x + a.y * b.y + a.z * b.z + a.w * b.w;
}

__device__ __forceinline__ void fma4(float4& acc, float s, float4 v) {
  acc.x = fmaf(s, v.x, acc.x);
  acc.y = fmaf(s, v.y, acc.y);
  acc.z = fmaf(s, v.z, acc.z);
  acc.w = fmaf(s, v.w, acc.w);
}

// Decay table Dt[i*LDD + (j+1)] = prod_{r=j+1}^{i-1} al[r] for i in [0, FC],
// j in [-1, FC-1] (1 for the empty product, 0 where i <= j). Threads 0..FC.
__device__ __forceinline__ void decay_table(float* Dt, const float* al, int tid) {
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
}

// Rows of a global matrix into a float32 shared-memory tile (row stride ld, a multiple
// of 4), in groups of 4 elements (width % 4 == 0; rows 16-byte aligned for float, 8-byte
// for bf16); rows at or past n_valid read as zero. Each thread issues all its loads of a
// pass before it stores any of them, so their latencies overlap instead of adding up
// (the compiler cannot prove that the global loads and shared stores do not alias).
constexpr int RB = 4;  // 4-element groups per thread per pass

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }
__device__ __forceinline__ float4 ld4(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xffff0000u),
                     __uint_as_float(u.y << 16), __uint_as_float(u.y & 0xffff0000u));
}

struct RowTile {
  float* dst;
  int ld, n_rows, width;
};

template <typename Tio>
__device__ __forceinline__ void fetch_rows(float4 (&v)[RB], const Tio* src, int n_rows,
                                           int n_valid, int width, int tid, int pass) {
  const int w4 = width >> 2, total = n_rows * w4;
#pragma unroll
  for (int u = 0; u < RB; ++u) {
    const int e = (pass * RB + u) * FT + tid;
    const int i = e / w4, k4 = e - i * w4;
    v[u] = (e < total && i < n_valid) ? ld4(src + (size_t)i * width + 4 * k4)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

__device__ __forceinline__ void put_rows(const RowTile& t, const float4 (&v)[RB], int tid,
                                         int pass) {
  const int w4 = t.width >> 2, total = t.n_rows * w4;
#pragma unroll
  for (int u = 0; u < RB; ++u) {
    const int e = (pass * RB + u) * FT + tid;
    if (e < total) {
      const int i = e / w4, k4 = e - i * w4;
      *reinterpret_cast<float4*>(&t.dst[i * t.ld + 4 * k4]) = v[u];
    }
  }
}

// Two matrices at once: both batches of loads are in flight before any store.
template <typename Ta, typename Tb>
__device__ __forceinline__ void load_rows2(const RowTile& ta, const Ta* sa, int va,
                                           const RowTile& tb, const Tb* sb, int vb, int tid) {
  const int na = (ta.n_rows * (ta.width >> 2) + RB * FT - 1) / (RB * FT);
  const int nb = (tb.n_rows * (tb.width >> 2) + RB * FT - 1) / (RB * FT);
  for (int pass = 0; pass < max(na, nb); ++pass) {
    float4 a[RB], b[RB];
    if (pass < na) fetch_rows(a, sa, ta.n_rows, va, ta.width, tid, pass);
    if (pass < nb) fetch_rows(b, sb, tb.n_rows, vb, tb.width, tid, pass);
    if (pass < na) put_rows(ta, a, tid, pass);
    if (pass < nb) put_rows(tb, b, tid, pass);
  }
}

// Four matrices at once (a tile with n_rows = 0 is skipped).
template <typename Ta, typename Tb, typename Tc, typename Td>
__device__ __forceinline__ void load_rows4(const RowTile& ta, const Ta* sa, int va,
                                           const RowTile& tb, const Tb* sb, int vb,
                                           const RowTile& tc, const Tc* sc, int vc,
                                           const RowTile& td, const Td* sd, int vd, int tid) {
  auto passes = [](const RowTile& t) { return (t.n_rows * (t.width >> 2) + RB * FT - 1) / (RB * FT); };
  const int na = passes(ta), nb = passes(tb), nc = passes(tc), nd = passes(td);
  const int np = max(max(na, nb), max(nc, nd));
  for (int pass = 0; pass < np; ++pass) {
    float4 a[RB], b[RB], c[RB], d[RB];
    if (pass < na) fetch_rows(a, sa, ta.n_rows, va, ta.width, tid, pass);
    if (pass < nb) fetch_rows(b, sb, tb.n_rows, vb, tb.width, tid, pass);
    if (pass < nc) fetch_rows(c, sc, tc.n_rows, vc, tc.width, tid, pass);
    if (pass < nd) fetch_rows(d, sd, td.n_rows, vd, td.width, tid, pass);
    if (pass < na) put_rows(ta, a, tid, pass);
    if (pass < nb) put_rows(tb, b, tid, pass);
    if (pass < nc) put_rows(tc, c, tid, pass);
    if (pass < nd) put_rows(td, d, tid, pass);
  }
}

template <typename Tio>
__device__ __forceinline__ void load_rows(const RowTile& t, const Tio* src, int n_valid, int tid) {
  const int n = (t.n_rows * (t.width >> 2) + RB * FT - 1) / (RB * FT);
  for (int pass = 0; pass < n; ++pass) {
    float4 v[RB];
    fetch_rows(v, src, t.n_rows, n_valid, t.width, tid, pass);
    put_rows(t, v, tid, pass);
  }
}

size_t fwd_smem_bytes(int din, int dout) {
  const int LDI = din + 4, LDO = dout + 4;
  return sizeof(float) * ((size_t)2 * dout * LDI + (size_t)FC * LDI + (size_t)FC * LDO +
                          (size_t)FC * LDC + (size_t)(FC + 1) * LDD + 2 * FC);
}

// Forward scan. y may be null (state sweep only); ckpt may be null. ckpt layout:
// float [B*H][n_chunks][d_out][d_in], the state at the start of each chunk.
template <typename Tio>
__global__ void __launch_bounds__(FT, 1) fwd_kernel(FwdArgs a) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  const int din = a.din, dout = a.dout, tid = threadIdx.x;
  const int LDI = din + 4, LDO = dout + 4;
  float* S = sm;
  float* W = S + dout * LDI;
  float* X = W + dout * LDI;
  float* G = X + FC * LDI;
  float* P = G + FC * LDO;
  float* Dt = P + FC * LDC;
  float* et = Dt + (FC + 1) * LDD;
  float* al = et + FC;

  // one CTA per (scan, segment); the segment walks chunks [c0, c1)
  const int bh = blockIdx.x / a.nseg, seg = blockIdx.x - bh * a.nseg, h = bh % a.H;
  const size_t tok0 = (size_t)bh * a.T;
  const int nch = (a.T + FC - 1) / FC;  // chunks of the whole scan (checkpoint indexing)
  const int c0 = seg * a.seg_chunks, c1 = min(nch, c0 + a.seg_chunks);
  const size_t seg_row = (size_t)bh * a.nseg + seg;
  const Tio* xg = static_cast<const Tio*>(a.x);
  const Tio* gg = static_cast<const Tio*>(a.g);
  Tio* yg = static_cast<Tio*>(a.y);
  const float* W0 = a.W0 + (size_t)h * dout * din;

  const float* S0 = a.S0 ? a.S0 + seg_row * dout * din : nullptr;
  for (int e = tid; e < dout * din; e += FT) {
    const int n = e / din, k = e - n * din;
    S[n * LDI + k] = S0 ? S0[e] : 0.f;
    W[n * LDI + k] = W0[e];
  }
  const int NG = dout / 4, NK4 = din / 4, NB4 = dout / 4;
  float lseg = 0.f;  // log2 of the product of alpha over the walked chunks (summary)

  for (int c = c0; c < c1; ++c) {
    const int t0 = c * FC;
    const int nt = min(FC, a.T - t0);
    __syncthreads();
    if (a.ckpt) {
      float* dst = a.ckpt + ((size_t)bh * nch + c) * dout * din;
      for (int e = tid; e < dout * din; e += FT) {
        const int n = e / din, k = e - n * din;
        dst[e] = S[n * LDI + k];
      }
    }
    if (tid < FC) {
      et[tid] = tid < nt ? a.eta[tok0 + t0 + tid] : 0.f;
      al[tid] = tid < nt ? a.alpha[tok0 + t0 + tid] : 1.f;
    }
    load_rows2(RowTile{X, LDI, FC, din}, xg + (tok0 + t0) * din, nt,
               RowTile{G, LDO, FC, dout}, gg + (tok0 + t0) * dout, nt, tid);
    __syncthreads();
    decay_table(Dt, al, tid);
    __syncthreads();

    if (yg) {
      // P_ij = (x_i . x_j) (-eta_j) D[i][j] for j < i (strictly causal), else 0. Threads
      // 0..127 take a 2 x 4 tile of X X^T each: rows i = ti + 16 q, j = tj + 8 r
      if (tid < 128) {
        const int ti = tid >> 3, tj = tid & 7;
        float acc[2][4];
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[q][r] = 0.f;
        for (int k = 0; k < din; k += 4) {
          float4 av[2], bv[4];
#pragma unroll
          for (int q = 0; q < 2; ++q) av[q] = *reinterpret_cast<const float4*>(&X[(ti + 16 * q) * LDI + k]);
#pragma unroll
          for (int r = 0; r < 4; ++r) bv[r] = *reinterpret_cast<const float4*>(&X[(tj + 8 * r) * LDI + k]);
#pragma unroll
          for (int q = 0; q < 2; ++q)
#pragma unroll
            for (int r = 0; r < 4; ++r) acc[q][r] += dot4(av[q], bv[r]);
        }
#pragma unroll
        for (int q = 0; q < 2; ++q)
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int i = ti + 16 * q, j = tj + 8 * r;
            P[i * LDC + j] = j < i ? acc[q][r] * (-et[j]) * Dt[i * LDD + j + 1] : 0.f;
          }
      }
      __syncthreads();
      // y_i = W0 x_i + D[i][-1] S_in x_i + sum_j P_ij g_j; thread tile 4 tokens x 4 outputs
      // (a wider tile than the reverse's: each W0 and S row it loads serves 4 tokens)
      for (int tile = tid; tile < (FC / 4) * NG; tile += FT) {
        const int ig = tile / NG, ng = tile - ig * NG;
        float a1[4][4], a2[4][4], a3[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int r = 0; r < 4; ++r) a1[q][r] = a2[q][r] = a3[q][r] = 0.f;
        for (int k = 0; k < din; k += 4) {
          float4 xv[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) xv[q] = *reinterpret_cast<const float4*>(&X[(ig * 4 + q) * LDI + k]);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float4 wv = *reinterpret_cast<const float4*>(&W[(ng + NG * r) * LDI + k]);
            const float4 sv = *reinterpret_cast<const float4*>(&S[(ng + NG * r) * LDI + k]);
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              a1[q][r] += dot4(xv[q], wv);
              a2[q][r] += dot4(xv[q], sv);
            }
          }
        }
        for (int j = 0; j < FC; ++j) {
          float gv[4];
#pragma unroll
          for (int r = 0; r < 4; ++r) gv[r] = G[j * LDO + ng + NG * r];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float pv = P[(ig * 4 + q) * LDC + j];
#pragma unroll
            for (int r = 0; r < 4; ++r) a3[q][r] = fmaf(pv, gv[r], a3[q][r]);
          }
        }
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int i = ig * 4 + q;
          if (i < nt) {
            const float gam = Dt[i * LDD];
#pragma unroll
            for (int r = 0; r < 4; ++r)
              yg[(tok0 + t0 + i) * dout + ng + NG * r] =
                  from_f32<Tio>(a1[q][r] + gam * a2[q][r] + a3[q][r]);
          }
        }
      }
      __syncthreads();
    }

    // carry: S <- D[FC][-1] S + sum_j (-eta_j D[FC][j]) g_j x_j^T
    const float gC = Dt[FC * LDD];
    lseg += log2f(gC);
    // item: 4 rows x 4 columns of the state, so that every thread has one at d = 64
    for (int item = tid; item < NB4 * NK4; item += FT) {
      const int nb = item / NK4, k4 = item - nb * NK4;
      float4 acc[4];
#pragma unroll
      for (int r = 0; r < 4; ++r) {
        const float4 s = *reinterpret_cast<const float4*>(&S[(nb * 4 + r) * LDI + 4 * k4]);
        acc[r] = make_float4(gC * s.x, gC * s.y, gC * s.z, gC * s.w);
      }
      for (int j = 0; j < nt; ++j) {
        const float w = -et[j] * Dt[FC * LDD + j + 1];
        const float4 xv = *reinterpret_cast<const float4*>(&X[j * LDI + 4 * k4]);
#pragma unroll
        for (int r = 0; r < 4; ++r) fma4(acc[r], w * G[j * LDO + nb * 4 + r], xv);
      }
#pragma unroll
      for (int r = 0; r < 4; ++r) *reinterpret_cast<float4*>(&S[(nb * 4 + r) * LDI + 4 * k4]) = acc[r];
    }
  }
  if (a.summary) {  // this segment's local end state and log-decay
    __syncthreads();
    float* dst = a.Sloc + seg_row * dout * din;
    for (int e = tid; e < dout * din; e += FT) {
      const int n = e / din, k = e - n * din;
      dst[e] = S[n * LDI + k];
    }
    if (tid == 0) a.segL[seg_row] = lseg;
  }
  if (a.ST && seg == a.nseg - 1) {  // the state after the last token (padded tokens left it unchanged)
    __syncthreads();
    float* dst = a.ST + (size_t)bh * dout * din;
    for (int e = tid; e < dout * din; e += FT) {
      const int n = e / din, k = e - n * din;
      dst[e] = S[n * LDI + k];
    }
  }
}

size_t bwd_smem_bytes(int din, int dout) {
  const int LDI = din + 4, LDO = dout + 4;
  const int NG = dout / 4, NK = din / 4;
  return sizeof(float) *
         ((size_t)2 * dout * LDI + (size_t)FC * LDI + (size_t)2 * FC * LDO + (size_t)5 * FC * LDC +
          (size_t)(FC + 1) * LDD + 2 * FC + (size_t)FC * (2 * NG + NK) + FT + 2 * FC + 4);
}

// Reverse scan. ckpt holds the chunk-start states (float [B*H][n_chunks][d_out][d_in]).
// dW0p receives this pair's sum_t u_t x_t^T (float [B*H][d_out][d_in]).
template <typename Tio>
__global__ void __launch_bounds__(FT, 1) bwd_kernel(BwdArgs a) {
  extern __shared__ float4 smem4[];
  float* sm = reinterpret_cast<float*>(smem4);
  const int din = a.din, dout = a.dout, tid = threadIdx.x;
  const int LDI = din + 4, LDO = dout + 4;
  const int NG = dout / 4, NK = din / 4, NB4 = dout / 4, NK4 = din / 4;
  float* L = sm;                    // Lam, [dout][LDI]
  float* Sin = L + dout * LDI;      // chunk-start state
  float* X = Sin + dout * LDI;      // [FC][LDI]
  float* G = X + FC * LDI;          // [FC][LDO]
  float* U = G + FC * LDO;          // [FC][LDO]
  float* K = U + FC * LDO;          // x_i . x_j
  float* Kug = K + FC * LDC;        // u_i . g_j
  float* Ar = Kug + FC * LDC;       // r intra weights
  float* Z = Ar + FC * LDC;         // dx intra weights
  float* Q = Z + FC * LDC;          // (u_s.g_j)(x_s.x_j)
  float* Dt = Q + FC * LDC;
  float* et = Dt + (FC + 1) * LDD;
  float* al = et + FC;
  float* qpart = al + FC;           // [FC][NG]
  float* epart = qpart + FC * NG;   // [FC][NG]
  float* ppart = epart + FC * NG;   // [FC][NK]
  float* red = ppart + FC * NK;     // [FT]
  float* qv = red + FT;             // [FC]
  float* pv = qv + FC;              // [FC]
  float* Esh = pv + FC;             // [1]

  // one CTA per (scan, segment); the segment walks chunks c1 - 1 down to c0
  const int bh = blockIdx.x / a.nseg, seg = blockIdx.x - bh * a.nseg, h = bh % a.H;
  const size_t tok0 = (size_t)bh * a.T;
  const int nch = (a.T + FC - 1) / FC;  // chunks of the whole scan (checkpoint indexing)
  const int c0 = seg * a.seg_chunks, c1 = min(nch, c0 + a.seg_chunks);
  const size_t seg_row = (size_t)bh * a.nseg + seg;
  const bool full = !a.summary;  // outputs, not just the adjoint carry
  const Tio* xg = static_cast<const Tio*>(a.x);
  const Tio* gg = static_cast<const Tio*>(a.g);
  const Tio* ug = static_cast<const Tio*>(a.dy);
  Tio* dxg = static_cast<Tio*>(a.dx);
  Tio* dgg = static_cast<Tio*>(a.dg);
  const float* W0 = a.W0 + (size_t)h * dout * din;

  const float* LamT = a.LamT ? a.LamT + seg_row * dout * din : nullptr;
  for (int e = tid; e < dout * din; e += FT) {
    const int n = e / din, k = e - n * din;
    L[n * LDI + k] = LamT ? LamT[e] : 0.f;
  }
  // dW0 partial sums in registers: items of 4 rows x 4 columns, up to 4 per thread
  // (d_in d_out <= 16384)
  float4 dw[4][4];
#pragma unroll
  for (int it = 0; it < 4; ++it)
#pragma unroll
    for (int r = 0; r < 4; ++r) dw[it][r] = make_float4(0.f, 0.f, 0.f, 0.f);

  float lseg = 0.f;  // log2 of the product of alpha over the walked chunks (summary)
  for (int c = c1 - 1; c >= c0; --c) {
    const int t0 = c * FC;
    const int nt = min(FC, a.T - t0);
    __syncthreads();
    if (tid < FC) {
      et[tid] = tid < nt ? a.eta[tok0 + t0 + tid] : 0.f;
      al[tid] = tid < nt ? a.alpha[tok0 + t0 + tid] : 1.f;
    }
    // X and U always; G and the chunk-start state S_in (the checkpoint) for the outputs
    const float* src = full ? a.ckpt + ((size_t)bh * nch + c) * dout * din : nullptr;
    load_rows4(RowTile{X, LDI, FC, din}, xg + (tok0 + t0) * din, nt,
               RowTile{U, LDO, FC, dout}, ug + (tok0 + t0) * dout, nt,
               RowTile{G, LDO, full ? FC : 0, dout}, gg + (tok0 + t0) * dout, nt,
               RowTile{Sin, LDI, full ? dout : 0, din}, src, dout, tid);
    __syncthreads();
    decay_table(Dt, al, tid);
    if (full) {
    // Gram matrices of the chunk, K = X X^T and Kug = U G^T: threads 0..127 take a 4 x 4
    // tile each, rows i = ti + 8 q and j = tj + 8 r (neighbouring rows of a warp's loads
    // fall in different banks); threads 128..255 the partial sums of <Lam_end, S_in>
    if (tid < 128) {
      const int which = tid >> 6, t = tid & 63, ti = t >> 3, tj = t & 7;
      const float* A = which ? U : X;
      const float* Bm = which ? G : X;
      const int ld = which ? LDO : LDI, width = which ? dout : din;
      float acc[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) acc[q][r] = 0.f;
      for (int k = 0; k < width; k += 4) {
        float4 av[4], bv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          av[q] = *reinterpret_cast<const float4*>(&A[(ti + 8 * q) * ld + k]);
          bv[q] = *reinterpret_cast<const float4*>(&Bm[(tj + 8 * q) * ld + k]);
        }
#pragma unroll
        for (int q = 0; q < 4; ++q)
#pragma unroll
          for (int r = 0; r < 4; ++r) acc[q][r] += dot4(av[q], bv[r]);
      }
      float* Out = which ? Kug : K;
#pragma unroll
      for (int q = 0; q < 4; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) Out[(ti + 8 * q) * LDC + tj + 8 * r] = acc[q][r];
      red[tid] = 0.f;
    } else {  // <Lam_end, S_in>
      float acc = 0.f;
      for (int e = tid - 128; e < dout * din; e += FT - 128) {
        const int n = e / din, k = e - n * din;
        acc = fmaf(L[n * LDI + k], Sin[n * LDI + k], acc);
      }
      red[tid] = acc;
    }
    __syncthreads();
    for (int e = tid; e < FC * FC; e += FT) {
      const int i = e / FC, j = e - i * FC;
      // r_i intra: sum_{s>i} D[s][i] K_si u_s
      Ar[i * LDC + j] = (j > i) ? Dt[j * LDD + i + 1] * K[j * LDC + i] : 0.f;
      float z = 0.f;
      if (j < i) z = -et[j] * Dt[i * LDD + j + 1] * Kug[i * LDC + j];
      else if (j > i) z = -et[i] * Dt[j * LDD + i + 1] * Kug[j * LDC + i];
      Z[i * LDC + j] = z;
      // Q[j][s] for j < s (here i plays j, j plays s)
      Q[i * LDC + j] = (j > i) ? Kug[j * LDC + i] * K[j * LDC + i] : 0.f;
    }
    if (tid < 32) {  // the fixed-order sum of the partials of <Lam_end, S_in>
      float e8 = 0.f;
#pragma unroll
      for (int w = 0; w < FT / 32; ++w) e8 += red[32 * w + tid];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) e8 += __shfl_xor_sync(0xffffffffu, e8, o);
      if (tid == 0) Esh[0] = e8;
    }
    __syncthreads();

    // r = D[FC][i] (Lam_end x_i) + sum_{s>i} Ar[i][s] u_s ; dg = -eta r ; partial sums.
    // Thread tile: 2 tokens x 4 outputs n = ng + NG r (rows of Lam in neighbouring banks).
    for (int tile = tid; tile < (FC / 2) * NG; tile += FT) {
      const int ig = tile / NG, ng = tile - ig * NG;
      float r1[2][4], ri[2][4];
#pragma unroll
      for (int q = 0; q < 2; ++q)
#pragma unroll
        for (int r = 0; r < 4; ++r) r1[q][r] = ri[q][r] = 0.f;
      for (int k = 0; k < din; k += 4) {
        float4 xv[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) xv[q] = *reinterpret_cast<const float4*>(&X[(ig * 2 + q) * LDI + k]);
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 lv = *reinterpret_cast<const float4*>(&L[(ng + NG * r) * LDI + k]);
#pragma unroll
          for (int q = 0; q < 2; ++q) r1[q][r] += dot4(xv[q], lv);
        }
      }
      for (int s = 0; s < FC; ++s) {
        float uv[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) uv[r] = U[s * LDO + ng + NG * r];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const float w = Ar[(ig * 2 + q) * LDC + s];
#pragma unroll
          for (int r = 0; r < 4; ++r) ri[q][r] = fmaf(w, uv[r], ri[q][r]);
        }
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = ig * 2 + q;
        const float dl = Dt[FC * LDD + i + 1];
        float pe = 0.f, pq = 0.f;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const int n = ng + NG * r;
          const float rr = dl * r1[q][r] + ri[q][r];
          const float gv = G[i * LDO + n];
          pe = fmaf(gv, rr, pe);
          pq = fmaf(gv, r1[q][r], pq);
          if (i < nt) dgg[(tok0 + t0 + i) * dout + n] = from_f32<Tio>(-et[i] * rr);
        }
        epart[i * NG + ng] = pe;
        qpart[i * NG + ng] = pq;
      }
    }

    // dx_i = W0^T u_i + D[i][-1] S_in^T u_i - eta_i D[FC][i] Lam_end^T g_i + sum_j Z_ij x_j.
    // Thread tile: 2 tokens x 4 contiguous columns k = 4 kg .. 4 kg + 3 (16-byte rows).
    for (int tile = tid; tile < (FC / 2) * NK; tile += FT) {
      const int ig = tile / NK, kg = tile - ig * NK;
      const int k0 = 4 * kg;
      float4 aw[2], as[2], alm[2], az[2];
#pragma unroll
      for (int q = 0; q < 2; ++q) aw[q] = as[q] = alm[q] = az[q] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int n = 0; n < dout; ++n) {
        float uq[2], gq[2];
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          uq[q] = U[(ig * 2 + q) * LDO + n];
          gq[q] = G[(ig * 2 + q) * LDO + n];
        }
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(&W0[(size_t)n * din + k0]));
        const float4 sv = *reinterpret_cast<const float4*>(&Sin[n * LDI + k0]);
        const float4 lv = *reinterpret_cast<const float4*>(&L[n * LDI + k0]);
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          fma4(aw[q], uq[q], w0);
          fma4(as[q], uq[q], sv);
          fma4(alm[q], gq[q], lv);
        }
      }
      for (int j = 0; j < FC; ++j) {
        const float4 xv = *reinterpret_cast<const float4*>(&X[j * LDI + k0]);
#pragma unroll
        for (int q = 0; q < 2; ++q) fma4(az[q], Z[(ig * 2 + q) * LDC + j], xv);
      }
#pragma unroll
      for (int q = 0; q < 2; ++q) {
        const int i = ig * 2 + q;
        const float gam = Dt[i * LDD];
        const float ed = et[i] * Dt[FC * LDD + i + 1];
        const float4 xi = *reinterpret_cast<const float4*>(&X[i * LDI + k0]);
        ppart[i * NK + kg] = dot4(xi, as[q]);
        if (i < nt) {
          const float o0 = aw[q].x + gam * as[q].x - ed * alm[q].x + az[q].x;
          const float o1 = aw[q].y + gam * as[q].y - ed * alm[q].y + az[q].y;
          const float o2 = aw[q].z + gam * as[q].z - ed * alm[q].z + az[q].z;
          const float o3 = aw[q].w + gam * as[q].w - ed * alm[q].w + az[q].w;
          Tio* o = dxg + (tok0 + t0 + i) * din + k0;
          o[0] = from_f32<Tio>(o0);
          o[1] = from_f32<Tio>(o1);
          o[2] = from_f32<Tio>(o2);
          o[3] = from_f32<Tio>(o3);
        }
      }
    }
    __syncthreads();
    if (tid < FC) {
      const int i = tid;
      float se = 0.f, sq = 0.f, sp = 0.f;
      for (int e = 0; e < NG; ++e) {
        se += epart[i * NG + e];
        sq += qpart[i * NG + e];
      }
      for (int e = 0; e < NK; ++e) sp += ppart[i * NK + e];
      qv[i] = sq;
      pv[i] = sp;
      if (i < nt) a.d_eta[tok0 + t0 + i] = -se;
    }
    // V_ij = sum_{s>i} D[s][i] Q[j][s] for j < i, on every thread (into K, whose last
    // readers, the chunk matrices, are done)
    float* V = K;
    for (int e = tid; e < FC * FC; e += FT) {
      const int i = e / FC, j = e - i * FC;
      float v = 0.f;
      if (j < i)
        for (int s2 = i + 1; s2 < FC; ++s2) v = fmaf(Dt[s2 * LDD + i + 1], Q[j * LDC + s2], v);
      V[i * LDC + j] = v;
    }
    __syncthreads();
    {
      // d_alpha_i = <Lam_{i+1}, S_i> as four cross terms (see file header): warp w takes
      // rows 4w .. 4w+3, lane l the term j = l (t2, t4) and s = l (t3); fixed-order sums
      const int w = tid >> 5, l = tid & 31;
      for (int i = (FC / 8) * w; i < (FC / 8) * (w + 1); ++i) {
        const float aij = l < i ? -et[l] * Dt[i * LDD + l + 1] : 0.f;
        const float bis = l > i ? Dt[l * LDD + i + 1] : 0.f;
        float t2 = aij * qv[l], t4 = aij * V[i * LDC + l], t3 = bis * pv[l];
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
          t2 += __shfl_xor_sync(0xffffffffu, t2, o);
          t3 += __shfl_xor_sync(0xffffffffu, t3, o);
          t4 += __shfl_xor_sync(0xffffffffu, t4, o);
        }
        if (l == 0 && i < nt) {
          const float gam = Dt[i * LDD], dl = Dt[FC * LDD + i + 1];
          a.d_alpha[tok0 + t0 + i] = gam * dl * Esh[0] + dl * t2 + gam * t3 + t4;
        }
      }
    }
    } else {
      __syncthreads();  // the decay table is complete
    }
    // Lam <- D[FC][-1] Lam + sum_s D[s][-1] u_s x_s^T ; dW0 += sum_s u_s x_s^T
    const float gC = Dt[FC * LDD];
    lseg += log2f(gC);
#pragma unroll
    for (int it = 0; it < 4; ++it) {
      const int item = tid + it * FT;
      if (item < NB4 * NK4) {
        const int nb = item / NK4, k4 = item - nb * NK4;
        float4 acc[4];
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const float4 l = *reinterpret_cast<const float4*>(&L[(nb * 4 + r) * LDI + 4 * k4]);
          acc[r] = make_float4(gC * l.x, gC * l.y, gC * l.z, gC * l.w);
        }
        for (int s = 0; s < nt; ++s) {
          const float gs = Dt[s * LDD];
          const float4 xv = *reinterpret_cast<const float4*>(&X[s * LDI + 4 * k4]);
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const float uv = U[s * LDO + nb * 4 + r];
            fma4(acc[r], gs * uv, xv);
            if (full) fma4(dw[it][r], uv, xv);
          }
        }
#pragma unroll
        for (int r = 0; r < 4; ++r) *reinterpret_cast<float4*>(&L[(nb * 4 + r) * LDI + 4 * k4]) = acc[r];
      }
    }
  }
  if (!full) {  // this segment's local adjoint and log-decay
    __syncthreads();
    float* dl = a.Lloc + seg_row * dout * din;
    for (int e = tid; e < dout * din; e += FT) {
      const int n = e / din, k = e - n * din;
      dl[e] = L[n * LDI + k];
    }
    if (tid == 0) a.segL[seg_row] = lseg;
    return;
  }
  if (a.dS0 && seg == 0) {  // the adjoint at the first token
    __syncthreads();
    float* ds = a.dS0 + (size_t)bh * dout * din;
    for (int e = tid; e < dout * din; e += FT) {
      const int n = e / din, k = e - n * din;
      ds[e] = L[n * LDI + k];
    }
  }
  // this (scan, segment)'s dW0 partial: [b][seg][h], summed over b and seg in a fixed order
  const int bb = bh / a.H;
  float* dst = a.dW0_part + (((size_t)bb * a.nseg + seg) * a.H + h) * dout * din;
#pragma unroll
  for (int it = 0; it < 4; ++it) {
    const int item = tid + it * FT;
    if (item < NB4 * NK4) {
      const int nb = item / NK4, k4 = item - nb * NK4;
#pragma unroll
      for (int r = 0; r < 4; ++r)
        *reinterpret_cast<float4*>(&dst[(size_t)(nb * 4 + r) * din + 4 * k4]) = dw[it][r];
    }
  }
}

// dW0[h] = sum_{b=0..B-1} part[b][h] in a fixed order (deterministic).
__global__ void reduce_dW0_kernel(const float* __restrict__ part, float* __restrict__ dW0, int B,
                                  int H, int dd) {
  const size_t n = (size_t)H * dd;
  for (size_t e = (size_t)blockIdx.x * blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int b = 0; b < B; ++b) s += part[(size_t)b * n + e];
    dW0[e] = s;
  }
}

// The dynamic shared-memory opt-in is per kernel and device; it is raised only when a launch
// needs more than the largest size set so far (kernel k, device dev < 64).
static cudaError_t ensure_smem(const void* kernel, int k, size_t smem) {
  static std::atomic<int> set[4][64];
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  if (dev >= 0 && dev < 64 && set[k][dev].load() >= (int)smem) return cudaSuccess;
  const cudaError_t e =
      cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && dev >= 0 && dev < 64) {
    int cur = set[k][dev].load();
    while (cur < (int)smem && !set[k][dev].compare_exchange_weak(cur, (int)smem)) {
    }
  }
  return e;
}

template <typename Tio>
static cudaError_t launch_fwd_t(const FwdArgs& a, cudaStream_t st) {
  const size_t smem = fwd_smem_bytes(a.din, a.dout);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(fwd_kernel<Tio>),
                              std::is_same<Tio, float>::value ? 0 : 1, smem);
  if (e != cudaSuccess) return e;
  fwd_kernel<Tio><<<a.B * a.H * a.nseg, FT, smem, st>>>(a);
  count_launch();
  return cudaGetLastError();
}

template <typename Tio>
static cudaError_t launch_bwd_t(const BwdArgs& a, cudaStream_t st) {
  const size_t smem = bwd_smem_bytes(a.din, a.dout);
  cudaError_t e = ensure_smem(reinterpret_cast<const void*>(bwd_kernel<Tio>),
                              std::is_same<Tio, float>::value ? 2 : 3, smem);
  if (e != cudaSuccess) return e;
  bwd_kernel<Tio><<<a.B * a.H * a.nseg, FT, smem, st>>>(a);
  count_launch();
  e = cudaGetLastError();
  if (e != cudaSuccess || a.summary) return e;
  const int dd = a.din * a.dout;
  const size_t n = (size_t)a.H * dd;
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  reduce_dW0_kernel<<<blocks, 256, 0, st>>>(a.dW0_part, a.dW0, a.B * a.nseg, a.H, dd);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_reduce_dW0(const float* part, float* dW0, int B, int H, int dd,
                              cudaStream_t st) {
  const size_t n = (size_t)H * dd;
  const int blocks = (int)((n + 255) / 256 < 1184 ? (n + 255) / 256 : 1184);
  reduce_dW0_kernel<<<blocks, 256, 0, st>>>(part, dW0, B, H, dd);
  count_launch();
  return cudaGetLastError();
}

cudaError_t launch_fwd(const FwdArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_fwd_t<__nv_bfloat16>(a, st) : launch_fwd_t<float>(a, st);
}

cudaError_t launch_bwd(const BwdArgs& a, bool bf16, cudaStream_t st) {
  return bf16 ? launch_bwd_t<__nv_bfloat16>(a, st) : launch_bwd_t<float>(a, st);
}

size_t ckpt_bytes(int B, int H, int T, int din, int dout) {
  const size_t nch = (size_t)(T + FC - 1) / FC;
  return (size_t)B * H * nch * din * dout * sizeof(float);
}

size_t dW0_part_bytes(int B, int H, int din, int dout) {
  return (size_t)B * H * din * dout * sizeof(float);
}

bool shape_ok(int din, int dout) {
  return din % 4 == 0 && dout % 8 == 0 && din >= 8 && dout >= 8 && din * dout <= 16384 &&
         bwd_smem_bytes(din, dout) <= 227 * 1024 && fwd_smem_bytes(din, dout) <= 227 * 1024;
}

}  // namespace ffma
}  // namespace gradlev
