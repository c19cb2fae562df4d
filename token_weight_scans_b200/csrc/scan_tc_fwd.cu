// Tensor-core (tcgen05/TMEM) forward GradLev scan for bf16 I/O, d_in = 128 and
// d_out a multiple of 128 (one CTA per (b, h, 128-wide slice of d_out)).
//
// Method (Cognaptus, "Parallelize the Training, Keep the Learning Serial",
// section "Once the gradient signals are known, the weight trajectory becomes
// parallelizable"; GradLev abstract): S_0 = 0, y_t = (W0 + S_t) x_t,
// S_{t+1} = alpha_t S_t - eta_t g_t x_t^T. The deviation is a discounted sum
// of rank-one updates, so within a chunk of C = 64 tokens starting at c0,
// with L_j = sum_{r<=j} log2 alpha_{c0+r} (chunk-local):
//
//   y_i = W0 x_i + 2^{L_{i-1}} S x_i + sum_{j<i} (x_i.x_j) (-eta_j) 2^{L_{i-1}-L_j} g_j
//   S'  = 2^{L_{C-1}} S + sum_j (-eta_j 2^{L_{C-1}-L_j}) g_j x_j^T
//
// Products (the output ones d-major: d_out on the 128 TMEM lanes, the chunk's
// tokens on the columns, so that every product but the Gram one has M = 128):
//   K     = X X^T                        (M=64 tokens, N=64, K=d_in)        -> TMEM
//   P_ij  = K_ij (-eta_j) 2^{L_{i-1}-L_j} (j < i), bf16 in shared memory
//   Y1^T  = W0 X^T + G^T P^T             (M=128, N=64, K=d_in then C; W0 is a
//                                         bf16 A operand kept in TMEM)      -> TMEM
//   Y2^T  = S X^T                        (M=128, N=64, K=d_in)              -> TMEM
//   dS    = G^T Xhat, Xhat_j = w_j x_j   (M=128, N=d_in, K=C)               -> TMEM
//   y_i   = Y1^T[:, i] + 2^{L_{i-1}} Y2^T[:, i];  S <- 2^{L_{C-1}} S + dS (fp32, registers)
//
// Warp roles (20 warps), each running through the chunks on its own, tied by
// mbarriers so that the roles overlap across chunks:
//   0      TMA producer (X and G tiles, 4 stages)
//   1      MMA issuer and TMEM owner
//   2      gate prep (log2 alpha cumulative sums, prefetched) + half of Xhat
//   3      the other half of Xhat (double-buffered)
//   4..7   mask: K -> P for each chunk, a chunk ahead of the output products
//   8..15  state: the fp32 state in registers (warpgroup h owns columns
//          [64h, 64h+64)), its bf16 copy for the S X^T product and the
//          chunk-start checkpoints (TMA-stored from that copy)
//   16..19 output epilogue: y from Y1^T and Y2^T, transposed into the chunk's
//          X tile (free by then) and TMA-stored
// Without y (state-carry summaries, checkpoint-only sweeps) only the producer,
// MMA, gate/Xhat and state roles run.

#include <cuda.h>
#include <cuda_bf16.h>
#include <atomic>

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include "common.cuh"
#include "scan_tc.h"
#include "sm100.cuh"

namespace gradlev {
namespace tc {

using namespace sm100;

namespace {

constexpr int C = 64;          // tokens per chunk
constexpr int NS = 4;          // TMA stages (X and G tiles)
constexpr int GS = 4;          // gate slots
constexpr int NTHREADS = 640;  // 20 warps
constexpr int TILE = C * 128;  // bytes of one [64 rows x 128 B] swizzled block
constexpr int BIG = 128 * 128; // bytes of one [128 rows x 128 B] swizzled block

// TMEM columns (512 allocated).
//   [0, 64)    K, an M=64 product: rows in lanes 0-15 of each 32-lane sub-partition
//   [64, 128)  W0 slice as a bf16 A operand (lane n = row n, two k per column)
//   [128, 384) two output buffers of 128 columns: Y1^T in the first 64, Y2^T in the next 64
//   [384, 512) dS
constexpr uint32_t COL_K = 0;
constexpr uint32_t COL_W0 = 64;
constexpr uint32_t COL_Y = 128;
constexpr uint32_t COL_DS = 384;

// With M = L_{31}, the mask factor -eta_j 2^{L_{i-1} - L_j} = ra_i ca_j whenever
// every exponent stays inside fp32 range: fac = (|L_{C-1}| <= 120).
struct GateSlot {
  float L[C];     // chunk-local inclusive cumulative sum of log2 alpha
  float eta[C];
  float gam[C];   // 2^{L_{i-1}}
  float w[C];     // -eta_j 2^{L_{C-1} - L_j}
  float ra[C];    // 2^{L_{i-1} - M}
  float ca[C];    // -eta_j 2^{M - L_j}
  float gC;       // 2^{L_{C-1}}
  int fac;
  float pad[2];
};

struct Smem {
  // 1024-byte aligned tiles first
  uint8_t X[NS][2 * TILE];     // k-blocks [0,64), [64,128): 64 token rows x 128 B; after the
                               // chunk's products, the y staging tile (n-blocks of the slice)
  uint8_t G[NS][2 * TILE];     // n-blocks of the slice: 64 token rows x 128 B
  uint8_t S[2][BIG];           // [k-block]: 128 n rows x 128 B (bf16 state)
  uint8_t Xh[2][2 * TILE];     // [buffer] scaled X, same layout as X
  uint8_t P[2][TILE];          // [buffer] 64 token rows (i) x 128 B (j)
  GateSlot gates[GS];
  uint64_t full[NS], empty[NS];
  uint64_t gfull[GS], gempty[GS];
  uint64_t kfull, kfree;
  uint64_t xhready[2], xhfree[2];
  uint64_t pready[2], pfree[2];
  uint64_t yfull[2], yfree[2];
  uint64_t dsfull, dsfree, sready, sfree, done;
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "over the 227 KB of shared memory a CTA may use");

// where-codes of the bounded waits (role << 8 | site)
enum : uint32_t {
  W_TMA_EMPTY = 0x001, W_TMA_DRAIN = 0x002,
  W_MMA_FULL = 0x101, W_MMA_KFREE, W_MMA_YFREE, W_MMA_XREADY, W_MMA_DSFREE, W_MMA_PREADY,
  W_MMA_SREADY, W_MMA_DONE,
  W_GATE_EMPTY = 0x201,
  W_XH_FULL = 0x301, W_XH_GFULL, W_XH_FREE,
  W_K_GFULL = 0x401, W_K_KFULL, W_K_PFREE,
  W_S_DSFULL = 0x501, W_S_SFREE,
  W_E_YFULL = 0x601, W_E_GFULL,
};

constexpr uint32_t BAR_EPI = 2;  // named barrier of the four epilogue warps

}  // namespace

__global__ void __launch_bounds__(NTHREADS, 1)
    fwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG,
               const __grid_constant__ CUtensorMap tmY, const __grid_constant__ CUtensorMap tmS,
               TcFwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nslice = p.dout >> 7;
  const int unit = blockIdx.x / p.nseg, seg = blockIdx.x - unit * p.nseg;
  const int bh = unit / nslice, slice = unit - bh * nslice;
  const int h = bh % p.H;
  const int n0 = slice * 128;
  const int T = p.T;
  const int nch_all = (T + C - 1) / C;           // chunks of the whole sequence
  const int c0 = seg * p.seg_chunks;             // this CTA's segment: chunks [c0, c1)
  const int c1 = min(nch_all, c0 + p.seg_chunks);
  const int nch = c1 - c0;                       // chunks this CTA walks
  // global chunk of the c-th chunk walked (a reverse summary walks the segment backwards)
  auto cg = [&](int c) { return p.reverse ? c1 - 1 - c : c0 + c; };
  const size_t seg_row = (size_t)bh * p.nseg + seg;  // [bh][seg] index of the segment states
  const WaitCtx wc{&sm.abort, p.status, p.timeout_ns};
  // y outputs (and with them the Gram, mask, output products and epilogue)
  const bool yout = !p.summary && p.y != nullptr;
  const bool has_ck = !p.summary && p.ckpt != nullptr;

  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    for (int g = 0; g < GS; ++g) {
      mbar_init(&sm.gfull[g], 32);
      // Xhat warps (2) + state warps (8) [+ mask warps (4) + epilogue warps (4)]
      mbar_init(&sm.gempty[g], yout ? 18 : 10);
    }
    mbar_init(&sm.kfull, 1);
    mbar_init(&sm.kfree, 4);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&sm.xhready[b], 2);
      mbar_init(&sm.xhfree[b], 1);
      mbar_init(&sm.pready[b], 4);
      mbar_init(&sm.pfree[b], 1);
      mbar_init(&sm.yfull[b], 1);
      mbar_init(&sm.yfree[b], 4);
    }
    mbar_init(&sm.dsfull, 1);
    mbar_init(&sm.dsfree, 8);
    mbar_init(&sm.sready, 8);
    mbar_init(&sm.sfree, 1);
    mbar_init(&sm.done, 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmG);
    if (yout) prefetch_tmap(&tmY);
    if (has_ck) prefetch_tmap(&tmS);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;
  if (yout && warp >= 4 && warp < 8) {
    // the bf16 W0 slice into TMEM (A operand of W0 X^T): lane n = row n, column c holds
    // elements 2c and 2c + 1
    const int q = warp & 3, n = 32 * q + lane;
    const float* W0r = p.W0 + ((size_t)h * p.dout + n0 + n) * 128;
#pragma unroll
    for (int hf = 0; hf < 2; ++hf) {
      float v[32];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const float4 a = *reinterpret_cast<const float4*>(W0r + 64 * hf + 2 * e);
        const float4 b = *reinterpret_cast<const float4*>(W0r + 64 * hf + 2 * e + 4);
        v[e] = __uint_as_float(pack_bf16(a.x, a.y));
        v[e + 1] = __uint_as_float(pack_bf16(a.z, a.w));
        v[e + 2] = __uint_as_float(pack_bf16(b.x, b.y));
        v[e + 3] = __uint_as_float(pack_bf16(b.z, b.w));
      }
      tmem_st32(tbase + COL_W0 + ((uint32_t)(32 * q) << 16) + 32 * hf, v);
    }
    tmem_st_wait();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    int issued = 0;
    if (lane == 0) {
      for (int c = 0; c < nch; ++c) {
        const int s = c % NS;
        if (!mbar_wait(&sm.empty[s], ((c / NS) & 1) ^ 1, wc, W_TMA_EMPTY)) break;
        mbar_arrive_expect_tx(&sm.full[s], 4 * TILE);
        const int t0 = cg(c) * C;
        tma_load_3d(sm.X[s], &tmX, &sm.full[s], 0, t0, bh);
        tma_load_3d(sm.X[s] + TILE, &tmX, &sm.full[s], 64, t0, bh);
        tma_load_3d(sm.G[s], &tmG, &sm.full[s], n0, t0, bh);
        tma_load_3d(sm.G[s] + TILE, &tmG, &sm.full[s], n0 + 64, t0, bh);
        issued = c + 1;
      }
      // teardown: let every load this thread issued land before the CTA exits
      for (int c = issued > NS ? issued - NS : 0; c < issued; ++c)
        mbar_drain(&sm.full[c % NS], (c / NS) & 1, wc, W_TMA_DRAIN);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_k = idesc_bf16(64, 64, false, false);    // X X^T
      const uint32_t id_y = idesc_bf16(128, 64, false, false);   // W0 X^T (W0 in TMEM), S X^T
      const uint32_t id_gp = idesc_bf16(128, 64, true, false);   // G^T P^T (G n-contiguous)
      const uint32_t id_ds = idesc_bf16(128, 128, true, true);   // G^T Xhat
      const uint32_t sS = smem_u32(sm.S[0]);
      // K_c (the mask warps have read K_{c-1})
      auto issue_k = [&](int c) -> bool {
        const int s = c % NS;
        if (!mbar_wait(&sm.full[s], (c / NS) & 1, wc, W_MMA_FULL)) return false;
        if (!mbar_wait(&sm.kfree, (c & 1) ^ 1, wc, W_MMA_KFREE)) return false;
        tc_fence_after();
        const uint32_t sX = smem_u32(sm.X[s]);
        const uint64_t dX = sw128_desc(sX, 16, 1024);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t off = (kk >> 2) * TILE + (kk & 3) * 32;
          umma_bf16(tbase + COL_K, desc_at(dX, off), desc_at(dX, off), id_k, kk > 0);
        }
        if (!(p.inject == 1 && c == 1)) umma_commit(&sm.kfull);
        return true;
      };
      bool ok = true;
      if (yout && nch > 0) ok = issue_k(0);
      for (int c = 0; c < nch && ok; ++c) {
        const int s = c % NS, b = c & 1;
        const uint32_t sX = smem_u32(sm.X[s]), sG = smem_u32(sm.G[s]);
        const uint32_t sXh = smem_u32(sm.Xh[b]);
        // ---- dS_c = G^T Xhat (the state warps have read dS_{c-1})
        if (!(ok = mbar_wait(&sm.full[s], (c / NS) & 1, wc, W_MMA_FULL))) break;
        if (!(ok = mbar_wait(&sm.xhready[b], (c >> 1) & 1, wc, W_MMA_XREADY))) break;
        if (!(ok = mbar_wait(&sm.dsfree, (c & 1) ^ 1, wc, W_MMA_DSFREE))) break;
        tc_fence_after();
        {
          const uint64_t dG = sw128_desc(sG, TILE, 1024), dXh = sw128_desc(sXh, TILE, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_DS, desc_at(dG, kk * 2048), desc_at(dXh, kk * 2048), id_ds,
                      kk > 0);
        }
        if (!(p.inject == 3 && c == 1)) umma_commit(&sm.dsfull);
        umma_commit(&sm.xhfree[b]);
        if (!yout) {  // state carry only: the stage is free once dS has read it
          umma_commit(&sm.empty[s]);
          continue;
        }
        // ---- K of the next chunk (the mask warps build its P while chunk c's products run)
        if (c + 1 < nch && !(ok = issue_k(c + 1))) break;
        // ---- Y1^T_c = W0 X^T + G^T P^T into buffer b (the epilogue of chunk c - 2 read it)
        const uint32_t tY1 = tbase + COL_Y + 128 * b, tY2 = tY1 + 64;
        if (!(ok = mbar_wait(&sm.yfree[b], ((c >> 1) & 1) ^ 1, wc, W_MMA_YFREE))) break;
        tc_fence_after();
        {
          const uint64_t dX = sw128_desc(sX, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16_tmem_a(tY1, tbase + COL_W0 + 8 * kk,
                             desc_at(dX, (kk >> 2) * TILE + (kk & 3) * 32), id_y, kk > 0);
        }
        if (!(ok = mbar_wait(&sm.pready[b], (c >> 1) & 1, wc, W_MMA_PREADY))) break;
        tc_fence_after();
        {
          const uint64_t dG = sw128_desc(sG, TILE, 1024), dP = sw128_desc(smem_u32(sm.P[b]), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tY1, desc_at(dG, kk * 2048), desc_at(dP, kk * 32), id_gp, 1);
        }
        umma_commit(&sm.pfree[b]);
        // ---- Y2^T_c = S_c X^T (S_c written by the state update of chunk c - 1)
        if (!(ok = mbar_wait(&sm.sready, c & 1, wc, W_MMA_SREADY))) break;
        tc_fence_after();
        {
          const uint64_t dX = sw128_desc(sX, 16, 1024), dS = sw128_desc(sS, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t aoff = (kk >> 2) * BIG + (kk & 3) * 32;
            const uint32_t boff = (kk >> 2) * TILE + (kk & 3) * 32;
            umma_bf16(tY2, desc_at(dS, aoff), desc_at(dX, boff), id_y, kk > 0);
          }
        }
        umma_commit(&sm.sfree);
        umma_commit(&sm.yfull[b]);
      }
      // teardown: every issued MMA completes before TMEM is released
      umma_commit(&sm.done);
      mbar_drain(&sm.done, 0, wc, W_MMA_DONE);
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------ gates + scaled X
    // Warp 2 also prepares the gates of each chunk (alpha / eta prefetched PD chunks
    // ahead so the global-load latency is off the chain); both warps then write
    // half of Xhat = w (.) X with packed bf16 multiplies.
    constexpr int PD = 4;
    const size_t gbase = (size_t)bh * T;
    const bool gate_warp = warp == 2;
    float ra[PD][2], re[PD][2];
    float Lseg = 0.f;  // sum of log2 alpha over the walked chunks (lane-uniform)
    // gates of the c-th walked chunk (alpha = 1, eta = 0 past the walk or past T)
    auto gate_load = [&](int c, float (&a)[2], float (&e)[2]) {
      const bool in = c < nch;
      const int t0 = (in ? cg(c) : 0) * C + lane, t1 = t0 + 32;
      a[0] = in && t0 < T ? p.alpha[gbase + t0] : 1.f;
      a[1] = in && t1 < T ? p.alpha[gbase + t1] : 1.f;
      e[0] = in && t0 < T ? p.eta[gbase + t0] : 0.f;
      e[1] = in && t1 < T ? p.eta[gbase + t1] : 0.f;
    };
    if (gate_warp) {
#pragma unroll
      for (int k = 0; k < PD; ++k) gate_load(k, ra[k], re[k]);
    }
    bool ok = true;
    for (int cb = 0; cb < nch && ok; cb += PD) {
#pragma unroll
      for (int k = 0; k < PD; ++k) {
        const int c = cb + k;
        if (c >= nch) break;
        const int s = c % NS, g = c % GS;
        GateSlot& gs = sm.gates[g];
        if (gate_warp) {
          if (!mbar_wait_warp(&sm.gempty[g], ((c / GS) & 1) ^ 1, wc, W_GATE_EMPTY)) { ok = false; break; }
          const float a0 = ra[k][0], a1 = ra[k][1], e0 = re[k][0], e1 = re[k][1];
          gate_load(c + PD, ra[k], re[k]);  // prefetch chunk c + PD into this register slot
          float l0 = fmaxf(log2f(a0), -100.f), l1 = fmaxf(log2f(a1), -100.f);
#pragma unroll
          for (int o = 1; o < 32; o <<= 1) {
            const float u0 = __shfl_up_sync(0xffffffffu, l0, o);
            const float u1 = __shfl_up_sync(0xffffffffu, l1, o);
            if (lane >= o) {
              l0 += u0;
              l1 += u1;
            }
          }
          const float last0 = __shfl_sync(0xffffffffu, l0, 31);
          l1 += last0;
          const float Lend = __shfl_sync(0xffffffffu, l1, 31);
          Lseg += Lend;
          const float pm0 = __shfl_up_sync(0xffffffffu, l0, 1);
          const float pm1 = __shfl_up_sync(0xffffffffu, l1, 1);
          gs.L[lane] = l0;
          gs.L[lane + 32] = l1;
          gs.eta[lane] = e0;
          gs.eta[lane + 32] = e1;
          gs.gam[lane] = lane == 0 ? 1.f : exp2f(pm0);
          gs.gam[lane + 32] = exp2f(lane == 0 ? last0 : pm1);
          gs.w[lane] = -e0 * exp2f(Lend - l0);
          gs.w[lane + 32] = -e1 * exp2f(Lend - l1);
          gs.ra[lane] = exp2f((lane == 0 ? 0.f : pm0) - last0);
          gs.ra[lane + 32] = exp2f((lane == 0 ? last0 : pm1) - last0);
          gs.ca[lane] = -e0 * exp2f(last0 - l0);
          gs.ca[lane + 32] = -e1 * exp2f(last0 - l1);
          if (lane == 0) {
            gs.gC = exp2f(Lend);
            gs.fac = (Lend >= -120.f) ? 1 : 0;
          }
          __syncwarp();
          mbar_arrive(&sm.gfull[g]);
        }
        if (!mbar_wait_warp(&sm.full[s], (c / NS) & 1, wc, W_XH_FULL)) { ok = false; break; }
        if (!mbar_wait_warp(&sm.gfull[g], (c / GS) & 1, wc, W_XH_GFULL)) { ok = false; break; }
        if (!mbar_wait_warp(&sm.xhfree[c & 1], ((c >> 1) & 1) ^ 1, wc, W_XH_FREE)) { ok = false; break; }
        const uint32_t src = smem_u32(sm.X[s]), dst = smem_u32(sm.Xh[c & 1]);
#pragma unroll 4
        for (int idx = (warp - 2) * 32 + lane; idx < 2 * TILE / 16; idx += 64) {
          const uint32_t off = idx * 16;
          const int j = (off & (TILE - 1)) >> 7;  // token row
          // forward: -eta_j 2^{L_{C-1}-L_j}; reverse (adjoint) summary: 2^{L_{j-1}}
          const __nv_bfloat162 w2 = __float2bfloat162_rn(p.reverse ? gs.gam[j] : gs.w[j]);
          const uint32_t wv = *reinterpret_cast<const uint32_t*>(&w2);
          uint4 v = ld_shared_v4(src + off);
          v.x = hmul2_bf16(v.x, wv);
          v.y = hmul2_bf16(v.y, wv);
          v.z = hmul2_bf16(v.z, wv);
          v.w = hmul2_bf16(v.w, wv);
          st_shared_v4(dst + off, v.x, v.y, v.z, v.w);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&sm.xhready[c & 1]);
          mbar_arrive(&sm.gempty[g]);
        }
      }
    }
    if (ok && gate_warp && lane == 0 && p.seg_L && slice == 0) p.seg_L[seg_row] = Lseg;
  } else if (warp < 8) {
    // ------------------------------------------------------------ mask warps
    // Warp q: token rows [16q, 16q+16) of K, in lanes 0-15 of its sub-partition.
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    bool ok = true;
    for (int c = 0; c < nch && yout && ok; ++c) {
      const int g = c % GS, b = c & 1;
      const GateSlot& gs = sm.gates[g];
      ok = ok && mbar_wait_warp(&sm.gfull[g], (c / GS) & 1, wc, W_K_GFULL);
      ok = ok && mbar_wait_warp(&sm.kfull, c & 1, wc, W_K_KFULL);
      // P buffer b was last read by the G^T P^T product of chunk c - 2
      ok = ok && mbar_wait_warp(&sm.pfree[b], ((c >> 1) & 1) ^ 1, wc, W_K_PFREE);
      if (!ok) break;
      tc_fence_after();
      const bool mine = lane < 16;
      const int i = 16 * q + (lane & 15);
      const uint32_t prow = smem_u32(sm.P[b]);
      const float Lm1 = i == 0 ? 0.f : gs.L[i - 1];
      const float rai = gs.ra[i];
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        float v[32];
        tmem_ld32(tbase + COL_K + lane_off + 32 * hf, v);
        tmem_ld_wait();
        if (hf == 1) {
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.kfree);
        }
        if (mine) {
          uint32_t pk[16];
          if (gs.fac) {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int j = 32 * hf + e;
              const float p0 = (j < i) ? v[e] * rai * gs.ca[j] : 0.f;
              const float p1 = (j + 1 < i) ? v[e + 1] * rai * gs.ca[j + 1] : 0.f;
              pk[e >> 1] = pack_bf16(p0, p1);
            }
          } else {
#pragma unroll
            for (int e = 0; e < 32; e += 2) {
              const int j = 32 * hf + e;
              const float f0 = exp2f(fminf(Lm1 - gs.L[j], 0.f));
              const float f1 = exp2f(fminf(Lm1 - gs.L[j + 1], 0.f));
              const float p0 = (j < i) ? v[e] * (-gs.eta[j]) * f0 : 0.f;
              const float p1 = (j + 1 < i) ? v[e + 1] * (-gs.eta[j + 1]) * f1 : 0.f;
              pk[e >> 1] = pack_bf16(p0, p1);
            }
          }
#pragma unroll
          for (int cc = 0; cc < 4; ++cc)
            st_shared_v4(prow + sw128_off(i, 4 * hf + cc), pk[4 * cc], pk[4 * cc + 1],
                         pk[4 * cc + 2], pk[4 * cc + 3]);
        }
      }
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.pready[b]);
        mbar_arrive(&sm.gempty[g]);
      }
    }
  } else if (warp < 16) {
    // ------------------------------------------------------------ state warps
    const int q = warp & 3;          // TMEM lane quadrant
    const int hh = (warp - 8) >> 2;  // warpgroup: state columns [64hh, 64hh+64)
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int n = 32 * q + lane;     // row of the d_out slice owned by this thread
    const uint32_t srow = smem_u32(sm.S[hh]);
    float Sreg[64];  // fp32 state: row n, columns [64hh, 64hh+64)
    if (p.S_init) {
      const float4* si = reinterpret_cast<const float4*>(
          p.S_init + (seg_row * p.dout + n0 + n) * 128 + 64 * hh);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float4 v = si[e];
        Sreg[4 * e] = v.x;
        Sreg[4 * e + 1] = v.y;
        Sreg[4 * e + 2] = v.z;
        Sreg[4 * e + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 64; ++e) Sreg[e] = 0.f;
    }
    const bool copy = yout || has_ck;  // the bf16 copy feeds S X^T and the checkpoints
    // bf16 copy of the state (row n, this warpgroup's k-block) into the S tile
    auto write_copy = [&]() {
#pragma unroll
      for (int cc = 0; cc < 8; ++cc)
        st_shared_v4(srow + sw128_off(n, cc), pack_bf16(Sreg[8 * cc], Sreg[8 * cc + 1]),
                     pack_bf16(Sreg[8 * cc + 2], Sreg[8 * cc + 3]),
                     pack_bf16(Sreg[8 * cc + 4], Sreg[8 * cc + 5]),
                     pack_bf16(Sreg[8 * cc + 6], Sreg[8 * cc + 7]));
      fence_proxy_async_smem();
      __syncwarp();
    };
    // Each warp TMA-stores the 32 rows it wrote, one k-block wide, as its part of the
    // chunk-start checkpoint (bf16 [bh][chunk][dout][din], box of 32 rows).
    auto store_ck = [&](int gchunk) {
      if (lane == 0) {
        tma_store_3d(&tmS, sm.S[hh] + (uint32_t)(32 * q) * 128, 64 * hh, n0 + 32 * q,
                     bh * nch_all + gchunk);
        tma_store_commit();
      }
    };
    if (copy) {  // S at the segment's first chunk
      write_copy();
      if (lane == 0) mbar_arrive(&sm.sready);
      if (has_ck) store_ck(c0);
    }
    bool ok = true;
    for (int c = 0; c < nch; ++c) {
      const int g = c % GS;
      const GateSlot& gs = sm.gates[g];
      ok = ok && mbar_wait_warp(&sm.dsfull, c & 1, wc, W_S_DSFULL);
      if (!ok) break;
      tc_fence_after();
      const float gC = gs.gC;
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) {
        float v[16];
        tmem_ld16(tbase + COL_DS + lane_off + 64 * hh + 16 * qq, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) Sreg[16 * qq + e] = fmaf(gC, Sreg[16 * qq + e], v[e]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&sm.dsfree);
        mbar_arrive(&sm.gempty[g]);
      }
      if (!copy || c + 1 == nch) continue;  // no copy after the last chunk
      // the S X^T product of chunk c has read the old copy, and so has the last
      // checkpoint store from it
      if (yout) ok = ok && mbar_wait_warp(&sm.sfree, c & 1, wc, W_S_SFREE);
      if (!ok) break;
      if (has_ck && lane == 0) tma_store_wait_read();
      __syncwarp();
      write_copy();
      if (lane == 0) mbar_arrive(&sm.sready);
      if (has_ck) store_ck(cg(c) + 1);
    }
    if (lane == 0) tma_store_wait_all();
    if (ok && p.S_final) {  // the state after the walked chunks, fp32
      float4* so = reinterpret_cast<float4*>(p.S_final + (seg_row * p.dout + n0 + n) * 128 + 64 * hh);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        so[e] = make_float4(Sreg[4 * e], Sreg[4 * e + 1], Sreg[4 * e + 2], Sreg[4 * e + 3]);
    }
    if (ok && !p.summary && p.S_last && seg == p.nseg - 1) {  // S_T: padded tokens left it unchanged
      float4* so = reinterpret_cast<float4*>(p.S_last + ((size_t)bh * p.dout + n0 + n) * 128 + 64 * hh);
#pragma unroll
      for (int e = 0; e < 16; ++e)
        so[e] = make_float4(Sreg[4 * e], Sreg[4 * e + 1], Sreg[4 * e + 2], Sreg[4 * e + 3]);
    }
  } else {
    // ------------------------------------------------------------ output epilogue
    // Thread (q, lane) owns output row n = 32q + lane of the slice: Y1^T and Y2^T hold
    // y_i[n] for the chunk's 64 tokens i in its TMEM lane. y_i[n] is staged into
    // row i of the chunk's X tile (free once the chunk's products are done): lanes
    // n and n^1 exchange one value per token pair, so each writes a bf16 pair.
    // Every epilogue warp runs every iteration and reaches the named barrier, also
    // after a failed wait, so that none is left waiting at it.
    const int q = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int n = 32 * q + lane;
    const bool odd = lane & 1;
    const int ne = n & ~1;                       // the pair's first column
    const uint32_t nb = (uint32_t)(ne >> 6) * TILE;  // n-block of the staging tile
    const uint32_t cb = (uint32_t)((ne & 63) * 2);   // byte offset inside the 128-byte row
    const bool leader = warp == 16 && lane == 0;
    bool ok = true;
    int prev_s = -1;  // stage whose y store is still reading it
    for (int c = 0; c < nch && yout; ++c) {
      const int s = c % NS, g = c % GS, b = c & 1;
      const GateSlot& gs = sm.gates[g];
      if (leader && prev_s >= 0) {  // the last chunk's y store has read its stage
        tma_store_wait_read();
        mbar_arrive(&sm.empty[prev_s]);
        prev_s = -1;
      }
      ok = ok && mbar_wait_warp(&sm.gfull[g], (c / GS) & 1, wc, W_E_GFULL);
      ok = ok && mbar_wait_warp(&sm.yfull[b], (c >> 1) & 1, wc, W_E_YFULL);
      if (ok) {
        tc_fence_after();
        const uint32_t tY = tbase + COL_Y + 128 * b + lane_off;
        const uint32_t xs = smem_u32(sm.X[s]) + nb;
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          float v1[16], v2[16];
          tmem_ld16(tY + 16 * k, v1);
          tmem_ld16(tY + 64 + 16 * k, v2);
          tmem_ld_wait();
          if (k == 3) {
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&sm.yfree[b]);
          }
#pragma unroll
          for (int e = 0; e < 16; e += 2) {
            const int i0 = 16 * k + e;
            const float ya = fmaf(gs.gam[i0], v2[e], v1[e]);          // y_{i0}[n]
            const float yb = fmaf(gs.gam[i0 + 1], v2[e + 1], v1[e + 1]);  // y_{i0+1}[n]
            // the even lane keeps token i0 and receives y_{i0}[n+1]; the odd lane keeps
            // token i0 + 1 and receives y_{i0+1}[n-1]
            const float r = __shfl_xor_sync(0xffffffffu, odd ? ya : yb, 1);
            const int row = odd ? i0 + 1 : i0;
            const uint32_t w = odd ? pack_bf16(r, yb) : pack_bf16(ya, r);
            st_shared_b32(xs + row * 128 + ((((cb >> 4) ^ (row & 7)) << 4) | (cb & 15)), w);
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.gempty[g]);
      }
      named_bar_sync(BAR_EPI, 128);
      if (leader && ok) {  // the stage goes back to the producer once this store has read it
        tma_store_3d(&tmY, sm.X[s], n0, cg(c) * C, bh);
        tma_store_3d(&tmY, sm.X[s] + TILE, n0 + 64, cg(c) * C, bh);
        tma_store_commit();
        prev_s = s;
      }
    }
    if (leader) {
      tma_store_wait_all();
      if (prev_s >= 0) mbar_arrive(&sm.empty[prev_s]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  }
  return fn;
}

// 3-D bf16 map over [d2][d1][d0] (d0 innermost), box {64, box1, 1}, 128-byte swizzle.
bool make_map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t box1) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {d0 * 2, d0 * d1 * 2};
  cuuint32_t box[3] = {64, box1, 1};
  cuuint32_t es[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides,
                  box, es, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool fwd_shape_ok(int din, int dout) { return din == 128 && dout % 128 == 0 && dout <= 256; }

size_t ckpt_bytes(int B, int H, int T, int din, int dout) {
  const size_t nch = (size_t)(T + C - 1) / C;
  return (size_t)B * H * nch * dout * din * sizeof(__nv_bfloat16);
}

cudaError_t launch_fwd(const TcFwdParams& prm, const void* x, const void* g, cudaStream_t st) {
  CUtensorMap mx, mg, my, ms;
  const uint64_t BH = (uint64_t)prm.B * prm.H;
  const uint64_t nch = (uint64_t)(prm.T + C - 1) / C;
  // The y and checkpoint maps are only used when those outputs are requested; g
  // stands in as a well-formed base otherwise.
  if (!make_map_bf16_3d(&mx, x, prm.din, prm.T, BH, C) ||
      !make_map_bf16_3d(&mg, g, prm.dout, prm.T, BH, C) ||
      !make_map_bf16_3d(&my, prm.y ? (const void*)prm.y : g, prm.dout, prm.T, BH, C) ||
      !make_map_bf16_3d(&ms, prm.ckpt ? (const void*)prm.ckpt : g, 128, prm.dout,
                        prm.ckpt ? BH * nch : 1, 32))
    return cudaErrorInvalidValue;
  // The shared-memory opt-in is a per-device attribute: set it once on each device.
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(fwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  const int grid = prm.B * prm.H * (prm.dout / 128) * prm.nseg;
  fwd_kernel<<<grid, NTHREADS, kSmemBytes, st>>>(mx, mg, my, ms, prm);
  count_launch();
  return cudaGetLastError();
}

size_t fwd_smem_bytes() { return kSmemBytes; }

}  // namespace tc
}  // namespace gradlev
