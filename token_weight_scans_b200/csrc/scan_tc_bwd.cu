// Tensor-core (tcgen05/TMEM) reverse GradLev scan for bf16 I/O, d_in = 128 and
// one 128-row slice of d_out per launch.
//
// Reverse-mode derivative of S_{t+1} = alpha_t S_t - eta_t g_t x_t^T,
// y_t = (W0 + S_t) x_t (Cognaptus, "Parallelize the Training, Keep the Learning
// Serial", section "Once the gradient signals are known, the weight trajectory
// becomes parallelizable"; GradLev abstract: the reverse backpropagation is a
// scan too). With u = dL/dy and the state adjoint Lam_t = alpha_t Lam_{t+1} + u_t x_t^T:
//   dx_t = (W0 + S_t)^T u_t - eta_t Lam_{t+1}^T g_t,  dg_t = -eta_t Lam_{t+1} x_t,
//   deta_t = -g_t . Lam_{t+1} x_t,  dalpha_t = <Lam_{t+1}, S_t>,  dW0 = sum u_t x_t^T.
//
// One CTA per (b, h) walks the 64-token chunks backwards, carrying Lam (fp32 in
// TMEM, a bf16 copy in shared memory). The chunk-start state S_in comes from
// the bf16 checkpoints of the forward scan. Inside a chunk (local i, with
// L_j = sum_{r<=j} log2 alpha, gam_i = 2^{L_{i-1}}, del_i = 2^{L_{C-1}-L_i},
// a_ij = -eta_j 2^{L_{i-1}-L_j} (j<i), b_is = 2^{L_{s-1}-L_i} (s>i)):
//   r_i  = del_i Lam x_i + sum_{s>i} b_is (x_s.x_i) u_s
//   dx_i = W0^T u_i + gam_i S_in^T u_i - eta_i del_i Lam^T g_i + sum_j Z_ij x_j
//   Z_ij = a_ij (u_i.g_j) (j<i),  -eta_i b_ij (g_i.u_j) (j>i)
//   deta_i = -(del_i q_i + t_i), q_i = g_i^T Lam x_i, t_i = sum_{s>i} b_is (x_i.x_s)(g_i.u_s)
//   dalpha_i = gam_i del_i <Lam,S_in> + del_i sum_{j<i} a_ij q_j + gam_i sum_{s>i} b_is p_s
//              + sum_{j<i} a_ij V_ij,  p_s = u_s^T S_in x_s,
//   V_ij = sum_{s>i} b_is Q_js, Q_js = (u_s.g_j)(x_s.x_j) (j<s)
//   Lam <- 2^{L_{C-1}} Lam + sum_s gam_s u_s x_s^T ;  dW0 += sum_s u_s x_s^T
// (dalpha is the exact four-term expansion of <Lam_{i+1}, S_i>; no division by alpha.)
//
// Products (d on the 128 TMEM lanes, tokens on the columns; M=64 ones use the
// two 16-lane halves of each TMEM sub-partition):
//   phase 1: K = X X^T | Kug = U G^T (M=64), KugT = G U^T (M=64), dW0 += U^T X,
//            DXb = U S_in, R1 = X Lam^T (M=64, token-major)
//   phase 2: V^T = Bm Q^T (M=64), r += Ar U, dx += U W0 + Z X + Gs Lam (token-major)
//   phase 3: Lam += U^T Xg
// where Ar, Z, Q^T, Bm are built by the math warps from K, Kug, KugT into the
// shared memory that held S_in, Gs = diag(-eta del) G is written in place once
// the unscaled G has been used, and Xg = diag(gam) X is a tile of its own that
// the math warps write as soon as X arrives. The fp32 adjoint Lam
// lives in TMEM: the math warps scale it by 2^{L_{C-1}} in place and the MMA
// accumulates U^T Xg onto it; likewise the rows del_i R1_i and gam_i DXb_i are
// written back so that the remaining terms accumulate onto them (r and dx).
//
// Warp roles (20 warps): 0 TMA producer and gate prep, 1..3 three MMA issuers
// (1 owns TMEM), 4..19 four math warpgroups (warpgroup w: tokens [16w, 16w+16) of
// each chunk and state columns [32w, 32w+32)).
//
// A tcgen05.mma is issued by one thread, and that thread shares its scheduler
// with the math warps of its TMEM lane quadrant: with those warps busy, one
// thread's issue rate drops several-fold. The 76 products of a chunk are
// therefore split over three issuers on three schedulers (A: the Gram products,
// dW0, V^T; B: the r accumulator and the Lam update; C: the dx accumulator), so
// that each accumulator has a single issuer.
//
// A later slice of d_out (accumulate) adds its dx to the earlier slices' by one bulk
// reduction per chunk in L2 (staged row-major) and its d_eta and d_alpha by atomic
// adds, one per element, so that no load of the earlier values sits on its chain;
// with one add per element onto a completed launch's result, the sums do not depend
// on timing.

#include <cuda.h>
#include <cuda_bf16.h>
#include <atomic>

#include <cuda_runtime.h>
#include <cudaTypedefs.h>

#include <type_traits>

#include "common.cuh"
#include "scan_tc.h"
#include "sm100.cuh"

namespace gradlev {
namespace tc {

bool make_map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t box1);

using namespace sm100;

namespace {

constexpr int C = kChunk;       // 64 tokens per chunk
constexpr int NS = 2;           // stages of the X, G, U tiles
constexpr int GS = 2;           // gate slots
constexpr int NMATH = 16;                   // math warps: 4 warpgroups
constexpr int NTHREADS = 128 + 32 * NMATH;  // + TMA, MMA, gate and helper warps
constexpr int TILE = C * 128;   // [64 rows x 128 B] swizzled block
constexpr int BIG = 128 * 128;  // [128 rows x 128 B] swizzled block

// TMEM columns (512 allocated)
constexpr uint32_t COL_KK = 0;    // K (lanes 0-15 of each sub-partition) | Kug (lanes 16-31)
constexpr uint32_t COL_KT = 64;   // KugT (lanes 0-15) | V^T (lanes 16-31)
// r and dx are token-major M=64 products (token row i at lane 32 (i/16) + i%16):
// r in the lower 16 lanes and dx in the upper 16 lanes of the same 128 columns, so
// one load gives a warp the r and dx rows of the same tokens.
constexpr uint32_t COL_RX = 128;  // R1 -> del (.) R1 -> + Ar U = r  |  DXb -> gam (.) DXb -> + ... = dx
constexpr uint32_t COL_L = 256;   // Lam, fp32 (128 columns)
constexpr uint32_t COL_W = 384;   // dW0 accumulator (128 columns)
constexpr uint32_t LANE16 = 16u << 16;

// chunk-by-chunk matrices built by the math warps, aliased onto the S_in tile
constexpr int CC_AR = 0, CC_Z = TILE, CC_QT = 2 * TILE, CC_BM = 3 * TILE;

// Per-chunk gate quantities (16-byte aligned rows for vector loads). With M = L_{31} (mid-chunk) the decay factors
// split into row and column factors, a_ij = ra_i ca_j and b_ij = rb_i cb_j, as
// long as every exponent stays inside fp32 range: fac = (|L_{C-1}| <= 120).
struct alignas(16) GateSlot {
  float L[C];
  float eta[C];
  float gam[C];
  float del[C];
  float ra[C];   // 2^{L_{i-1} - M}
  float ca[C];   // -eta_j 2^{M - L_j}
  float rb[C];   // 2^{M - L_i}
  float cb[C];   // 2^{L_{j-1} - M}
  float gC;
  int fac;
  float pad[2];
};

struct Smem {
  uint8_t X[NS][2 * TILE];    // [s rows][k]: k-blocks
  uint8_t G[NS][2 * TILE];    // [s rows][n]: n-blocks
  uint8_t U[NS][2 * TILE];    // [s rows][n]
  // Two regions that swap roles every chunk. Chunk it loads S_in into SL[it & 1], builds
  // its chunk matrices (Ar | Z | Q^T | Bm) there once S_in is read, and leaves the bf16
  // Lam for the next chunk there once those are read; it reads the bf16 Lam of the chunk
  // before from SL[(it & 1) ^ 1], which then takes the next S_in.
  uint8_t SL[2][2 * BIG];     // [k-block][n rows x 128 B]
  uint8_t W0[2 * BIG];        // [k-block][n rows x 128 B]
  uint8_t Xg[2 * TILE];       // diag(gam) X for the Lam update, same layout as X
  GateSlot gates[GS];
  float redq[4][C], redp[4][C];
  float tv[4][C], t2v[4][C], t3v[4][C], hv[4][C];
  alignas(16) float qv[C];
  alignas(16) float pv[C];
  alignas(16) float ered[2][NMATH];  // by chunk parity: the d_alpha of chunk it reads its
                                     // slots while faster warps start chunk it + 1
  uint64_t xfull[NS], xempty[NS];
  uint64_t staged[NS];  // the dg / dx staging tiles of the stage are written
  uint64_t gfull[GS], gempty[GS];
  uint64_t sfull;  // S_in tile loaded
  uint64_t ccfull, b1full, b2full;
  uint64_t m1a, m1done, m2done, lscaled, xgready, lbfree, lbready, done[3];
  uint32_t tmem_base;
  int abort;
};

constexpr size_t kSmemBytes = sizeof(Smem) + 1024;
static_assert(kSmemBytes <= 227 * 1024, "over the 227 KB of shared memory a CTA may use");

enum : uint32_t {
  W_TMA_XEMPTY = 0x001, W_TMA_SEMPTY, W_TMA_DRAIN, W_TMA_STAGED,
  W_MMA_XFULL = 0x101, W_MMA_M2, W_MMA_SFULL, W_MMA_LB, W_MMA_M1, W_MMA_XS, W_MMA_DONE,
  W_MMA_M1A,
  W_GATE_EMPTY = 0x201, W_XG_FULL, W_XG_GFULL, W_XG_FREE,
  W_M_GFULL = 0x401, W_M_CC, W_M_B1, W_M_B2,
};

__device__ __forceinline__ void named_sync_math() {
  asm volatile("bar.sync 1, %0;" ::"n"(32 * NMATH) : "memory");
}


}  // namespace

__global__ void __launch_bounds__(NTHREADS, 1)
    bwd_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmG,
               const __grid_constant__ CUtensorMap tmU, const __grid_constant__ CUtensorMap tmS,
               const __grid_constant__ CUtensorMap tmDX, const __grid_constant__ CUtensorMap tmDG,
               TcBwdParams p) {
  extern __shared__ uint8_t smem_raw[];
  Smem& sm = *reinterpret_cast<Smem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x / p.nseg, seg = blockIdx.x - bh * p.nseg, h = bh % p.H;
  const int T = p.T;
  const int nch_all = (T + C - 1) / C;         // chunks of the whole sequence
  const int c0 = seg * p.seg_chunks;           // this CTA's segment: chunks [c0, c1),
  const int c1 = min(nch_all, c0 + p.seg_chunks);  // walked from c1 - 1 down to c0
  const int nch = c1 - c0;
  const size_t seg_row = (size_t)bh * p.nseg + seg;  // [bh][seg] index of the segment adjoints
  const WaitCtx wc{&sm.abort, p.status, p.timeout_ns};

  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < NS; ++s) {
      mbar_init(&sm.xfull[s], 1);
      mbar_init(&sm.xempty[s], 4);  // the three issuers' last products on X, G, U + the dg / dx stores' read
      mbar_init(&sm.staged[s], 1);
    }
    for (int g = 0; g < GS; ++g) {
      mbar_init(&sm.gfull[g], 32);
      mbar_init(&sm.gempty[g], NMATH);
    }
    mbar_init(&sm.sfull, 1);
    mbar_init(&sm.lbfree, 2);  // R1 (issuer B) and Gs Lam (issuer C)
    mbar_init(&sm.ccfull, 1);
    mbar_init(&sm.b1full, 2);  // R1 (B) and DXb (C)
    mbar_init(&sm.b2full, 3);  // all three issuers
    mbar_init(&sm.m1a, NMATH);
    mbar_init(&sm.m1done, NMATH);
    mbar_init(&sm.m2done, NMATH);
    mbar_init(&sm.lscaled, NMATH);
    mbar_init(&sm.xgready, NMATH);
    mbar_init(&sm.lbready, NMATH);
    for (int i = 0; i < 3; ++i) mbar_init(&sm.done[i], 1);
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmX);
    prefetch_tmap(&tmG);
    prefetch_tmap(&tmU);
    prefetch_tmap(&tmS);
    prefetch_tmap(&tmDX);
    prefetch_tmap(&tmDG);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 512);
    tmem_relinquish();
  }
  if (warp >= 4) {
    // W0 -> bf16 swizzled [k-block][n rows]; the bf16 adjoint at the segment's end
    // (Lam_T = 0 for the last segment)
    const int t = threadIdx.x - 128;
    const float* W0 = p.W0 + ((size_t)h * p.dout + p.n0) * 128;
    for (int idx = t; idx < 128 * 16; idx += 32 * NMATH) {
      const int n = idx >> 4, ck = idx & 15;
      const int kb = ck >> 3, c = ck & 7;
      const float4 a = *reinterpret_cast<const float4*>(W0 + (size_t)n * 128 + ck * 8);
      const float4 b = *reinterpret_cast<const float4*>(W0 + (size_t)n * 128 + ck * 8 + 4);
      st_shared_v4(smem_u32(sm.W0 + kb * BIG) + sw128_off(n, c), pack_bf16(a.x, a.y),
                   pack_bf16(a.z, a.w), pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
      if (p.L_init) {
        const float* li = p.L_init + (seg_row * p.dout + p.n0 + n) * 128 + ck * 8;
        const float4 u = *reinterpret_cast<const float4*>(li);
        const float4 v = *reinterpret_cast<const float4*>(li + 4);
        st_shared_v4(smem_u32(sm.SL[1] + kb * BIG) + sw128_off(n, c), pack_bf16(u.x, u.y),
                     pack_bf16(u.z, u.w), pack_bf16(v.x, v.y), pack_bf16(v.z, v.w));
      } else {
        st_shared_v4(smem_u32(sm.SL[1] + kb * BIG) + sw128_off(n, c), 0u, 0u, 0u, 0u);
      }
    }
    fence_proxy_async_smem();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  if (warp < 4) {
    if (warp == 0) {
      // ---------------------------------------------------------- TMA producer + gate prep
      // Per chunk: lane 0 issues the tile loads (X, G, U into the stage, then S_in into
      // the region the chunk before left its bf16 Lam in), then the warp prepares the
      // gates, whose alpha / eta were loaded one chunk ahead.
      const size_t gbase = (size_t)bh * T;
      int xi = 0, si = 0;
      bool ok = true;
      float a0 = 1.f, a1 = 1.f, e0 = 0.f, e1 = 0.f;  // gates of the chunk prepared next
      auto gate_load = [&](int it, float& x0, float& x1, float& y0, float& y1) {
        const int c = c1 - 1 - it, t0 = c * C + lane, t1 = t0 + 32;
        const bool in = it < nch;
        x0 = in && t0 < T ? p.alpha[gbase + t0] : 1.f;
        x1 = in && t1 < T ? p.alpha[gbase + t1] : 1.f;
        y0 = in && t0 < T ? p.eta[gbase + t0] : 0.f;
        y1 = in && t1 < T ? p.eta[gbase + t1] : 0.f;
      };
      auto store_staged = [&](int j) -> bool {
        const int sj = j % NS, t0j = (c1 - 1 - j) * C;
        if (!mbar_wait(&sm.staged[sj], (j / NS) & 1, wc, W_TMA_STAGED)) return false;
        tma_store_3d(&tmDG, sm.G[sj], p.n0, t0j, bh);
        tma_store_3d(&tmDG, sm.G[sj] + TILE, p.n0 + 64, t0j, bh);
        if (!p.accumulate) {
          tma_store_3d(&tmDX, sm.U[sj], 0, t0j, bh);
          tma_store_3d(&tmDX, sm.U[sj] + TILE, 64, t0j, bh);
        } else {  // later slices: the staged rows (row-major) are added onto dx in L2
          const int rows = min(C, T - t0j);
          bulk_reduce_add_bf16(p.dx + ((size_t)bh * T + t0j) * 128, sm.U[sj], (uint32_t)rows * 256u);
        }
        tma_store_commit();
        tma_store_wait_read();
        mbar_arrive(&sm.xempty[sj]);
        return true;
      };
      gate_load(0, a0, a1, e0, e1);
      for (int it = 0; it < nch && ok; ++it) {
        const int c = c1 - 1 - it, st = it % NS, g = it % GS;
        int tok = 1;
        if (lane == 0) {
          // dg and dx of chunk it - NS, staged in this stage's G and U tiles; the stage is
          // free for chunk it once the stores have read them (rows past T are clipped)
          if (it >= NS && !store_staged(it - NS)) {
            tok = 0;
          } else if (!mbar_wait(&sm.xempty[st], ((it / NS) & 1) ^ 1, wc, W_TMA_XEMPTY)) {
            tok = 0;
          } else {
            mbar_arrive_expect_tx(&sm.xfull[st], 6 * TILE);
            tma_load_3d(sm.X[st], &tmX, &sm.xfull[st], 0, c * C, bh);
            tma_load_3d(sm.X[st] + TILE, &tmX, &sm.xfull[st], 64, c * C, bh);
            tma_load_3d(sm.G[st], &tmG, &sm.xfull[st], p.n0, c * C, bh);
            tma_load_3d(sm.G[st] + TILE, &tmG, &sm.xfull[st], p.n0 + 64, c * C, bh);
            tma_load_3d(sm.U[st], &tmU, &sm.xfull[st], p.n0, c * C, bh);
            tma_load_3d(sm.U[st] + TILE, &tmU, &sm.xfull[st], p.n0 + 64, c * C, bh);
            xi = it + 1;
            // S_in goes to SL[it & 1], which last held the bf16 Lam that chunk it - 1 read:
            // load once that chunk's last products on it have completed
            if (it > 0 && !mbar_wait(&sm.lbfree, (it - 1) & 1, wc, W_TMA_SEMPTY)) {
              tok = 0;
            } else {
              mbar_arrive_expect_tx(&sm.sfull, 2 * BIG);
              tma_load_3d(sm.SL[it & 1], &tmS, &sm.sfull, 0, p.n0, bh * nch_all + c);
              tma_load_3d(sm.SL[it & 1] + BIG, &tmS, &sm.sfull, 64, p.n0, bh * nch_all + c);
              si = it + 1;
            }
          }
        }
        ok = __shfl_sync(0xffffffffu, tok, 0) != 0;
        ok = ok && mbar_wait_warp(&sm.gempty[g], ((it / GS) & 1) ^ 1, wc, W_GATE_EMPTY);
        if (!ok) break;
        GateSlot& gs = sm.gates[g];
        const float x0 = a0, x1 = a1, y0 = e0, y1 = e1;
        gate_load(it + 1, a0, a1, e0, e1);  // the next chunk's gates, in flight meanwhile
        float l0 = fmaxf(log2f(x0), -100.f), l1 = fmaxf(log2f(x1), -100.f);
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
        const float pm0 = __shfl_up_sync(0xffffffffu, l0, 1);
        const float pm1 = __shfl_up_sync(0xffffffffu, l1, 1);
        gs.L[lane] = l0;
        gs.L[lane + 32] = l1;
        gs.eta[lane] = y0;
        gs.eta[lane + 32] = y1;
        gs.gam[lane] = lane == 0 ? 1.f : exp2f(pm0);
        gs.gam[lane + 32] = exp2f(lane == 0 ? last0 : pm1);
        gs.del[lane] = exp2f(Lend - l0);
        gs.del[lane + 32] = exp2f(Lend - l1);
        {
          const float Mid = last0;  // L_{31}
          const float lm0 = lane == 0 ? 0.f : pm0, lm1 = lane == 0 ? last0 : pm1;  // L_{i-1}
          gs.ra[lane] = exp2f(lm0 - Mid);
          gs.ra[lane + 32] = exp2f(lm1 - Mid);
          gs.ca[lane] = -y0 * exp2f(Mid - l0);
          gs.ca[lane + 32] = -y1 * exp2f(Mid - l1);
          gs.rb[lane] = exp2f(Mid - l0);
          gs.rb[lane + 32] = exp2f(Mid - l1);
          gs.cb[lane] = exp2f(lm0 - Mid);
          gs.cb[lane + 32] = exp2f(lm1 - Mid);
        }
        if (lane == 0) {
          gs.gC = exp2f(Lend);
          gs.fac = (Lend >= -120.f) ? 1 : 0;
        }
        __syncwarp();
        mbar_arrive(&sm.gfull[g]);
      }
      if (lane == 0) {
        // the last chunks' dg and dx
        for (int j = nch > NS ? nch - NS : 0; ok && j < nch; ++j) ok = store_staged(j);
        tma_store_wait_all();
        for (int it = xi > NS ? xi - NS : 0; it < xi; ++it)
          mbar_drain(&sm.xfull[it % NS], (it / NS) & 1, wc, W_TMA_DRAIN);
        if (si > 0) mbar_drain(&sm.sfull, (si - 1) & 1, wc, W_TMA_DRAIN);
      }
    } else if (lane == 0) {
      // ---------------------------------------------------------- MMA issuers
      // A (warp 1): the Gram products K | Kug and KugT, dW0, and V^T = Bm Q^T.
      // B (warp 2): the r accumulator (R1 = X Lam^T, then + Ar U) and the Lam update.
      // C (warp 3): the dx accumulator (DXb = U S_in, then + U W0 + Gs Lam + Z X).
      // Each accumulator has one issuer; where one issuer's product follows another's
      // (a scaling pass of the math warps in between), the math warps' barrier orders them.
      const int ii = warp - 1;
      const uint32_t id_cc = idesc_bf16(64, 64, false, false);      // X X^T, U G^T, G U^T
      const uint32_t id_w = idesc_bf16(128, 128, true, true);       // U^T X, U^T Xg
      const uint32_t id_tb = idesc_bf16(64, 128, false, true);      // U S_in, U W0, Ar U, ...
      const uint32_t id_r1 = idesc_bf16(64, 128, false, false);     // X Lam^T
      const uint32_t id_v = idesc_bf16(64, 64, false, true);        // Bm Q^T
      const uint32_t sW0 = smem_u32(sm.W0);
      bool ok = true;
      for (int it = 0; it < nch && ok; ++it) {
        const int st = it % NS;
        const uint32_t sX = smem_u32(sm.X[st]), sG = smem_u32(sm.G[st]), sU = smem_u32(sm.U[st]);
        const uint32_t sS = smem_u32(sm.SL[it & 1]);        // S_in, then the chunk matrices
        const uint32_t sL = smem_u32(sm.SL[(it & 1) ^ 1]);  // the bf16 Lam of the chunk before
        ok = mbar_wait(&sm.xfull[st], (it / NS) & 1, wc, W_MMA_XFULL);
        if (!ok) break;
        if (ii == 0) {
          // K | Kug and dW0: the previous chunk's matrix build has read K | Kug
          ok = it == 0 || mbar_wait(&sm.m1done, (it - 1) & 1, wc, W_MMA_M1);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * TILE + (kk & 3) * 32;
            const uint64_t dX = desc_at(sw128_desc(sX, 16, 1024), off);
            umma_bf16(tbase + COL_KK, dX, dX, id_cc, kk > 0);
            umma_bf16(tbase + COL_KK + LANE16, desc_at(sw128_desc(sU, 16, 1024), off),
                      desc_at(sw128_desc(sG, 16, 1024), off), id_cc, kk > 0);
          }
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_W, desc_at(sw128_desc(sU, TILE, 1024), kk * 2048),
                      desc_at(sw128_desc(sX, TILE, 1024), kk * 2048), id_w, (it > 0 || kk > 0));
          // KugT: its columns neighbour V^T, which the previous output phase reads until m2done
          ok = it == 0 || mbar_wait(&sm.m2done, (it - 1) & 1, wc, W_MMA_M2);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t off = (kk >> 2) * TILE + (kk & 3) * 32;
            umma_bf16(tbase + COL_KT, desc_at(sw128_desc(sG, 16, 1024), off),
                      desc_at(sw128_desc(sU, 16, 1024), off), id_cc, kk > 0);
          }
          umma_commit(&sm.ccfull);  // the Gram products (the last readers of unscaled G)
          // V^T = Bm Q^T from the chunk matrices
          ok = mbar_wait(&sm.m1done, it & 1, wc, W_MMA_M1);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_KT + LANE16, desc_at(sw128_desc(sS, 16, 1024), CC_BM + kk * 32),
                      desc_at(sw128_desc(sS, TILE, 1024), CC_QT + kk * 2048), id_v, kk > 0);
        } else if (ii == 1) {
          // R1 = X Lam^T: r was read by the previous output phase, the bf16 Lam is in place
          ok = it == 0 || (mbar_wait(&sm.m2done, (it - 1) & 1, wc, W_MMA_M2) &&
                           mbar_wait(&sm.lbready, (it - 1) & 1, wc, W_MMA_LB));
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tbase + COL_RX, desc_at(sw128_desc(sX, 16, 1024), (kk >> 2) * TILE + (kk & 3) * 32),
                      desc_at(sw128_desc(sL, 16, 1024), (kk >> 2) * BIG + (kk & 3) * 32), id_r1, kk > 0);
          if (!(p.inject == 2 && it == 1)) umma_commit(&sm.b1full);
          umma_commit(&sm.lbfree);  // one of the two products reading the bf16 Lam
          // Lam += U^T Xg once the math warps have scaled Lam and written Xg
          ok = mbar_wait(&sm.lscaled, it & 1, wc, W_MMA_XS) && mbar_wait(&sm.xgready, it & 1, wc, W_MMA_XS);
          if (!ok) break;
          tc_fence_after();
          const uint32_t sXg = smem_u32(sm.Xg);
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_L, desc_at(sw128_desc(sU, TILE, 1024), kk * 2048),
                      desc_at(sw128_desc(sXg, TILE, 1024), kk * 2048), id_w, 1);
          // r = del (.) R1 + Ar U
          ok = mbar_wait(&sm.m1done, it & 1, wc, W_MMA_M1);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_RX, desc_at(sw128_desc(sS, 16, 1024), CC_AR + kk * 32),
                      desc_at(sw128_desc(sU, TILE, 1024), kk * 2048), id_tb, 1);
        } else {
          // DXb = U S_in: dx was read by the previous output phase, S_in has landed
          ok = (it == 0 || mbar_wait(&sm.m2done, (it - 1) & 1, wc, W_MMA_M2)) &&
               mbar_wait(&sm.sfull, it & 1, wc, W_MMA_SFULL);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tbase + COL_RX + LANE16, desc_at(sw128_desc(sU, 16, 1024), (kk >> 2) * TILE + (kk & 3) * 32),
                      desc_at(sw128_desc(sS, BIG, 1024), kk * 2048), id_tb, kk > 0);
          umma_commit(&sm.b1full);
          // dx = gam (.) DXb + U W0 + Gs Lam, once DXb is scaled and G is scaled in place
          ok = mbar_wait(&sm.m1a, it & 1, wc, W_MMA_M1A);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            umma_bf16(tbase + COL_RX + LANE16, desc_at(sw128_desc(sU, 16, 1024), (kk >> 2) * TILE + (kk & 3) * 32),
                      desc_at(sw128_desc(sW0, BIG, 1024), kk * 2048), id_tb, 1);
          if (!p.local) {
            #pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              umma_bf16(tbase + COL_RX + LANE16, desc_at(sw128_desc(sG, 16, 1024), (kk >> 2) * TILE + (kk & 3) * 32),
                        desc_at(sw128_desc(sL, BIG, 1024), kk * 2048), id_tb, 1);
          }
          umma_commit(&sm.lbfree);  // the other product reading the bf16 Lam
          // dx += Z X
          ok = mbar_wait(&sm.m1done, it & 1, wc, W_MMA_M1);
          if (!ok) break;
          tc_fence_after();
          #pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16(tbase + COL_RX + LANE16, desc_at(sw128_desc(sS, 16, 1024), CC_Z + kk * 32),
                      desc_at(sw128_desc(sX, TILE, 1024), kk * 2048), id_tb, 1);
        }
        umma_commit(&sm.b2full);      // this issuer's products of the chunk
        umma_commit(&sm.xempty[st]);  // its last reads of X, G and U
      }
      // teardown: every MMA this thread issued completes before TMEM is released
      umma_commit(&sm.done[ii]);
      mbar_drain(&sm.done[ii], 0, wc, W_MMA_DONE);
    }
  } else {
    // ------------------------------------------------------------ math warpgroups
    const int q = warp & 3;          // TMEM lane quadrant
    const int wg = (warp - 4) >> 2;  // warpgroup: tokens [16wg, +16), Lam columns [32wg, +32)
    const int mt = threadIdx.x - 128;
    const uint32_t lane_off = (uint32_t)(32 * q) << 16;
    const int n = 32 * q + lane;             // d row owned in the 128-lane products
    const int ir = 16 * q + (lane & 15);     // chunk row owned in the 64-row products
    const bool lo = lane < 16;
    const int j0w = 16 * wg;                 // first chunk token / column of this warpgroup
    const uint32_t tL = tbase + COL_L + lane_off + 32 * wg;  // this thread's Lam columns
    {  // the fp32 adjoint at the segment's end (Lam_T = 0 for the last segment)
      float z[32];
      if (p.L_init) {
        const float4* li = reinterpret_cast<const float4*>(
            p.L_init + (seg_row * p.dout + p.n0 + n) * 128 + 32 * wg);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          const float4 v = li[e];
          z[4 * e] = v.x;
          z[4 * e + 1] = v.y;
          z[4 * e + 2] = v.z;
          z[4 * e + 3] = v.w;
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) z[e] = 0.f;
      }
      tmem_st32(tL, z);
      tmem_st_wait();
    }

    // Every math thread executes the same sequence of named barriers in every
    // iteration, whatever happens to its waits: after a failed (timed-out or
    // aborted) wait the warp skips the work but keeps the barrier schedule, so no
    // warp can be left at a bar.sync that its peers never reach.
    bool ok = true;
    for (int it = 0; it < nch; ++it) {
      const int c = c1 - 1 - it, st = it % NS, g = it % GS;
      const GateSlot& gs = sm.gates[g];
      const int t0 = c * C;
      const size_t tokbase = (size_t)bh * T + t0;
      const uint32_t sX = smem_u32(sm.X[st]), sG = smem_u32(sm.G[st]);
      const uint32_t sS = smem_u32(sm.SL[it & 1]);  // S_in, then the chunk matrices
      ok = ok && mbar_wait_warp(&sm.gfull[g], (it / GS) & 1, wc, W_M_GFULL);
      ok = ok && mbar_wait_warp(&sm.xfull[st], (it / NS) & 1, wc, W_M_GFULL);
      if (ok) {
        // ---- Xg = diag(gam) X for the Lam update (the previous update has read Xg: the
        //      previous chunk's b2full covers it); two 16-byte pieces per thread
        const uint32_t dst = smem_u32(sm.Xg);
#pragma unroll
        for (int k = 0; k < (2 * TILE / 16) / (32 * NMATH); ++k) {
          const uint32_t off = (uint32_t)(mt + 32 * NMATH * k) * 16;
          const int sr = (off & (TILE - 1)) >> 7;  // token row
          const __nv_bfloat162 f2 = __float2bfloat162_rn(gs.gam[sr]);
          const uint32_t fv = *reinterpret_cast<const uint32_t*>(&f2);
          const uint4 v = ld_shared_v4(sX + off);
          st_shared_v4(dst + off, hmul2_bf16(v.x, fv), hmul2_bf16(v.y, fv), hmul2_bf16(v.z, fv),
                       hmul2_bf16(v.w, fv));
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.xgready);
      }
      // S_in has landed (Xg above needs only the X tile, so it goes first)
      ok = ok && mbar_wait_warp(&sm.sfull, it & 1, wc, W_M_GFULL);
      tc_fence_after();
      if (ok) {
        // ---- <Lam_end, S_in>, then Lam <- 2^{L_{C-1}} Lam in place (Lam_end is complete
        //      since the previous chunk's b2full; this overlaps the R1 and DXb products)
        {
          const float gC = gs.gC;
          const uint32_t row = sS + (wg >> 1) * BIG;
          float v[32];
          tmem_ld32(tL, v);
          tmem_ld_wait();
          float ac4[4] = {0.f, 0.f, 0.f, 0.f};  // four chains, summed in a fixed order
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint4 sv = ld_shared_v4(row + sw128_off(n, 4 * (wg & 1) + cc));
            ac4[cc] = fmaf(v[8 * cc + 0], bf16_lo(sv.x), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 1], bf16_hi(sv.x), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 2], bf16_lo(sv.y), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 3], bf16_hi(sv.y), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 4], bf16_lo(sv.z), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 5], bf16_hi(sv.z), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 6], bf16_lo(sv.w), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 7], bf16_hi(sv.w), ac4[cc]);
          }
          float acc = (ac4[0] + ac4[1]) + (ac4[2] + ac4[3]);
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= gC;
          tmem_st32(tL, v);
#pragma unroll
          for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
          if (lane == 0) sm.ered[it & 1][warp - 4] = acc;
          // the scaled Lam is in place: the Lam update of this chunk may be issued
          tmem_st_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.lscaled);
        }
      }
      ok = ok && mbar_wait_warp(&sm.b1full, it & 1, wc, W_M_B1);
      tc_fence_after();
      if (ok) {
        // ---- one pass for q and p: lanes 0-15 hold row i of R1 (q_i = g_i . R1_i,
        //      then R1_i <- del_i R1_i), lanes 16-31 row i of DXb (p_i = x_i . DXb_i,
        //      then DXb_i <- gam_i DXb_i); this warp covers columns [32 wg, 32 wg + 32)
        {
          float v[32];
          tmem_ld32(tbase + COL_RX + lane_off + 32 * wg, v);
          tmem_ld_wait();
          const int i = ir;
          const uint32_t row = (lo ? sG : sX) + (wg >> 1) * TILE;
          float ac4[4] = {0.f, 0.f, 0.f, 0.f};  // four chains, summed in a fixed order
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const uint4 sv = ld_shared_v4(row + sw128_off(i, 4 * (wg & 1) + cc));
            ac4[cc] = fmaf(v[8 * cc + 0], bf16_lo(sv.x), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 1], bf16_hi(sv.x), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 2], bf16_lo(sv.y), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 3], bf16_hi(sv.y), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 4], bf16_lo(sv.z), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 5], bf16_hi(sv.z), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 6], bf16_lo(sv.w), ac4[cc]);
            ac4[cc] = fmaf(v[8 * cc + 7], bf16_hi(sv.w), ac4[cc]);
          }
          const float acc = (ac4[0] + ac4[1]) + (ac4[2] + ac4[3]);
          const float sc = lo ? gs.del[i] : gs.gam[i];
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] *= sc;
          tmem_st32(tbase + COL_RX + lane_off + 32 * wg, v);
          if (lo) sm.redq[wg][i] = acc;
          else sm.redp[wg][i] = acc;
        }
        tmem_st_wait();
      }
      named_sync_math();  // (B1) S_in read; partial sums of q, p and E written; G read
      if (ok && mt < C) {
        const int j = mt;
        sm.qv[j] = sm.redq[0][j] + sm.redq[1][j] + sm.redq[2][j] + sm.redq[3][j];
        sm.pv[j] = sm.redp[0][j] + sm.redp[1][j] + sm.redp[2][j] + sm.redp[3][j];
      }
      // the Gram products (which read G) are complete before G is scaled in place
      ok = ok && mbar_wait_warp(&sm.ccfull, it & 1, wc, W_M_CC);
      tc_fence_after();
      if (ok) {  // G <- diag(-eta del) G, rows scaled with packed bf16 multiplies
#pragma unroll
        for (int k = 0; k < (2 * TILE / 16) / (32 * NMATH); ++k) {
          const uint32_t off = (uint32_t)(mt + 32 * NMATH * k) * 16;
          const int j = (off & (TILE - 1)) >> 7;
          const __nv_bfloat162 f2 = __float2bfloat162_rn(-gs.eta[j] * gs.del[j]);
          const uint32_t fv = *reinterpret_cast<const uint32_t*>(&f2);
          uint4 v = ld_shared_v4(sG + off);
          st_shared_v4(sG + off, hmul2_bf16(v.x, fv), hmul2_bf16(v.y, fv), hmul2_bf16(v.z, fv),
                       hmul2_bf16(v.w, fv));
        }
        // Gs and gam (.) DXb are in place (the TMEM writes finished before B1)
        fence_proxy_async_smem();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.m1a);
      }
      named_sync_math();  // (B2) q and p complete; the S_in buffer may be overwritten

      if (ok) {
        // ---- chunk matrices from K | Kug and KugT, plus the t, t2, t3 partial sums
        float vkk[16], vkt[16];
        tmem_ld16(tbase + COL_KK + lane_off + j0w, vkk);
        tmem_ld16(tbase + COL_KT + lane_off + j0w, vkt);
        tmem_ld_wait();
        // lanes < 16 hold the K and KugT rows, lanes >= 16 the Kug row of the same i;
        // each value is exchanged with the partner lane (l ^ 16) as it is consumed
        const int i = ir;
        const float Li = gs.L[i], Lim1 = i == 0 ? 0.f : gs.L[i - 1], eti = gs.eta[i];
        const float zb = p.local ? 0.f : 1.f;  // keeps the adjoint's intra-chunk term of Z
        const float rai = gs.ra[i], rbi = gs.rb[i];
        const uint32_t b1 = sS + (lo ? CC_AR : CC_QT), b2 = sS + (lo ? CC_Z : CC_BM);
        float tpart = 0.f, t2part = 0.f, t3part = 0.f;
        auto build = [&](auto fac_tag) {
          constexpr bool FAC = decltype(fac_tag)::value;
          // Both lane halves run the same straight-line code on their own data
          // (selects, no divergent branches): lanes < 16 produce Ar and Z and the t2
          // sum, lanes >= 16 produce Q^T and Bm and the t and t3 sums.
          const float selA = lo ? 1.f : 0.f, selB = 1.f - selA;
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            uint32_t m1[4], m2[4];
#pragma unroll
            for (int e4 = 0; e4 < 8; e4 += 4) {
              const int jb = j0w + 8 * cc + e4;
              float4 cb4, ca4, L4, Lm4, et4;
              if (FAC) {
                cb4 = *reinterpret_cast<const float4*>(&gs.cb[jb]);
                ca4 = *reinterpret_cast<const float4*>(&gs.ca[jb]);
              } else {
                L4 = *reinterpret_cast<const float4*>(&gs.L[jb]);
                et4 = *reinterpret_cast<const float4*>(&gs.eta[jb]);
                Lm4 = make_float4(jb == 0 ? 0.f : gs.L[jb - 1], L4.x, L4.y, L4.z);
              }
              const float4 q4 = *reinterpret_cast<const float4*>(&sm.qv[jb]);
              const float4 p4 = *reinterpret_cast<const float4*>(&sm.pv[jb]);
              const float cbv[4] = {cb4.x, cb4.y, cb4.z, cb4.w};
              const float cav[4] = {ca4.x, ca4.y, ca4.z, ca4.w};
              const float Lv[4] = {L4.x, L4.y, L4.z, L4.w};
              const float Lmv[4] = {Lm4.x, Lm4.y, Lm4.z, Lm4.w};
              const float etv[4] = {et4.x, et4.y, et4.z, et4.w};
              const float qvv[4] = {q4.x, q4.y, q4.z, q4.w};
              const float pvv[4] = {p4.x, p4.y, p4.z, p4.w};
              float v0[4], v1[4];
#pragma unroll
              for (int d = 0; d < 4; ++d) {
                const int e = 8 * cc + e4 + d;
                const int j = jb + d;
                const float o1 = __shfl_xor_sync(0xffffffffu, vkk[e], 16);
                const float o2 = __shfl_xor_sync(0xffffffffu, vkt[e], 16);
                const float kr = lo ? vkk[e] : o1;  // x_i . x_j
                const float kg = lo ? o1 : vkk[e];  // u_i . g_j
                const float kt = lo ? vkt[e] : o2;  // g_i . u_j
                float bij, aij;                     // b_ij (j > i), a_ij (j < i)
                if (FAC) {
                  bij = cbv[d] * rbi;
                  aij = rai * cav[d];
                } else {
                  bij = exp2f(fminf(Lmv[d] - Li, 0.f));
                  aij = -etv[d] * exp2f(fminf(Lim1 - Lv[d], 0.f));
                }
                const float lt = (j < i) ? 1.f : 0.f, gt = (j > i) ? 1.f : 0.f;
                const float bg = gt * bij, al = lt * aij;
                // lanes < 16: Ar = b kr, Z = a kg - eta_i b kt ; lanes >= 16: Q^T = kg kr, Bm = b
                v0[d] = kr * (lo ? bg : lt * kg);
                v1[d] = lo ? fmaf(al, kg, -zb * eti * bg * kt) : bg;
                t2part = fmaf(selA * al, qvv[d], t2part);
                tpart = fmaf(selB * bg * kr, kt, tpart);
                t3part = fmaf(selB * bg, pvv[d], t3part);
              }
              m1[e4 >> 1] = pack_bf16(v0[0], v0[1]);
              m1[(e4 >> 1) + 1] = pack_bf16(v0[2], v0[3]);
              m2[e4 >> 1] = pack_bf16(v1[0], v1[1]);
              m2[(e4 >> 1) + 1] = pack_bf16(v1[2], v1[3]);
            }
            st_shared_v4(b1 + sw128_off(i, 2 * wg + cc), m1[0], m1[1], m1[2], m1[3]);
            st_shared_v4(b2 + sw128_off(i, 2 * wg + cc), m2[0], m2[1], m2[2], m2[3]);
          }
        };
        // With the factored decays, a warp whose 16 x 16 block lies wholly above
        // (wg > q: every j > i) or below (wg < q: every j < i) the diagonal needs no
        // masks, and fewer exchanges: above, each lane already holds what it needs
        // (lanes < 16: K and KugT; lanes >= 16 produce only Bm and t3); below, one
        // exchange gives both halves K_ij Kug_ij.
        auto store_pair = [&](int cc, const float (&v0)[8], const float (&v1)[8]) {
          st_shared_v4(b1 + sw128_off(i, 2 * wg + cc), pack_bf16(v0[0], v0[1]),
                       pack_bf16(v0[2], v0[3]), pack_bf16(v0[4], v0[5]), pack_bf16(v0[6], v0[7]));
          st_shared_v4(b2 + sw128_off(i, 2 * wg + cc), pack_bf16(v1[0], v1[1]),
                       pack_bf16(v1[2], v1[3]), pack_bf16(v1[4], v1[5]), pack_bf16(v1[6], v1[7]));
        };
        auto build_above = [&]() {
          const float neti = -zb * eti;  // the j > i part of Z (zero in hidden-costate mode)
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float v0[8], v1[8];
#pragma unroll
            for (int e4 = 0; e4 < 8; e4 += 4) {
              const int jb = j0w + 8 * cc + e4;
              const float4 cb4 = *reinterpret_cast<const float4*>(&gs.cb[jb]);
              const float4 p4 = *reinterpret_cast<const float4*>(&sm.pv[jb]);
              const float cbv[4] = {cb4.x, cb4.y, cb4.z, cb4.w};
              const float pvv[4] = {p4.x, p4.y, p4.z, p4.w};
#pragma unroll
              for (int d = 0; d < 4; ++d) {
                const int e = 8 * cc + e4 + d;
                const float bij = cbv[d] * rbi;
                const float pa = bij * vkk[e];                  // lanes < 16: b_ij K_ij
                v0[e4 + d] = lo ? pa : 0.f;                     // Ar | Q^T = 0
                v1[e4 + d] = lo ? neti * bij * vkt[e] : bij;    // Z | Bm
                tpart += lo ? pa * vkt[e] : 0.f;
                t3part += lo ? 0.f : bij * pvv[d];
              }
            }
            store_pair(cc, v0, v1);
          }
        };
        auto build_below = [&]() {
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            float v0[8], v1[8];
#pragma unroll
            for (int e4 = 0; e4 < 8; e4 += 4) {
              const int jb = j0w + 8 * cc + e4;
              const float4 ca4 = *reinterpret_cast<const float4*>(&gs.ca[jb]);
              const float4 q4 = *reinterpret_cast<const float4*>(&sm.qv[jb]);
              const float cav[4] = {ca4.x, ca4.y, ca4.z, ca4.w};
              const float qvv[4] = {q4.x, q4.y, q4.z, q4.w};
#pragma unroll
              for (int d = 0; d < 4; ++d) {
                const int e = 8 * cc + e4 + d;
                const float o = __shfl_xor_sync(0xffffffffu, vkk[e], 16);  // the other half
                const float aij = rai * cav[d];
                v0[e4 + d] = lo ? 0.f : vkk[e] * o;  // Ar = 0 | Q^T = K Kug
                v1[e4 + d] = lo ? aij * o : 0.f;     // Z = a Kug | Bm = 0
                t2part += lo ? aij * qvv[d] : 0.f;
              }
            }
            store_pair(cc, v0, v1);
          }
        };
        // A diagonal block with the factored decays: the lane pair of row i splits the
        // 16 columns (lo: the first 8, hi: the last 8) and each lane produces all four
        // matrices for its columns. Lo holds K and KugT of the row, hi holds Kug; one
        // exchange per column gives lo the Kug and hi the K of its own columns, a second
        // gives hi the KugT.
        auto build_diag = [&]() {
          const int h = lo ? 0 : 1;
          const int jb = j0w + 8 * h;
          const float neti = -zb * eti;
          float cbv[8], cav[8], qvv[8], pvv[8];
#pragma unroll
          for (int e4 = 0; e4 < 8; e4 += 4) {
            const float4 cb4 = *reinterpret_cast<const float4*>(&gs.cb[jb + e4]);
            const float4 ca4 = *reinterpret_cast<const float4*>(&gs.ca[jb + e4]);
            const float4 q4 = *reinterpret_cast<const float4*>(&sm.qv[jb + e4]);
            const float4 p4 = *reinterpret_cast<const float4*>(&sm.pv[jb + e4]);
            cbv[e4] = cb4.x; cbv[e4 + 1] = cb4.y; cbv[e4 + 2] = cb4.z; cbv[e4 + 3] = cb4.w;
            cav[e4] = ca4.x; cav[e4 + 1] = ca4.y; cav[e4 + 2] = ca4.z; cav[e4 + 3] = ca4.w;
            qvv[e4] = q4.x; qvv[e4 + 1] = q4.y; qvv[e4 + 2] = q4.z; qvv[e4 + 3] = q4.w;
            pvv[e4] = p4.x; pvv[e4 + 1] = p4.y; pvv[e4 + 2] = p4.z; pvv[e4 + 3] = p4.w;
          }
          float ar[8], zz[8], qq[8], bm[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            // lo sends K of column 8+e and receives Kug of column e; hi the reverse
            const float x1 = __shfl_xor_sync(0xffffffffu, lo ? vkk[8 + e] : vkk[e], 16);
            // lo sends KugT of column 8+e (hi's value is not used)
            const float x2 = __shfl_xor_sync(0xffffffffu, vkt[8 + e], 16);
            const float kr = lo ? vkk[e] : x1;      // x_i . x_j
            const float kg = lo ? x1 : vkk[8 + e];  // u_i . g_j
            const float kt = lo ? vkt[e] : x2;      // g_i . u_j
            const int j = jb + e;
            const float bij = cbv[e] * rbi, aij = rai * cav[e];
            const bool up = j > i, dn = j < i;
            const float bu = up ? bij : 0.f, ad = dn ? aij : 0.f;
            ar[e] = bu * kr;                               // Ar = b K (j > i)
            zz[e] = fmaf(ad, kg, neti * bu * kt);          // Z = a Kug (j < i) - eta_i b KugT (j > i)
            qq[e] = dn ? kr * kg : 0.f;                    // Q^T: K Kug (j < i)
            bm[e] = bu;                                    // Bm = b (j > i)
            t2part = fmaf(ad, qvv[e], t2part);
            tpart = fmaf(ar[e], kt, tpart);
            t3part = fmaf(bu, pvv[e], t3part);
          }
          const uint32_t cidx = 2 * wg + h;
          st_shared_v4(sS + CC_AR + sw128_off(i, cidx), pack_bf16(ar[0], ar[1]), pack_bf16(ar[2], ar[3]),
                       pack_bf16(ar[4], ar[5]), pack_bf16(ar[6], ar[7]));
          st_shared_v4(sS + CC_Z + sw128_off(i, cidx), pack_bf16(zz[0], zz[1]), pack_bf16(zz[2], zz[3]),
                       pack_bf16(zz[4], zz[5]), pack_bf16(zz[6], zz[7]));
          st_shared_v4(sS + CC_QT + sw128_off(i, cidx), pack_bf16(qq[0], qq[1]), pack_bf16(qq[2], qq[3]),
                       pack_bf16(qq[4], qq[5]), pack_bf16(qq[6], qq[7]));
          st_shared_v4(sS + CC_BM + sw128_off(i, cidx), pack_bf16(bm[0], bm[1]), pack_bf16(bm[2], bm[3]),
                       pack_bf16(bm[4], bm[5]), pack_bf16(bm[6], bm[7]));
        };
        if (gs.fac && wg > q) build_above();
        else if (gs.fac && wg < q) build_below();
        else if (gs.fac) build_diag();
        else build(std::false_type{});
        // each partial is nonzero in one lane half only; combine the pair
        tpart += __shfl_xor_sync(0xffffffffu, tpart, 16);
        t2part += __shfl_xor_sync(0xffffffffu, t2part, 16);
        t3part += __shfl_xor_sync(0xffffffffu, t3part, 16);
        if (lo) {
          sm.t2v[wg][i] = t2part;
          sm.tv[wg][i] = tpart;
          sm.t3v[wg][i] = t3part;
        }
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.m1done);
      }

      // ---- phase 2: dg from r, dx from dx, and the V part of dalpha
      ok = ok && mbar_wait_warp(&sm.b2full, it & 1, wc, W_M_B2);
      tc_fence_after();
      if (ok && it + 1 < nch) {
        // bf16 copy of the updated Lam for the next chunk's products, into this chunk's
        // region: b2full covers the Lam update and the last products on the chunk matrices
        const uint32_t lrow = sS + (wg >> 1) * BIG;
        float v[32];
        tmem_ld32(tL, v);
        tmem_ld_wait();
#pragma unroll
        for (int cc = 0; cc < 4; ++cc)
          st_shared_v4(lrow + sw128_off(n, 4 * (wg & 1) + cc), pack_bf16(v[8 * cc], v[8 * cc + 1]),
                       pack_bf16(v[8 * cc + 2], v[8 * cc + 3]),
                       pack_bf16(v[8 * cc + 4], v[8 * cc + 5]),
                       pack_bf16(v[8 * cc + 6], v[8 * cc + 7]));
        tc_fence_before();
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sm.lbready);
      }
      if (ok) {
        {
          float vv[16];
          tmem_ld16(tbase + COL_KT + lane_off + j0w, vv);
          tmem_ld_wait();
          if (!lo) {
            const int i = ir;
            float hpart = 0.f;
            if (gs.fac && wg > q) {
              // every j > i in this block: no term
            } else if (gs.fac && wg < q) {  // every j < i
              float acc = 0.f;
#pragma unroll
              for (int e4 = 0; e4 < 16; e4 += 4) {
                const float4 ca4 = *reinterpret_cast<const float4*>(&gs.ca[j0w + e4]);
                acc = fmaf(ca4.x, vv[e4], acc);
                acc = fmaf(ca4.y, vv[e4 + 1], acc);
                acc = fmaf(ca4.z, vv[e4 + 2], acc);
                acc = fmaf(ca4.w, vv[e4 + 3], acc);
              }
              hpart = gs.ra[i] * acc;
            } else if (gs.fac) {
              const float rai = gs.ra[i];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int j = j0w + e;
                if (j < i) hpart = fmaf(rai * gs.ca[j], vv[e], hpart);
              }
            } else {
              const float Lim1 = i == 0 ? 0.f : gs.L[i - 1];
#pragma unroll
              for (int e = 0; e < 16; ++e) {
                const int j = j0w + e;
                const float aij = -gs.eta[j] * exp2f(fminf(Lim1 - gs.L[j], 0.f));
                if (j < i) hpart = fmaf(aij, vv[e], hpart);
              }
            }
            sm.hv[wg][i] = hpart;
          }
        }
        {
          // dg_i = -eta_i r_i (lanes 0-15) and dx_i (lanes 16-31) -> staging tiles [i rows][d]
          // in this chunk's G and U tiles: every product that reads them has completed
          float v[32];
          tmem_ld32(tbase + COL_RX + lane_off + 32 * wg, v);
          tmem_ld_wait();
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&sm.m2done);
          const int i = ir;
          if (lo) {
            const float ne = -gs.eta[i];
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] *= ne;
          } else if (p.local) {  // hidden-costate mode: (1 - x^2) (.) (W0 + S)^T dy
            const uint32_t xrow = smem_u32(sm.X[st]) + (wg >> 1) * TILE;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              const uint4 xv = ld_shared_v4(xrow + sw128_off(i, 4 * (wg & 1) + cc));
              const uint32_t xw[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const float a0 = bf16_lo(xw[k]), a1 = bf16_hi(xw[k]);
                v[8 * cc + 2 * k] *= 1.f - a0 * a0;
                v[8 * cc + 2 * k + 1] *= 1.f - a1 * a1;
              }
            }
          }
          if (!lo && p.accumulate) {
            // this slice's dx is added onto that of the slices already done by one bulk
            // reduction of the chunk's rows (issued with the stores of the stage), so it is
            // staged row-major: row i at 256 i bytes
            const uint32_t trow = smem_u32(sm.U[st]) + (uint32_t)i * 256u + 64u * wg;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              st_shared_v4(trow + 16u * cc, pack_bf16(v[8 * cc], v[8 * cc + 1]),
                           pack_bf16(v[8 * cc + 2], v[8 * cc + 3]),
                           pack_bf16(v[8 * cc + 4], v[8 * cc + 5]),
                           pack_bf16(v[8 * cc + 6], v[8 * cc + 7]));
            }
          } else {
            const uint32_t trow = smem_u32(lo ? sm.G[st] : sm.U[st]) + (wg >> 1) * TILE;
#pragma unroll
            for (int cc = 0; cc < 4; ++cc)
              st_shared_v4(trow + sw128_off(i, 4 * (wg & 1) + cc), pack_bf16(v[8 * cc], v[8 * cc + 1]),
                           pack_bf16(v[8 * cc + 2], v[8 * cc + 3]),
                           pack_bf16(v[8 * cc + 4], v[8 * cc + 5]),
                           pack_bf16(v[8 * cc + 6], v[8 * cc + 7]));
          }
          fence_proxy_async_smem();
        }
      }
      named_sync_math();  // (B4) t, hv of all warpgroups and the dg / dx staging tiles written
      if (ok && mt == 0) mbar_arrive(&sm.staged[st]);  // warp 0 stores dg and dx from here
      if (ok && mt < C) {  // d_eta_j = -(del_j q_j + t_j)
        const int j = mt;
        const float deta =
            -(gs.del[j] * sm.qv[j] + sm.tv[0][j] + sm.tv[1][j] + sm.tv[2][j] + sm.tv[3][j]);
        if (t0 + j < T) {  // later slices add (one fire-and-forget add per element)
          if (p.accumulate)
            atomicAdd(p.d_eta + tokbase + j, deta);
          else
            p.d_eta[tokbase + j] = deta;
        }
      }
      if (ok && mt >= C && mt < 2 * C) {
        const int i = mt - C;
        const float t2 = sm.t2v[0][i] + sm.t2v[1][i] + sm.t2v[2][i] + sm.t2v[3][i];
        const float t3 = sm.t3v[0][i] + sm.t3v[1][i] + sm.t3v[2][i] + sm.t3v[3][i];
        const float h4 = sm.hv[0][i] + sm.hv[1][i] + sm.hv[2][i] + sm.hv[3][i];
        float E = 0.f;  // <Lam_end, S_in>: sum of the math warps' partials
#pragma unroll
        for (int w = 0; w < NMATH; w += 4) {
          const float4 e4 = *reinterpret_cast<const float4*>(&sm.ered[it & 1][w]);
          E += (e4.x + e4.y) + (e4.z + e4.w);
        }
        const float da = gs.gam[i] * gs.del[i] * E + gs.del[i] * t2 + gs.gam[i] * t3 + h4;
        if (t0 + i < T) {
          if (p.accumulate)
            atomicAdd(p.d_alpha + tokbase + i, da);
          else
            p.d_alpha[tokbase + i] = da;
        }
      }

      __syncwarp();
      if (ok && lane == 0) mbar_arrive(&sm.gempty[g]);  // this chunk's gates are read
      // No barrier is needed here. Faster warps may start the next chunk while warps
      // 4-7 finish the scalars above, but what those read is rewritten only later:
      // q by warps 4-5 themselves, the t, t2, t3 and h partials after the next B2
      // (which warps 4-7 must reach), the E partials in the other parity slot, and
      // the gates only after every math warp has arrived on gempty. The next tiles of
      // this stage land in the staging tiles only after their stores have read them.
    }

    // ---- this scan's dW0 partial: the last b2full wait covered every product
    if (ok) {
      float v[32];
      tmem_ld32(tbase + COL_W + lane_off + 32 * wg, v);
      tmem_ld_wait();
      // partial of (b, seg, h): the fixed-order reduction sums over b and seg
      const size_t part = ((size_t)(bh / p.H) * p.nseg + seg) * p.H + h;
      float4* dst = reinterpret_cast<float4*>(p.dW0_part + (part * p.dout + p.n0 + n) * 128 + 32 * wg);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
    // ---- the adjoint at the scan's first token, dL/dS_0 (segment 0 ends there)
    if (ok && p.L_first && seg == 0) {
      float v[32];
      tmem_ld32(tL, v);
      tmem_ld_wait();
      float4* dst = reinterpret_cast<float4*>(p.L_first + ((size_t)bh * p.dout + p.n0 + n) * 128 + 32 * wg);
#pragma unroll
      for (int e = 0; e < 8; ++e) dst[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 512);
  }
}

bool bwd_shape_ok(int din, int dout) { return din == 128 && (dout == 128 || dout == 256); }

cudaError_t launch_bwd(const TcBwdParams& prm, const void* x, const void* g, const void* dy,
                       const void* ckpt, cudaStream_t st) {
  CUtensorMap mx, mg, mu, ms, mdx, mdg;
  const uint64_t BH = (uint64_t)prm.B * prm.H;
  const uint64_t nch = (uint64_t)(prm.T + C - 1) / C;
  const uint64_t D = (uint64_t)prm.dout;
  if (!make_map_bf16_3d(&mx, x, 128, prm.T, BH, C) || !make_map_bf16_3d(&mg, g, D, prm.T, BH, C) ||
      !make_map_bf16_3d(&mu, dy, D, prm.T, BH, C) ||
      !make_map_bf16_3d(&ms, ckpt, 128, D, BH * nch, 128) ||
      !make_map_bf16_3d(&mdx, prm.dx, 128, prm.T, BH, C) ||
      !make_map_bf16_3d(&mdg, prm.dg, D, prm.T, BH, C))
    return cudaErrorInvalidValue;
  // The shared-memory opt-in is a per-device attribute: set it once on each device.
  static std::atomic<uint64_t> attr_set{0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(bwd_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  bwd_kernel<<<(int)BH * prm.nseg, NTHREADS, kSmemBytes, st>>>(mx, mg, mu, ms, mdx, mdg, prm);
  count_launch();
  return cudaGetLastError();
}

}  // namespace tc
}  // namespace gradlev
