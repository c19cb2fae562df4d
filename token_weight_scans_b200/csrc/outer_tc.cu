// Sum over a sequence of outer products on the tensor cores: out[bh] = sum_t a_t b_t^T
// for [T, 128] bf16 sequences a and b per (b, h), out [128][128] float32.
//
// In the two-layer reconstruction of the synthetic test (Cognaptus, "Parallelize
// the Training, Keep the Learning Serial", section "The synthetic test checks the
// mechanism, not model quality") this is the first matrix's gradient,
// dW1 = sum_t g1til_t x_t^T. It has the shape of the reverse scan's dW0 product:
// A^T B with the sequence as the contraction index.
//
// One CTA per (b, h). Warp 0 streams 64-token tiles of a and b through an
// NST-stage TMA pipeline. Warp 1 issues four 128 x 128 x 16 MMAs per tile into a
// TMEM accumulator. Both operands are MN-major: a tile holds 64 token rows of 128
// features. All four warps then read the accumulator out (warp w: rows 32w..32w+31).
// Every wait is bounded and reports through the device status word.

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>

#include "common.cuh"
#include "mlp2.h"
#include "scan_tc.h"
#include "sm100.cuh"

namespace gradlev {
namespace tc {
bool make_map_bf16_3d(CUtensorMap* m, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
                      uint32_t box1);
}  // namespace tc

namespace mlp2 {

using namespace sm100;

namespace {

constexpr int NST = 4;            // pipeline stages
constexpr int CT = 64;            // tokens per tile
constexpr int TILE = CT * 128;    // one [64 rows x 128 B] swizzled block
constexpr uint64_t kTimeoutNs = 2000000000ull;

enum : uint32_t { W_OT_EMPTY = 0x801, W_OT_FULL, W_OT_DONE, W_OT_DRAIN };

struct alignas(1024) OtSmem {
  uint8_t A[NST][2 * TILE];  // [64 tokens][128 features] as two 64-feature blocks
  uint8_t B[NST][2 * TILE];
  uint64_t full[NST], empty[NST], done;
  uint32_t tmem_base;
  int abort;
};
constexpr size_t kOtSmem = sizeof(OtSmem) + 1024;  // + alignment slack

__global__ void __launch_bounds__(128, 1)
    outer_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    float* __restrict__ out, int T, DeviceStatus* status) {
  extern __shared__ uint8_t smem_raw[];
  OtSmem& sm = *reinterpret_cast<OtSmem*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;
  const int ntile = (T + CT - 1) / CT;
  const WaitCtx wc{&sm.abort, status, kTimeoutNs};
  if (threadIdx.x == 0) {
    sm.abort = 0;
    for (int s = 0; s < NST; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], 1);
    }
    mbar_init(&sm.done, 1);
    fence_mbar_init();
    prefetch_tmap(&tmA);
    prefetch_tmap(&tmB);
  }
  if (warp == 1) {
    tmem_alloc(&sm.tmem_base, 128);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = sm.tmem_base;

  if (warp == 0 && lane == 0) {  // TMA producer (rows past T read as zeros)
    int issued = 0;
    for (int c = 0; c < ntile; ++c) {
      const int s = c % NST;
      if (!mbar_wait(&sm.empty[s], ((c / NST) & 1) ^ 1, wc, W_OT_EMPTY)) break;
      mbar_arrive_expect_tx(&sm.full[s], 4 * TILE);
      tma_load_3d(sm.A[s], &tmA, &sm.full[s], 0, c * CT, bh);
      tma_load_3d(sm.A[s] + TILE, &tmA, &sm.full[s], 64, c * CT, bh);
      tma_load_3d(sm.B[s], &tmB, &sm.full[s], 0, c * CT, bh);
      tma_load_3d(sm.B[s] + TILE, &tmB, &sm.full[s], 64, c * CT, bh);
      issued = c + 1;
    }
    // loads still in flight must land before the CTA exits
    for (int c = issued > NST ? issued - NST : 0; c < issued; ++c)
      mbar_drain(&sm.full[c % NST], (c / NST) & 1, wc, W_OT_DRAIN);
  } else if (warp == 1 && lane == 0) {  // MMA issuer
    const uint32_t id = idesc_bf16(128, 128, true, true);
    bool ok = true;
    for (int c = 0; c < ntile && ok; ++c) {
      const int s = c % NST;
      ok = mbar_wait(&sm.full[s], (c / NST) & 1, wc, W_OT_FULL);
      if (!ok) break;
      tc_fence_after();
      const uint64_t dA = sw128_desc(smem_u32(sm.A[s]), TILE, 1024);
      const uint64_t dB = sw128_desc(smem_u32(sm.B[s]), TILE, 1024);
#pragma unroll
      for (int kk = 0; kk < 4; ++kk)  // 16 tokens per MMA
        umma_bf16(tbase, desc_at(dA, kk * 2048), desc_at(dB, kk * 2048), id, (c > 0 || kk > 0));
      umma_commit(&sm.empty[s]);
    }
    umma_commit(&sm.done);
  }
  __syncwarp();
  // epilogue: every warp reads its 32 accumulator rows
  const bool ok = mbar_wait_warp(&sm.done, 0, wc, W_OT_DONE);
  tc_fence_after();
  if (ok) {
    const uint32_t lane_off = (uint32_t)(32 * warp) << 16;
    float* dst = out + ((size_t)bh * 128 + 32 * warp + lane) * 128;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float v[32];
      tmem_ld32(tbase + lane_off + 32 * j, v);
      tmem_ld_wait();
      float4* d4 = reinterpret_cast<float4*>(dst + 32 * j);
#pragma unroll
      for (int e = 0; e < 8; ++e) d4[e] = make_float4(v[4 * e], v[4 * e + 1], v[4 * e + 2], v[4 * e + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tbase, 128);
  }
}

}  // namespace

bool outer_tc_ok(int dh, int dx) { return dh == 128 && dx == 128; }

cudaError_t launch_outer_tc(const void* a, const void* b, float* out, int BH, int T,
                            DeviceStatus* status, cudaStream_t st) {
  CUtensorMap ma, mb;
  if (!tc::make_map_bf16_3d(&ma, a, 128, T, BH, CT) || !tc::make_map_bf16_3d(&mb, b, 128, T, BH, CT))
    return cudaErrorInvalidValue;
  static std::atomic<uint64_t> attr_set{0};  // the opt-in is per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return cudaErrorInvalidDevice;
  const uint64_t bit = dev < 64 ? (1ull << dev) : 0;
  if (!bit || !(attr_set.load() & bit)) {
    cudaError_t e = cudaFuncSetAttribute(outer_tc_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kOtSmem);
    if (e != cudaSuccess) return e;
    attr_set.fetch_or(bit);
  }
  outer_tc_kernel<<<BH, 128, kOtSmem, st>>>(ma, mb, out, T, status);
  count_launch();
  return cudaGetLastError();
}

}  // namespace mlp2
}  // namespace gradlev
