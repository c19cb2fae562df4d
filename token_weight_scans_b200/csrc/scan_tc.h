// Host-side interface of the tensor-core (tcgen05) GradLev scan kernels.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "common.cuh"

namespace gradlev {
namespace tc {

// The forward kernel walks one segment of chunks per CTA: CTA (b, h, slice, seg)
// covers chunks [seg * seg_chunks, min(n_chunks, (seg + 1) * seg_chunks)) of
// its scan. With nseg > 1 the segments' start states come from S_init, which a
// summary pass (summary = 1: the state carry alone, from a zero start, ending in
// S_final and seg_L) and a combine pass (combine_segments) produce beforehand.
// reverse = 1 walks the segment backwards and weights row j of the G-operand by
// 2^{L_{j-1}} instead of -eta_j 2^{L_{C-1}-L_j}: with dy in place of g, that is the
// adjoint recursion Lam <- 2^{L_{C-1}} Lam + sum_j 2^{L_{j-1}} u_j x_j^T.
constexpr float kSummaryRescaleLog2 = 64.f;  // default bound of the summary passes' deferred decay

struct TcFwdParams {
  int B, H, T, din, dout;   // din == 128, dout % 128 == 0
  const float* eta;         // [B,H,T]
  const float* alpha;       // [B,H,T]
  const float* W0;          // [H,dout,din] float32
  __nv_bfloat16* y;         // [B,H,T,dout], or null (state checkpoints only)
  __nv_bfloat16* ckpt;      // [B*H][n_chunks][dout][din] chunk-start states, or null
  DeviceStatus* status;     // device status word (workspace head)
  uint64_t timeout_ns;      // bound of every wait inside the kernel
  int inject;               // test hook: 1 = withhold one completion signal of the main
                            // pass, 3 = of the state carry (summary passes)
  int nseg = 1;             // segments per scan
  int seg_chunks = 1 << 30; // chunks per segment (the last one may be shorter)
  const float* S_init = nullptr;  // [B*H][nseg][dout][din] segment start states, or null (= 0)
  float* S_final = nullptr;       // [B*H][nseg][dout][din] state after the walk, or null
  float* seg_L = nullptr;         // [B*H][nseg] sum of log2 alpha over the segment, or null
  int summary = 0;          // 1: state carry only (no y, no checkpoints)
  int reverse = 0;          // 1: adjoint summary (see above)
  float* S_last = nullptr;  // [B*H][dout][din] the state after the scan's last token, or null
                            // (written by the last segment's CTAs; not in summary mode)
  // summary mode: the decay since the last in-place rescale of the state is kept as a
  // scale 2^E, and the state is rescaled once E would drop below -rescale_log2 (0..126)
  float rescale_log2 = kSummaryRescaleLog2;
  // summary mode at d_out = 256: 1 = one CTA carries both 128-row slices (grid B*H*nseg)
  int two_slices = 0;
};

// The reverse scan of one 128-row slice [n0, n0+128) of d_out: the rows of the
// state and adjoint evolve independently, so a d_out = 256 problem is two
// slice problems whose dx, d_eta and d_alpha add up (accumulate = 1 on the
// second slice) and whose dg and dW0 rows are disjoint.
//
// The reverse kernel walks one segment per CTA, like the forward one; L_init
// holds the adjoint at each segment's end (zero for the last segment), from the
// reverse summary and combine passes.
struct TcBwdParams {
  int B, H, T, din, dout;   // din == 128, dout in {128, 256}
  int n0;                   // first d_out row of this slice
  int accumulate;           // add dx, d_eta, d_alpha onto the values already there
  const float* eta;
  const float* alpha;
  const float* W0;          // [H,dout,128] float32
  __nv_bfloat16* dx;        // [B,H,T,128]
  __nv_bfloat16* dg;        // [B,H,T,dout]
  float* d_eta;             // [B,H,T]
  float* d_alpha;           // [B,H,T]
  float* dW0_part;          // [B][nseg][H][dout][128] float32 per-(scan, segment) partials
  DeviceStatus* status;
  uint64_t timeout_ns;
  int nseg = 1;             // segments per scan
  int seg_chunks = 1 << 30; // chunks per segment (the last one may be shorter)
  const float* L_init = nullptr;  // [B*H][nseg][dout][din] adjoint at each segment's end, or null
  float* L_first = nullptr;  // [B*H][dout][din] the adjoint at the scan's first token (dL/dS_0),
                             // or null (written by segment 0's CTAs)
  // Hidden-costate mode: dx_t = (1 - x_t^2) (.) ((W0 + S_t)^T dy_t), the layer's input
  // gradient at frozen weights through tanh (no adjoint terms). dg, d_eta, d_alpha and
  // the dW0 partials are then scratch.
  int local = 0;
  int inject = 0;           // test hook: 2 = withhold one completion signal
};

constexpr int kChunk = 64;  // tokens per chunk of the tensor-core kernels

bool fwd_shape_ok(int din, int dout);
bool bwd_shape_ok(int din, int dout);
// bytes of the bf16 chunk-start state checkpoints the tensor-core kernels exchange
size_t ckpt_bytes(int B, int H, int T, int din, int dout);
cudaError_t launch_fwd(const TcFwdParams& p, const void* x, const void* g, cudaStream_t st);
cudaError_t launch_bwd(const TcBwdParams& p, const void* x, const void* g, const void* dy,
                       const void* ckpt, cudaStream_t st);
size_t fwd_smem_bytes();
// Segments for `units` CTAs per segment index over a scan of n_chunks chunks.
void segment_plan(int units, int n_chunks, int* nseg, int* seg_chunks);
// The serial recursion over segment summaries (forward: start states; reverse:
// end adjoints), element by element for `scans` scans of per_scan elements. `init`
// ([scans][per_scan], or null for zero) is the value entering the first segment walked:
// the carried start state forward, the adjoint flowing in at the end in reverse.
// out_every > 1 (forward only): out keeps the start states of segments 0, out_every,
// 2 out_every, ... as [scans][ceil(nseg / out_every)]. out may alias loc only when
// out_every == 1.
cudaError_t combine_segments(const float* loc, const float* segL, const float* init, float* out,
                             int scans, int nseg, int per_scan, int reverse, cudaStream_t st,
                             int out_every = 1);

}  // namespace tc
}  // namespace gradlev
