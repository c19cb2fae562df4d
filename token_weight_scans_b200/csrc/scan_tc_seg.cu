// Segment combine for long scans on the tensor-core path.
//
// A scan of n_chunks chunks can be cut into nseg segments that separate CTAs
// walk in parallel. Each segment first gets a summary from a zero start: its
// local state Sloc_k and the sum L_k of log2 alpha over its tokens. The carried
// quantity is linear, so the state entering each segment follows from those
// summaries by a short serial recursion over segments (Cognaptus, "Parallelize
// the Training, Keep the Learning Serial", section "Once the gradient signals
// are known, the weight trajectory becomes parallelizable": a discounted sum of
// rank-one updates composes segment by segment):
//   forward (state S):    S_start(0) = 0,  S_start(k) = 2^{L_{k-1}} S_start(k-1) + Sloc_{k-1}
//   reverse (adjoint Lam): Lam_end(nseg-1) = 0,
//                          Lam_end(k) = 2^{L_{k+1}} Lam_end(k+1) + Lloc_{k+1}
// The forward may keep only every out_every-th start state (the summary pass then cut each
// segment of the main pass into out_every pieces): out holds [scan][ceil(nseg / out_every)].
// The recursion runs element by element in fp32: one thread per element of the
// d_out x d_in matrix, looping over the segments of its scan. A carried start
// state (forward) or an adjoint flowing in at the sequence's end (reverse)
// replaces the zero that enters the first segment walked.

#include <cuda_runtime.h>

#include "common.cuh"
#include "scan_tc.h"

namespace gradlev {
namespace tc {

__global__ void combine_kernel(const float* __restrict__ loc, const float* __restrict__ segL,
                               const float* __restrict__ init, float* __restrict__ out, int nseg,
                               int per_scan, int reverse, int out_every) {
  const int scan = blockIdx.y;
  const int e = blockIdx.x * blockDim.x + threadIdx.x;
  if (e >= per_scan) return;
  const size_t base = (size_t)scan * nseg;
  const size_t obase = (size_t)scan * ((nseg + out_every - 1) / out_every);
  float acc = init ? init[(size_t)scan * per_scan + e] : 0.f;
  for (int i = 0; i < nseg; ++i) {
    const int k = reverse ? nseg - 1 - i : i;
    const size_t at = (base + k) * per_scan + e;
    const float l = loc[at];  // read before the write below when loc and out alias
    if (k % out_every == 0) out[(obase + k / out_every) * per_scan + e] = acc;
    acc = fmaf(exp2f(segL[base + k]), acc, l);
  }
}

cudaError_t combine_segments(const float* loc, const float* segL, const float* init, float* out,
                             int scans, int nseg, int per_scan, int reverse, cudaStream_t st,
                             int out_every) {
  if (out_every < 1 || (reverse && out_every != 1)) return cudaErrorInvalidValue;
  const dim3 grid((per_scan + 255) / 256, scans);
  combine_kernel<<<grid, 256, 0, st>>>(loc, segL, init, out, nseg, per_scan, reverse, out_every);
  count_launch();
  return cudaGetLastError();
}

void segment_plan(int units, int n_chunks, int* nseg, int* seg_chunks) {
  // Enough segments to give every SM of a B200 (148) a CTA, of at least two chunks each.
  constexpr int kTargetCtas = 148, kMinSegChunks = 2;
  int n = 1;
  if (units > 0 && 2 * units <= kTargetCtas) {
    n = kTargetCtas / units;
    const int cap = (n_chunks + kMinSegChunks - 1) / kMinSegChunks;
    if (n > cap) n = cap;
    if (n < 1) n = 1;
  }
  int len = (n_chunks + n - 1) / n;
  if (len < 1) len = 1;
  *seg_chunks = n > 1 ? len : (1 << 30);
  *nseg = n > 1 ? (n_chunks + len - 1) / len : 1;
}

}  // namespace tc
}  // namespace gradlev
