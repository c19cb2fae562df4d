// Host side of the C ABI declared in include/gradlev.h: argument validation,
// workspace sizing and kernel dispatch. No device memory is allocated here.
//
// Kernel families:
//   * tcgen05 kernels (scan_tc_fwd.cu, scan_tc_bwd.cu): bf16 I/O, d_in = 128 and
//     d_out in {128, 256} (one 128-row slice of d_out per CTA / per backward launch);
//   * CUDA-core kernels (scan_ffma.cu): everything else that is supported
//     (float32 I/O, or bf16 with d_in * d_out <= 16384).
// The two families exchange state checkpoints in different formats; a
// checkpoint buffer written by gradlev_scan_fwd is consumed by gradlev_scan_bwd
// of the same shape and dtype, which always picks the same family.

#include <cuda_runtime.h>
#include <stdint.h>
#include <string.h>

#include "common.cuh"
#include "dispatch.h"
#include "gradlev.h"
#include "consistency.h"
#include "mlp2.h"
#include "scan_ffma.h"
#include "scan_tc.h"

namespace gradlev {

static constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bound of device-side waits

static thread_local int t_launches = 0;
void count_launch() { ++t_launches; }
void reset_launch_count() { t_launches = 0; }

// Test hook state (gradlev_debug_inject_timeout): the site of the next launch that
// withholds one completion signal (0 = none), consumed by that launch.
enum InjectSite { INJ_NONE = 0, INJ_FWD = 1, INJ_BWD = 2, INJ_FWD_SUMMARY = 3, INJ_BWD_SUMMARY = 4 };
static int g_inject = INJ_NONE;
static uint64_t g_inject_timeout_ns = 0;
// Test hook state (gradlev_debug_summary_rescale): bound of the summary passes' deferred decay
static float g_rescale_log2 = tc::kSummaryRescaleLog2;

// The kernel's inject code and wait bound for a launch at `site` (one-shot).
static int take_inject(int site, int code, uint64_t* timeout_ns) {
  if (g_inject != site) {
    *timeout_ns = kWaitTimeoutNs;
    return 0;
  }
  g_inject = INJ_NONE;
  *timeout_ns = g_inject_timeout_ns;
  return code;
}

static size_t align_up(size_t v, size_t a) { return (v + a - 1) / a * a; }

bool use_tc(int din, int dout, gradlev_dtype dt) {
  return dt == GRADLEV_BF16 && tc::bwd_shape_ok(din, dout);
}

static gradlev_status check_shape(int B, int H, int T, int din, int dout, gradlev_dtype dt) {
  if (B <= 0 || H <= 0 || T <= 0 || din <= 0 || dout <= 0) return GRADLEV_ERR_INVALID_ARG;
  if (dt != GRADLEV_F32 && dt != GRADLEV_BF16) return GRADLEV_ERR_INVALID_ARG;
  if ((long long)B * H * T >= (1LL << 31)) return GRADLEV_ERR_UNSUPPORTED;
  if (!use_tc(din, dout, dt) && !ffma::shape_ok(din, dout)) return GRADLEV_ERR_UNSUPPORTED;
  return GRADLEV_OK;
}

static size_t ckpt_bytes_of(int B, int H, int T, int din, int dout, gradlev_dtype dt) {
  return use_tc(din, dout, dt) ? tc::ckpt_bytes(B, H, T, din, dout)
                               : ffma::ckpt_bytes(B, H, T, din, dout);
}

// ---- segmented long scans (both kernel families)
//
// When the scans of a call cannot fill the GPU, each scan is cut into segments
// that separate CTAs walk at the same time. Forward: a summary pass gives each
// segment's local state and log-decay, combine_segments turns them into the
// segments' start states, and the main pass walks every segment from its start
// state. Reverse: the same with the adjoint, walked backwards.
struct SegPlan {
  int nseg = 1, seg_chunks = 1 << 30;
};

static SegPlan fwd_plan(int B, int H, int T, int dout) {
  SegPlan s;
  tc::segment_plan(B * H * (dout / 128), (T + tc::kChunk - 1) / tc::kChunk, &s.nseg,
                   &s.seg_chunks);
  return s;
}

// The forward's summary pass at d_out = 256 carries both 128-row slices in one CTA, so it has
// half the units of the main pass and may cut each main segment into `ratio` equal pieces
// (the main segments' boundaries stay segment boundaries, and the combine keeps their start
// states). Without such a split it runs as the main pass does, one slice per CTA.
struct SumPlan {
  SegPlan seg;
  int two = 0, ratio = 1;
};

static SumPlan fwd_summary_plan(int B, int H, int T, int dout, const SegPlan& m) {
  SumPlan p;
  p.seg = m;
  if (dout != 256 || m.nseg <= 1) return p;
  const int n_chunks = (T + tc::kChunk - 1) / tc::kChunk;
  int r = (148 / (B * H)) / m.nseg;  // pieces per main segment that still fit one wave
  while (r > 1 && m.seg_chunks % r) --r;
  if (r < 2) return p;
  p.seg.seg_chunks = m.seg_chunks / r;
  p.seg.nseg = (n_chunks + p.seg.seg_chunks - 1) / p.seg.seg_chunks;
  p.two = 1;
  p.ratio = r;
  return p;
}

static SegPlan bwd_plan(int B, int H, int T) {
  SegPlan s;
  tc::segment_plan(B * H, (T + tc::kChunk - 1) / tc::kChunk, &s.nseg, &s.seg_chunks);
  return s;
}

// The CUDA-core kernels: one CTA per (scan, segment) in both directions.
static SegPlan ffma_plan(int B, int H, int T) {
  SegPlan s;
  tc::segment_plan(B * H, (T + ffma::kChunk - 1) / ffma::kChunk, &s.nseg, &s.seg_chunks);
  return s;
}

// Scratch of the segment passes: local summaries and combined states
// ([B*H][nseg][dout][din] fp32 each) and the segment log-decays ([B*H][nseg]).
static size_t seg_bytes(int B, int H, int din, int dout, int nseg) {
  if (nseg <= 1) return 0;
  const size_t mats = (size_t)B * H * nseg * dout * din * sizeof(float);
  return 2 * align_up(mats, 256) + align_up((size_t)B * H * nseg * sizeof(float), 256);
}

struct SegBufs {
  float *loc, *comb, *L;
};

static SegBufs seg_bufs(char* base, int B, int H, int din, int dout, int nseg) {
  const size_t mats = align_up((size_t)B * H * nseg * dout * din * sizeof(float), 256);
  return {reinterpret_cast<float*>(base), reinterpret_cast<float*>(base + mats),
          reinterpret_cast<float*>(base + 2 * mats)};
}

// segments of the forward's summary pass (at least as many as the main pass's)
static int fwd_seg_count(int B, int H, int T, int dout) {
  const SegPlan m = fwd_plan(B, H, T, dout);
  return fwd_summary_plan(B, H, T, dout, m).seg.nseg;
}

static size_t fwd_scratch_bytes(int B, int H, int T, int din, int dout, gradlev_dtype dt) {
  if (!use_tc(din, dout, dt)) return kStatusBytes + seg_bytes(B, H, din, dout, ffma_plan(B, H, T).nseg);
  return kStatusBytes + seg_bytes(B, H, din, dout, fwd_seg_count(B, H, T, dout));
}

static size_t dW0_part_bytes(int B, int H, int T, int din, int dout, gradlev_dtype dt) {
  const int nseg = use_tc(din, dout, dt) ? bwd_plan(B, H, T).nseg : ffma_plan(B, H, T).nseg;
  return align_up((size_t)B * H * nseg * din * dout * sizeof(float), 256);
}

size_t bwd_scratch_bytes(int B, int H, int T, int din, int dout, gradlev_dtype dt,
                         bool own_states) {
  size_t ws = kStatusBytes + dW0_part_bytes(B, H, T, din, dout, dt);
  if (own_states) ws += align_up(ckpt_bytes_of(B, H, T, din, dout, dt), 256);
  if (use_tc(din, dout, dt)) {
    const size_t fseg = own_states ? seg_bytes(B, H, din, dout, fwd_seg_count(B, H, T, dout)) : 0;
    const size_t bseg = seg_bytes(B, H, din, dout, bwd_plan(B, H, T).nseg);
    ws += fseg > bseg ? fseg : bseg;
  } else {  // the same plan in both directions
    ws += seg_bytes(B, H, din, dout, ffma_plan(B, H, T).nseg);
  }
  return ws;
}

static gradlev_status launch_fwd_impl(int B, int H, int T, int din, int dout, gradlev_dtype dt,
                                      const void* x, const void* g, const float* eta,
                                      const float* alpha, const float* W0, void* y, void* ckpt,
                                      DeviceStatus* status, char* seg_ws, cudaStream_t st,
                                      const float* S0, float* ST) {
  if (use_tc(din, dout, dt)) {
    uint64_t tmo = kWaitTimeoutNs;
    const int inject = y ? take_inject(INJ_FWD, 1, &tmo) : 0;
    const SegPlan sp = fwd_plan(B, H, T, dout);
    tc::TcFwdParams prm{B, H, T, din, dout, eta, alpha, W0, static_cast<__nv_bfloat16*>(y),
                        static_cast<__nv_bfloat16*>(ckpt), status, tmo, inject};
    if (sp.nseg > 1) {
      const SumPlan ss = fwd_summary_plan(B, H, T, dout, sp);
      const SegBufs sb = seg_bufs(seg_ws, B, H, din, dout, ss.seg.nseg);
      tc::TcFwdParams sum = prm;  // each segment's local state and log-decay
      sum.y = nullptr;
      sum.ckpt = nullptr;
      sum.inject = take_inject(INJ_FWD_SUMMARY, 3, &sum.timeout_ns);
      sum.nseg = ss.seg.nseg;
      sum.seg_chunks = ss.seg.seg_chunks;
      sum.S_final = sb.loc;
      sum.seg_L = sb.L;
      sum.summary = 1;
      sum.rescale_log2 = g_rescale_log2;
      sum.two_slices = ss.two;
      if (tc::launch_fwd(sum, x, g, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
      // the first segment starts from the carried state S0; the main pass's segments start
      // at every ratio-th summary segment
      if (tc::combine_segments(sb.loc, sb.L, S0, sb.comb, B * H, ss.seg.nseg, dout * din, 0, st,
                               ss.ratio) != cudaSuccess)
        return GRADLEV_ERR_CUDA;
      prm.nseg = sp.nseg;
      prm.seg_chunks = sp.seg_chunks;
      prm.S_init = sb.comb;
    } else {
      prm.S_init = S0;  // [B*H][1][dout][din]: the one segment's start state
    }
    prm.S_last = ST;
    return tc::launch_fwd(prm, x, g, st) == cudaSuccess ? GRADLEV_OK : GRADLEV_ERR_CUDA;
  }
  ffma::FwdArgs a{B, H, T, din, dout, x, g, eta, alpha, W0, y, static_cast<float*>(ckpt)};
  const SegPlan sp = ffma_plan(B, H, T);
  a.S0 = S0;  // [B*H][1][dout][din]: the one segment's start state
  if (sp.nseg > 1) {
    const SegBufs sb = seg_bufs(seg_ws, B, H, din, dout, sp.nseg);
    ffma::FwdArgs sum = a;  // each segment's local state and log-decay, from zero
    sum.y = nullptr;
    sum.ckpt = nullptr;
    sum.S0 = nullptr;
    sum.nseg = sp.nseg;
    sum.seg_chunks = sp.seg_chunks;
    sum.summary = 1;
    sum.Sloc = sb.loc;
    sum.segL = sb.L;
    if (ffma::launch_fwd(sum, dt == GRADLEV_BF16, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
    // the first segment starts from the carried state S0
    if (tc::combine_segments(sb.loc, sb.L, S0, sb.comb, B * H, sp.nseg, dout * din, 0, st) !=
        cudaSuccess)
      return GRADLEV_ERR_CUDA;
    a.nseg = sp.nseg;
    a.seg_chunks = sp.seg_chunks;
    a.S0 = sb.comb;
  }
  a.ST = ST;
  return ffma::launch_fwd(a, dt == GRADLEV_BF16, st) == cudaSuccess ? GRADLEV_OK
                                                                   : GRADLEV_ERR_CUDA;
}

gradlev_status bwd_run(int B, int H, int T, int din, int dout, gradlev_dtype dt, const void* x,
                       const void* g, const float* eta, const float* alpha, const float* W0,
                       const void* dy, void* dx, void* dg, float* d_eta, float* d_alpha,
                       float* dW0, const void* ckpt, char* ws, cudaStream_t st,
                       const StateIO& io, bool clear_status) {
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  float* dW0_part = reinterpret_cast<float*>(ws + kStatusBytes);
  char* own = ws + kStatusBytes + dW0_part_bytes(B, H, T, din, dout, dt);
  char* seg_ws = own + (ckpt ? 0 : align_up(ckpt_bytes_of(B, H, T, din, dout, dt), 256));
  if (clear_status && cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  const void* states = ckpt;
  if (!states) {
    gradlev_status s = launch_fwd_impl(B, H, T, din, dout, dt, x, g, eta, alpha, W0, nullptr,
                                       own, status, seg_ws, st, io.S0, nullptr);
    if (s != GRADLEV_OK) return s;
    states = own;
  }
  if (use_tc(din, dout, dt)) {
    const SegPlan sp = bwd_plan(B, H, T);
    const float* L_init = io.LamT;  // one segment: it ends where the adjoint flows in
    if (sp.nseg > 1) {
      // each segment's local adjoint (walked backwards from zero) and log-decay, then the
      // adjoint at each segment's end
      const SegBufs sb = seg_bufs(seg_ws, B, H, din, dout, sp.nseg);
      tc::TcFwdParams sum{B, H, T, din, dout, eta, alpha, W0, nullptr, nullptr, status,
                          kWaitTimeoutNs, 0};
      sum.inject = take_inject(INJ_BWD_SUMMARY, 3, &sum.timeout_ns);
      sum.nseg = sp.nseg;
      sum.seg_chunks = sp.seg_chunks;
      sum.S_final = sb.loc;
      sum.seg_L = sb.L;
      sum.summary = 1;
      sum.reverse = 1;
      sum.rescale_log2 = g_rescale_log2;
      sum.two_slices = dout == 256 ? 1 : 0;  // one CTA per (scan, segment): one wave
      if (tc::launch_fwd(sum, x, dy, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
      // the last segment ends where the adjoint LamT flows in
      if (tc::combine_segments(sb.loc, sb.L, io.LamT, sb.comb, B * H, sp.nseg, dout * din, 1,
                               st) != cudaSuccess)
        return GRADLEV_ERR_CUDA;
      L_init = sb.comb;
    }
    // one launch per 128-row slice of d_out; later slices accumulate dx, d_eta, d_alpha
    for (int n0 = 0; n0 < dout; n0 += 128) {
      tc::TcBwdParams prm{B, H, T, din, dout, n0, n0 > 0 ? 1 : 0, eta, alpha, W0,
                          static_cast<__nv_bfloat16*>(dx), static_cast<__nv_bfloat16*>(dg),
                          d_eta, d_alpha, dW0_part, status, kWaitTimeoutNs};
      prm.nseg = sp.nseg;
      prm.seg_chunks = sp.seg_chunks;
      prm.L_init = L_init;
      prm.L_first = io.dS0;
      prm.inject = take_inject(INJ_BWD, 2, &prm.timeout_ns);
      if (tc::launch_bwd(prm, x, g, dy, states, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
    }
    // partials are [B][nseg][H]: a fixed-order sum over b and the segments
    if (ffma::launch_reduce_dW0(dW0_part, dW0, B * sp.nseg, H, din * dout, st) != cudaSuccess)
      return GRADLEV_ERR_CUDA;
    return GRADLEV_OK;
  }
  ffma::BwdArgs a{B, H, T, din, dout, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha, dW0,
                  static_cast<const float*>(states), dW0_part};
  const SegPlan sp = ffma_plan(B, H, T);
  a.LamT = io.LamT;  // one segment: it ends where the adjoint flows in
  if (sp.nseg > 1) {
    // each segment's local adjoint (walked backwards from zero) and log-decay, then the
    // adjoint at each segment's end
    const SegBufs sb = seg_bufs(seg_ws, B, H, din, dout, sp.nseg);
    ffma::BwdArgs sum = a;
    sum.LamT = nullptr;
    sum.dS0 = nullptr;
    sum.nseg = sp.nseg;
    sum.seg_chunks = sp.seg_chunks;
    sum.summary = 1;
    sum.Lloc = sb.loc;
    sum.segL = sb.L;
    if (ffma::launch_bwd(sum, dt == GRADLEV_BF16, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
    // the last segment ends where the adjoint LamT flows in
    if (tc::combine_segments(sb.loc, sb.L, io.LamT, sb.comb, B * H, sp.nseg, dout * din, 1,
                             st) != cudaSuccess)
      return GRADLEV_ERR_CUDA;
    a.nseg = sp.nseg;
    a.seg_chunks = sp.seg_chunks;
    a.LamT = sb.comb;
  }
  a.dS0 = io.dS0;
  return ffma::launch_bwd(a, dt == GRADLEV_BF16, st) == cudaSuccess ? GRADLEV_OK
                                                                   : GRADLEV_ERR_CUDA;
}

static bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace gradlev

using namespace gradlev;

extern "C" {

const char* gradlev_status_string(gradlev_status s) {
  switch (s) {
    case GRADLEV_OK: return "GRADLEV_OK";
    case GRADLEV_ERR_INVALID_ARG: return "GRADLEV_ERR_INVALID_ARG";
    case GRADLEV_ERR_UNSUPPORTED: return "GRADLEV_ERR_UNSUPPORTED";
    case GRADLEV_ERR_WORKSPACE: return "GRADLEV_ERR_WORKSPACE";
    case GRADLEV_ERR_CUDA: return "GRADLEV_ERR_CUDA";
    case GRADLEV_ERR_TIMEOUT: return "GRADLEV_ERR_TIMEOUT";
  }
  return "GRADLEV_UNKNOWN_STATUS";
}

gradlev_status gradlev_scan_supported(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt) {
  return check_shape(B, H, T, d_in, d_out, dt);
}

size_t gradlev_scan_ckpt_bytes(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt) {
  if (check_shape(B, H, T, d_in, d_out, dt) != GRADLEV_OK) return 0;
  return ckpt_bytes_of(B, H, T, d_in, d_out, dt);
}

size_t gradlev_scan_workspace_bytes(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                    int is_bwd) {
  if (check_shape(B, H, T, d_in, d_out, dt) != GRADLEV_OK) return 0;
  return is_bwd ? bwd_scratch_bytes(B, H, T, d_in, d_out, dt, true)
                : fwd_scratch_bytes(B, H, T, d_in, d_out, dt);
}

}  // extern "C"

namespace gradlev {

static gradlev_status fwd_entry(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, const float* S0, void* y,
                                float* ST, void* ckpt, void* workspace, size_t ws_bytes,
                                void* stream) {
  gradlev_status s = check_shape(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (!x || !g || !eta || !alpha || !W0 || !y || !workspace) return GRADLEV_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(y, 16) || !aligned(W0, 16) ||
      !aligned(eta, 4) || !aligned(alpha, 4) || (ckpt && !aligned(ckpt, 16)) ||
      (S0 && !aligned(S0, 16)) || (ST && !aligned(ST, 16)) || !aligned(workspace, 16))
    return GRADLEV_ERR_INVALID_ARG;
  if (ws_bytes < gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, 0))
    return GRADLEV_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  t_launches = 0;
  DeviceStatus* status = static_cast<DeviceStatus*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  return launch_fwd_impl(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, y, ckpt, status,
                         static_cast<char*>(workspace) + kStatusBytes, st, S0, ST);
}

static gradlev_status bwd_entry(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, const void* dy, void* dx,
                                void* dg, float* d_eta, float* d_alpha, float* dW0,
                                const void* ckpt, void* workspace, size_t ws_bytes, void* stream,
                                const StateIO& io) {
  gradlev_status s = check_shape(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (!x || !g || !eta || !alpha || !W0 || !dy || !dx || !dg || !d_eta || !d_alpha || !dW0 ||
      !workspace)
    return GRADLEV_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(dy, 16) || !aligned(dx, 16) ||
      !aligned(dg, 16) || !aligned(W0, 16) || !aligned(dW0, 16) || !aligned(eta, 4) ||
      !aligned(alpha, 4) || !aligned(d_eta, 4) || !aligned(d_alpha, 4) ||
      (ckpt && !aligned(ckpt, 16)) || (io.S0 && !aligned(io.S0, 16)) ||
      (io.LamT && !aligned(io.LamT, 16)) || (io.dS0 && !aligned(io.dS0, 16)) ||
      !aligned(workspace, 16))
    return GRADLEV_ERR_INVALID_ARG;
  if (ws_bytes < gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, 1))
    return GRADLEV_ERR_WORKSPACE;
  t_launches = 0;
  return bwd_run(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha,
                 dW0, ckpt, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream), io);
}

}  // namespace gradlev

extern "C" {

gradlev_status gradlev_scan_fwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, void* y, void* ckpt,
                                void* workspace, size_t ws_bytes, void* stream) {
  return fwd_entry(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, nullptr, y, nullptr, ckpt,
                   workspace, ws_bytes, stream);
}

gradlev_status gradlev_scan_fwd_state(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                      const void* x, const void* g, const float* eta,
                                      const float* alpha, const float* W0, const float* S0,
                                      void* y, float* ST, void* ckpt, void* workspace,
                                      size_t ws_bytes, void* stream) {
  return fwd_entry(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, S0, y, ST, ckpt, workspace,
                   ws_bytes, stream);
}

gradlev_status gradlev_scan_bwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, const void* dy, void* dx,
                                void* dg, float* d_eta, float* d_alpha, float* dW0,
                                const void* ckpt, void* workspace, size_t ws_bytes,
                                void* stream) {
  return bwd_entry(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha,
                   dW0, ckpt, workspace, ws_bytes, stream, StateIO{});
}

gradlev_status gradlev_scan_bwd_state(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                      const void* x, const void* g, const float* eta,
                                      const float* alpha, const float* W0, const float* S0,
                                      const void* dy, const float* LamT, void* dx, void* dg,
                                      float* d_eta, float* d_alpha, float* dW0, float* dS0,
                                      const void* ckpt, void* workspace, size_t ws_bytes,
                                      void* stream) {
  StateIO io;
  io.S0 = S0;
  io.LamT = LamT;
  io.dS0 = dS0;
  return bwd_entry(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha,
                   dW0, ckpt, workspace, ws_bytes, stream, io);
}

size_t gradlev_consistency_workspace_bytes(int B, int H, int T, int d_in, int d_out,
                                           gradlev_dtype dt) {
  if (check_shape(B, H, T, d_in, d_out, dt) != GRADLEV_OK || d_out % 4 != 0) return 0;
  // the reverse scan's scratch, then the forward's checkpoints that it consumes
  return bwd_scratch_bytes(B, H, T, d_in, d_out, dt, true) +
         align_up(ckpt_bytes_of(B, H, T, d_in, d_out, dt), 256);
}

gradlev_status gradlev_consistency_step(int B, int H, int T, int d_in, int d_out,
                                        gradlev_dtype dt, const void* x, const void* ghat,
                                        const float* eta, const float* alpha, const float* W0,
                                        const void* v, float lam, void* y, void* gtil,
                                        float* loss_tok, float* loss_c, void* dx, void* dghat,
                                        float* d_eta, float* d_alpha, float* dW0, void* dv,
                                        void* workspace, size_t ws_bytes, void* stream) {
  gradlev_status s = check_shape(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (d_out % 4 != 0) return GRADLEV_ERR_UNSUPPORTED;
  if (!x || !ghat || !eta || !alpha || !W0 || !v || !y || !gtil || !loss_tok || !loss_c || !dx ||
      !dghat || !d_eta || !d_alpha || !dW0 || !workspace)
    return GRADLEV_ERR_INVALID_ARG;
  const size_t ea = dt == GRADLEV_BF16 ? 8 : 16;  // 4-element vectors of the residual pass
  if (!aligned(x, 16) || !aligned(ghat, 16) || !aligned(y, 16) || !aligned(dx, 16) ||
      !aligned(dghat, 16) || !aligned(W0, 16) || !aligned(dW0, 16) || !aligned(v, ea) ||
      !aligned(gtil, 16) || (dv && !aligned(dv, ea)) || !aligned(eta, 4) ||
      !aligned(alpha, 4) || !aligned(d_eta, 4) || !aligned(d_alpha, 4) ||
      !aligned(loss_tok, 4) || !aligned(loss_c, 4) || !aligned(workspace, 256))
    return GRADLEV_ERR_INVALID_ARG;
  if (ws_bytes < gradlev_consistency_workspace_bytes(B, H, T, d_in, d_out, dt))
    return GRADLEV_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  t_launches = 0;
  char* ws = static_cast<char*>(workspace);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  void* ckpt = ws + bwd_scratch_bytes(B, H, T, d_in, d_out, dt, true);
  if (cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  // 1. forward on the predicted costates, checkpoints for the reverse scan
  s = launch_fwd_impl(B, H, T, d_in, d_out, dt, x, ghat, eta, alpha, W0, y, ckpt, status,
                      ws + kStatusBytes, st, nullptr, nullptr);
  if (s != GRADLEV_OK) return s;
  // 2. reconstructed costates gtil = y - v (the token loss's output gradient), the losses
  const size_t ntok = (size_t)B * H * T;
  consistency::ResidualArgs ra{ntok, d_out, y, ghat, v, gtil, dv, loss_tok, loss_c};
  if (consistency::launch_residual(ra, dt == GRADLEV_BF16, st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  // 3. the token loss's gradients: the reverse scan with dy = gtil
  s = bwd_run(B, H, T, d_in, d_out, dt, x, ghat, eta, alpha, W0, gtil, dx, dghat, d_eta, d_alpha,
              dW0, ckpt, ws, st, StateIO{}, false);
  if (s != GRADLEV_OK) return s;
  // 4. the consistency term pushes ghat toward gtil: d ghat += 2 lam (ghat - gtil)
  if (consistency::launch_finish(dghat, ghat, gtil, lam, ntok * d_out, dt == GRADLEV_BF16, st) !=
      cudaSuccess)
    return GRADLEV_ERR_CUDA;
  return GRADLEV_OK;
}

}  // extern "C"

namespace gradlev {

// Workspace of the two-layer reconstruction. The tensor-core route (second layer a
// tensor-core shape, no control) lays it out as:
//   [0, r0)  status word, the forward scans' segment scratch, the reverse scan's partials
//   ckpt     the second layer's checkpoints
//   dg, de, da  scratch for the reverse scan's outputs that this call does not return
// The CUDA-core route needs only the first part.
struct Mlp2Ws {
  size_t r0, ckpt, dg, de, da, total;
};

static Mlp2Ws mlp2_ws(int B, int H, int T, int dx, int dh, int dy, gradlev_dtype dt) {
  Mlp2Ws w{};
  const size_t f1 = fwd_scratch_bytes(B, H, T, dx, dh, dt);
  const size_t f2 = fwd_scratch_bytes(B, H, T, dh, dy, dt);
  w.r0 = f1 > f2 ? f1 : f2;
  if (use_tc(dh, dy, dt)) {
    const size_t b = bwd_scratch_bytes(B, H, T, dh, dy, dt, false);
    w.r0 = align_up(w.r0 > b ? w.r0 : b, 256);
    const size_t es = dt == GRADLEV_BF16 ? 2 : 4;
    const size_t ntok = (size_t)B * H * T;
    w.ckpt = align_up(ckpt_bytes_of(B, H, T, dh, dy, dt), 256);
    w.dg = align_up(ntok * dy * es, 256);
    w.de = w.da = align_up(ntok * 4, 256);
  }
  w.total = w.r0 + w.ckpt + w.dg + w.de + w.da;
  return w;
}

}  // namespace gradlev

extern "C" {

size_t gradlev_mlp2_workspace_bytes(int B, int H, int T, int d_x, int d_h, int d_y,
                                    gradlev_dtype dt) {
  if (check_shape(B, H, T, d_x, d_h, dt) != GRADLEV_OK ||
      check_shape(B, H, T, d_h, d_y, dt) != GRADLEV_OK || !mlp2::shape_ok(d_x, d_h, d_y))
    return 0;
  return mlp2_ws(B, H, T, d_x, d_h, d_y, dt).total;
}

gradlev_status gradlev_mlp2_recon(int B, int H, int T, int d_x, int d_h, int d_y,
                                  gradlev_dtype dt, const void* x, const void* g1hat,
                                  const void* g2hat, const void* v, const float* eta,
                                  const float* alpha, const float* W1, const float* W2,
                                  int control, void* a, void* h, void* y, void* g2til,
                                  void* g1til, float* dW1, void* workspace, size_t ws_bytes,
                                  void* stream) {
  gradlev_status s = check_shape(B, H, T, d_x, d_h, dt);
  if (s != GRADLEV_OK) return s;
  s = check_shape(B, H, T, d_h, d_y, dt);
  if (s != GRADLEV_OK) return s;
  if (!mlp2::shape_ok(d_x, d_h, d_y)) return GRADLEV_ERR_UNSUPPORTED;
  if (!x || !g1hat || !g2hat || !v || !eta || !alpha || !W1 || !W2 || !a || !h || !y ||
      !g2til || !g1til || !dW1 || !workspace)
    return GRADLEV_ERR_INVALID_ARG;
  const size_t es = dt == GRADLEV_BF16 ? 2 : 4;
  if (!aligned(x, 16) || !aligned(g1hat, 16) || !aligned(g2hat, 16) || !aligned(a, 16) ||
      !aligned(h, 16) || !aligned(y, 16) || !aligned(W1, 16) || !aligned(W2, 16) ||
      !aligned(dW1, 16) || !aligned(v, es) || !aligned(g2til, 16) || !aligned(g1til, 16) ||
      !aligned(eta, 4) || !aligned(alpha, 4) || !aligned(workspace, 256))
    return GRADLEV_ERR_INVALID_ARG;
  const Mlp2Ws w = mlp2_ws(B, H, T, d_x, d_h, d_y, dt);
  if (ws_bytes < w.total) return GRADLEV_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  t_launches = 0;
  char* ws = static_cast<char*>(workspace);
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  if (cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  const bool bf = dt == GRADLEV_BF16;
  const bool tc_route = use_tc(d_h, d_y, dt) && !control;
  char* ckpt = tc_route ? ws + w.r0 : nullptr;
  // first layer: a = scan(x; g1hat, W1), h = tanh(a)
  s = launch_fwd_impl(B, H, T, d_x, d_h, dt, x, g1hat, eta, alpha, W1, a, nullptr, status,
                      ws + kStatusBytes, st, nullptr, nullptr);
  if (s != GRADLEV_OK) return s;
  const size_t ntok = (size_t)B * H * T;
  if (mlp2::launch_tanh(a, h, ntok * d_h, bf, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
  // second layer: y = scan(h; g2hat, W2), with its checkpoints on the tensor-core route
  s = launch_fwd_impl(B, H, T, d_h, d_y, dt, h, g2hat, eta, alpha, W2, y, ckpt, status,
                      ws + kStatusBytes, st, nullptr, nullptr);
  if (s != GRADLEV_OK) return s;
  if (!tc_route) {
    // the reconstruction kernel on CUDA cores (every shape, and the control)
    mlp2::TqueryArgs ta{B, H, T, d_x, d_h, d_y, control ? 1 : 0, x, h, g2hat, y, v, eta, alpha,
                        W2, g2til, g1til, dW1};
    return mlp2::launch_tquery(ta, bf, st) == cudaSuccess ? GRADLEV_OK : GRADLEV_ERR_CUDA;
  }
  // tensor-core route: g2til = y - v, then the reverse scan of the second layer in its
  // hidden-costate mode gives g1til = (1 - h^2) (.) (W2 + S2_t)^T g2til directly
  if (mlp2::launch_sub(y, v, g2til, ntok * d_y, bf, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
  char* dg = ckpt + w.ckpt;
  float* de = reinterpret_cast<float*>(dg + w.dg);
  float* da = reinterpret_cast<float*>(dg + w.dg + w.de);
  float* parts = reinterpret_cast<float*>(ws + kStatusBytes);
  for (int n0 = 0; n0 < d_y; n0 += 128) {
    tc::TcBwdParams prm{B, H, T, d_h, d_y, n0, n0 > 0 ? 1 : 0, eta, alpha, W2,
                        static_cast<__nv_bfloat16*>(g1til), reinterpret_cast<__nv_bfloat16*>(dg),
                        de, da, parts, status, kWaitTimeoutNs};
    prm.local = 1;
    if (tc::launch_bwd(prm, h, g2hat, g2til, ckpt, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
  }
  // the first matrix's gradient over the sequence (tensor cores when d_x = 128 too)
  const cudaError_t e =
      mlp2::outer_tc_ok(d_h, d_x)
          ? mlp2::launch_outer_tc(g1til, x, dW1, B * H, T, status, st)
          : mlp2::launch_outer_sum(g1til, x, dW1, B * H, T, d_h, d_x, bf, st);
  return e == cudaSuccess ? GRADLEV_OK : GRADLEV_ERR_CUDA;
}

gradlev_status gradlev_device_status(const void* workspace, void* stream) {
  if (!workspace) return GRADLEV_ERR_INVALID_ARG;
  DeviceStatus h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GRADLEV_ERR_CUDA;
  if (h.code == 0) return GRADLEV_OK;
  return h.code == GRADLEV_ERR_TIMEOUT ? GRADLEV_ERR_TIMEOUT : GRADLEV_ERR_CUDA;
}

int gradlev_last_launch_count(void) { return t_launches; }

void gradlev_debug_inject_timeout(int site, int timeout_ms) {
  g_inject = (site >= INJ_FWD && site <= INJ_BWD_SUMMARY) ? site : INJ_NONE;
  g_inject_timeout_ns = (uint64_t)(timeout_ms > 0 ? timeout_ms : 1) * 1000000ull;
}

void gradlev_debug_summary_rescale(float log2_bound) {
  g_rescale_log2 = !(log2_bound >= 0.f) ? tc::kSummaryRescaleLog2 : fminf(log2_bound, 126.f);
}

}  // extern "C"
