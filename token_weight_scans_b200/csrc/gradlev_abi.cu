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
#include "scan_ffma.h"
#include "scan_tc.h"

namespace gradlev {

static thread_local int t_launches = 0;
void count_launch() { ++t_launches; }

// Test hook state (gradlev_debug_inject_timeout): consumed by the next fwd call.
static int g_inject = 0;
static uint64_t g_inject_timeout_ns = 0;
static constexpr uint64_t kWaitTimeoutNs = 2000000000ull;  // bound of device-side waits

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

size_t bwd_scratch_bytes(int B, int H, int T, int din, int dout, gradlev_dtype dt,
                         bool own_states) {
  size_t ws = kStatusBytes + align_up((size_t)B * H * din * dout * sizeof(float), 256);
  if (own_states) ws += align_up(ckpt_bytes_of(B, H, T, din, dout, dt), 256);
  return ws;
}

static gradlev_status launch_fwd_impl(int B, int H, int T, int din, int dout, gradlev_dtype dt,
                                      const void* x, const void* g, const float* eta,
                                      const float* alpha, const float* W0, void* y, void* ckpt,
                                      DeviceStatus* status, cudaStream_t st) {
  if (use_tc(din, dout, dt)) {
    const int inject = y ? g_inject : 0;
    const uint64_t tmo = inject ? g_inject_timeout_ns : kWaitTimeoutNs;
    if (y) g_inject = 0;
    tc::TcFwdParams prm{B, H, T, din, dout, eta, alpha, W0, static_cast<__nv_bfloat16*>(y),
                        static_cast<__nv_bfloat16*>(ckpt), status, tmo, inject};
    return tc::launch_fwd(prm, x, g, st) == cudaSuccess ? GRADLEV_OK : GRADLEV_ERR_CUDA;
  }
  ffma::FwdArgs a{B, H, T, din, dout, x, g, eta, alpha, W0, y, static_cast<float*>(ckpt)};
  return ffma::launch_fwd(a, dt == GRADLEV_BF16, st) == cudaSuccess ? GRADLEV_OK
                                                                   : GRADLEV_ERR_CUDA;
}

gradlev_status bwd_run(int B, int H, int T, int din, int dout, gradlev_dtype dt, const void* x,
                       const void* g, const float* eta, const float* alpha, const float* W0,
                       const void* dy, void* dx, void* dg, float* d_eta, float* d_alpha,
                       float* dW0, const void* ckpt, char* ws, cudaStream_t st) {
  DeviceStatus* status = reinterpret_cast<DeviceStatus*>(ws);
  float* dW0_part = reinterpret_cast<float*>(ws + kStatusBytes);
  void* own = ws + kStatusBytes + align_up((size_t)B * H * din * dout * sizeof(float), 256);
  if (cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  const void* states = ckpt;
  if (!states) {
    gradlev_status s = launch_fwd_impl(B, H, T, din, dout, dt, x, g, eta, alpha, W0, nullptr,
                                       own, status, st);
    if (s != GRADLEV_OK) return s;
    states = own;
  }
  if (use_tc(din, dout, dt)) {
    // one launch per 128-row slice of d_out; later slices accumulate dx, d_eta, d_alpha
    for (int n0 = 0; n0 < dout; n0 += 128) {
      tc::TcBwdParams prm{B, H, T, din, dout, n0, n0 > 0 ? 1 : 0, eta, alpha, W0,
                          static_cast<__nv_bfloat16*>(dx), static_cast<__nv_bfloat16*>(dg),
                          d_eta, d_alpha, dW0_part, status, kWaitTimeoutNs};
      if (tc::launch_bwd(prm, x, g, dy, states, st) != cudaSuccess) return GRADLEV_ERR_CUDA;
    }
    if (ffma::launch_reduce_dW0(dW0_part, dW0, B, H, din * dout, st) != cudaSuccess)
      return GRADLEV_ERR_CUDA;
    return GRADLEV_OK;
  }
  ffma::BwdArgs a{B, H, T, din, dout, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha, dW0,
                  static_cast<const float*>(states), dW0_part};
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
  return is_bwd ? bwd_scratch_bytes(B, H, T, d_in, d_out, dt, true) : kStatusBytes;
}

gradlev_status gradlev_scan_fwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, void* y, void* ckpt,
                                void* workspace, size_t ws_bytes, void* stream) {
  gradlev_status s = check_shape(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (!x || !g || !eta || !alpha || !W0 || !y || !workspace) return GRADLEV_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(y, 16) || !aligned(W0, 16) ||
      !aligned(eta, 4) || !aligned(alpha, 4) || (ckpt && !aligned(ckpt, 16)) ||
      !aligned(workspace, 16))
    return GRADLEV_ERR_INVALID_ARG;
  if (ws_bytes < gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, 0))
    return GRADLEV_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  t_launches = 0;
  DeviceStatus* status = static_cast<DeviceStatus*>(workspace);
  if (cudaMemsetAsync(status, 0, sizeof(DeviceStatus), st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  return launch_fwd_impl(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, y, ckpt, status, st);
}

gradlev_status gradlev_scan_bwd(int B, int H, int T, int d_in, int d_out, gradlev_dtype dt,
                                const void* x, const void* g, const float* eta,
                                const float* alpha, const float* W0, const void* dy, void* dx,
                                void* dg, float* d_eta, float* d_alpha, float* dW0,
                                const void* ckpt, void* workspace, size_t ws_bytes,
                                void* stream) {
  gradlev_status s = check_shape(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (!x || !g || !eta || !alpha || !W0 || !dy || !dx || !dg || !d_eta || !d_alpha || !dW0 ||
      !workspace)
    return GRADLEV_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(dy, 16) || !aligned(dx, 16) ||
      !aligned(dg, 16) || !aligned(W0, 16) || !aligned(dW0, 16) || !aligned(eta, 4) ||
      !aligned(alpha, 4) || !aligned(d_eta, 4) || !aligned(d_alpha, 4) ||
      (ckpt && !aligned(ckpt, 16)) || !aligned(workspace, 16))
    return GRADLEV_ERR_INVALID_ARG;
  if (ws_bytes < gradlev_scan_workspace_bytes(B, H, T, d_in, d_out, dt, 1))
    return GRADLEV_ERR_WORKSPACE;
  t_launches = 0;
  return bwd_run(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha,
                 dW0, ckpt, static_cast<char*>(workspace), static_cast<cudaStream_t>(stream));
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

void gradlev_debug_inject_timeout(int enable, int timeout_ms) {
  g_inject = enable ? 1 : 0;
  g_inject_timeout_ns = (uint64_t)(timeout_ms > 0 ? timeout_ms : 1) * 1000000ull;
}

}  // extern "C"
