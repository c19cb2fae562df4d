// gradlev_scan_bwd_noalloc: the reverse scan for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a workspace: code that runs while the
// process's allocator is unavailable or forbidden to grow (a fixed-pool
// serving runtime, a plugin handed only its tensors, a host language binding
// with no CUDA allocator of its own). gradlev_scan_bwd needs a caller-provided
// workspace; this variant instead takes its scratch from one file-scope
// __device__ array of GRADLEV_NOALLOC_SCRATCH_BYTES, which exists once per GPU
// that loads the library and lives until the process exits. The caller still
// passes every input and output buffer.
//
// Host code may not hand the array's name to a kernel: on the host that name
// is only a stand-in for the symbol, not a device address. The device address
// is looked up once per device with cudaGetSymbolAddress, with that device
// current, the first time the entry point runs on it, and cached.
//
// A bounded device-side wait that gives up writes its status word into the
// start of the array, as it would into a workspace; gradlev_noalloc_device_status
// reads it back.
//
// Nothing here calls cudaMalloc, cudaFree or any allocating routine.

#include <cuda_runtime.h>
#include <stdint.h>

#include <mutex>

#include "common.cuh"
#include "dispatch.h"
#include "gradlev.h"

namespace gradlev {
namespace {

constexpr size_t kScratchBytes = GRADLEV_NOALLOC_SCRATCH_BYTES;
constexpr int kMaxDevices = 64;

// The scratch itself. Every call on a device shares it; it keeps the last
// call's contents, so each call clears what must start at zero (the status word).
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

std::mutex g_mu;
void* g_addr[kMaxDevices] = {};

// Device address of g_noalloc_scratch on the current device (looked up once per device).
gradlev_status scratch_address(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess) return GRADLEV_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GRADLEV_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_addr[dev] == nullptr) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) return GRADLEV_ERR_CUDA;
    g_addr[dev] = p;
  }
  *out = g_addr[dev];
  return GRADLEV_OK;
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

}  // namespace
}  // namespace gradlev

using namespace gradlev;

extern "C" GRADLEV_API gradlev_status gradlev_scan_bwd_noalloc(
    int B, int H, int T, int d_in, int d_out, gradlev_dtype dt, const void* x, const void* g,
    const float* eta, const float* alpha, const float* W0, const void* dy, void* dx, void* dg,
    float* d_eta, float* d_alpha, float* dW0, const void* ckpt, void* stream) {
  // Shape and size checks first: they need no GPU and launch nothing.
  gradlev_status s = gradlev_scan_supported(B, H, T, d_in, d_out, dt);
  if (s != GRADLEV_OK) return s;
  if (bwd_scratch_bytes(B, H, T, d_in, d_out, dt, ckpt == nullptr) > kScratchBytes)
    return GRADLEV_ERR_WORKSPACE;
  if (!x || !g || !eta || !alpha || !W0 || !dy || !dx || !dg || !d_eta || !d_alpha || !dW0)
    return GRADLEV_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(dy, 16) || !aligned(dx, 16) ||
      !aligned(dg, 16) || !aligned(W0, 16) || !aligned(dW0, 16) || !aligned(eta, 4) ||
      !aligned(alpha, 4) || !aligned(d_eta, 4) || !aligned(d_alpha, 4) ||
      (ckpt && !aligned(ckpt, 16)))
    return GRADLEV_ERR_INVALID_ARG;

  void* base = nullptr;
  s = scratch_address(&base);
  if (s != GRADLEV_OK) return s;
  reset_launch_count();
  // The status word is cleared by bwd_run; the dW0 partials and the states are
  // fully overwritten by the kernels before they are read.
  return bwd_run(B, H, T, d_in, d_out, dt, x, g, eta, alpha, W0, dy, dx, dg, d_eta, d_alpha,
                 dW0, ckpt, static_cast<char*>(base), static_cast<cudaStream_t>(stream));
}

extern "C" GRADLEV_API size_t gradlev_scan_bwd_noalloc_scratch_bytes(int B, int H, int T, int d_in,
                                                                   int d_out, gradlev_dtype dt,
                                                                   int has_ckpt) {
  if (gradlev_scan_supported(B, H, T, d_in, d_out, dt) != GRADLEV_OK) return 0;
  return bwd_scratch_bytes(B, H, T, d_in, d_out, dt, has_ckpt == 0);
}

extern "C" GRADLEV_API gradlev_status gradlev_noalloc_device_status(void* stream) {
  void* base = nullptr;
  const gradlev_status s = scratch_address(&base);
  if (s != GRADLEV_OK) return s;
  DeviceStatus h;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&h, base, sizeof(h), cudaMemcpyDeviceToHost, st) != cudaSuccess)
    return GRADLEV_ERR_CUDA;
  if (cudaStreamSynchronize(st) != cudaSuccess) return GRADLEV_ERR_CUDA;
  if (h.code == 0) return GRADLEV_OK;
  return h.code == GRADLEV_ERR_TIMEOUT ? GRADLEV_ERR_TIMEOUT : GRADLEV_ERR_CUDA;
}
