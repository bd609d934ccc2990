// Whole-forward entry point for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or a caching allocator at all: code running under
// a runtime that owns every allocation (an engine with a fixed memory pool, a plugin
// host that forbids allocation inside its execute call, a process whose allocator is not
// initialised on the calling thread). For them this file keeps the forward's scratch --
// the quantized Q/K/V^T codes, their scale tiles, the K mean and the binary64 partial
// sums -- in one file-scope device array of fixed size. Every GPU that loads the library
// holds that array until the process exits.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "sage_fp4.h"

namespace {

// 16 MiB: enough for B*H = 16 heads of N = 4096, D = 128 (about 13.7 MiB of scratch).
constexpr size_t kStaticScratchBytes = size_t(16) << 20;

__device__ __align__(256) uint8_t g_noalloc_scratch[kStaticScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
std::mutex g_scratch_mu;

// Device address of the array on the current device. Host code must not use the
// symbol itself: on the host it names a stand-in object, not device memory. The address
// is cached per device for the life of the process, so it is only valid while the
// device's primary context lives: the library must not be used on a device after a
// cudaDeviceReset() or another teardown of that context.
sage_status_t scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return SAGE_ERR_CUDA;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return SAGE_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return SAGE_OK;
}

}  // namespace

extern "C" sage_status_t sage_fp4_attn_fwd_noalloc(const void* q, const void* k, const void* v,
                                                   void* out, sage_dtype_t dtype, int B, int H,
                                                   int N, int D, int causal, float sm_scale,
                                                   void* stream) {
  const size_t need = sage_fp4_workspace_bytes(B, H, N, D);
  if (need == 0) {
    // Empty problem or bad shape: the regular entry point reports which, launching nothing.
    return sage_fp4_attn_fwd_ex(q, k, v, out, dtype, B, H, N, D, causal, sm_scale, nullptr, 0, stream);
  }
  if (need > kStaticScratchBytes) return SAGE_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if (sage_status_t st = scratch_address(&scratch); st != SAGE_OK) return st;
  return sage_fp4_attn_fwd_ex(q, k, v, out, dtype, B, H, N, D, causal, sm_scale, scratch,
                              kStaticScratchBytes, stream);
}
