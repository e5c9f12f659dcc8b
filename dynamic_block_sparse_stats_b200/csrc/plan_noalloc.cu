// prism_plan_noalloc: prism_plan for callers that cannot allocate device
// memory.  The scratch that prism_plan takes from its caller's workspace
// (zone statistics, per-zone block offsets and the status word) lives here
// in one file-scope device array instead, so a call needs nothing but its
// inputs and outputs.
#include <stdio.h>

#include <mutex>

#include "internal.h"

namespace prism {
namespace {

// Largest scratch the entry point can use.  The native-2K grid with 24 heads
// needs about 1.8 MiB; this holds a bit more than twice that.
constexpr size_t kNoAllocScratchBytes = 4u << 20;

// Every GPU that loads the library reserves this array until the process
// exits.  Host code may not use its name as a device address: the address is
// fetched per device with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_plan_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 256;
std::mutex g_mu;
void *g_scratch_addr[kMaxDevices] = {};

// Device address of g_plan_scratch on the current device, looked up once per
// device (with that device current) and cached.
cudaError_t scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_scratch_addr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_plan_scratch);
    if (e != cudaSuccess) return e;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return cudaSuccess;
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" int prism_plan_noalloc(const prism_params *p, const uint16_t *V, const float *a2v_norm,
                                  const prism_plan_t *out, prism_stream_t stream) {
  int rc = check_plan_call(p, V, a2v_norm, out);
  if (rc != PRISM_OK) return rc;
  const size_t need = plan_ws_bytes(*p);
  if (need > kNoAllocScratchBytes) {
    char msg[256];
    snprintf(msg, sizeof(msg),
             "prism_plan_noalloc: this grid needs %zu bytes of scratch but the built-in scratch holds %zu; "
             "call prism_plan with a caller-owned workspace instead",
             need, kNoAllocScratchBytes);
    return report_error(PRISM_ERR_CAPACITY, msg);
  }
  void *scratch = nullptr;
  cudaError_t e = scratch_address(&scratch);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "prism_plan_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
    return report_error(PRISM_ERR_CUDA, msg);
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // the status word must start at zero; the rest is fully rewritten per call
  e = cudaMemsetAsync(scratch, 0, kWsHeader, st);
  if (e == cudaSuccess) e = launch_plan(*p, V, a2v_norm, *out, scratch, st);
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "prism_plan_noalloc: %s", cudaGetErrorString(e));
    return report_error(PRISM_ERR_CUDA, msg);
  }
  clear_error();
  return PRISM_OK;
}
