// prism_plan_noalloc: prism_plan for callers that cannot allocate device
// memory.  The scratch that prism_plan takes from its caller's workspace
// (zone statistics, per-zone block offsets and the status word) lives here
// in one file-scope device array instead, so a call needs nothing but its
// inputs and outputs.
#include <stdio.h>

#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"

namespace prism {
namespace {

// Largest scratch the entry point can use.  The native-2K grid with 24 heads
// needs about 1.8 MiB; this holds a bit more than twice that.
constexpr size_t kNoAllocScratchBytes = 4u << 20;

// Every CUDA context that loads the library reserves this array until the
// context is destroyed (for the primary context: until the process exits).
// Host code may not use its name as a device address: the address is fetched
// per context with cudaGetSymbolAddress below.
static __device__ __align__(256) unsigned char g_plan_scratch[kNoAllocScratchBytes];

// A __device__ array exists once per CUDA context that loaded the library's
// module, not once per device: a second context on the same device
// (cuCtxCreate) has its own copy at another address, and so has the primary
// context that the runtime creates again after cudaDeviceReset.  The address
// is therefore cached per context, keyed by the context's id (cuCtxGetId: an
// id is never reused within a process, unlike a context handle).
typedef CUresult (*CtxGetCurrentFn)(CUcontext *);
typedef CUresult (*CtxGetIdFn)(CUcontext, unsigned long long *);

std::mutex g_mu;
std::vector<std::pair<unsigned long long, void *>> g_scratch_addr;  // (context id, address)

template <typename F>
F driver_entry(const char *name) {
  void *fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &fn, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess)
    return nullptr;
  return reinterpret_cast<F>(fn);
}

// Id of the context current on this thread, or false when the driver cannot
// say (no context current, or a driver without cuCtxGetId).
bool current_context_id(unsigned long long *id) {
  static CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return false;
  CUcontext ctx = nullptr;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of g_plan_scratch in the context current on this thread.
// The first call in a context looks it up with cudaGetSymbolAddress (which
// also sets up the runtime's context on a thread that has none yet); later
// calls in the same context take it from the cache.
cudaError_t scratch_address(void **out) {
  unsigned long long id = 0;
  std::lock_guard<std::mutex> lock(g_mu);
  if (current_context_id(&id)) {
    for (const auto &e : g_scratch_addr)
      if (e.first == id) {
        *out = e.second;
        return cudaSuccess;
      }
  }
  void *p = nullptr;
  cudaError_t e = cudaGetSymbolAddress(&p, g_plan_scratch);
  if (e != cudaSuccess) return e;
  // key by the context the lookup ran in (the runtime may only now have made
  // its context current); without an id the address is simply not cached
  if (current_context_id(&id)) g_scratch_addr.emplace_back(id, p);
  *out = p;
  return cudaSuccess;
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" int prism_plan_noalloc(const prism_params *p, const uint16_t *V, const float *a2v_norm,
                                  const prism_plan_t *out, prism_stream_t stream) {
  NvtxRange nvtx_("prism_plan_noalloc");
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
