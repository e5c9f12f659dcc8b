// Diagnostics:
//   * the FMA-pipe exponential the attention kernels can use for a share of
//     their softmax weights (they take all of them from MUFU today, which
//     measured faster), exposed so that its error can be checked against
//     exp2 on the device;
//   * a self-test of the failure path every kernel wait takes: a wait on an
//     mbarrier that nothing will complete gives up after a bounded number of
//     cycles and records PRISM_ERR_TIMEOUT in the workspace status word,
//     leaving the context usable.
#include <cstdio>

#include "common.cuh"
#include "internal.h"

namespace prism {
namespace {

__global__ void exp2_check_kernel(const float *__restrict__ x, float *__restrict__ y_poly,
                                  float *__restrict__ y_mufu, long long n) {
  const long long i = 2 * ((long long)blockIdx.x * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float2 v = make_float2(x[i], i + 1 < n ? x[i + 1] : 0.f);
  const float2 p = exp2_poly2(v);
  y_poly[i] = p.x;
  y_mufu[i] = ex2f(v.x);
  if (i + 1 < n) {
    y_poly[i + 1] = p.y;
    y_mufu[i + 1] = ex2f(v.y);
  }
}

// One warp waits on an mbarrier whose only expected arrival never comes,
// with the same try_wait loop as the kernels but a caller-chosen limit.
__global__ void wait_timeout_kernel(int *status, long long limit) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_barrier_init();
  }
  __syncwarp();
  bool done = mbar_try_wait(&bar, 0);
  const long long t0 = clock64();
  while (!done && clock64() - t0 <= limit) done = mbar_try_wait(&bar, 0);
  if (!__all_sync(0xffffffffu, done) && threadIdx.x == 0) record_timeout(status, 900);
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" int prism_diag_exp2(const float *x, float *y_poly, float *y_mufu, int64_t n, prism_stream_t stream) {
  if (n < 0 || (n > 0 && (!x || !y_poly || !y_mufu)))
    return report_error(PRISM_ERR_INVALID_ARG, "prism_diag_exp2: bad arguments");
  if (n == 0) {
    clear_error();
    return PRISM_OK;
  }
  const long long pairs = (n + 1) / 2;
  exp2_check_kernel<<<(unsigned)((pairs + 255) / 256), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      x, y_poly, y_mufu, (long long)n);
  count_launches(1);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "prism_diag_exp2: %s", cudaGetErrorString(e));
    return report_error(PRISM_ERR_CUDA, msg);
  }
  clear_error();
  return PRISM_OK;
}

extern "C" int prism_diag_wait_timeout(void *workspace, size_t ws_bytes, int64_t limit_cycles,
                                       prism_stream_t stream) {
  if (!workspace || ws_bytes < kWsHeader || limit_cycles < 0 || limit_cycles > 1000000000LL)
    return report_error(PRISM_ERR_INVALID_ARG,
                        "prism_diag_wait_timeout: workspace of >= 256 bytes and 0 <= limit <= 1e9 cycles");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess) {
    wait_timeout_kernel<<<1, 32, 0, st>>>(&static_cast<WsHeader *>(workspace)->status, (long long)limit_cycles);
    count_launches(1);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    char msg[160];
    snprintf(msg, sizeof(msg), "prism_diag_wait_timeout: %s", cudaGetErrorString(e));
    return report_error(PRISM_ERR_CUDA, msg);
  }
  clear_error();
  return PRISM_OK;
}
