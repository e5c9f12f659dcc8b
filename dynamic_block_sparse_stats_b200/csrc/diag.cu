// Diagnostics: the FMA-pipe exponential the attention forward uses for a
// share of its softmax weights, exposed so that its error can be checked
// against exp2 on the device.
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
