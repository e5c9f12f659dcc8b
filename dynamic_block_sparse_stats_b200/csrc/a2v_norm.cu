// The A2V guidance signal: the L2 norm of the audio-to-video bridge output
// at every video token, a_{t,h,w} = ||h_hat_{t,h,w}||_2 (Prism digest, section
// on the zone guidance signals: the length of each video position's
// audio-to-video cross-attention output is its audio injection strength;
// review "Prism: динамическое разреженное внимание ...", Method section 1).
// A layer's plan reads the norms its predecessor left behind, so this runs
// once per layer on the bridge output and the next layer's prism_plan
// consumes the fp32 [N] map.
//
// HBM-bound: every row is read once (2*width bytes) and 4 bytes are written.
// One warp per row; each lane streams 16-byte vectors of the row with
// UNROLL loads in flight, keeps eight fp32 partial sums (one per bf16 slot
// of a vector), and the warp combines them with a butterfly.  bf16 squares
// are exact in fp32, so the only rounding is in the sums: a row of width w
// adds at most w/256 terms per partial, then 3 + 5 tree levels.
#include <algorithm>
#include <cstdio>

#include "common.cuh"
#include "internal.h"

namespace prism {
namespace {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;

__device__ __forceinline__ void add_squares(float (&acc)[8], const uint4 &x) {
  const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float lo = __uint_as_float(w[k] << 16);
    const float hi = __uint_as_float(w[k] & 0xffff0000u);
    acc[2 * k] = fmaf(lo, lo, acc[2 * k]);
    acc[2 * k + 1] = fmaf(hi, hi, acc[2 * k + 1]);
  }
}

__global__ void __launch_bounds__(kThreads, 8) a2v_norm_kernel(const uint4 *__restrict__ hhat, long long n,
                                                             int vec_per_row, long long ld_vec,
                                                             float *__restrict__ a) {
  const int lane = threadIdx.x & 31;
  const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
  for (long long row = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5; row < n; row += nwarps) {
    const uint4 *r = hhat + row * ld_vec;
    float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
    int v = lane;
    for (; v + 32 * (kUnroll - 1) < vec_per_row; v += 32 * kUnroll) {
      uint4 x[kUnroll];
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) x[u] = __ldcs(r + v + 32 * u);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u) add_squares(acc, x[u]);
    }
    for (; v < vec_per_row; v += 32) add_squares(acc, __ldcs(r + v));
    float s = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
    s = warp_sum(s);
    if (lane == 0) a[row] = sqrtf(s);
  }
}

int sm_count() {
  static int count = 0;
  if (count == 0) {
    int dev = 0, c = 0;
    if (cudaGetDevice(&dev) == cudaSuccess &&
        cudaDeviceGetAttribute(&c, cudaDevAttrMultiProcessorCount, dev) == cudaSuccess && c > 0)
      count = c;
    else
      return 148;
  }
  return count;
}

}  // namespace
}  // namespace prism

using namespace prism;

extern "C" int prism_a2v_norm(const uint16_t *hhat, int64_t n, int32_t width, int64_t ld, float *a2v_norm,
                              prism_stream_t stream) {
  NvtxRange nvtx_("prism_a2v_norm");
  if (n < 0) return report_error(PRISM_ERR_INVALID_ARG, "prism_a2v_norm: n must be >= 0");
  if (width <= 0 || width % 8 || width > (1 << 20))
    return report_error(PRISM_ERR_INVALID_ARG, "prism_a2v_norm: width must be a positive multiple of 8, <= 2^20");
  if (ld < width || ld % 8)
    return report_error(PRISM_ERR_INVALID_ARG, "prism_a2v_norm: ld must be a multiple of 8 and >= width");
  if (n == 0) {
    clear_error();
    return PRISM_OK;
  }
  if (!hhat || !a2v_norm) return report_error(PRISM_ERR_INVALID_ARG, "prism_a2v_norm: NULL pointer");
  if (reinterpret_cast<uintptr_t>(hhat) % 16)
    return report_error(PRISM_ERR_INVALID_ARG, "prism_a2v_norm: hhat must be 16-byte aligned");
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const long long warps_needed = n;
  const long long resident = (long long)sm_count() * (2048 / kThreads);  // full occupancy, 8 CTAs per SM
  const int grid = (int)std::min<long long>(resident, (warps_needed + kThreads / 32 - 1) / (kThreads / 32));
  {
    KernelTimer kt_(KT_A2V_NORM, st);
    a2v_norm_kernel<<<grid, kThreads, 0, st>>>(reinterpret_cast<const uint4 *>(hhat), (long long)n, width / 8,
                                               (long long)(ld / 8), a2v_norm);
  }
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    char msg[256];
    snprintf(msg, sizeof(msg), "prism_a2v_norm: %s", cudaGetErrorString(e));
    return report_error(PRISM_ERR_CUDA, msg);
  }
  clear_error();
  return PRISM_OK;
}
