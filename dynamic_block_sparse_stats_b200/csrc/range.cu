// Full bf16 range for the attention operands.  The tensor-core operands are
// fp16, to which bf16 converts exactly for 2^-17 <= |x| <= 65504.  The token
// gather (permute3, and the backward's dO preparation) converts with no scale
// and flags every (tensor, head) that holds a value above 65504.  For those
// only, these kernels find the head's largest magnitude and convert it again
// with a power-of-two pre-scale 2^-e (the smallest e that brings the maximum
// to 65504 or below for Q and K, to 16 or below for V and dO, whose products
// dP = dO V^T feed dS, which must stay within fp16 too).  The attention kernels fold the scales back exactly:
// Q and K into the score scale, V and dO into the output stores and into
// Delta, which the fix-up divides by 2^(e_dO + e_V) for the heads concerned.
// A head with no flag keeps e = 0 and its results are bit-identical to the
// unscaled path.  A non-finite input records PRISM_ERR_RANGE.
#include <math.h>

#include "internal.h"

namespace prism {
namespace range {

// per (tensor, head): largest |x| of the flagged heads (float bits; a
// non-negative float orders like its bits)
__global__ void __launch_bounds__(256) range_max_kernel(RangeSrc src, int N, int heads, int D,
                                                        const int32_t *__restrict__ flag,
                                                        unsigned *__restrict__ maxbits, int *status) {
  const int t = blockIdx.z, h = blockIdx.y;
  const uint16_t *X = src.p[t];
  if (!X || !flag[t * heads + h]) return;  // uniform over the block
  const int G = D / 8;                     // 16-byte vectors per row
  float mx = 0.f;
  bool nonfinite = false;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < (size_t)N * G; q += stride) {
    const size_t n = q / G;
    const int v = (int)(q % G);
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(X + ((size_t)n * heads + h) * D + v * 8));
    const uint32_t w[4] = {a.x, a.y, a.z, a.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float lo = fabsf(bf16lo(w[k])), hi = fabsf(bf16hi(w[k]));
      nonfinite |= !(lo < INFINITY) || !(hi < INFINITY);
      mx = fmaxf(mx, fmaxf(lo, hi));
    }
  }
  if (nonfinite) record_status(status, PRISM_ERR_RANGE, 110);
  mx = warp_max(mx);
  __shared__ float red[8];
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = mx;
  __syncthreads();
  if (threadIdx.x == 0) {
    for (int w = 1; w < (int)(blockDim.x >> 5); ++w) mx = fmaxf(mx, red[w]);
    atomicMax(&maxbits[t * heads + h], __float_as_uint(mx));
  }
}

// dst[t][h][p][:] = fp16(src[t][perm[h][p]][h][:] * 2^-e) for the flagged
// (tensor, head) pairs; Delta of the heads with e_dO + e_V > 0 divided by
// 2^(e_dO + e_V) (by the blocks of tensor 3).  Grid (blocks per head, heads,
// 4): a block whose (tensor, head) needs nothing returns at once.
__global__ void __launch_bounds__(256) range_fix_kernel(const int32_t *__restrict__ perm, int N, int heads, int D,
                                                        RangeSrc src, RangeDst dst, const int32_t *__restrict__ flag,
                                                        const unsigned *__restrict__ maxbits,
                                                        float *__restrict__ delta) {
  const int t = blockIdx.z, h = blockIdx.y;
  const int es = (t == 3 && delta) ? range_exp(maxbits[3 * heads + h], 3) + range_exp(maxbits[2 * heads + h], 2) : 0;
  const int e = (src.p[t] && flag[t * heads + h]) ? range_exp(maxbits[t * heads + h], t) : 0;
  if (es == 0 && e == 0) return;  // uniform over the block; e = 0 also for a non-finite maximum
  const int G = D / 8;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < (size_t)N * G; q += stride) {
    const size_t r = (size_t)h * N + q / G;  // permuted row of head h
    const int v = (int)(q % G);
    if (es > 0 && v == 0) delta[r] = ldexpf(delta[r], -es);
    if (e > 0) {
      const int n = perm[r];
      const uint4 a = __ldg(reinterpret_cast<const uint4 *>(src.p[t] + ((size_t)n * heads + h) * D + v * 8));
      const uint32_t w[4] = {a.x, a.y, a.z, a.w};
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) o[k] = pack_f16(ldexpf(bf16lo(w[k]), -e), ldexpf(bf16hi(w[k]), -e));
      *reinterpret_cast<uint4 *>(dst.p[t] + r * D + v * 8) = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

}  // namespace range

cudaError_t launch_range_fix(const int32_t *perm, int N, int heads, int D, RangeSrc src, RangeDst dst,
                             int32_t *flag, unsigned *maxbits, float *delta, int *status, cudaStream_t st) {
  {
    KernelTimer kt_(KT_RANGE_FIX, st);
    dim3 g1(148, heads, 4);  // grid-stride over each head's rows
    range::range_max_kernel<<<g1, 256, 0, st>>>(src, N, heads, D, flag, maxbits, status);
    dim3 g2(148, heads, 4);
    range::range_fix_kernel<<<g2, 256, 0, st>>>(perm, N, heads, D, src, dst, flag, maxbits, delta);
  }
  count_launches(2);
  return cudaGetLastError();
}

}  // namespace prism
