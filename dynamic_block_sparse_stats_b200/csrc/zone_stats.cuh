// Per (zone, head) statistics of V: the arithmetic of prism_plan's K1,
// shared by the zone-statistics kernel (which reads V from global memory)
// and the value projection's epilogue (which reads the tile it has just
// computed from shared memory), so that both give bit-identical results.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// section on zone guidance (channel variance of the mean-pooled V along T, H
// and W) and the rho_raw equation (intra-zone spatial variance plus the
// variance of frame-to-frame differences); xyznot.com review, Method
// section 1 (sigma^2_{v,d}).
//
// 256 threads (tid 0..255), 8 warps; warp t owns frame t of the zone.  Lane
// = (channel vector cv of 8 channels, token group xg).  For every row y the
// warp forms the fp32 row sum over x (fixed shuffle tree, identical for every
// frame so that equal frames give bit-equal frame sums), keeps fp32 column
// sums over y, and a sum of squares.  The 8-term partial sums are combined
// in float64.
//   o[0..4] = sigma2_T, sigma2_H, sigma2_W, spatial, temporal
// load(t, y, x, cv) returns the 16-byte vector of channels [8cv, 8cv + 8) of
// the zone's token (t, y, x); smem holds 2*8*8*D floats; sync() is a barrier
// of the 256 threads.
#pragma once

#include "common.cuh"

namespace prism {

template <int D, typename Load, typename Sync>
__device__ __forceinline__ void zone_stats_core(Load load, int tid, float *smem, double (*red)[8], double *o,
                                                Sync sync) {
  constexpr int CV = D / 8;     // 16-byte channel vectors per token
  constexpr int GPL = 32 / CV;  // token groups per warp row
  constexpr int TPL = 8 / GPL;  // tokens per lane
  float(*rowsum)[8][D] = reinterpret_cast<float(*)[8][D]>(smem);              // [t][y][c]
  float(*colsum)[8][D] = reinterpret_cast<float(*)[8][D]>(smem + 8 * 8 * D);  // [t][x][c]
  const int warp = tid >> 5, lane = tid & 31;
  const int t = warp;
  const int cv = lane % CV, xg = lane / CV;

  float colacc[TPL][8];
#pragma unroll
  for (int i = 0; i < TPL; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) colacc[i][c] = 0.f;
  double sq = 0.0;

#pragma unroll 2
  for (int y = 0; y < 8; ++y) {
    uint4 raw[TPL];
#pragma unroll
    for (int i = 0; i < TPL; ++i) raw[i] = load(t, y, xg * TPL + i, cv);
    float r[8];
    float s2 = 0.f;
#pragma unroll
    for (int c = 0; c < 8; ++c) r[c] = 0.f;
#pragma unroll
    for (int i = 0; i < TPL; ++i) {
      const uint32_t w4[4] = {raw[i].x, raw[i].y, raw[i].z, raw[i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16lo(w4[q]), b = bf16hi(w4[q]);
        r[2 * q] += a;
        r[2 * q + 1] += b;
        colacc[i][2 * q] += a;
        colacc[i][2 * q + 1] += b;
        s2 = fmaf(a, a, s2);
        s2 = fmaf(b, b, s2);
      }
    }
    sq += (double)s2;
    // combine the token groups of this row: fixed tree
#pragma unroll
    for (int o = CV; o < 32; o <<= 1)
#pragma unroll
      for (int c = 0; c < 8; ++c) r[c] += __shfl_xor_sync(0xffffffffu, r[c], o);
    if (xg == 0) {
#pragma unroll
      for (int c = 0; c < 8; ++c) rowsum[t][y][cv * 8 + c] = r[c];
    }
  }
#pragma unroll
  for (int i = 0; i < TPL; ++i)
#pragma unroll
    for (int c = 0; c < 8; ++c) colsum[t][xg * TPL + i][cv * 8 + c] = colacc[i][c];
  sq = warp_sum(sq);
  if (lane == 0) red[warp][5] = sq;
  sync();

  // Per channel (first D threads): profiles along T, H, W in float64.
  double acc[5] = {0, 0, 0, 0, 0};  // var_T, var_H, var_W, temporal, sum_t mu_t^2
  if (tid < D) {
    const int c = tid;
    double pT[8], pH[8], pW[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pT[i] = 0.0;
      pH[i] = 0.0;
      pW[i] = 0.0;
    }
#pragma unroll
    for (int a = 0; a < 8; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const double rv = (double)rowsum[a][b][c];
        pT[a] += rv;
        pH[b] += rv;
        pW[b] += (double)colsum[a][b][c];
      }
    const double inv64 = 1.0 / 64.0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      pT[i] *= inv64;
      pH[i] *= inv64;
      pW[i] *= inv64;
    }
    double mT = 0, mH = 0, mW = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      mT += pT[i];
      mH += pH[i];
      mW += pW[i];
    }
    mT *= 0.125;
    mH *= 0.125;
    mW *= 0.125;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      acc[0] += (pT[i] - mT) * (pT[i] - mT);
      acc[1] += (pH[i] - mH) * (pH[i] - mH);
      acc[2] += (pW[i] - mW) * (pW[i] - mW);
      acc[4] += pT[i] * pT[i];
    }
    acc[0] *= 0.125;
    acc[1] *= 0.125;
    acc[2] *= 0.125;
#pragma unroll
    for (int i = 0; i < 7; ++i) acc[3] += (pT[i + 1] - pT[i]) * (pT[i + 1] - pT[i]);
    acc[3] *= (1.0 / 7.0);
  }
#pragma unroll
  for (int k = 0; k < 5; ++k) acc[k] = warp_sum(acc[k]);
  if (lane == 0)
#pragma unroll
    for (int k = 0; k < 5; ++k) red[warp][k] = acc[k];
  sync();
  if (tid == 0) {
    double tot[6] = {0, 0, 0, 0, 0, 0};
    for (int w = 0; w < 8; ++w)
      for (int k = 0; k < 6; ++k) tot[k] += red[w][k];
    o[0] = tot[0] / D;
    o[1] = tot[1] / D;
    o[2] = tot[2] / D;
    // sum over t,y,x,c of (V - frame mean)^2 = sum V^2 - 64 sum_{t,c} mu_t,c^2
    double sp = (tot[5] - 64.0 * tot[4]) / (512.0 * D);
    o[3] = sp > 0.0 ? sp : 0.0;
    o[4] = tot[3] / D;
  }
}

}  // namespace prism
