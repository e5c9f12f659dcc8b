// prism_plan kernels: zone statistics (HBM-bound single pass over V), the
// per-head finalisation (density normalisation, volume, variation indicator,
// closed-form l*, nearest candidate, block table) and the permutation.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// sections on zone guidance (r_v, abar, vhat), information density
// (rho_raw equation, thresholds 0.5/0.25, 16 candidates) and the shape loss J;
// xyznot.com review ("Prism: динамическое разреженное внимание ..."), Method
// sections 1 and 2 (sigma^2_{v,d}, r_{v,d}, g_d, B(m), l*_d, nearest
// candidate in log2 space).
#include "internal.h"
#include "zone_stats.cuh"

namespace prism {

// Candidate shapes, built by enumerating edges {2,4,8} with product in
// {64,128,256}: volume ascending, then (bT,bH,bW) lexicographic.
struct ShapeTable {
  int8_t lT[16], lH[16], lW[16];  // log2 edges
  int16_t vol[16];
};
__host__ __device__ constexpr ShapeTable make_shape_table() {
  ShapeTable t{};
  int n = 0;
  for (int lv = 6; lv <= 8; ++lv)
    for (int a = 1; a <= 3; ++a)
      for (int b = 1; b <= 3; ++b)
        for (int c = 1; c <= 3; ++c)
          if (a + b + c == lv) {
            t.lT[n] = (int8_t)a;
            t.lH[n] = (int8_t)b;
            t.lW[n] = (int8_t)c;
            t.vol[n] = (int16_t)(1 << lv);
            ++n;
          }
  return t;
}
__constant__ ShapeTable c_shapes = make_shape_table();

// ---------------------------------------------------------------------------
// K1: per (zone, head) statistics of V (arithmetic in zone_stats.cuh, shared
// with the value projection's epilogue).  One 256-thread CTA per (zone, head).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) zone_video_stats_kernel(const uint16_t *__restrict__ V, int T, int H, int W,
                                                               int heads, double *__restrict__ out) {
  extern __shared__ __align__(16) float zs_smem[];
  __shared__ double red[8][8];
  const int z = blockIdx.x, h = blockIdx.y;
  const int ZH = H / 8, ZW = W / 8;
  const int zt = z / (ZH * ZW), zh = (z / ZW) % ZH, zw = z % ZW;
  const size_t tok_stride = (size_t)heads * D;  // elements between tokens
  const uint16_t *base = V + (size_t)h * D;
  const auto load = [&](int t, int y, int x, int cv) {
    const size_t n = ((size_t)(zt * 8 + t) * H + (zh * 8 + y)) * W + zw * 8 + x;
    return __ldg(reinterpret_cast<const uint4 *>(base + n * tok_stride + cv * 8));
  };
  zone_stats_core<D>(load, threadIdx.x, zs_smem, red, out + ((size_t)h * gridDim.x + z) * 5,
                     [] { __syncthreads(); });
}

// ---------------------------------------------------------------------------
// K1a: per-zone statistics of the A2V norm map a [N] (head independent).
//   out[z][0..3] = zone mean, sigma2_T, sigma2_H, sigma2_W of a's profiles.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(64) zone_a2v_stats_kernel(const float *__restrict__ a, int T, int H, int W,
                                                            double *__restrict__ out) {
  __shared__ float v[8][8][8];
  const int z = blockIdx.x;
  const int ZH = H / 8, ZW = W / 8;
  const int zt = z / (ZH * ZW), zh = (z / ZW) % ZH, zw = z % ZW;
  const int t = threadIdx.x >> 3, y = threadIdx.x & 7;
  const size_t n0 = ((size_t)(zt * 8 + t) * H + (zh * 8 + y)) * W + zw * 8;
  const float4 p0 = __ldg(reinterpret_cast<const float4 *>(a + n0));
  const float4 p1 = __ldg(reinterpret_cast<const float4 *>(a + n0 + 4));
  v[t][y][0] = p0.x; v[t][y][1] = p0.y; v[t][y][2] = p0.z; v[t][y][3] = p0.w;
  v[t][y][4] = p1.x; v[t][y][5] = p1.y; v[t][y][6] = p1.z; v[t][y][7] = p1.w;
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int d = lane >> 3, i = lane & 7;  // lanes 0-23: (axis, position)
    double p = 0.0;
    if (d < 3) {
      for (int u = 0; u < 8; ++u)
        for (int w = 0; w < 8; ++w)
          p += (double)(d == 0 ? v[i][u][w] : d == 1 ? v[u][i][w] : v[u][w][i]);
      p *= (1.0 / 64.0);
    }
    // mean of each axis' profile over its 8 positions
    double s = p;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    const double mu = s * 0.125;
    double dev = (d < 3) ? (p - mu) * (p - mu) : 0.0;
    dev += __shfl_xor_sync(0xffffffffu, dev, 1);
    dev += __shfl_xor_sync(0xffffffffu, dev, 2);
    dev += __shfl_xor_sync(0xffffffffu, dev, 4);
    double *o = out + (size_t)z * 4;
    if (lane == 0) o[0] = mu;  // mean of the T profile = zone mean
    if (i == 0 && d < 3) o[1 + d] = dev * 0.125;
  }
}

// ---------------------------------------------------------------------------
// K2: per-head finalisation.  One CTA per head.
// ---------------------------------------------------------------------------
__device__ __forceinline__ double block_max_d(double v, double *sh) {
  v = warp_max(v);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) sh[warp] = v;
  __syncthreads();
  double r = -1.0e300;
  for (int w = 0; w < (int)(blockDim.x >> 5); ++w) r = max(r, sh[w]);
  return r;
}

__global__ void __launch_bounds__(1024) plan_finalize_kernel(const double *__restrict__ vstats,
                                                             const double *__restrict__ astats, int Z, int T,
                                                             int H, int W, int heads, int NB, float tau128,
                                                             float tau256, float eps, float map_exponent,
                                                             int guidance, int density,
                                                             uint8_t *__restrict__ zone_shape,
                                                             double *__restrict__ zone_g,
                                                             double *__restrict__ zone_rho,
                                                             int32_t *__restrict__ n_blocks,
                                                             int32_t *__restrict__ blocks,
                                                             int32_t *__restrict__ zone_first) {
  __shared__ double sh[32];
  __shared__ int scan_sh[32];
  __shared__ int carry_sh;
  const int h = blockIdx.x;
  const double *vs = vstats + (size_t)h * Z * 5;

  // rho_raw(m) of the chosen density variant (0: spatial + temporal terms)
  auto rho_raw = [&](int m) -> double {
    switch (density) {
      case 1: return vs[m * 5 + 3];
      case 2: return vs[m * 5 + 4];
      case 3: return astats[m * 4 + 0];
      default: return vs[m * 5 + 3] + vs[m * 5 + 4];
    }
  };
  double mx = 0.0, ma = 0.0;
  for (int m = threadIdx.x; m < Z; m += blockDim.x) {
    mx = max(mx, rho_raw(m));
    if (astats) ma = max(ma, astats[m * 4 + 0]);
  }
  const double rho_max = block_max_d(mx, sh);
  const double a_max = block_max_d(ma, sh);
  if (threadIdx.x == 0) carry_sh = 0;
  __syncthreads();

  const int ZH = H / 8, ZW = W / 8;
  const double t128 = (double)tau128, t256 = (double)tau256, e = (double)eps;
  for (int m0 = 0; m0 < Z; m0 += blockDim.x) {
    const int m = m0 + threadIdx.x;
    int cnt = 0, sid = 0, vol = 0;
    if (m < Z) {
      const double *s = vs + (size_t)m * 5;
      const double sv = s[0] + s[1] + s[2];
      double r[3];
      for (int d = 0; d < 3; ++d) r[d] = sv > 0.0 ? s[d] / sv : (1.0 / 3.0);
      // g_d = r_{v,d} + abar * vhat_{a,d} + eps, less the terms the guidance variant drops
      double g[3];
      for (int d = 0; d < 3; ++d) g[d] = (guidance & 1) ? 0.0 : r[d];
      if (astats && !(guidance & 2)) {
        const double *as = astats + (size_t)m * 4;
        const double abar = a_max > 0.0 ? as[0] / a_max : 0.0;
        const double sa = as[1] + as[2] + as[3];
        for (int d = 0; d < 3; ++d) g[d] = g[d] + abar * (sa > 0.0 ? as[1 + d] / sa : (1.0 / 3.0));
      }
      for (int d = 0; d < 3; ++d) g[d] = g[d] + e;
      const double rho = rho_max > 0.0 ? rho_raw(m) / rho_max : 0.0;
      vol = rho >= t128 ? 64 : (rho >= t256 ? 128 : 256);
      const double S = vol == 64 ? 6.0 : (vol == 128 ? 7.0 : 8.0);
      // l*_d for b*_d proportional to g_d^(-alpha); alpha = 1/2 is the Lagrange optimum of J
      const double alpha = map_exponent > 0.f ? (double)map_exponent : 0.5;
      const double lg0 = log2(g[0]), lg1 = log2(g[1]), lg2 = log2(g[2]);
      const double shift = (S + alpha * (lg0 + lg1 + lg2)) / 3.0;
      const double l0 = -alpha * lg0 + shift, l1 = -alpha * lg1 + shift, l2 = -alpha * lg2 + shift;
      double best = 1.0e300;
      for (int c = 0; c < 16; ++c) {
        if (c_shapes.vol[c] != vol) continue;
        const double d0 = c_shapes.lT[c] - l0, d1 = c_shapes.lH[c] - l1, d2 = c_shapes.lW[c] - l2;
        const double dist = d0 * d0 + d1 * d1 + d2 * d2;
        if (dist < best) {
          best = dist;
          sid = c;
        }
      }
      zone_shape[(size_t)h * Z + m] = (uint8_t)sid;
      if (zone_g) {
        zone_g[((size_t)h * Z + m) * 3 + 0] = g[0];
        zone_g[((size_t)h * Z + m) * 3 + 1] = g[1];
        zone_g[((size_t)h * Z + m) * 3 + 2] = g[2];
      }
      if (zone_rho) zone_rho[(size_t)h * Z + m] = rho;
      cnt = 512 / vol;
    }
    // exclusive scan of cnt over this chunk of zones
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int incl = cnt;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) scan_sh[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int v = lane < (int)(blockDim.x >> 5) ? scan_sh[lane] : 0;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += y;
      }
      scan_sh[lane] = v;  // inclusive over warps
    }
    __syncthreads();
    const int first = carry_sh + (warp > 0 ? scan_sh[warp - 1] : 0) + incl - cnt;
    if (m < Z) {
      zone_first[(size_t)h * Z + m] = first;
      const int bT = 1 << c_shapes.lT[sid], bH = 1 << c_shapes.lH[sid], bW = 1 << c_shapes.lW[sid];
      const int nbH = 8 / bH, nbW = 8 / bW;
      const int zt = m / (ZH * ZW), zh = (m / ZW) % ZH, zw = m % ZW;
      for (int b = 0; b < cnt; ++b) {
        const int it = b / (nbH * nbW), ih = (b / nbW) % nbH, iw = b % nbW;
        const int t0 = zt * 8 + it * bT, y0 = zh * 8 + ih * bH, x0 = zw * 8 + iw * bW;
        int32_t *e4 = blocks + ((size_t)h * NB + first + b) * 4;
        e4[0] = m * 512 + b * vol;
        e4[1] = vol;
        e4[2] = (t0 * H + y0) * W + x0;
        e4[3] = sid;
      }
    }
    __syncthreads();
    if (threadIdx.x == 0) carry_sh += scan_sh[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (threadIdx.x == 0) n_blocks[h] = carry_sh;
}

// ---------------------------------------------------------------------------
// K3: permutation.  perm[h][p] = natural index; inv_perm[h][n] = p.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) perm_kernel(const uint8_t *__restrict__ zone_shape, int T, int H, int W,
                                                   int Z, int32_t *__restrict__ perm, int32_t *__restrict__ inv_perm) {
  const int h = blockIdx.y;
  const int N = T * H * W;
  const int p = blockIdx.x * blockDim.x + threadIdx.x;
  if (p >= N) return;
  const int m = p >> 9, local = p & 511;
  const int sid = zone_shape[(size_t)h * Z + m];
  const int lT = c_shapes.lT[sid], lH = c_shapes.lH[sid], lW = c_shapes.lW[sid];
  const int lB = lT + lH + lW;
  const int b = local >> lB, r = local & ((1 << lB) - 1);
  const int nbH = 3 - lH, nbW = 3 - lW;  // log2 of blocks per zone edge
  const int iw = b & ((1 << nbW) - 1), ih = (b >> nbW) & ((1 << nbH) - 1), it = b >> (nbW + nbH);
  const int xx = r & ((1 << lW) - 1), yy = (r >> lW) & ((1 << lH) - 1), tt = r >> (lW + lH);
  const int ZH = H / 8, ZW = W / 8;
  const int zt = m / (ZH * ZW), zh = (m / ZW) % ZH, zw = m % ZW;
  const int t = zt * 8 + (it << lT) + tt, y = zh * 8 + (ih << lH) + yy, x = zw * 8 + (iw << lW) + xx;
  const int n = (t * H + y) * W + x;
  perm[(size_t)h * N + p] = n;
  if (inv_perm) inv_perm[(size_t)h * N + n] = p;
}

// ---------------------------------------------------------------------------
// host launchers
// ---------------------------------------------------------------------------
size_t plan_ws_bytes(const prism_params &p) {
  const size_t Z = (size_t)(p.T / 8) * (p.H / 8) * (p.W / 8);
  size_t s = kWsHeader;
  s += align_up(sizeof(double) * p.heads * Z * 5, 256);
  s += align_up(sizeof(double) * Z * 4, 256);
  s += align_up(sizeof(int32_t) * p.heads * Z, 256);
  return s;
}

double *plan_vstats(void *ws) { return reinterpret_cast<double *>(static_cast<char *>(ws) + kWsHeader); }

cudaError_t launch_plan_tail(const prism_params &p, const float *a, const prism_plan_t &out, void *ws,
                             cudaStream_t st) {
  const int Z = (p.T / 8) * (p.H / 8) * (p.W / 8);
  const int N = p.T * p.H * p.W;
  const int NB = N / 64;
  char *w = static_cast<char *>(ws) + kWsHeader;
  double *vstats = reinterpret_cast<double *>(w);
  w += align_up(sizeof(double) * p.heads * Z * 5, 256);
  double *astats = reinterpret_cast<double *>(w);
  w += align_up(sizeof(double) * Z * 4, 256);
  int32_t *zone_first = reinterpret_cast<int32_t *>(w);
  if (a) {
    KernelTimer kt_(KT_ZONE_A2V_STATS, st);
    zone_a2v_stats_kernel<<<Z, 64, 0, st>>>(a, p.T, p.H, p.W, astats);
  }
  {
    KernelTimer kt_(KT_PLAN_FINALIZE, st);
    plan_finalize_kernel<<<p.heads, 1024, 0, st>>>(vstats, a ? astats : nullptr, Z, p.T, p.H, p.W, p.heads, NB,
                                                   p.tau128, p.tau256, p.eps, p.map_exponent, p.guidance,
                                                   p.density, out.zone_shape, out.zone_g,
                                                   out.zone_rho, out.n_blocks, out.blocks, zone_first);
  }
  dim3 g3((N + 255) / 256, p.heads);
  {
    KernelTimer kt_(KT_PERM, st);
    perm_kernel<<<g3, 256, 0, st>>>(out.zone_shape, p.T, p.H, p.W, Z, out.perm, out.inv_perm);
  }
  count_launches(a ? 3 : 2);
  return cudaGetLastError();
}

cudaError_t launch_plan(const prism_params &p, const uint16_t *V, const float *a, const prism_plan_t &out, void *ws,
                        cudaStream_t st) {
  const int Z = (p.T / 8) * (p.H / 8) * (p.W / 8);
  double *vstats = plan_vstats(ws);
  dim3 g1(Z, p.heads);
  {
  KernelTimer kt_(KT_ZONE_STATS, st);
  if (p.head_dim == 128) {
    const int sm = 2 * 8 * 8 * 128 * sizeof(float);
    cudaFuncSetAttribute(zone_video_stats_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    zone_video_stats_kernel<128><<<g1, 256, sm, st>>>(V, p.T, p.H, p.W, p.heads, vstats);
  } else {
    const int sm = 2 * 8 * 8 * 64 * sizeof(float);
    zone_video_stats_kernel<64><<<g1, 256, sm, st>>>(V, p.T, p.H, p.W, p.heads, vstats);
  }
  }
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  return launch_plan_tail(p, a, out, ws, st);
}

}  // namespace prism
