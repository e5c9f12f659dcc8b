// prism_select kernels: block means, fp32 block scores, per-row hybrid
// Top-k U Top-p selection by radix select, CSR assembly and its transpose.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// section on hybrid block selection (mean-pooled block representatives,
// dot product then softmax, union of a fixed Top-k and an adaptive Top-p
// that accumulates relevance from the top until it passes the threshold);
// xyznot.com review, Method section 3 (S_i = Top-k(P_i,k) U Top-p(P_i,p)).
#include <math.h>

#include "internal.h"

namespace prism {

struct SelShape {
  int8_t lT[16], lH[16], lW[16];
};
__host__ __device__ constexpr SelShape make_sel_shapes() {
  SelShape t{};
  int n = 0;
  for (int lv = 6; lv <= 8; ++lv)
    for (int a = 1; a <= 3; ++a)
      for (int b = 1; b <= 3; ++b)
        for (int c = 1; c <= 3; ++c)
          if (a + b + c == lv) {
            t.lT[n] = (int8_t)a;
            t.lH[n] = (int8_t)b;
            t.lW[n] = (int8_t)c;
            ++n;
          }
  return t;
}
__constant__ SelShape c_sel_shapes = make_sel_shapes();

// ---------------------------------------------------------------------------
// K4: block means.  One CTA per (block, head); D threads: the first D/2
// threads pool Q (two channels each), the rest pool K.  Each channel's sum
// runs left to right over the block's tokens in raster (t,y,x) order in
// fp32, then is multiplied by 1/B (exact).
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(D) block_mean_kernel(const uint16_t *__restrict__ Q, const uint16_t *__restrict__ K,
                                                       const int32_t *__restrict__ blocks,
                                                       const int32_t *__restrict__ n_blocks, int H, int W, int heads,
                                                       int NB, float *__restrict__ Qbar, float *__restrict__ Kbar) {
  __shared__ int toff[256];
  const int b = blockIdx.x, h = blockIdx.y;
  if (b >= n_blocks[h]) return;
  const int32_t *e = blocks + ((size_t)h * NB + b) * 4;
  const int B = e[1], n0 = e[2], sid = e[3];
  const int lH = c_sel_shapes.lH[sid], lW = c_sel_shapes.lW[sid];
  for (int r = threadIdx.x; r < B; r += blockDim.x) {
    const int tt = r >> (lH + lW), yy = (r >> lW) & ((1 << lH) - 1), xx = r & ((1 << lW) - 1);
    toff[r] = (tt * H + yy) * W + xx;
  }
  __syncthreads();
  const int half = D / 2;
  const int which = threadIdx.x / half, pair = threadIdx.x % half;
  const uint32_t *src = reinterpret_cast<const uint32_t *>(which ? K : Q);
  float a0 = 0.f, a1 = 0.f;
  for (int r0 = 0; r0 < B; r0 += 8) {
    uint32_t v[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) v[u] = __ldg(src + ((size_t)(n0 + toff[r0 + u]) * heads + h) * half + pair);
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      a0 = __fadd_rn(a0, bf16lo(v[u]));
      a1 = __fadd_rn(a1, bf16hi(v[u]));
    }
  }
  const float inv = 1.0f / (float)B;  // exact: B is a power of two
  float *dst = (which ? Kbar : Qbar) + ((size_t)h * NB + b) * D + 2 * pair;
  dst[0] = __fmul_rn(a0, inv);
  dst[1] = __fmul_rn(a1, inv);
}

// ---------------------------------------------------------------------------
// K5a: scores of one head.  128x128 tile per CTA, 8x8 per thread.  Every
// score is the fp32 running sum over channels c = 0..D-1 of the separately
// rounded products Qbar_ic * Kbar_jc, then one rounded multiply by the scale.
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) block_score_kernel(const float *__restrict__ Qbar,
                                                          const float *__restrict__ Kbar,
                                                          const int32_t *__restrict__ nb_ptr, int NB, float scale,
                                                          float *__restrict__ S) {
  __shared__ __align__(16) float As[32][132];
  __shared__ __align__(16) float Bs[32][132];
  const int nb = *nb_ptr;
  const int i0 = blockIdx.y * 128, j0 = blockIdx.x * 128;
  if (i0 >= nb || j0 >= nb) return;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[8][8];
#pragma unroll
  for (int a = 0; a < 8; ++a)
#pragma unroll
    for (int b = 0; b < 8; ++b) acc[a][b] = 0.f;
  for (int c0 = 0; c0 < D; c0 += 32) {
    for (int idx = threadIdx.x; idx < 128 * 8; idx += 256) {
      const int row = idx >> 3, q = idx & 7;
      float4 va = make_float4(0.f, 0.f, 0.f, 0.f), vb = va;
      if (i0 + row < nb) va = *reinterpret_cast<const float4 *>(Qbar + (size_t)(i0 + row) * D + c0 + 4 * q);
      if (j0 + row < nb) vb = *reinterpret_cast<const float4 *>(Kbar + (size_t)(j0 + row) * D + c0 + 4 * q);
      As[4 * q + 0][row] = va.x; As[4 * q + 1][row] = va.y; As[4 * q + 2][row] = va.z; As[4 * q + 3][row] = va.w;
      Bs[4 * q + 0][row] = vb.x; Bs[4 * q + 1][row] = vb.y; Bs[4 * q + 2][row] = vb.z; Bs[4 * q + 3][row] = vb.w;
    }
    __syncthreads();
#pragma unroll 4
    for (int c = 0; c < 32; ++c) {
      const float4 a0 = *reinterpret_cast<const float4 *>(&As[c][ty * 8]);
      const float4 a1 = *reinterpret_cast<const float4 *>(&As[c][ty * 8 + 4]);
      const float4 b0 = *reinterpret_cast<const float4 *>(&Bs[c][tx * 8]);
      const float4 b1 = *reinterpret_cast<const float4 *>(&Bs[c][tx * 8 + 4]);
      const float av[8] = {a0.x, a0.y, a0.z, a0.w, a1.x, a1.y, a1.z, a1.w};
      const float bv[8] = {b0.x, b0.y, b0.z, b0.w, b1.x, b1.y, b1.z, b1.w};
#pragma unroll
      for (int a = 0; a < 8; ++a)
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = __fadd_rn(acc[a][b], __fmul_rn(av[a], bv[b]));
    }
    __syncthreads();
  }
#pragma unroll
  for (int a = 0; a < 8; ++a) {
    const int row = i0 + ty * 8 + a;
    if (row >= nb) break;
    float *dst = S + (size_t)row * NB + j0 + tx * 8;
    const int col = j0 + tx * 8;
    if (col + 8 <= nb) {
      *reinterpret_cast<float4 *>(dst) = make_float4(__fmul_rn(acc[a][0], scale), __fmul_rn(acc[a][1], scale),
                                                     __fmul_rn(acc[a][2], scale), __fmul_rn(acc[a][3], scale));
      *reinterpret_cast<float4 *>(dst + 4) = make_float4(__fmul_rn(acc[a][4], scale), __fmul_rn(acc[a][5], scale),
                                                         __fmul_rn(acc[a][6], scale), __fmul_rn(acc[a][7], scale));
    } else {
#pragma unroll
      for (int b = 0; b < 8; ++b)
        if (col + b < nb) dst[b] = __fmul_rn(acc[a][b], scale);
    }
  }
}

// ---------------------------------------------------------------------------
// K5b: hybrid selection of one query block (row).  Scores become ordered
// uint32 keys (larger score -> larger key).  e_j = exp(s_j - max) in fp32 from
// the exact float64 difference, then quantised to an integer multiple of
// 2^-qb (qb chosen so that the row's total fits 62 bits; quantum <= 2^-48 at
// the 2K grid).  Top-p sums are exact integer sums of those, so the crossing
// does not depend on the order of the atomic additions: the selection is
// deterministic.  With p >= 1 every block is kept (in exact arithmetic the
// cumulative probability reaches 1 only at the last block).  A
// most-significant-digit radix descent over the keys (8-bit digits, from the
// highest bit in which the row's keys differ) finds the Top-p crossing
// key and the Top-k threshold without sorting; the kept ids are emitted in
// ascending order into the row's own scratch, and the count into counts[i].
// ---------------------------------------------------------------------------
constexpr int kSelThreads = 512;

__device__ __forceinline__ uint32_t score_key(float s) {
  if (s == 0.0f) s = 0.0f;  // -0 and +0 are the same score
  const uint32_t b = __float_as_uint(s);
  return (b & 0x80000000u) ? ~b : (b | 0x80000000u);
}
__device__ __forceinline__ float key_score(uint32_t u) {
  return __uint_as_float((u & 0x80000000u) ? (u & 0x7fffffffu) : ~u);
}
__device__ __forceinline__ float score_weight(float s, double m) {
  const double x = (double)s - m;  // exact
  const float xh = (float)x;
  const float xl = (float)(x - (double)xh);
  const float ex = expf(xh);
  return fmaf(ex, xl, ex);  // exp(xh) * (1 + xl)
}

// quantised weight: round(e * 2^qb), e in [0, 1]
__device__ __forceinline__ unsigned long long quant_weight(float e, double qscale) {
  return __double2ull_rn((double)e * qscale);
}

struct SelShared {
  int hcnt[256];
  unsigned long long hsum[256];
  int wtot[kSelThreads / 32];
  int wtot2[kSelThreads / 32];
  unsigned long long zred[kSelThreads / 32];
  uint32_t ured[kSelThreads / 32];
  uint32_t ured2[kSelThreads / 32];
  // descent state broadcast
  uint32_t prefix;
  int found;
  int cabove;
  unsigned long long sabove;
};

// Descending scan of the 256-bucket histogram by warp 0.  Finds the first
// bucket (from the top) where `above + running >= target` (sum mode) or
// `cabove + running count >= target_n` (count mode).  Returns bucket or -1.
__device__ void bucket_descent(SelShared &sh, bool by_sum, unsigned long long target, int target_n, int shift) {
  const int lane = threadIdx.x & 31;
  // lane l owns buckets 255-8l ... 255-8l-7 (descending)
  int c[8];
  unsigned long long s[8];
  int csum = 0;
  unsigned long long ssum = 0;
#pragma unroll
  for (int k = 0; k < 8; ++k) {
    const int b = 255 - 8 * lane - k;
    c[k] = sh.hcnt[b];
    s[k] = sh.hsum[b];
    csum += c[k];
    ssum += s[k];
  }
  int cex = csum;
  unsigned long long sex = ssum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int yc = __shfl_up_sync(0xffffffffu, cex, o);
    const unsigned long long ys = __shfl_up_sync(0xffffffffu, sex, o);
    if (lane >= o) {
      cex += yc;
      sex += ys;
    }
  }
  cex -= csum;  // exclusive
  sex -= ssum;
  int hit = -1, hc = 0;
  unsigned long long hs = 0;
  {
    int rc = cex;
    unsigned long long rs = sex;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const bool reach = by_sum ? (sh.sabove + rs + s[k] >= target) : (sh.cabove + rc + c[k] >= target_n);
      if (hit < 0 && reach && c[k] > 0) {
        hit = 255 - 8 * lane - k;
        hc = rc;
        hs = rs;
      }
      rc += c[k];
      rs += s[k];
    }
  }
  const unsigned ball = __ballot_sync(0xffffffffu, hit >= 0);
  if (ball == 0) {
    if (lane == 0) sh.found = 0;
    return;
  }
  const int src = __ffs(ball) - 1;
  if (lane == src) {
    sh.found = 1;
    sh.prefix |= ((uint32_t)hit) << shift;
    sh.cabove += hc;
    sh.sabove += hs;
  }
}

__device__ __forceinline__ void block_excl_scan2(int v0, int v1, int &e0, int &e1, int &t0, int &t1,
                                                 SelShared &sh) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int i0 = v0, i1 = v1;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y0 = __shfl_up_sync(0xffffffffu, i0, o), y1 = __shfl_up_sync(0xffffffffu, i1, o);
    if (lane >= o) {
      i0 += y0;
      i1 += y1;
    }
  }
  if (lane == 31) {
    sh.wtot[warp] = i0;
    sh.wtot2[warp] = i1;
  }
  __syncthreads();
  int b0 = 0, b1 = 0;
  t0 = 0;
  t1 = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    if (w < warp) {
      b0 += sh.wtot[w];
      b1 += sh.wtot2[w];
    }
    t0 += sh.wtot[w];
    t1 += sh.wtot2[w];
  }
  e0 = b0 + i0 - v0;
  e1 = b1 + i1 - v1;
  __syncthreads();
}

// One histogram update per distinct bucket and warp instead of one per key:
// rows whose scores are close together put most keys of a digit into a few
// buckets, and per-key shared-memory atomics on those serialise.  The lanes
// with the same bucket sum their counts and weights (each weight < 2^62,
// at most 32 of them, summed exactly in three 21-bit parts) and the lowest
// of them adds.  Integer sums, so the histogram is the same in any order.
// b < 0: the lane adds nothing.  Every lane of the warp calls it.
__device__ __forceinline__ void hist_add(SelShared &sh, int b, unsigned long long w, bool with_sum) {
  const unsigned peers = __match_any_sync(0xffffffffu, b);
  if (b < 0) return;
  const bool leader = (int)(threadIdx.x & 31) == __ffs(peers) - 1;
  if (with_sum) {
    const unsigned s0 = __reduce_add_sync(peers, (unsigned)(w & 0x1fffffu));
    const unsigned s1 = __reduce_add_sync(peers, (unsigned)((w >> 21) & 0x1fffffu));
    const unsigned s2 = __reduce_add_sync(peers, (unsigned)(w >> 42));
    if (leader)
      atomicAdd(&sh.hsum[b], (unsigned long long)s0 + ((unsigned long long)s1 << 21) + ((unsigned long long)s2 << 42));
  }
  if (leader) atomicAdd(&sh.hcnt[b], __popc(peers));
}

__global__ void __launch_bounds__(kSelThreads) select_row_kernel(float *__restrict__ S, int NB,
                                                                 const int32_t *__restrict__ nb_ptr, float topk_frac,
                                                                 int topk_abs, float top_p,
                                                                 int32_t *__restrict__ counts) {
  extern __shared__ __align__(16) uint32_t sel_smem[];
  __shared__ SelShared sh;
  const int nb = *nb_ptr;
  const int i = blockIdx.x;
  if (i >= nb) return;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t *key = sel_smem;
  float *ev = reinterpret_cast<float *>(sel_smem + ((NB + 3) & ~3));
  float *row = S + (size_t)i * NB;

  // 1. keys, their maximum and minimum
  uint32_t kmax = 0, kmin = 0xffffffffu;
  for (int j = tid; j < nb; j += kSelThreads) {
    const uint32_t u = score_key(row[j]);
    key[j] = u;
    kmax = max(kmax, u);
    kmin = min(kmin, u);
  }
  kmax = warp_max(kmax);
  kmin = ~warp_max(~kmin);
  if (lane == 0) {
    sh.ured[warp] = kmax;
    sh.ured2[warp] = kmin;
  }
  __syncthreads();
  kmax = 0;
  kmin = 0xffffffffu;
  for (int w = 0; w < kSelThreads / 32; ++w) {
    kmax = max(kmax, sh.ured[w]);
    kmin = min(kmin, sh.ured2[w]);
  }
  const double m = (double)key_score(kmax);
  // The radix descent below only resolves the bits in which the row's keys
  // differ: the bits above the highest differing bit hb are common to every
  // key, so the first 8-bit digit is taken just below them, where the keys
  // spread over all 256 buckets (starting at the top byte would put nearly
  // every key of a row into one or two buckets).  At least one full digit.
  const int hb = max(31 - __clz((int)(kmax ^ kmin)), 7);  // clz(0) = 32 gives -1
  const uint32_t common = hb >= 31 ? 0u : ~((2u << hb) - 1u);

  // 2. weights, quantised to multiples of 2^-qb, and their exact total
  const int qb = 62 - (32 - __clz(nb));  // nb < 2^(32 - clz(nb)), so the total stays below 2^62
  const double qscale = ldexp(1.0, qb);
  unsigned long long zp = 0;
  for (int j = tid; j < nb; j += kSelThreads) {
    const float e = score_weight(key_score(key[j]), m);
    ev[j] = e;
    zp += quant_weight(e, qscale);
  }
  zp = warp_sum(zp);
  if (lane == 0) sh.zred[warp] = zp;
  __syncthreads();
  unsigned long long Z = 0;
  for (int w = 0; w < kSelThreads / 32; ++w) Z += sh.zred[w];

  // 3. counts: k and n_p
  int k;
  if (topk_abs > 0)
    k = min(nb, topk_abs);
  else
    k = min(nb, max(1, (int)ceil((double)topk_frac * (double)nb)));
  // target = ceil(p * Z) exactly: p = pm * 2^(e2 - 24) with a 24-bit integer pm
  unsigned long long target = 0;
  if (top_p > 0.0f && top_p < 1.0f) {
    int e2;
    const float mant = frexpf(top_p, &e2);
    const unsigned long long pm = (unsigned long long)ldexpf(mant, 24);
    const unsigned __int128 prod = (unsigned __int128)pm * Z;
    const int rs = 24 - e2;  // >= 24 for p < 1
    if (rs >= 127)
      target = prod != 0 ? 1ull : 0ull;
    else
      target = (unsigned long long)((prod + (((unsigned __int128)1 << rs) - 1)) >> rs);
  }

  int n_p = 0;
  uint32_t thr = 0;
  int need = 0;
  bool have_thr = false;
  if (top_p >= 1.0f) {
    n_p = nb;
  } else if (top_p > 0.0f) {
    if (tid == 0) {
      sh.prefix = kmax & common;
      sh.cabove = 0;
      sh.sabove = 0;
      sh.found = 1;
    }
    __syncthreads();
    uint32_t pmask = common, last_mask = 255u;
    bool ok = true;
    for (int hi = hb + 1; hi > 0; hi -= 8) {  // digit = key bits [lo, hi)
      const int shift = max(hi - 8, 0);
      const uint32_t dmask = (1u << (hi - shift)) - 1u;
      last_mask = dmask;
      for (int b = tid; b < 256; b += kSelThreads) {
        sh.hcnt[b] = 0;
        sh.hsum[b] = 0;
      }
      __syncthreads();
      const uint32_t prefix = sh.prefix;
      for (int j0 = 0; j0 < nb; j0 += kSelThreads) {  // the same trip count for every thread
        const int j = j0 + tid;
        int b = -1;
        unsigned long long wq = 0;
        if (j < nb) {
          const uint32_t u = key[j];
          if ((u & pmask) == prefix) {
            b = (int)((u >> shift) & dmask);
            wq = quant_weight(ev[j], qscale);
          }
        }
        hist_add(sh, b, wq, true);
      }
      __syncthreads();
      if (warp == 0) bucket_descent(sh, true, target, 0, shift);
      __syncthreads();
      if (!sh.found) {
        ok = false;
        break;
      }
      pmask |= dmask << shift;
    }
    if (!ok) {
      n_p = nb;  // cannot happen for p < 1 (target <= Z); kept as a safe bound
    } else {
      // every key of the final bucket is the same score, hence the same weight
      const uint32_t ustar = sh.prefix;
      const int cstar = sh.hcnt[ustar & last_mask];  // the last digit is bits [0, width)
      const unsigned long long estar = quant_weight(score_weight(key_score(ustar), m), qscale);
      const unsigned long long sab = sh.sabove;
      int q = 1;
      if (estar > 0 && target > sab) q = (int)min((unsigned long long)cstar, (target - sab + estar - 1) / estar);
      q = max(1, min(q, cstar));
      n_p = sh.cabove + q;
      thr = ustar;
      need = q;
      have_thr = true;
    }
    __syncthreads();
  }
  const int n = min(nb, max(k, n_p));
  if (!(have_thr && n == n_p)) {
    // count-based radix select of the n-th largest key
    if (tid == 0) {
      sh.prefix = kmax & common;
      sh.cabove = 0;
      sh.sabove = 0;
      sh.found = 1;
    }
    __syncthreads();
    uint32_t pmask = common;
    for (int hi = hb + 1; hi > 0; hi -= 8) {  // digit = key bits [lo, hi)
      const int shift = max(hi - 8, 0);
      const uint32_t dmask = (1u << (hi - shift)) - 1u;
      for (int b = tid; b < 256; b += kSelThreads) {
        sh.hcnt[b] = 0;
        sh.hsum[b] = 0;
      }
      __syncthreads();
      const uint32_t prefix = sh.prefix;
      for (int j0 = 0; j0 < nb; j0 += kSelThreads) {  // the same trip count for every thread
        const int j = j0 + tid;
        int b = -1;
        if (j < nb) {
          const uint32_t u = key[j];
          if ((u & pmask) == prefix) b = (int)((u >> shift) & dmask);
        }
        hist_add(sh, b, 0ull, false);
      }
      __syncthreads();
      if (warp == 0) bucket_descent(sh, false, 0ull, n, shift);
      __syncthreads();
      pmask |= dmask << shift;
    }
    thr = sh.prefix;
    need = n - sh.cabove;
    __syncthreads();
  }

  // 4. emit kept ids in ascending order into the row's scratch.  Thread t
  // owns the contiguous keys [t*Lp, t*Lp + Lp) (Lp odd, so that the threads'
  // shared-memory reads fall in different banks); the keys above thr are
  // kept, and of the keys equal to thr the first `need` in id order.  Two
  // block scans give each thread its tie rank and its output offset.
  int32_t *out = reinterpret_cast<int32_t *>(row);
  const int Lp = ((nb + kSelThreads - 1) / kSelThreads) | 1;
  const int jb = min(nb, tid * Lp), je = min(nb, jb + Lp);
  int n_gt = 0, n_tie = 0;
  for (int j = jb; j < je; ++j) {
    const uint32_t u = key[j];
    n_gt += u > thr;
    n_tie += u == thr;
  }
  int e_tie, e0, t_tie, t0;
  block_excl_scan2(n_tie, 0, e_tie, e0, t_tie, t0, sh);
  const int keep_tie = min(n_tie, max(0, need - e_tie));
  int e_sel, e1, t_sel, t1;
  block_excl_scan2(n_gt + keep_tie, 0, e_sel, e1, t_sel, t1, sh);
  int o = e_sel, ties_left = keep_tie;
  for (int j = jb; j < je; ++j) {
    const uint32_t u = key[j];
    if (u > thr || (u == thr && ties_left > 0)) {
      out[o++] = j;
      ties_left -= (u == thr);
    }
  }
  if (tid == 0) counts[i] = t_sel;
}

// ---------------------------------------------------------------------------
// CSR assembly and transpose
// ---------------------------------------------------------------------------
// Exclusive scan of in[0..n) into out[0..n] (out[n] = total), adding *base
// (when non-null) and advancing it by the total.  Single CTA of 1024 threads.
__global__ void __launch_bounds__(1024) scan_kernel(const int32_t *__restrict__ in, int n,
                                                    int32_t *__restrict__ out, long long *base, int write_total) {
  __shared__ long long wsum[32];
  __shared__ long long carry;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) carry = base ? *base : 0;
  __syncthreads();
  for (int i0 = 0; i0 < n; i0 += 1024) {
    const int i = i0 + threadIdx.x;
    const long long v = i < n ? in[i] : 0;
    long long incl = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const long long y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    long long before = 0, total = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < warp) before += wsum[w];
      total += wsum[w];
    }
    if (i < n) out[i] = (int32_t)(carry + before + incl - v);
    __syncthreads();
    if (threadIdx.x == 0) carry += total;
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    if (write_total) out[n] = (int32_t)carry;
    if (base) *base = carry;
  }
}

__global__ void __launch_bounds__(128) csr_fill_kernel(const float *__restrict__ S, int NB,
                                                       const int32_t *__restrict__ nb_ptr,
                                                       const int32_t *__restrict__ counts,
                                                       const int32_t *__restrict__ row_ptr_h,
                                                       int32_t *__restrict__ col, long long cap) {
  const int i = blockIdx.x;
  if (i >= *nb_ptr) return;
  const long long start = row_ptr_h[i];
  const int n = counts[i];
  const int32_t *src = reinterpret_cast<const int32_t *>(S + (size_t)i * NB);
  for (int r = threadIdx.x; r < n; r += blockDim.x)
    if (start + r < cap) col[start + r] = src[r];
}

__global__ void __launch_bounds__(128) csc_count_kernel(const int32_t *__restrict__ row_ptr,
                                                        const int32_t *__restrict__ col, int NB, long long cap,
                                                        int32_t *__restrict__ colcnt) {
  const int r = blockIdx.y * NB + blockIdx.x;
  const long long b = row_ptr[r], e = min((long long)row_ptr[r + 1], cap);
  for (long long q = b + threadIdx.x; q < e; q += blockDim.x) atomicAdd(&colcnt[blockIdx.y * NB + col[q]], 1);
}

__global__ void __launch_bounds__(128) csc_fill_kernel(const int32_t *__restrict__ row_ptr,
                                                       const int32_t *__restrict__ col, int NB, long long cap,
                                                       const int32_t *__restrict__ col_ptr,
                                                       int32_t *__restrict__ cursor, int32_t *__restrict__ rows) {
  const int i = blockIdx.x;
  const int r = blockIdx.y * NB + i;
  const long long b = row_ptr[r], e = min((long long)row_ptr[r + 1], cap);
  for (long long q = b + threadIdx.x; q < e; q += blockDim.x) {
    const int s = blockIdx.y * NB + col[q];
    const long long pos = (long long)col_ptr[s] + atomicAdd(&cursor[s], 1);
    if (pos < cap) rows[pos] = i;
  }
}

// Sort each CSC segment ascending with a bitmap (ids are distinct and < NB).
__global__ void __launch_bounds__(256) csc_sort_kernel(const int32_t *__restrict__ col_ptr, int NB, long long cap,
                                                       int32_t *__restrict__ rows) {
  extern __shared__ uint32_t bm[];
  __shared__ int wtot[8];
  const int s = blockIdx.y * NB + blockIdx.x;
  const long long b = col_ptr[s], e = min((long long)col_ptr[s + 1], cap);
  if (e - b <= 1) return;
  const int words = (NB + 31) / 32;
  for (int w = threadIdx.x; w < words; w += blockDim.x) bm[w] = 0;
  __syncthreads();
  for (long long q = b + threadIdx.x; q < e; q += blockDim.x) atomicOr(&bm[rows[q] >> 5], 1u << (rows[q] & 31));
  __syncthreads();
  // each thread owns a contiguous range of words
  const int per = (words + blockDim.x - 1) / blockDim.x;
  const int w0 = threadIdx.x * per, w1 = min(words, w0 + per);
  int cnt = 0;
  for (int w = w0; w < w1; ++w) cnt += __popc(bm[w]);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = cnt;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) wtot[warp] = incl;
  __syncthreads();
  int before = 0;
  for (int w = 0; w < warp; ++w) before += wtot[w];
  long long pos = b + before + incl - cnt;
  for (int w = w0; w < w1; ++w) {
    uint32_t bits = bm[w];
    while (bits) {
      const int k = __ffs(bits) - 1;
      bits &= bits - 1;
      rows[pos++] = w * 32 + k;
    }
  }
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
size_t select_max_nb(const prism_params &) {
  // two 4-byte arrays per row in shared memory of the selection kernel
  return (size_t)((220 * 1024 - sizeof(SelShared)) / 8) & ~(size_t)3;
}

struct SelWs {
  WsHeader *hdr;
  float *qbar, *kbar, *S;
  int32_t *counts, *colcnt, *cursor;
};

static SelWs carve_select(const prism_params &p, void *ws) {
  const size_t N = (size_t)p.T * p.H * p.W, NB = N / 64, h = p.heads, D = p.head_dim;
  char *w = static_cast<char *>(ws);
  SelWs s;
  s.hdr = reinterpret_cast<WsHeader *>(w);
  w += kWsHeader;
  s.qbar = reinterpret_cast<float *>(w);
  w += align_up(sizeof(float) * h * NB * D, 256);
  s.kbar = reinterpret_cast<float *>(w);
  w += align_up(sizeof(float) * h * NB * D, 256);
  s.S = reinterpret_cast<float *>(w);
  w += align_up(sizeof(float) * NB * NB, 256);
  s.counts = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * NB, 256);
  s.colcnt = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * NB, 256);
  s.cursor = reinterpret_cast<int32_t *>(w);
  return s;
}

size_t select_ws_bytes(const prism_params &p) {
  const size_t N = (size_t)p.T * p.H * p.W, NB = N / 64, h = p.heads, D = p.head_dim;
  return kWsHeader + 2 * align_up(sizeof(float) * h * NB * D, 256) + align_up(sizeof(float) * NB * NB, 256) +
         3 * align_up(sizeof(int32_t) * h * NB, 256);
}

cudaError_t launch_select(const prism_params &p, const prism_plan_t &plan, const uint16_t *Q, const uint16_t *K,
                          prism_select_t &out, void *ws, cudaStream_t st, long long *nnz_out) {
  const int N = p.T * p.H * p.W, NB = N / 64, D = p.head_dim;
  SelWs w = carve_select(p, ws);
  cudaError_t err;
  if ((err = cudaMemsetAsync(&w.hdr->nnz, 0, sizeof(long long), st)) != cudaSuccess) return err;
  if ((err = cudaMemsetAsync(w.counts, 0, sizeof(int32_t) * p.heads * NB, st)) != cudaSuccess) return err;

  dim3 gm(NB, p.heads);
  {
  KernelTimer kt_(KT_BLOCK_MEAN, st);
  if (D == 128)
    block_mean_kernel<128><<<gm, 128, 0, st>>>(Q, K, plan.blocks, plan.n_blocks, p.H, p.W, p.heads, NB, w.qbar,
                                               w.kbar);
  else
    block_mean_kernel<64><<<gm, 64, 0, st>>>(Q, K, plan.blocks, plan.n_blocks, p.H, p.W, p.heads, NB, w.qbar,
                                             w.kbar);
  }
  const float scale = effective_scale(p);
  const int tiles = (NB + 127) / 128;
  const size_t sel_smem = (size_t)8 * ((NB + 3) & ~3);
  cudaFuncSetAttribute(select_row_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sel_smem);
  for (int h = 0; h < p.heads; ++h) {
    const float *qb = w.qbar + (size_t)h * NB * D;
    const float *kb = w.kbar + (size_t)h * NB * D;
    {
      KernelTimer kt_(KT_BLOCK_SCORE, st);
      if (D == 128)
        block_score_kernel<128><<<dim3(tiles, tiles), 256, 0, st>>>(qb, kb, plan.n_blocks + h, NB, scale, w.S);
      else
        block_score_kernel<64><<<dim3(tiles, tiles), 256, 0, st>>>(qb, kb, plan.n_blocks + h, NB, scale, w.S);
    }
    {
      KernelTimer kt_(KT_SELECT_ROW, st);
      select_row_kernel<<<NB, kSelThreads, sel_smem, st>>>(w.S, NB, plan.n_blocks + h, p.topk_frac, p.topk_abs,
                                                           p.top_p, w.counts + (size_t)h * NB);
    }
    {
      KernelTimer kt_(KT_SELECT_SCAN, st);
      scan_kernel<<<1, 1024, 0, st>>>(w.counts + (size_t)h * NB, NB, out.row_ptr + (size_t)h * NB, &w.hdr->nnz,
                                      h == p.heads - 1);
    }
    {
      KernelTimer kt_(KT_CSR_FILL, st);
      csr_fill_kernel<<<NB, 128, 0, st>>>(w.S, NB, plan.n_blocks + h, w.counts + (size_t)h * NB,
                                          out.row_ptr + (size_t)h * NB, out.col, out.cap);
    }
  }
  count_launches(1 + 4 * p.heads);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  long long nnz = 0;
  if ((err = cudaMemcpyAsync(&nnz, &w.hdr->nnz, sizeof(long long), cudaMemcpyDeviceToHost, st)) != cudaSuccess)
    return err;
  if ((err = cudaStreamSynchronize(st)) != cudaSuccess) return err;
  *nnz_out = nnz;
  if (nnz > out.cap || nnz > 0x7fffffffLL) return cudaSuccess;  // caller reports capacity
  if (out.col_ptr && out.row) {
    const size_t HN = (size_t)p.heads * NB;
    if ((err = cudaMemsetAsync(w.colcnt, 0, sizeof(int32_t) * HN, st)) != cudaSuccess) return err;
    if ((err = cudaMemsetAsync(w.cursor, 0, sizeof(int32_t) * HN, st)) != cudaSuccess) return err;
    {
      KernelTimer kt_(KT_CSC_COUNT, st);
      csc_count_kernel<<<gm, 128, 0, st>>>(out.row_ptr, out.col, NB, out.cap, w.colcnt);
    }
    {
      KernelTimer kt_(KT_CSC_SCAN, st);
      scan_kernel<<<1, 1024, 0, st>>>(w.colcnt, (int)HN, out.col_ptr, nullptr, 1);
    }
    {
      KernelTimer kt_(KT_CSC_FILL, st);
      csc_fill_kernel<<<gm, 128, 0, st>>>(out.row_ptr, out.col, NB, out.cap, out.col_ptr, w.cursor, out.row);
    }
    {
      KernelTimer kt_(KT_CSC_SORT, st);
      csc_sort_kernel<<<gm, 256, sizeof(uint32_t) * ((NB + 31) / 32), st>>>(out.col_ptr, NB, out.cap, out.row);
    }
    count_launches(4);
  }
  return cudaGetLastError();
}

}  // namespace prism
