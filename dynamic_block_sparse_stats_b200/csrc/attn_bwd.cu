// prism_attn_bwd: gradients of the block-sparse attention through the
// selected blocks only, on tcgen05 tensor cores.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// training section: shape assignment and block selection are constants; the
// gradient flows only through the sparse attention of the selected blocks.
// The arithmetic is the softmax-attention backward with the softmax recomputed
// from the forward's log-sum-exp:
//   P = exp(s*scale - lse), dP = dO V^T, Delta_q = sum_c dO_qc O_qc,
//   dS = P (dP - Delta), dQ = scale dS K, dK = scale dS^T Q, dV = P^T dO.
//
// Two paths.  The default (head_dim 128) is dkdvq_kernel, one CTA per
// 128-key tile that forms dK, dV and its share of dQ, summed into an fp32
// accumulator by bulk reductions (described at the kernel), then
// dq_convert_kernel.  The deterministic path is two kernels without
// reductions:
//   dq_kernel    one CTA per 128-query tile; walks the CSR like the forward,
//                two key units (128 keys) per step: S = Q K^T and dP = dO V^T
//                with Q and dO held in TMEM (TS MMAs), dS -> TMEM (fp16),
//                dQ += dS K (TS MMA).
//   dkdv_kernel  one CTA per 128-key tile; walks the transpose (CSC), two
//                query units per step: S^T = K Q^T, dP^T = V dO^T (TMEM),
//                P^T and dS^T -> TMEM (fp16), dV += P^T dO, dK += dS^T Q (TS
//                MMAs), issued dV(i-1), S^T(i), dK(i-1), dP^T(i): the
//                softmax of step i overlaps dK(i-1) and dP^T(i), and S^T(i)
//                waits only for dV(i-1) to have read P^T(i-1).
// Operands are fp16 conversions of the bf16 inputs (exact for 2^-17 <= |x| <=
// 65504 and for 0, see the forward; heads beyond that range are pre-scaled by
// a power of two that the kernels fold back).
// Roles: warp 0 TMA producer, warp 1 TMEM owner and MMA issuer, warps 4-11
// two compute warpgroups (one thread per TMEM lane), each taking one of the
// step's two 64-token units.
#include "attn_walk.cuh"

namespace prism {
namespace bwd {
using namespace attn;

constexpr int kThreads = 384;  // warp 0 TMA, warp 1 MMA, warps 4-11 two compute warpgroups
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------------------
// prep: dOp[h][p] = fp16(dO[perm][h]), delta[h][p] = sum_c dO*(O + O_res)
// (O_res, the forward's bf16 rounding residual, may be NULL), lse2 = lse*log2e,
// and, for the fused kernel, the fp32 dQ accumulator's row p zeroed;
// a dO value outside the fp16 range flags its head in range_flag_do
// ---------------------------------------------------------------------------
template <int D>
__global__ void __launch_bounds__(256) bwd_prep_kernel(const int32_t *__restrict__ perm, int N, int heads,
                                                       const uint16_t *__restrict__ dO,
                                                       const uint16_t *__restrict__ O,
                                                       const uint16_t *__restrict__ O_res,
                                                       const float *__restrict__ lse, uint16_t *__restrict__ dOp,
                                                       float *__restrict__ lse2p, float *__restrict__ deltap,
                                                       int32_t *__restrict__ range_flag_do,
                                                       float *__restrict__ dq_acc) {
  constexpr int G = D / 8;  // lanes per row
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t r = g / G;
  const int v = (int)(g % G);
  const size_t rows = (size_t)heads * N;
  const bool live = r < rows;
  float acc = 0.f;
  if (live) {
    const int h = (int)(r / N);
    const int n = perm[r];
    const size_t src = ((size_t)n * heads + h) * D + v * 8;
    const uint4 a = __ldg(reinterpret_cast<const uint4 *>(dO + src));
    const uint4 b = __ldg(reinterpret_cast<const uint4 *>(O + src));
    bool bad = false;
    *reinterpret_cast<uint4 *>(dOp + r * D + v * 8) =
        make_uint4(bf16x2_to_f16x2(a.x, bad), bf16x2_to_f16x2(a.y, bad), bf16x2_to_f16x2(a.z, bad),
                   bf16x2_to_f16x2(a.w, bad));
    if (bad) atomicOr(&range_flag_do[h], 1);  // range.cu converts this head again, pre-scaled
    const uint4 c = O_res ? __ldg(reinterpret_cast<const uint4 *>(O_res + src)) : make_uint4(0, 0, 0, 0);
    const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, bw[4] = {b.x, b.y, b.z, b.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      acc = fmaf(bf16lo(aw[q]), bf16lo(bw[q]) + bf16lo(cw[q]), acc);
      acc = fmaf(bf16hi(aw[q]), bf16hi(bw[q]) + bf16hi(cw[q]), acc);
    }
    if (v == 0) lse2p[r] = lse[(size_t)h * N + n] * kLog2e;
    if (dq_acc) {  // the fused kernel adds into it
      float4 *z = reinterpret_cast<float4 *>(dq_acc + r * D + v * 8);
      z[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      z[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
#pragma unroll
  for (int o = 1; o < G; o <<= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (live && v == 0) deltap[r] = acc;
}

// ---------------------------------------------------------------------------
// Shared pieces of the two kernels.  Both walk the streamed side's 64-token
// units in pairs: one step is up to 128 streamed tokens, so every S-like
// product is a full-width M=128, N=128 tcgen05.mma (narrower products run
// the tensor pipe at a fraction of its rate).  The two compute warpgroups
// share the TMEM lanes (one thread per row of the CTA's tile) and split a
// step by unit: warpgroup g takes the step's unit g (fp32 columns
// [64g, 64g+64) of a product).  Each writes its fp16 results, packed two per
// column, into the first 32 columns of its own range, so neither overwrites
// columns the other may still be reading.  The TS MMA's 16-wide K slice ks
// therefore starts at column pk_col(ks).
// ---------------------------------------------------------------------------
constexpr int NS = 2;  // ring depth (steps of up to two 64-token units)
constexpr int kPolyPairs = 0;  // of every 16 column pairs, this many take exp2_poly2 (none: measured no faster)

__host__ __device__ constexpr uint32_t pk_col(int ks) { return (uint32_t)((ks >> 2) * 64 + (ks & 3) * 8); }

template <int D>
__device__ __forceinline__ void store_row(void *out, bool fp32, size_t off, const uint32_t (&o)[32], float mul) {
  if (fp32) {
    float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(out) + off);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(__uint_as_float(o[4 * i]) * mul, __uint_as_float(o[4 * i + 1]) * mul,
                           __uint_as_float(o[4 * i + 2]) * mul, __uint_as_float(o[4 * i + 3]) * mul);
  } else {
    uint4 v[4];
    uint32_t *pv = reinterpret_cast<uint32_t *>(v);
#pragma unroll
    for (int i = 0; i < 16; ++i) pv[i] = pack_bf16(__uint_as_float(o[2 * i]) * mul, __uint_as_float(o[2 * i + 1]) * mul);
    uint4 *dst = reinterpret_cast<uint4 *>(static_cast<uint16_t *>(out) + off);
#pragma unroll
    for (int i = 0; i < 4; ++i) dst[i] = v[i];
  }
}

// P = 2^(s * scale_log2 - lse2) for 32 fp32 scores; a share of the
// exponentials on the FMA pipe.  neg_lse2(k) gives -lse2 of column k's pair
// partner (per column for dK/dV, one value per row for dQ).
template <typename F>
__device__ __forceinline__ void softmax_p32(const uint32_t (&sv)[32], float scale_log2, F neg_lse2, float *pf) {
#pragma unroll
  for (int k = 0; k < 32; k += 2) {
    const float2 x = ffma2(make_float2(__uint_as_float(sv[k]), __uint_as_float(sv[k + 1])),
                           make_float2(scale_log2, scale_log2), neg_lse2(k));
    const float2 p = k < 2 * kPolyPairs ? exp2_poly2(x) : make_float2(ex2f(x.x), ex2f(x.y));
    pf[k] = p.x;
    pf[k + 1] = p.y;
  }
}

// ---------------------------------------------------------------------------
// dQ kernel: one CTA per 128-query tile; steps over pairs of the key units of
// the union of its rows' selections.
//   TMEM: dQ [0, 128); Q and dO as fp16 MMA operands [128, 192) and
//   [192, 256) (loaded once, so S and dP are TS products that read only K
//   and V from shared memory); S [256, 384); dP [384, 512), dS packed into
//   the dP columns.
//   Per step the MMA issue order is S(i+1), dQ(i), dP(i+1): the next S runs
//   while the compute warps turn dP(i) into dS(i).
// ---------------------------------------------------------------------------
constexpr int NSQ = 3;  // K/V ring depth of the dQ kernel

template <int D>
struct DqSmem {
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE = 128 * D * 2;  // 128 rows of fp16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + NSQ * TILE;
  static constexpr int OFF_BAR = OFF_V + NSQ * TILE;
  static constexpr int BYTES = OFF_BAR + 256;
};

struct DqBars {
  uint64_t k_full[NSQ], v_full[NSQ], k_empty[NSQ], v_empty[NSQ];
  uint64_t qdo_ready;  // Q and dO are in TMEM (256 arrivals)
  uint64_t s_full, s_free, dp_full, ds_ready, dq_done;
  uint64_t fin;    // single use: every MMA of the tile has completed
  uint64_t drain;  // single use: the MMA thread's in-flight products after an abort
  int meta[NSQ];  // units | mask_a << 4 | mask_b << 8 (bit = 64-row half of the tile)
  uint32_t tmem_base;
  int nsteps, nunits, abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dq_kernel(const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
              const uint16_t *__restrict__ Qp, const uint16_t *__restrict__ dOp,
              const int32_t *__restrict__ row_ptr, const int32_t *__restrict__ col, const int32_t *__restrict__ blocks,
              const int32_t *__restrict__ unit_block, const int32_t *__restrict__ tile_units,
              const int32_t *__restrict__ perm, const float *__restrict__ lse2p, const float *__restrict__ deltap,
              void *__restrict__ dQ, int grad_fp32, int N, int heads, float scale_log2_in, float sm_scale_in,
              const unsigned *__restrict__ range_max, int *status) {
  using L = DqSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  DqBars &bar = *reinterpret_cast<DqBars *>(smem + L::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, h = blockIdx.y;
  const int NB = N / 64;
  const int32_t *blocks_h = blocks + (size_t)h * NB * 4;
  // operands pre-scaled by 2^-e (range.cu; e = 0, no change, for in-range
  // heads): S = scale Q K^T takes 2^(eQ + eK) back, Delta already carries
  // 2^-(edO + eV) like dP, and dQ = scale dS K takes 2^(edO + eV + eK)
  const int eQ = range_exp(range_max[h], 0), eK = range_exp(range_max[heads + h], 1);
  const int eV = range_exp(range_max[2 * heads + h], 2), eO = range_exp(range_max[3 * heads + h], 3);
  const float scale_log2 = ldexpf(scale_log2_in, eQ + eK);
  const float sm_scale = ldexpf(sm_scale_in, eO + eV + eK);

  if (threadIdx.x == 0) bar.abort = *reinterpret_cast<volatile int *>(status);
  __syncthreads();
  if (bar.abort) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSQ; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    mbar_init(&bar.qdo_ready, 256);
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.s_free, 256);
    mbar_init(&bar.dp_full, 1);
    mbar_init(&bar.ds_ready, 256);
    mbar_init(&bar.dq_done, 1);
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.drain, 1);
    bar.nunits = tile_units[(size_t)h * (N / 128) + tile];
    bar.nsteps = (bar.nunits + 1) >> 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int nsteps = bar.nsteps, nunits = bar.nunits;
  const uint32_t tQacc = tmem, tQ16 = tmem + 128, tdO16 = tmem + 192, tS = tmem + 256, tdP = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const int blk[2] = {unit_block[(size_t)h * NB + 2 * tile], unit_block[(size_t)h * NB + 2 * tile + 1]};
    UnitWalk<2> w;
    walk_init<2>(w, blk, 2, row_ptr, h * NB);
    int k_issued = 0, v_issued = 0;
    for (int j = 0; j < nsteps; ++j) {
      const int s = j % NSQ;
      uint32_t ua, ub = 0;
      int ma, mb = 0, nu = 1;
      walk_next<2>(w, col, blocks_h, ua, ma);
      if (2 * j + 2 <= nunits) {
        walk_next<2>(w, col, blocks_h, ub, mb);
        nu = 2;
      }
      PRISM_CHECK(ua < (uint32_t)NB && ub < (uint32_t)NB, status, 125);
      ua = min(ua, (uint32_t)(NB - 1));  // a well-formed walk never clamps
      ub = min(ub, (uint32_t)(NB - 1));
      if (lane == 0) {
        bool ok = true;
        if (j >= NSQ) ok = mbar_wait(&bar.k_empty[s], ((j / NSQ) - 1) & 1, status, 21);
        if (ok) {
          bar.meta[s] = nu | (ma << 4) | (mb << 8);
          uint8_t *ks = smem + L::OFF_K + s * L::TILE;
          mbar_arrive_expect_tx(&bar.k_full[s], nu * 64 * D * 2);
#pragma unroll
          for (int c = 0; c < L::CHUNKS; ++c) {
            tma_load_2d(ks + c * (128 * 128), &mapK, &bar.k_full[s], c * 64, h * N + (int)ua * 64);
            if (nu == 2) tma_load_2d(ks + c * (128 * 128) + 64 * 128, &mapK, &bar.k_full[s], c * 64, h * N + (int)ub * 64);
          }
          ++k_issued;
        }
        if (ok && j >= NSQ) ok = mbar_wait(&bar.v_empty[s], ((j / NSQ) - 1) & 1, status, 20);
        if (ok) {
          uint8_t *vs = smem + L::OFF_V + s * L::TILE;
          mbar_arrive_expect_tx(&bar.v_full[s], nu * 64 * D * 2);
#pragma unroll
          for (int c = 0; c < L::CHUNKS; ++c) {
            tma_load_2d(vs + c * (128 * 128), &mapV, &bar.v_full[s], c * 64, h * N + (int)ua * 64);
            if (nu == 2) tma_load_2d(vs + c * (128 * 128) + 64 * 128, &mapV, &bar.v_full[s], c * 64, h * N + (int)ub * 64);
          }
          ++v_issued;
        }
        if (!ok) bar.abort = 1;
      }
      __syncwarp();
      if (*reinterpret_cast<volatile int *>(&bar.abort)) break;
    }
    if (lane == 0) {  // no copy may still be writing when the CTA leaves
      drain_loads(bar.k_full, NSQ, k_issued, status, 31);
      drain_loads(bar.v_full, NSQ, v_issued, status, 32);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_full = idesc_f16(128, 128, 0), id_half = idesc_f16(128, 64, 0);
      const uint32_t id_acc = idesc_f16(128, D, 1);
      // S(i) = Q K_i^T (TS); waits for the stage's K and for the compute warps
      // to have read S(i-1)
      auto issue_s = [&](int i) -> bool {
        const int s = i % NSQ;
        bool ok = mbar_wait(&bar.k_full[s], (i / NSQ) & 1, status, 24);
        if (ok && i >= 1) ok = mbar_wait(&bar.s_free, (i - 1) & 1, status, 26);
        if (!ok) return false;
        tc_fence_after();
        const int nu = bar.meta[s] & 15;  // written before the stage's K arrived
        const uint64_t dK = sdesc_sw128(smem_u32(smem + L::OFF_K + s * L::TILE), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tS, tQ16 + kk * 8, dK + kslice16(kk, 128 * 128), nu == 2 ? id_full : id_half, kk > 0 ? 1u : 0u);
        mma_commit(&bar.s_full);
        return true;
      };
      // dP(i) = dO V_i^T (TS) into the dP columns, free once dQ(i-1) read dS(i-1)
      auto issue_dp = [&](int i) -> bool {
        const int s = i % NSQ;
        bool ok = mbar_wait(&bar.v_full[s], (i / NSQ) & 1, status, 25);
        if (ok && i >= 1) ok = mbar_wait(&bar.dq_done, (i - 1) & 1, status, 27);
        if (!ok) return false;
        tc_fence_after();
        const int nu = bar.meta[s] & 15;
        const uint64_t dV = sdesc_sw128(smem_u32(smem + L::OFF_V + s * L::TILE), 16, 1024);
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ts(tdP, tdO16 + kk * 8, dV + kslice16(kk, 128 * 128), nu == 2 ? id_full : id_half, kk > 0 ? 1u : 0u);
        mma_commit(&bar.dp_full);
        mma_commit(&bar.v_empty[s]);
        return true;
      };
      bool ok = mbar_wait(&bar.qdo_ready, 0, status, 22);
      tc_fence_after();
      if (ok && nsteps > 0) ok = issue_s(0) && issue_dp(0);
      for (int i = 0; ok && i < nsteps; ++i) {
        if (i + 1 < nsteps && !(ok = issue_s(i + 1))) break;
        // dQ += dS(i) K(i)
        const int s = i % NSQ;
        ok = mbar_wait(&bar.ds_ready, i & 1, status, 23);
        if (!ok) break;
        tc_fence_after();
        const int nu = bar.meta[s] & 15;
        const uint64_t dKmn = sdesc_sw128(smem_u32(smem + L::OFF_K + s * L::TILE), 128 * 128, 1024);
        for (int ks = 0; ks < 4 * nu; ++ks)
          mma_ts(tQacc, tdP + pk_col(ks), dKmn + (uint64_t)ks * 128, id_acc, (i > 0 || ks > 0) ? 1u : 0u);
        mma_commit(&bar.dq_done);
        mma_commit(&bar.k_empty[s]);
        if (i + 1 < nsteps && !(ok = issue_dp(i + 1))) break;
      }
      if (ok && nsteps > 0) mma_commit(&bar.fin);
      if (!ok) {
        bar.abort = 1;
        mma_drain(&bar.drain, status, 33);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ compute
    const int g = (warp - 4) >> 2;  // warpgroup: key unit g of every step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int half = row >> 6;  // warp-uniform
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const size_t prow = (size_t)h * N + (size_t)tile * 128 + row;
    const float lse2 = lse2p[prow], dl = deltap[prow];
    const auto row_lse = [lse2](int) { return make_float2(-lse2, -lse2); };
    // Q and dO rows into TMEM as fp16 operands (two elements per column):
    // warpgroup g stores elements [g D/2, (g+1) D/2) of the row
    {
      const uint4 *qs = reinterpret_cast<const uint4 *>(Qp + prow * D + (D / 2) * g);
      const uint4 *os = reinterpret_cast<const uint4 *>(dOp + prow * D + (D / 2) * g);
      uint32_t q[32], o[32];
#pragma unroll
      for (int v = 0; v < D / 16; ++v) {
        const uint4 a = __ldg(qs + v), b = __ldg(os + v);
        q[4 * v] = a.x, q[4 * v + 1] = a.y, q[4 * v + 2] = a.z, q[4 * v + 3] = a.w;
        o[4 * v] = b.x, o[4 * v + 1] = b.y, o[4 * v + 2] = b.z, o[4 * v + 3] = b.w;
      }
      if (D == 128) {
        tmem_st32(tQ16 + lane_off + 32 * g, q);
        tmem_st32(tdO16 + lane_off + 32 * g, o);
      } else {
        tmem_st16(tQ16 + lane_off + 16 * g, q);
        tmem_st16(tdO16 + lane_off + 16 * g, o);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.qdo_ready);
    }
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % NSQ;
      ok = mbar_wait_warp(&bar.s_full, i & 1, status, 28);
      if (!ok) break;
      tc_fence_after();
      const int meta = bar.meta[s];
      const bool active = g < (meta & 15);
      const bool valid = active && (((meta >> (4 + 4 * g)) >> half) & 1);  // warp-uniform
      float pf[64];
      if (valid) {
        uint32_t sv[2][32];
        tmem_ld32(tS + lane_off + 64 * g, sv[0]);
        tmem_ld32(tS + lane_off + 64 * g + 32, sv[1]);
        tmem_wait_ld();
        softmax_p32(sv[0], scale_log2, row_lse, pf);
        softmax_p32(sv[1], scale_log2, row_lse, pf + 32);
      }
      tc_fence_before();
      mbar_arrive(&bar.s_free);  // S(i) read: S(i+1) may overwrite it
      ok = mbar_wait_warp(&bar.dp_full, i & 1, status, 29);
      if (!ok) break;
      tc_fence_after();
      uint32_t dv[2][32];
      if (valid) tmem_ld32(tdP + lane_off + 64 * g, dv[0]);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        if (valid) {
          tmem_wait_ld_r(dv[c]);
          if (c == 0) tmem_ld32(tdP + lane_off + 64 * g + 32, dv[1]);
#pragma unroll
          for (int k = 0; k < 32; k += 2) {
            const float2 d = fmul2(make_float2(pf[32 * c + k], pf[32 * c + k + 1]),
                                   fsub2(make_float2(__uint_as_float(dv[c][k]), __uint_as_float(dv[c][k + 1])),
                                         make_float2(dl, dl)));
            pk[k / 2] = pack_f16(d.x, d.y);
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        }
        // dS goes into the first half of this warpgroup's own dP columns,
        // below the chunk-1 values still loading
        if (active) tmem_st16(tdP + lane_off + 64 * g + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.ds_ready);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nsteps > 0) ok = mbar_wait_warp(&bar.fin, 0, status, 30);
    if (ok) {
      tc_fence_after();
      int n = perm[prow];
      if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 127)) n = 0;
      const size_t off = ((size_t)n * heads + h) * D;
#pragma unroll 1
      for (int c = g * (D / 2); c < (g + 1) * (D / 2); c += 32) {
        uint32_t o[32];
        if (nsteps > 0) {
          tmem_ld32(tQacc + lane_off + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        store_row<D>(dQ, grad_fp32 != 0, off + c, o, sm_scale);
      }
    } else {
      bar.abort = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// ---------------------------------------------------------------------------
// dK/dV kernel: one CTA per 128-key tile; steps over pairs of the query units
// of the union of its blocks' columns (the transpose of the selection).
//   TMEM: dV [0, 128), dK [128, 256), S^T [256, 384) (P^T packed into it),
//   dP^T [384, 512) (dS^T packed into it).
// ---------------------------------------------------------------------------
template <int D>
struct KvSmem {
  static constexpr int CHUNKS = D / 64;
  static constexpr int TILE = 128 * D * 2;
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;                // ring of query-unit pairs
  static constexpr int OFF_DO = OFF_Q + NS * TILE;          // ring of dO-unit pairs
  static constexpr int OFF_STAT = OFF_DO + NS * TILE;       // [NS][lse2 128, delta 128] floats
  static constexpr int OFF_BAR = OFF_STAT + NS * 256 * 4;
  static constexpr int BYTES = OFF_BAR + 256;
};

struct KvBars {
  uint64_t kv_full;
  uint64_t q_full[NS], q_empty[NS];
  uint64_t s_full, dp_full, p_ready, ds_ready, dv_done, dk_done;
  uint64_t fin;    // single use: every MMA of the tile has completed
  uint64_t drain;  // single use: the MMA thread's in-flight products after an abort
  int meta[NS];    // units | mask_a << 4 | mask_b << 8 (bit = 64-row half of the key tile)
  uint32_t tmem_base;
  int nsteps, nunits, abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    dkdv_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapDO,
                const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                const int32_t *__restrict__ col_ptr, const int32_t *__restrict__ rowidx,
                const int32_t *__restrict__ blocks, const int32_t *__restrict__ unit_block,
                const int32_t *__restrict__ tile_units, const int32_t *__restrict__ perm,
                const float *__restrict__ lse2p, const float *__restrict__ deltap, void *__restrict__ dK,
                void *__restrict__ dV, int grad_fp32, int N, int heads, float scale_log2_in, float sm_scale_in,
                const unsigned *__restrict__ range_max, int *status) {
  using L = KvSmem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  KvBars &bar = *reinterpret_cast<KvBars *>(smem + L::OFF_BAR);
  float *stat = reinterpret_cast<float *>(smem + L::OFF_STAT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, h = blockIdx.y;
  const int NB = N / 64;
  const int32_t *blocks_h = blocks + (size_t)h * NB * 4;
  // operands pre-scaled by 2^-e (range.cu; e = 0, no change, for in-range
  // heads): S^T takes 2^(eQ + eK) back, dV = P^T dO takes 2^edO, and
  // dK = scale dS^T Q takes 2^(edO + eV + eQ) (Delta carries 2^-(edO + eV))
  const int eQ = range_exp(range_max[h], 0), eK = range_exp(range_max[heads + h], 1);
  const int eV = range_exp(range_max[2 * heads + h], 2), eO = range_exp(range_max[3 * heads + h], 3);
  const float scale_log2 = ldexpf(scale_log2_in, eQ + eK);
  const float sm_scale = ldexpf(sm_scale_in, eO + eV + eQ);
  const float dv_scale = ldexpf(1.0f, eO);

  if (threadIdx.x == 0) bar.abort = *reinterpret_cast<volatile int *>(status);
  __syncthreads();
  if (bar.abort) return;
  if (threadIdx.x == 0) {
    mbar_init(&bar.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
    }
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.dp_full, 1);
    mbar_init(&bar.p_ready, 256);
    mbar_init(&bar.ds_ready, 256);
    mbar_init(&bar.dv_done, 1);
    mbar_init(&bar.dk_done, 1);
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.drain, 1);
    bar.nunits = tile_units[(size_t)h * (N / 128) + tile];
    bar.nsteps = (bar.nunits + 1) >> 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int nsteps = bar.nsteps, nunits = bar.nunits;
  const uint32_t tV = tmem, tK = tmem + 128, tS = tmem + 256, tP = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const int blk[2] = {unit_block[(size_t)h * NB + 2 * tile], unit_block[(size_t)h * NB + 2 * tile + 1]};
    UnitWalk<2> w;
    walk_init<2>(w, blk, 2, col_ptr, h * NB);
    int q_issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar.kv_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < L::CHUNKS; ++c) {
        tma_load_2d(smem + L::OFF_K + c * (128 * 128), &mapK, &bar.kv_full, c * 64, h * N + tile * 128);
        tma_load_2d(smem + L::OFF_V + c * (128 * 128), &mapV, &bar.kv_full, c * 64, h * N + tile * 128);
      }
    }
    for (int j = 0; j < nsteps; ++j) {
      const int s = j % NS;
      uint32_t ua, ub = 0;
      int ma, mb = 0, nu = 1;
      walk_next<2>(w, rowidx, blocks_h, ua, ma);
      if (2 * j + 2 <= nunits) {
        walk_next<2>(w, rowidx, blocks_h, ub, mb);
        nu = 2;
      }
      PRISM_CHECK(ua < (uint32_t)NB && ub < (uint32_t)NB, status, 126);
      ua = min(ua, (uint32_t)(NB - 1));
      ub = min(ub, (uint32_t)(NB - 1));
      if (lane == 0) {
        bool ok = true;
        if (j >= NS) ok = mbar_wait(&bar.q_empty[s], ((j / NS) - 1) & 1, status, 41);
        if (!ok) bar.abort = 1;
        if (ok) {
          bar.meta[s] = nu | (ma << 4) | (mb << 8);
          uint8_t *qs = smem + L::OFF_Q + s * L::TILE;
          uint8_t *os = smem + L::OFF_DO + s * L::TILE;
          float *st = stat + s * 256;
          mbar_arrive_expect_tx(&bar.q_full[s], nu * (2 * 64 * D * 2 + 2 * 64 * 4));
#pragma unroll
          for (int c = 0; c < L::CHUNKS; ++c) {
            tma_load_2d(qs + c * (128 * 128), &mapQ, &bar.q_full[s], c * 64, h * N + (int)ua * 64);
            tma_load_2d(os + c * (128 * 128), &mapDO, &bar.q_full[s], c * 64, h * N + (int)ua * 64);
            if (nu == 2) {
              tma_load_2d(qs + c * (128 * 128) + 64 * 128, &mapQ, &bar.q_full[s], c * 64, h * N + (int)ub * 64);
              tma_load_2d(os + c * (128 * 128) + 64 * 128, &mapDO, &bar.q_full[s], c * 64, h * N + (int)ub * 64);
            }
          }
          bulk_load(st, lse2p + (size_t)h * N + (size_t)ua * 64, 256, &bar.q_full[s]);
          bulk_load(st + 128, deltap + (size_t)h * N + (size_t)ua * 64, 256, &bar.q_full[s]);
          if (nu == 2) {
            bulk_load(st + 64, lse2p + (size_t)h * N + (size_t)ub * 64, 256, &bar.q_full[s]);
            bulk_load(st + 192, deltap + (size_t)h * N + (size_t)ub * 64, 256, &bar.q_full[s]);
          }
          ++q_issued;
        }
      }
      __syncwarp();
      if (*reinterpret_cast<volatile int *>(&bar.abort)) break;
    }
    if (lane == 0) {  // no copy may still be writing when the CTA leaves
      drain_loads(&bar.kv_full, 1, 1, status, 52);
      drain_loads(bar.q_full, NS, q_issued, status, 53);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_full = idesc_f16(128, 128, 0), id_half = idesc_f16(128, 64, 0);
      const uint32_t id_acc = idesc_f16(128, D, 1);
      const uint64_t dKd = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, 1024);
      const uint64_t dVd = sdesc_sw128(smem_u32(smem + L::OFF_V), 16, 1024);
      bool ok = mbar_wait(&bar.kv_full, 0, status, 42);
      tc_fence_after();
      // Step i's products, in the order dV(i-1), S^T(i), dK(i-1), dP^T(i):
      // S^T(i) is issued as soon as dV(i-1) has read P^T(i-1), so the
      // softmax of step i can follow the compute warps' dS of step i-1
      // without waiting for dK(i-1).
      for (int i = 0; ok && i <= nsteps; ++i) {
        const int s = i % NS, sp = (i + NS - 1) % NS;
        const int nup = i >= 1 ? (bar.meta[sp] & 15) : 0;  // stage sp is not refilled before dK(i-1)
        if (i >= 1) {  // dV += P^T(i-1) dO(i-1)
          ok = mbar_wait(&bar.p_ready, (i - 1) & 1, status, 43);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dDOmn = sdesc_sw128(smem_u32(smem + L::OFF_DO + sp * L::TILE), 128 * 128, 1024);
          for (int ks = 0; ks < 4 * nup; ++ks)
            mma_ts(tV, tS + pk_col(ks), dDOmn + (uint64_t)ks * 128, id_acc, (i > 1 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.dv_done);
        }
        uint32_t id = id_full;
        uint64_t dDOs = 0;
        if (i < nsteps) {  // S^T(i) = K Q(i)^T, into the columns dV(i-1) read P^T(i-1) from
          ok = mbar_wait(&bar.q_full[s], (i / NS) & 1, status, 44);
          if (ok && i >= 1) ok = mbar_wait(&bar.dv_done, (i - 1) & 1, status, 45);
          if (!ok) break;
          tc_fence_after();
          const int nu = bar.meta[s] & 15;  // written before the stage's Q arrived
          id = nu == 2 ? id_full : id_half;
          const uint64_t dQs = sdesc_sw128(smem_u32(smem + L::OFF_Q + s * L::TILE), 16, 1024);
          dDOs = sdesc_sw128(smem_u32(smem + L::OFF_DO + s * L::TILE), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tS, dKd + kslice16(kk, 128 * 128), dQs + kslice16(kk, 128 * 128), id, kk > 0 ? 1u : 0u);
          mma_commit(&bar.s_full);
        }
        if (i >= 1) {  // dK += dS^T(i-1) Q(i-1)
          ok = mbar_wait(&bar.ds_ready, (i - 1) & 1, status, 47);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dQmn = sdesc_sw128(smem_u32(smem + L::OFF_Q + sp * L::TILE), 128 * 128, 1024);
          for (int ks = 0; ks < 4 * nup; ++ks)
            mma_ts(tK, tP + pk_col(ks), dQmn + (uint64_t)ks * 128, id_acc, (i > 1 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.dk_done);
          mma_commit(&bar.q_empty[sp]);
        }
        if (i < nsteps) {  // dP^T(i) = V dO(i)^T, into the columns dK(i-1) read dS^T(i-1) from
          if (i >= 1) ok = mbar_wait(&bar.dk_done, (i - 1) & 1, status, 46);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tP, dVd + kslice16(kk, 128 * 128), dDOs + kslice16(kk, 128 * 128), id, kk > 0 ? 1u : 0u);
          mma_commit(&bar.dp_full);
        }
      }
      if (ok && nsteps > 0) mma_commit(&bar.fin);
      if (!ok) {
        bar.abort = 1;
        mma_drain(&bar.drain, status, 54);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ compute
    const int g = (warp - 4) >> 2;   // warpgroup: query unit g of every step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // key row of the tile
    const int half = row >> 6;       // warp-uniform
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % NS;
      ok = mbar_wait_warp(&bar.s_full, i & 1, status, 48);
      // the stage's statistics were written by the async proxy: observe the
      // stage's own barrier (already complete; the stage cannot be refilled
      // before this step releases it) so those writes are visible here
      if (ok) ok = mbar_wait_warp(&bar.q_full[s], (i / NS) & 1, status, 50);
      if (!ok) break;
      tc_fence_after();
      const int meta = bar.meta[s];
      const bool active = g < (meta & 15);
      const bool valid = active && (((meta >> (4 + 4 * g)) >> half) & 1);  // warp-uniform
      const float *st = stat + s * 256 + 64 * g;
      float pf[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        if (valid) {
          uint32_t sv[32];
          float nl[32];
          tmem_ld32(tS + lane_off + 64 * g + 32 * c, sv);
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 lq = reinterpret_cast<const float4 *>(st + 32 * c)[k4];
            nl[4 * k4] = -lq.x;
            nl[4 * k4 + 1] = -lq.y;
            nl[4 * k4 + 2] = -lq.z;
            nl[4 * k4 + 3] = -lq.w;
          }
          tmem_wait_ld();
          softmax_p32(sv, scale_log2, [&nl](int k) { return make_float2(nl[k], nl[k + 1]); }, pf + 32 * c);
#pragma unroll
          for (int k = 0; k < 32; k += 2) pk[k / 2] = pack_f16(pf[32 * c + k], pf[32 * c + k + 1]);
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        }
        if (active) tmem_st16(tS + lane_off + 64 * g + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_ready);
      ok = mbar_wait_warp(&bar.dp_full, i & 1, status, 49);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        if (valid) {
          uint32_t dv[32];
          tmem_ld32(tP + lane_off + 64 * g + 32 * c, dv);
          tmem_wait_ld();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 dq = reinterpret_cast<const float4 *>(st + 128 + 32 * c)[k4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int k = 4 * k4 + 2 * u;
              const float2 dd = u ? make_float2(dq.z, dq.w) : make_float2(dq.x, dq.y);
              const float2 d = fmul2(make_float2(pf[32 * c + k], pf[32 * c + k + 1]),
                                     fsub2(make_float2(__uint_as_float(dv[k]), __uint_as_float(dv[k + 1])), dd));
              pk[k / 2] = pack_f16(d.x, d.y);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        }
        if (active) tmem_st16(tP + lane_off + 64 * g + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.ds_ready);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nsteps > 0) ok = mbar_wait_warp(&bar.fin, 0, status, 51);
    if (ok) {
      tc_fence_after();
      const size_t prow = (size_t)h * N + (size_t)tile * 128 + row;
      int n = perm[prow];
      if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 128)) n = 0;
      const size_t off = ((size_t)n * heads + h) * D;
      // warpgroup 0 writes dV, warpgroup 1 writes dK
      const uint32_t src = g == 0 ? tV : tK;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (nsteps > 0) {
          tmem_ld32(src + lane_off + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        store_row<D>(g == 0 ? dV : dK, grad_fp32 != 0, off + c, o, g == 0 ? dv_scale : sm_scale);
      }
    } else {
      bar.abort = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}


// ---------------------------------------------------------------------------
// Fused dK/dV/dQ kernel (head_dim 128): the dK/dV kernel's walk over a
// 128-key tile's query units, plus dQ^T(i) = K^T dS^T(i) per step, added
// into an fp32 [heads][N][128] accumulator in permuted order by bulk
// reductions (cp.reduce.async.bulk .add.f32, performed at L2).  No S or dP
// is recomputed for dQ, so the backward issues 10 P D flops instead of the
// two-kernel path's 14 P D.  The order of the reductions is not fixed: dQ is
// not bitwise reproducible from run to run (dK and dV are; each CTA owns its
// key rows).
//   TMEM: dV [0, 128), dK [128, 256), S^T [256, 384) (P^T packed into it,
//   read by dV as a TS product), dP^T [384, 512), and dQ^T of the same step
//   in those columns once the compute warps have read dP^T.
//   Shared memory (FusedSmem; 1024-byte-aligned window, no slack): the K and
//   V tiles; a ring of two stages, each a Q tile (with its rows' lse) and a
//   dO tile (with their Delta), filled and released separately; dS^T (fp16,
//   128 keys x 128 queries, 128-byte swizzle), the K-major A operand of
//   dK += dS^T Q and the MN-major B operand of dQ^T = K^T dS^T, whose A is
//   the resident K tile read MN-major.
//   Per step the compute warps load dQ^T(i) from TMEM (freeing the columns
//   for dP^T(i+1)) and stage it as [64 queries][128] fp32 per unit:
//   warpgroup 0 into the stage's dO slot, warpgroup 1 into the dS^T buffer
//   (both free once dQ^T(i), the last product issued that reads them, is
//   done).  Warp 2 issues one 32 KB bulk reduction per unit (the unit's 64
//   accumulator rows are contiguous) and releases the two buffers when the
//   copies have read them, so the reductions run behind the next step.
//   MMA issue order of iteration i: dV(i-1), dK(i-1), dQ^T(i-1), S^T(i),
//   dP^T(i): dQ^T(i-1), which the compute warps wait for, goes ahead of
//   S^T(i), which they need only after staging it.
// ---------------------------------------------------------------------------
struct FusedSmem {
  static constexpr int TILE = 128 * 128 * 2;  // 128 rows of 128 fp16
  static constexpr int OFF_K = 0;
  static constexpr int OFF_V = OFF_K + TILE;
  static constexpr int OFF_Q = OFF_V + TILE;        // ring of query-unit pairs
  static constexpr int OFF_DO = OFF_Q + NS * TILE;  // ring of dO-unit pairs; warpgroup 0's dQ staging
  static constexpr int OFF_DS = OFF_DO + NS * TILE;  // dS^T; warpgroup 1's dQ staging
  static constexpr int OFF_STAT = OFF_DS + TILE;     // [NS][lse2 128, delta 128] floats
  static constexpr int OFF_BAR = OFF_STAT + NS * 256 * 4;
  static constexpr int BYTES = OFF_BAR + 256;
};

struct FusedBars {
  uint64_t kv_full;
  uint64_t q_full[NS], o_full[NS];      // Q + lse2, dO + Delta of a stage have arrived
  uint64_t q_empty[NS], o_empty[NS];    // the Q slot (after dK), the dO slot (after its staging was read)
  uint64_t s_full, dp_full, p_ready, ds_ready, dv_done, dq_full, dq_free;
  uint64_t staged[2];  // warpgroup g has staged its unit's dQ^T
  uint64_t ds_free;    // the dS^T buffer's staging has been read
  uint64_t fin;        // single use: every MMA of the tile has completed
  uint64_t drain;      // single use: the MMA thread's in-flight products after an abort
  int meta[NS];        // units | mask_a << 4 | mask_b << 8 (bit = 64-row half of the key tile)
  int unit[NS][2];     // the stage's query units
  // step i's unit count and units for the reducer, copied by warpgroup 0
  // (the producer may refill the stage's meta and unit before the reducer
  // is done with step i)
  int red_job[2][3];
  uint32_t tmem_base;
  int nsteps, nunits, abort;
};

__device__ __forceinline__ void bulk_reduce_add_f32(float *gdst, const void *ssrc, uint32_t bytes) {
  asm volatile("cp.reduce.async.bulk.global.shared::cta.bulk_group.add.f32 [%0], [%1], %2;" ::"l"(gdst),
               "r"(smem_u32(ssrc)), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void bulk_wait_read() {
  asm volatile("cp.async.bulk.wait_group.read %0;" ::"n"(N) : "memory");
}
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__global__ void __launch_bounds__(kThreads, 1)
    dkdvq_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapDO,
                 const __grid_constant__ CUtensorMap mapK, const __grid_constant__ CUtensorMap mapV,
                 const int32_t *__restrict__ col_ptr, const int32_t *__restrict__ rowidx,
                 const int32_t *__restrict__ blocks, const int32_t *__restrict__ unit_block,
                 const int32_t *__restrict__ tile_units, const int32_t *__restrict__ perm,
                 const float *__restrict__ lse2p, const float *__restrict__ deltap, float *__restrict__ dq_acc,
                 void *__restrict__ dK, void *__restrict__ dV, int grad_fp32, int N, int heads,
                 float scale_log2_in, float sm_scale_in, const unsigned *__restrict__ range_max, int *status) {
  constexpr int D = 128;
  using L = FusedSmem;
  static_assert(sizeof(FusedBars) <= L::BYTES - L::OFF_BAR, "barrier block");
  extern __shared__ __align__(1024) uint8_t smem[];
  // the layout fills the window: it needs the window 1024-byte aligned (as
  // the B200 places it) and has no slack to align it here
  if (smem_u32(smem) & 1023u) {
    if (threadIdx.x == 0) record_status(status, PRISM_ERR_UNSUPPORTED, 77);
    return;
  }
  FusedBars &bar = *reinterpret_cast<FusedBars *>(smem + L::OFF_BAR);
  float *stat = reinterpret_cast<float *>(smem + L::OFF_STAT);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x, h = blockIdx.y;
  const int NB = N / 64;
  const int32_t *blocks_h = blocks + (size_t)h * NB * 4;
  // operand pre-scales as in dkdv_kernel; dQ's 2^(edO + eV + eK) is applied
  // by the conversion pass
  const int eQ = range_exp(range_max[h], 0), eK = range_exp(range_max[heads + h], 1);
  const int eV = range_exp(range_max[2 * heads + h], 2), eO = range_exp(range_max[3 * heads + h], 3);
  const float scale_log2 = ldexpf(scale_log2_in, eQ + eK);
  const float sm_scale = ldexpf(sm_scale_in, eO + eV + eQ);
  const float dv_scale = ldexpf(1.0f, eO);

  if (threadIdx.x == 0) bar.abort = *reinterpret_cast<volatile int *>(status);
  __syncthreads();
  if (bar.abort) return;
  if (threadIdx.x == 0) {
    mbar_init(&bar.kv_full, 1);
    for (int s = 0; s < NS; ++s) {
      mbar_init(&bar.q_full[s], 1);
      mbar_init(&bar.o_full[s], 1);
      mbar_init(&bar.q_empty[s], 1);
      mbar_init(&bar.o_empty[s], 1);
    }
    mbar_init(&bar.s_full, 1);
    mbar_init(&bar.dp_full, 1);
    mbar_init(&bar.p_ready, 256);
    mbar_init(&bar.ds_ready, 256);
    mbar_init(&bar.dv_done, 1);
    mbar_init(&bar.dq_full, 1);
    mbar_init(&bar.dq_free, 256);
    mbar_init(&bar.staged[0], 128);
    mbar_init(&bar.staged[1], 128);
    mbar_init(&bar.ds_free, 1);
    mbar_init(&bar.fin, 1);
    mbar_init(&bar.drain, 1);
    bar.nunits = tile_units[(size_t)h * (N / 128) + tile];
    bar.nsteps = (bar.nunits + 1) >> 1;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;
  const int nsteps = bar.nsteps, nunits = bar.nunits;
  const uint32_t tV = tmem, tK = tmem + 128, tS = tmem + 256, tP = tmem + 384;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    const int blk[2] = {unit_block[(size_t)h * NB + 2 * tile], unit_block[(size_t)h * NB + 2 * tile + 1]};
    UnitWalk<2> w;
    walk_init<2>(w, blk, 2, col_ptr, h * NB);
    int q_issued = 0, o_issued = 0;
    if (lane == 0) {
      mbar_arrive_expect_tx(&bar.kv_full, 2 * L::TILE);
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        tma_load_2d(smem + L::OFF_K + c * (128 * 128), &mapK, &bar.kv_full, c * 64, h * N + tile * 128);
        tma_load_2d(smem + L::OFF_V + c * (128 * 128), &mapV, &bar.kv_full, c * 64, h * N + tile * 128);
      }
    }
    for (int j = 0; j < nsteps; ++j) {
      const int s = j % NS;
      uint32_t ua, ub = 0;
      int ma, mb = 0, nu = 1;
      walk_next<2>(w, rowidx, blocks_h, ua, ma);
      if (2 * j + 2 <= nunits) {
        walk_next<2>(w, rowidx, blocks_h, ub, mb);
        nu = 2;
      }
      PRISM_CHECK(ua < (uint32_t)NB && ub < (uint32_t)NB, status, 129);
      ua = min(ua, (uint32_t)(NB - 1));
      ub = min(ub, (uint32_t)(NB - 1));
      if (lane == 0) {
        bool ok = true;
        if (j >= NS) ok = mbar_wait(&bar.q_empty[s], ((j / NS) - 1) & 1, status, 61);
        if (ok) {
          bar.meta[s] = nu | (ma << 4) | (mb << 8);
          bar.unit[s][0] = (int)ua;
          bar.unit[s][1] = (int)ub;
          uint8_t *qs = smem + L::OFF_Q + s * L::TILE;
          float *st = stat + s * 256;
          mbar_arrive_expect_tx(&bar.q_full[s], nu * (64 * D * 2 + 64 * 4));
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(qs + c * (128 * 128), &mapQ, &bar.q_full[s], c * 64, h * N + (int)ua * 64);
            if (nu == 2)
              tma_load_2d(qs + c * (128 * 128) + 64 * 128, &mapQ, &bar.q_full[s], c * 64, h * N + (int)ub * 64);
          }
          bulk_load(st, lse2p + (size_t)h * N + (size_t)ua * 64, 256, &bar.q_full[s]);
          if (nu == 2) bulk_load(st + 64, lse2p + (size_t)h * N + (size_t)ub * 64, 256, &bar.q_full[s]);
          ++q_issued;
        }
        if (ok && j >= NS) ok = mbar_wait(&bar.o_empty[s], ((j / NS) - 1) & 1, status, 62);
        if (ok) {
          uint8_t *os = smem + L::OFF_DO + s * L::TILE;
          float *st = stat + s * 256;
          mbar_arrive_expect_tx(&bar.o_full[s], nu * (64 * D * 2 + 64 * 4));
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            tma_load_2d(os + c * (128 * 128), &mapDO, &bar.o_full[s], c * 64, h * N + (int)ua * 64);
            if (nu == 2)
              tma_load_2d(os + c * (128 * 128) + 64 * 128, &mapDO, &bar.o_full[s], c * 64, h * N + (int)ub * 64);
          }
          bulk_load(st + 128, deltap + (size_t)h * N + (size_t)ua * 64, 256, &bar.o_full[s]);
          if (nu == 2) bulk_load(st + 192, deltap + (size_t)h * N + (size_t)ub * 64, 256, &bar.o_full[s]);
          ++o_issued;
        }
        if (!ok) bar.abort = 1;
      }
      __syncwarp();
      if (*reinterpret_cast<volatile int *>(&bar.abort)) break;
    }
    if (lane == 0) {  // no copy may still be writing when the CTA leaves
      drain_loads(&bar.kv_full, 1, 1, status, 63);
      drain_loads(bar.q_full, NS, q_issued, status, 63);
      drain_loads(bar.o_full, NS, o_issued, status, 63);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t id_full = idesc_f16(128, 128, 0), id_half = idesc_f16(128, 64, 0);
      const uint32_t id_acc = idesc_f16(128, D, 1);
      const uint64_t dKd = sdesc_sw128(smem_u32(smem + L::OFF_K), 16, 1024);
      const uint64_t dVd = sdesc_sw128(smem_u32(smem + L::OFF_V), 16, 1024);
      const uint64_t dKmn = sdesc_sw128(smem_u32(smem + L::OFF_K), 128 * 128, 1024);  // K^T as an MN-major A
      const uint64_t dSmn = sdesc_sw128(smem_u32(smem + L::OFF_DS), 128 * 128, 1024);  // dS^T as an MN-major B
      const uint64_t dSk = sdesc_sw128(smem_u32(smem + L::OFF_DS), 16, 1024);          // dS^T as a K-major A
      bool ok = mbar_wait(&bar.kv_full, 0, status, 64);
      tc_fence_after();
      for (int i = 0; ok && i <= nsteps; ++i) {
        const int s = i % NS, sp = (i + NS - 1) % NS;
        const int nup = i >= 1 ? (bar.meta[sp] & 15) : 0;  // stage sp is not refilled before dK(i-1)
        if (i >= 1) {  // dV += P^T(i-1) dO(i-1)
          ok = mbar_wait(&bar.p_ready, (i - 1) & 1, status, 65);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dDOmn = sdesc_sw128(smem_u32(smem + L::OFF_DO + sp * L::TILE), 128 * 128, 1024);
          for (int ks = 0; ks < 4 * nup; ++ks)
            mma_ts(tV, tS + pk_col(ks), dDOmn + (uint64_t)ks * 128, id_acc, (i > 1 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.dv_done);
        }
        if (i >= 1) {  // dK += dS^T(i-1) Q(i-1); dQ^T(i-1) = K^T dS^T(i-1) into the dP^T columns
          ok = mbar_wait(&bar.ds_ready, (i - 1) & 1, status, 68);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dQmn = sdesc_sw128(smem_u32(smem + L::OFF_Q + sp * L::TILE), 128 * 128, 1024);
          for (int ks = 0; ks < 4 * nup; ++ks)
            mma_ss(tK, dSk + kslice16(ks, 128 * 128), dQmn + (uint64_t)ks * 128, id_acc, (i > 1 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.q_empty[sp]);
          const uint32_t id_q = idesc_f16_amn(128, 64 * nup, 1);
#pragma unroll
          for (int ks = 0; ks < 8; ++ks)
            mma_ss(tP, dKmn + (uint64_t)ks * 128, dSmn + (uint64_t)ks * 128, id_q, ks > 0 ? 1u : 0u);
          mma_commit(&bar.dq_full);  // also covers dK(i-1), issued before
        }
        uint32_t id = id_full;
        if (i < nsteps) {  // S^T(i) = K Q(i)^T, into the columns dV(i-1) read P^T(i-1) from
          ok = mbar_wait(&bar.q_full[s], (i / NS) & 1, status, 66);
          if (ok && i >= 1) ok = mbar_wait(&bar.dv_done, (i - 1) & 1, status, 67);
          if (!ok) break;
          tc_fence_after();
          const int nu = bar.meta[s] & 15;  // written before the stage's Q arrived
          id = nu == 2 ? id_full : id_half;
          const uint64_t dQs = sdesc_sw128(smem_u32(smem + L::OFF_Q + s * L::TILE), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tS, dKd + kslice16(kk, 128 * 128), dQs + kslice16(kk, 128 * 128), id, kk > 0 ? 1u : 0u);
          mma_commit(&bar.s_full);
        }
        if (i < nsteps) {  // dP^T(i) = V dO(i)^T, once the compute warps have read dQ^T(i-1)
          ok = mbar_wait(&bar.o_full[s], (i / NS) & 1, status, 69);
          if (ok && i >= 1) ok = mbar_wait(&bar.dq_free, (i - 1) & 1, status, 70);
          if (!ok) break;
          tc_fence_after();
          const uint64_t dDOs = sdesc_sw128(smem_u32(smem + L::OFF_DO + s * L::TILE), 16, 1024);
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk)
            mma_ss(tP, dVd + kslice16(kk, 128 * 128), dDOs + kslice16(kk, 128 * 128), id, kk > 0 ? 1u : 0u);
          mma_commit(&bar.dp_full);
        }
      }
      if (ok && nsteps > 0) mma_commit(&bar.fin);
      if (!ok) {
        bar.abort = 1;
        mma_drain(&bar.drain, status, 71);
      }
    }
    __syncwarp();
  } else if (warp == 2) {
    // ------------------------------------------------------------ dQ reducer
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; ok && i < nsteps; ++i) {
        const int s = i % NS;
        // the dS^T buffer first: the compute warps write the next dS^T into
        // it, while the dO slot is refilled only for step i + 2
        ok = mbar_wait(&bar.staged[1], i & 1, status, 82);
        if (ok) ok = mbar_wait(&bar.staged[0], i & 1, status, 81);
        if (!ok) break;
        const int *job = bar.red_job[i & 1];  // written before staged[0] (step i+2 rewrites it only
                                              // after this step's reductions have been read)
        const int nu = job[0];
        int ua = job[1], ub = job[2];
        if (!PRISM_CHECK((unsigned)ua < (unsigned)NB && (unsigned)ub < (unsigned)NB, status, 130)) ua = ub = 0;
        if (nu == 2)
          bulk_reduce_add_f32(dq_acc + ((size_t)h * N + (size_t)ub * 64) * D, smem + L::OFF_DS, 64 * D * 4);
        bulk_commit();
        bulk_reduce_add_f32(dq_acc + ((size_t)h * N + (size_t)ua * 64) * D, smem + L::OFF_DO + s * L::TILE,
                            64 * D * 4);
        bulk_commit();
        bulk_wait_read<1>();  // the dS^T buffer's staging has been read
        mbar_arrive(&bar.ds_free);
        bulk_wait_read<0>();  // and the dO slot's
        mbar_arrive(&bar.o_empty[s]);
      }
      if (!ok) bar.abort = 1;
      bulk_wait_all();  // every reduction has been performed before the CTA leaves
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ compute
    const int g = (warp - 4) >> 2;   // warpgroup: query unit g of every step
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;  // key row of the tile; the feature index d of dQ^T
    const int half = row >> 6;       // warp-uniform
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % NS;
      ok = mbar_wait_warp(&bar.s_full, i & 1, status, 72);
      // the stage's statistics were written by the async proxy: observe the
      // stage's own barriers (already complete) so those writes are visible
      if (ok) ok = mbar_wait_warp(&bar.q_full[s], (i / NS) & 1, status, 72);
      if (!ok) break;
      tc_fence_after();
      // the stage's meta and units, read before this step releases the stage
      const int meta = bar.meta[s], unit0 = bar.unit[s][0], unit1 = bar.unit[s][1];
      const bool active = g < (meta & 15);
      const bool valid = active && (((meta >> (4 + 4 * g)) >> half) & 1);  // warp-uniform
      const float *st = stat + s * 256 + 64 * g;
      float pf[64];
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        uint32_t pk[16];
        if (valid) {
          uint32_t sv[32];
          float nl[32];
          tmem_ld32(tS + lane_off + 64 * g + 32 * c, sv);
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 lq = reinterpret_cast<const float4 *>(st + 32 * c)[k4];
            nl[4 * k4] = -lq.x;
            nl[4 * k4 + 1] = -lq.y;
            nl[4 * k4 + 2] = -lq.z;
            nl[4 * k4 + 3] = -lq.w;
          }
          tmem_wait_ld();
          softmax_p32(sv, scale_log2, [&nl](int k) { return make_float2(nl[k], nl[k + 1]); }, pf + 32 * c);
#pragma unroll
          for (int k = 0; k < 32; k += 2) pk[k / 2] = pack_f16(pf[32 * c + k], pf[32 * c + k + 1]);
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) pk[k] = 0u;
        }
        if (active) tmem_st16(tS + lane_off + 64 * g + 16 * c, pk);
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_ready);
      ok = mbar_wait_warp(&bar.dp_full, i & 1, status, 73);
      if (ok) ok = mbar_wait_warp(&bar.o_full[s], (i / NS) & 1, status, 73);
      if (!ok) break;
      tc_fence_after();
      uint32_t ds[32];  // dS^T of this row and unit, fp16 pairs
#pragma unroll
      for (int c = 0; c < 2; ++c) {
        if (valid) {
          uint32_t dv[32];
          tmem_ld32(tP + lane_off + 64 * g + 32 * c, dv);
          tmem_wait_ld();
#pragma unroll
          for (int k4 = 0; k4 < 8; ++k4) {
            const float4 dq = reinterpret_cast<const float4 *>(st + 128 + 32 * c)[k4];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              const int k = 4 * k4 + 2 * u;
              const float2 dd = u ? make_float2(dq.z, dq.w) : make_float2(dq.x, dq.y);
              const float2 d = fmul2(make_float2(pf[32 * c + k], pf[32 * c + k + 1]),
                                     fsub2(make_float2(__uint_as_float(dv[k]), __uint_as_float(dv[k + 1])), dd));
              ds[16 * c + k / 2] = pack_f16(d.x, d.y);
            }
          }
        } else {
#pragma unroll
          for (int k = 0; k < 16; ++k) ds[16 * c + k] = 0u;
        }
      }
      // the dS^T buffer held the previous step's staging until its reduction read it
      if (i >= 1) ok = mbar_wait_warp(&bar.ds_free, (i - 1) & 1, status, 74);
      if (!ok) break;
      if (active) {
        uint8_t *rowp = smem + L::OFF_DS + g * (128 * 128) + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j)
          *reinterpret_cast<uint4 *>(rowp + ((j ^ (row & 7)) << 4)) =
              make_uint4(ds[4 * j], ds[4 * j + 1], ds[4 * j + 2], ds[4 * j + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      mbar_arrive(&bar.ds_ready);
      // dQ^T(i): TMEM lane = feature d, column = query of unit g.  Once it is
      // done (and with it every product issued before: dV(i), dP^T(i) and
      // dK(i), the last readers of the dO slot and of the dS^T buffer), it
      // is staged as [64 queries][128] fp32, warpgroup 0 into the stage's
      // dO slot, warpgroup 1 into the dS^T buffer.  Then dP^T(i+1) may take
      // the columns.
      ok = mbar_wait_warp(&bar.dq_full, i & 1, status, 75);
      if (!ok) break;
      tc_fence_after();
      if (active) {
        float *stg = reinterpret_cast<float *>(smem + (g == 0 ? L::OFF_DO + s * L::TILE : L::OFF_DS));
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          uint32_t qv[32];
          tmem_ld32(tP + lane_off + 64 * g + 32 * c, qv);
          tmem_wait_ld();
#pragma unroll
          for (int k = 0; k < 32; ++k) stg[(32 * c + k) * D + row] = __uint_as_float(qv[k]);
        }
      }
      tc_fence_before();
      mbar_arrive(&bar.dq_free);
      if (g == 0 && q4 == 0 && lane == 0) {
        bar.red_job[i & 1][0] = meta & 15;
        bar.red_job[i & 1][1] = unit0;
        bar.red_job[i & 1][2] = unit1;
      }
      fence_async_smem();
      mbar_arrive(&bar.staged[g]);
    }
    ok = __all_sync(0xffffffffu, ok);
    if (ok && nsteps > 0) ok = mbar_wait_warp(&bar.fin, 0, status, 78);
    if (ok) {
      tc_fence_after();
      const size_t prow = (size_t)h * N + (size_t)tile * 128 + row;
      int n = perm[prow];
      if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 131)) n = 0;
      const size_t off = ((size_t)n * heads + h) * D;
      // warpgroup 0 writes dV, warpgroup 1 writes dK
      const uint32_t src = g == 0 ? tV : tK;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (nsteps > 0) {
          tmem_ld32(src + lane_off + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int k = 0; k < 32; ++k) o[k] = 0u;
        }
        store_row<D>(g == 0 ? dV : dK, grad_fp32 != 0, off + c, o, g == 0 ? dv_scale : sm_scale);
      }
    } else {
      bar.abort = 1;
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

// dQ[n][h][:] = 2^(edO + eV + eK) * scale * dq_acc[h][p][:] for n = perm[h][p]:
// the fused kernel's fp32 accumulator in natural order, bf16 or fp32.
template <int D>
__global__ void __launch_bounds__(256) dq_convert_kernel(const int32_t *__restrict__ perm, int N, int heads,
                                                         const float *__restrict__ acc, void *__restrict__ dQ,
                                                         int grad_fp32, float sm_scale_in,
                                                         const unsigned *__restrict__ range_max, int *status) {
  constexpr int G = D / 8;  // 8-feature vectors per row
  const size_t total = (size_t)heads * N * G;
  for (size_t q = (size_t)blockIdx.x * blockDim.x + threadIdx.x; q < total; q += (size_t)gridDim.x * blockDim.x) {
    const size_t r = q / G;
    const int v = (int)(q % G);
    const int h = (int)(r / N);
    const float mul = ldexpf(sm_scale_in, range_exp(range_max[3 * heads + h], 3) +
                                              range_exp(range_max[2 * heads + h], 2) +
                                              range_exp(range_max[heads + h], 1));
    int n = perm[r];
    if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 132)) n = 0;
    const float4 a = __ldg(reinterpret_cast<const float4 *>(acc + r * D + v * 8));
    const float4 b = __ldg(reinterpret_cast<const float4 *>(acc + r * D + v * 8 + 4));
    const size_t off = ((size_t)n * heads + h) * D + v * 8;
    if (grad_fp32) {
      float4 *dst = reinterpret_cast<float4 *>(static_cast<float *>(dQ) + off);
      dst[0] = make_float4(a.x * mul, a.y * mul, a.z * mul, a.w * mul);
      dst[1] = make_float4(b.x * mul, b.y * mul, b.z * mul, b.w * mul);
    } else {
      *reinterpret_cast<uint4 *>(static_cast<uint16_t *>(dQ) + off) =
          make_uint4(pack_bf16(a.x * mul, a.y * mul), pack_bf16(a.z * mul, a.w * mul), pack_bf16(b.x * mul, b.y * mul),
                     pack_bf16(b.z * mul, b.w * mul));
    }
  }
}

}  // namespace bwd

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct BwdWs {
  WsHeader *hdr;
  uint16_t *Qp, *Kp, *Vp, *dOp;
  float *lse2p, *deltap;
  int32_t *unit_block, *tu_q, *tu_k;
  int32_t *range_flag;   // [4][heads]
  unsigned *range_max;   // [4][heads]
  float *dq_acc;         // [heads][N][128] fp32, permuted rows (fused path; head_dim 128 only)
};
static BwdWs carve_bwd(const prism_params &p, void *ws) {
  const size_t N = (size_t)p.T * p.H * p.W, h = p.heads, D = p.head_dim;
  const size_t tens = align_up(sizeof(uint16_t) * h * N * D, 256);
  char *w = static_cast<char *>(ws);
  BwdWs b;
  b.hdr = reinterpret_cast<WsHeader *>(w);
  w += kWsHeader;
  b.Qp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  b.Kp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  b.Vp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  b.dOp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  b.lse2p = reinterpret_cast<float *>(w);
  w += align_up(sizeof(float) * h * N, 256);
  b.deltap = reinterpret_cast<float *>(w);
  w += align_up(sizeof(float) * h * N, 256);
  b.unit_block = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * (N / 64), 256);
  b.tu_q = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * (N / 128), 256);
  b.tu_k = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * (N / 128), 256);
  b.range_flag = reinterpret_cast<int32_t *>(w);
  b.range_max = reinterpret_cast<unsigned *>(w + sizeof(int32_t) * 4 * h);
  w += align_up(sizeof(int32_t) * 8 * h, 256);
  b.dq_acc = D == 128 ? reinterpret_cast<float *>(w) : nullptr;
  return b;
}

size_t attn_bwd_ws_bytes(const prism_params &p) {
  const size_t N = (size_t)p.T * p.H * p.W, h = p.heads, D = p.head_dim;
  return kWsHeader + 4 * align_up(sizeof(uint16_t) * h * N * D, 256) + 2 * align_up(sizeof(float) * h * N, 256) +
         align_up(sizeof(int32_t) * h * (N / 64), 256) + 2 * align_up(sizeof(int32_t) * h * (N / 128), 256) +
         align_up(sizeof(int32_t) * 8 * h, 256) + (D == 128 ? align_up(sizeof(float) * h * N * D, 256) : 0);
}

template <int D>
static cudaError_t run_bwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                           const BwdWs &w, void *dQ, void *dK, void *dV, int grad_fp32, cudaStream_t st) {
  const int N = p.T * p.H * p.W;
  const long long rows = (long long)p.heads * N;
  CUtensorMap mK64, mV64, mQ64, mDO64, mK128, mV128;  // box rows 128 or 64
  cudaError_t e;
  if ((e = make_rows_map(&mK64, w.Kp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mV64, w.Vp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mQ64, w.Qp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mDO64, w.dOp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mK128, w.Kp, rows, D, 128)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mV128, w.Vp, rows, D, 128)) != cudaSuccess) return e;
  const float scale = effective_scale(p);
  const float scale_log2 = scale * bwd::kLog2e;
  dim3 grid(N / 128, p.heads);
  const int s1 = bwd::KvSmem<D>::BYTES + 1024;
  cudaFuncSetAttribute(bwd::dkdv_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
  {
  KernelTimer kt_(KT_ATTN_DKDV, st);
  bwd::dkdv_kernel<D><<<grid, bwd::kThreads, s1, st>>>(mQ64, mDO64, mK128, mV128, sel.col_ptr, sel.row, plan.blocks,
                                                       w.unit_block, w.tu_k, plan.perm, w.lse2p, w.deltap, dK, dV,
                                                       grad_fp32, N, p.heads, scale_log2, scale, w.range_max,
                                                       &w.hdr->status);
  }
  const int s2 = bwd::DqSmem<D>::BYTES + 1024;
  cudaFuncSetAttribute(bwd::dq_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, s2);
  {
  KernelTimer kt_(KT_ATTN_DQ, st);
  bwd::dq_kernel<D><<<grid, bwd::kThreads, s2, st>>>(mK64, mV64, w.Qp, w.dOp, sel.row_ptr, sel.col, plan.blocks,
                                                     w.unit_block, w.tu_q, plan.perm, w.lse2p, w.deltap, dQ,
                                                     grad_fp32, N, p.heads, scale_log2, scale, w.range_max,
                                                     &w.hdr->status);
  }
  count_launches(2);
  return cudaGetLastError();
}

static cudaError_t run_bwd_fused(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                                 const BwdWs &w, void *dQ, void *dK, void *dV, int grad_fp32, cudaStream_t st) {
  constexpr int D = 128;
  const int N = p.T * p.H * p.W;
  const long long rows = (long long)p.heads * N;
  CUtensorMap mQ64, mDO64, mK128, mV128;
  cudaError_t e;
  if ((e = make_rows_map(&mQ64, w.Qp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mDO64, w.dOp, rows, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mK128, w.Kp, rows, D, 128)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mV128, w.Vp, rows, D, 128)) != cudaSuccess) return e;
  const float scale = effective_scale(p);
  const float scale_log2 = scale * bwd::kLog2e;
  dim3 grid(N / 128, p.heads);
  const int s1 = bwd::FusedSmem::BYTES;  // exactly the layout: the window's base is 1024-byte aligned
  cudaFuncSetAttribute(bwd::dkdvq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, s1);
  {
    KernelTimer kt_(KT_ATTN_BWD_FUSED, st);
    bwd::dkdvq_kernel<<<grid, bwd::kThreads, s1, st>>>(mQ64, mDO64, mK128, mV128, sel.col_ptr, sel.row, plan.blocks,
                                                        w.unit_block, w.tu_k, plan.perm, w.lse2p, w.deltap, w.dq_acc,
                                                        dK, dV, grad_fp32, N, p.heads, scale_log2, scale,
                                                        w.range_max, &w.hdr->status);
  }
  {
    KernelTimer kt_(KT_DQ_CONVERT, st);
    bwd::dq_convert_kernel<D><<<148 * 8, 256, 0, st>>>(plan.perm, N, p.heads, w.dq_acc, dQ, grad_fp32, scale,
                                                       w.range_max, &w.hdr->status);
  }
  count_launches(2);
  return cudaGetLastError();
}

cudaError_t launch_attn_bwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                            const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *O,
                            const uint16_t *O_res, const uint16_t *dO, const float *lse, void *dQ, void *dK,
                            void *dV, int grad_fp32, int deterministic, void *ws, cudaStream_t st) {
  const int N = p.T * p.H * p.W, NB = N / 64, D = p.head_dim;
  BwdWs w = carve_bwd(p, ws);
  const bool fused = D == 128 && !deterministic;
  cudaError_t e;
  if ((e = cudaMemsetAsync(w.range_flag, 0, sizeof(int32_t) * 8 * p.heads, st)) != cudaSuccess) return e;
  if ((e = launch_permute3(plan.perm, N, p.heads, D, Q, K, V, w.Qp, w.Kp, w.Vp, w.range_flag, &w.hdr->status,
                           st)) != cudaSuccess)
    return e;
  const size_t total = (size_t)p.heads * N * (D / 8);
  {
  KernelTimer kt_(KT_BWD_PREP, st);
  if (D == 128)
    bwd::bwd_prep_kernel<128><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(plan.perm, N, p.heads, dO, O, O_res, lse,
                                                                              w.dOp, w.lse2p, w.deltap,
                                                                              w.range_flag + 3 * p.heads,
                                                                              fused ? w.dq_acc : nullptr);
  else
    bwd::bwd_prep_kernel<64><<<(unsigned)((total + 255) / 256), 256, 0, st>>>(plan.perm, N, p.heads, dO, O, O_res, lse,
                                                                             w.dOp, w.lse2p, w.deltap,
                                                                             w.range_flag + 3 * p.heads, nullptr);
  }
  count_launches(1);
  if ((e = launch_range_fix(plan.perm, N, p.heads, D, RangeSrc{{Q, K, V, dO}}, RangeDst{{w.Qp, w.Kp, w.Vp, w.dOp}},
                            w.range_flag, w.range_max, w.deltap, &w.hdr->status, st)) != cudaSuccess)
    return e;
  if ((e = launch_unit_block(plan.blocks, plan.n_blocks, NB, p.heads, w.unit_block, st)) != cudaSuccess) return e;
  if ((e = launch_tile_units(sel.row_ptr, sel.col, plan.blocks, w.unit_block, N, p.heads, 2, w.tu_q, st)) !=
      cudaSuccess)
    return e;
  if ((e = launch_tile_units(sel.col_ptr, sel.row, plan.blocks, w.unit_block, N, p.heads, 2, w.tu_k, st)) !=
      cudaSuccess)
    return e;
  if (fused) return run_bwd_fused(p, plan, sel, w, dQ, dK, dV, grad_fp32, st);
  return D == 128 ? run_bwd<128>(p, plan, sel, w, dQ, dK, dV, grad_fp32, st)
                  : run_bwd<64>(p, plan, sel, w, dQ, dK, dV, grad_fp32, st);
}

}  // namespace prism
