// prism_attn_fwd: exact attention of each query over the tokens of its
// selected key blocks, on tcgen05 tensor cores with TMEM accumulators.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// section on hybrid block selection (exact attention with the full query
// tokens and the selected key/value blocks, online softmax, no full attention
// matrix; the output goes back to the original order) and the training
// section (the kernel walks blocks of any volume in 64-token units).
//
// Work unit: one CTA per 256 permuted query positions of one head (grid
// N/256 x heads): four 64-token query units, two 128-row tiles.  The CTA walks
// the merged selections of the (up to four) distinct blocks of its units once,
// in ascending 64-token key units; every key tile feeds both query tiles, and
// each key unit carries a mask of the 64-row quarters whose block selected it
// (the rows of other quarters give it weight 0).  Keys are streamed as tiles
// of two 64-token units (any two units of the walk).
//
// Roles (384 threads, two 128-row query tiles t = 0, 1 per CTA):
//   warp 0      TMA producer: Q once, then per key tile j the K tile j and
//               the V tile j-1 into two 2-stage rings (K runs one ahead).
//   warp 1      allocates TMEM; lane 0 issues tcgen05.mma:
//                 S_t = Q_t K^T  (SS, fp32 in TMEM)
//                 O_t += P_t V   (TS: P_t is read from TMEM where S_t was)
//               in the order PV_0(j), S_0(j+1), PV_1(j), S_1(j+1): each
//               tile's next S waits only for its own PV, so the softmax of
//               one tile runs while the tensor pipe works for the other.
//   warps 4-11  two softmax warpgroups (tile t = warpgroup), one thread per
//               query row: reads S_t, online max with lazy rescaling of O_t
//               (only when the max grows by more than 2^8), writes P_t as
//               fp16 into TMEM, and finally normalises O_t and scatters it
//               to natural token order.
#include "attn_walk.cuh"

namespace prism {

namespace fwd {
using namespace attn;

constexpr int BQ = 256;          // query rows per CTA: two 128-row tiles
constexpr int NSTAGE = 2;        // K/V ring depth
constexpr int kThreads = 384;    // 12 warps
constexpr uint32_t kTmemCols = 512;
constexpr float kRescaleLog2 = 8.0f;  // lazy-rescale threshold (factor 256)
constexpr int kPolyPairs = 0;         // of every 16 column pairs, this many take exp2_poly2 (none: measured slower here)

template <int D>
struct Smem {
  static constexpr int CHUNKS = D / 64;                     // 128-byte swizzle chunks per row
  static constexpr int TILE = 128 * D * 2;                  // 128 rows of fp16
  static constexpr int OFF_Q = 0;                           // two query tiles
  static constexpr int OFF_K = OFF_Q + 2 * TILE;
  static constexpr int OFF_V = OFF_K + NSTAGE * TILE;
  static constexpr int OFF_BAR = OFF_V + NSTAGE * TILE;
  static constexpr int BYTES = OFF_BAR + 256;
};

constexpr int NMETA = 4;  // ring of per-key-tile descriptors

struct Bars {
  uint64_t q_full;
  uint64_t k_full[NSTAGE], k_empty[NSTAGE];
  uint64_t v_full[NSTAGE], v_empty[NSTAGE];
  uint64_t s_full[2];   // per query tile
  uint64_t p_full[2];
  uint64_t pv_done[2];
  uint64_t drain;  // single use: the MMA thread's in-flight products after an abort
  // per key tile j, slot j % NMETA: units | maskA << 4 | maskB << 8 (masks:
  // bit = 64-row quarter).  Written with K(j); slot j is rewritten for tile
  // j + 4 only after both softmax warpgroups have finished tile j.
  int meta[NMETA];
  uint32_t tmem_base;
  int ntiles;
  int nunits;
  int abort;
};

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    attn_fwd_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                    const __grid_constant__ CUtensorMap mapV, const int32_t *__restrict__ row_ptr,
                    const int32_t *__restrict__ col, const int32_t *__restrict__ blocks,
                    const int32_t *__restrict__ unit_block, const int32_t *__restrict__ tile_units,
                    const int32_t *__restrict__ perm, uint16_t *__restrict__ O, uint16_t *__restrict__ O_res,
                    float *__restrict__ lse, int N, int heads, float scale_log2_in,
                    const unsigned *__restrict__ range_max, int *status) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars &bar = *reinterpret_cast<Bars *>(smem + L::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int quad = blockIdx.x, h = blockIdx.y;
  const int NB = N / 64;
  const int32_t *blocks_h = blocks + (size_t)h * NB * 4;
  // operands pre-scaled by 2^-e (range.cu): Q and K fold into the score
  // scale, V into the output; e = 0 (no change at all) for in-range heads
  const float scale_log2 = ldexpf(scale_log2_in, range_exp(range_max[h], 0) + range_exp(range_max[heads + h], 1));
  const float out_scale = ldexpf(1.0f, range_exp(range_max[2 * heads + h], 2));

  // a CTA that starts after another one gave up does no work
  if (threadIdx.x == 0) bar.abort = *reinterpret_cast<volatile int *>(status);
  __syncthreads();
  if (bar.abort) return;

  if (threadIdx.x == 0) {
    mbar_init(&bar.q_full, 1);
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&bar.k_full[s], 1);
      mbar_init(&bar.k_empty[s], 1);
      mbar_init(&bar.v_full[s], 1);
      mbar_init(&bar.v_empty[s], 1);
    }
    for (int t = 0; t < 2; ++t) {
      mbar_init(&bar.s_full[t], 1);
      mbar_init(&bar.p_full[t], 128);
      mbar_init(&bar.pv_done[t], 1);
    }
    mbar_init(&bar.drain, 1);
    bar.nunits = tile_units[(size_t)h * (N / BQ) + quad];
    bar.ntiles = (bar.nunits + 1) >> 1;
    bar.abort = 0;
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
  const int ntiles = bar.ntiles;
  const int nunits = bar.nunits;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    int blk[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) blk[q] = unit_block[(size_t)h * NB + 4 * quad + q];
    UnitWalk<4> w;
    walk_init<4>(w, blk, 4, row_ptr, h * NB);
    if (lane == 0) {
      prefetch_tensormap(&mapQ);
      prefetch_tensormap(&mapK);
      prefetch_tensormap(&mapV);
      mbar_arrive_expect_tx(&bar.q_full, 2 * L::TILE);
#pragma unroll
      for (int t = 0; t < 2; ++t)
#pragma unroll
        for (int c = 0; c < L::CHUNKS; ++c)
          tma_load_2d(smem + L::OFF_Q + t * L::TILE + c * (128 * 128), &mapQ, &bar.q_full, c * 64,
                      h * N + quad * BQ + t * 128);
    }
    // iteration j loads K(j) and V(j-1): the next S needs K one tile before
    // the PV that needs V
    uint32_t pa = 0, pb = 0;  // units of tile j-1, for its V
    int pnu = 0;
    int k_issued = 0, v_issued = 0;
    for (int j = 0; j <= ntiles; ++j) {
      uint32_t ua = 0, ub = 0;
      int ma = 0, mb = 0, nu = 1;
      if (j < ntiles) {
        walk_next<4>(w, col, blocks_h, ua, ma);
        if (2 * j + 2 <= nunits) {
          walk_next<4>(w, col, blocks_h, ub, mb);
          nu = 2;
        }
        PRISM_CHECK(ua < (uint32_t)NB && ub < (uint32_t)NB, status, 123);
        ua = min(ua, (uint32_t)(NB - 1));  // a well-formed walk never clamps
        ub = min(ub, (uint32_t)(NB - 1));
      }
      if (lane == 0) {
        bool ok = true;
        if (j < ntiles) {
          const int s = j % NSTAGE;
          if (j >= NSTAGE) ok = mbar_wait(&bar.k_empty[s], ((j / NSTAGE) - 1) & 1, status, 1);
          if (ok) {
            bar.meta[j % NMETA] = nu | (ma << 4) | (mb << 8);
            uint8_t *ks = smem + L::OFF_K + s * L::TILE;
            mbar_arrive_expect_tx(&bar.k_full[s], nu * 64 * D * 2);
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c) {
              tma_load_2d(ks + c * (128 * 128), &mapK, &bar.k_full[s], c * 64, h * N + (int)ua * 64);
              if (nu == 2)
                tma_load_2d(ks + c * (128 * 128) + 64 * 128, &mapK, &bar.k_full[s], c * 64, h * N + (int)ub * 64);
            }
            ++k_issued;
          }
        }
        if (ok && j >= 1) {
          const int jv = j - 1, s = jv % NSTAGE;
          if (jv >= NSTAGE) ok = mbar_wait(&bar.v_empty[s], ((jv / NSTAGE) - 1) & 1, status, 10);
          if (ok) {
            uint8_t *vs = smem + L::OFF_V + s * L::TILE;
            mbar_arrive_expect_tx(&bar.v_full[s], pnu * 64 * D * 2);
#pragma unroll
            for (int c = 0; c < L::CHUNKS; ++c) {
              tma_load_2d(vs + c * (128 * 128), &mapV, &bar.v_full[s], c * 64, h * N + (int)pa * 64);
              if (pnu == 2)
                tma_load_2d(vs + c * (128 * 128) + 64 * 128, &mapV, &bar.v_full[s], c * 64, h * N + (int)pb * 64);
            }
            ++v_issued;
          }
        }
        if (!ok) bar.abort = 1;
      }
      pa = ua;
      pb = ub;
      pnu = nu;
      __syncwarp();
      if (*reinterpret_cast<volatile int *>(&bar.abort)) break;
    }
    if (lane == 0) {  // no copy may still be writing when the CTA leaves
      drain_loads(bar.k_full, NSTAGE, k_issued, status, 11);
      drain_loads(bar.v_full, NSTAGE, v_issued, status, 12);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc_s_full = idesc_f16(128, 128, 0);
      const uint32_t idesc_s_half = idesc_f16(128, 64, 0);
      const uint32_t idesc_o = idesc_f16(128, D, 1);
      const uint64_t dQ0 = sdesc_sw128(smem_u32(smem + L::OFF_Q), 16, 1024);
      const uint64_t dQ1 = sdesc_sw128(smem_u32(smem + L::OFF_Q + L::TILE), 16, 1024);
      // S_t(jj) = Q_t K(jj)^T into S_t's columns; K(jj) is in stage jj % NSTAGE
      auto issue_s = [&](int t, int jj) {
        const int nu = bar.meta[jj % NMETA] & 15;
        const uint32_t idesc_s = nu == 2 ? idesc_s_full : idesc_s_half;
        const uint64_t dK = sdesc_sw128(smem_u32(smem + L::OFF_K + (jj % NSTAGE) * L::TILE), 16, 1024);
        const uint64_t dQt = t ? dQ1 : dQ0;
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk)
          mma_ss(tmem + 128 * t, dQt + kslice16(kk, 128 * 128), dK + kslice16(kk, 128 * 128), idesc_s,
                 kk > 0 ? 1u : 0u);
        mma_commit(&bar.s_full[t]);
      };
      bool ok = mbar_wait(&bar.q_full, 0, status, 2);
      if (ok && ntiles > 0) ok = mbar_wait(&bar.k_full[0], 0, status, 3);
      if (ok && ntiles > 0) {
        tc_fence_after();
        issue_s(0, 0);
        issue_s(1, 0);
        mma_commit(&bar.k_empty[0]);
      }
      for (int j = 0; ok && j < ntiles; ++j) {
        const int sv = j % NSTAGE;
        const int nu = bar.meta[j % NMETA] & 15;
        const bool next = j + 1 < ntiles;
        ok = mbar_wait(&bar.v_full[sv], (j / NSTAGE) & 1, status, 6);
        if (ok && next) ok = mbar_wait(&bar.k_full[(j + 1) % NSTAGE], ((j + 1) / NSTAGE) & 1, status, 3);
        if (!ok) break;
        const uint64_t dV = sdesc_sw128(smem_u32(smem + L::OFF_V + sv * L::TILE), 128 * 128, 1024);
        for (int t = 0; ok && t < 2; ++t) {
          ok = mbar_wait(&bar.p_full[t], j & 1, status, 5);
          if (!ok) break;
          tc_fence_after();
          const uint32_t tOt = tmem + 256 + t * D, tPt = tmem + 128 * t;
          for (int ks = 0; ks < nu * 4; ++ks)
            mma_ts(tOt, tPt + ks * 8, dV + (uint64_t)ks * 128, idesc_o, (j > 0 || ks > 0) ? 1u : 0u);
          mma_commit(&bar.pv_done[t]);
          if (t == 1) mma_commit(&bar.v_empty[sv]);
          if (next) {
            // S_t(j+1) overwrites the columns PV_t(j) reads P_t from
            ok = mbar_wait(&bar.pv_done[t], j & 1, status, 4);
            if (!ok) break;
            tc_fence_after();
            issue_s(t, j + 1);
            if (t == 1) mma_commit(&bar.k_empty[(j + 1) % NSTAGE]);
          }
        }
      }
      if (!ok) {
        bar.abort = 1;
        mma_drain(&bar.drain, status, 13);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ softmax
    const int t = (warp - 4) >> 2;  // query tile of this warpgroup
    const int q4 = warp & 3;
    const int row = q4 * 32 + lane;
    const int qbit = 2 * t + (row >> 6);  // 64-row quarter of the CTA (warp-uniform)
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    const uint32_t tS = tmem + 128 * t, tO = tmem + 256 + t * D;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    for (int j = 0; j < ntiles; ++j) {
      ok = mbar_wait_warp(&bar.s_full[t], j & 1, status, 7);
      if (!ok) break;
      tc_fence_after();
      const int meta = bar.meta[j % NMETA];
      const int nu = meta & 15;
      const bool v0 = ((meta >> 4) >> qbit) & 1;
      const bool v1 = nu == 2 && (((meta >> 8) >> qbit) & 1);
      // Fast path (after the first valid tile): P against the running maximum
      // in one pass over S, kept packed in registers; it is stored only if no
      // P reached 2^8, i.e. no row's maximum grew past the lazy threshold.
      bool done = false;
      if (__all_sync(0xffffffffu, m > -INFINITY)) {
        uint32_t pk[64];
        float2 ls2 = make_float2(0.f, 0.f);
        uint32_t pmax = 0u;
        // 32-column chunks of S; chunk c+1 loads while chunk c is computed
        const bool cv[4] = {v0, v0, nu == 2 && v1, nu == 2 && v1};  // warp-uniform
        uint32_t rr[2][32];
        if (cv[0]) tmem_ld32(tS + lane_off, rr[0]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          uint32_t(&r)[32] = rr[c & 1];
          if (cv[c]) tmem_wait_ld_r(r);
          if (c + 1 < 4 && cv[c + 1]) tmem_ld32(tS + lane_off + (c + 1) * 32, rr[(c + 1) & 1]);
          if (cv[c]) {
#pragma unroll
            for (int i = 0; i < 32; i += 2) {
              const float2 x = ffma2(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), scale_log2, -m);
              // a share of the exponentials on the FMA pipe, the rest on MUFU
              const float2 p = i < 2 * kPolyPairs ? exp2_poly2(x) : make_float2(ex2f(x.x), ex2f(x.y));
              ls2 = fadd2(ls2, p);
              const uint32_t h2 = pack_f16(p.x, p.y);
              pmax = hmax2u(pmax, h2);
              pk[c * 16 + i / 2] = h2;
            }
          } else {
#pragma unroll
            for (int i = 0; i < 16; ++i) pk[c * 16 + i] = 0u;
          }
        }
        // P >= 0, so fp16 bit patterns order like values; 0x5C00 is 256.0
        const bool over = (pmax & 0xffffu) >= 0x5C00u || (pmax >> 16) >= 0x5C00u;
        if (!__any_sync(0xffffffffu, over)) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            if (c < 2 * nu) tmem_st16(tS + lane_off + c * 16, &pk[c * 16]);
          l += ls2.x + ls2.y;
          done = true;
        }
      }
      if (!done) {
      // slow path, pass 1: maximum over the valid columns of this row
      float mt = -INFINITY;
      for (int c = 0; c < 2 * nu; ++c) {
        if (!((c < 2) ? v0 : v1)) continue;  // warp-uniform
        uint32_t r[32];
        tmem_ld32(tS + lane_off + c * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; i += 2) mt = fmax3f(mt, __uint_as_float(r[i]), __uint_as_float(r[i + 1]));
      }
      mt *= scale_log2;
      // A row takes a new reference maximum only when it grows by more than
      // 2^8 (or on its first valid key).  The decision to touch O is made per
      // warp, because tcgen05.ld/st are warp-collective; rows that keep their
      // maximum use alpha = 1.
      const bool want = mt > m + kRescaleLog2 || (m == -INFINITY && mt > -INFINITY);
      if (__any_sync(0xffffffffu, want)) {
        const float m_new = want ? mt : m;
        const float alpha = (m == -INFINITY) ? 0.f : ex2f(m - m_new);
        if (j > 0 && __any_sync(0xffffffffu, want && m != -INFINITY)) {
          ok = mbar_wait_warp(&bar.pv_done[t], (j - 1) & 1, status, 8);
          if (!ok) break;
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < D; c += 32) {
            uint32_t o[32];
            tmem_ld32(tO + lane_off + c, o);
            tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(tO + lane_off + c, o);
          }
          tmem_wait_st();
        }
        l *= alpha;
        m = m_new;
      }
      // slow path, pass 2: P = exp2(s * scale_log2 - m) in fp16, two keys per column
      float2 ls = make_float2(0.f, 0.f);
      for (int c = 0; c < 2 * nu; ++c) {
        uint32_t pk[16];
        if ((c < 2) ? v0 : v1) {
          uint32_t r[32];
          tmem_ld32(tS + lane_off + c * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; i += 2) {
            float2 x = ffma2(make_float2(__uint_as_float(r[i]), __uint_as_float(r[i + 1])), scale_log2, -m);
            float2 p = make_float2(ex2f(x.x), ex2f(x.y));
            ls = fadd2(ls, p);
            pk[i / 2] = pack_f16(p.x, p.y);
          }
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) pk[i] = 0u;
        }
        tmem_st16(tS + lane_off + c * 16, pk);
      }
      l += ls.x + ls.y;
      }
      tmem_wait_st();
      tc_fence_before();
      mbar_arrive(&bar.p_full[t]);
    }
    // epilogue
    ok = __all_sync(0xffffffffu, ok);
    if (ok && ntiles > 0) ok = mbar_wait_warp(&bar.pv_done[t], (ntiles - 1) & 1, status, 9);
    if (ok) {
      tc_fence_after();
      const int p = quad * BQ + t * 128 + row;
      int n = perm[(size_t)h * N + p];
      if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 124)) n = 0;
      const float inv = (l > 0.f) ? (1.0f / l) * out_scale : 0.f;
      uint16_t *dst = O + ((size_t)n * heads + h) * D;
#pragma unroll 1
      for (int c = 0; c < D; c += 32) {
        uint32_t o[32];
        if (ntiles > 0) {
          tmem_ld32(tO + lane_off + c, o);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = 0u;
        }
        uint4 v[4], rv[4];
        uint32_t *pv = reinterpret_cast<uint32_t *>(v), *pr = reinterpret_cast<uint32_t *>(rv);
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float x0 = __uint_as_float(o[2 * i]) * inv, x1 = __uint_as_float(o[2 * i + 1]) * inv;
          pv[i] = pack_bf16(x0, x1);
          pr[i] = pack_bf16(x0 - bf16lo(pv[i]), x1 - bf16hi(pv[i]));  // rounding residual
        }
#pragma unroll
        for (int i = 0; i < 4; ++i) reinterpret_cast<uint4 *>(dst + c)[i] = v[i];
        if (O_res) {
          uint16_t *rdst = O_res + ((size_t)n * heads + h) * D;
#pragma unroll
          for (int i = 0; i < 4; ++i) reinterpret_cast<uint4 *>(rdst + c)[i] = rv[i];
        }
      }
      // natural-log LSE: ln 2 * (m + log2 l)
      lse[(size_t)h * N + n] = (l > 0.f) ? 0.69314718055994531f * (m + log2f(l)) : -INFINITY;
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
// pre-passes
// ---------------------------------------------------------------------------
// unit_block[h][u] = block of 64-token unit u.
__global__ void unit_block_kernel(const int32_t *__restrict__ blocks, const int32_t *__restrict__ n_blocks, int NB,
                                  int32_t *__restrict__ unit_block) {
  const int h = blockIdx.y;
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b >= n_blocks[h]) return;
  const int32_t *e = blocks + ((size_t)h * NB + b) * 4;
  const int u0 = e[0] >> 6, nu = e[1] >> 6;
  for (int k = 0; k < nu; ++k) unit_block[(size_t)h * NB + u0 + k] = b;
}

// tile_units[h][t] = 64-token units walked by tile t (UPT units) over the
// union of the rows of its distinct blocks (CSR rows for query tiles, CSC
// rows for key tiles).  One warp per tile.
template <int UPT>
__global__ void tile_units_kernel(const int32_t *__restrict__ ptr, const int32_t *__restrict__ idx,
                                  const int32_t *__restrict__ blocks, const int32_t *__restrict__ unit_block, int N,
                                  int heads, int32_t *__restrict__ tile_units) {
  const int NB = N / 64, NT = N / (64 * UPT);
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (gw >= NT * heads) return;
  const int h = gw / NT, t = gw % NT;
  const int32_t *blocks_h = blocks + (size_t)h * NB * 4;
  int b[UPT];
#pragma unroll
  for (int q = 0; q < UPT; ++q) b[q] = unit_block[(size_t)h * NB + UPT * t + q];
  long long cnt = 0;
#pragma unroll
  for (int q = 0; q < UPT; ++q) {
    bool dup = false;
#pragma unroll
    for (int r = 0; r < q; ++r) dup |= (b[r] == b[q]);
    if (dup) continue;
    const int s = ptr[h * NB + b[q]], e = ptr[h * NB + b[q] + 1];
    for (int k = s + lane; k < e; k += 32) {
      const int j = idx[k];
      bool seen = false;  // already counted through an earlier distinct block's row
#pragma unroll
      for (int r = 0; r < q; ++r) {
        bool first = true;
#pragma unroll
        for (int u = 0; u < r; ++u) first &= (b[u] != b[r]);
        if (!first || seen) continue;
        int lo = ptr[h * NB + b[r]], hi = ptr[h * NB + b[r] + 1];
        while (lo < hi) {
          const int mid = (lo + hi) >> 1;
          if (idx[mid] < j)
            lo = mid + 1;
          else
            hi = mid;
        }
        seen = lo < ptr[h * NB + b[r] + 1] && idx[lo] == j;
      }
      if (!seen) cnt += blocks_h[(size_t)j * 4 + 1] >> 6;
    }
  }
  cnt = warp_sum(cnt);
  if (lane == 0) tile_units[(size_t)h * NT + t] = (int32_t)cnt;
}

__device__ __forceinline__ uint4 to_f16x8(uint4 v, bool &bad) {
  return make_uint4(bf16x2_to_f16x2(v.x, bad), bf16x2_to_f16x2(v.y, bad), bf16x2_to_f16x2(v.z, bad),
                    bf16x2_to_f16x2(v.w, bad));
}

// dst[h][p][:] = fp16(src[perm[h][p]][h][:]), rounded to nearest: exact for
// 2^-17 <= |x| <= 65504 and for 0 (bf16's 8 significant bits fit fp16's 11
// down to its subnormal spacing 2^-24); smaller magnitudes move by at most
// 2^-25.  A value outside the fp16 range flags its (operand, head) in
// range_flag [3][heads] (operands s0, s1, s2); range.cu converts those heads
// again with a pre-scale.
__global__ void permute3_kernel(const int32_t *__restrict__ perm, int N, int heads, int D,
                                const uint16_t *__restrict__ s0, const uint16_t *__restrict__ s1,
                                const uint16_t *__restrict__ s2, uint16_t *__restrict__ d0, uint16_t *__restrict__ d1,
                                uint16_t *__restrict__ d2, int32_t *__restrict__ range_flag, int *status) {
  const int vpr = D / 8;  // 16-byte vectors per row
  const size_t g = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  const size_t rows = (size_t)heads * N;
  if (g >= rows * vpr) return;
  const size_t r = g / vpr;
  const int v = (int)(g % vpr);
  const int h = (int)(r / N);
  const int n = perm[r];
  if (!PRISM_CHECK((unsigned)n < (unsigned)N, status, 122)) return;
  const size_t src = ((size_t)n * heads + h) * D + v * 8, dst = r * D + v * 8;
  bool bad0 = false, bad1 = false, bad2 = false;
  *reinterpret_cast<uint4 *>(d0 + dst) = to_f16x8(__ldg(reinterpret_cast<const uint4 *>(s0 + src)), bad0);
  if (s1) *reinterpret_cast<uint4 *>(d1 + dst) = to_f16x8(__ldg(reinterpret_cast<const uint4 *>(s1 + src)), bad1);
  if (s2) *reinterpret_cast<uint4 *>(d2 + dst) = to_f16x8(__ldg(reinterpret_cast<const uint4 *>(s2 + src)), bad2);
  if (bad0) atomicOr(&range_flag[h], 1);
  if (bad1) atomicOr(&range_flag[heads + h], 1);
  if (bad2) atomicOr(&range_flag[2 * heads + h], 1);
}

}  // namespace fwd

cudaError_t launch_permute3(const int32_t *perm, int N, int heads, int D, const uint16_t *s0, const uint16_t *s1,
                            const uint16_t *s2, uint16_t *d0, uint16_t *d1, uint16_t *d2, int32_t *range_flag,
                            int *status, cudaStream_t st) {
  const size_t total = (size_t)heads * N * (D / 8);
  KernelTimer kt_(KT_PERMUTE3, st);
  fwd::permute3_kernel<<<(unsigned)((total + 255) / 256), 256, 0, st>>>(perm, N, heads, D, s0, s1, s2, d0, d1, d2,
                                                                       range_flag, status);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_unit_block(const int32_t *blocks, const int32_t *n_blocks, int NB, int heads,
                              int32_t *unit_block, cudaStream_t st) {
  KernelTimer kt_(KT_UNIT_BLOCK, st);
  fwd::unit_block_kernel<<<dim3((NB + 255) / 256, heads), 256, 0, st>>>(blocks, n_blocks, NB, unit_block);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_tile_units(const int32_t *ptr, const int32_t *idx, const int32_t *blocks,
                              const int32_t *unit_block, int N, int heads, int units_per_tile, int32_t *tile_units,
                              cudaStream_t st) {
  const int warps = (N / (64 * units_per_tile)) * heads;
  KernelTimer kt_(KT_TILE_UNITS, st);
  if (units_per_tile == 4)
    fwd::tile_units_kernel<4><<<(warps * 32 + 255) / 256, 256, 0, st>>>(ptr, idx, blocks, unit_block, N, heads,
                                                                        tile_units);
  else
    fwd::tile_units_kernel<2><<<(warps * 32 + 255) / 256, 256, 0, st>>>(ptr, idx, blocks, unit_block, N, heads,
                                                                        tile_units);
  count_launches(1);
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn get_encode() {
  static EncodeTiledFn fn = nullptr;
  if (!fn) {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D fp16 map over rows of D elements: box = 64 elements x box_rows, 128B swizzle.
cudaError_t make_rows_map(CUtensorMap *map, const void *base, long long rows, int D, int box_rows) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  const cuuint64_t dims[2] = {(cuuint64_t)D, (cuuint64_t)rows};
  const cuuint64_t strides[1] = {(cuuint64_t)D * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  const cuuint32_t estr[2] = {1, 1};
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2, const_cast<void *>(base), dims, strides, box,
                         estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// bf16 map of rank 2..5 (dims and boxes innermost first, strides in bytes for
// dims 1..rank-1), 128-byte swizzle.
cudaError_t make_bf16_map(CUtensorMap *map, const void *base, int rank, const unsigned long long *dims,
                          const unsigned long long *strides, const unsigned *box) {
  EncodeTiledFn enc = get_encode();
  if (!enc) return cudaErrorNotSupported;
  cuuint64_t d[5], st[4];
  cuuint32_t b[5], e[5];
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    b[i] = box[i];
    e[i] = 1;
    if (i + 1 < rank) st[i] = strides[i];
  }
  const CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, (cuuint32_t)rank, const_cast<void *>(base), d, st, b,
                         e, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct FwdWs {
  WsHeader *hdr;
  uint16_t *Qp, *Kp, *Vp;
  int32_t *unit_block, *tile_units;
  int32_t *range_flag;   // [4][heads]
  unsigned *range_max;   // [4][heads]
};
static FwdWs carve_fwd(const prism_params &p, void *ws) {
  const size_t N = (size_t)p.T * p.H * p.W, h = p.heads, D = p.head_dim;
  const size_t tens = align_up(sizeof(uint16_t) * h * N * D, 256);
  char *w = static_cast<char *>(ws);
  FwdWs f;
  f.hdr = reinterpret_cast<WsHeader *>(w);
  w += kWsHeader;
  f.Qp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  f.Kp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  f.Vp = reinterpret_cast<uint16_t *>(w);
  w += tens;
  f.unit_block = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * (N / 64), 256);
  f.tile_units = reinterpret_cast<int32_t *>(w);
  w += align_up(sizeof(int32_t) * h * (N / 256), 256);
  f.range_flag = reinterpret_cast<int32_t *>(w);
  f.range_max = reinterpret_cast<unsigned *>(w + sizeof(int32_t) * 4 * h);
  return f;
}

size_t attn_fwd_ws_bytes(const prism_params &p) {
  const size_t N = (size_t)p.T * p.H * p.W, h = p.heads, D = p.head_dim;
  return kWsHeader + 3 * align_up(sizeof(uint16_t) * h * N * D, 256) + align_up(sizeof(int32_t) * h * (N / 64), 256) +
         align_up(sizeof(int32_t) * h * (N / 256), 256) + align_up(sizeof(int32_t) * 8 * h, 256);
}

template <int D>
static cudaError_t run_fwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                           const FwdWs &w, uint16_t *O, uint16_t *O_res, float *lse, cudaStream_t st) {
  const int N = p.T * p.H * p.W;
  CUtensorMap mQ, mK, mV;
  cudaError_t e;
  if ((e = make_rows_map(&mQ, w.Qp, (long long)p.heads * N, D, 128)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mK, w.Kp, (long long)p.heads * N, D, 64)) != cudaSuccess) return e;
  if ((e = make_rows_map(&mV, w.Vp, (long long)p.heads * N, D, 64)) != cudaSuccess) return e;
  const int smem = fwd::Smem<D>::BYTES + 1024;
  cudaFuncSetAttribute(fwd::attn_fwd_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  const float scale_log2 = effective_scale(p) * 1.4426950408889634f;
  dim3 grid(N / fwd::BQ, p.heads);
  KernelTimer kt_(KT_ATTN_FWD, st);
  fwd::attn_fwd_kernel<D><<<grid, fwd::kThreads, smem, st>>>(mQ, mK, mV, sel.row_ptr, sel.col, plan.blocks,
                                                             w.unit_block, w.tile_units, plan.perm, O, O_res, lse,
                                                             N, p.heads, scale_log2, w.range_max, &w.hdr->status);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_attn_fwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                            const uint16_t *Q, const uint16_t *K, const uint16_t *V, uint16_t *O, uint16_t *O_res,
                            float *lse, void *ws, cudaStream_t st) {
  const int N = p.T * p.H * p.W, NB = N / 64, D = p.head_dim;
  FwdWs w = carve_fwd(p, ws);
  cudaError_t e;
  if ((e = cudaMemsetAsync(w.range_flag, 0, sizeof(int32_t) * 8 * p.heads, st)) != cudaSuccess) return e;
  if ((e = launch_permute3(plan.perm, N, p.heads, D, Q, K, V, w.Qp, w.Kp, w.Vp, w.range_flag, &w.hdr->status,
                           st)) != cudaSuccess)
    return e;
  if ((e = launch_range_fix(plan.perm, N, p.heads, D, RangeSrc{{Q, K, V, nullptr}},
                            RangeDst{{w.Qp, w.Kp, w.Vp, nullptr}}, w.range_flag, w.range_max, nullptr,
                            &w.hdr->status, st)) != cudaSuccess)
    return e;
  if ((e = launch_unit_block(plan.blocks, plan.n_blocks, NB, p.heads, w.unit_block, st)) != cudaSuccess) return e;
  if ((e = launch_tile_units(sel.row_ptr, sel.col, plan.blocks, w.unit_block, N, p.heads, 4, w.tile_units, st)) !=
      cudaSuccess)
    return e;
  return D == 128 ? run_fwd<128>(p, plan, sel, w, O, O_res, lse, st) : run_fwd<64>(p, plan, sel, w, O, O_res, lse, st);
}

}  // namespace prism
