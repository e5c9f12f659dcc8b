// prism_project_v_plan: the value projection V = X Wv^T of a layer's video
// tokens on tcgen05 tensor cores, with prism_plan's zone statistics computed
// in the GEMM's epilogue from the tile it has just produced, so that
// planning never reads V back from HBM.
//
// Method: Prism digest ("Prism：为原生 2K 视频音频联合生成设计的动态稀疏注意力"),
// section on zone guidance and Figure 4: the zone statistics are taken from
// the value features that the video self-attention computes anyway; the
// density section gives the rho_raw terms.  The projection itself is the
// layer's plain linear map of the video tokens to the value features.
//
// Work unit: one CTA per (head, macro-zone), heads fastest so that the CTAs
// of one zone run together and share its X tile in L2.  The CTA computes the
// zone's 512 tokens x head_dim outputs as four 128-token accumulators in TMEM
// (two frames each: the A tile of one accumulator is a 4-D TMA box of
// 2 x 8 x 8 tokens x 64 channels of X), over the K loop of X's C channels in
// steps of 64.
// Roles (384 threads): warp 0 TMA producer, warp 1 TMEM owner and MMA issuer
// (one thread), warps 4-11 the epilogue: TMEM -> bf16 V (to HBM and to a
// shared-memory copy of the zone's tile), then the zone statistics of that
// copy with the very arithmetic of the zone-statistics kernel (zone_stats.cuh).
#include "internal.h"
#include "zone_stats.cuh"

namespace prism {
namespace proj {

constexpr int kThreads = 384;
constexpr int NSTAGE = 2;
constexpr int BK = 64;  // channels of X per stage: one 128-byte swizzle row

template <int D>
struct Smem {
  static constexpr int A_SUB = 128 * BK * 2;      // 128 tokens (two frames) x 64 channels
  static constexpr int A_STAGE = 4 * A_SUB;       // the zone's 512 tokens
  static constexpr int B_STAGE = D * BK * 2;      // D output channels x 64
  static constexpr int STAGE = A_STAGE + B_STAGE;
  static constexpr int MAIN = NSTAGE * STAGE;
  // epilogue: reuses the stage buffers once every product has completed
  static constexpr int OFF_TILE = 0;                              // bf16 [512 tokens][D], 16-byte chunks swizzled
  static constexpr int OFF_STATS = 512 * D * 2;                   // float [2][8][8][D] row and column sums
  static constexpr int OFF_RED = OFF_STATS + 2 * 8 * 8 * D * 4;   // double [8][8]
  static constexpr int EPI = OFF_RED + 8 * 8 * 8;
  static constexpr int OFF_BAR = MAIN > EPI ? MAIN : EPI;
  static constexpr int BYTES = OFF_BAR + 256;
};

struct Bars {
  uint64_t full[NSTAGE], empty[NSTAGE];
  uint64_t acc_full;  // single use: every product of the CTA has completed
  uint64_t drain;     // single use: the MMA thread's in-flight products after an abort
  uint32_t tmem_base;
  int abort;
  int epi_abort;  // written by the epilogue warps only: whether the statistics run
};

__device__ __forceinline__ void tma_load_4d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int c0, int c1,
                                            int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5, %6}], [%2];" ::
          "r"(smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
      : "memory");
}
// barrier 1 of the 256 epilogue threads
__device__ __forceinline__ void epilogue_sync() { asm volatile("bar.sync 1, 256;" ::: "memory"); }

// Position of 16-byte chunk j of tile row tok: chunks are XOR-swizzled by the
// row's low three bits, so that the epilogue's row-per-thread stores do not
// all hit the same banks.
__device__ __forceinline__ int tile_chunk(int tok, int j) { return j ^ (tok & 7); }

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
    project_v_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW, int C,
                     int T, int H, int W, int heads, uint16_t *__restrict__ V, double *__restrict__ vstats,
                     int *status) {
  using L = Smem<D>;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  Bars &bar = *reinterpret_cast<Bars *>(smem + L::OFF_BAR);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int h = blockIdx.x, z = blockIdx.y;
  const int ZH = H / 8, ZW = W / 8;
  const int zt = z / (ZH * ZW), zh = (z / ZW) % ZH, zw = z % ZW;
  const int nk = C / BK;

  if (threadIdx.x == 0) bar.abort = *reinterpret_cast<volatile int *>(status);
  __syncthreads();
  if (bar.abort) return;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NSTAGE; ++s) {
      mbar_init(&bar.full[s], 1);
      mbar_init(&bar.empty[s], 1);
    }
    mbar_init(&bar.acc_full, 1);
    mbar_init(&bar.drain, 1);
    bar.epi_abort = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar.tmem_base, 4 * D);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = bar.tmem_base;

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      prefetch_tensormap(&mapX);
      prefetch_tensormap(&mapW);
      int issued = 0;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % NSTAGE;
        if (kc >= NSTAGE && !mbar_wait(&bar.empty[s], ((kc / NSTAGE) - 1) & 1, status, 301)) {
          bar.abort = 1;
          break;
        }
        if (*reinterpret_cast<volatile int *>(&bar.abort)) break;
        uint8_t *st = smem + s * L::STAGE;
        mbar_arrive_expect_tx(&bar.full[s], L::STAGE);
#pragma unroll
        for (int a = 0; a < 4; ++a)
          tma_load_4d(st + a * L::A_SUB, &mapX, &bar.full[s], kc * BK, zw * 8, zh * 8, zt * 8 + 2 * a);
        tma_load_2d(st + L::A_STAGE, &mapW, &bar.full[s], kc * BK, h * D);
        ++issued;
      }
      drain_loads(bar.full, NSTAGE, issued, status, 302);  // no copy may still be writing when the CTA leaves
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16(128, D, 0);
      bool ok = true;
      for (int kc = 0; kc < nk; ++kc) {
        const int s = kc % NSTAGE;
        if (!(ok = mbar_wait(&bar.full[s], (kc / NSTAGE) & 1, status, 303))) break;
        tc_fence_after();
        const uint32_t st = smem_u32(smem + s * L::STAGE);
        const uint64_t db = sdesc_sw128(st + L::A_STAGE, 16, 1024);
#pragma unroll
        for (int a = 0; a < 4; ++a) {
          const uint64_t da = sdesc_sw128(st + a * L::A_SUB, 16, 1024);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            mma_ss(tmem + a * D, da + kslice16(kk, 0), db + kslice16(kk, 0), idesc, (kc > 0 || kk > 0) ? 1u : 0u);
        }
        mma_commit(&bar.empty[s]);
      }
      if (ok) {
        mma_commit(&bar.acc_full);
      } else {
        bar.abort = 1;
        mma_drain(&bar.drain, status, 304);
      }
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    const int tid = threadIdx.x - 128;  // 0..255
    const int q4 = warp & 3;            // TMEM lane quarter of this warp
    const int pair = (warp - 4) >> 2;   // accumulators 2*pair and 2*pair + 1
    const uint32_t lane_off = (uint32_t)(q4 * 32) << 16;
    bool ok = mbar_wait_warp(&bar.acc_full, 0, status, 305);
    if (ok) {
      tc_fence_after();
      uint16_t *tile = reinterpret_cast<uint16_t *>(smem + L::OFF_TILE);
      const int r = q4 * 32 + lane;  // row of the accumulator: (frame t', y, x) = (r / 64, r / 8 % 8, r % 8)
#pragma unroll 1
      for (int aa = 0; aa < 2; ++aa) {
        const int a = 2 * pair + aa;
        const int tok = a * 128 + r;  // (t, y, x) raster index within the zone
        const int t = tok >> 6, y = (tok >> 3) & 7, x = tok & 7;
        const size_t n = ((size_t)(zt * 8 + t) * H + (zh * 8 + y)) * W + zw * 8 + x;
        uint16_t *dst = V + (n * heads + h) * D;
#pragma unroll 1
        for (int c0 = 0; c0 < D; c0 += 32) {
          uint32_t o[32];
          tmem_ld32(tmem + a * D + c0 + lane_off, o);
          tmem_wait_ld();
          uint4 v[4];
          uint32_t *pv = reinterpret_cast<uint32_t *>(v);
#pragma unroll
          for (int i = 0; i < 16; ++i) pv[i] = pack_bf16(__uint_as_float(o[2 * i]), __uint_as_float(o[2 * i + 1]));
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            reinterpret_cast<uint4 *>(dst + c0)[i] = v[i];
            reinterpret_cast<uint4 *>(tile + tok * D)[tile_chunk(tok, c0 / 8 + i)] = v[i];
          }
        }
      }
    }
    // every epilogue thread reaches the barriers of the statistics below, or
    // none does: the decision is taken from a flag only the epilogue writes
    ok = __all_sync(0xffffffffu, ok);
    if (!ok) bar.epi_abort = 1;
    epilogue_sync();
    if (!*reinterpret_cast<volatile int *>(&bar.epi_abort)) {
      const uint16_t *tile = reinterpret_cast<const uint16_t *>(smem + L::OFF_TILE);
      const auto load = [tile](int t, int y, int x, int cv) {
        const int tok = (t * 8 + y) * 8 + x;
        return reinterpret_cast<const uint4 *>(tile + tok * D)[tile_chunk(tok, cv)];
      };
      zone_stats_core<D>(load, tid, reinterpret_cast<float *>(smem + L::OFF_STATS),
                         reinterpret_cast<double(*)[8]>(smem + L::OFF_RED),
                         vstats + ((size_t)h * gridDim.y + z) * 5, [] { epilogue_sync(); });
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, 4 * D);
  }
}

}  // namespace proj

cudaError_t launch_project_v(const prism_params &p, const uint16_t *X, int C, const uint16_t *Wv, uint16_t *V,
                             double *vstats, int *status, cudaStream_t st) {
  const int D = p.head_dim;
  const int Z = (p.T / 8) * (p.H / 8) * (p.W / 8);
  CUtensorMap mX, mW;
  // X viewed as [T][H][W][C]: box 2 frames x 8 rows x 8 columns x 64 channels
  const unsigned long long xd[4] = {(unsigned long long)C, (unsigned long long)p.W, (unsigned long long)p.H,
                                    (unsigned long long)p.T};
  const unsigned long long xs[3] = {2ull * C, 2ull * C * p.W, 2ull * C * p.W * p.H};
  const unsigned xb[4] = {(unsigned)proj::BK, 8, 8, 2};
  cudaError_t e = make_bf16_map(&mX, X, 4, xd, xs, xb);
  if (e != cudaSuccess) return e;
  // Wv [heads * D][C]: box D output channels x 64
  const unsigned long long wd[2] = {(unsigned long long)C, (unsigned long long)p.heads * D};
  const unsigned long long ws[1] = {2ull * C};
  const unsigned wb[2] = {(unsigned)proj::BK, (unsigned)D};
  if ((e = make_bf16_map(&mW, Wv, 2, wd, ws, wb)) != cudaSuccess) return e;
  dim3 grid(p.heads, Z);
  KernelTimer kt_(KT_PROJECT_V, st);
  if (D == 128) {
    const int sm = proj::Smem<128>::BYTES + 1024;
    cudaFuncSetAttribute(proj::project_v_kernel<128>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    proj::project_v_kernel<128><<<grid, proj::kThreads, sm, st>>>(mX, mW, C, p.T, p.H, p.W, p.heads, V, vstats,
                                                                  status);
  } else {
    const int sm = proj::Smem<64>::BYTES + 1024;
    cudaFuncSetAttribute(proj::project_v_kernel<64>, cudaFuncAttributeMaxDynamicSharedMemorySize, sm);
    proj::project_v_kernel<64><<<grid, proj::kThreads, sm, st>>>(mX, mW, C, p.T, p.H, p.W, p.heads, V, vstats,
                                                                 status);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace prism
