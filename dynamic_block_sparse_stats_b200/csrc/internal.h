// Internal declarations shared by the translation units of libprism.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"

namespace prism {

// NVTX range around a C-ABI call (a no-op unless a profiler is attached).
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
  NvtxRange(const NvtxRange &) = delete;
  NvtxRange &operator=(const NvtxRange &) = delete;
};

// plan.cu
size_t plan_ws_bytes(const prism_params &p);
cudaError_t launch_plan(const prism_params &p, const uint16_t *V, const float *a, const prism_plan_t &out, void *ws,
                        cudaStream_t st);
// the plan after the zone statistics of V (K1a, K2, K3), from the statistics
// already in the workspace (plan_vstats)
cudaError_t launch_plan_tail(const prism_params &p, const float *a, const prism_plan_t &out, void *ws,
                             cudaStream_t st);
// where the workspace holds the per-(head, zone) statistics of V: double [heads][Z][5]
double *plan_vstats(void *ws);

// project.cu
cudaError_t launch_project_v(const prism_params &p, const uint16_t *X, int C, const uint16_t *Wv, uint16_t *V,
                             double *vstats, int *status, cudaStream_t st);

// select.cu
size_t select_ws_bytes(const prism_params &p);
size_t select_max_nb(const prism_params &p);
cudaError_t launch_select(const prism_params &p, const prism_plan_t &plan, const uint16_t *Q, const uint16_t *K,
                          prism_select_t &out, void *ws, cudaStream_t st, long long *nnz_out);

// attn_fwd.cu
size_t attn_fwd_ws_bytes(const prism_params &p);
cudaError_t launch_attn_fwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                            const uint16_t *Q, const uint16_t *K, const uint16_t *V, uint16_t *O, uint16_t *O_res,
                            float *lse, void *ws, cudaStream_t st);

// attn_bwd.cu
size_t attn_bwd_ws_bytes(const prism_params &p);
cudaError_t launch_attn_bwd(const prism_params &p, const prism_plan_t &plan, const prism_select_t &sel,
                            const uint16_t *Q, const uint16_t *K, const uint16_t *V, const uint16_t *O,
                            const uint16_t *O_res, const uint16_t *dO, const float *lse, void *dQ, void *dK,
                            void *dV, int grad_fp32, int deterministic, void *ws, cudaStream_t st);

// shared launch helper: token gather into permuted head-major order with the
// bf16 -> fp16 conversion of the attention operands:
// dst[h][p][:] = fp16(src[perm[h][p]][h][:]) for up to three tensors at once
// (operand ids 0, 1, 2 = Q, K, V); a value outside the fp16 range sets
// range_flag[id][h] (range.cu then converts that head again, pre-scaled).
cudaError_t launch_permute3(const int32_t *perm, int N, int heads, int D, const uint16_t *s0, const uint16_t *s1,
                            const uint16_t *s2, uint16_t *d0, uint16_t *d1, uint16_t *d2, int32_t *range_flag,
                            int *status, cudaStream_t st);

// range.cu: full bf16 range of the attention operands (ids 0..3 = Q, K, V,
// dO).  For every (operand, head) flagged by the gather: its largest
// magnitude into range_max[id][h] (float bits), then the gather again with the
// pre-scale 2^-range_exp(range_max[id][h]); Delta (when given) divided by
// 2^(e_dO + e_V).  range_flag and range_max are [4][heads], zeroed by the
// caller before the gather.
struct RangeSrc {
  const uint16_t *p[4];
};
struct RangeDst {
  uint16_t *p[4];
};
cudaError_t launch_range_fix(const int32_t *perm, int N, int heads, int D, RangeSrc src, RangeDst dst,
                             int32_t *range_flag, unsigned *range_max, float *delta, int *status, cudaStream_t st);

float effective_scale(const prism_params &p);

// attention pre-passes (attn_fwd.cu), shared by the backward
cudaError_t launch_unit_block(const int32_t *blocks, const int32_t *n_blocks, int NB, int heads,
                              int32_t *unit_block, cudaStream_t st);
// tile_units[h][t]: 64-token units walked by tile t (units_per_tile = 2 or 4
// units) over the union of the rows (ptr, idx) of its distinct blocks (CSR
// for query tiles, CSC for key tiles).
cudaError_t launch_tile_units(const int32_t *ptr, const int32_t *idx, const int32_t *blocks,
                              const int32_t *unit_block, int N, int heads, int units_per_tile, int32_t *tile_units,
                              cudaStream_t st);
// 2-D fp16 tensor map over rows of D elements, box 64 x box_rows, 128B swizzle.
cudaError_t make_rows_map(CUtensorMap *map, const void *base, long long rows, int D, int box_rows);
// bf16 tensor map of rank 2..5, 128B swizzle (dims, box innermost first;
// strides in bytes for dims 1..rank-1).
cudaError_t make_bf16_map(CUtensorMap *map, const void *base, int rank, const unsigned long long *dims,
                          const unsigned long long *strides, const unsigned *box);

// host-side count of kernel launches (prism_kernel_launches)
void count_launches(int n);

// timing.cu: optional event timing of every kernel (prism_kernel_timing)
enum KernelTimingId {
  KT_ZONE_STATS = 0,
  KT_BLOCK_MEAN,
  KT_BLOCK_SCORE,
  KT_SELECT_ROW,
  KT_ATTN_FWD,
  KT_ATTN_DKDV,
  KT_ATTN_DQ,
  KT_A2V_NORM,
  KT_ZONE_A2V_STATS,
  KT_PLAN_FINALIZE,
  KT_PERM,
  KT_SELECT_SCAN,
  KT_CSR_FILL,
  KT_CSC_COUNT,
  KT_CSC_SCAN,
  KT_CSC_FILL,
  KT_CSC_SORT,
  KT_PERMUTE3,
  KT_UNIT_BLOCK,
  KT_TILE_UNITS,
  KT_BWD_PREP,
  KT_PROJECT_V,
  KT_RANGE_FIX,
  KT_ATTN_BWD_FUSED,
  KT_DQ_CONVERT,
  KT_COUNT
};
static_assert(KT_COUNT == PRISM_KERNEL_TIMING_IDS, "timing ids");
// Records an event on `st` at construction and at destruction when timing is
// enabled; wrap exactly one kernel launch.
class KernelTimer {
 public:
  KernelTimer(int id, cudaStream_t st);
  ~KernelTimer();

 private:
  cudaStream_t st_;
  int idx_;
};

// api.cu: prism_plan's argument checks; error reporting for prism_last_error
int check_plan_call(const prism_params *p, const uint16_t *V, const float *a2v_norm, const prism_plan_t *out);
int report_error(int code, const char *msg);
void clear_error();

}  // namespace prism
