// C-ABI entry points of libprism: argument validation, workspace sizing,
// error reporting and dispatch to the kernels.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <string>

#include "internal.h"

namespace prism {

static thread_local std::string g_last_error;
static std::atomic<uint64_t> g_launches{0};

void count_launches(int n) { g_launches.fetch_add((uint64_t)n, std::memory_order_relaxed); }

static int fail(int code, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
  return code;
}

static int cuda_fail(cudaError_t e, const char *where) {
  return fail(PRISM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

float effective_scale(const prism_params &p) {
  if (p.sm_scale > 0.0f) return p.sm_scale;
  return (float)(1.0 / sqrt((double)p.head_dim));
}

// Common parameter checks.  Returns PRISM_OK or an error code with message.
static int check_params(const prism_params *p) {
  if (!p) return fail(PRISM_ERR_INVALID_ARG, "params is NULL");
  if (p->T <= 0 || p->H <= 0 || p->W <= 0 || p->heads <= 0 || p->head_dim <= 0)
    return fail(PRISM_ERR_INVALID_ARG, "non-positive size (T=%d H=%d W=%d heads=%d head_dim=%d)", p->T, p->H,
                p->W, p->heads, p->head_dim);
  if (p->T % 8 || p->H % 8 || p->W % 8)
    return fail(PRISM_ERR_UNSUPPORTED, "T, H and W must be multiples of the zone edge 8 (got %d, %d, %d)", p->T,
                p->H, p->W);
  if (p->head_dim != 64 && p->head_dim != 128)
    return fail(PRISM_ERR_UNSUPPORTED, "head_dim must be 64 or 128 (got %d)", p->head_dim);
  const long long N = (long long)p->T * p->H * p->W;
  if (N * p->heads * p->head_dim >= (1LL << 40) || N >= (1LL << 30))
    return fail(PRISM_ERR_UNSUPPORTED, "grid too large (N=%lld)", N);
  if (!(p->tau128 >= p->tau256) || !(p->tau256 >= 0.f) || !isfinite(p->tau128))
    return fail(PRISM_ERR_INVALID_ARG, "thresholds must satisfy tau128 >= tau256 >= 0");
  if (!(p->eps > 0.f) || !isfinite(p->eps)) return fail(PRISM_ERR_INVALID_ARG, "eps must be positive");
  if (!(p->top_p >= 0.f) || !isfinite(p->top_p)) return fail(PRISM_ERR_INVALID_ARG, "top_p must be >= 0");
  if (p->topk_abs < 0 || !(p->topk_frac >= 0.f) || !isfinite(p->topk_frac))
    return fail(PRISM_ERR_INVALID_ARG, "top-k must be non-negative");
  if (p->sm_scale < 0.f || !isfinite(p->sm_scale)) return fail(PRISM_ERR_INVALID_ARG, "sm_scale must be >= 0");
  if (!(p->map_exponent >= 0.f && p->map_exponent <= 8.f))
    return fail(PRISM_ERR_INVALID_ARG, "map_exponent must lie in [0, 8] (0 selects 1/2)");
  if (p->guidance < 0 || p->guidance > 3) return fail(PRISM_ERR_INVALID_ARG, "guidance must be 0..3");
  if (p->density < 0 || p->density > 3) return fail(PRISM_ERR_INVALID_ARG, "density must be 0..3");
  return PRISM_OK;
}

// The kernels move tensor rows in 16-byte vectors (and the plan table in
// int4 rows), so every such pointer must be 16-byte aligned.
static int check_aligned16(const void *ptr, const char *name) {
  if (reinterpret_cast<uintptr_t>(ptr) % 16) return fail(PRISM_ERR_INVALID_ARG, "%s is not 16-byte aligned", name);
  return PRISM_OK;
}

static int check_plan(const prism_plan_t *pl) {
  if (!pl || !pl->zone_shape || !pl->n_blocks || !pl->blocks || !pl->perm)
    return fail(PRISM_ERR_INVALID_ARG, "plan arrays (zone_shape, n_blocks, blocks, perm) must be non-NULL");
  return check_aligned16(pl->blocks, "plan blocks");
}

static int check_ws(void *ws, size_t bytes, size_t need) {
  if (!ws) return fail(PRISM_ERR_INVALID_ARG, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(ws) % 256) return fail(PRISM_ERR_INVALID_ARG, "workspace not 256-byte aligned");
  if (bytes < need) return fail(PRISM_ERR_CAPACITY, "workspace too small: %zu bytes, need %zu", bytes, need);
  return PRISM_OK;
}

// Argument checks of prism_plan, for other entry points that plan the same way.
int check_plan_call(const prism_params *p, const uint16_t *V, const float *a2v_norm, const prism_plan_t *out) {
  int rc;
  if ((rc = check_params(p)) != PRISM_OK) return rc;
  if (!V) return fail(PRISM_ERR_INVALID_ARG, "V is NULL");
  if ((rc = check_aligned16(V, "V")) != PRISM_OK) return rc;
  if (p->density == 3 && !a2v_norm) return fail(PRISM_ERR_INVALID_ARG, "density 3 (A2V strength) needs a2v_norm");
  return check_plan(out);
}

int report_error(int code, const char *msg) { return fail(code, "%s", msg); }

void clear_error() { g_last_error.clear(); }

}  // namespace prism

using namespace prism;

extern "C" {

const char *prism_version(void) { return "0.1.0"; }

uint64_t prism_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

const char *prism_last_error(void) { return g_last_error.c_str(); }

size_t prism_plan_workspace_size(const prism_params *p) {
  if (check_params(p) != PRISM_OK) return 0;
  return plan_ws_bytes(*p);
}

int prism_plan(const prism_params *p, const uint16_t *V, const float *a2v_norm, const prism_plan_t *out,
               void *workspace, size_t ws_bytes, prism_stream_t stream) {
  NvtxRange nvtx_("prism_plan");
  int rc;
  if ((rc = check_plan_call(p, V, a2v_norm, out)) != PRISM_OK) return rc;
  if ((rc = check_ws(workspace, ws_bytes, plan_ws_bytes(*p))) != PRISM_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess) e = launch_plan(*p, V, a2v_norm, *out, workspace, st);
  if (e != cudaSuccess) return cuda_fail(e, "prism_plan");
  g_last_error.clear();
  return PRISM_OK;
}

int prism_project_v_plan(const prism_params *p, const uint16_t *X, int32_t C, const uint16_t *Wv, uint16_t *V,
                         const float *a2v_norm, const prism_plan_t *out, void *workspace, size_t ws_bytes,
                         prism_stream_t stream) {
  NvtxRange nvtx_("prism_project_v_plan");
  int rc;
  if ((rc = check_plan_call(p, V, a2v_norm, out)) != PRISM_OK) return rc;
  if (!X || !Wv) return fail(PRISM_ERR_INVALID_ARG, "X or Wv is NULL");
  if ((rc = check_aligned16(X, "X")) != PRISM_OK || (rc = check_aligned16(Wv, "Wv")) != PRISM_OK) return rc;
  if (C <= 0 || C % 64 || C > (1 << 16))
    return fail(PRISM_ERR_INVALID_ARG, "C must be a positive multiple of 64, at most 65536 (got %d)", C);
  if ((rc = check_ws(workspace, ws_bytes, plan_ws_bytes(*p))) != PRISM_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess)
    e = launch_project_v(*p, X, C, Wv, V, plan_vstats(workspace), &static_cast<WsHeader *>(workspace)->status, st);
  if (e == cudaSuccess) e = launch_plan_tail(*p, a2v_norm, *out, workspace, st);
  if (e != cudaSuccess) return cuda_fail(e, "prism_project_v_plan");
  g_last_error.clear();
  return PRISM_OK;
}

size_t prism_select_workspace_size(const prism_params *p) {
  if (check_params(p) != PRISM_OK) return 0;
  return select_ws_bytes(*p);
}

int prism_select(const prism_params *p, const prism_plan_t *plan, const uint16_t *Q, const uint16_t *K,
                 prism_select_t *out, void *workspace, size_t ws_bytes, prism_stream_t stream) {
  NvtxRange nvtx_("prism_select");
  int rc;
  if ((rc = check_params(p)) != PRISM_OK) return rc;
  if (!Q || !K) return fail(PRISM_ERR_INVALID_ARG, "Q or K is NULL");
  if ((rc = check_aligned16(Q, "Q")) != PRISM_OK || (rc = check_aligned16(K, "K")) != PRISM_OK) return rc;
  if ((rc = check_plan(plan)) != PRISM_OK) return rc;
  if (!out || !out->row_ptr || !out->col || out->cap < 0)
    return fail(PRISM_ERR_INVALID_ARG, "select output (row_ptr, col, cap) invalid");
  if ((out->col_ptr == nullptr) != (out->row == nullptr))
    return fail(PRISM_ERR_INVALID_ARG, "col_ptr and row must both be set or both be NULL");
  const size_t NB = (size_t)p->T * p->H * p->W / 64;
  if (NB > select_max_nb(*p))
    return fail(PRISM_ERR_UNSUPPORTED, "too many blocks per head for the selection kernel (%zu > %zu)", NB,
                select_max_nb(*p));
  if ((rc = check_ws(workspace, ws_bytes, select_ws_bytes(*p))) != PRISM_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  long long nnz = 0;
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess) e = launch_select(*p, *plan, Q, K, *out, workspace, st, &nnz);
  if (e != cudaSuccess) return cuda_fail(e, "prism_select");
  out->nnz = nnz;
  if (nnz > out->cap) return fail(PRISM_ERR_CAPACITY, "selection needs %lld entries, capacity %lld", nnz, out->cap);
  if (nnz > 0x7fffffffLL) return fail(PRISM_ERR_CAPACITY, "selection of %lld entries exceeds int32 offsets", nnz);
  g_last_error.clear();
  return PRISM_OK;
}

size_t prism_attn_workspace_size(const prism_params *p, int backward) {
  if (check_params(p) != PRISM_OK) return 0;
  return backward ? attn_bwd_ws_bytes(*p) : attn_fwd_ws_bytes(*p);
}

int prism_attn_fwd(const prism_params *p, const prism_plan_t *plan, const prism_select_t *sel, const uint16_t *Q,
                   const uint16_t *K, const uint16_t *V, uint16_t *O, uint16_t *O_res, float *lse, void *workspace,
                   size_t ws_bytes, prism_stream_t stream) {
  NvtxRange nvtx_("prism_attn_fwd");
  int rc;
  if ((rc = check_params(p)) != PRISM_OK) return rc;
  if (!Q || !K || !V || !O || !lse) return fail(PRISM_ERR_INVALID_ARG, "Q, K, V, O or lse is NULL");
  {
    const void *ptrs[5] = {Q, K, V, O, O_res};
    const char *names[5] = {"Q", "K", "V", "O", "O_res"};
    for (int k = 0; k < 5; ++k)
      if ((rc = check_aligned16(ptrs[k], names[k])) != PRISM_OK) return rc;
  }
  if ((rc = check_plan(plan)) != PRISM_OK) return rc;
  if (!sel || !sel->row_ptr || !sel->col) return fail(PRISM_ERR_INVALID_ARG, "selection is NULL");
  if ((rc = check_ws(workspace, ws_bytes, attn_fwd_ws_bytes(*p))) != PRISM_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess) e = launch_attn_fwd(*p, *plan, *sel, Q, K, V, O, O_res, lse, workspace, st);
  if (e != cudaSuccess) return cuda_fail(e, "prism_attn_fwd");
  g_last_error.clear();
  return PRISM_OK;
}

int prism_attn_bwd(const prism_params *p, const prism_plan_t *plan, const prism_select_t *sel, const uint16_t *Q,
                   const uint16_t *K, const uint16_t *V, const uint16_t *O, const uint16_t *O_res, const uint16_t *dO,
                   const float *lse, void *dQ, void *dK, void *dV, int grad_fp32, int deterministic,
                   void *workspace, size_t ws_bytes, prism_stream_t stream) {
  NvtxRange nvtx_("prism_attn_bwd");
  int rc;
  if ((rc = check_params(p)) != PRISM_OK) return rc;
  if (deterministic != 0 && deterministic != 1) return fail(PRISM_ERR_INVALID_ARG, "deterministic must be 0 or 1");
  if (!Q || !K || !V || !O || !dO || !lse || !dQ || !dK || !dV)
    return fail(PRISM_ERR_INVALID_ARG, "a tensor argument is NULL");
  {
    const void *ptrs[9] = {Q, K, V, O, O_res, dO, dQ, dK, dV};
    const char *names[9] = {"Q", "K", "V", "O", "O_res", "dO", "dQ", "dK", "dV"};
    for (int k = 0; k < 9; ++k)
      if ((rc = check_aligned16(ptrs[k], names[k])) != PRISM_OK) return rc;
  }
  if ((rc = check_plan(plan)) != PRISM_OK) return rc;
  if (!sel || !sel->row_ptr || !sel->col || !sel->col_ptr || !sel->row)
    return fail(PRISM_ERR_INVALID_ARG, "selection with its transpose (col_ptr, row) is required");
  if ((rc = check_ws(workspace, ws_bytes, attn_bwd_ws_bytes(*p))) != PRISM_OK) return rc;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemsetAsync(workspace, 0, kWsHeader, st);
  if (e == cudaSuccess)
    e = launch_attn_bwd(*p, *plan, *sel, Q, K, V, O, O_res, dO, lse, dQ, dK, dV, grad_fp32, deterministic,
                        workspace, st);
  if (e != cudaSuccess) return cuda_fail(e, "prism_attn_bwd");
  g_last_error.clear();
  return PRISM_OK;
}

int prism_workspace_status(const void *workspace, prism_stream_t stream) {
  if (!workspace) return fail(PRISM_ERR_INVALID_ARG, "workspace is NULL");
  int st_word = 0;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(&st_word, workspace, sizeof(int), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "prism_workspace_status");
  return st_word;
}

}  // extern "C"
