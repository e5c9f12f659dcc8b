// Optional per-kernel timing for measurement: CUDA event pairs recorded on the
// launching stream around every kernel launch of the library.
#include <mutex>
#include <vector>

#include "internal.h"

namespace prism {
namespace {

const char *const kNames[KT_COUNT] = {
    "zone_video_stats", "block_mean",  "block_score", "select_row", "attn_fwd",  "attn_bwd_dkdv", "attn_bwd_dq",
    "a2v_norm",         "zone_a2v_stats", "plan_finalize", "perm",   "select_scan", "csr_fill",    "csc_count",
    "csc_scan",         "csc_fill",    "csc_sort",    "permute3",   "unit_block", "tile_units",    "bwd_prep",
    "project_v",        "range_fix",
    "attn_bwd_fused",   "dq_convert"};

struct Rec {
  cudaEvent_t a, b;
  int id;
};
std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

void give_event(cudaEvent_t e) {
  if (e) g_pool.push_back(e);
}

}  // namespace

KernelTimer::KernelTimer(int id, cudaStream_t st) : st_(st), idx_(-1) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_on) return;
  Rec r{take_event(), take_event(), id};
  if (!r.a || !r.b || cudaEventRecord(r.a, st) != cudaSuccess) {
    give_event(r.a);  // keep the events for the next launch
    give_event(r.b);
    return;
  }
  idx_ = (int)g_recs.size();
  g_recs.push_back(r);
}

KernelTimer::~KernelTimer() {
  if (idx_ < 0) return;
  std::lock_guard<std::mutex> lock(g_mu);
  if (idx_ < (int)g_recs.size()) cudaEventRecord(g_recs[idx_].b, st_);
}

}  // namespace prism

using namespace prism;

extern "C" int prism_kernel_timing(int enable) {
  std::lock_guard<std::mutex> lock(g_mu);
  for (auto &r : g_recs) {
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  g_on = enable != 0;
  return PRISM_OK;
}

extern "C" int prism_kernel_timing_read(int id, int *launches, double *total_ms, const char **name) {
  if (id < 0 || id >= KT_COUNT) return report_error(PRISM_ERR_INVALID_ARG, "kernel timing id out of range");
  std::lock_guard<std::mutex> lock(g_mu);
  int n = 0;
  double ms = 0.0;
  for (auto &r : g_recs) {
    if (r.id != id) continue;
    if (cudaEventSynchronize(r.b) != cudaSuccess) return report_error(PRISM_ERR_CUDA, "event synchronize failed");
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess) return report_error(PRISM_ERR_CUDA, "event timing failed");
    ms += t;
    ++n;
  }
  if (launches) *launches = n;
  if (total_ms) *total_ms = ms;
  if (name) *name = kNames[id];
  return PRISM_OK;
}
