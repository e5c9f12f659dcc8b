// Shared device code of the attention kernels: the walk over a CSR (or CSC)
// row pair in 64-token units.
#pragma once

#include "internal.h"

namespace prism {
namespace attn {

// Packed CSR entry for the walk: unit base (p0/64) | (units-1) << 28.
__device__ __forceinline__ uint32_t pack_entry(const int32_t *__restrict__ blocks_h, int j) {
  const int2 pb = *reinterpret_cast<const int2 *>(blocks_h + (size_t)j * 4);
  return (uint32_t)(pb.x >> 6) | ((uint32_t)((pb.y >> 6) - 1) << 28);
}
constexpr uint32_t kEnd = 0xffffffffu;

// Warp-cooperative cursor over one CSR row: 32 entries are loaded at a time,
// one per lane, and read back with shuffles.  All lanes call it uniformly.
struct Cursor {
  int pos, end, base;
  uint32_t reg;
};
__device__ __forceinline__ void cursor_init(Cursor &c, int b, int e) {
  c.pos = b;
  c.end = e;
  c.base = -1000000;
  c.reg = kEnd;
}
__device__ __forceinline__ uint32_t cursor_peek(Cursor &c, const int32_t *__restrict__ col,
                                                const int32_t *__restrict__ blocks_h) {
  if (c.pos >= c.end) return kEnd;
  if (c.pos - c.base >= 32 || c.pos < c.base) {
    c.base = c.pos;
    const int e = c.pos + (threadIdx.x & 31);
    c.reg = e < c.end ? pack_entry(blocks_h, col[e]) : kEnd;
  }
  return __shfl_sync(0xffffffffu, c.reg, c.pos - c.base);
}

struct UnitWalk {
  Cursor a, b;
  int mask_a, mask_b;
  uint32_t cur_ub;
  int cur_cnt, cur_k, cur_mask;
};
__device__ __forceinline__ void walk_next(UnitWalk &w, const int32_t *__restrict__ col,
                                          const int32_t *__restrict__ blocks_h, uint32_t &unit, int &mask) {
  if (w.cur_k >= w.cur_cnt) {
    const uint32_t ea = cursor_peek(w.a, col, blocks_h);
    const uint32_t eb = cursor_peek(w.b, col, blocks_h);
    const uint32_t ka = ea == kEnd ? kEnd : (ea & 0x0fffffffu);
    const uint32_t kb = eb == kEnd ? kEnd : (eb & 0x0fffffffu);
    uint32_t e;
    if (ka < kb) {
      e = ea;
      w.cur_mask = w.mask_a;
      ++w.a.pos;
    } else if (kb < ka) {
      e = eb;
      w.cur_mask = w.mask_b;
      ++w.b.pos;
    } else {
      e = ea;
      w.cur_mask = w.mask_a | w.mask_b;
      ++w.a.pos;
      ++w.b.pos;
    }
    w.cur_ub = e & 0x0fffffffu;
    w.cur_cnt = (int)(e >> 28) + 1;
    w.cur_k = 0;
  }
  unit = w.cur_ub + (uint32_t)w.cur_k;
  mask = w.cur_mask;
  ++w.cur_k;
}

}  // namespace attn
}  // namespace prism
