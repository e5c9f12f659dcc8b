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

// Merge of up to NL sorted rows (the distinct blocks of a query or key tile)
// into one ascending stream of 64-token units.  Each unit carries a mask:
// bit q is set when the block of the tile's q-th 64-row quarter selected it.
template <int NL>
struct UnitWalk {
  Cursor c[NL];
  int mask[NL];
  uint32_t cur_ub;
  int cur_cnt, cur_k, cur_mask;
};

// Set up the walk for a tile made of `nq` units whose blocks are blk[0..nq):
// slot q holds the row of quarter q's block unless an earlier quarter has
// the same block (then the slot stays empty and that quarter's bit is added
// to the earlier slot's mask).  All indices are compile-time after unrolling.
template <int NL>
__device__ __forceinline__ void walk_init(UnitWalk<NL> &w, const int (&blk)[NL], int nq,
                                          const int32_t *__restrict__ ptr, int row0) {
#pragma unroll
  for (int q = 0; q < NL; ++q) {
    bool dup = false;
#pragma unroll
    for (int r = 0; r < q; ++r) dup |= (blk[r] == blk[q]);
    const bool live = q < nq && !dup;
    if (live)
      cursor_init(w.c[q], ptr[row0 + blk[q]], ptr[row0 + blk[q] + 1]);
    else
      cursor_init(w.c[q], 0, 0);
    int m = 0;
#pragma unroll
    for (int r = q; r < NL; ++r)
      if (r < nq && blk[r] == blk[q]) m |= 1 << r;
    w.mask[q] = live ? m : 0;
  }
  w.cur_cnt = 0;
  w.cur_k = 0;
  w.cur_ub = 0;
  w.cur_mask = 0;
}

template <int NL>
__device__ __forceinline__ void walk_next(UnitWalk<NL> &w, const int32_t *__restrict__ col,
                                          const int32_t *__restrict__ blocks_h, uint32_t &unit, int &mask) {
  if (w.cur_k >= w.cur_cnt) {
    uint32_t e[NL], key[NL];
    uint32_t kmin = kEnd;
#pragma unroll
    for (int r = 0; r < NL; ++r) {
      e[r] = cursor_peek(w.c[r], col, blocks_h);
      key[r] = e[r] == kEnd ? kEnd : (e[r] & 0x0fffffffu);
      kmin = min(kmin, key[r]);
    }
    uint32_t ent = kEnd;
    int m = 0;
#pragma unroll
    for (int r = 0; r < NL; ++r)
      if (key[r] == kmin && kmin != kEnd) {
        ent = e[r];
        m |= w.mask[r];
        ++w.c[r].pos;
      }
    w.cur_ub = ent & 0x0fffffffu;
    w.cur_cnt = (int)(ent >> 28) + 1;
    w.cur_k = 0;
    w.cur_mask = m;
  }
  unit = w.cur_ub + (uint32_t)w.cur_k;
  mask = w.cur_mask;
  ++w.cur_k;
}

}  // namespace attn
}  // namespace prism
