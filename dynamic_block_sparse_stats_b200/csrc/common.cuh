// Device helpers shared by the Prism kernels: status word, bf16 unpacking,
// and thin inline-PTX wrappers for mbarrier, TMA and tcgen05 (sm_100a).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/prism.h"

namespace prism {

// ---------------------------------------------------------------------------
// Workspace header.  Every workspace starts with this 256-byte block; the
// first int is the status word kernels write when they give up on a wait.
// ---------------------------------------------------------------------------
constexpr size_t kWsHeader = 256;
struct WsHeader {
  int status;       // PRISM_OK or PRISM_ERR_TIMEOUT
  int where;        // kernel-specific code of the wait that timed out
  long long nnz;    // prism_select: running total of selected entries
  long long pad[30];
};
static_assert(sizeof(WsHeader) == kWsHeader, "header size");

inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Longest a kernel spins on one wait before it records PRISM_ERR_TIMEOUT
// (cycles of the SM clock; about 2 s at 1.9 GHz).
constexpr long long kWaitLimitCycles = 4000000000LL;

__device__ __forceinline__ void record_status(int *status, int code, int where) {
  if (status) {
    atomicCAS(status, 0, code);
    atomicExch(status + 1, where);
  }
}
// Debug builds (-DPRISM_DEBUG, `build --debug`): device-side bounds checks
// that record PRISM_ERR_INVALID_ARG and the check's site in the status word,
// and let the caller skip the access, instead of trapping; release builds
// compile every check to `true`.
#ifdef PRISM_DEBUG
#define PRISM_CHECK(cond, status, where) \
  ((cond) ? true : (record_status((status), (int)PRISM_ERR_INVALID_ARG, (where)), false))
#else
#define PRISM_CHECK(cond, status, where) true
#endif

__device__ __forceinline__ void record_timeout(int *status, int where) {
  if (status) {
    atomicExch(status, (int)PRISM_ERR_TIMEOUT);
    atomicExch(status + 1, where);
  }
}

// ---------------------------------------------------------------------------
// bf16 helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float bf16lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

// round-to-nearest-even fp32 -> bf16 bits (inputs are finite)
__device__ __forceinline__ uint32_t f2bf(float f) {
  uint32_t u = __float_as_uint(f);
  u += 0x7fffu + ((u >> 16) & 1u);
  return u >> 16;
}
__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ uint32_t pack_f16(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
// bf16 pair -> fp16 pair, rounded to nearest: exact for 2^-17 <= |x| <= 65504
// and for 0 (bf16's 8 significant bits fit fp16's grid down to its subnormal
// spacing 2^-24); sets *bad when a value lies outside the fp16 range.
__device__ __forceinline__ uint32_t bf16x2_to_f16x2(uint32_t v, bool &bad) {
  const float lo = bf16lo(v), hi = bf16hi(v);
  bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
  return pack_f16(lo, hi);
}

// Power-of-two pre-scale exponent of attention operand `id` (0..3 = Q, K, V,
// dO) of a head from its largest magnitude (float bits; 0 when the head was
// never scanned, i.e. every value fits fp16).  Q and K: the smallest e with
// max * 2^-e <= 65504, the largest fp16 value.  V and dO: the smallest e with
// max * 2^-e <= 16, because they meet in dP = dO V^T, whose D-term sums must
// keep dS = P (dP - Delta) within fp16 (|dP| <= D * 16 * 16).  0 when the
// maximum fits fp16 or is not finite.
__device__ __forceinline__ int range_exp(unsigned bits, int id) {
  const float m = __uint_as_float(bits);
  if (!(m > 65504.f) || !(m < INFINITY)) return 0;
  const float limit = id < 2 ? 65504.f : 16.f;
  int e = 1;
  while (ldexpf(m, -e) > limit) ++e;
  return e;
}

// ---------------------------------------------------------------------------
// shared-memory address
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
                   smem_u32(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: returns false (and records the timeout) if the phase with the
// given parity does not complete within kWaitLimitCycles.
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status, int where) {
  if (mbar_try_wait(bar, parity)) return true;
  long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      record_timeout(status, where);
      return false;
    }
  }
  return true;
}

// Before a CTA leaves: wait (bounded) for the last `nstage` loads a producer
// issued into a ring of `nstage` full barriers (load j went to barrier
// j % nstage, completing its phase j / nstage), so that no copy still writes
// into shared memory the CTA gives back.  After a normal run they are long
// complete.
__device__ __forceinline__ void drain_loads(uint64_t *full, int nstage, int issued, int *status, int where) {
  for (int j = issued > nstage ? issued - nstage : 0; j < issued; ++j)
    mbar_wait(&full[j % nstage], (uint32_t)((j / nstage) & 1), status, where);
}

// Bounded wait whose outcome is the same for every lane of the warp, so that
// the .sync.aligned tcgen05 instructions that follow stay convergent.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t *bar, uint32_t parity, int *status, int where) {
  const bool ok = mbar_wait(bar, parity, status, where);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------------------
// TMA (tiled; each CTA loads into its own shared memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_2d(void *smem_dst, const CUtensorMap *map, uint64_t *bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          smem_u32(smem_dst)),
      "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}
// Untiled bulk copy global -> this CTA's shared memory; both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_load(void *smem_dst, const void *gsrc, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(smem_dst)),
               "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (cta_group::1)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t *smem_dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(smem_dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// D[tmem] (+)= A[smem] * B[smem] per the descriptors; kind::f16 (fp16 or bf16
// operands, as the instruction descriptor says), fp32 accumulation.
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// Arrive on `bar` when all previously issued tcgen05.mma of this thread complete.
__device__ __forceinline__ void mma_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}
// After an abort: wait (bounded) for this thread's MMAs still in flight, so
// that the CTA does not free TMEM under them.  `bar` is a fresh barrier
// (count 1) used for nothing else.
__device__ __forceinline__ void mma_drain(uint64_t *bar, int *status, int where) {
  mma_commit(bar);
  mbar_wait(bar, 0, status, where);
}
// Make this thread's generic-proxy shared-memory writes visible to the async
// proxy (tcgen05.mma operand reads) before the barrier that publishes them.
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
// Fire-and-forget fp32 add to global memory (performed at L2).
__device__ __forceinline__ void red_add_f32(float *p, float v) {
  asm volatile("red.relaxed.gpu.global.add.f32 [%0], %1;" ::"l"(p), "f"(v) : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }
// tcgen05.wait::ld that also names the registers of the load it completes,
// so that no use of them can be scheduled before the wait (needed when other
// work runs between a tcgen05.ld and its wait).
__device__ __forceinline__ void tmem_wait_ld_r(uint32_t (&r)[32]) {
  asm volatile("tcgen05.wait::ld.sync.aligned;"
               : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
                 "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]),
                 "+r"(r[15]), "+r"(r[16]), "+r"(r[17]), "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]),
                 "+r"(r[22]), "+r"(r[23]), "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]),
                 "+r"(r[29]), "+r"(r[30]), "+r"(r[31])
               :
               : "memory");
}

// 32 lanes x 32 consecutive 32-bit columns: thread i of the warp gets lane
// (base_lane + i), columns [col, col+32).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), "=r"(r[8]),
        "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]),
        "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%"
      "18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]),
      "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]),
      "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
      "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

// ---------------------------------------------------------------------------
// UMMA descriptors (sm_100 format)
// ---------------------------------------------------------------------------
// Shared-memory matrix descriptor, 128-byte swizzle:
//   bits  0-13 start address >> 4, 16-29 leading byte offset >> 4,
//   32-45 stride byte offset >> 4, 46-47 version (1), 49-51 base offset (0),
//   52 LBO mode (0), 61-63 layout (2 = SWIZZLE_128B).
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;
  d |= (uint64_t)2 << 61;
  return d;
}
// Offset (in the descriptor's 16-byte units) of the 16-element K slice kk of
// a K-major SW128 tile whose 64-element column chunks are chunk_bytes apart.
// Adding it to a descriptor is exact: shared-memory addresses stay below
// 2^18, so the 14-bit address field never carries.
__host__ __device__ constexpr uint64_t kslice16(int kk, int chunk_bytes) {
  return (uint64_t)(((kk >> 2) * chunk_bytes + (kk & 3) * 32) >> 4);
}

// Instruction descriptor for kind::f16 with fp32 accumulation.
//   bits 4-5 D format (1 = f32), 7-9 A format, 10-12 B format (0 = f16,
//   1 = bf16; A and B always the same type), 15 A major (0 = K), 16 B major
//   (0 = K, 1 = MN), 17-22 N >> 3, 24-28 M >> 4.
__host__ __device__ constexpr uint32_t idesc_bf16(uint32_t M, uint32_t N, uint32_t b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (b_mn_major << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
__host__ __device__ constexpr uint32_t idesc_f16(uint32_t M, uint32_t N, uint32_t b_mn_major) {
  return (1u << 4) | (b_mn_major << 16) | ((N >> 3) << 17) | ((M >> 4) << 24);
}
// fp16 operands with A MN-major (bit 15) as well: A read as the transpose of a
// K-major tile already in shared memory.
__host__ __device__ constexpr uint32_t idesc_f16_amn(uint32_t M, uint32_t N, uint32_t b_mn_major) {
  return idesc_f16(M, N, b_mn_major) | (1u << 15);
}

// ---------------------------------------------------------------------------
// fast arithmetic for the attention softmax
// ---------------------------------------------------------------------------
// 2^x by the MUFU instruction (flush-to-zero; relative error ~2^-22, far below
// the fp16 rounding the result goes through).
__device__ __forceinline__ float ex2f(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, for a share of the softmax exponentials (the MUFU unit
// is otherwise as busy as the tensor pipe).  Cody-Waite style range
// reduction x = n + f, n = floor(x), f in [0, 1): n comes from adding
// 1.5 * 2^23 with rounding toward -inf, 2^f from a degree-3 polynomial whose
// coefficients are a minimax fit of 2^f on [0, 1) in relative error
// (computed here by linear programming; max relative error 7.5e-5 in fp32,
// below half an fp16 ulp), and 2^n is added to the exponent field.
// x is clamped to [-125, 64]: below, the result is far under the smallest
// fp16 subnormal; above, it is +inf after fp16 conversion like the MUFU
// result it replaces.
__device__ __forceinline__ float2 fadd2_rm(float2 a, float2 b) {
  uint64_t d;
  asm("add.rm.f32x2 %0, %1, %2;"
      : "=l"(d)
      : "l"(*reinterpret_cast<uint64_t *>(&a)), "l"(*reinterpret_cast<uint64_t *>(&b)));
  return *reinterpret_cast<float2 *>(&d);
}
__device__ __forceinline__ float fmax3f(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t hmax2u(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2u(float2 a) { return *reinterpret_cast<uint64_t *>(&a); }
__device__ __forceinline__ float2 u2f(uint64_t a) { return *reinterpret_cast<float2 *>(&a); }
// paired fp32 lanes (one instruction for two values)
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)), "l"(f2u(c)));
  return u2f(d);
}
__device__ __forceinline__ float2 ffma2(float2 a, float b, float c) {
  return ffma2(a, make_float2(b, b), make_float2(c, c));
}
__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 fsub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
// 2^x for a pair, on the FMA pipe (see fadd2_rm above for the method)
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  constexpr float c0 = 0.9999251961708069f, c1 = 0.6958335638046265f, c2 = 0.22606714069843292f,
                  c3 = 0.07802452892065048f;
  x.x = fminf(fmaxf(x.x, -125.0f), 64.0f);
  x.y = fminf(fmaxf(x.y, -125.0f), 64.0f);
  const float2 t = fadd2_rm(x, make_float2(kMagic, kMagic));    // floor(x) + 1.5 * 2^23, exactly
  const float2 f = fsub2(x, fsub2(t, make_float2(kMagic, kMagic)));
  float2 p = ffma2(f, make_float2(c3, c3), make_float2(c2, c2));
  p = ffma2(p, f, make_float2(c1, c1));
  p = ffma2(p, f, make_float2(c0, c0));
  // the low mantissa bits of t hold floor(x) (two's complement); shifted
  // into the exponent field they scale p by 2^floor(x)
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// ---------------------------------------------------------------------------
// block-wide helpers
// ---------------------------------------------------------------------------
template <typename T>
__device__ __forceinline__ T warp_sum(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
template <typename T>
__device__ __forceinline__ T warp_max(T v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = max(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

}  // namespace prism
