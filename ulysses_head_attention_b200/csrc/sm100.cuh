// Thin inline-PTX wrappers for the sm_100a features the kernels use:
// mbarriers, TMA tensor loads, tcgen05 MMA / commit / TMEM allocation and
// TMEM <-> register moves.  Only what the kernels here need; no templates
// beyond the register-count helpers.
#pragma once

#include <cuda.h>
#include <cstdint>

namespace uly {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t globaltimer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------------------------
// mbarrier
// ----------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

// try_wait without a suspend-time hint: the hardware's own (short) limit
// applies before it returns false and the caller polls again.  Measured on
// B200 the waiting warp then sees a completed phase sooner than when it is
// parked with a long hint (about 4% per backward step).
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Error words written to the caller's status slot: a wait gave up, a
// kernel found its dynamic shared memory too poorly aligned for its tiles,
// or (debug build only) an index fell outside its buffer.
enum : int {
  kDevOk = 0,
  kDevTimeout = 1,
  kDevSmemAlign = 2,
  kDevBounds = 3,
};

// The bounds-checked debug build (compiled with ULY_DEBUG_BOUNDS) checks every
// global index and TMA tile coordinate before the access: one outside its
// buffer is recorded as kDevBounds in the status word (the first error code
// wins) and the access is skipped, so a wait that then never completes gives
// up on its time limit instead of reading or writing stray memory.  The
// release build compiles every check away.
#ifdef ULY_DEBUG_BOUNDS
constexpr bool kDebugBounds = true;
#else
constexpr bool kDebugBounds = false;
#endif

__device__ __forceinline__ bool in_bounds(bool ok, int* status) {
  if constexpr (!kDebugBounds) {
    return true;
  } else {
    if (!ok && status) atomicCAS(status, 0, kDevBounds);
    return ok;
  }
}

// Bounded wait on an mbarrier phase.  Repeats the (suspending) try_wait;
// every 16 tries it checks the CTA-wide abort flag (set by any warp that gave
// up) and the elapsed time.  Returns false when it gave up: the caller must stop its
// loop, and the kernel reports kDevTimeout through the status word.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                          int* status, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 15u) == 0) {
      if (abort_flag && *abort_flag) return false;
      if (globaltimer_ns() - t0 > limit_ns) {
        if (abort_flag) *abort_flag = 1;
        if (status) atomicExch(status, kDevTimeout);
        return false;
      }
    }
  }
}

// mbar_wait for a whole converged warp: every lane polls, and every lane
// returns the same value, so the warp stays converged for the *_warp issue
// forms that follow.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, volatile int* abort_flag,
                                               int* status, uint64_t limit_ns) {
  if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t it = 1;; ++it) {
    if (__all_sync(0xffffffffu, mbar_try_wait(bar, parity))) return true;
    if ((it & 15u) == 0) {
      const bool stop = abort_flag && *abort_flag;
      const bool late = globaltimer_ns() - t0 > limit_ns;
      if (__any_sync(0xffffffffu, late)) {
        if ((threadIdx.x & 31) == 0) {
          if (abort_flag) *abort_flag = 1;
          if (status) atomicExch(status, kDevTimeout);
        }
        return false;
      }
      if (__any_sync(0xffffffffu, stop)) return false;
    }
  }
}

// ----------------------------------------------------------------------------
// TMA (cp.async.bulk.tensor), no multicast
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

__device__ __forceinline__ void tma_load_4d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int c0, int c1, int c2, int c3) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4, %5}], [%6];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(c3),
        "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tma_load_2d(const CUtensorMap* map, uint64_t* bar, void* dst,
                                            int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Contiguous global -> shared copy (bulk copy engine); 16-byte aligned
// addresses, size a multiple of 16.  Completes bytes on *bar.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

// Make generic-proxy shared-memory writes visible to the async proxy
// (tensor core operand reads, TMA stores).
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM allocation
// ----------------------------------------------------------------------------
// Whole warp executes; the allocated TMEM base address is written to *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
               ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
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

// ----------------------------------------------------------------------------
// tcgen05: descriptors
// ----------------------------------------------------------------------------
// Instruction descriptor, kind::f16 with bf16 A/B and fp32 D.
//   bits 4-5 D format (1 = f32), 7-9 A format (1 = bf16), 10-12 B format,
//   15 A major (1 = MN-major), 16 B major, 17-22 N>>3, 24-28 M>>4.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// The same descriptor with fp16 A and B (format code 0): the backward's
// operands are fp16 copies of its inputs (finer rounding of P and dS).
__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         (uint32_t(N >> 3) << 17) | (uint32_t(M >> 4) << 24);
}

// Shared-memory matrix descriptor for a 128-byte-swizzled operand.
//   bits 0-13 start>>4, 16-29 leading byte offset>>4, 32-45 stride byte
//   offset>>4, 46-47 version (1), 61-63 layout (2 = 128B swizzle).
// K-major: rows of 128 B (64 bf16 of K), 8-row atoms of 1024 B; SBO = 1024,
//   LBO unused (1).  Moving along K inside the 128-B row adds bytes to start.
// MN-major: rows of 128 B hold 64 consecutive M/N elements, one K per row;
//   SBO = distance between 8-row K groups (1024), LBO = distance between
//   64-element M/N chunks.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes) {
  return uint64_t((saddr >> 4) & 0x3FFFu) | (uint64_t((lbo_bytes >> 4) & 0x3FFFu) << 16) |
         (uint64_t((sbo_bytes >> 4) & 0x3FFFu) << 32) | (1ull << 46) | (2ull << 61);
}

// Byte offset of element (row, col16) of a 128B-swizzled tile whose rows are
// 128 bytes: the 16-byte chunk index is XORed with (row mod 8).
__device__ __forceinline__ uint32_t sw128_offset(uint32_t row, uint32_t byte_in_row) {
  return row * 128u + ((((byte_in_row >> 4) ^ (row & 7u)) << 4) | (byte_in_row & 15u));
}

// ----------------------------------------------------------------------------
// tcgen05: MMA and commit (issued by one thread)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive once on *bar when every tcgen05 op issued so far by this thread completes.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               ::"r"(smem_u32(bar)) : "memory");
}

// Whole-warp forms: every lane of the warp executes them convergently and
// elect.sync picks the lane that issues, with no branch around the
// instruction.  Measured on B200, a converged warp issuing this way keeps
// back-to-back M=N=128 MMAs at full rate and a ready-check between groups
// costs ~60 cycles, against ~170 when a lone lane issues and polls.
__device__ __forceinline__ void umma_ss_warp(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_ts_warp(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\tsetp.ne.b32 p, %4, 0;\n\telect.sync _|e, 0xffffffff;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}"
      ::"r"(d_tmem), "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit_warp(uint64_t* bar) {
  asm volatile("{\n\t.reg .pred e;\n\telect.sync _|e, 0xffffffff;\n\t"
               "@e tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n\t}"
               ::"r"(smem_u32(bar)) : "memory");
}

// Register split for warp-specialised kernels of 384 threads launched at
// 168 registers: the first warpgroup (producers, MMA issuer) drops to LO,
// the two softmax warpgroups rise to HI, with 4*32*LO + 8*32*HI <= 384*168.
// ptxas allocates each region to its own limit.
template <int LO, int HI>
__device__ __forceinline__ void regs_split(bool softmax_warpgroup) {
  static_assert(LO % 8 == 0 && HI % 8 == 0 && 128 * LO + 256 * HI <= 384 * 168, "register split over budget");
  if (softmax_warpgroup) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(HI) : "memory");
  else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(LO) : "memory");
}

// The same for NT threads launched at RL registers each: the first warpgroup
// takes LO, the other NT - 128 threads HI, with 128 LO + (NT - 128) HI <= NT RL.
template <int LO, int HI, int NT, int RL>
__device__ __forceinline__ void regs_split_n(bool softmax_warpgroup) {
  static_assert(LO % 8 == 0 && HI % 8 == 0 && 128 * LO + (NT - 128) * HI <= NT * RL, "register split over budget");
  if (softmax_warpgroup) asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(HI) : "memory");
  else asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(LO) : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM <-> registers (warp-collective; warp w touches lanes 32*(w%4)..)
// ----------------------------------------------------------------------------
#define ULY_R8(i) "=r"(r[i]), "=r"(r[i + 1]), "=r"(r[i + 2]), "=r"(r[i + 3]), \
                  "=r"(r[i + 4]), "=r"(r[i + 5]), "=r"(r[i + 6]), "=r"(r[i + 7])
#define ULY_W8(i) "r"(r[i]), "r"(r[i + 1]), "r"(r[i + 2]), "r"(r[i + 3]), \
                  "r"(r[i + 4]), "r"(r[i + 5]), "r"(r[i + 6]), "r"(r[i + 7])

// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : ULY_R8(0), ULY_R8(8), ULY_R8(16), ULY_R8(24)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : ULY_R8(0), ULY_R8(8)
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), ULY_W8(0), ULY_W8(8), ULY_W8(16), ULY_W8(24)
      : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};"
      ::"r"(taddr), ULY_W8(0), ULY_W8(8)
      : "memory");
}

__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

#undef ULY_R8
#undef ULY_W8

// Pack two floats into a bf16x2 word (round to nearest even), lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// Pack two floats into an fp16x2 word (round to nearest even), lo in bits 0-15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x of both halves of an fp16x2 word (one MUFU operation), and the two
// halves widened to float.
__device__ __forceinline__ uint32_t ex2_f16x2(uint32_t x) {
  uint32_t y;
  asm("ex2.approx.f16x2 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}
__device__ __forceinline__ void unpack_f16x2(uint32_t v, float& lo, float& hi) {
  asm("{\n\t.reg .f16 l, h;\n\tmov.b32 {l, h}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, h;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(v));
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// ----------------------------------------------------------------------------
// Packed fp32 pairs (Blackwell f32x2 FMA-pipe instructions)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ uint64_t f2_mul(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// Three-input maximum (one instruction on sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the FMA/ALU pipes, for x <= 126 (arguments here are <= 8).
// Range reduction 2^x = 2^n * 2^f with n = round(x), f in [-1/2, 1/2]: adding
// 1.5 * 2^23 rounds x to an integer held in the low mantissa bits, and those
// bits shifted into the exponent field scale p(f) by 2^n.  p is the degree-3
// polynomial minimising the maximum relative error of 2^f on [-1/2, 1/2]
// (Lawson's iteratively reweighted least squares; fit_exp2_poly.py next to
// this file derives the coefficients): max relative error 7.5e-5 in fp32.
// x is clamped at -125, so anything smaller returns about 2^-125 instead of 0.
constexpr float kExp2PolyC3 = 0.05517167f;   // p(f) = ((c3 f + c2) f + c1) f + c0
constexpr float kExp2PolyC2 = 0.24261114f;
constexpr float kExp2PolyC1 = 0.69326097f;
constexpr float kExp2PolyC0 = 0.99992806f;
constexpr float kExp2Round = 12582912.f;     // 1.5 * 2^23

__device__ __forceinline__ float exp2_poly(float x) {
  x = fmaxf(x, -125.f);
  const float t = x + kExp2Round;
  const float f = x - (t - kExp2Round);
  float q = fmaf(kExp2PolyC3, f, kExp2PolyC2);
  q = fmaf(q, f, kExp2PolyC1);
  q = fmaf(q, f, kExp2PolyC0);
  return __int_as_float(__float_as_int(q) + (__float_as_int(t) << 23));
}

// exp2_poly of both halves of a packed pair, with the same operations in
// packed f32x2 form (bitwise the same results): about 10 instructions for
// the pair instead of 18.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x2 = f2_pack(fmaxf(x0, -125.f), fmaxf(x1, -125.f));
  const uint64_t t = f2_add(x2, f2_pack(kExp2Round, kExp2Round));
  const uint64_t u = f2_add(t, f2_pack(-kExp2Round, -kExp2Round));   // t - 1.5 * 2^23, exact
  const uint64_t f = f2_fma(u, f2_pack(-1.f, -1.f), x2);             // x - u, one rounding
  uint64_t q = f2_fma(f2_pack(kExp2PolyC3, kExp2PolyC3), f, f2_pack(kExp2PolyC2, kExp2PolyC2));
  q = f2_fma(q, f, f2_pack(kExp2PolyC1, kExp2PolyC1));
  q = f2_fma(q, f, f2_pack(kExp2PolyC0, kExp2PolyC0));
  float q0, q1, t0, t1;
  f2_unpack(q, q0, q1);
  f2_unpack(t, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(q0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(q1) + (__float_as_int(t1) << 23)));
}

__device__ __forceinline__ int elect_one_lane() { return (threadIdx.x & 31) == 0; }

}  // namespace uly
