// Thin inline-PTX wrappers for the sm_100a features the FLARE kernels use:
// mbarriers, TMA tensor loads, tcgen05 (TMEM allocation, UMMA, TMEM load/store)
// and the UMMA descriptor encodings.  Every wait on an mbarrier is bounded by
// a wall-clock limit read from %globaltimer; on expiry the wait records an
// error bit in device memory, raises a CTA-local abort flag and returns false,
// so no kernel ever spins forever.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

#include "flare_internal.h"

namespace flare {

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
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
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}
// One arrive per warp (all 32 lanes call it, lane 0 arrives after the warp
// has converged); barriers signalled this way count warps, not threads.
__device__ __forceinline__ void mbar_arrive_warp(uint64_t* bar) {
  __syncwarp();
  if ((threadIdx.x & 31) == 0) mbar_arrive(bar);
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Non-blocking test of the phase with the given parity (for event loops that
// poll several barriers).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Per-CTA context for bounded waits.
struct WaitCtx {
  uint32_t* gerr;        // device error word (FLARE_DEV_* bits)
  volatile int* abort;   // CTA-local abort flag in shared memory
  uint64_t timeout_ns;   // wall-clock limit for one wait
};

// Wait until the phase with the given parity of `bar` has completed.
// Returns false (and raises the abort flag) if the limit expires or another
// thread of the CTA has already aborted.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t spins = 0;
  while (true) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((++spins & 15u) == 0) {
      if (*w.abort) return false;
      if (global_timer_ns() - t0 > w.timeout_ns) {
        atomicOr(w.gerr, FLARE_DEV_TIMEOUT);
        *w.abort = 1;
        return false;
      }
    }
  }
}

// Wait of the single MMA-issuing thread.  A failed poll is followed by a
// pause (FLARE_MMA_WAIT_SLEEP_NS nanoseconds, or a suspend-time hint of
// FLARE_MMA_WAIT_HINT_NS on the poll itself), so that the polling does not
// take the issue slots of the softmax warp that shares its sub-partition.
#ifndef FLARE_MMA_WAIT_SLEEP_NS
#define FLARE_MMA_WAIT_SLEEP_NS 0
#endif
#ifndef FLARE_MMA_WAIT_HINT_NS
#define FLARE_MMA_WAIT_HINT_NS 0
#endif
__device__ __forceinline__ bool mbar_try_wait_hint(uint64_t* bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_mma(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  uint32_t spins = 0;
  while (true) {
#if FLARE_MMA_WAIT_SLEEP_NS > 0
    __nanosleep(FLARE_MMA_WAIT_SLEEP_NS);
#endif
#if FLARE_MMA_WAIT_HINT_NS > 0
    if (mbar_try_wait_hint(bar, parity, FLARE_MMA_WAIT_HINT_NS)) return true;
#else
    if (mbar_try_wait(bar, parity)) return true;
#endif
    if ((++spins & 15u) == 0) {
      if (*w.abort) return false;
      if (global_timer_ns() - t0 > w.timeout_ns) {
        atomicOr(w.gerr, FLARE_DEV_TIMEOUT);
        *w.abort = 1;
        return false;
      }
    }
  }
}

// Warp-collective wait (all 32 lanes call it): the verdict is made uniform
// across the warp so that a following .sync.aligned instruction is never
// executed by part of a warp.
__device__ __forceinline__ bool mbar_wait_warp(uint64_t* bar, uint32_t parity, const WaitCtx& w) {
  const bool ok = mbar_wait(bar, parity, w);
  return __all_sync(0xffffffffu, ok);
}

// Like mbar_wait but ignores the abort flag: used only to drain asynchronous
// copies that are already in flight before a CTA exits.
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint64_t timeout_ns) {
  const uint64_t t0 = global_timer_ns();
  while (!mbar_try_wait(bar, parity)) {
    if (global_timer_ns() - t0 > timeout_ns) return false;
  }
  return true;
}

// Programmatic dependent launch (see LaunchCfg): wait until the previous
// kernel on the stream has completed and its writes are visible (returns at
// once for a kernel launched normally), and let the next kernel start
// launching once every CTA of this grid has called it or exited.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

__device__ __forceinline__ void named_bar_sync(uint32_t id, uint32_t nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ----------------------------------------------------------------------------
// TMA (tiled tensor loads, no multicast)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}
__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, uint64_t* bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ----------------------------------------------------------------------------
// tcgen05: TMEM allocation, fences, MMA, commit
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {  // whole warp
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // whole warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T  (kind::f16, one CTA)
__device__ __forceinline__ void umma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T  (kind::f16, one CTA, A K-major in TMEM)
__device__ __forceinline__ void umma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, {%5, %6, %7, %8}, p;\n\t}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate), "r"(0u), "r"(0u), "r"(0u), "r"(0u)
      : "memory");
}
// Arrive once on `bar` when every MMA previously issued by this thread is done.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_u32(bar))
               : "memory");
}

// UMMA shared-memory matrix descriptor (sm_100 format):
//   [0,14) start>>4, [16,30) leading byte offset>>4, [32,46) stride byte
//   offset>>4, [46,48) version = 1, [61,64) layout (0 none, 2 SW128, 4 SW64,
//   6 SW32).
enum : uint32_t { LAYOUT_SW128 = 2u, LAYOUT_SW64 = 4u, LAYOUT_SW32 = 6u };

__device__ __forceinline__ uint64_t umma_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo, uint32_t layout) {
  uint64_t d = 0;
  d |= static_cast<uint64_t>((saddr >> 4) & 0x3FFFu);
  d |= static_cast<uint64_t>((lbo >> 4) & 0x3FFFu) << 16;
  d |= static_cast<uint64_t>((sbo >> 4) & 0x3FFFu) << 32;
  d |= static_cast<uint64_t>(1u) << 46;
  d |= static_cast<uint64_t>(layout & 7u) << 61;
  return d;
}

// Instruction descriptor for kind::f16 with bf16 A/B and an fp32 accumulator.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((a_mn_major ? 1u : 0u) << 15) |
         ((b_mn_major ? 1u : 0u) << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
// The same with fp16 A/B (type fields 0).
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N, bool a_mn_major, bool b_mn_major) {
  return idesc_bf16_f32(M, N, a_mn_major, b_mn_major) & ~((7u << 7) | (7u << 10));
}

// ----------------------------------------------------------------------------
// TMEM <-> registers, 32 lanes x 32 bit per warp (thread i <-> lane base+i)
// ----------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]),
        "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]),
        "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
               "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
               : "memory");
}
// N consecutive columns (N a multiple of 16; st: a multiple of 8) as 32/16/8-column pieces.
template <int N>
__device__ __forceinline__ void tmem_ld_cols(uint32_t taddr, uint32_t (&r)[N]) {
  static_assert(N % 16 == 0, "tmem_ld_cols: N must be a multiple of 16");
  if constexpr (N >= 32) {
    tmem_ld32(taddr, *reinterpret_cast<uint32_t(*)[32]>(&r[0]));
    if constexpr (N > 32) tmem_ld_cols<N - 32>(taddr + 32, *reinterpret_cast<uint32_t(*)[N - 32]>(&r[32]));
  } else {
    tmem_ld16(taddr, *reinterpret_cast<uint32_t(*)[16]>(&r[0]));
  }
}
template <int N>
__device__ __forceinline__ void tmem_st_cols(uint32_t taddr, const uint32_t (&r)[N]) {
  static_assert(N % 8 == 0, "tmem_st_cols: N must be a multiple of 8");
  if constexpr (N >= 32) {
    tmem_st32(taddr, *reinterpret_cast<const uint32_t(*)[32]>(&r[0]));
    if constexpr (N > 32) tmem_st_cols<N - 32>(taddr + 32, *reinterpret_cast<const uint32_t(*)[N - 32]>(&r[32]));
  } else if constexpr (N >= 16) {
    tmem_st16(taddr, *reinterpret_cast<const uint32_t(*)[16]>(&r[0]));
    if constexpr (N > 16) tmem_st_cols<N - 16>(taddr + 16, *reinterpret_cast<const uint32_t(*)[N - 16]>(&r[16]));
  } else {
    tmem_st8(taddr, *reinterpret_cast<const uint32_t(*)[8]>(&r[0]));
  }
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// ----------------------------------------------------------------------------
// arithmetic helpers
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi);
// Pack two floats to fp16x2 (round to nearest even): lo -> bits [0,16), hi -> [16,32).
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x on the special-function unit (flushes subnormal results to zero).
__device__ __forceinline__ float ex2_mufu(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
// 2^x on the FMA pipe, for x <= ~0 (inputs below -125 are clamped; the
// result is then 2^-125 instead of 0, which the callers' sums absorb).
// Cody-Waite range reduction x = j + f, j = rint(x), f in [-1/2, 1/2]:
// t = x + 1.5*2^23 leaves j in the low mantissa bits of t, so (bits(t) << 23)
// is j shifted into the exponent field; p(f) ~ 2^f is the degree-3 minimax
// polynomial (max relative error 7.5e-5) derived by gen_exp2_poly.py.
__device__ __forceinline__ float ex2_poly(float x) {
  x = fmaxf(x, -125.0f);
  const float t = x + 12582912.0f;
  const float f = x - (t - 12582912.0f);
  float p = fmaf(0x1.c3f76p-5f, f, 0x1.f0de1ap-3f);
  p = fmaf(p, f, 0x1.62f31ap-1f);
  p = fmaf(p, f, 0x1.fff692p-1f);
  return __int_as_float(__float_as_int(p) + (__float_as_int(t) << 23));
}

// ----------------------------------------------------------------------------
// packed fp32 pairs (sm_100: one instruction computes two lanes' worth)
// ----------------------------------------------------------------------------
__device__ __forceinline__ uint64_t f2_pack(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}
__device__ __forceinline__ void f2_unpack(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
// a * b + c, elementwise, round to nearest
__device__ __forceinline__ uint64_t f2_fma(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(a), "l"(b), "l"(c));
  return r;
}
__device__ __forceinline__ uint64_t f2_add(uint64_t a, uint64_t b) {
  uint64_t r;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(r) : "l"(a), "l"(b));
  return r;
}

// ex2_poly of two values with the paired instructions: the same operations,
// each rounded as in ex2_poly, so the results are bitwise the same.
__device__ __forceinline__ void ex2_poly_x2(float x0, float x1, float& e0, float& e1) {
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f), neg_magic = f2_pack(-12582912.0f, -12582912.0f);
  const uint64_t x = f2_pack(fmaxf(x0, -125.0f), fmaxf(x1, -125.0f));
  const uint64_t t = f2_add(x, magic);
  const uint64_t r = f2_add(t, neg_magic);                       // t - magic, exact
  const uint64_t f = f2_fma(r, f2_pack(-1.0f, -1.0f), x);       // x - r, exact
  uint64_t p = f2_fma(f2_pack(0x1.c3f76p-5f, 0x1.c3f76p-5f), f, f2_pack(0x1.f0de1ap-3f, 0x1.f0de1ap-3f));
  p = f2_fma(p, f, f2_pack(0x1.62f31ap-1f, 0x1.62f31ap-1f));
  p = f2_fma(p, f, f2_pack(0x1.fff692p-1f, 0x1.fff692p-1f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  e0 = __int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23));
  e1 = __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23));
}

// Exponentials of one 64-column chunk of scores (raw fp32 bits in a[0..31],
// b[0..31]): e = 2^(s * c - shift), packed to bf16 pairs.  NPOLY of the 32
// pairs use ex2_poly (FMA pipe), spread evenly; the rest use the MUFU.
template <int NPOLY>
__device__ __forceinline__ void exp2_chunk64(const uint32_t (&a)[32], const uint32_t (&b)[32], float c, float shift,
                                             uint32_t (&pk)[32]) {
#pragma unroll
  for (int q = 0; q < 32; ++q) {
    const uint32_t* src = q < 16 ? a : b;
    const int k = q & 15;
    const float x0 = fmaf(__uint_as_float(src[2 * k]), c, -shift);
    const float x1 = fmaf(__uint_as_float(src[2 * k + 1]), c, -shift);
    const bool poly = ((q * NPOLY) % 32) < NPOLY;
    float e0, e1;
    if (poly) {
      e0 = ex2_poly(x0);
      e1 = ex2_poly(x1);
    } else {
      e0 = ex2_mufu(x0);
      e1 = ex2_mufu(x1);
    }
    pk[q] = pack_bf16x2(e0, e1);
  }
}

// Exponentials of one row of NV scores (raw fp32 bits in s[0..NV)): e =
// 2^(s * c - shift), packed to bf16 pairs pk[0..NV/2).  NPOLY of every 32
// pairs use ex2_poly (FMA pipe), spread evenly; the rest use the MUFU.  A row
// exponentiated in pieces passes each piece's first pair index as Q0, so the
// pattern runs on across the pieces.
#ifndef FLARE_PACKED_F32X2
#define FLARE_PACKED_F32X2 1
#endif
template <int NV, int NPOLY, int Q0 = 0, bool F16 = false>
__device__ __forceinline__ void exp2_row(const uint32_t (&s)[NV], float c, float shift, uint32_t (&pk)[NV / 2]) {
#if FLARE_PACKED_F32X2
  // the scale-and-shift of a pair of scores is one paired fma
  const uint64_t c2 = f2_pack(c, c), ms2 = f2_pack(-shift, -shift);
#endif
#pragma unroll
  for (int q = 0; q < NV / 2; ++q) {
    float x0, x1;
#if FLARE_PACKED_F32X2
    f2_unpack(f2_fma(f2_pack(__uint_as_float(s[2 * q]), __uint_as_float(s[2 * q + 1])), c2, ms2), x0, x1);
#else
    x0 = fmaf(__uint_as_float(s[2 * q]), c, -shift);
    x1 = fmaf(__uint_as_float(s[2 * q + 1]), c, -shift);
#endif
    const bool poly = ((((q + Q0) % 32) * NPOLY) % 32) < NPOLY;
    float e0, e1;
    if (poly) {
#if FLARE_PACKED_F32X2
      ex2_poly_x2(x0, x1, e0, e1);
#else
      e0 = ex2_poly(x0);
      e1 = ex2_poly(x1);
#endif
    } else {
      e0 = ex2_mufu(x0);
      e1 = ex2_mufu(x1);
    }
    pk[q] = F16 ? pack_f16x2(e0, e1) : pack_bf16x2(e0, e1);
  }
}

// Pack two floats to bf16x2 (round to nearest even): lo -> bits [0,16), hi -> [16,32).
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}
__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace flare
