// Device helpers for sm_100a: shared-memory barriers, bulk (TMA) copies,
// tensor-core mma, byte permutes and the pair rebuild of the codec.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/zf.h"

namespace zf {

// A bounded wait gives up after this many nanoseconds of wall time.
constexpr uint64_t kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// ----------------------------------------------------------- mbarriers

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// One bounded-time test of a barrier phase: the thread is suspended in
// hardware until the phase with `parity` completes or about `hint_ns` pass.
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity, uint32_t hint_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(hint_ns)
      : "memory");
  return ok != 0;
}

// Wait until the phase with the given parity has completed; false after
// kWaitLimitNs without completion.  Waiting threads sleep in try_wait rather
// than spin, so they take no issue slots from the warps doing work.
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity) {
  constexpr uint32_t kHintNs = 100000;  // 0.1 ms per suspended try
  if (mbar_try_wait(bar, parity, kHintNs)) return true;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (mbar_try_wait(bar, parity, kHintNs)) return true;
    if (global_timer_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Outcome of a wait that another warp can call off.
enum WaitResult : int { kWaitDone = 1, kWaitAborted = 0, kWaitTimedOut = -1 };

// As mbar_wait_bounded, but a wait that does not complete at the first try
// also gives up as soon as *abort becomes non-zero (another warp of the CTA
// has timed out).  The common case (phase already complete) costs one
// try_wait and no shared-memory load.
__device__ __forceinline__ WaitResult mbar_wait_or_abort(uint32_t bar, uint32_t parity,
                                                         const volatile int32_t* abort) {
  constexpr uint32_t kHintNs = 100000;
  if (mbar_try_wait(bar, parity, kHintNs)) return kWaitDone;
  const uint64_t t0 = global_timer_ns();
  for (;;) {
    if (*abort) return kWaitAborted;
    if (mbar_try_wait(bar, parity, kHintNs)) return kWaitDone;
    if (global_timer_ns() - t0 > kWaitLimitNs) return kWaitTimedOut;
  }
}

// ------------------------------------------------------- bulk copy (TMA)

// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
// src and dst 16-byte aligned, bytes a multiple of 16.  No multicast.
__device__ __forceinline__ void bulk_copy_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar)
      : "memory");
}

// Fetch `bytes` (a multiple of 16, 16-byte aligned) from global memory into
// L2 without waiting for them.
__device__ __forceinline__ void bulk_prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// Order this CTA's earlier generic-proxy shared-memory accesses (made
// visible to this thread through a barrier) before later async-proxy
// (bulk copy) writes to the same shared memory.
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Acquire-release fence at GPU scope (orders this thread's earlier memory
// accesses before its later ones for every thread of the GPU).
__device__ __forceinline__ void fence_acq_rel_gpu() { asm volatile("fence.acq_rel.gpu;" ::: "memory"); }

// ------------------------------------------------------- named barriers

__device__ __forceinline__ void named_barrier_sync(int id, int threads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(threads) : "memory");
}

// ------------------------------------------------------- register split

// Per-warpgroup register budget (all four warps of the warpgroup execute
// it).  A warpgroup that needs few registers gives some back to the pool
// the CTA was launched with; one that needs many then takes them.  The sum
// over warpgroups must not exceed the launch allocation, or the increase
// never completes.
template <int kRegs>
__device__ __forceinline__ void warpgroup_regs_dec() {
  static_assert(kRegs % 8 == 0 && kRegs >= 24 && kRegs <= 256, "setmaxnreg range");
  asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegs));
}
template <int kRegs>
__device__ __forceinline__ void warpgroup_regs_inc() {
  static_assert(kRegs % 8 == 0 && kRegs >= 24 && kRegs <= 256, "setmaxnreg range");
  asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegs));
}

// ------------------------------------------ programmatic dependent launch

// Wait until the grids this one depends on (the previous kernel in the
// stream, when launched with programmatic stream serialization) have
// completed and their memory is visible.  A no-op otherwise.
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// Allow the next kernel in the stream to start launching (it still waits for
// this grid's completion before it touches memory).
__device__ __forceinline__ void launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------- tensor cores

// D += A * B, m16n8k16, bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                          uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Transpose an 8x8 matrix of 16-bit values held in the mma fragment layout
// (lane 4r + c holds row r, columns 2c and 2c+1, the lower column in the low
// half): afterwards lane 4r + c holds row r, columns 2c, 2c+1 of the
// transpose.  All 32 lanes take part.
__device__ __forceinline__ uint32_t transpose8x8_b16(uint32_t x) {
  uint32_t y;
  asm("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

// D += A * B, m16n8k16, f16 inputs, fp32 accumulate (the FP8 comparator:
// E4M3 values are exact in f16).
__device__ __forceinline__ void mma_16816_f16(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                              uint32_t b0, uint32_t b1) {
  asm("mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Two floats -> f16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_f16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ __forceinline__ float f16_lo_to_f32(uint32_t x) {
  float f;
  asm("{\n\t.reg .f16 h;\n\tmov.b32 {h, _}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(x));
  return f;
}
__device__ __forceinline__ float f16_hi_to_f32(uint32_t x) {
  float f;
  asm("{\n\t.reg .f16 h;\n\tmov.b32 {_, h}, %1;\n\tcvt.f32.f16 %0, h;\n\t}" : "=f"(f) : "r"(x));
  return f;
}

// Two E4M3 codes (bits 0..7 and 8..15 of x) -> f16x2, exact.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t x) {
  uint32_t r;
  const uint16_t h = static_cast<uint16_t>(x);
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(h));
  return r;
}

// Two floats -> two E4M3 codes (round to nearest even, saturating at +-448);
// `lo` lands in bits 0..7.
__device__ __forceinline__ uint32_t f32x2_to_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Two floats -> bf16x2 (round to nearest even); `lo` lands in bits 0..15.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// 2^x with the hardware approximation (MUFU.EX2); 2^-inf = +0.
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ float bf16_lo_to_f32(uint32_t x) { return __uint_as_float(x << 16); }
__device__ __forceinline__ float bf16_hi_to_f32(uint32_t x) { return __uint_as_float(x & 0xFFFF0000u); }

// ------------------------------------------------------------- the codec

// Rebuild two consecutive values (2p, 2p+1) of an eligible block.
//   sm4: four sign/mantissa bytes of values 4k..4k+3, byte j = (m_j << 1) | s_(j^1)
//   e4:  four rebuilt exponents (offset + base, one add for four values)
//   sel: 0x5140 for the pair (4k, 4k+1), 0x7362 for (4k+2, 4k+3)
// The permute lays the pair out as [e1][m1 s0][e0][m0 s1], which is the pair
// word (v0 | v1 << 16) rotated left by one bit; rotating right restores it.
__device__ __forceinline__ uint32_t rebuild_pair(uint32_t sm4, uint32_t e4, uint32_t sel) {
  const uint32_t r = __byte_perm(sm4, e4, sel);
  return __funnelshift_r(r, r, 1);
}

// Offsets of four values (low or high nibbles of a nibble-plane word) plus
// the base exponent in every byte: the single integer addition per value
// (base + offset <= 255, so no carry crosses a byte).
__device__ __forceinline__ uint32_t exponents4(uint32_t nib_word, uint32_t shift, uint32_t base4) {
  return ((nib_word >> shift) & 0x0F0F0F0Fu) + base4;
}

__device__ __forceinline__ uint32_t splat_byte(uint32_t b) { return b * 0x01010101u; }

__device__ __forceinline__ void set_error(uint32_t* err, uint32_t bits) {
  if (err) atomicOr(err, bits);
}

}  // namespace zf
