// Check of the bounded barrier waits that the decode kernels rely on: one
// CTA runs the same wait functions on a shared-memory barrier whose
// completion the check controls, so each outcome (completed, called off by
// another warp, given up at the time limit) can be observed on a device
// without any fault or hang.  The waiting thread records what it saw; a wait
// that gives up sets ZF_DEVERR_TIMEOUT exactly as the kernels do.
#include <cuda_runtime.h>

#include <cstdint>

#include "zf_device.cuh"
#include "zf_internal.h"
#include "zf_scan.cuh"

namespace zf {
namespace {

// How long the second warp waits before it calls the wait off or completes
// the barrier (long enough that the first try_wait has already failed).
constexpr uint64_t kOtherWarpDelayNs = 1000000;  // 1 ms

__global__ void __launch_bounds__(64) bounded_wait_check_kernel(int mode, int64_t* result, uint32_t* err) {
  __shared__ __align__(8) uint64_t bar;
  __shared__ int32_t abort_flag;
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t b = smem_addr(&bar);
  if (threadIdx.x == 0) {
    mbar_init(b, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (lane != 0) return;
  if (warp == 0) {
    const uint64_t t0 = global_timer_ns();
    int outcome;
    if (mode == ZF_WAITCHECK_PLAIN_TIMEOUT)
      outcome = mbar_wait_bounded(b, 0) ? kWaitDone : kWaitTimedOut;
    else
      outcome = mbar_wait_or_abort(b, 0, &abort_flag);
    result[0] = outcome;
    result[1] = static_cast<int64_t>(global_timer_ns() - t0);
    if (outcome == kWaitTimedOut) set_error(err, ZF_DEVERR_TIMEOUT);
  } else if (mode == ZF_WAITCHECK_ABORT || mode == ZF_WAITCHECK_COMPLETE) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < kOtherWarpDelayNs) {
    }
    if (mode == ZF_WAITCHECK_ABORT)
      atomicExch(&abort_flag, 1);
    else
      mbar_arrive(b);
  }
}

// Tile states of the look-back check (test only; every call rewrites them).
__device__ uint64_t g_lookback_check_states[8];
constexpr int64_t kCheckTile = 5;
constexpr uint32_t kCheckPrefix = 10 + 7 + 7 + 5 + 3;

// The compress kernel's look-back, run by warp 0 for tile 5 over fabricated
// predecessor states: tile 0 inclusive 10, tiles 1 and 2 aggregate 7, tile 4
// aggregate 3, and tile 3 nothing (ZF_WAITCHECK_LOOKBACK_TIMEOUT) or, after
// 1 ms, aggregate 5 published by warp 1 (ZF_WAITCHECK_LOOKBACK_COMPLETE).
__global__ void __launch_bounds__(64) lookback_check_kernel(int mode, int64_t* result, uint32_t* err) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  uint64_t* st = g_lookback_check_states;
  if (threadIdx.x == 0) {
    st_relaxed_u64(&st[0], kStateInclusive | 10u);
    st_relaxed_u64(&st[1], kStateAggregate | 7u);
    st_relaxed_u64(&st[2], kStateAggregate | 7u);
    st_relaxed_u64(&st[3], 0);
    st_relaxed_u64(&st[4], kStateAggregate | 3u);
    __threadfence();
  }
  __syncthreads();
  if (warp == 0) {
    const uint64_t t0 = global_timer_ns();
    uint32_t prefix = 0;
    const bool ok = lookback_prefix<kLookBackPerLane>(st, kCheckTile, lane, prefix);
    if (lane == 0) {
      result[0] = ok ? (prefix == kCheckPrefix ? 1 : 2) : -1;
      result[1] = static_cast<int64_t>(global_timer_ns() - t0);
      if (!ok) set_error(err, ZF_DEVERR_TIMEOUT);
    }
  } else if (mode == ZF_WAITCHECK_LOOKBACK_COMPLETE && lane == 0) {
    const uint64_t t0 = global_timer_ns();
    while (global_timer_ns() - t0 < kOtherWarpDelayNs) {
    }
    st_relaxed_u64(&st[3], kStateAggregate | 5u);
  }
}

}  // namespace
}  // namespace zf

namespace zf {
// The compress kernel with a withheld stage fill (zf_codec.cu).
zf_status compress_stall_check(int64_t* result, uint32_t* err, cudaStream_t s);
}  // namespace zf

extern "C" zf_status zf_check_bounded_wait(int mode, int64_t* result, uint32_t* err, zf_stream_t stream) {
  using namespace zf;
  if (mode < ZF_WAITCHECK_TIMEOUT || mode > ZF_WAITCHECK_COMPRESS_STALL) return ZF_ERR_INVALID_ARG;
  if (!result || !aligned(result, 8) || !err || !aligned(err, 4)) return ZF_ERR_INVALID_ARG;
  if (mode == ZF_WAITCHECK_COMPRESS_STALL) return compress_stall_check(result, err, reinterpret_cast<cudaStream_t>(stream));
  if (mode >= ZF_WAITCHECK_LOOKBACK_TIMEOUT)
    lookback_check_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(mode, result, err);
  else
    bounded_wait_check_kernel<<<1, 64, 0, reinterpret_cast<cudaStream_t>(stream)>>>(mode, result, err);
  return cuda_status(cudaGetLastError());
}
