// Decoupled look-back for the single-pass prefix sum of the compress kernel
// (Merrill and Garland, "Single-pass Parallel Prefix Scan with Decoupled
// Look-back"): every tile publishes its aggregate as soon as it is known and
// its inclusive prefix once its own look-back ends; a tile's exclusive prefix
// is the sum of its predecessors' aggregates down to the nearest one that has
// published an inclusive prefix.  Shared by the compress kernel and by the
// check that makes the look-back's bounded wait run out on a device.
#pragma once

#include <cstdint>

#include "zf_device.cuh"

namespace zf {

// Tile states each lane of the look-back reads per round trip (wider windows,
// 2, 4 or 8 per lane, measured slower: more L2 traffic while a window is re-read).
constexpr int kLookBackPerLane = 1;

// Tile state word: status << 32 | units (status 0: nothing published yet).
constexpr uint64_t kStateAggregate = 1ull << 32;
constexpr uint64_t kStateInclusive = 2ull << 32;

__device__ __forceinline__ uint64_t ld_relaxed_u64(const uint64_t* p) {
  uint64_t v;
  asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_relaxed_u64(uint64_t* p, uint64_t v) {
  asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// Exclusive prefix of tile `tile` > 0, run by one whole warp.  Lane i reads
// the states of tiles hi - kPerLane*i - k (k < kPerLane) in one round trip.
// The window is summed, nearest tile first, down to the nearest tile that
// has published its inclusive prefix; a window without one adds all its
// aggregates and moves 32*kPerLane tiles further back.  Every tile in the
// summed range must have published at least its aggregate, else the window
// is read again.  Tile 0 publishes its inclusive prefix at once, so the walk
// ends; if a predecessor publishes nothing for kWaitLimitNs the wait gives
// up, returns false and the prefix is unusable.
template <int kPerLane>
__device__ __forceinline__ bool lookback_prefix(const uint64_t* tile_state, int64_t tile, int lane,
                                                uint32_t& prefix) {
  constexpr unsigned kAll = 0xFFFFFFFFu;
  prefix = 0;
  int64_t hi = tile - 1;
  uint64_t t0 = 0;
  for (;;) {
    uint64_t st[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int64_t j = hi - kPerLane * lane - i;
      st[i] = j >= 0 ? ld_relaxed_u64(&tile_state[j]) : kStateInclusive;
    }
    // nearest inclusive tile: its lane, then its place within the lane
    int first_incl = kPerLane;
#pragma unroll
    for (int i = kPerLane - 1; i >= 0; --i)
      if (static_cast<uint32_t>(st[i] >> 32) == 2u) first_incl = i;
    const uint32_t incl = __ballot_sync(kAll, first_incl < kPerLane);
    const int last_lane = incl ? __ffs(incl) - 1 : 31;  // deepest lane summed
    // items of this lane inside the summed range
    const int n_in = lane < last_lane ? kPerLane : (lane == last_lane ? (incl ? first_incl + 1 : kPerLane) : 0);
    bool missing = false;
    uint32_t part = 0;
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      if (i < n_in) {
        missing |= static_cast<uint32_t>(st[i] >> 32) == 0u;
        part += static_cast<uint32_t>(st[i]);
      }
    }
    if (__any_sync(kAll, missing)) {
      const uint64_t now = __shfl_sync(kAll, global_timer_ns(), 0);
      if (t0 == 0) {
        t0 = now;
      } else if (now - t0 > kWaitLimitNs) {
        return false;
      }
      continue;
    }
    t0 = 0;
#pragma unroll
    for (int d = 16; d >= 1; d >>= 1) part += __shfl_xor_sync(kAll, part, d);
    prefix += part;
    if (incl) return true;
    hi -= kPerLane * 32;
  }
}

}  // namespace zf
