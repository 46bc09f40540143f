// Host-side helpers shared by the C-ABI translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/zf.h"

namespace zf {

constexpr int kBlockValues = 64;      // values per codec block
constexpr int kUnitBytes = 16;        // offset-table unit
constexpr int kHeadDim = 128;
constexpr int kPageTokens = 16;
constexpr int kChunkValues = kPageTokens * kHeadDim;       // one (page, kv head)
constexpr int kChunkBlocks = kChunkValues / kBlockValues;  // 32
// Paged form: every chunk extent starts with 32 base bytes, the u32
// eligibility mask and 12 zero bytes.
constexpr int kChunkHeaderBytes = 48;
constexpr int kMaxGroup = 8;
constexpr int kMaxBatch = 4096;
constexpr size_t kErrBytes = 16;      // device error word + padding at ws start

inline bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

inline zf_status cuda_status(cudaError_t e) { return e == cudaSuccess ? ZF_OK : ZF_ERR_CUDA; }

inline int current_sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
  return n;
}

}  // namespace zf
