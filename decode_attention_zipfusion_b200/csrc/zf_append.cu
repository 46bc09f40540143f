// Append-time compression into a paged-form pool: each decode step adds one
// token per sequence, i.e. two blocks (64 values each) per kv head, and they
// are compressed at once instead of waiting for a separate pass (the summary
// leaves initial compression out of its timing; a serving loop needs it).
//
// Layout (see zf_kv_paged): the chunk of a page that is still filling lives
// in a staging extent of the largest size (header + 32 raw blocks), one per
// (sequence, kv head); its blocks are appended in token order, so earlier
// blocks never move.  When the page's last token arrives the warp moves the
// finished extent to the packed region (bump allocation) and points the
// chunk table there, so full pages take their compressed size.  The data
// buffer is [packed region | staging extents]: the packed region is
// [0, staging offset) and the cursor counts its used 16-byte units.
#include <cuda_runtime.h>

#include <cstdint>

#include "zf_device.cuh"
#include "zf_internal.h"

namespace zf {
namespace {

constexpr unsigned kAll = 0xFFFFFFFFu;
constexpr uint32_t kExtentUnits = (kChunkHeaderBytes + 2 * kChunkValues) / kUnitBytes;  // 259

__device__ __forceinline__ uint32_t rotl1(uint32_t x) { return __funnelshift_l(x, x, 1); }

// One pool's side of an append launch.
struct AppendTarget {
  uint8_t* data;
  uint32_t* chunk_tab;
  int64_t cap_units;
  const uint16_t* vals;   // [B][Hkv][128]
  uint32_t staging_base;  // 16-byte units
  uint32_t* packed_cursor;
};

// One warp per (sequence b, kv head h) of one pool.  Lane l holds values
// 4l..4l+3 of the token's 128: block 2i + (l >> 4) of the chunk (i = token
// slot in its page), in-block values 4 (l & 15) .. + 3.
__device__ __forceinline__ void append_warp(const AppendTarget& tg, int64_t w, int lane,
                                            const int32_t* __restrict__ page_table, int max_pages,
                                            const int32_t* __restrict__ positions, int Hkv, int num_pages,
                                            uint32_t* err) {
  uint8_t* __restrict__ data = tg.data;
  uint32_t* __restrict__ chunk_tab = tg.chunk_tab;
  const int64_t cap_units = tg.cap_units;
  const uint16_t* __restrict__ vals = tg.vals;
  const uint32_t staging_base = tg.staging_base;
  uint32_t* packed_cursor = tg.packed_cursor;
  const int b = static_cast<int>(w / Hkv);
  const int h = static_cast<int>(w - int64_t(b) * Hkv);
  const int32_t t = __ldg(positions + b);
  if (t < 0) return;  // no token for this sequence in this step
  if (t >= max_pages * kPageTokens) {
    if (lane == 0) set_error(err, ZF_DEVERR_SEQ_LEN);
    return;
  }
  const int32_t pid = __ldg(page_table + int64_t(b) * max_pages + t / kPageTokens);
  if (pid < 0 || pid >= num_pages) {
    if (lane == 0) set_error(err, ZF_DEVERR_PAGE_ID);
    return;
  }
  const int64_t c = int64_t(pid) * Hkv + h;
  const int i = t % kPageTokens;  // token slot: blocks 2i, 2i + 1
  const uint32_t slot = staging_base + static_cast<uint32_t>(w) * kExtentUnits;
  uint8_t* ext = data + uint64_t(slot) * kUnitBytes;

  // ---- the token's values and its two blocks' exponent ranges
  const uint2 x = __ldg(reinterpret_cast<const uint2*>(vals + w * kHeadDim) + lane);
  const uint32_t e2a = (x.x >> 7) & 0x00FF00FFu;
  const uint32_t e2b = (x.y >> 7) & 0x00FF00FFu;
  const uint32_t expw = __byte_perm(e2a, e2b, 0x6420);  // four exponent fields
  uint32_t mn = min(min(expw & 0xFF, (expw >> 8) & 0xFF), min((expw >> 16) & 0xFF, expw >> 24));
  uint32_t mx = max(max(expw & 0xFF, (expw >> 8) & 0xFF), max((expw >> 16) & 0xFF, expw >> 24));
#pragma unroll
  for (int d = 1; d < 16; d <<= 1) {  // over the 16 lanes of this lane's block
    mn = min(mn, __shfl_xor_sync(kAll, mn, d));
    mx = max(mx, __shfl_xor_sync(kAll, mx, d));
  }
  const uint32_t el = (mx - mn <= 15u) ? 1u : 0u;
  const uint32_t half = lane >> 4;  // which of the two blocks
  const uint32_t q = lane & 15;
  const uint32_t el0 = __shfl_sync(kAll, el, 0), el1 = __shfl_sync(kAll, el, 16);
  const uint32_t size0 = el0 ? 6u : 8u, size1 = el1 ? 6u : 8u;  // 16-byte units

  // ---- where the two blocks go in the extent
  uint32_t u0 = 3u;  // header only for the first token of a page
  if (i > 0) u0 = __ldcg(chunk_tab + 2 * c + 1);
  if (u0 < 3u || u0 + size0 + size1 > kExtentUnits || uint64_t(slot) + kExtentUnits > uint64_t(cap_units)) {
    if (lane == 0) set_error(err, ZF_DEVERR_EXTENT);
    return;
  }
  uint8_t* blk = ext + (uint64_t(u0) + (half ? size0 : 0u)) * kUnitBytes;

  // ---- encode: sign/mantissa plane, then nibbles (eligible) or exponents (raw)
  const uint32_t smw = __byte_perm(rotl1(x.x), rotl1(x.y), 0x6420);
  reinterpret_cast<uint32_t*>(blk)[q] = smw;
  const uint32_t offw = expw - mn * 0x01010101u;  // four 4-bit offsets (eligible blocks)
  const uint32_t hiw = __shfl_down_sync(kAll, offw, 8);  // values + 32 of the same block
  if (el) {
    if (q < 8) reinterpret_cast<uint32_t*>(blk + 64)[q] = offw | (hiw << 4);
  } else {
    reinterpret_cast<uint32_t*>(blk + 64)[q] = expw;
  }
  // ---- header: base exponents and mask bits of the two new blocks
  if (i == 0 && lane < 3) reinterpret_cast<uint4*>(ext)[lane] = make_uint4(0u, 0u, 0u, 0u);
  __syncwarp();
  if (q == 0) ext[2 * i + half] = static_cast<uint8_t>(mn);
  if (lane == 0) {
    uint32_t* maskp = reinterpret_cast<uint32_t*>(ext + 32);
    const uint32_t old = (i == 0) ? 0u : *maskp;
    *maskp = old | (el0 << (2 * i)) | (el1 << (2 * i + 1));
  }
  const uint32_t units = u0 + size0 + size1;
  __syncwarp();
  if (i < kPageTokens - 1) {
    if (lane == 0) {
      chunk_tab[2 * c] = slot;
      chunk_tab[2 * c + 1] = units;
    }
    return;
  }
  // ---- the page is full: move its extent to the packed region
  uint32_t dst = 0;
  if (lane == 0) dst = atomicAdd(packed_cursor, units);
  dst = __shfl_sync(kAll, dst, 0);
  // the packed region is [0, staging_base): full extents never reach staging
  if (uint64_t(dst) + units > uint64_t(staging_base)) {
    if (lane == 0) {
      set_error(err, ZF_DEVERR_EXTENT);
      chunk_tab[2 * c] = slot;  // stays readable in staging until the slot is reused
      chunk_tab[2 * c + 1] = units;
    }
    return;
  }
  const uint4* from = reinterpret_cast<const uint4*>(ext);
  uint4* to = reinterpret_cast<uint4*>(data + uint64_t(dst) * kUnitBytes);
  for (uint32_t k = lane; k < units; k += 32) to[k] = from[k];
  if (lane == 0) {
    chunk_tab[2 * c] = dst;
    chunk_tab[2 * c + 1] = units;
  }
}

// n_targets pools (1: K or V alone; 2: K and V of the same step, one launch):
// warps [0, B * Hkv) append to t0, the next B * Hkv to t1.
__global__ void __launch_bounds__(256)
    append_kernel(AppendTarget t0, AppendTarget t1, int n_targets, const int32_t* __restrict__ page_table,
                  int max_pages, const int32_t* __restrict__ positions, int B, int Hkv, int num_pages,
                  uint32_t* err) {
  const int lane = threadIdx.x & 31;
  const int64_t gw = (int64_t(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t per = int64_t(B) * Hkv;
  if (gw >= per * n_targets) return;
  const bool second = gw >= per;
  append_warp(second ? t1 : t0, second ? gw - per : gw, lane, page_table, max_pages, positions, Hkv, num_pages,
              err);
}

// Host checks of a pool alone (also for B == 0).
zf_status check_pool(const zf_kv_paged* pool, int Hkv) {
  if (!pool || !pool->data || !pool->chunk_tab || !aligned(pool->data, 16) || !aligned(pool->chunk_tab, 8) ||
      pool->num_chunks < 0 || pool->data_cap_bytes < 0 || Hkv <= 0 || pool->num_chunks % Hkv)
    return ZF_ERR_INVALID_ARG;
  return ZF_OK;
}

// Host checks of one pool's side of an append (B > 0); fills its launch
// arguments.
zf_status append_target(const zf_kv_paged* pool, const uint16_t* vals, int B, int Hkv, int64_t staging_offset,
                        uint32_t* packed_cursor, AppendTarget& tg, int64_t& num_pages) {
  if (!vals || !aligned(vals, 8) || !packed_cursor) return ZF_ERR_INVALID_ARG;
  if (staging_offset < 0 || staging_offset % kUnitBytes) return ZF_ERR_INVALID_ARG;
  const int64_t cap_units = pool->data_cap_bytes / kUnitBytes;
  const int64_t staging_units = staging_offset / kUnitBytes;
  if (staging_units + int64_t(B) * Hkv * kExtentUnits > cap_units) return ZF_ERR_WORKSPACE;
  if (cap_units > 0xFFFFFFFFll) return ZF_ERR_UNSUPPORTED;  // u32 units in the chunk table
  num_pages = pool->num_chunks / Hkv;
  if (num_pages > 0x7FFFFFFF) return ZF_ERR_UNSUPPORTED;
  tg = AppendTarget{static_cast<uint8_t*>(pool->data), pool->chunk_tab, cap_units, vals,
                    static_cast<uint32_t>(staging_units), packed_cursor};
  return ZF_OK;
}

zf_status launch_append(const AppendTarget& t0, const AppendTarget& t1, int n_targets, const int32_t* page_table,
                        int max_pages_per_seq, const int32_t* positions, int B, int Hkv, int64_t num_pages,
                        uint32_t* err, zf_stream_t stream) {
  const int64_t threads = int64_t(B) * Hkv * n_targets * 32;
  const int64_t blocks = (threads + 255) / 256;
  append_kernel<<<static_cast<unsigned>(blocks), 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      t0, t1, n_targets, page_table, max_pages_per_seq, positions, B, Hkv, static_cast<int>(num_pages), err);
  return cuda_status(cudaGetLastError());
}

}  // namespace
}  // namespace zf

using namespace zf;

extern "C" {

size_t zf_append_staging_bytes(int B, int Hkv) {
  if (B < 0 || Hkv <= 0) return 0;
  return static_cast<size_t>(B) * Hkv * kExtentUnits * kUnitBytes;
}

zf_status zf_append_paged(const zf_kv_paged* pool, const uint16_t* vals, const int32_t* page_table,
                          int max_pages_per_seq, const int32_t* positions, int B, int Hkv, int64_t staging_offset,
                          uint32_t* packed_cursor, uint32_t* err, zf_stream_t stream) {
  if (check_pool(pool, Hkv) != ZF_OK || B < 0 || max_pages_per_seq <= 0) return ZF_ERR_INVALID_ARG;
  if (B == 0) return ZF_OK;
  if (!page_table || !positions) return ZF_ERR_INVALID_ARG;
  AppendTarget tg{};
  int64_t num_pages = 0;
  const zf_status st = append_target(pool, vals, B, Hkv, staging_offset, packed_cursor, tg, num_pages);
  if (st != ZF_OK) return st;
  return launch_append(tg, tg, 1, page_table, max_pages_per_seq, positions, B, Hkv, num_pages, err, stream);
}

zf_status zf_append_paged_kv(const zf_kv_paged* k_pool, const zf_kv_paged* v_pool, const uint16_t* k_vals,
                             const uint16_t* v_vals, const int32_t* page_table, int max_pages_per_seq,
                             const int32_t* positions, int B, int Hkv, int64_t k_staging_offset,
                             int64_t v_staging_offset, uint32_t* k_packed_cursor, uint32_t* v_packed_cursor,
                             uint32_t* err, zf_stream_t stream) {
  if (check_pool(k_pool, Hkv) != ZF_OK || check_pool(v_pool, Hkv) != ZF_OK || B < 0 || max_pages_per_seq <= 0)
    return ZF_ERR_INVALID_ARG;
  if (k_pool->num_chunks != v_pool->num_chunks || k_pool->data == v_pool->data ||
      k_pool->chunk_tab == v_pool->chunk_tab)
    return ZF_ERR_INVALID_ARG;
  if (B == 0) return ZF_OK;
  if (!page_table || !positions || k_packed_cursor == v_packed_cursor) return ZF_ERR_INVALID_ARG;
  AppendTarget tk{}, tv{};
  int64_t num_pages = 0;
  zf_status st = append_target(k_pool, k_vals, B, Hkv, k_staging_offset, k_packed_cursor, tk, num_pages);
  if (st != ZF_OK) return st;
  st = append_target(v_pool, v_vals, B, Hkv, v_staging_offset, v_packed_cursor, tv, num_pages);
  if (st != ZF_OK) return st;
  return launch_append(tk, tv, 2, page_table, max_pages_per_seq, positions, B, Hkv, num_pages, err, stream);
}

}  // extern "C"
