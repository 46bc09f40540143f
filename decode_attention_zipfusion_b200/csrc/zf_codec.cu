// Lossless BF16 block codec ("ZipFusion", summary chapter "Twelve Bits and
// One Addition"): compress, decompress and validate kernels + C-ABI calls.
//
// Compress is one pass over the input, in tiles of 384 blocks (48 KB of
// input) taken in order from an atomic counter by one persistent CTA per SM.
// The offset table is an exclusive scan of block sizes done with a decoupled
// look-back across tiles, so the input is read once.  Inside a CTA the work
// is pipelined over four shared-memory stages, one tile each:
//   loader warp     takes tile indices one fill ahead (prefetching that
//                   tile into L2) and copies a tile's input into a free
//                   stage with one 1-D bulk copy;
//   12 compute warps analyse a tile (exponent range of every block, hence
//                   its size; the block bases and eligibility words stay in
//                   shared memory) and publish the tile's total size; then
//                   write the tile analysed two fills earlier, whose prefix
//                   is known by then;
//   look-back warp  turns each published tile size into the tile's prefix.
// So no warp waits on the look-back's L2 round trips while there is a tile
// to analyse, and DRAM keeps streaming the next stages meanwhile.  A warp
// owns 32 consecutive blocks (one eligibility word) and four lanes own one
// block, 16 values (32 bytes) each, so every warp-wide store touches
// contiguous memory.
#include <cuda_runtime.h>

#include <cstdint>

#include "zf_device.cuh"
#include "zf_internal.h"
#include "zf_scan.cuh"

namespace zf {
namespace {

constexpr int kCompressWarps = 12;                    // warps that analyse and write tiles
constexpr int kLoaderWarp = kCompressWarps;           // copies tiles into stages
constexpr int kLookBackWarp = kCompressWarps + 1;     // resolves each tile's prefix
constexpr int kCompressThreads = (kCompressWarps + 2) * 32;
constexpr int kTileBlocks = kCompressWarps * 32;      // one 32-block group per warp (4 KB of input each)
constexpr int kCompressStages = 4;
// A tile is written kWriteLag tiles after it was analysed, so its look-back
// has that long to resolve; a stage is refilled kCompressStages - kWriteLag
// tiles before it is analysed again.
constexpr int kWriteLag = 2;
static_assert(kWriteLag >= 1 && kCompressStages > kWriteLag, "stages must cover the write lag");
constexpr uint32_t kTileBytes = uint32_t(kTileBlocks) * kBlockValues * 2;  // 48 KB
constexpr unsigned kFull = 0xFFFFFFFFu;

// Compress workspace: [0,4) error word, [4,8) tile counter, [16, ...) one
// 8-byte scan state per tile (status << 32 | units).
constexpr size_t kCompressStateOffset = 16;

// Shared memory after the stages.  Each barrier completes one phase per
// stage fill (k-th fill of a stage: parity k & 1).
struct CompressShared {
  uint64_t full[kCompressStages];    // loader -> compute: tile input landed (or: no more tiles)
  uint64_t units[kCompressStages];   // compute warps -> warp 0: per-warp sizes written
  uint64_t agg[kCompressStages];     // warp 0 -> look-back: tile size published
  uint64_t pre[kCompressStages];     // look-back -> compute: tile prefix known
  uint64_t empty[kCompressStages];   // compute -> loader: stage read for the last time
  int64_t tile[kCompressStages];     // tile in the stage; -1: no more tiles
  uint32_t warp_units[kCompressStages][kCompressWarps];
  uint32_t warp_excl[kCompressStages][kCompressWarps];
  uint32_t warp_word[kCompressStages][kCompressWarps];  // eligibility word of each warp's group
  uint8_t blk_base[kCompressStages][kTileBlocks];       // base exponent of every block
  uint32_t aggregate[kCompressStages];
  uint32_t prefix[kCompressStages];
  int32_t abort;  // set by a warp whose wait ran out; the others stop too
};
constexpr size_t kCompressSmem = size_t(kCompressStages) * kTileBytes + sizeof(CompressShared);

__device__ __forceinline__ uint32_t rotl1(uint32_t x) { return __funnelshift_l(x, x, 1); }

__device__ __forceinline__ void payload_store(uint8_t* dst, uint4 v) { *reinterpret_cast<uint4*>(dst) = v; }

// Exponent statistics of the 32 blocks of a warp in a stage: lane (sub, q)
// reads quarter q (values [16q, 16q + 16)) of block 8r + sub of the warp's
// group, r = 0..3; el_r / base_r: that block's eligibility (exponent spread
// <= 15) and base (smallest exponent), the same on its four lanes.  Blocks
// at or past n_blocks are not eligible.  The order of a lane's values does
// not matter here, so they are used as loaded.
__device__ __forceinline__ void block_stats(const uint8_t* stage, int warp, int lane, int64_t warp_first,
                                            int64_t n_blocks, uint32_t (&el_r)[4], uint32_t (&base_r)[4]) {
  const int q = lane & 3;
  const int sub = lane >> 2;
  // Odd blocks read the upper half of their quarter first, so the 8 lanes of
  // one shared-memory phase hit 8 different 16-byte bank groups.
  const int sw = (sub & 1) * 16;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const bool exists = warp_first + 8 * r + sub < n_blocks;
    uint32_t w[8];
    if (exists) {
      const uint8_t* p = stage + size_t(warp * 32 + 8 * r + sub) * (kBlockValues * 2) + 32 * q;
      const uint4 u = *reinterpret_cast<const uint4*>(p + sw);
      const uint4 v = *reinterpret_cast<const uint4*>(p + (16 - sw));
      w[0] = u.x; w[1] = u.y; w[2] = u.z; w[3] = u.w;
      w[4] = v.x; w[5] = v.y; w[6] = v.z; w[7] = v.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) w[k] = 0;
    }
    // the two exponent fields of a word, masked in place (bits 7..14 of each half)
    uint32_t mn = 0x7F807F80u, mx = 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      const uint32_t e2 = w[k] & 0x7F807F80u;
      mn = __vminu2(mn, e2);
      mx = __vmaxu2(mx, e2);
    }
    uint32_t emin = min(mn & 0xFFFFu, mn >> 16) >> 7;
    uint32_t emax = max(mx & 0xFFFFu, mx >> 16) >> 7;
    uint32_t key = ((255u - emin) << 16) | emax;
    key = __vmaxu2(key, __shfl_xor_sync(kFull, key, 1));
    key = __vmaxu2(key, __shfl_xor_sync(kFull, key, 2));
    emin = 255u - (key >> 16);
    emax = key & 0xFFFFu;
    el_r[r] = (exists && emax - emin <= 15u) ? 1u : 0u;
    base_r[r] = emin;
  }
}

// The values of the same blocks in value order (lane (sub, q): quarter q of
// block 8r + sub in x[r]), for the write pass.  Its loads take a 2-way bank
// conflict (two blocks of a shared-memory phase start on the same bank)
// rather than selects to undo a swapped order: measured the faster of the two.
__device__ __forceinline__ void load_blocks(const uint8_t* stage, int warp, int lane, int64_t warp_first,
                                            int64_t n_blocks, uint32_t (&x)[4][8]) {
  const int q = lane & 3;
  const int sub = lane >> 2;
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    if (warp_first + 8 * r + sub < n_blocks) {
      const uint4* p = reinterpret_cast<const uint4*>(stage + size_t(warp * 32 + 8 * r + sub) * (kBlockValues * 2) +
                                                      32 * q);
      const uint4 a = p[0];
      const uint4 b = p[1];
      x[r][0] = a.x; x[r][1] = a.y; x[r][2] = a.z; x[r][3] = a.w;
      x[r][4] = b.x; x[r][5] = b.y; x[r][6] = b.z; x[r][7] = b.w;
    } else {
#pragma unroll
      for (int k = 0; k < 8; ++k) x[r][k] = 0;
    }
  }
}

// The 8 bits at positions 0, 4, ..., 28 of x, packed into bits 0..7.
__device__ __forceinline__ uint32_t every_fourth_bit(uint32_t x) {
  x &= 0x11111111u;
  x = (x | (x >> 3)) & 0x03030303u;
  x = (x | (x >> 6)) & 0x000F000Fu;
  return (x | (x >> 12)) & 0xFFu;
}

__device__ __forceinline__ uint32_t blocks_in_group(int64_t n_blocks, int64_t warp_first) {
  const int64_t left = n_blocks - warp_first;
  return left <= 0 ? 0u : (left >= 32 ? 32u : static_cast<uint32_t>(left));
}

// kPaged: write the paged form instead (one extent per chunk of 32 blocks: a
// 48-byte header, then the chunk's blocks; chunk_tab[c] = {start, extent}).
// A warp owns exactly one chunk, so a chunk's extent starts at the flat
// offset of its first block plus 3 header units for every chunk before and
// including it.
// The group's eligibility word and block bases come from the analysis pass
// (written by this warp's lanes), so only the values are read again.
template <bool kPaged>
__device__ __forceinline__ void write_group(const uint8_t* stage, int warp, int lane, int64_t warp_first,
                                            int64_t n_blocks, uint32_t warp_prefix, uint32_t word,
                                            const uint8_t* grp_base, uint8_t* __restrict__ payload,
                                            uint32_t* __restrict__ offs, uint8_t* __restrict__ base,
                                            uint32_t* __restrict__ elig, uint32_t* __restrict__ chunk_tab) {
  const int q = lane & 3;
  const int sub = lane >> 2;
  __syncwarp();  // the analysis pass's shared-memory writes by the other lanes
  uint32_t x[4][8], el_r[4], base_r[4];
  load_blocks(stage, warp, lane, warp_first, n_blocks, x);
#pragma unroll
  for (int r = 0; r < 4; ++r) {
    el_r[r] = (word >> (8 * r + sub)) & 1u;
    base_r[r] = grp_base[8 * r + sub];
  }
  const uint32_t my_base = grp_base[lane];
  const uint32_t nb_warp = blocks_in_group(n_blocks, warp_first);
  const uint32_t warp_units = 8u * nb_warp - 2u * __popc(word);

  // ---- metadata (owner lanes) and payload (4 lanes per block)
  const int64_t chunk = warp_first >> 5;
  // paged form: this warp's chunk header, and the shift of its payload
  const uint64_t hdr_unit = uint64_t(warp_prefix) + 3ull * uint64_t(chunk);
  const uint64_t payload_shift = kPaged ? 3ull * uint64_t(chunk + 1) : 0ull;
  if constexpr (kPaged) {
    uint8_t* hdr = payload + hdr_unit * kUnitBytes;
    if (lane < static_cast<int>(nb_warp)) hdr[lane] = static_cast<uint8_t>(my_base);
    if (lane == 0 && nb_warp > 0) {
      reinterpret_cast<uint4*>(hdr + 32)[0] = make_uint4(word, 0u, 0u, 0u);
      chunk_tab[2 * chunk] = static_cast<uint32_t>(hdr_unit);
      chunk_tab[2 * chunk + 1] = 3u + warp_units;
    }
  } else {
    if (lane < static_cast<int>(nb_warp)) {
      const uint32_t below = (lane == 0) ? 0u : (word & ((1u << lane) - 1u));
      offs[warp_first + lane] = warp_prefix + 8u * lane - 2u * __popc(below);
      base[warp_first + lane] = static_cast<uint8_t>(my_base);
    }
    if (lane == 0 && nb_warp > 0) elig[warp_first >> 5] = word;
  }

#pragma unroll
  for (int r = 0; r < 4; ++r) {
    const int li = 8 * r + sub;
    const int64_t blk = warp_first + li;
    const uint32_t below = (li == 0) ? 0u : (word & ((1u << li) - 1u));
    const uint32_t unit = warp_prefix + 8u * li - 2u * __popc(below);
    uint8_t* dst = payload + (static_cast<uint64_t>(unit) + payload_shift) * kUnitBytes;
    const uint32_t b4 = splat_byte(base_r[r]);
    uint32_t expw[4], offw[4], smw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t e2a = (x[r][2 * k] >> 7) & 0x00FF00FFu;
      const uint32_t e2b = (x[r][2 * k + 1] >> 7) & 0x00FF00FFu;
      expw[k] = __byte_perm(e2a, e2b, 0x6420);  // four exponent fields, one per byte
      offw[k] = expw[k] - b4;                    // four 4-bit offsets (eligible blocks)
      smw[k] = __byte_perm(rotl1(x[r][2 * k]), rotl1(x[r][2 * k + 1]), 0x6420);
    }
    uint32_t hiw[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) hiw[k] = __shfl_down_sync(kFull, offw[k], 2);  // values + 32
    if (blk < n_blocks) {
      // sign/mantissa plane: the same for both kinds of block
      payload_store(dst + 16 * q, make_uint4(smw[0], smw[1], smw[2], smw[3]));
      if (el_r[r]) {
        if (q < 2) {
          payload_store(dst + 64 + 16 * q, make_uint4(offw[0] | (hiw[0] << 4), offw[1] | (hiw[1] << 4),
                                                      offw[2] | (hiw[2] << 4), offw[3] | (hiw[3] << 4)));
        }
      } else {
        // raw: the exponent plane, one whole exponent field per value
        payload_store(dst + 64 + 16 * q, make_uint4(expw[0], expw[1], expw[2], expw[3]));
      }
    }
  }
}

template <bool kPaged>
__global__ void __launch_bounds__(kCompressThreads, 1)
    compress_kernel(const uint16_t* __restrict__ src, int64_t n_blocks, uint8_t* __restrict__ payload,
                    uint32_t* __restrict__ offs, uint8_t* __restrict__ base, uint32_t* __restrict__ elig,
                    uint32_t* __restrict__ chunk_tab, uint32_t* ws_err, uint32_t* tile_counter,
                    uint64_t* tile_state, int withhold_fill) {
  extern __shared__ __align__(128) uint8_t smem[];
  CompressShared& sh = *reinterpret_cast<CompressShared*>(smem + size_t(kCompressStages) * kTileBytes);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  auto stage_of = [&](int s) { return smem + size_t(s) * kTileBytes; };
  auto fail = [&](WaitResult w) {  // a wait that did not complete
    if (w == kWaitTimedOut && lane == 0) {
      set_error(ws_err, ZF_DEVERR_TIMEOUT);
      atomicExch(&sh.abort, 1);
    }
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < kCompressStages; ++s) {
      mbar_init(smem_addr(&sh.full[s]), 1);
      mbar_init(smem_addr(&sh.units[s]), kCompressWarps);
      mbar_init(smem_addr(&sh.agg[s]), 1);
      mbar_init(smem_addr(&sh.pre[s]), 1);
      mbar_init(smem_addr(&sh.empty[s]), kCompressWarps);
    }
    sh.abort = 0;
    fence_mbar_init();
  }
  __syncthreads();

  if (warp == kLoaderWarp) {
    // ---- fill the stages in turn: fill k goes to stage k % kCompressStages
    if (lane == 0) {
      int k = 0;
      // The next fill's tile index is taken one fill ahead, so the counter's
      // round trip overlaps the wait for a free stage.  Holding an index
      // before its stage is free is safe: this CTA's earlier tiles, which
      // free the stage, wait only on smaller tiles.
      int64_t t_next = atomicAdd(tile_counter, 1u);
      for (;;) {
        const int s = k % kCompressStages;
        const int64_t t = t_next;
        if (t < n_tiles) {
          t_next = atomicAdd(tile_counter, 1u);
          // Its input goes to L2 now: the stage copy that follows a fill
          // later then reads L2 (prefetching further ahead measured slower).
          if (t_next < n_tiles) {
            const int64_t pb = t_next * kTileBlocks;
            bulk_prefetch_l2(src + pb * kBlockValues,
                             static_cast<uint32_t>(n_blocks - pb < kTileBlocks ? n_blocks - pb : kTileBlocks) *
                                 (kBlockValues * 2));
          }
        }
        if (k >= kCompressStages) {
          const WaitResult w = mbar_wait_or_abort(smem_addr(&sh.empty[s]), ((k / kCompressStages) - 1) & 1,
                                                  &sh.abort);
          if (w != kWaitDone) {
            fail(w);
            break;
          }
        }
        if (t >= n_tiles) {
          sh.tile[s] = -1;
          mbar_arrive(smem_addr(&sh.full[s]));
          ++k;
          break;
        }
        sh.tile[s] = t;
        if (blockIdx.x == 0 && k == withhold_fill) {
          // The bounded-wait check: this fill is never delivered (no copy,
          // no arrival), so the compute warps' wait on it runs out.
          ++k;
          continue;
        }
        const int64_t b0 = t * kTileBlocks;
        const uint32_t bytes = static_cast<uint32_t>(n_blocks - b0 < kTileBlocks ? n_blocks - b0 : kTileBlocks) *
                               (kBlockValues * 2);
        mbar_arrive_expect_tx(smem_addr(&sh.full[s]), bytes);
        bulk_copy_g2s(smem_addr(stage_of(s)), src + b0 * kBlockValues, bytes, smem_addr(&sh.full[s]));
        ++k;
      }
      // Copies may still be in flight after an abort: wait (bounded) for the
      // last fill of every stage before the CTA can exit.
      for (int j = k > kCompressStages ? k - kCompressStages : 0; j < k; ++j)
        mbar_wait_bounded(smem_addr(&sh.full[j % kCompressStages]), (j / kCompressStages) & 1);
    }
    return;
  }

  if (warp == kLookBackWarp) {
    // ---- each published tile size -> the tile's exclusive prefix
    for (int k = 0;; ++k) {
      const int s = k % kCompressStages;
      const WaitResult w = mbar_wait_or_abort(smem_addr(&sh.agg[s]), (k / kCompressStages) & 1, &sh.abort);
      if (w != kWaitDone) {
        fail(w);
        return;
      }
      const int64_t t = sh.tile[s];
      if (t < 0) return;
      const uint32_t aggregate = sh.aggregate[s];
      uint32_t prefix = 0;
      if (t > 0) {
        if (!lookback_prefix<kLookBackPerLane>(tile_state, t, lane, prefix) && lane == 0)
          set_error(ws_err, ZF_DEVERR_TIMEOUT);
        if (lane == 0) st_relaxed_u64(&tile_state[t], kStateInclusive | (prefix + aggregate));
      }
      if (lane == 0) {
        sh.prefix[s] = prefix;
        if (!kPaged && t == n_tiles - 1) offs[n_blocks] = prefix + aggregate;
        mbar_arrive(smem_addr(&sh.pre[s]));
      }
      __syncwarp();
    }
  }

  // ---- compute warps: analyse fill k, then write fill k - kWriteLag
  auto write_fill = [&](int k) {
    const int s = k % kCompressStages;
    const WaitResult w = mbar_wait_or_abort(smem_addr(&sh.pre[s]), (k / kCompressStages) & 1, &sh.abort);
    if (w != kWaitDone) {
      fail(w);
      return;
    }
    const int64_t warp_first = sh.tile[s] * kTileBlocks + warp * 32;
    write_group<kPaged>(stage_of(s), warp, lane, warp_first, n_blocks, sh.prefix[s] + sh.warp_excl[s][warp],
                        sh.warp_word[s][warp], &sh.blk_base[s][warp * 32], payload, offs, base, elig, chunk_tab);
    __syncwarp();
    if (lane == 0) mbar_arrive(smem_addr(&sh.empty[s]));
  };
  for (int k = 0;; ++k) {
    const int s = k % kCompressStages;
    const uint32_t parity = (k / kCompressStages) & 1;
    bool more = false;
    const WaitResult w = mbar_wait_or_abort(smem_addr(&sh.full[s]), parity, &sh.abort);
    if (w == kWaitDone) {
      const int64_t t = sh.tile[s];
      if (t >= 0) {
        more = true;
        const int64_t warp_first = t * kTileBlocks + warp * 32;
        uint32_t el_r[4], base_r[4];
        block_stats(stage_of(s), warp, lane, warp_first, n_blocks, el_r, base_r);
        // the group's eligibility word: block 8r + sub's bit from lane 4 sub
        // of round r's ballot; its base from the same lane
        uint32_t word = 0;
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          word |= every_fourth_bit(__ballot_sync(kFull, el_r[r] != 0)) << (8 * r);
          if ((lane & 3) == 0) sh.blk_base[s][warp * 32 + 8 * r + (lane >> 2)] = static_cast<uint8_t>(base_r[r]);
        }
        const uint32_t units = 8u * blocks_in_group(n_blocks, warp_first) - 2u * __popc(word);
        if (lane == 0) {
          sh.warp_word[s][warp] = word;
          sh.warp_units[s][warp] = units;
          mbar_arrive(smem_addr(&sh.units[s]));
        }
        if (warp == 0) {
          // the tile's scan over its warps, then publish the tile size
          const WaitResult wu = mbar_wait_or_abort(smem_addr(&sh.units[s]), parity, &sh.abort);
          if (wu == kWaitDone) {
            uint32_t v = lane < kCompressWarps ? sh.warp_units[s][lane] : 0u;
            const uint32_t own = v;
#pragma unroll
            for (int d = 1; d < kCompressWarps; d <<= 1) {
              const uint32_t y = __shfl_up_sync(kFull, v, d);
              if (lane >= d) v += y;
            }
            if (lane < kCompressWarps) sh.warp_excl[s][lane] = v - own;
            const uint32_t aggregate = __shfl_sync(kFull, v, kCompressWarps - 1);
            __syncwarp();
            if (lane == 0) {
              sh.aggregate[s] = aggregate;
              st_relaxed_u64(&tile_state[t], (t == 0 ? kStateInclusive : kStateAggregate) | aggregate);
              mbar_arrive(smem_addr(&sh.agg[s]));
            }
          } else {
            fail(wu);
          }
        }
      } else if (warp == 0 && lane == 0) {
        mbar_arrive(smem_addr(&sh.agg[s]));  // no more tiles: the look-back warp stops
      }
    } else {
      fail(w);
    }
    if (k >= kWriteLag) write_fill(k - kWriteLag);
    if (!more) {
      for (int j = k - kWriteLag + 1 > 0 ? k - kWriteLag + 1 : 0; j < k; ++j) write_fill(j);
      break;
    }
  }
}

__global__ void __launch_bounds__(256)
    decompress_kernel(const uint8_t* __restrict__ payload, int64_t cap_units, const uint32_t* __restrict__ offs,
                      const uint8_t* __restrict__ base, const uint32_t* __restrict__ elig, int64_t n_blocks,
                      uint16_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int q = lane & 3;
  const int sub = lane >> 2;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t b8 = warp_id * 8; b8 < n_blocks; b8 += n_warps * 8) {
    const int64_t blk = b8 + sub;
    if (blk >= n_blocks) continue;
    const uint32_t unit = __ldg(offs + blk);
    const uint32_t el = (__ldg(elig + (blk >> 5)) >> (blk & 31)) & 1u;
    // a block whose payload would pass the end of the buffer is skipped
    if (static_cast<int64_t>(unit) + (el ? 6 : 8) > cap_units) continue;
    const uint8_t* p = payload + static_cast<uint64_t>(unit) * kUnitBytes;
    // Both kinds of block: sign/mantissa plane, then the exponents (eligible:
    // base + 4-bit offset from the nibble plane; raw: the exponent plane).
    const uint4 sm = __ldg(reinterpret_cast<const uint4*>(p + 16 * q));
    const uint4 ex = __ldg(reinterpret_cast<const uint4*>(p + 64 + 16 * (el ? (q & 1) : q)));
    const uint32_t shift = (el && q >= 2) ? 4u : 0u;
    const uint32_t mask = el ? 0x0F0F0F0Fu : 0xFFFFFFFFu;
    const uint32_t b4 = el ? splat_byte(__ldg(base + blk)) : 0u;
    const uint32_t smv[4] = {sm.x, sm.y, sm.z, sm.w};
    const uint32_t exv[4] = {ex.x, ex.y, ex.z, ex.w};
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t e4 = ((exv[k] >> shift) & mask) + b4;
      w[2 * k] = rebuild_pair(smv[k], e4, 0x5140);
      w[2 * k + 1] = rebuild_pair(smv[k], e4, 0x7362);
    }
    uint4* d = reinterpret_cast<uint4*>(dst + blk * kBlockValues + 16 * q);
    __stcs(d, make_uint4(w[0], w[1], w[2], w[3]));
    __stcs(d + 1, make_uint4(w[4], w[5], w[6], w[7]));
  }
}

// Decompress the paged form: block blk = 32 c + i of chunk c sits in the
// chunk's extent after the 48-byte header and the blocks before it.  A chunk
// whose largest possible extent would pass the end of data is skipped (its
// values in dst are left as they were).
__global__ void __launch_bounds__(256)
    decompress_paged_kernel(const uint8_t* __restrict__ data, int64_t cap_units,
                            const uint32_t* __restrict__ chunk_tab, int64_t n_blocks, uint16_t* __restrict__ dst) {
  const int lane = threadIdx.x & 31;
  const int q = lane & 3;
  const int sub = lane >> 2;
  const int64_t warp_id = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t n_warps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t b8 = warp_id * 8; b8 < n_blocks; b8 += n_warps * 8) {
    const int64_t blk = b8 + sub;
    if (blk >= n_blocks) continue;
    const int64_t c = blk >> 5;
    const uint32_t i = static_cast<uint32_t>(blk & 31);
    const uint32_t start = __ldg(chunk_tab + 2 * c);
    if (int64_t(start) + (kChunkHeaderBytes + 2 * kChunkValues) / kUnitBytes > cap_units) continue;
    const uint8_t* hdr = data + static_cast<uint64_t>(start) * kUnitBytes;
    const uint32_t mask = __ldg(reinterpret_cast<const uint32_t*>(hdr + 32));
    const uint32_t el = (mask >> i) & 1u;
    const uint32_t below = i ? (mask & ((1u << i) - 1u)) : 0u;
    const uint8_t* p = hdr + 48 + 128u * i - 32u * __popc(below);
    const uint4 sm = __ldg(reinterpret_cast<const uint4*>(p + 16 * q));
    const uint4 ex = __ldg(reinterpret_cast<const uint4*>(p + 64 + 16 * (el ? (q & 1) : q)));
    const uint32_t shift = (el && q >= 2) ? 4u : 0u;
    const uint32_t msk = el ? 0x0F0F0F0Fu : 0xFFFFFFFFu;
    const uint32_t b4 = el ? splat_byte(__ldg(hdr + i)) : 0u;
    const uint32_t smv[4] = {sm.x, sm.y, sm.z, sm.w};
    const uint32_t exv[4] = {ex.x, ex.y, ex.z, ex.w};
    uint32_t w[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t e4 = ((exv[k] >> shift) & msk) + b4;
      w[2 * k] = rebuild_pair(smv[k], e4, 0x5140);
      w[2 * k + 1] = rebuild_pair(smv[k], e4, 0x7362);
    }
    uint4* d = reinterpret_cast<uint4*>(dst + blk * kBlockValues + 16 * q);
    __stcs(d, make_uint4(w[0], w[1], w[2], w[3]));
    __stcs(d + 1, make_uint4(w[4], w[5], w[6], w[7]));
  }
}

__global__ void __launch_bounds__(256)
    validate_kernel(const uint8_t* __restrict__ payload, const uint32_t* __restrict__ offs,
                    const uint8_t* __restrict__ base, const uint32_t* __restrict__ elig, int64_t n_blocks,
                    int64_t cap_units, int32_t* bad_count) {
  __shared__ int32_t s_bad;
  if (threadIdx.x == 0) s_bad = 0;
  __syncthreads();
  int32_t bad = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_blocks; i += stride) {
    const uint32_t u0 = offs[i], u1 = offs[i + 1];
    const uint32_t el = (elig[i >> 5] >> (i & 31)) & 1u;
    bool ok = u1 >= u0 && (u1 - u0) == (el ? 6u : 8u) && static_cast<int64_t>(u1) <= cap_units;
    if (ok && el) {
      const uint4* nb = reinterpret_cast<const uint4*>(payload + static_cast<uint64_t>(u0) * kUnitBytes + 64);
      uint32_t mx = 0;
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const uint4 v = nb[k];
        const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          mx = __vmaxu4(mx, w[j] & 0x0F0F0F0Fu);
          mx = __vmaxu4(mx, (w[j] >> 4) & 0x0F0F0F0Fu);
        }
      }
      mx = max(max(mx & 0xFF, (mx >> 8) & 0xFF), max((mx >> 16) & 0xFF, mx >> 24));
      ok = base[i] + mx <= 255u;
    }
    bad += ok ? 0 : 1;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0 && offs[0] != 0) bad += 1;
  if (bad) atomicAdd(&s_bad, bad);
  __syncthreads();
  if (threadIdx.x == 0 && s_bad) atomicAdd(bad_count, s_bad);
}

// One persistent CTA per SM (fewer for small inputs); tiles are taken in
// order from the counter in the workspace.
cudaError_t launch_compress_kernel(bool paged, const uint16_t* src, int64_t n_blocks, uint8_t* payload,
                                   uint32_t* offs, uint8_t* base, uint32_t* elig, uint32_t* chunk_tab, uint8_t* ws,
                                   cudaStream_t s) {
  const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  uint32_t* err = reinterpret_cast<uint32_t*>(ws);
  uint32_t* counter = reinterpret_cast<uint32_t*>(ws + 4);
  uint64_t* state = reinterpret_cast<uint64_t*>(ws + kCompressStateOffset);
  const int sms = current_sm_count();
  if (sms <= 0) return cudaErrorInvalidDevice;
  const unsigned grid = static_cast<unsigned>(n_tiles < sms ? n_tiles : sms);  // one persistent CTA per SM
  auto kern = paged ? compress_kernel<true> : compress_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(kCompressSmem));
  if (e != cudaSuccess) return e;
  kern<<<grid, kCompressThreads, kCompressSmem, s>>>(src, n_blocks, payload, offs, base, elig, chunk_tab, err,
                                                     counter, state, -1);
  return cudaGetLastError();
}

// ---- The compress kernel's own waits, made to run out (zf_check_bounded_wait,
// ZF_WAITCHECK_COMPRESS_STALL): 4 tiles of zeros in the library's own device
// memory, compressed with CTA 0's first stage fill withheld.
constexpr size_t up256(size_t x) { return (x + 255) / 256 * 256; }
constexpr int kStallTiles = 4;
constexpr int64_t kStallBlocks = int64_t(kStallTiles) * kTileBlocks;
constexpr size_t kStallSrc = 0;
constexpr size_t kStallPayload = kStallSrc + size_t(kStallBlocks) * kBlockValues * 2;
constexpr size_t kStallOffs = kStallPayload + size_t(kStallBlocks) * kBlockValues * 2;
constexpr size_t kStallBase = kStallOffs + up256(size_t(kStallBlocks + 1) * 4);
constexpr size_t kStallElig = kStallBase + up256(size_t(kStallBlocks));
constexpr size_t kStallWs = kStallElig + up256(size_t(kStallBlocks / 32) * 4);
constexpr size_t kStallBytes = kStallWs + kCompressStateOffset + size_t(kStallTiles) * 8;
__device__ __align__(256) uint8_t g_stall_check[kStallBytes];

__global__ void stall_check_start(int64_t* result) {
  result[0] = 0;
  result[1] = static_cast<int64_t>(global_timer_ns());
}

__global__ void stall_check_end(int64_t* result, const uint32_t* err) {
  result[1] = static_cast<int64_t>(global_timer_ns()) - result[1];
  result[0] = (*err & ZF_DEVERR_TIMEOUT) ? -1 : 1;
}

}  // namespace

zf_status compress_stall_check(int64_t* result, uint32_t* err, cudaStream_t s) {
  void* base = nullptr;
  if (cudaGetSymbolAddress(&base, g_stall_check) != cudaSuccess) return ZF_ERR_CUDA;
  uint8_t* b = static_cast<uint8_t*>(base);
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  auto kern = compress_kernel<false>;
  if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kCompressSmem)) !=
      cudaSuccess)
    return ZF_ERR_CUDA;
  if (cudaMemsetAsync(b + kStallWs, 0, kCompressStateOffset + size_t(kStallTiles) * 8, s) != cudaSuccess)
    return ZF_ERR_CUDA;
  stall_check_start<<<1, 1, 0, s>>>(result);
  const unsigned grid = static_cast<unsigned>(kStallTiles < sms ? kStallTiles : sms);
  kern<<<grid, kCompressThreads, kCompressSmem, s>>>(
      reinterpret_cast<const uint16_t*>(b + kStallSrc), kStallBlocks, b + kStallPayload,
      reinterpret_cast<uint32_t*>(b + kStallOffs), b + kStallBase, reinterpret_cast<uint32_t*>(b + kStallElig),
      nullptr, err, reinterpret_cast<uint32_t*>(b + kStallWs + 4),
      reinterpret_cast<uint64_t*>(b + kStallWs + kCompressStateOffset), 0);
  stall_check_end<<<1, 1, 0, s>>>(result, err);
  return cuda_status(cudaGetLastError());
}

namespace {

bool valid_compressed_desc(const zf_kv_compressed* c) {
  return c && c->payload && c->offs && c->base && c->elig && c->n_values >= 0 &&
         c->n_values % kBlockValues == 0 && c->payload_cap_bytes >= 0 && aligned(c->payload, 16) &&
         aligned(c->offs, 4) && aligned(c->base, 16) && aligned(c->elig, 4);
}

}  // namespace
}  // namespace zf

using namespace zf;

extern "C" {

size_t zf_compressed_bound(int64_t n_values) {
  if (n_values < 0 || n_values % kBlockValues) return 0;
  return static_cast<size_t>(n_values) * 2;
}

size_t zf_compress_workspace_size(int64_t n_values) {
  if (n_values < 0 || n_values % kBlockValues) return 0;
  const int64_t n_blocks = n_values / kBlockValues;
  const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  return kCompressStateOffset + static_cast<size_t>(n_tiles) * 8;
}

zf_status zf_compress_kv(const uint16_t* src, int64_t n_values, const zf_kv_compressed* dst, void* ws,
                         size_t ws_bytes, zf_stream_t stream) {
  if (!valid_compressed_desc(dst) || n_values < 0 || n_values % kBlockValues || dst->n_values != n_values)
    return ZF_ERR_INVALID_ARG;
  if (n_values > 0 && (!src || !aligned(src, 16) || !ws || !aligned(ws, 16))) return ZF_ERR_INVALID_ARG;
  if (static_cast<size_t>(dst->payload_cap_bytes) < zf_compressed_bound(n_values)) return ZF_ERR_WORKSPACE;
  if (n_values / kBlockValues > (int64_t(1) << 28)) return ZF_ERR_UNSUPPORTED;  // u32 offsets
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n_blocks = n_values / kBlockValues;
  if (n_blocks == 0) {
    return cuda_status(cudaMemsetAsync(dst->offs, 0, sizeof(uint32_t), s));
  }
  if (ws_bytes < zf_compress_workspace_size(n_values)) return ZF_ERR_WORKSPACE;
  const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  if (n_tiles > 0x7FFFFFFF) return ZF_ERR_UNSUPPORTED;
  cudaError_t e = cudaMemsetAsync(ws, 0, zf_compress_workspace_size(n_values), s);
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  return cuda_status(launch_compress_kernel(false, src, n_blocks, static_cast<uint8_t*>(dst->payload), dst->offs, dst->base,
                                            dst->elig, nullptr, static_cast<uint8_t*>(ws), s));
}

zf_status zf_decompress_kv(const zf_kv_compressed* src, uint16_t* dst, zf_stream_t stream) {
  if (!valid_compressed_desc(src)) return ZF_ERR_INVALID_ARG;
  const int64_t n_blocks = src->n_values / kBlockValues;
  if (n_blocks == 0) return ZF_OK;
  if (!dst || !aligned(dst, 16)) return ZF_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const int64_t want = (n_blocks + 63) / 64;
  const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  decompress_kernel<<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(src->payload),
                                         src->payload_cap_bytes / kUnitBytes, src->offs, src->base, src->elig,
                                         n_blocks, dst);
  return cuda_status(cudaGetLastError());
}

zf_status zf_validate_compressed(const zf_kv_compressed* c, int32_t* d_bad_count, zf_stream_t stream) {
  if (!valid_compressed_desc(c) || !d_bad_count) return ZF_ERR_INVALID_ARG;
  const int64_t n_blocks = c->n_values / kBlockValues;
  if (n_blocks == 0) return ZF_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const int64_t want = (n_blocks + 255) / 256;
  const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  validate_kernel<<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(c->payload), c->offs, c->base, c->elig,
                                       n_blocks, c->payload_cap_bytes / kUnitBytes, d_bad_count);
  return cuda_status(cudaGetLastError());
}

size_t zf_paged_bound(int64_t num_chunks) {
  if (num_chunks < 0) return 0;
  return static_cast<size_t>(num_chunks) * (kChunkHeaderBytes + 2 * kChunkValues);
}

zf_status zf_compress_paged(const uint16_t* src, int64_t num_chunks, const zf_kv_paged* dst, void* ws,
                            size_t ws_bytes, zf_stream_t stream) {
  if (!dst || !dst->data || !dst->chunk_tab || dst->num_chunks != num_chunks || num_chunks < 0 ||
      !aligned(dst->data, 16) || !aligned(dst->chunk_tab, 8))
    return ZF_ERR_INVALID_ARG;
  const int64_t n_values = num_chunks * kChunkValues;
  if (num_chunks == 0) return ZF_OK;
  if (!src || !aligned(src, 16) || !ws || !aligned(ws, 16)) return ZF_ERR_INVALID_ARG;
  if (dst->data_cap_bytes < 0 || static_cast<size_t>(dst->data_cap_bytes) < zf_paged_bound(num_chunks))
    return ZF_ERR_WORKSPACE;
  if (zf_paged_bound(num_chunks) / kUnitBytes > 0xFFFFFFFFull) return ZF_ERR_UNSUPPORTED;  // u32 units
  if (ws_bytes < zf_compress_workspace_size(n_values)) return ZF_ERR_WORKSPACE;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int64_t n_blocks = n_values / kBlockValues;
  const int64_t n_tiles = (n_blocks + kTileBlocks - 1) / kTileBlocks;
  if (n_tiles > 0x7FFFFFFF) return ZF_ERR_UNSUPPORTED;
  cudaError_t e = cudaMemsetAsync(ws, 0, zf_compress_workspace_size(n_values), s);
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  return cuda_status(launch_compress_kernel(true, src, n_blocks, static_cast<uint8_t*>(dst->data), nullptr, nullptr, nullptr,
                                           dst->chunk_tab, static_cast<uint8_t*>(ws), s));
}

zf_status zf_decompress_paged(const zf_kv_paged* src, uint16_t* dst, zf_stream_t stream) {
  if (!src || !src->data || !src->chunk_tab || src->num_chunks < 0 || src->data_cap_bytes < 0 ||
      !aligned(src->data, 16) || !aligned(src->chunk_tab, 8))
    return ZF_ERR_INVALID_ARG;
  const int64_t n_blocks = src->num_chunks * kChunkBlocks;
  if (n_blocks == 0) return ZF_OK;
  if (!dst || !aligned(dst, 16)) return ZF_ERR_INVALID_ARG;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const int64_t want = (n_blocks + 63) / 64;
  const unsigned grid = static_cast<unsigned>(want < int64_t(sms) * 8 ? want : int64_t(sms) * 8);
  decompress_paged_kernel<<<grid, 256, 0, s>>>(static_cast<const uint8_t*>(src->data),
                                               src->data_cap_bytes / kUnitBytes, src->chunk_tab, n_blocks, dst);
  return cuda_status(cudaGetLastError());
}

}  // extern "C"
