// Fused split-K GQA decode attention over a compressed (or raw) paged BF16
// KV cache, for B200 (sm_100a).
//
// Method: "Run AI Faster With Lossless Compressed Memory" (ZipFusion summary),
// chapters "Why Memory Sets the Speed" and "Twelve Bits and One Addition":
// the cache stays compressed in HBM, attention reads the compressed bytes and
// rebuilds every K/V value in registers with one integer addition, so decode
// moves ~25% fewer bytes than a raw BF16 cache.
//
// Design (B200-first):
//  * Persistent grid, 2 CTAs per SM.  All work is the list of (sequence, kv
//    head, page) items in sequence-major order; CTA i takes the contiguous
//    share [i*W/G, (i+1)*W/G), so every CTA moves the same number of pages
//    whatever the length mix.  The split points come from seq_lens on the
//    device (each CTA scans them into shared memory), so no host round trip.
//  * One producer warp streams each page's K and V chunks (variable-size
//    compressed extents, base exponents) into an 8-stage shared-memory ring
//    with 1-D bulk (TMA) copies completed on mbarriers.  Page ids and chunk
//    metadata for the next 32 pages are fetched one batch ahead by the 32
//    lanes of the producer warp.
//  * Four consumer warps take pages round-robin.  Per page (16 tokens) a warp
//    rebuilds K and V straight into mma.sync m16n8k16 operand registers:
//    S^T = Q K^T puts the query heads of the GQA group on M and tokens on N,
//    so the S accumulator is already the B operand of O^T = V^T P^T.  P is fed
//    as a bf16 hi + lo pair (two mma), which keeps P to ~16 bits of precision.
//  * Online softmax in base 2 (scale * log2 e folded into one FMA); the
//    running max is reduced over the 4 lanes that hold one head's tokens.
//  * At the end of each (sequence, kv head) piece the consumer warps merge
//    their states through shared memory in a fixed order.  A CTA that covers
//    a whole sequence/head writes the output directly; otherwise it writes a
//    partial (m, l, acc[128]) slot and a second kernel merges the slots.
//  * The raw-BF16 twin is the same template with the decode step replaced by
//    plain loads: same plan, same arithmetic, same order, so its output is
//    bitwise identical to the compressed kernel's.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>

#include "zf_device.cuh"
#include "zf_internal.h"

namespace zf {
namespace {

#ifndef ZF_CONSUMER_WARPS
#define ZF_CONSUMER_WARPS 4
#endif
#ifndef ZF_STAGES
#define ZF_STAGES 8
#endif
#ifndef ZF_CTAS_PER_SM
#define ZF_CTAS_PER_SM 2
#endif
constexpr int kConsumerWarps = ZF_CONSUMER_WARPS;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = ZF_STAGES;
constexpr int kCtasPerSm = ZF_CTAS_PER_SM;
// Page j lives in stage j % kStages and is consumed by warp j % kConsumerWarps.
// Every stage must always belong to the same consumer warp: a warp then never
// waits on a stage more than one barrier phase ahead of it, which the parity
// waits need (two phases ahead would alias).
static_assert(kStages % kConsumerWarps == 0, "each ring stage must map to one consumer warp");
constexpr int kChunkBytes = kChunkValues * 2;  // 4096 raw bytes per (page, head)
// Stage layout: K payload | V payload | K bases | V bases | header
constexpr int kStageK = 0;
constexpr int kStageV = kChunkBytes;
constexpr int kStageKBase = 2 * kChunkBytes;
constexpr int kStageVBase = kStageKBase + 32;
constexpr int kStageHdr = kStageVBase + 32;
constexpr int kStageBytes = kStageHdr + 128;  // 8384: every stage starts 16-byte aligned
constexpr int kPartStride = 132;              // floats per (slot, head): m, l, pad, pad, acc[128]
constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xFFFFFFFFu;

struct DecodeParams {
  const uint16_t* q;
  // compressed pools
  const uint8_t* k_payload;
  const uint32_t* k_offs;
  const uint8_t* k_base;
  const uint32_t* k_elig;
  int64_t k_cap_units;
  const uint8_t* v_payload;
  const uint32_t* v_offs;
  const uint8_t* v_base;
  const uint32_t* v_elig;
  int64_t v_cap_units;
  // raw pools
  const uint16_t* k_pool;
  const uint16_t* v_pool;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint16_t* out;
  float* lse;
  float* part;
  int32_t* plan;
  uint32_t* err;
  int num_pages;
  int max_pages;
  int B;
  int Hq;
  int Hkv;
  int group;
  float sm_scale;
  float scale_log2;  // sm_scale * log2(e)
};

// Shared-memory layout after the stage ring.
struct SmemTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  float red_m[kConsumerWarps][kMaxGroup];
  float red_l[kConsumerWarps][kMaxGroup];
  int32_t abort_flag;
  int32_t pad[3];
};

__host__ __device__ constexpr size_t smem_fixed_bytes() {
  return size_t(kStages) * kStageBytes + sizeof(SmemTail) +
         size_t(kConsumerWarps) * kMaxGroup * kHeadDim * sizeof(float);
}
__host__ __device__ inline size_t smem_bytes(int B) {
  return smem_fixed_bytes() + size_t(2 * B + 2) * sizeof(int32_t);
}

// Largest CTA index whose range [i*W/G, (i+1)*W/G) starts at or before x.
__device__ __forceinline__ int64_t cta_of(int64_t x, int64_t W, int64_t G) {
  return ((x + 1) * G + W - 1) / W - 1;
}

struct Piece {
  int b, h;
  int64_t page0;   // first page of the piece within the sequence
  int64_t npages;  // pages in the piece
  int64_t n_b;     // pages of the whole sequence
  bool whole;      // the piece is the whole (sequence, kv head) segment
};

// Locate linear work index x (sequence-major, then kv head, then page).
__device__ __forceinline__ void locate(const int32_t* s_pfx, int B, int Hkv, int64_t x, int& b, int& h,
                                       int64_t& page, int64_t& n_b) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {  // largest b with pfx[b] * Hkv <= x
    const int mid = (lo + hi + 1) >> 1;
    if (int64_t(s_pfx[mid]) * Hkv <= x) lo = mid; else hi = mid - 1;
  }
  b = lo;
  n_b = s_pfx[b + 1] - s_pfx[b];
  const int64_t rem = x - int64_t(s_pfx[b]) * Hkv;  // < Hkv * n_b
  if (rem < (int64_t(1) << 32) && n_b < (int64_t(1) << 32)) {
    const uint32_t hh = static_cast<uint32_t>(rem) / static_cast<uint32_t>(n_b);
    h = static_cast<int>(hh);
  } else {
    h = static_cast<int>(rem / n_b);
  }
  page = rem - int64_t(h) * n_b;
}


// ------------------------------------------------------------------ kernel

template <bool kCompressed>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_attn_kernel(const DecodeParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  SmemTail& tail = *reinterpret_cast<SmemTail*>(smem + size_t(kStages) * kStageBytes);
  float* red_acc = reinterpret_cast<float*>(smem + size_t(kStages) * kStageBytes + sizeof(SmemTail));
  int32_t* s_pfx = reinterpret_cast<int32_t*>(red_acc + kConsumerWarps * kMaxGroup * kHeadDim);
  int32_t* s_len = s_pfx + p.B + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int B = p.B;
  const int Hkv = p.Hkv;
  const int group = p.group;
  const int max_tokens = p.max_pages * kPageTokens;

  // Inputs may come from the previous kernel in the stream (q, the cache
  // append): wait for it before reading anything, then let the next kernel
  // (the split merge) start launching.
  grid_dependency_wait();
  launch_dependents();

  // ---- plan: clamped lengths and page prefix sums (warp 0), barriers (thread 0)
  if (warp == 0) {
    const int per = (B + 31) / 32;
    const int b0 = lane * per;
    int32_t run = 0;
    for (int i = 0; i < per; ++i) {
      const int b = b0 + i;
      if (b < B) {
        int32_t len = __ldg(p.seq_lens + b);
        if (len < 0 || len > max_tokens) {
          set_error(p.err, ZF_DEVERR_SEQ_LEN);
          len = len < 0 ? 0 : max_tokens;
        }
        s_len[b] = len;
        run += (len + kPageTokens - 1) / kPageTokens;
      }
    }
    int32_t incl = run;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const int32_t t = __shfl_up_sync(kFull, incl, d);
      if (lane >= d) incl += t;
    }
    int32_t acc = incl - run;
    for (int i = 0; i < per; ++i) {
      const int b = b0 + i;
      if (b < B) {
        s_pfx[b] = acc;
        acc += (s_len[b] + kPageTokens - 1) / kPageTokens;
      }
    }
    if (lane == 31) s_pfx[B] = incl;
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&tail.full[s]), 1);
      mbar_init(smem_addr(&tail.empty[s]), 1);
    }
    tail.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int i = threadIdx.x; i <= B; i += blockDim.x) p.plan[i] = s_pfx[i];
  }

  const int64_t G = gridDim.x;
  const int64_t W = int64_t(s_pfx[B]) * Hkv;
  const int64_t lo = W * blockIdx.x / G;
  const int64_t hi = W * (blockIdx.x + 1) / G;
  const int64_t n_items = hi - lo;

  if (warp == kConsumerWarps) {
    // =========================== producer warp ===========================
    // Three-step software pipeline over batches of 32 pages (one per lane):
    //   A: locate the page and load its id      (two batches ahead)
    //   B: load the chunk's offset / mask words  (one batch ahead)
    //   C: lane 0 issues the bulk copies, in page order
    struct StepA { int64_t h; int32_t pid; bool valid; };
    struct StepB { int64_t chunk; uint32_t ku, vu, ke, ve; bool valid; };
    auto step_a = [&](int64_t j) {
      StepA a{0, 0, j < n_items};
      if (a.valid) {
        int b, h;
        int64_t page, n_b;
        locate(s_pfx, B, Hkv, lo + j, b, h, page, n_b);
        a.h = h;
        a.pid = __ldg(p.page_table + int64_t(b) * p.max_pages + page);
      }
      return a;
    };
    auto step_b = [&](const StepA& a) {
      StepB m{0, 0, 0, 0, 0, a.valid};
      if (a.valid) {
        int32_t pid = a.pid;
        if (pid < 0 || pid >= p.num_pages) {
          set_error(p.err, ZF_DEVERR_PAGE_ID);
          pid = 0;
        }
        m.chunk = int64_t(pid) * Hkv + a.h;
        if constexpr (kCompressed) {
          m.ku = __ldg(p.k_offs + m.chunk * kChunkBlocks);
          m.vu = __ldg(p.v_offs + m.chunk * kChunkBlocks);
          m.ke = __ldg(p.k_elig + m.chunk);
          m.ve = __ldg(p.v_elig + m.chunk);
        }
      }
      return m;
    };

    // Lane i < kStages owns ring stage i and issues the copies of every page
    // j with j % kStages == i, in order; the kStages lanes work in parallel.
    static_assert(kStages <= 32, "one producer lane per stage");
    int64_t my_last = -1;  // last page this lane issued
    auto issue = [&](int64_t j, int64_t chunk, uint32_t ku, uint32_t vu, uint32_t ke, uint32_t ve) {
      const int s = lane;
      const uint32_t parity = static_cast<uint32_t>((j / kStages) & 1) ^ 1u;
      if (!mbar_wait_bounded(smem_addr(&tail.empty[s]), parity)) {
        set_error(p.err, ZF_DEVERR_TIMEOUT);
        atomicExch(&tail.abort_flag, 1);
        return;
      }
      // The consumer's reads of this stage's previous page (ordered before
      // us by the empty barrier) must precede the bulk copies' writes.
      fence_proxy_async_smem();
      uint8_t* st = smem + size_t(s) * kStageBytes;
      const uint32_t full = smem_addr(&tail.full[s]);
      const uint8_t* ksrc;
      const uint8_t* vsrc;
      uint32_t kb, vb;
      if constexpr (kCompressed) {
        const uint32_t k_units = 8u * kChunkBlocks - 2u * __popc(ke);
        const uint32_t v_units = 8u * kChunkBlocks - 2u * __popc(ve);
        kb = k_units * kUnitBytes;
        vb = v_units * kUnitBytes;
        if (int64_t(ku) + k_units > p.k_cap_units) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          kb = 0;
        }
        if (int64_t(vu) + v_units > p.v_cap_units) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          vb = 0;
        }
        ksrc = p.k_payload + uint64_t(ku) * kUnitBytes;
        vsrc = p.v_payload + uint64_t(vu) * kUnitBytes;
        reinterpret_cast<uint32_t*>(st + kStageHdr)[0] = ke;
        reinterpret_cast<uint32_t*>(st + kStageHdr)[1] = ve;
      } else {
        ksrc = reinterpret_cast<const uint8_t*>(p.k_pool + chunk * kChunkValues);
        vsrc = reinterpret_cast<const uint8_t*>(p.v_pool + chunk * kChunkValues);
        kb = vb = kChunkBytes;
      }
      mbar_arrive_expect_tx(full, kb + vb + (kCompressed ? 64u : 0u));
      if (kb) bulk_copy_g2s(smem_addr(st + kStageK), ksrc, kb, full);
      if (vb) bulk_copy_g2s(smem_addr(st + kStageV), vsrc, vb, full);
      if constexpr (kCompressed) {
        bulk_copy_g2s(smem_addr(st + kStageKBase), p.k_base + chunk * kChunkBlocks, 32, full);
        bulk_copy_g2s(smem_addr(st + kStageVBase), p.v_base + chunk * kChunkBlocks, 32, full);
      }
      my_last = j;
    };

    StepB cur = step_b(step_a(lane));
    StepA ahead = step_a(32 + lane);
    for (int64_t j0 = 0; j0 < n_items; j0 += 32) {
      const StepA ahead2 = step_a(j0 + 64 + lane);
      const StepB nxt = step_b(ahead);
      const int count = static_cast<int>(n_items - j0 < 32 ? n_items - j0 : 32);
      const int jm = static_cast<int>(j0 % kStages);
      const int l0 = ((lane - jm) % kStages + kStages) % kStages;  // first batch slot of my stage
      for (int r = 0; r * kStages < 32; ++r) {
        const int l = l0 + r * kStages;
        const int src = l < 32 ? l : 0;
        const int64_t chunk = __shfl_sync(kFull, cur.chunk, src);
        uint32_t ku = 0, vu = 0, ke = 0, ve = 0;
        if constexpr (kCompressed) {
          ku = __shfl_sync(kFull, cur.ku, src);
          vu = __shfl_sync(kFull, cur.vu, src);
          ke = __shfl_sync(kFull, cur.ke, src);
          ve = __shfl_sync(kFull, cur.ve, src);
        }
        if (lane < kStages && l < count && !*reinterpret_cast<volatile int32_t*>(&tail.abort_flag))
          issue(j0 + l, chunk, ku, vu, ke, ve);
        __syncwarp();
      }
      cur = nxt;
      ahead = ahead2;
    }
    // Copies still in flight must land before the CTA may exit; in normal
    // operation the consumers have waited for all of them already.
    if (lane < kStages && my_last >= 0 && *reinterpret_cast<volatile int32_t*>(&tail.abort_flag))
      mbar_wait_bounded(smem_addr(&tail.full[lane]), static_cast<uint32_t>((my_last / kStages) & 1));
  } else {
    // =========================== consumer warps ==========================
    const int g = lane >> 2;  // mma group: query head (rows) / token (cols)
    const int c = lane & 3;   // thread in group
    const float sl = p.scale_log2;
    int64_t x = lo;
    int64_t j_base = 0;  // CTA-local index of the piece's first page
    while (x < hi) {
      Piece pc;
      {
        int64_t page, n_b;
        locate(s_pfx, B, Hkv, x, pc.b, pc.h, page, n_b);
        const int64_t seg_start = int64_t(s_pfx[pc.b]) * Hkv + int64_t(pc.h) * n_b;
        const int64_t seg_end = seg_start + n_b;
        const int64_t end = seg_end < hi ? seg_end : hi;
        pc.page0 = page;
        pc.npages = end - x;
        pc.n_b = n_b;
        pc.whole = (x == seg_start) && (end == seg_end);
      }
      const int seq_len = s_len[pc.b];

      // Q operand (A of S^T = Q K^T): head g, the 32 dims lane c owns:
      // run0 = dims 64*(c>>1) + 16*(c&1) + [0,16), run1 = run0 + 32.
      uint32_t qa[8][2];
      {
        const int hq = pc.h * group + g;
        if (g < group) {
          const uint16_t* qp = p.q + (int64_t(pc.b) * p.Hq + hq) * kHeadDim + 64 * (c >> 1) + 16 * (c & 1);
          const uint4* q4 = reinterpret_cast<const uint4*>(qp);
          const uint4 r0a = __ldg(q4), r0b = __ldg(q4 + 1), r1a = __ldg(q4 + 4), r1b = __ldg(q4 + 5);
          const uint32_t r0[8] = {r0a.x, r0a.y, r0a.z, r0a.w, r0b.x, r0b.y, r0b.z, r0b.w};
          const uint32_t r1[8] = {r1a.x, r1a.y, r1a.z, r1a.w, r1b.x, r1b.y, r1b.z, r1b.w};
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            qa[s][0] = r0[s];
            qa[s][1] = r1[s];
          }
        } else {
#pragma unroll
          for (int s = 0; s < 8; ++s) qa[s][0] = qa[s][1] = 0u;
        }
      }

      float m_run = kNegInf;  // running max of raw scores, head g
      float l_run = 0.f;      // this lane's share of the running sum
      float acc[8][4];        // O^T rows (dims) x cols (heads 2c, 2c+1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = 0.f;

      const int64_t jj0 = (warp - j_base % kConsumerWarps + kConsumerWarps) % kConsumerWarps;
      for (int64_t jj = jj0; jj < pc.npages; jj += kConsumerWarps) {
        const int64_t j = j_base + jj;
        if (*reinterpret_cast<volatile int32_t*>(&tail.abort_flag)) continue;
        const int s = static_cast<int>(j % kStages);
        const uint32_t parity = static_cast<uint32_t>((j / kStages) & 1);
        if (!mbar_wait_bounded(smem_addr(&tail.full[s]), parity)) {
          if (lane == 0) {
            set_error(p.err, ZF_DEVERR_TIMEOUT);
            atomicExch(&tail.abort_flag, 1);
          }
          __syncwarp();
          continue;
        }
        const uint8_t* st = smem + size_t(s) * kStageBytes;
        const int64_t page = pc.page0 + jj;
        const int64_t left = int64_t(seq_len) - page * kPageTokens;
        const int n_valid = left >= kPageTokens ? kPageTokens : static_cast<int>(left);
        const int tk[4] = {2 * c, 2 * c + 1, 8 + 2 * c, 9 + 2 * c};
        const int kk = 8 * (g & 3);

        // ---- 1. copy this lane's share of the page into registers, then
        // hand the stage back to the producer at once.
        // K: tokens g and g+8, half v = c&1 of block 2*tok + (c>>1).
        //   eligible: kw = {nibbles, sign/mantissa lo, sign/mantissa hi}
        //   raw:      kw = 64 bytes (values [16v,16v+16) and [32+16v,+16))
        // V: tokens tk[u], 16 values from block 2*tk[u] + (g>>2).
        //   eligible: vw[0] = {nibbles(8 B), sign/mantissa lo(8 B)}, vw[1].xy = hi
        //   raw:      vw = 32 bytes (values [kk,kk+8) and [32+kk,+8))
        uint4 kw[2][4];
        uint4 vw[4][2];
        uint32_t kbase4[2] = {0u, 0u}, vbase4[4] = {0u, 0u, 0u, 0u};
        bool kel[2] = {false, false}, vel[4] = {false, false, false, false};
        {
          uint32_t ke = 0, ve = 0;
          if constexpr (kCompressed) {
            ke = reinterpret_cast<const uint32_t*>(st + kStageHdr)[0];
            ve = reinterpret_cast<const uint32_t*>(st + kStageHdr)[1];
          }
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const int blk = 2 * (g + 8 * nt) + (c >> 1);
            const int v = c & 1;
            uint32_t off = 128u * blk;
            if constexpr (kCompressed) {
              const uint32_t below = blk ? (ke & ((1u << blk) - 1u)) : 0u;
              off = 16u * (8u * blk - 2u * __popc(below));
              kel[nt] = (ke >> blk) & 1u;
            }
            const uint8_t* bp = st + kStageK + off;
            if (kel[nt]) {
              kw[nt][0] = *reinterpret_cast<const uint4*>(bp + 64 + 16 * v);
              kw[nt][1] = *reinterpret_cast<const uint4*>(bp + 16 * v);
              kw[nt][2] = *reinterpret_cast<const uint4*>(bp + 32 + 16 * v);
              kw[nt][3] = make_uint4(0u, 0u, 0u, 0u);
              kbase4[nt] = splat_byte(st[kStageKBase + blk]);
            } else {
              const uint4* r = reinterpret_cast<const uint4*>(bp + 32 * v);
              kw[nt][0] = r[0];
              kw[nt][1] = r[1];
              kw[nt][2] = r[4];
              kw[nt][3] = r[5];
            }
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int blk = 2 * tk[u] + (g >> 2);
            uint32_t off = 128u * blk;
            if constexpr (kCompressed) {
              const uint32_t below = blk ? (ve & ((1u << blk) - 1u)) : 0u;
              off = 16u * (8u * blk - 2u * __popc(below));
              vel[u] = (ve >> blk) & 1u;
            }
            const uint8_t* bp = st + kStageV + off;
            if (vel[u]) {
              const uint2 nb = *reinterpret_cast<const uint2*>(bp + 64 + kk);
              const uint2 s0 = *reinterpret_cast<const uint2*>(bp + kk);
              const uint2 s1 = *reinterpret_cast<const uint2*>(bp + 32 + kk);
              vw[u][0] = make_uint4(nb.x, nb.y, s0.x, s0.y);
              vw[u][1] = make_uint4(s1.x, s1.y, 0u, 0u);
              vbase4[u] = splat_byte(st[kStageVBase + blk]);
            } else {
              vw[u][0] = *reinterpret_cast<const uint4*>(bp + 2 * kk);
              vw[u][1] = *reinterpret_cast<const uint4*>(bp + 64 + 2 * kk);
            }
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&tail.empty[s]));

        // ---- 2. K -> B operand of S^T = Q K^T (token g and g+8)
        uint32_t kb[2][8][2];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          if (kel[nt]) {
            const uint32_t nbv[4] = {kw[nt][0].x, kw[nt][0].y, kw[nt][0].z, kw[nt][0].w};
            const uint32_t s0v[4] = {kw[nt][1].x, kw[nt][1].y, kw[nt][1].z, kw[nt][1].w};
            const uint32_t s1v[4] = {kw[nt][2].x, kw[nt][2].y, kw[nt][2].z, kw[nt][2].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t elo = exponents4(nbv[w], 0, kbase4[nt]);
              const uint32_t ehi = exponents4(nbv[w], 4, kbase4[nt]);
              kb[nt][2 * w][0] = rebuild_pair(s0v[w], elo, 0x5140);
              kb[nt][2 * w + 1][0] = rebuild_pair(s0v[w], elo, 0x7362);
              kb[nt][2 * w][1] = rebuild_pair(s1v[w], ehi, 0x5140);
              kb[nt][2 * w + 1][1] = rebuild_pair(s1v[w], ehi, 0x7362);
            }
          } else {
            const uint32_t r0[8] = {kw[nt][0].x, kw[nt][0].y, kw[nt][0].z, kw[nt][0].w,
                                    kw[nt][1].x, kw[nt][1].y, kw[nt][1].z, kw[nt][1].w};
            const uint32_t r1[8] = {kw[nt][2].x, kw[nt][2].y, kw[nt][2].z, kw[nt][2].w,
                                    kw[nt][3].x, kw[nt][3].y, kw[nt][3].z, kw[nt][3].w};
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              kb[nt][s2][0] = r0[s2];
              kb[nt][s2][1] = r1[s2];
            }
          }
        }

        // ---- S^T[head g][token] for tokens 2c, 2c+1 (nt 0) and 8+2c, 9+2c (nt 1)
        float sc[2][4];
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
          for (int k = 0; k < 4; ++k) sc[nt][k] = 0.f;
#pragma unroll
          for (int s2 = 0; s2 < 8; ++s2)
            mma_16816(sc[nt], qa[s2][0], 0u, qa[s2][1], 0u, kb[nt][s2][0], kb[nt][s2][1]);
        }
        float sv[4] = {sc[0][0], sc[0][1], sc[1][0], sc[1][1]};
#pragma unroll
        for (int k = 0; k < 4; ++k)
          if (tk[k] >= n_valid) sv[k] = kNegInf;

        // ---- online softmax (base 2), head g over the 4 lanes of group g
        float mx = fmaxf(fmaxf(sv[0], sv[1]), fmaxf(sv[2], sv[3]));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(kFull, mx, 2));
        const float m_new = fmaxf(m_run, mx);
        const float alpha = fast_exp2((m_run - m_new) * sl);
        const float neg = -m_new * sl;
        float pr[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) pr[k] = fast_exp2(fmaf(sv[k], sl, neg));
        l_run = fmaf(l_run, alpha, (pr[0] + pr[1]) + (pr[2] + pr[3]));
        m_run = m_new;
        // P^T as the B operand: hi + lo bf16 parts
        const uint32_t ph0 = pack_bf16x2(pr[0], pr[1]);
        const uint32_t ph1 = pack_bf16x2(pr[2], pr[3]);
        const uint32_t pl0 = pack_bf16x2(pr[0] - bf16_lo_to_f32(ph0), pr[1] - bf16_hi_to_f32(ph0));
        const uint32_t pl1 = pack_bf16x2(pr[2] - bf16_lo_to_f32(ph1), pr[3] - bf16_hi_to_f32(ph1));
        // rescale O^T columns (heads 2c, 2c+1) by their alpha
        const float a_even = __shfl_sync(kFull, alpha, 8 * c);
        const float a_odd = __shfl_sync(kFull, alpha, 8 * c + 4);
        if (__any_sync(kFull, a_even != 1.f || a_odd != 1.f)) {
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            acc[i][0] *= a_even;
            acc[i][1] *= a_odd;
            acc[i][2] *= a_even;
            acc[i][3] *= a_odd;
          }
        }

        // ---- 3. V -> A operand of O^T = V^T P^T: tokens 2c, 2c+1, 2c+8, 2c+9;
        // dims r(i) = 64*(g>>2) + 32*hi + 8*(g&3) + 4*w + 2*t for m-tile
        // i = 4*w + 2*hi + t, rows g and g+8 = dims r(i) and r(i)+1.
        uint32_t xv[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if (vel[u]) {
            const uint32_t nbv[2] = {vw[u][0].x, vw[u][0].y};
            const uint32_t s0v[2] = {vw[u][0].z, vw[u][0].w};
            const uint32_t s1v[2] = {vw[u][1].x, vw[u][1].y};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const uint32_t elo = exponents4(nbv[w], 0, vbase4[u]);
              const uint32_t ehi = exponents4(nbv[w], 4, vbase4[u]);
              xv[u][4 * w + 0] = rebuild_pair(s0v[w], elo, 0x5140);
              xv[u][4 * w + 1] = rebuild_pair(s0v[w], elo, 0x7362);
              xv[u][4 * w + 2] = rebuild_pair(s1v[w], ehi, 0x5140);
              xv[u][4 * w + 3] = rebuild_pair(s1v[w], ehi, 0x7362);
            }
          } else {
            const uint4 r0 = vw[u][0], r1 = vw[u][1];
            xv[u][0] = r0.x; xv[u][1] = r0.y; xv[u][2] = r1.x; xv[u][3] = r1.y;
            xv[u][4] = r0.z; xv[u][5] = r0.w; xv[u][6] = r1.z; xv[u][7] = r1.w;
          }
          if (tk[u] >= n_valid) {
#pragma unroll
            for (int i = 0; i < 8; ++i) xv[u][i] = 0u;
          }
        }

#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t a0 = __byte_perm(xv[0][i], xv[1][i], 0x5410);
          const uint32_t a1 = __byte_perm(xv[0][i], xv[1][i], 0x7632);
          const uint32_t a2 = __byte_perm(xv[2][i], xv[3][i], 0x5410);
          const uint32_t a3 = __byte_perm(xv[2][i], xv[3][i], 0x7632);
          mma_16816(acc[i], a0, a1, a2, a3, ph0, ph1);
          mma_16816(acc[i], a0, a1, a2, a3, pl0, pl1);
        }
      }

      // ---- merge the consumer warps' states for this piece
      float l_row = l_run + __shfl_xor_sync(kFull, l_run, 1);
      l_row = l_row + __shfl_xor_sync(kFull, l_row, 2);
      if (c == 0 && g < group) {
        tail.red_m[warp][g] = m_run;
        tail.red_l[warp][g] = l_row;
      }
      {
        const int kk = 8 * (g & 3);
        float* ra = red_acc + warp * kMaxGroup * kHeadDim;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int w = i >> 2, hi2 = (i >> 1) & 1, t = i & 1;
          const int r = 64 * (g >> 2) + 32 * hi2 + kk + 4 * w + 2 * t;
          if (2 * c < group) {
            ra[(2 * c) * kHeadDim + r] = acc[i][0];
            ra[(2 * c) * kHeadDim + r + 1] = acc[i][2];
          }
          if (2 * c + 1 < group) {
            ra[(2 * c + 1) * kHeadDim + r] = acc[i][1];
            ra[(2 * c + 1) * kHeadDim + r + 1] = acc[i][3];
          }
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);
      {
        const int64_t seg = int64_t(pc.b) * Hkv + pc.h;
        const int64_t slot = seg + blockIdx.x;
        for (int item = threadIdx.x; item < group * kHeadDim; item += kConsumerWarps * 32) {
          const int hh = item / kHeadDim;
          const int d = item - hh * kHeadDim;
          float M = kNegInf;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, tail.red_m[w][hh]);
          float L = 0.f, A = 0.f;
#pragma unroll
          for (int w = 0; w < kConsumerWarps; ++w) {
            const float mw = tail.red_m[w][hh];
            const float f = (mw == kNegInf) ? 0.f : fast_exp2((mw - M) * sl);
            L = fmaf(tail.red_l[w][hh], f, L);
            A = fmaf(red_acc[(w * kMaxGroup + hh) * kHeadDim + d], f, A);
          }
          if (pc.whole) {
            const int64_t row = int64_t(pc.b) * p.Hq + pc.h * group + hh;
            const float o = A / L;
            p.out[row * kHeadDim + d] = static_cast<uint16_t>(pack_bf16x2(o, 0.f) & 0xFFFFu);
            if (d == 0 && p.lse) p.lse[row] = M * p.sm_scale + logf(L);
          } else {
            float* ps = p.part + (slot * group + hh) * kPartStride;
            if (d == 0) {
              ps[0] = M;
              ps[1] = L;
            }
            ps[4 + d] = A;
          }
        }
      }
      named_barrier_sync(1, kConsumerWarps * 32);
      j_base += pc.npages;
      x += pc.npages;
    }
  }
  __syncthreads();
}

// Merge the partial slots of every (sequence, kv head) that more than one
// CTA covered; also writes zeros / -inf for empty sequences.
__global__ void __launch_bounds__(kHeadDim) merge_kernel(const DecodeParams p, int64_t G) {
  __shared__ int64_t s_first, s_last, s_W;
  grid_dependency_wait();  // partials and plan of the attention kernel
  launch_dependents();
  const int seg = blockIdx.x;
  const int b = seg / p.Hkv;
  const int h = seg - b * p.Hkv;
  const int d = threadIdx.x;
  const int group = p.group;
  const int64_t n_b = p.plan[b + 1] - p.plan[b];
  if (n_b == 0) {
    for (int hh = 0; hh < group; ++hh) {
      const int64_t row = int64_t(b) * p.Hq + h * group + hh;
      p.out[row * kHeadDim + d] = 0;
      if (d == 0 && p.lse) p.lse[row] = kNegInf;
    }
    return;
  }
  if (threadIdx.x == 0) {
    const int64_t W = int64_t(p.plan[p.B]) * p.Hkv;
    const int64_t x0 = int64_t(p.plan[b]) * p.Hkv + int64_t(h) * n_b;
    s_first = cta_of(x0, W, G);
    s_last = cta_of(x0 + n_b - 1, W, G);
    s_W = W;
  }
  __syncthreads();
  const int64_t first = s_first, last = s_last, W = s_W;
  if (first == last) return;  // that CTA wrote the output itself
  // With more CTAs than work items some ranges are empty and wrote no slot.
  const bool check = G > W;
  auto live = [&](int64_t i) { return !check || (W * i / G != W * (i + 1) / G); };
  const float sl = p.scale_log2;
  for (int hh = 0; hh < group; ++hh) {
    float M = kNegInf;
    for (int64_t i = first; i <= last; ++i)
      if (live(i)) M = fmaxf(M, p.part[((seg + i) * group + hh) * kPartStride]);
    float L = 0.f, A = 0.f;
    for (int64_t i = first; i <= last; ++i) {
      if (!live(i)) continue;
      const float* ps = p.part + ((seg + i) * group + hh) * kPartStride;
      const float f = (ps[0] == kNegInf) ? 0.f : fast_exp2((ps[0] - M) * sl);
      L = fmaf(ps[1], f, L);
      A = fmaf(ps[4 + d], f, A);
    }
    const int64_t row = int64_t(b) * p.Hq + h * group + hh;
    p.out[row * kHeadDim + d] = static_cast<uint16_t>(pack_bf16x2(A / L, 0.f) & 0xFFFFu);
    if (d == 0 && p.lse) p.lse[row] = M * p.sm_scale + logf(L);
  }
}

// Workspace: [0,16) error word | plan (B+1 int32, 256-aligned) | partial slots
struct WsLayout {
  size_t plan_off, part_off, total;
  int64_t grid;
};

WsLayout ws_layout(int B, int Hq, int Hkv, int max_seq_len, int num_sms) {
  WsLayout w{};
  const int64_t max_pages = (int64_t(max_seq_len) + kPageTokens - 1) / kPageTokens;
  int64_t work = int64_t(B) * Hkv * max_pages;
  int64_t grid = int64_t(num_sms) * kCtasPerSm;
  if (work < grid) grid = work;
  if (grid < 1) grid = 1;
  w.grid = grid;
  w.plan_off = 256;
  w.part_off = round_up(w.plan_off + size_t(B + 1) * sizeof(int32_t), 256);
  const int group = Hkv > 0 ? Hq / Hkv : 1;
  const size_t slots = size_t(B) * Hkv + size_t(grid);
  w.total = w.part_off + slots * size_t(group) * kPartStride * sizeof(float);
  return w;
}

zf_status check_common(const uint16_t* q, int num_pages, const int32_t* page_table, int max_pages_per_seq,
                       const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv, int head_dim,
                       float sm_scale, const uint16_t* out, const void* ws) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || max_pages_per_seq <= 0 || max_seq_len < 0)
    return ZF_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || Hq % Hkv != 0 || Hq / Hkv > kMaxGroup || B > kMaxBatch) return ZF_ERR_UNSUPPORTED;
  if (!std::isfinite(sm_scale)) return ZF_ERR_INVALID_ARG;
  if (int64_t(num_pages) * Hkv * kChunkBlocks > (int64_t(1) << 31)) return ZF_ERR_UNSUPPORTED;
  if (B == 0) return ZF_OK;
  if (!q || !page_table || !seq_lens || !out || !ws) return ZF_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
      !aligned(ws, 256))
    return ZF_ERR_INVALID_ARG;
  return ZF_OK;
}

template <bool kCompressed>
zf_status launch(DecodeParams prm, int max_seq_len, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const WsLayout L = ws_layout(prm.B, prm.Hq, prm.Hkv, max_seq_len, sms);
  if (ws_bytes < L.total) return ZF_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  prm.err = reinterpret_cast<uint32_t*>(w);
  prm.plan = reinterpret_cast<int32_t*>(w + L.plan_off);
  prm.part = reinterpret_cast<float*>(w + L.part_off);
  prm.group = prm.Hq / prm.Hkv;
  prm.scale_log2 = prm.sm_scale * 1.4426950408889634f;
  const size_t smem = smem_bytes(prm.B);
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<kCompressed>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  // Both kernels are launched with programmatic stream serialization: each
  // may be scheduled while the previous kernel in the stream drains, and
  // waits for it (griddepcontrol.wait) before touching memory.
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(L.grid));
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, decode_attn_kernel<kCompressed>, prm);
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  cfg.gridDim = dim3(static_cast<unsigned>(prm.B * prm.Hkv));
  cfg.blockDim = dim3(kHeadDim);
  cfg.dynamicSmemBytes = 0;
  e = cudaLaunchKernelEx(&cfg, merge_kernel, prm, static_cast<int64_t>(L.grid));
  return cuda_status(e);
}

}  // namespace
}  // namespace zf

using namespace zf;

extern "C" {

size_t zf_decode_workspace_size(int B, int Hq, int Hkv, int max_seq_len, int num_sms) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || max_seq_len < 0) return 0;
  if (num_sms <= 0) num_sms = current_sm_count();
  if (num_sms <= 0) return 0;
  return ws_layout(B, Hq, Hkv, max_seq_len, num_sms).total;
}

zf_status zf_decode_attention(const uint16_t* q, const zf_kv_compressed* k, const zf_kv_compressed* v,
                              int num_pages, const int32_t* page_table, int max_pages_per_seq,
                              const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv, int head_dim,
                              float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                              zf_stream_t stream) {
  zf_status st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                              head_dim, sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  if (!k || !v) return ZF_ERR_INVALID_ARG;
  const int64_t pool_values = int64_t(num_pages) * Hkv * kChunkValues;
  for (const zf_kv_compressed* c : {k, v}) {
    if (!c->payload || !c->offs || !c->base || !c->elig || c->n_values != pool_values ||
        c->payload_cap_bytes < 0 || !aligned(c->payload, 16) || !aligned(c->offs, 4) || !aligned(c->base, 16) ||
        !aligned(c->elig, 4))
      return ZF_ERR_INVALID_ARG;
  }
  if (lse && !aligned(lse, 4)) return ZF_ERR_INVALID_ARG;
  DecodeParams prm{};
  prm.q = q;
  prm.k_payload = static_cast<const uint8_t*>(k->payload);
  prm.k_offs = k->offs;
  prm.k_base = k->base;
  prm.k_elig = k->elig;
  prm.k_cap_units = k->payload_cap_bytes / kUnitBytes;
  prm.v_payload = static_cast<const uint8_t*>(v->payload);
  prm.v_offs = v->offs;
  prm.v_base = v->base;
  prm.v_elig = v->elig;
  prm.v_cap_units = v->payload_cap_bytes / kUnitBytes;
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.lse = lse;
  prm.num_pages = num_pages;
  prm.max_pages = max_pages_per_seq;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.sm_scale = sm_scale;
  return launch<true>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

zf_status zf_decode_attention_raw(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                                  int num_pages, const int32_t* page_table, int max_pages_per_seq,
                                  const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                  int head_dim, float sm_scale, uint16_t* out, float* lse, void* ws,
                                  size_t ws_bytes, zf_stream_t stream) {
  zf_status st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                              head_dim, sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  if (!k_pool || !v_pool || !aligned(k_pool, 16) || !aligned(v_pool, 16)) return ZF_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return ZF_ERR_INVALID_ARG;
  DecodeParams prm{};
  prm.q = q;
  prm.k_pool = k_pool;
  prm.v_pool = v_pool;
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.lse = lse;
  prm.num_pages = num_pages;
  prm.max_pages = max_pages_per_seq;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  prm.sm_scale = sm_scale;
  return launch<false>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Decode attention without any caller-provided workspace.
//
// Some callers cannot hand this library scratch memory: a plugin that a host
// inference engine invokes with nothing but its input and output buffers, or
// a process that reserves all of its device memory up front and forbids new
// allocations while serving.  For them the scratch (error word, split plan,
// partial results) lives in one fixed array that the library carries in its
// own device image.  Each GPU that loads the library holds this array until
// the process exits.
#include <mutex>

namespace zf {
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(4) << 20;  // 4 MiB
constexpr int kNoAllocMaxDevices = 64;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mu;

// Device address of the scratch array for the current device, looked up once
// per device (host code may not use the array's name as an address).
zf_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return ZF_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ZF_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return ZF_OK;
}
}  // namespace
}  // namespace zf

extern "C" zf_status zf_decode_attention_noalloc(const uint16_t* q, const zf_kv_compressed* k,
                                                 const zf_kv_compressed* v, int num_pages,
                                                 const int32_t* page_table, int max_pages_per_seq,
                                                 const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                                 int head_dim, float sm_scale, uint16_t* out, float* lse,
                                                 zf_stream_t stream) {
  void* ws = nullptr;
  zf_status st = zf::noalloc_scratch(&ws);
  if (st != ZF_OK) return st;
  st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv, head_dim,
                    sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  const size_t need = zf_decode_workspace_size(B, Hq, Hkv, max_seq_len, 0);
  if (need == 0) return ZF_ERR_CUDA;
  if (need > zf::kNoAllocScratchBytes) return ZF_ERR_WORKSPACE;
  // Nothing in the scratch has to start at zero; the error word is cleared so
  // that it describes this call only.
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ZF_ERR_CUDA;
  return zf_decode_attention(q, k, v, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                             head_dim, sm_scale, out, lse, ws, zf::kNoAllocScratchBytes, stream);
}
