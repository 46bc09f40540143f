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
//  * Persistent grid, one CTA per SM.  All work is the list of W (sequence,
//    kv head, page) items in sequence-major order, cut into equal contiguous
//    units, one per consumer warp of the grid, so every warp moves the same
//    number of pages whatever the length mix.  The split points come from
//    seq_lens on the device (each CTA scans them into shared memory), so
//    there is no host round trip.
//  * Four producer warps (one warpgroup) stream the pages of the CTA's
//    twelve consumer warps, round-robin, into a 24-stage shared-memory ring
//    with 1-D bulk (TMA) copies completed on mbarriers: each page's K and V
//    chunks (variable-size compressed extents) and their base exponents.
//    Page ids and chunk metadata are prepared 32 pages at a time by the
//    producer's lanes, two batches ahead.
//  * Per page (16 tokens) a consumer warp copies its share of the page into
//    registers, releases the stage, and rebuilds K and V straight into
//    mma.sync m16n8k16 operand registers: S^T = Q K^T puts the query heads of
//    the GQA group on M and tokens on N, so the S accumulator is already the
//    B operand of O^T = V^T P^T.  P is fed as a bf16 hi + lo pair (two mma),
//    which keeps P to ~16 bits of precision.  When every block of both
//    chunks is eligible (the common case) all block offsets are fixed and the
//    per-block tests are skipped.
//  * Online softmax in base 2 (scale * log2 e folded into one FMA); the
//    running max is reduced over the 4 lanes that hold one head's tokens.
//  * Three consumer warps and one producer warp share each SM sub-partition;
//    the producers hand registers to the consumers (setmaxnreg).
//  * A warp whose unit covers a whole sequence/head writes the output
//    directly; otherwise it writes a partial (m, l, acc[128]) slot and
//    counts it in on a per-segment counter: the warp that completes the
//    segment merges its slots in unit order (no second kernel).
//  * The raw-BF16 twin is the same template with the decode step replaced by
//    plain loads: same plan, same arithmetic, same order, so its output is
//    bitwise identical to the compressed kernel's.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <type_traits>

#include "zf_device.cuh"
#include "zf_internal.h"

namespace zf {
namespace {

#ifndef ZF_CONSUMER_WARPS
#define ZF_CONSUMER_WARPS 12
#endif
#ifndef ZF_PRODUCER_WARPS
#define ZF_PRODUCER_WARPS 4
#endif
#ifndef ZF_STAGES
#define ZF_STAGES 24
#endif
#ifndef ZF_CTAS_PER_SM
#define ZF_CTAS_PER_SM 1
#endif
constexpr int kConsumerWarps = ZF_CONSUMER_WARPS;
constexpr int kProducerWarps = ZF_PRODUCER_WARPS;
constexpr int kThreads = (kConsumerWarps + kProducerWarps) * 32;
constexpr int kStages = ZF_STAGES;
constexpr int kCtasPerSm = ZF_CTAS_PER_SM;
// Registers: the CTA is launched with kLaunchRegs per thread (the SM's 64K
// over its threads); the producer warpgroup then gives registers back and the
// consumer warpgroups take them (the consumers hold the O accumulator, the Q
// operand and a page's compressed words at once).  Each SM sub-partition
// runs one warp of every warpgroup, so the split also balances per
// sub-partition.
constexpr int kLaunchRegs = 65536 / (kThreads * kCtasPerSm) / 8 * 8;
constexpr int kProducerRegs = 56;
constexpr int kConsumerRegs = 152;
static_assert(kConsumerWarps * 32 * kConsumerRegs + kProducerWarps * 32 * kProducerRegs <=
                  kThreads * kLaunchRegs,
              "register split exceeds the launch allocation");
static_assert(kConsumerWarps % 4 == 0 && kProducerWarps % 4 == 0, "roles are whole warpgroups");
// Issue slot j (pages are handed out round-robin: slot j is page j / kConsumerWarps
// of consumer warp j % kConsumerWarps) lives in stage j % kStages.  Every stage
// must always belong to the same consumer warp: a warp then never waits on a
// stage more than one barrier phase ahead of it, which the parity waits need
// (two phases ahead would alias).  Likewise each stage belongs to one producer.
static_assert(kStages % kConsumerWarps == 0, "each ring stage must map to one consumer warp");
static_assert(kStages % kProducerWarps == 0, "each ring stage must map to one producer warp");
static_assert(kConsumerWarps % 4 == 0, "consumer warps spread evenly over the four SM sub-partitions");
constexpr int kChunkBytes = kChunkValues * 2;  // 4096 raw bytes per (page, head)
// KV cache formats of the decode kernel.
constexpr int kFmtRaw = 0;         // BF16 pools
constexpr int kFmtCompressed = 1;  // the lossless block codec
constexpr int kFmtFp8 = 2;         // E4M3 codes, one scale per pool (the lossy comparator)
constexpr int kFmtPaged = 3;       // the lossless block codec, paged form (one extent per chunk)
// Stage layout: K payload | V payload | K bases | V bases | header
constexpr int kStageK = 0;
constexpr int kStageV = kChunkBytes;
constexpr int kStageKBase = 2 * kChunkBytes;
constexpr int kStageVBase = kStageKBase + 32;
constexpr int kStageHdr = kStageVBase + 32;
// Paged form: the K chunk extent (header + blocks) at 0, the V extent after it.
constexpr int kExtentMax = kChunkHeaderBytes + kChunkBytes;  // 4144 = 259 units
constexpr int kStagePagedV = kExtentMax;
constexpr int kStageBytes = (kStageHdr + 16 > 2 * kExtentMax) ? kStageHdr + 16 : 2 * kExtentMax;  // 8288
static_assert(kStageBytes % 16 == 0 && kStagePagedV % 16 == 0, "stages and extents 16-byte aligned");
constexpr int kPartStride = 132;             // floats per (slot, head): m, l, pad, pad, acc[128]
constexpr float kNegInf = -INFINITY;
constexpr unsigned kFull = 0xFFFFFFFFu;
// Shared memory of one SM and what the hardware keeps back per resident CTA.
constexpr size_t kSmemPerSm = 228 * 1024;
constexpr size_t kSmemReservedPerCta = 1024;

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
  // paged-form pools: data, chunk_tab ({start, extent} in 16-byte units)
  const uint8_t* k_data;
  const uint32_t* k_tab;
  const uint8_t* v_data;
  const uint32_t* v_tab;
  // E4M3 pools (their K scale is folded into sm_scale / scale_log2)
  const uint8_t* k_fp8;
  const uint8_t* v_fp8;
  const int32_t* page_table;
  const int32_t* seq_lens;
  uint16_t* out;
  float* lse;
  float* part;
  uint32_t* count;  // per (sequence, kv head): partial slots written so far
  uint32_t* err;
  int num_pages;
  int max_pages;
  int B;
  int Hq;
  int Hkv;
  int group;
  float sm_scale;
  float scale_log2;  // sm_scale * log2(e)
  float out_scale;   // multiplies the output (the V scale of E4M3 pools; 1 otherwise)
};

// Shared-memory layout after the stage ring.
struct SmemTail {
  uint64_t full[kStages];
  uint64_t empty[kStages];
  int64_t unit_lo[kConsumerWarps + 1];  // work ranges of this CTA's consumer warps
  int32_t abort_flag;
  uint8_t last_issue[kStages];  // per stage: 0x80 | parity of the last page issued into it
};

__host__ __device__ constexpr size_t smem_fixed_bytes() {
  return size_t(kStages) * kStageBytes + ((sizeof(SmemTail) + 15) / 16) * 16;
}
// Dynamic shared memory: stage ring, tail, page prefix sums (B + 1).
__host__ __device__ inline size_t smem_bytes(int B) {
  return smem_fixed_bytes() + size_t(B + 1) * sizeof(int32_t);
}
// Resident CTAs per SM for batch size B (the shared-memory limit).
inline int ctas_per_sm(int B) {
  const size_t per_cta = smem_bytes(B) + kSmemReservedPerCta;
  const int fit = static_cast<int>(kSmemPerSm / per_cta);
  return fit < kCtasPerSm ? (fit < 1 ? 1 : fit) : kCtasPerSm;
}

// Largest unit index whose range [i*W/U, (i+1)*W/U) starts at or before x.
__device__ __forceinline__ int64_t unit_of(int64_t x, int64_t W, int64_t U) {
  return ((x + 1) * U + W - 1) / W - 1;
}

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

// Clamped length of sequence b (the plan reports out-of-range lengths).
__device__ __forceinline__ int32_t clamped_len(const int32_t* seq_lens, int b, int max_tokens) {
  const int32_t len = __ldg(seq_lens + b);
  return len < 0 ? 0 : (len > max_tokens ? max_tokens : len);
}

// Combine the partial (m, l, acc) slots of segment seg = (b, h), written by
// units first..last (empty units skipped), into the output rows of its query
// heads; one warp.  Slots are read through L2 (other SMs wrote them during
// this launch).  Lane j holds slot first + j's (m, l) of every head and lane
// l accumulates dims [4l, 4l+4) of every head, kSteps slots per step; the
// (m, l) loads and the first step's accumulator loads go out together, so a
// merge of up to 32 slots costs about ceil(slots / kSteps) L2 round trips.
// kHeads bounds the heads of the group (kHeads x kSteps float4 in flight).
template <int kHeads, int kSteps>
__device__ __forceinline__ void merge_slots(const DecodeParams& p, int b, int h, int64_t seg, int64_t i0,
                                            int n, int64_t last, int64_t W, int64_t U, int lane, float (&M)[kHeads],
                                            float (&L)[kHeads], float4 (&A)[kHeads], bool with_max) {
  constexpr unsigned kAll = 0xFFFFFFFFu;
  const float sl = p.scale_log2;
  const int group = p.group;
  const bool check = U > W;
  auto live = [&](int64_t i) { return i <= last && (!check || (W * i / U != W * (i + 1) / U)); };
  auto slot = [&](int64_t i, int hh) { return p.part + ((seg + i) * group + hh) * kPartStride; };
  auto load_step = [&](int t0, float4 (&a)[kSteps][kHeads]) {
#pragma unroll
    for (int t = 0; t < kSteps; ++t) {
      const bool ok = t0 + t < n && live(i0 + t0 + t);
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh)
        a[t][hh] = (hh < group && ok) ? __ldcg(reinterpret_cast<const float4*>(slot(i0 + t0 + t, hh) + 4) + lane)
                                      : make_float4(0.f, 0.f, 0.f, 0.f);
    }
  };
  // (m, l) of this lane's slot, and the first step's accumulators
  float2 ml[kHeads];
  {
    const bool ok = lane < n && live(i0 + lane);
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh)
      ml[hh] = (hh < group && ok) ? __ldcg(reinterpret_cast<const float2*>(slot(i0 + lane, hh)))
                                  : make_float2(kNegInf, 0.f);
  }
  float4 a[kSteps][kHeads];
  load_step(0, a);
  float f[kHeads];
#pragma unroll
  for (int hh = 0; hh < kHeads; ++hh) {
    if (with_max) {
      float m = ml[hh].x;
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) m = fmaxf(m, __shfl_xor_sync(kAll, m, d));
      M[hh] = m;
    }
    f[hh] = (ml[hh].x == kNegInf) ? 0.f : fast_exp2((ml[hh].x - M[hh]) * sl);
    L[hh] = fmaf(ml[hh].y, f[hh], L[hh]);
  }
  for (int t0 = 0;;) {
#pragma unroll
    for (int t = 0; t < kSteps; ++t)
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh) {
        const float ft = __shfl_sync(kAll, f[hh], (t0 + t) & 31);
        A[hh].x = fmaf(a[t][hh].x, ft, A[hh].x);
        A[hh].y = fmaf(a[t][hh].y, ft, A[hh].y);
        A[hh].z = fmaf(a[t][hh].z, ft, A[hh].z);
        A[hh].w = fmaf(a[t][hh].w, ft, A[hh].w);
      }
    t0 += kSteps;
    if (t0 >= n) break;
    load_step(t0, a);
  }
}

template <int kHeads, int kSteps>
__device__ __forceinline__ void merge_segment_g(const DecodeParams& p, int b, int h, int64_t seg, int64_t first,
                                                int64_t last, int64_t W, int64_t U, int lane) {
  constexpr unsigned kAll = 0xFFFFFFFFu;
  const int group = p.group;
  const bool check = U > W;
  float M[kHeads], L[kHeads];
  float4 A[kHeads];
#pragma unroll
  for (int hh = 0; hh < kHeads; ++hh) {
    M[hh] = kNegInf;
    L[hh] = 0.f;
    A[hh] = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const int64_t n_all = last - first + 1;
  if (n_all > 32) {
    // more than one round of slots: the maxima first, over every round
    for (int64_t i0 = first; i0 <= last; i0 += 32) {
      const int64_t i = i0 + lane;
      const bool ok = i <= last && (!check || (W * i / U != W * (i + 1) / U));
#pragma unroll
      for (int hh = 0; hh < kHeads; ++hh)
        if (hh < group && ok) M[hh] = fmaxf(M[hh], __ldcg(p.part + ((seg + i) * group + hh) * kPartStride));
    }
#pragma unroll
    for (int hh = 0; hh < kHeads; ++hh)
#pragma unroll
      for (int d = 16; d > 0; d >>= 1) M[hh] = fmaxf(M[hh], __shfl_xor_sync(kAll, M[hh], d));
  }
  for (int64_t i0 = first; i0 <= last; i0 += 32) {
    const int n = static_cast<int>(last - i0 + 1 < 32 ? last - i0 + 1 : 32);
    merge_slots<kHeads, kSteps>(p, b, h, seg, i0, n, last, W, U, lane, M, L, A, n_all <= 32);
  }
#pragma unroll
  for (int hh = 0; hh < kHeads; ++hh) {
#pragma unroll
    for (int d = 16; d > 0; d >>= 1) L[hh] += __shfl_xor_sync(kAll, L[hh], d);
    if (hh < group) {
      const int64_t row = int64_t(b) * p.Hq + h * group + hh;
      uint2* o = reinterpret_cast<uint2*>(p.out + row * kHeadDim) + lane;
      *o = make_uint2(pack_bf16x2(A[hh].x / L[hh], A[hh].y / L[hh]), pack_bf16x2(A[hh].z / L[hh], A[hh].w / L[hh]));
      if (lane == 0 && p.lse) p.lse[row] = M[hh] * p.sm_scale + logf(L[hh]);
    }
  }
}

__device__ __forceinline__ void merge_segment(const DecodeParams& p, int b, int h, int64_t seg, int64_t first,
                                              int64_t last, int64_t W, int64_t U, int lane) {
  if (p.group <= 4)
    merge_segment_g<4, 4>(p, b, h, seg, first, last, W, U, lane);
  else
    merge_segment_g<kMaxGroup, 1>(p, b, h, seg, first, last, W, U, lane);
}

// ------------------------------------------------------------------ kernel

template <int kFmt>
__global__ void __launch_bounds__(kThreads, kCtasPerSm) decode_attn_kernel(const DecodeParams p) {
  constexpr bool kCompressed = kFmt == kFmtCompressed;
  constexpr bool kPaged = kFmt == kFmtPaged;
  constexpr bool kCodec = kCompressed || kPaged;  // values rebuilt by the block codec
  constexpr bool kFp8 = kFmt == kFmtFp8;
  // Where a stage keeps K / V payload blocks, base exponents and masks.
  constexpr int kPayK = kPaged ? kChunkHeaderBytes : kStageK;
  constexpr int kPayV = kPaged ? kStagePagedV + kChunkHeaderBytes : kStageV;
  constexpr int kBaseK = kPaged ? 0 : kStageKBase;
  constexpr int kBaseV = kPaged ? kStagePagedV : kStageVBase;
  constexpr int kMaskK = kPaged ? 32 : kStageHdr;
  constexpr int kMaskV = kPaged ? kStagePagedV + 32 : kStageHdr + 4;
  extern __shared__ __align__(128) uint8_t smem[];
  SmemTail& tail = *reinterpret_cast<SmemTail*>(smem + size_t(kStages) * kStageBytes);
  int32_t* s_pfx = reinterpret_cast<int32_t*>(smem + smem_fixed_bytes());

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int B = p.B;
  const int Hkv = p.Hkv;
  const int group = p.group;
  const int max_tokens = p.max_pages * kPageTokens;

  // Inputs may come from the previous kernel in the stream (q, the cache
  // append): wait for it before reading anything, then let the next kernel
  // in the stream start launching.
  grid_dependency_wait();
  launch_dependents();

  // ---- plan: page prefix sums of the clamped lengths (warp 0), barriers
  if (warp == 0) {
    const int per = (B + 31) / 32;
    const int b0 = lane * per;
    int32_t run = 0;
    for (int i = 0; i < per; ++i) {
      const int b = b0 + i;
      if (b < B) {
        const int32_t len = __ldg(p.seq_lens + b);
        if (len < 0 || len > max_tokens) set_error(p.err, ZF_DEVERR_SEQ_LEN);
        run += (clamped_len(p.seq_lens, b, max_tokens) + kPageTokens - 1) / kPageTokens;
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
        acc += (clamped_len(p.seq_lens, b, max_tokens) + kPageTokens - 1) / kPageTokens;
      }
    }
    if (lane == 31) s_pfx[B] = incl;
  }
  if (threadIdx.x == 32) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(smem_addr(&tail.full[s]), 1);
      mbar_init(smem_addr(&tail.empty[s]), 1);
      tail.last_issue[s] = 0;
    }
    tail.abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  // Sequences without tokens: output 0 and lse = -inf (no unit covers them).
  for (int b = blockIdx.x; b < B; b += gridDim.x) {
    if (s_pfx[b + 1] != s_pfx[b]) continue;
    uint32_t* o = reinterpret_cast<uint32_t*>(p.out + int64_t(b) * p.Hq * kHeadDim);
    for (int i = threadIdx.x; i < p.Hq * kHeadDim / 2; i += blockDim.x) o[i] = 0u;
    if (p.lse)
      for (int i = threadIdx.x; i < p.Hq; i += blockDim.x) p.lse[int64_t(b) * p.Hq + i] = kNegInf;
  }
  // All work is the list of W (sequence, kv head, page) items; it is cut
  // into U = grid * kConsumerWarps equal contiguous units, one per consumer
  // warp, so every warp moves the same number of pages whatever the length
  // mix.  This CTA owns units [blockIdx.x * kConsumerWarps, +kConsumerWarps).
  const int64_t U = int64_t(gridDim.x) * kConsumerWarps;
  const int64_t W = int64_t(s_pfx[B]) * Hkv;
  if (threadIdx.x <= kConsumerWarps)
    tail.unit_lo[threadIdx.x] = W * (int64_t(blockIdx.x) * kConsumerWarps + threadIdx.x) / U;
  __syncthreads();

  if (warp >= kConsumerWarps) {
    // =========================== producer warps ==========================
    // Pages are handed to the consumer warps round-robin: issue slot j is
    // page j / kConsumerWarps of warp j % kConsumerWarps' unit (slots past
    // the end of a shorter unit are empty) and goes to stage j % kStages.
    // Producer pw issues the slots j = pw, pw + P, ... (P producer warps;
    // it fills the stages s with s % P == pw) in order.  Its 32 lanes
    // prepare the metadata of 32 of its slots at a time in a software
    // pipeline (one lane per slot, all in one SIMT pass):
    //   A: locate the page and load its id                (two batches ahead)
    //   B: load the chunk's offset / mask words             (one batch ahead)
    //   C: derive the copy addresses and sizes            (this batch)
    // and then issues the batch slot by slot: the lane that holds the page
    // waits for its stage to be released, stores the mask words and issues
    // the bulk copies (payloads and base exponents of K and V).  All but the
    // wait and the copies runs once per 32 pages.
    warpgroup_regs_dec<kProducerRegs>();
    const int pw = warp - kConsumerWarps;
    constexpr int P = kProducerWarps;
    const int64_t n_round = (tail.unit_lo[kConsumerWarps] - tail.unit_lo[0] + kConsumerWarps - 1) / kConsumerWarps;
    const int64_t n_slots = n_round * kConsumerWarps;
    const int64_t n_mine = n_slots > pw ? (n_slots - pw + P - 1) / P : 0;
    struct StepA { int32_t h; int32_t pid; bool valid; };
    struct StepB { int64_t chunk; uint32_t ku, vu, ke, ve; bool valid; };
    struct StepC { const uint8_t* ksrc; const uint8_t* vsrc; const uint8_t* kbase; const uint8_t* vbase;
                   uint32_t kbytes, vbytes; uint32_t ke, ve; bool valid; };
    auto step_a = [&](int64_t i) {
      StepA a{0, 0, false};
      if (i < n_mine) {
        const int64_t j = pw + int64_t(P) * i;
        const int w = static_cast<int>(j % kConsumerWarps);
        const int64_t k = j / kConsumerWarps;
        const int64_t x = tail.unit_lo[w] + k;
        if (x < tail.unit_lo[w + 1]) {
          int b, h;
          int64_t page, n_b;
          locate(s_pfx, B, Hkv, x, b, h, page, n_b);
          a.h = h;
          a.pid = __ldg(p.page_table + int64_t(b) * p.max_pages + page);
          a.valid = true;
        }
      }
      return a;
    };
    auto step_b = [&](const StepA& a) {
      StepB m{};
      m.valid = a.valid;
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
        } else if constexpr (kPaged) {  // {start, extent} of each chunk
          const uint2 kt = __ldg(reinterpret_cast<const uint2*>(p.k_tab) + m.chunk);
          const uint2 vt = __ldg(reinterpret_cast<const uint2*>(p.v_tab) + m.chunk);
          m.ku = kt.x;
          m.ke = kt.y;
          m.vu = vt.x;
          m.ve = vt.y;
        }
      }
      return m;
    };
    auto step_c = [&](const StepB& m) {
      StepC d{};
      d.valid = m.valid;
      if constexpr (kCompressed) {
        const uint32_t k_units = 8u * kChunkBlocks - 2u * __popc(m.ke);
        const uint32_t v_units = 8u * kChunkBlocks - 2u * __popc(m.ve);
        d.kbytes = k_units * kUnitBytes;
        d.vbytes = v_units * kUnitBytes;
        if (m.valid && int64_t(m.ku) + k_units > p.k_cap_units) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          d.kbytes = 0;
        }
        if (m.valid && int64_t(m.vu) + v_units > p.v_cap_units) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          d.vbytes = 0;
        }
        d.ksrc = p.k_payload + uint64_t(m.ku) * kUnitBytes;
        d.vsrc = p.v_payload + uint64_t(m.vu) * kUnitBytes;
        d.kbase = p.k_base + m.chunk * kChunkBlocks;
        d.vbase = p.v_base + m.chunk * kChunkBlocks;
        d.ke = m.ke;
        d.ve = m.ve;
      } else if constexpr (kPaged) {
        // extents: one header + at most 32 raw blocks, inside the data buffer
        d.kbytes = m.ke * kUnitBytes;
        d.vbytes = m.ve * kUnitBytes;
        if (m.valid && (m.ke > kExtentMax / kUnitBytes || int64_t(m.ku) + m.ke > p.k_cap_units)) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          d.kbytes = 0;
        }
        if (m.valid && (m.ve > kExtentMax / kUnitBytes || int64_t(m.vu) + m.ve > p.v_cap_units)) {
          set_error(p.err, ZF_DEVERR_EXTENT);
          d.vbytes = 0;
        }
        d.ksrc = p.k_data + uint64_t(m.ku) * kUnitBytes;
        d.vsrc = p.v_data + uint64_t(m.vu) * kUnitBytes;
      } else if constexpr (kFp8) {
        d.ksrc = p.k_fp8 + m.chunk * kChunkValues;
        d.vsrc = p.v_fp8 + m.chunk * kChunkValues;
        d.kbytes = d.vbytes = kChunkValues;
      } else {
        d.ksrc = reinterpret_cast<const uint8_t*>(p.k_pool + m.chunk * kChunkValues);
        d.vsrc = reinterpret_cast<const uint8_t*>(p.v_pool + m.chunk * kChunkValues);
        d.kbytes = d.vbytes = kChunkBytes;
      }
      return d;
    };
    // Wait for stage s to be released (barrier phase parity `parity`), then
    // fill it; false if the wait was called off or timed out.
    auto issue = [&](int s, uint32_t parity, const StepC& d) -> bool {
      const WaitResult w = mbar_wait_or_abort(smem_addr(&tail.empty[s]), parity, &tail.abort_flag);
      if (w != kWaitDone) {
        if (w == kWaitTimedOut) {
          set_error(p.err, ZF_DEVERR_TIMEOUT);
          atomicExch(&tail.abort_flag, 1);
        }
        return false;
      }
      // The consumer's reads of this stage's previous page (ordered before
      // us by the empty barrier) must precede the bulk copies' writes.
      fence_proxy_async_smem();
      uint8_t* st = smem + size_t(s) * kStageBytes;
      const uint32_t full = smem_addr(&tail.full[s]);
      // The mask words are a plain store, released by the arrive below.
      if constexpr (kCompressed) *reinterpret_cast<uint2*>(st + kStageHdr) = make_uint2(d.ke, d.ve);
      mbar_arrive_expect_tx(full, d.kbytes + d.vbytes + (kCompressed ? 2u * kChunkBlocks : 0u));
      if (d.kbytes) bulk_copy_g2s(smem_addr(st + kStageK), d.ksrc, d.kbytes, full);
      if (d.vbytes) bulk_copy_g2s(smem_addr(st + (kPaged ? kStagePagedV : kStageV)), d.vsrc, d.vbytes, full);
      if constexpr (kCompressed) {
        bulk_copy_g2s(smem_addr(st + kStageKBase), d.kbase, kChunkBlocks, full);
        bulk_copy_g2s(smem_addr(st + kStageVBase), d.vbase, kChunkBlocks, full);
      }
      tail.last_issue[s] = static_cast<uint8_t>(0x80u | (parity ^ 1u));
      return true;
    };

    StepB nb = step_b(step_a(lane));
    StepA ahead = step_a(32 + lane);
    int stage = pw;      // stage of the next slot, same on all lanes
    uint32_t phase = 0;  // its barrier round parity
    bool stop = false;
    for (int64_t i0 = 0; i0 < n_mine && !stop; i0 += 32) {
      const StepC cur = step_c(nb);
      const StepA ahead2 = step_a(i0 + 64 + lane);
      nb = step_b(ahead);
      ahead = ahead2;
      const int count = static_cast<int>(n_mine - i0 < 32 ? n_mine - i0 : 32);
      const uint32_t has_page = __ballot_sync(kFull, cur.valid);
      for (int l = 0; l < count; ++l) {
        if ((has_page >> l) & 1u) {
          int ok = 1;
          if (lane == l) ok = issue(stage, phase ^ 1u, cur);
          if (!__shfl_sync(kFull, ok, l)) {
            stop = true;
            break;
          }
        }
        stage += P;
        if (stage >= kStages) {
          stage -= kStages;
          phase ^= 1u;
        }
      }
    }
    // After an abort, copies still in flight must land before the CTA may
    // exit: lane l waits for the last page this producer issued into its
    // l-th stage.
    __syncwarp();
    if (stop) {
      for (int s = pw + P * lane; s < kStages && lane < 32; s += P * 32) {
        const uint32_t li = tail.last_issue[s];
        if (li & 0x80u) mbar_wait_bounded(smem_addr(&tail.full[s]), li & 1u);
      }
    }
  } else {
    // =========================== consumer warps ==========================
    warpgroup_regs_inc<kConsumerRegs>();
    const int g = lane >> 2;  // mma group: query head (rows) / token (cols)
    const int c = lane & 3;   // thread in group
    const float sl = p.scale_log2;
    // Tokens of this lane in the P / V operands, and its V dims offset.
    const int tk[4] = {2 * c, 2 * c + 1, 8 + 2 * c, 9 + 2 * c};
    const int kk = 8 * (g & 3);
    const int kv = c & 1;  // half of a K block this lane reads
    // Raw pools: the lanes of the upper half of a token's dims (c >= 2) take
    // their two 16-dim runs in the other order (a k-order permutation that Q
    // follows), so the four lanes of a token row in one shared-memory phase
    // read four different bank groups; and for V those lanes load their
    // upper 8 dims first (then swap back in registers).
    const int run_sw = (kFmt == kFmtRaw && (c >> 1)) ? 4 : 0;  // in 16-byte pieces
    // Blocks this lane reads in every page: K block of token g + 8 nt, V block
    // of token tk[u]; and the mask of the blocks before each (offsets).
    uint32_t kblk[2], kbelow[2], vblk[4], vbelow[4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt) {
      kblk[nt] = 2 * (g + 8 * nt) + (c >> 1);
      kbelow[nt] = (1u << kblk[nt]) - 1u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      vblk[u] = 2 * tk[u] + (g >> 2);
      vbelow[u] = (1u << vblk[u]) - 1u;
    }
    const int64_t unit = int64_t(blockIdx.x) * kConsumerWarps + warp;
    const int64_t x_hi = tail.unit_lo[warp + 1];
    // This warp's k-th page is issue slot k * kConsumerWarps + warp: stage
    // (slot % kStages), barrier phase parity (slot / kStages) & 1, tracked
    // incrementally (kStages is a multiple of kConsumerWarps, so the stage
    // index wraps exactly at kStages).
    int stage = warp;
    uint32_t phase = 0;
    bool dead = false;  // set once a wait failed: skip the remaining pages
    for (int64_t x = tail.unit_lo[warp]; x < x_hi;) {
      // ---- the piece of this unit inside one (sequence, kv head) segment
      int b, h;
      int64_t page0_64, n_b;
      locate(s_pfx, B, Hkv, x, b, h, page0_64, n_b);
      const int64_t seg_start = int64_t(s_pfx[b]) * Hkv + int64_t(h) * n_b;
      const int64_t seg_end = seg_start + n_b;
      const int64_t end = seg_end < x_hi ? seg_end : x_hi;
      const int32_t npages = static_cast<int32_t>(end - x);
      const bool whole = (x == seg_start) && (end == seg_end);
      const int32_t page0 = static_cast<int32_t>(page0_64);
      const int seq_len = clamped_len(p.seq_lens, b, max_tokens);

      // Q operand (B of S = K Q^T): head g (column), the 32 dims lane c owns
      // (the k index order of the contraction is a free permutation, the
      // same for K and Q): run0 = dims 64*(c>>1) + 16*(c&1) + [0,16),
      // run1 = run0 + 32 (swapped when run_sw); k-step s2 takes the pair
      // 2*s2 of each run.
      uint32_t qa[8][2];
      {
        const int hq = h * group + g;
        if (g < group) {
          const uint16_t* qp = p.q + (int64_t(b) * p.Hq + hq) * kHeadDim + 64 * (c >> 1) + 16 * (c & 1);
          const uint4* q4 = reinterpret_cast<const uint4*>(qp);
          const uint4 r0a = __ldg(q4 + run_sw), r0b = __ldg(q4 + run_sw + 1);
          const uint4 r1a = __ldg(q4 + 4 - run_sw), r1b = __ldg(q4 + 5 - run_sw);
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
        if constexpr (kFp8) {  // the E4M3 path multiplies in f16
#pragma unroll
          for (int s = 0; s < 8; ++s)
#pragma unroll
            for (int t = 0; t < 2; ++t) qa[s][t] = pack_f16x2(bf16_lo_to_f32(qa[s][t]), bf16_hi_to_f32(qa[s][t]));
        }
      }

      // Online softmax state of this lane's two heads 2c ("e") and 2c+1
      // ("o"): running max (the same on the 8 lanes of a column) and this
      // lane's share of the running sum (its two tokens per page).
      float m_e = kNegInf, m_o = kNegInf;
      float l_e = 0.f, l_o = 0.f;
      float acc[8][4];  // O^T rows (dims) x cols (heads 2c, 2c+1)
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] = 0.f;

      for (int32_t jj = 0; jj < npages; ++jj) {
        const int s = stage;
        const uint32_t parity = phase;
        stage += kConsumerWarps;
        if (stage >= kStages) {
          stage -= kStages;
          phase ^= 1u;
        }
        if (dead) continue;
        {
          // The lanes must agree: a page is used only if every lane saw it.
          const WaitResult w = mbar_wait_or_abort(smem_addr(&tail.full[s]), parity, &tail.abort_flag);
          if (!__all_sync(kFull, w == kWaitDone)) {
            if (__any_sync(kFull, w == kWaitTimedOut) && lane == 0) {
              set_error(p.err, ZF_DEVERR_TIMEOUT);
              atomicExch(&tail.abort_flag, 1);
            }
            dead = true;
            continue;
          }
        }
        const uint8_t* st = smem + size_t(s) * kStageBytes;
        const int32_t page = page0 + jj;
        const int32_t left = seq_len - page * kPageTokens;
        const int n_valid = left >= kPageTokens ? kPageTokens : left;

        // ---- 1. copy this lane's share of the page into registers, then
        // hand the stage back to the producer at once.
        // K: tokens g (nt 0) and g+8 (nt 1), half v = c&1 of block
        //    2*token + (c>>1): values [16v,16v+16) ("lo") and [32+16v,+16) ("hi").
        // V: tokens tk[u], 16 values of block 2*tk[u] + (g>>2): [kk,kk+8) and
        //    [32+kk,+8).
        // Compressed blocks of both kinds share the layout [sign/mantissa
        // plane | exponent plane]: eligible blocks hold 4-bit offsets (low
        // nibble: value k, high nibble: value k+32) to add to the base,
        // raw blocks the 8-bit exponent of each value; x0 / x1 below are
        // the exponent-plane words of the lo / hi values of a raw block (x0
        // holds both nibbles for an eligible one).
        uint4 ks0[2], ks1[2], kx0[2], kx1[2];  // compressed K (raw pools: 4 quads of values)
        uint2 vs0[4], vs1[4], vx0[4], vx1[4];  // compressed V (raw pools: vs0|vx0, vs1|vx1 hold 2 quads)
        uint4 vr0[4], vr1[4];
        uint32_t kbase[2] = {0u, 0u}, vbase[4] = {0u, 0u, 0u, 0u};
        uint32_t ke = 0u, ve = 0u;
        if constexpr (kCodec) {
          ke = *reinterpret_cast<const uint32_t*>(st + kMaskK);
          ve = *reinterpret_cast<const uint32_t*>(st + kMaskV);
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint32_t blk = kblk[nt];
            const uint8_t* bp = st + kPayK + (128u * blk - 32u * __popc(ke & kbelow[nt])) + 16 * kv;
            ks0[nt] = *reinterpret_cast<const uint4*>(bp);
            ks1[nt] = *reinterpret_cast<const uint4*>(bp + 32);
            kx0[nt] = *reinterpret_cast<const uint4*>(bp + 64);
            kx1[nt] = *reinterpret_cast<const uint4*>(bp + 96);
            kbase[nt] = st[kBaseK + blk];
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint32_t blk = vblk[u];
            const uint8_t* bp = st + kPayV + (128u * blk - 32u * __popc(ve & vbelow[u])) + kk;
            vs0[u] = *reinterpret_cast<const uint2*>(bp);
            vs1[u] = *reinterpret_cast<const uint2*>(bp + 32);
            vx0[u] = *reinterpret_cast<const uint2*>(bp + 64);
            vx1[u] = *reinterpret_cast<const uint2*>(bp + 96);
            vbase[u] = st[kBaseV + blk];
          }
        } else if constexpr (kFp8) {
          // E4M3 chunk: token t at bytes [128 t, 128 t + 128); K: the lane's two
          // runs of 16 dims of tokens g and g+8; V: 8 + 8 dims of tokens tk[u].
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint8_t* tp = st + kStageK + 128 * (g + 8 * nt) + 64 * (c >> 1) + 16 * (c & 1);
            ks0[nt] = *reinterpret_cast<const uint4*>(tp);
            ks1[nt] = *reinterpret_cast<const uint4*>(tp + 32);
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint8_t* tp = st + kStageV + 128 * tk[u] + 64 * (g >> 2) + kk;
            vs0[u] = *reinterpret_cast<const uint2*>(tp);
            vs1[u] = *reinterpret_cast<const uint2*>(tp + 32);
          }
        } else {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt) {
            const uint4* r = reinterpret_cast<const uint4*>(st + kStageK + 128 * kblk[nt] + 32 * kv);
            ks0[nt] = r[run_sw];
            ks1[nt] = r[run_sw + 1];
            kx0[nt] = r[4 - run_sw];
            kx1[nt] = r[5 - run_sw];
          }
          const int vsw = 16 * run_sw;  // bytes
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const uint8_t* bp = st + kStageV + 128 * vblk[u] + 2 * kk;
            const uint4 va = *reinterpret_cast<const uint4*>(bp + vsw);
            const uint4 vb = *reinterpret_cast<const uint4*>(bp + (64 - vsw));
            vr0[u] = vsw ? vb : va;
            vr1[u] = vsw ? va : vb;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(smem_addr(&tail.empty[s]));

        // ---- 2. K -> A operand of S = K Q^T (rows: tokens g, g+8)
        uint32_t kb[2][8][2];  // [token row][k-step][k-pair c, c+4]
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
          if constexpr (kCodec) {
            const bool el = (ke >> kblk[nt]) & 1u;
            const uint32_t mask = el ? 0x0F0F0F0Fu : 0xFFFFFFFFu;
            const uint32_t b4 = el ? splat_byte(kbase[nt]) : 0u;
            const uint32_t sh = el ? 4u : 32u;
            const uint32_t s0v[4] = {ks0[nt].x, ks0[nt].y, ks0[nt].z, ks0[nt].w};
            const uint32_t s1v[4] = {ks1[nt].x, ks1[nt].y, ks1[nt].z, ks1[nt].w};
            const uint32_t x0v[4] = {kx0[nt].x, kx0[nt].y, kx0[nt].z, kx0[nt].w};
            const uint32_t x1v[4] = {kx1[nt].x, kx1[nt].y, kx1[nt].z, kx1[nt].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              const uint32_t elo = (x0v[w] & mask) + b4;
              const uint32_t ehi = (__funnelshift_rc(x0v[w], x1v[w], sh) & mask) + b4;
              kb[nt][2 * w][0] = rebuild_pair(s0v[w], elo, 0x5140);
              kb[nt][2 * w + 1][0] = rebuild_pair(s0v[w], elo, 0x7362);
              kb[nt][2 * w][1] = rebuild_pair(s1v[w], ehi, 0x5140);
              kb[nt][2 * w + 1][1] = rebuild_pair(s1v[w], ehi, 0x7362);
            }
          } else if constexpr (kFp8) {
            const uint32_t r0[4] = {ks0[nt].x, ks0[nt].y, ks0[nt].z, ks0[nt].w};
            const uint32_t r1[4] = {ks1[nt].x, ks1[nt].y, ks1[nt].z, ks1[nt].w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
              kb[nt][2 * w][0] = e4m3x2_to_f16x2(r0[w]);
              kb[nt][2 * w + 1][0] = e4m3x2_to_f16x2(r0[w] >> 16);
              kb[nt][2 * w][1] = e4m3x2_to_f16x2(r1[w]);
              kb[nt][2 * w + 1][1] = e4m3x2_to_f16x2(r1[w] >> 16);
            }
          } else {
            const uint32_t r0[8] = {ks0[nt].x, ks0[nt].y, ks0[nt].z, ks0[nt].w,
                                    ks1[nt].x, ks1[nt].y, ks1[nt].z, ks1[nt].w};
            const uint32_t r1[8] = {kx0[nt].x, kx0[nt].y, kx0[nt].z, kx0[nt].w,
                                    kx1[nt].x, kx1[nt].y, kx1[nt].z, kx1[nt].w};
#pragma unroll
            for (int s2 = 0; s2 < 8; ++s2) {
              kb[nt][s2][0] = r0[s2];
              kb[nt][s2][1] = r1[s2];
            }
          }
        }

        // ---- S[token][head]: c0 = (g, 2c), c1 = (g, 2c+1), c2 = (g+8, 2c), c3 = (g+8, 2c+1)
        float sc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int s2 = 0; s2 < 8; ++s2) {
          if constexpr (kFp8)
            mma_16816_f16(sc, kb[0][s2][0], kb[1][s2][0], kb[0][s2][1], kb[1][s2][1], qa[s2][0], qa[s2][1]);
          else
            mma_16816(sc, kb[0][s2][0], kb[1][s2][0], kb[0][s2][1], kb[1][s2][1], qa[s2][0], qa[s2][1]);
        }
        const bool partial = n_valid < kPageTokens;  // same on every lane
        // ---- 3. V -> A operand of O^T = V^T P^T (independent of the scores,
        // so its integer work overlaps the QK^T mma and the softmax chain):
        // tokens 2c, 2c+1, 2c+8, 2c+9;
        // dims r(i) = 64*(g>>2) + 32*hi + 8*(g&3) + 4*w + 2*t for m-tile
        // i = 4*w + 2*hi + t, rows g and g+8 = dims r(i) and r(i)+1.
        uint32_t xv[4][8];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          if constexpr (kCodec) {
            const bool el = (ve >> vblk[u]) & 1u;
            const uint32_t mask = el ? 0x0F0F0F0Fu : 0xFFFFFFFFu;
            const uint32_t b4 = el ? splat_byte(vbase[u]) : 0u;
            const uint32_t sh = el ? 4u : 32u;
            const uint32_t s0v[2] = {vs0[u].x, vs0[u].y};
            const uint32_t s1v[2] = {vs1[u].x, vs1[u].y};
            const uint32_t x0v[2] = {vx0[u].x, vx0[u].y};
            const uint32_t x1v[2] = {vx1[u].x, vx1[u].y};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              const uint32_t elo = (x0v[w] & mask) + b4;
              const uint32_t ehi = (__funnelshift_rc(x0v[w], x1v[w], sh) & mask) + b4;
              xv[u][4 * w + 0] = rebuild_pair(s0v[w], elo, 0x5140);
              xv[u][4 * w + 1] = rebuild_pair(s0v[w], elo, 0x7362);
              xv[u][4 * w + 2] = rebuild_pair(s1v[w], ehi, 0x5140);
              xv[u][4 * w + 3] = rebuild_pair(s1v[w], ehi, 0x7362);
            }
          } else if constexpr (kFp8) {
            const uint32_t s0v[2] = {vs0[u].x, vs0[u].y};
            const uint32_t s1v[2] = {vs1[u].x, vs1[u].y};
#pragma unroll
            for (int w = 0; w < 2; ++w) {
              xv[u][4 * w + 0] = e4m3x2_to_f16x2(s0v[w]);
              xv[u][4 * w + 1] = e4m3x2_to_f16x2(s0v[w] >> 16);
              xv[u][4 * w + 2] = e4m3x2_to_f16x2(s1v[w]);
              xv[u][4 * w + 3] = e4m3x2_to_f16x2(s1v[w] >> 16);
            }
          } else {
            const uint4 r0 = vr0[u], r1 = vr1[u];
            xv[u][0] = r0.x; xv[u][1] = r0.y; xv[u][2] = r1.x; xv[u][3] = r1.y;
            xv[u][4] = r0.z; xv[u][5] = r0.w; xv[u][6] = r1.z; xv[u][7] = r1.w;
          }
        }
        // Tokens past the end of the sequence: their P is 0, and their V
        // (whatever the slot holds, NaN included) must not reach the sum.
        if (partial) {
#pragma unroll
          for (int u = 0; u < 4; ++u)
            if (tk[u] >= n_valid) {
#pragma unroll
              for (int i = 0; i < 8; ++i) xv[u][i] = 0u;
            }
        }

        if (partial) {
          if (g >= n_valid) sc[0] = sc[1] = kNegInf;
          if (g + 8 >= n_valid) sc[2] = sc[3] = kNegInf;
        }

        // ---- online softmax (base 2) per head column, over the 8 lanes of it
        float mx_e = fmaxf(sc[0], sc[2]), mx_o = fmaxf(sc[1], sc[3]);
#pragma unroll
        for (int d = 4; d < 32; d <<= 1) {
          mx_e = fmaxf(mx_e, __shfl_xor_sync(kFull, mx_e, d));
          mx_o = fmaxf(mx_o, __shfl_xor_sync(kFull, mx_o, d));
        }
        const float mn_e = fmaxf(m_e, mx_e), mn_o = fmaxf(m_o, mx_o);
        const float a_e = fast_exp2((m_e - mn_e) * sl), a_o = fast_exp2((m_o - mn_o) * sl);
        const float ng_e = -mn_e * sl, ng_o = -mn_o * sl;
        const float p0 = fast_exp2(fmaf(sc[0], sl, ng_e)), p1 = fast_exp2(fmaf(sc[1], sl, ng_o));
        const float p2 = fast_exp2(fmaf(sc[2], sl, ng_e)), p3 = fast_exp2(fmaf(sc[3], sl, ng_o));
        l_e = fmaf(l_e, a_e, p0 + p2);
        l_o = fmaf(l_o, a_o, p1 + p3);
        m_e = mn_e;
        m_o = mn_o;
        // P as bf16 hi + lo parts; each 8x8 (tokens x heads) piece is
        // transposed in registers into the B operand of O^T = V^T P^T
        // (k: tokens 2c, 2c+1 and 2c+8, 2c+9; n: head g).
        uint32_t ph0, ph1, pl0, pl1;
        if constexpr (kFp8) {
          ph0 = pack_f16x2(p0, p1);
          ph1 = pack_f16x2(p2, p3);
          pl0 = pack_f16x2(p0 - f16_lo_to_f32(ph0), p1 - f16_hi_to_f32(ph0));
          pl1 = pack_f16x2(p2 - f16_lo_to_f32(ph1), p3 - f16_hi_to_f32(ph1));
        } else {
          ph0 = pack_bf16x2(p0, p1);
          ph1 = pack_bf16x2(p2, p3);
          pl0 = pack_bf16x2(p0 - bf16_lo_to_f32(ph0), p1 - bf16_hi_to_f32(ph0));
          pl1 = pack_bf16x2(p2 - bf16_lo_to_f32(ph1), p3 - bf16_hi_to_f32(ph1));
        }
        const uint32_t bh0 = transpose8x8_b16(ph0), bh1 = transpose8x8_b16(ph1);
        const uint32_t bl0 = transpose8x8_b16(pl0), bl1 = transpose8x8_b16(pl1);
        // Rescale always (no branch: the block stays one scheduling region).
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          acc[i][0] *= a_e;
          acc[i][1] *= a_o;
          acc[i][2] *= a_e;
          acc[i][3] *= a_o;
        }

#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const uint32_t a0 = __byte_perm(xv[0][i], xv[1][i], 0x5410);
          const uint32_t a1 = __byte_perm(xv[0][i], xv[1][i], 0x7632);
          const uint32_t a2 = __byte_perm(xv[2][i], xv[3][i], 0x5410);
          const uint32_t a3 = __byte_perm(xv[2][i], xv[3][i], 0x7632);
          if constexpr (kFp8) {
            mma_16816_f16(acc[i], a0, a1, a2, a3, bh0, bh1);
            mma_16816_f16(acc[i], a0, a1, a2, a3, bl0, bl1);
          } else {
            mma_16816(acc[i], a0, a1, a2, a3, bh0, bh1);
            mma_16816(acc[i], a0, a1, a2, a3, bl0, bl1);
          }
        }
      }

      // ---- this warp's result for the piece: the output itself when the
      // piece is the whole segment, else a partial (m, l, acc) slot that the
      // last unit of the segment combines with the other units' slots.
      float L_e = l_e, L_o = l_o;
#pragma unroll
      for (int d = 4; d < 32; d <<= 1) {
        L_e += __shfl_xor_sync(kFull, L_e, d);
        L_o += __shfl_xor_sync(kFull, L_o, d);
      }
      const int he = 2 * c, ho = 2 * c + 1;
#pragma unroll
      for (int i = 0; i < 8; ++i)
#pragma unroll
        for (int k = 0; k < 4; ++k) acc[i][k] *= p.out_scale;
      if (whole) {
        const int64_t row0 = int64_t(b) * p.Hq + h * group;
        uint32_t* oe = reinterpret_cast<uint32_t*>(p.out + (row0 + he) * kHeadDim);
        uint32_t* oo = reinterpret_cast<uint32_t*>(p.out + (row0 + ho) * kHeadDim);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 64 * (g >> 2) + 32 * ((i >> 1) & 1) + kk + 4 * (i >> 2) + 2 * (i & 1);
          if (he < group) oe[r >> 1] = pack_bf16x2(acc[i][0] / L_e, acc[i][2] / L_e);
          if (ho < group) oo[r >> 1] = pack_bf16x2(acc[i][1] / L_o, acc[i][3] / L_o);
        }
        if (g == 0 && p.lse) {
          if (he < group) p.lse[row0 + he] = m_e * p.sm_scale + logf(L_e);
          if (ho < group) p.lse[row0 + ho] = m_o * p.sm_scale + logf(L_o);
        }
      } else {
        const int64_t slot = int64_t(b) * Hkv + h + unit;
        float* pe = p.part + (slot * group + he) * kPartStride;
        float* po = p.part + (slot * group + ho) * kPartStride;
        if (g == 0) {
          if (he < group) {
            pe[0] = m_e;
            pe[1] = L_e;
          }
          if (ho < group) {
            po[0] = m_o;
            po[1] = L_o;
          }
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 64 * (g >> 2) + 32 * ((i >> 1) & 1) + kk + 4 * (i >> 2) + 2 * (i & 1);
          if (he < group) *reinterpret_cast<float2*>(pe + 4 + r) = make_float2(acc[i][0], acc[i][2]);
          if (ho < group) *reinterpret_cast<float2*>(po + 4 + r) = make_float2(acc[i][1], acc[i][3]);
        }
        // Publish the slot, then count it in.  The unit whose slot completes
        // the segment merges all of the segment's slots (in unit order) and
        // puts the counter back to zero for the next call.
        fence_acq_rel_gpu();
        __syncwarp();
        const int64_t seg = int64_t(b) * Hkv + h;
        const int64_t first = unit_of(seg_start, W, U), last = unit_of(seg_end - 1, W, U);
        // Every unit is non-empty when W >= U; otherwise each live unit holds one item.
        const uint32_t n_slots = static_cast<uint32_t>(W >= U ? last - first + 1 : n_b);
        uint32_t done = 0;
        if (lane == 0) done = (atomicAdd(p.count + seg, 1u) + 1u == n_slots) ? 1u : 0u;
        if (__shfl_sync(kFull, done, 0)) {
          fence_acq_rel_gpu();
          merge_segment(p, b, h, seg, first, last, W, U, lane);
          if (lane == 0) p.count[seg] = 0u;
        }
      }
      x = end;
    }
  }
  __syncthreads();
}

// Workspace: [0,16) error word | per-segment counters | partial slots.  The
// counter region has one fixed size (kMaxSegments words) whatever the shape,
// so no call's partial slots ever overlap another call's counters: a counter
// is zero before its first use (the workspace is zero-filled once when it is
// created) and the warp that merges a segment puts it back to zero, so every
// call leaves the region zeroed and a workspace may be reused with any shape.
constexpr int64_t kMaxSegments = int64_t(1) << 17;  // B * Hkv
constexpr int64_t kMinUnitPages = 4;
struct WsLayout {
  size_t count_off, part_off, total;
  int64_t grid;
};

WsLayout ws_layout(int B, int Hq, int Hkv, int max_seq_len, int num_sms) {
  WsLayout w{};
  const int64_t max_pages = (int64_t(max_seq_len) + kPageTokens - 1) / kPageTokens;
  const int64_t work = int64_t(B) * Hkv * max_pages;
  int64_t grid = int64_t(num_sms) * ctas_per_sm(B);
  // CTAs that can all be busy with at least kMinUnitPages pages per consumer
  // warp: spreading little work one page per warp would split every segment
  // into as many partial slots as it has pages, and their merge would walk
  // them a few per L2 round trip (64 pages: 25.0 us with one page per warp,
  // 15.6 us with four; eight or more starve mid-size work of SMs).
  const int64_t need = (work + kConsumerWarps * kMinUnitPages - 1) / (kConsumerWarps * kMinUnitPages);
  if (need < grid) grid = need;
  if (grid < 1) grid = 1;
  w.grid = grid;
  w.count_off = 256;
  w.part_off = w.count_off + size_t(kMaxSegments) * sizeof(uint32_t);
  const int group = Hkv > 0 ? Hq / Hkv : 1;
  const size_t slots = size_t(B) * Hkv + size_t(grid) * kConsumerWarps;
  w.total = w.part_off + slots * size_t(group) * kPartStride * sizeof(float);
  return w;
}

zf_status check_common(const uint16_t* q, int num_pages, const int32_t* page_table, int max_pages_per_seq,
                       const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv, int head_dim,
                       float sm_scale, const uint16_t* out, const void* ws) {
  if (B < 0 || Hq <= 0 || Hkv <= 0 || num_pages <= 0 || max_pages_per_seq <= 0 || max_seq_len < 0)
    return ZF_ERR_INVALID_ARG;
  if (head_dim != kHeadDim || Hq % Hkv != 0 || Hq / Hkv > kMaxGroup || B > kMaxBatch ||
      int64_t(B) * Hkv > kMaxSegments)
    return ZF_ERR_UNSUPPORTED;
  if (!std::isfinite(sm_scale)) return ZF_ERR_INVALID_ARG;
  if (int64_t(num_pages) * Hkv * kChunkBlocks > (int64_t(1) << 31)) return ZF_ERR_UNSUPPORTED;
  if (B == 0) return ZF_OK;
  if (!q || !page_table || !seq_lens || !out || !ws) return ZF_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(out, 16) || !aligned(page_table, 4) || !aligned(seq_lens, 4) ||
      !aligned(ws, 256))
    return ZF_ERR_INVALID_ARG;
  return ZF_OK;
}

zf_status check_compressed_pair(const zf_kv_compressed* k, const zf_kv_compressed* v, int64_t pool_values) {
  if (!k || !v) return ZF_ERR_INVALID_ARG;
  for (const zf_kv_compressed* c : {k, v}) {
    if (!c->payload || !c->offs || !c->base || !c->elig || c->n_values != pool_values ||
        c->payload_cap_bytes < 0 || !aligned(c->payload, 16) || !aligned(c->offs, 4) || !aligned(c->base, 16) ||
        !aligned(c->elig, 4))
      return ZF_ERR_INVALID_ARG;
  }
  return ZF_OK;
}

template <int kFmt>
zf_status launch(DecodeParams prm, int max_seq_len, void* ws, size_t ws_bytes, cudaStream_t stream) {
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const WsLayout L = ws_layout(prm.B, prm.Hq, prm.Hkv, max_seq_len, sms);
  if (ws_bytes < L.total) return ZF_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  prm.err = reinterpret_cast<uint32_t*>(w);
  prm.count = reinterpret_cast<uint32_t*>(w + L.count_off);
  prm.part = reinterpret_cast<float*>(w + L.part_off);
  prm.group = prm.Hq / prm.Hkv;
  prm.scale_log2 = prm.sm_scale * 1.4426950408889634f;
  // The register split inside the kernel draws on the launch allocation: a
  // build whose kernel was given fewer registers than the split assumes must
  // not run (its register increase would never complete).
  static const bool regs_ok = [] {
    cudaFuncAttributes a{};
    if (cudaFuncGetAttributes(&a, decode_attn_kernel<kFmt>) != cudaSuccess) return false;
    return a.numRegs >= kLaunchRegs;
  }();
  if (!regs_ok) return ZF_ERR_CUDA;
  const size_t smem = smem_bytes(prm.B);
  cudaError_t e = cudaFuncSetAttribute(decode_attn_kernel<kFmt>,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  // Launched with programmatic stream serialization: the kernel may be
  // scheduled while the previous kernel in the stream drains, and waits for
  // it (griddepcontrol.wait) before touching memory.
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
  e = cudaLaunchKernelEx(&cfg, decode_attn_kernel<kFmt>, prm);
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
  st = check_compressed_pair(k, v, int64_t(num_pages) * Hkv * kChunkValues);
  if (st != ZF_OK) return st;
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
  prm.out_scale = 1.0f;
  return launch<kFmtCompressed>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
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
  prm.out_scale = 1.0f;
  return launch<kFmtRaw>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

zf_status zf_decode_attention_paged(const uint16_t* q, const zf_kv_paged* k, const zf_kv_paged* v, int num_pages,
                                    const int32_t* page_table, int max_pages_per_seq, const int32_t* seq_lens,
                                    int max_seq_len, int B, int Hq, int Hkv, int head_dim, float sm_scale,
                                    uint16_t* out, float* lse, void* ws, size_t ws_bytes, zf_stream_t stream) {
  zf_status st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                              head_dim, sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  for (const zf_kv_paged* c : {k, v}) {
    if (!c || !c->data || !c->chunk_tab || c->data_cap_bytes < 0 || !aligned(c->data, 16) ||
        !aligned(c->chunk_tab, 8))
      return ZF_ERR_INVALID_ARG;
    if (c->num_chunks != int64_t(num_pages) * Hkv) return ZF_ERR_INVALID_ARG;
  }
  if (lse && !aligned(lse, 4)) return ZF_ERR_INVALID_ARG;
  DecodeParams prm{};
  prm.q = q;
  prm.k_data = static_cast<const uint8_t*>(k->data);
  prm.k_tab = k->chunk_tab;
  prm.k_cap_units = k->data_cap_bytes / kUnitBytes;
  prm.v_data = static_cast<const uint8_t*>(v->data);
  prm.v_tab = v->chunk_tab;
  prm.v_cap_units = v->data_cap_bytes / kUnitBytes;
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
  prm.out_scale = 1.0f;
  return launch<kFmtPaged>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
}

zf_status zf_decode_attention_fp8(const uint16_t* q, const uint8_t* k_pool, const uint8_t* v_pool, float k_scale,
                                  float v_scale, int num_pages, const int32_t* page_table, int max_pages_per_seq,
                                  const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                  int head_dim, float sm_scale, uint16_t* out, float* lse, void* ws,
                                  size_t ws_bytes, zf_stream_t stream) {
  zf_status st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                              head_dim, sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  if (!k_pool || !v_pool || !aligned(k_pool, 16) || !aligned(v_pool, 16)) return ZF_ERR_INVALID_ARG;
  if (!(std::isfinite(k_scale) && k_scale > 0.f) || !(std::isfinite(v_scale) && v_scale > 0.f))
    return ZF_ERR_INVALID_ARG;
  if (lse && !aligned(lse, 4)) return ZF_ERR_INVALID_ARG;
  DecodeParams prm{};
  prm.q = q;
  prm.k_fp8 = k_pool;
  prm.v_fp8 = v_pool;
  prm.page_table = page_table;
  prm.seq_lens = seq_lens;
  prm.out = out;
  prm.lse = lse;
  prm.num_pages = num_pages;
  prm.max_pages = max_pages_per_seq;
  prm.B = B;
  prm.Hq = Hq;
  prm.Hkv = Hkv;
  // Scores are formed on the unscaled E4M3 values: the K scale joins the
  // softmax scale, the V scale multiplies the output.
  prm.sm_scale = sm_scale * k_scale;
  prm.out_scale = v_scale;
  return launch<kFmtFp8>(prm, max_seq_len, ws, ws_bytes, reinterpret_cast<cudaStream_t>(stream));
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
constexpr size_t kNoAllocScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kNoAllocMaxDevices = 64;
__device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];
// Per device: the context the address was looked up in, and the address.
void* g_noalloc_ctx[kNoAllocMaxDevices] = {};
void* g_noalloc_ptr[kNoAllocMaxDevices] = {};
std::mutex g_noalloc_mu;

// The driver's current context, through the runtime's entry-point query (the
// library does not link the driver library itself); nullptr if unavailable.
void* current_context() {
  using GetCtx = int (*)(void**);
  static GetCtx get = [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<GetCtx>(nullptr);
    return reinterpret_cast<GetCtx>(fn);
  }();
  void* ctx = nullptr;
  if (!get || get(&ctx) != 0) return nullptr;
  return ctx;
}

// Device address of the scratch array for the current device.  It is looked
// up with the device current (host code may not use the array's name as an
// address) and kept; it is looked up again if the device's context has
// changed since (a device reset rebuilds the context and may move the array).
zf_status noalloc_scratch(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices) return ZF_ERR_CUDA;
  void* ctx = current_context();
  std::lock_guard<std::mutex> lock(g_noalloc_mu);
  if (!g_noalloc_ptr[dev] || !ctx || ctx != g_noalloc_ctx[dev]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) return ZF_ERR_CUDA;
    g_noalloc_ptr[dev] = p;
    g_noalloc_ctx[dev] = ctx;
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
  // Every argument check before anything is enqueued.
  st = check_common(q, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv, head_dim,
                    sm_scale, out, ws);
  if (st != ZF_OK || B == 0) return st;
  st = check_compressed_pair(k, v, int64_t(num_pages) * Hkv * kChunkValues);
  if (st != ZF_OK) return st;
  if (lse && !aligned(lse, 4)) return ZF_ERR_INVALID_ARG;
  const size_t need = zf_decode_workspace_size(B, Hq, Hkv, max_seq_len, 0);
  if (need == 0) return ZF_ERR_CUDA;
  if (need > zf::kNoAllocScratchBytes) return ZF_ERR_WORKSPACE;
  // The split counters must be zero when a kernel starts: the array is
  // zero-filled when the module loads and every call leaves them at zero
  // (the warp that merges a segment resets its counter, aborted calls
  // included).  Only the error word is cleared here, so that it describes
  // this call alone.
  if (cudaMemsetAsync(ws, 0, sizeof(uint32_t), reinterpret_cast<cudaStream_t>(stream)) != cudaSuccess)
    return ZF_ERR_CUDA;
  return zf_decode_attention(q, k, v, num_pages, page_table, max_pages_per_seq, seq_lens, max_seq_len, B, Hq, Hkv,
                             head_dim, sm_scale, out, lse, ws, zf::kNoAllocScratchBytes, stream);
}

extern "C" zf_status zf_noalloc_device_error(int* host_code) {
  if (!host_code) return ZF_ERR_INVALID_ARG;
  void* ws = nullptr;
  const zf_status st = zf::noalloc_scratch(&ws);
  if (st != ZF_OK) return st;
  uint32_t v = 0;
  if (cudaMemcpy(&v, ws, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return ZF_ERR_CUDA;
  *host_code = static_cast<int>(v);
  return ZF_OK;
}

// ---- decode attention with host buffers: the per-step inputs are copied in
// and the output copied out on the same stream, through staging regions that
// follow the decode workspace.
namespace zf {
namespace {

constexpr size_t kStagingAlign = 256;

size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

struct HostStaging {
  size_t q, pt, sl, out, lse, total;
};

HostStaging host_staging(size_t decode_bytes, int B, int Hq, int max_pages_per_seq) {
  HostStaging h{};
  h.q = align_up(decode_bytes, kStagingAlign);
  h.pt = align_up(h.q + size_t(B) * Hq * kHeadDim * sizeof(uint16_t), kStagingAlign);
  h.sl = align_up(h.pt + size_t(B) * max_pages_per_seq * sizeof(int32_t), kStagingAlign);
  h.out = align_up(h.sl + size_t(B) * sizeof(int32_t), kStagingAlign);
  h.lse = align_up(h.out + size_t(B) * Hq * kHeadDim * sizeof(uint16_t), kStagingAlign);
  h.total = h.lse + size_t(B) * Hq * sizeof(float);
  return h;
}

}  // namespace
}  // namespace zf

extern "C" size_t zf_decode_host_workspace_size(int B, int Hq, int Hkv, int max_pages_per_seq, int max_seq_len,
                                                int num_sms) {
  if (max_pages_per_seq <= 0) return 0;
  const size_t d = zf_decode_workspace_size(B, Hq, Hkv, max_seq_len, num_sms);
  if (d == 0) return 0;
  return zf::host_staging(d, B, Hq, max_pages_per_seq).total;
}

extern "C" zf_status zf_decode_attention_host(const uint16_t* q_host, const zf_kv_compressed* k,
                                              const zf_kv_compressed* v, int num_pages,
                                              const int32_t* page_table_host, int max_pages_per_seq,
                                              const int32_t* seq_lens_host, int max_seq_len, int B, int Hq, int Hkv,
                                              int head_dim, float sm_scale, uint16_t* out_host, float* lse_host,
                                              void* ws, size_t ws_bytes, zf_stream_t stream) {
  using namespace zf;
  // Shape checks (the device pointers handed to the kernel are carved from
  // ws below, so ws stands in for them here).
  zf_status st = check_common(static_cast<const uint16_t*>(ws), num_pages, static_cast<const int32_t*>(ws),
                              max_pages_per_seq, static_cast<const int32_t*>(ws), max_seq_len, B, Hq, Hkv,
                              head_dim, sm_scale, static_cast<const uint16_t*>(ws), ws);
  if (st != ZF_OK || B == 0) return st;
  if (!q_host || !page_table_host || !seq_lens_host || !out_host || !ws) return ZF_ERR_INVALID_ARG;
  st = check_compressed_pair(k, v, int64_t(num_pages) * Hkv * kChunkValues);
  if (st != ZF_OK) return st;
  const int sms = current_sm_count();
  if (sms <= 0) return ZF_ERR_CUDA;
  const size_t decode_bytes = ws_layout(B, Hq, Hkv, max_seq_len, sms).total;
  const HostStaging h = host_staging(decode_bytes, B, Hq, max_pages_per_seq);
  if (ws_bytes < h.total) return ZF_ERR_WORKSPACE;
  uint8_t* w = static_cast<uint8_t*>(ws);
  uint16_t* q_d = reinterpret_cast<uint16_t*>(w + h.q);
  int32_t* pt_d = reinterpret_cast<int32_t*>(w + h.pt);
  int32_t* sl_d = reinterpret_cast<int32_t*>(w + h.sl);
  uint16_t* out_d = reinterpret_cast<uint16_t*>(w + h.out);
  float* lse_d = reinterpret_cast<float*>(w + h.lse);
  const size_t q_bytes = size_t(B) * Hq * kHeadDim * sizeof(uint16_t);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = cudaMemcpyAsync(q_d, q_host, q_bytes, cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(pt_d, page_table_host, size_t(B) * max_pages_per_seq * sizeof(int32_t),
                        cudaMemcpyHostToDevice, s);
  if (e == cudaSuccess) e = cudaMemcpyAsync(sl_d, seq_lens_host, size_t(B) * sizeof(int32_t), cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return ZF_ERR_CUDA;
  st = zf_decode_attention(q_d, k, v, num_pages, pt_d, max_pages_per_seq, sl_d, max_seq_len, B, Hq, Hkv, head_dim,
                           sm_scale, out_d, lse_host ? lse_d : nullptr, ws, decode_bytes, stream);
  if (st != ZF_OK) return st;
  e = cudaMemcpyAsync(out_host, out_d, q_bytes, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess && lse_host)
    e = cudaMemcpyAsync(lse_host, lse_d, size_t(B) * Hq * sizeof(float), cudaMemcpyDeviceToHost, s);
  return cuda_status(e);
}
