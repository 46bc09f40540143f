/*
 * zf.h -- C ABI of the ZipFusion-style lossless BF16 KV-cache library for
 * NVIDIA B200 (sm_100a).
 *
 * The method ("Run AI Faster With Lossless Compressed Memory", the ZipFusion
 * summary, chapter "Twelve Bits and One Addition"): the KV cache stays
 * compressed in GPU memory; each block of BF16 values keeps one shared base
 * exponent and a four-bit exponent offset per value, with sign and mantissa
 * kept verbatim, so an eligible block costs twelve bits per value (75% of
 * BF16); blocks whose exponents are too spread out stay uncompressed; decode
 * attention rebuilds each value in registers with one integer addition.
 *
 * Conventions for every call below:
 *   - Pointers are DEVICE pointers unless a comment says "host".  The caller
 *     owns all memory; the library never allocates, frees or synchronises
 *     (except zf_get_device_error, which reads 4 bytes back).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL = legacy default
 *     stream) of the current device and runs asynchronously.
 *   - Argument errors are detected on the host before anything is enqueued
 *     and returned as a zf_status.  Data errors found on the device (a page
 *     id out of range, a sequence longer than its page-table row, a payload
 *     extent past the buffer's capacity) never cause an out-of-bounds access:
 *     the offending value is clamped and a bit is OR-ed into the device error
 *     word at the start of the workspace (see zf_get_device_error).
 *   - Every wait inside a kernel is bounded (about two seconds); a wait that
 *     gives up sets ZF_DEVERR_TIMEOUT and the kernel returns.
 *   - The library keeps no global state (the one exception is the fixed
 *     scratch of zf_decode_attention_noalloc); calls on different streams may
 *     run concurrently as long as they use different workspaces and outputs.
 *
 * Canonical compressed layout (one flat buffer of n_values BF16 words):
 *   block i = values [64 i, 64 i + 64); e_j = exponent field (bits 7..14).
 *   base[i]  = min_j e_j (u8), for every block.
 *   eligible = max_j e_j - base[i] <= 15;  elig bit i%32 of word i/32.
 *   offs[i]  = start of block i's payload in 16-byte units (u32), exclusive
 *              prefix sum of sizes (6 units eligible, 8 raw); offs[n_blocks]
 *              is the total.
 *   eligible payload (96 bytes):
 *     bytes [0, 64):  byte j = (mantissa_j << 1) | sign_(j xor 1)
 *     bytes [64, 96): byte k = (e_k - base) | (e_(k+32) - base) << 4
 *   raw payload (128 bytes), 16 bits per value as two byte planes:
 *     bytes [0, 64):   byte j = (mantissa_j << 1) | sign_(j xor 1), as above
 *     bytes [64, 128): byte j = e_j
 *   (every bit of the block is kept; both kinds share the sign/mantissa
 *   plane, so one decode sequence rebuilds either kind).
 * Paged use: a K (or V) pool is [num_pages][Hkv][16][128] BF16, so the
 * (page, kv head) chunk c = page * Hkv + head is blocks [32 c, 32 c + 32) and
 * one eligibility word.
 */
#ifndef ZF_H_
#define ZF_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t. */
typedef struct CUstream_st* zf_stream_t;

typedef enum {
  ZF_OK = 0,
  ZF_ERR_INVALID_ARG = 1,   /* null/misaligned pointer, negative size, ...   */
  ZF_ERR_UNSUPPORTED = 2,   /* head_dim != 128, Hq % Hkv, group > 8, ...      */
  ZF_ERR_WORKSPACE = 3,     /* workspace (or payload capacity) too small      */
  ZF_ERR_CUDA = 4,          /* a CUDA runtime call failed                     */
  ZF_ERR_BAD_INPUT = 5,     /* device error word reports clamped data         */
  ZF_ERR_TIMEOUT = 6        /* device error word reports a bounded wait expired */
} zf_status;

/* Bits of the device error word (first 4 bytes of a workspace). */
#define ZF_DEVERR_PAGE_ID 1u    /* page id outside [0, num_pages): read page 0     */
#define ZF_DEVERR_SEQ_LEN 2u    /* seq_len < 0 or > 16 * max_pages_per_seq: clamped */
#define ZF_DEVERR_EXTENT 4u     /* compressed chunk past payload capacity: skipped  */
#define ZF_DEVERR_TIMEOUT 8u    /* a bounded wait gave up                           */

/* One compressed flat BF16 buffer.  The struct itself is host memory; its
 * pointers are device memory owned by the caller. */
typedef struct {
  void* payload;              /* 16-byte aligned, payload_cap_bytes long          */
  uint32_t* offs;             /* [n_blocks + 1], 4-byte aligned                   */
  uint8_t* base;              /* [n_blocks], 16-byte aligned                      */
  uint32_t* elig;             /* [ceil(n_blocks / 32)], 4-byte aligned            */
  int64_t n_values;           /* multiple of 64                                   */
  int64_t payload_cap_bytes;  /* >= zf_compressed_bound(n_values) for compress   */
} zf_kv_compressed;

/* Paged form of a K or V pool (the two-level-metadata variant): every
 * (page, kv head) chunk of 2048 values (32 blocks) is one extent of `data`,
 * 16-byte aligned:
 *   chunk_tab[2c]     start of chunk c, in 16-byte units of data
 *   chunk_tab[2c + 1] its extent in 16-byte units (3 + its blocks' units)
 *   extent = 48-byte header (byte i: base exponent of block i; bytes 32..35:
 *            eligibility mask, bit i for block i, little-endian; 12 zero
 *            bytes), then the chunk's blocks in order, each laid out as in the
 *            canonical form.
 * The metadata is 8 bytes per chunk outside data (instead of 4 per block)
 * and a chunk is fetched with one copy.  A chunk whose page is still being
 * filled (zf_append_paged) names only the blocks written so far. */
typedef struct {
  void* data;               /* 16-byte aligned, data_cap_bytes long            */
  uint32_t* chunk_tab;      /* [num_chunks][2], 8-byte aligned                 */
  int64_t num_chunks;       /* num_pages * Hkv                                 */
  int64_t data_cap_bytes;   /* >= zf_paged_bound(num_chunks) for compress      */
} zf_kv_paged;

/* Library version (major * 10000 + minor * 100 + patch). */
int zf_version(void);

/* Human-readable name of a status (static string). */
const char* zf_status_string(zf_status s);

/* Host.  Worst-case payload bytes for n_values (every block raw):
 * 2 * n_values.  Returns 0 when n_values < 0 or not a multiple of 64. */
size_t zf_compressed_bound(int64_t n_values);

/* Host.  Scratch bytes zf_compress_kv needs for n_values (error word, tile
 * counter and one 8-byte scan state per 256 blocks). */
size_t zf_compress_workspace_size(int64_t n_values);

/* Compress `src` (n_values BF16 words, 16-byte aligned) into dst's buffers:
 * per-block min/max exponent, eligibility bits, the prefix-sum offset table
 * and the packed sign|mantissa and 4-bit offset planes (one pass over the
 * input, decoupled look-back scan, 16-byte stores).  dst->n_values must equal
 * n_values and dst->payload_cap_bytes must be >= zf_compressed_bound(n_values).
 * `ws` (ws_bytes >= zf_compress_workspace_size(n_values), 16-byte aligned) is
 * cleared by this call.  The total size lands in dst->offs[n_blocks] on the
 * device; read it after the stream completes to size an exact copy.
 * Source: ZipFusion summary, "Twelve Bits and One Addition" (shared base
 * exponent, 4-bit offsets, raw fallback). */
zf_status zf_compress_kv(const uint16_t* src, int64_t n_values, const zf_kv_compressed* dst, void* ws,
                         size_t ws_bytes, zf_stream_t stream);

/* Rebuild src's n_values BF16 words into dst (16-byte aligned): each eligible
 * value as base + 4-bit offset (one integer add), raw blocks copied.  A block
 * whose payload (from offs[i]) would pass payload_cap_bytes is skipped and
 * its values in dst are left as they were; this call has no error word, and
 * zf_validate_compressed reports such buffers.
 * Source: ZipFusion summary, "Twelve Bits and One Addition". */
zf_status zf_decompress_kv(const zf_kv_compressed* src, uint16_t* dst, zf_stream_t stream);

/* Read-only consistency check of a compressed buffer: every block size is 6
 * or 8 units and agrees with its eligibility bit, offs[0] == 0, offs is the
 * running sum, offs[n_blocks] * 16 <= payload_cap_bytes, and base + every
 * stored offset of an eligible block <= 255.  Adds the number of bad blocks
 * (plus one if offs[0] or the total is wrong) to *d_bad_count (device int32,
 * caller zeroes it). */
zf_status zf_validate_compressed(const zf_kv_compressed* c, int32_t* d_bad_count, zf_stream_t stream);

/* Host.  Workspace bytes for a decode-attention call with these shapes on a
 * device with num_sms SMs (num_sms <= 0: ask the current device).  The same
 * workspace serves zf_decode_attention and zf_decode_attention_raw. */
size_t zf_decode_workspace_size(int B, int Hq, int Hkv, int max_seq_len, int num_sms);

/* Fused split-K GQA decode attention over the COMPRESSED paged cache.
 *   q            [B][Hq][128] BF16, 16-byte aligned
 *   k, v         host structs describing compressed pools of
 *                num_pages * Hkv * 16 * 128 values each
 *   page_table   [B][max_pages_per_seq] int32, row b lists sequence b's pages
 *   seq_lens     [B] int32 tokens per sequence (device), 0 allowed
 *   max_seq_len  host upper bound of seq_lens (sizes the split plan only)
 *   Hq % Hkv == 0, Hq / Hkv <= 8, head_dim == 128, B <= 4096
 *   sm_scale     softmax scale (usually 1/sqrt(128))
 *   out          [B][Hq][128] BF16 (round to nearest even), 16-byte aligned
 *   lse          [B][Hq] float natural-log sum-exp, or NULL
 *   ws           >= zf_decode_workspace_size(B, Hq, Hkv, max_seq_len, 0)
 *                bytes, 256-byte aligned, ZERO-FILLED before its first use
 *                (e.g. cudaMemset); its first 16 bytes are the sticky device
 *                error word (see zf_clear_device_error), then come the split
 *                counters, which every call leaves at zero, so one workspace
 *                serves any later call whose shape fits it.  B * Hkv <= 131072.
 * One kernel: each of the twelve consumer warps of a persistent CTA per SM
 * takes an equal share of all (sequence, kv head, page) work; producer warps
 * stream the pages' compressed K/V chunks into shared memory with bulk (TMA)
 * copies; the consumers rebuild the values in registers and run the online
 * softmax; the warp that finishes a sequence/head last merges the other
 * warps' partial results.  A sequence of length 0 gives out = 0 and
 * lse = -inf.  The result is bitwise identical to zf_decode_attention_raw on
 * the same values.
 * Source: ZipFusion summary, "Twelve Bits and One Addition" and "Why Memory
 * Sets the Speed" (compressed cache read directly by attention). */
zf_status zf_decode_attention(const uint16_t* q, const zf_kv_compressed* k, const zf_kv_compressed* v,
                              int num_pages, const int32_t* page_table, int max_pages_per_seq,
                              const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv, int head_dim,
                              float sm_scale, uint16_t* out, float* lse, void* ws, size_t ws_bytes,
                              zf_stream_t stream);

/* The same attention over an UNCOMPRESSED paged cache: k_pool, v_pool are
 * [num_pages][Hkv][16][128] BF16 (16-byte aligned).  Same plan, same
 * arithmetic, same reduction order as zf_decode_attention: the in-library
 * comparison for the compressed kernel. */
zf_status zf_decode_attention_raw(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                                  int num_pages, const int32_t* page_table, int max_pages_per_seq,
                                  const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                  int head_dim, float sm_scale, uint16_t* out, float* lse, void* ws,
                                  size_t ws_bytes, zf_stream_t stream);

/* ---- Paged form (see zf_kv_paged). */

/* Host.  Worst-case data bytes of num_chunks chunks (every block raw). */
size_t zf_paged_bound(int64_t num_chunks);

/* Compress num_chunks * 2048 BF16 values (a pool [num_pages][Hkv][16][128],
 * 16-byte aligned) into the paged form, chunks laid end to end in chunk
 * order.  Same block encoding, one pass and workspace as zf_compress_kv
 * (ws >= zf_compress_workspace_size(num_chunks * 2048)). */
zf_status zf_compress_paged(const uint16_t* src, int64_t num_chunks, const zf_kv_paged* dst, void* ws,
                            size_t ws_bytes, zf_stream_t stream);

/* Rebuild the num_chunks * 2048 values of a paged pool into dst (16-byte
 * aligned); blocks a filling chunk has not written yet are rebuilt from
 * whatever its extent holds, and a chunk whose start is within 4144 bytes of
 * the end of data (past data_cap_bytes) is skipped. */
zf_status zf_decompress_paged(const zf_kv_paged* src, uint16_t* dst, zf_stream_t stream);

/* zf_decode_attention over paged-form pools: per page one bulk copy per K
 * or V chunk (header and blocks together).  Arguments, workspace, errors
 * and results otherwise as zf_decode_attention; the output is bitwise
 * identical to it (and to the raw twin) on the same values.  An extent
 * longer than a chunk can be, or past data_cap_bytes, is skipped and sets
 * ZF_DEVERR_EXTENT. */
zf_status zf_decode_attention_paged(const uint16_t* q, const zf_kv_paged* k, const zf_kv_paged* v, int num_pages,
                                    const int32_t* page_table, int max_pages_per_seq, const int32_t* seq_lens,
                                    int max_seq_len, int B, int Hq, int Hkv, int head_dim, float sm_scale,
                                    uint16_t* out, float* lse, void* ws, size_t ws_bytes, zf_stream_t stream);

/* ---- Append-time compression into a paged pool.  A decode step adds one
 * token per sequence; zf_append_paged compresses its two blocks per kv head
 * at once (the summary leaves this step, initial compression, out of its
 * timing).  Layout of pool->data: [packed region | staging extents].  The
 * chunk of a page that is still filling sits in the staging extent of its
 * (sequence, kv head) (header + up to 32 raw blocks, 4144 bytes) and grows
 * there; when the page's 16th token arrives the finished extent is moved to
 * the packed region at *packed_cursor (16-byte units, advanced atomically)
 * and chunk_tab points there.  Decode reads filling and full pages alike. */

/* Host.  Bytes of staging extents for B sequences x Hkv heads. */
size_t zf_append_staging_bytes(int B, int Hkv);

/* Append one token per sequence.
 *   vals          [B][Hkv][128] BF16 (device, 8-byte aligned): the new K (or
 *                 V) of each sequence
 *   page_table    [B][max_pages_per_seq] (device); the page of the token
 *                 must already be assigned
 *   positions     [B] int32 (device): index of the token in its sequence, or
 *                 -1 to skip the sequence.  Tokens of a sequence must be
 *                 appended in order, each once; a page is filled by one
 *                 sequence only.
 *   staging_offset byte offset of the staging extents in pool->data
 *                 (multiple of 16; the packed region is [0, staging_offset),
 *                 staging takes zf_append_staging_bytes(B, Hkv) after it)
 *   packed_cursor device u32: used 16-byte units of the packed region
 *   err           device u32 error word (ZF_DEVERR_* bits) or NULL
 * Errors: a position past the page-table row, a bad page id, or a full
 * packed region set a bit of *err and leave that chunk unchanged (a full
 * page that found no room stays in staging until its slot is reused). */
zf_status zf_append_paged(const zf_kv_paged* pool, const uint16_t* vals, const int32_t* page_table,
                          int max_pages_per_seq, const int32_t* positions, int B, int Hkv, int64_t staging_offset,
                          uint32_t* packed_cursor, uint32_t* err, zf_stream_t stream);

/* The K and V appends of one decode step in one launch: the same chunks as
 * zf_append_paged(k_pool, k_vals, ...) followed by zf_append_paged(v_pool,
 * v_vals, ...) with the same page_table and positions (where a filled page
 * lands in the packed region follows the order of the cursor's atomic
 * updates, in both forms), at the cost of one launch (an append moves about
 * 0.3 KB per (sequence, kv head), so its time is launch latency).  k_pool and v_pool: two distinct pools with the same
 * num_chunks whose data buffers do not overlap; each has its own staging
 * offset and packed cursor (the cursors must differ).  Device errors of both
 * go to *err.  Argument errors as zf_append_paged, plus ZF_ERR_INVALID_ARG
 * for pools that share a buffer or a cursor or differ in num_chunks. */
zf_status zf_append_paged_kv(const zf_kv_paged* k_pool, const zf_kv_paged* v_pool, const uint16_t* k_vals,
                             const uint16_t* v_vals, const int32_t* page_table, int max_pages_per_seq,
                             const int32_t* positions, int B, int Hkv, int64_t k_staging_offset,
                             int64_t v_staging_offset, uint32_t* k_packed_cursor, uint32_t* v_packed_cursor,
                             uint32_t* err, zf_stream_t stream);

/* ---- FP8 E4M3 comparator (lossy).  The summary's chapter "Lossless or FP8"
 * sets the method against an FP8 KV cache, which halves the cache but changes
 * the values; these two calls give that comparison on the same kernel.
 * E4M3 = OCP 8-bit floating point: 1 sign bit, 4 exponent bits (bias 7), 3
 * mantissa bits, no infinities, S.1111.111 NaN, largest finite 448.  A pool
 * keeps one scale: value = E4M3(code) * scale. */

/* Quantize n_values BF16 values (device, 16-byte aligned, n_values a
 * multiple of 8) into E4M3 codes (device, 8-byte aligned, n_values bytes):
 * code = E4M3 nearest to (float)value * inv_scale, the product in single
 * precision, round to nearest even, saturating at +-448 (inf too).
 * inv_scale = 1 / scale, finite and > 0.  NaN inputs give a NaN code. */
zf_status zf_fp8_quantize(const uint16_t* src, int64_t n_values, float inv_scale, uint8_t* dst,
                          zf_stream_t stream);

/* Decode attention over E4M3 pools k_pool, v_pool ([num_pages][Hkv][16][128]
 * codes, 16-byte aligned) with scales k_scale, v_scale (finite, > 0): the
 * same plan and softmax as zf_decode_attention, values rebuilt as
 * E4M3 -> f16 (exact) and multiplied in f16 (q converted once, P as f16 hi +
 * lo); scores use sm_scale * k_scale and the output is multiplied by
 * v_scale.  All other arguments, the workspace and the error reporting are
 * those of zf_decode_attention. */
zf_status zf_decode_attention_fp8(const uint16_t* q, const uint8_t* k_pool, const uint8_t* v_pool, float k_scale,
                                  float v_scale, int num_pages, const int32_t* page_table, int max_pages_per_seq,
                                  const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                  int head_dim, float sm_scale, uint16_t* out, float* lse, void* ws,
                                  size_t ws_bytes, zf_stream_t stream);

/* zf_decode_attention for callers that cannot give the library any scratch
 * memory: for example a plugin that a host inference engine calls with only
 * its input and output buffers, or a process that reserves all device memory
 * at start-up and allows no allocation while it serves.  The source summary
 * has no counterpart to this call; it exists for those callers.
 *
 * Arguments and results are those of zf_decode_attention, without ws and
 * ws_bytes.  The scratch (error word, split plan, partial results) is one
 * fixed 8 MiB array inside the library's device image: every GPU that loads
 * the library holds it until the process exits.  Shapes whose scratch
 * (zf_decode_workspace_size) exceeds 8 MiB are rejected with
 * ZF_ERR_WORKSPACE, e.g. B = 32, Hq = 32, Hkv = 8 fits on a 148-SM B200.
 * The call allocates nothing: no cudaMalloc, no cudaFree.
 * The first call on a device looks up the array's device address (once per
 * device, with that device current, and again only if the device's context
 * has changed, e.g. after cudaDeviceReset); make that first call before any
 * stream capture.  All calls on a device share the one array and it keeps
 * the last call's contents, so calls whose kernels overlap on the GPU
 * (different streams, or without ordering between them) race and give wrong
 * results.  Every argument is checked before anything is enqueued; the
 * device error word is cleared at the start of each call and
 * zf_noalloc_device_error reads it back. */
zf_status zf_decode_attention_noalloc(const uint16_t* q, const zf_kv_compressed* k, const zf_kv_compressed* v,
                                      int num_pages, const int32_t* page_table, int max_pages_per_seq,
                                      const int32_t* seq_lens, int max_seq_len, int B, int Hq, int Hkv,
                                      int head_dim, float sm_scale, uint16_t* out, float* lse, zf_stream_t stream);

/* The device error word of the current device's zf_decode_attention_noalloc
 * scratch (ZF_DEVERR_* bits of the last call on that device), for the same
 * callers; it allocates nothing.  Blocking: it waits for all earlier work on
 * the device (a synchronous 4-byte copy).  host_code: host int*. */
zf_status zf_noalloc_device_error(int* host_code);

/* ---- Decode attention with HOST buffers: one call per decode step for a
 * caller whose per-step inputs and output live in host memory.  Enqueued on
 * stream, in order:
 *   1. copies of q_host [B][Hq][128] BF16, page_table_host
 *      [B][max_pages_per_seq] int32 and seq_lens_host [B] int32 into staging
 *      regions that follow the decode scratch inside ws;
 *   2. zf_decode_attention on the staged copies (k, v: device pools as for
 *      zf_decode_attention);
 *   3. copies of the output to out_host [B][Hq][128] BF16 and, when lse_host
 *      is not NULL, of the log-sum-exp to lse_host [B][Hq] float.
 * The host buffers need no alignment.  With page-locked (pinned) host memory
 * the copies are asynchronous; the caller synchronises the stream before it
 * reads out_host or lse_host, and keeps every host buffer alive until then.
 * With pageable memory the CUDA runtime may block inside the copies.
 * ws: device, 256-byte aligned, at least zf_decode_host_workspace_size bytes,
 * zero-filled once before first use like the zf_decode_attention workspace
 * (its first zf_decode_workspace_size bytes are that workspace, so the device
 * error word is read the same way).  Argument errors return before anything
 * is enqueued; shapes and limits are those of zf_decode_attention. */

/* Host.  Bytes of ws for zf_decode_attention_host (0 on invalid arguments;
 * num_sms <= 0 queries the current device). */
size_t zf_decode_host_workspace_size(int B, int Hq, int Hkv, int max_pages_per_seq, int max_seq_len,
                                     int num_sms);

zf_status zf_decode_attention_host(const uint16_t* q_host, const zf_kv_compressed* k, const zf_kv_compressed* v,
                                   int num_pages, const int32_t* page_table_host, int max_pages_per_seq,
                                   const int32_t* seq_lens_host, int max_seq_len, int B, int Hq, int Hkv,
                                   int head_dim, float sm_scale, uint16_t* out_host, float* lse_host, void* ws,
                                   size_t ws_bytes, zf_stream_t stream);

/* ---- Check of the bounded waits.  Every wait inside the kernels is a
 * shared-memory barrier wait that gives up after about two seconds (and,
 * inside the decode kernel, as soon as another warp of its CTA has given
 * up); a wait that gives up sets ZF_DEVERR_TIMEOUT and the kernel returns, so
 * the context stays usable.  zf_check_bounded_wait runs those same wait
 * functions in a one-CTA kernel on a barrier whose completion the check
 * controls, so each outcome can be observed on a device:
 *   ZF_WAITCHECK_TIMEOUT        nothing completes the barrier: the wait that
 *                               can be called off gives up at the limit;
 *   ZF_WAITCHECK_ABORT          a second warp raises the CTA's abort flag
 *                               after 1 ms: the wait is called off;
 *   ZF_WAITCHECK_COMPLETE       a second warp completes the barrier after
 *                               1 ms: the wait succeeds;
 *   ZF_WAITCHECK_PLAIN_TIMEOUT  nothing completes the barrier: the plain
 *                               bounded wait gives up at the limit.
 * Two more modes run the compress kernel's look-back (the single-pass prefix
 * sum's wait for predecessor tiles) for tile 5 over fabricated predecessor
 * states in the library's own device memory (tile 0 inclusive 10, tiles 1
 * and 2 aggregate 7, tile 4 aggregate 3):
 *   ZF_WAITCHECK_LOOKBACK_TIMEOUT   tile 3 never publishes: the look-back
 *                                   gives up at the limit;
 *   ZF_WAITCHECK_LOOKBACK_COMPLETE  a second warp publishes tile 3's
 *                                   aggregate 5 after 1 ms: the look-back
 *                                   ends with the prefix 32.
 * Concurrent look-back checks share those states and must not overlap.
 * One more runs the compress kernel itself, on 4 tiles of zeros in the
 * library's own device memory, with CTA 0's first stage fill withheld (no
 * copy, no arrival):
 *   ZF_WAITCHECK_COMPRESS_STALL     the compute warps' wait on that stage
 *                                   gives up at the limit and stops the CTA
 *                                   (its loader and look-back warp follow),
 *                                   and the other CTAs' look-backs give up on
 *                                   the tile that never publishes; result[0]
 *                                   = -1 when ZF_DEVERR_TIMEOUT was set, 1
 *                                   otherwise; result[1] = nanoseconds the
 *                                   whole launch took.  It keeps a few SMs
 *                                   busy for about four seconds; overlapping
 *                                   stall checks share the tiles.
 * result: device int64[2], 8-byte aligned: result[0] = 1 (completed, and
 * for the look-back with the right prefix), 2 (look-back completed with a
 * wrong prefix), 0 (called off) or -1 (gave up); result[1] = nanoseconds
 * the wait took
 * (%globaltimer).  err: device u32 error word (for example the first word of
 * a decode workspace, so zf_get_device_error reads it); a wait that gives up
 * ORs ZF_DEVERR_TIMEOUT into it.  The two timeout modes keep the GPU busy
 * for about two seconds on one SM. */
typedef enum {
  ZF_WAITCHECK_TIMEOUT = 0,
  ZF_WAITCHECK_ABORT = 1,
  ZF_WAITCHECK_COMPLETE = 2,
  ZF_WAITCHECK_PLAIN_TIMEOUT = 3,
  ZF_WAITCHECK_LOOKBACK_TIMEOUT = 4,
  ZF_WAITCHECK_LOOKBACK_COMPLETE = 5,
  ZF_WAITCHECK_COMPRESS_STALL = 6
} zf_waitcheck_mode;

zf_status zf_check_bounded_wait(int mode, int64_t* result, uint32_t* err, zf_stream_t stream);

/* Zero the device error word of a workspace (async on stream). */
zf_status zf_clear_device_error(void* ws, zf_stream_t stream);

/* Copy the device error word of a workspace to *host_code (host int; this
 * call synchronises with the device).  Returns ZF_ERR_TIMEOUT if the timeout
 * bit is set, ZF_ERR_BAD_INPUT if any other bit is set, else ZF_OK. */
zf_status zf_get_device_error(const void* ws, int* host_code);

#ifdef __cplusplus
}
#endif

#endif /* ZF_H_ */
