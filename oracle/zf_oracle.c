/*
 * CPU oracle for lossless BF16 KV-cache compression ("ZipFusion") and for
 * paged GQA decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the tests, the smoke check and the CPU
 * baseline leg of the benchmark may load this library.  It shares no code,
 * header, table or constant with the CUDA path in
 * decode_attention_zipfusion_b200/csrc and must never be linked into it.
 *
 * It is deliberately plain: one value at a time, no blocking, no
 * vectorisation, no threads.  Floating point is fp64.
 *
 * Source of the method: "Run AI Faster With Lossless Compressed Memory"
 * (chooseto.ai video summary of the ZipFusion preprint), the paragraph on
 * "Twelve Bits and One Addition":
 *   - each block keeps one shared base exponent;
 *   - each value keeps a four-bit exponent offset, so an eligible block
 *     costs twelve bits per value (75% of BF16);
 *   - blocks whose exponents are too spread out stay uncompressed;
 *   - values are rebuilt with a single integer addition.
 * The pages fix nothing else.  The readings taken where they are silent:
 *   R1 block = 64 consecutive values of the flat buffer;
 *   R2 base exponent = the smallest 8-bit exponent field in the block,
 *      so every offset is an unsigned 0..15;
 *   R3 eligible  <=>  emax - emin <= 15 (the spread fits in four bits);
 *   R4 the raw exponent field is used for every bit pattern (zeros,
 *      subnormals, Inf and NaN need no special case);
 *   R5 payload layout of an eligible block of n values (n even):
 *        bytes [0, n):      one sign/mantissa byte per value j:
 *                           (mantissa_j << 1) | sign_(j xor 1)
 *                           i.e. each byte carries its own 7 mantissa bits
 *                           and the sign of its pair partner (values 2p and
 *                           2p+1 form a pair);
 *        bytes [n, 3n/2):   byte k holds offset_k in its low nibble and
 *                           offset_(k + n/2) in its high nibble;
 *      an ineligible ("raw") block stays at 16 bits per value, laid out
 *      as two byte planes: bytes [0, n) the same sign/mantissa bytes as
 *      above, bytes [n, 2n) the 8-bit exponent field of each value.  The
 *      pages only say such blocks stay uncompressed; this byte order keeps
 *      every bit (it is a permutation of the block's bits) and gives both
 *      kinds of block the same sign/mantissa plane, so a decoder rebuilds
 *      either kind with the same steps (exponent = byte of the exponent
 *      plane instead of base + offset);
 *   R6 blocks are laid end to end; the offset table is the exclusive prefix
 *      sum of block sizes.  The canonical (n = 64) form counts it in
 *      16-byte units (eligible 6, raw 8), with one extra final entry.
 *   R7 decode attention: s_t = scale * q.k_t over t < seq_len, softmax,
 *      o = sum_t p_t v_t, lse = natural log of sum exp(s_t); query head h
 *      reads kv head h / (Hq / Hkv).
 *   R9 paged form (one extent per (page, kv head) chunk): see below.
 *   R8 the lossy comparator of the chapter "Lossless or FP8" (FP8 halves
 *      the cache and is lossy): values are stored as FP8 E4M3 codes with one
 *      scale per pool, value = decode(code) * scale; a value is quantized as
 *      the E4M3 code nearest to (float)value * (float)(1/scale), ties to the
 *      even code, saturating at +-448 (the single-precision product is the
 *      one the GPU forms before its own rounding, so both sides decide each
 *      code on the same number).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ---------------------------------------------------------------- codec */

static int exponent_field(uint16_t w) { return (w >> 7) & 0xFF; }
static int sign_bit(uint16_t w) { return (w >> 15) & 1; }
static int mantissa_bits(uint16_t w) { return w & 0x7F; }

/* Smallest and largest exponent field of one block (base-exponent rule). */
void zfo_block_stats(const uint16_t* w, int n, int* emin, int* emax) {
  int lo = 255, hi = 0;
  for (int j = 0; j < n; ++j) {
    int e = exponent_field(w[j]);
    if (e < lo) lo = e;
    if (e > hi) hi = e;
  }
  *emin = lo;
  *emax = hi;
}

/* A block is stored compressed iff every exponent is base + a 4-bit offset. */
int zfo_block_eligible(const uint16_t* w, int n) {
  int emin, emax;
  zfo_block_stats(w, n, &emin, &emax);
  return (emax - emin) <= 15;
}

/* Bytes one block of n values takes: 12 bits per value when eligible,
 * 16 bits per value when stored raw. */
int64_t zfo_block_bytes(int n, int eligible) {
  return eligible ? (int64_t)n * 12 / 8 : (int64_t)n * 2;
}

/* Encode one block into out[]; returns its size in bytes. */
int64_t zfo_pack_block(const uint16_t* w, int n, uint8_t* out, uint8_t* base_out,
                       int* eligible_out) {
  int emin, emax;
  zfo_block_stats(w, n, &emin, &emax);
  int eligible = (emax - emin) <= 15;
  *base_out = (uint8_t)emin;
  *eligible_out = eligible;
  for (int j = 0; j < n; ++j) {
    int partner = j ^ 1;
    out[j] = (uint8_t)((mantissa_bits(w[j]) << 1) | sign_bit(w[partner]));
  }
  if (eligible) {
    for (int k = 0; k < n / 2; ++k) {
      int off_lo = exponent_field(w[k]) - emin;
      int off_hi = exponent_field(w[k + n / 2]) - emin;
      out[n + k] = (uint8_t)(off_lo | (off_hi << 4));
    }
  } else {
    for (int j = 0; j < n; ++j) out[n + j] = (uint8_t)exponent_field(w[j]);
  }
  return zfo_block_bytes(n, eligible);
}

/* Decode one block.  For an eligible block the exponent of value j is
 * rebuilt as base + offset_j: the single integer addition of the method; a
 * raw block stores it whole. */
void zfo_unpack_block(const uint8_t* in, int n, uint8_t base, int eligible, uint16_t* w) {
  for (int j = 0; j < n; ++j) {
    int e;
    if (eligible) {
      int off = (j < n / 2) ? (in[n + j] & 0x0F) : (in[n + j - n / 2] >> 4);
      e = base + off;
    } else {
      e = in[n + j];
    }
    int m = in[j] >> 1;
    int s = in[j ^ 1] & 1;
    w[j] = (uint16_t)(((s << 15) | ((e & 0xFF) << 7) | m) & 0xFFFF);
  }
}

/* Compress n_values (a multiple of n) with block size n.  offs_bytes has
 * n_blocks + 1 entries; eligible has one byte (0/1) per block.  Returns the
 * total payload size in bytes. */
int64_t zfo_compress_general(const uint16_t* src, int64_t n_values, int n, uint8_t* payload,
                             int64_t* offs_bytes, uint8_t* base, uint8_t* eligible) {
  int64_t n_blocks = n_values / n;
  int64_t pos = 0;
  for (int64_t i = 0; i < n_blocks; ++i) {
    int el;
    offs_bytes[i] = pos;
    pos += zfo_pack_block(src + i * n, n, payload + pos, &base[i], &el);
    eligible[i] = (uint8_t)el;
  }
  offs_bytes[n_blocks] = pos;
  return pos;
}

/* Decompress blocks [i0, i1) of a buffer produced by zfo_compress_general;
 * dst receives values [i0*n, i1*n). */
void zfo_decompress_general(const uint8_t* payload, const int64_t* offs_bytes, const uint8_t* base,
                            const uint8_t* eligible, int n, int64_t i0, int64_t i1,
                            uint16_t* dst) {
  for (int64_t i = i0; i < i1; ++i)
    zfo_unpack_block(payload + offs_bytes[i], n, base[i], eligible[i], dst + (i - i0) * n);
}

/* Canonical form (block = 64 values): offsets in 16-byte units (u32),
 * eligibility as a bitmask (bit i%32 of word i/32).  Returns payload units. */
int64_t zfo_compress(const uint16_t* src, int64_t n_values, uint8_t* payload, uint32_t* offs,
                     uint8_t* base, uint32_t* elig) {
  const int n = 64;
  int64_t n_blocks = n_values / n;
  int64_t pos = 0;
  for (int64_t w = 0; w < (n_blocks + 31) / 32; ++w) elig[w] = 0;
  for (int64_t i = 0; i < n_blocks; ++i) {
    int el;
    offs[i] = (uint32_t)(pos / 16);
    pos += zfo_pack_block(src + i * n, n, payload + pos, &base[i], &el);
    if (el) elig[i / 32] |= (uint32_t)1 << (i % 32);
  }
  offs[n_blocks] = (uint32_t)(pos / 16);
  return pos / 16;
}

/* Decompress canonical blocks [i0, i1); dst receives values [64*i0, 64*i1). */
void zfo_decompress(const uint8_t* payload, const uint32_t* offs, const uint8_t* base,
                    const uint32_t* elig, int64_t i0, int64_t i1, uint16_t* dst) {
  for (int64_t i = i0; i < i1; ++i) {
    int el = (elig[i / 32] >> (i % 32)) & 1;
    zfo_unpack_block(payload + (int64_t)offs[i] * 16, 64, base[i], el, dst + (i - i0) * 64);
  }
}

/* ---------------------------------------------------------- paged form */

/* Reading R9: a paged pool keeps each (page, kv head) chunk of 32 blocks
 * (2048 values) as one extent, so that a chunk can be fetched in one piece
 * and grown while its page fills:
 *   chunk_tab[2c]     start of chunk c in 16-byte units of `data`
 *   chunk_tab[2c + 1] its extent in 16-byte units: 3 + its blocks' units
 *   extent = header (48 bytes: the base exponent of each of its 32 blocks,
 *            the eligibility mask as a little-endian u32 with bit i for
 *            block i, 12 zero bytes), then its blocks in order, each laid
 *            out as in R5.
 * The header of a chunk whose page is still filling describes only the
 * blocks written so far (the others: base 0, mask bit 0). */

/* Header and the first n_blocks blocks of the chunk whose 2048 values are
 * at src; returns the extent in bytes. */
int64_t zfo_pack_chunk(const uint16_t* src, int n_blocks, uint8_t* out) {
  uint32_t mask = 0;
  int64_t p = 48;
  memset(out, 0, 48);
  for (int i = 0; i < n_blocks; ++i) {
    int el;
    p += zfo_pack_block(src + (int64_t)i * 64, 64, out + p, &out[i], &el);
    if (el) mask |= (uint32_t)1 << i;
  }
  out[32] = (uint8_t)(mask & 0xFF);
  out[33] = (uint8_t)((mask >> 8) & 0xFF);
  out[34] = (uint8_t)((mask >> 16) & 0xFF);
  out[35] = (uint8_t)(mask >> 24);
  return p;
}

/* Compress num_chunks full chunks laid end to end in chunk order.  Returns
 * the total size in 16-byte units. */
int64_t zfo_compress_paged(const uint16_t* src, int64_t num_chunks, uint8_t* data, uint32_t* chunk_tab) {
  int64_t pos = 0;
  for (int64_t c = 0; c < num_chunks; ++c) {
    int64_t bytes = zfo_pack_chunk(src + c * 2048, 32, data + pos);
    chunk_tab[2 * c] = (uint32_t)(pos / 16);
    chunk_tab[2 * c + 1] = (uint32_t)(bytes / 16);
    pos += bytes;
  }
  return pos / 16;
}

/* Decompress the first n_blocks blocks of every chunk (values
 * [2048 c, 2048 c + 64 n_blocks) of dst). */
void zfo_decompress_paged(const uint8_t* data, const uint32_t* chunk_tab, int64_t num_chunks, int n_blocks,
                          uint16_t* dst) {
  for (int64_t c = 0; c < num_chunks; ++c) {
    const uint8_t* hdr = data + (int64_t)chunk_tab[2 * c] * 16;
    uint32_t mask = (uint32_t)hdr[32] | ((uint32_t)hdr[33] << 8) | ((uint32_t)hdr[34] << 16) |
                    ((uint32_t)hdr[35] << 24);
    int64_t p = 48;
    for (int i = 0; i < n_blocks; ++i) {
      int el = (mask >> i) & 1;
      zfo_unpack_block(hdr + p, 64, hdr[i], el, dst + c * 2048 + (int64_t)i * 64);
      p += zfo_block_bytes(64, el);
    }
  }
}

/* ------------------------------------------------------------ attention */

static double bf16_to_double(uint16_t w) {
  uint32_t bits = (uint32_t)w << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* ------------------------------------------------------------- FP8 E4M3 */

/* E4M3 as defined by the OCP 8-bit floating point specification: 1 sign bit,
 * 4 exponent bits with bias 7, 3 mantissa bits; no infinities; S.1111.111 is
 * NaN; the largest finite magnitude is 1.75 * 2^8 = 448; exponent field 0
 * holds the subnormals m * 2^-9. */
double zfo_e4m3_decode(uint8_t c) {
  int s = c >> 7, e = (c >> 3) & 0xF, m = c & 7;
  double v;
  if (e == 15 && m == 7) return NAN;
  if (e == 0)
    v = m * ldexp(1.0, -9);
  else
    v = (1.0 + m / 8.0) * ldexp(1.0, e - 7);
  return s ? -v : v;
}

/* The E4M3 code nearest to x: ties go to the even code (even mantissa),
 * magnitudes at or beyond 448 saturate to +-448, NaN gives 0x7F. */
uint8_t zfo_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  int sign = signbit(x) ? 0x80 : 0;
  double a = fabs(x);
  if (a >= 448.0) return (uint8_t)(sign | 0x7E);
  /* codes 0x00..0x7E are the finite non-negative values in increasing order */
  int hi = 0;
  while (zfo_e4m3_decode((uint8_t)hi) < a) ++hi; /* first code whose value >= a */
  if (hi == 0) return (uint8_t)sign;
  double dh = zfo_e4m3_decode((uint8_t)hi) - a;
  double dl = a - zfo_e4m3_decode((uint8_t)(hi - 1));
  int c = dl < dh ? hi - 1 : (dh < dl ? hi : ((hi & 1) ? hi - 1 : hi));
  return (uint8_t)(sign | c);
}

/* Values of n E4M3 codes times scale. */
void zfo_fp8_dequantize(const uint8_t* c, int64_t n, double scale, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = zfo_e4m3_decode(c[i]) * scale;
}

static float bf16_to_float(uint16_t w) {
  uint32_t bits = (uint32_t)w << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return f;
}

/* Quantize n bf16 values: code_i = zfo_e4m3_encode((float)value_i * inv_scale)
 * with the product formed in single precision. */
void zfo_fp8_quantize(const uint16_t* w, int64_t n, float inv_scale, uint8_t* out) {
  for (int64_t i = 0; i < n; ++i) {
    volatile float prod = bf16_to_float(w[i]) * inv_scale;
    out[i] = zfo_e4m3_encode((double)prod);
  }
}

/* Paged GQA decode attention in fp64.
 *   q          [B][Hq][D] bf16
 *   k_pool     [num_pages][Hkv][page_size][D] bf16 (v_pool alike)
 *   page_table [B][max_pages] logical page -> physical page
 *   seq_lens   [B]
 *   out        [B][Hq][D] fp64, lse [B][Hq] fp64 (natural log)
 *   p_out      optional [B][Hq][max_pages*page_size] softmax weights
 * A sequence of length 0 gives out = 0 and lse = -inf.  Returns 0, or -1
 * when a page id or a length is out of range (nothing is read then). */
/* Where the attention reads its K or V values: bf16 words, or E4M3 codes
 * times a scale. */
typedef struct {
  const void* pool;
  int fp8;
  double scale;
} kv_source;

static double kv_value(const kv_source* src, int64_t i) {
  if (src->fp8) return zfo_e4m3_decode(((const uint8_t*)src->pool)[i]) * src->scale;
  return bf16_to_double(((const uint16_t*)src->pool)[i]);
}

static int attention(const uint16_t* q, const kv_source* ksrc, const kv_source* vsrc, int64_t num_pages,
                     const int32_t* page_table, int max_pages, const int32_t* seq_lens, int B, int Hq,
                     int Hkv, int D, int page_size, double sm_scale, double* out, double* lse,
                     double* p_out) {
  if (Hkv <= 0 || Hq % Hkv != 0) return -1;
  int group = Hq / Hkv;
  int max_tokens = max_pages * page_size;
  for (int b = 0; b < B; ++b) {
    if (seq_lens[b] < 0 || seq_lens[b] > max_tokens) return -1;
    for (int t = 0; t < seq_lens[b]; t += page_size) {
      int32_t pid = page_table[(int64_t)b * max_pages + t / page_size];
      if (pid < 0 || pid >= num_pages) return -1;
    }
  }
  double* s = (double*)malloc(sizeof(double) * (max_tokens > 0 ? max_tokens : 1));
  if (!s) return -1;
  for (int b = 0; b < B; ++b) {
    int len = seq_lens[b];
    for (int hq = 0; hq < Hq; ++hq) {
      int hk = hq / group;
      const uint16_t* qv = q + ((int64_t)b * Hq + hq) * D;
      double* o = out + ((int64_t)b * Hq + hq) * D;
      double* p = p_out ? p_out + ((int64_t)b * Hq + hq) * max_tokens : 0;
      for (int d = 0; d < D; ++d) o[d] = 0.0;
      if (p)
        for (int t = 0; t < max_tokens; ++t) p[t] = 0.0;
      if (len == 0) {
        lse[(int64_t)b * Hq + hq] = -INFINITY;
        continue;
      }
      double m = -INFINITY;
      for (int t = 0; t < len; ++t) {
        int64_t pid = page_table[(int64_t)b * max_pages + t / page_size];
        int64_t kv = ((pid * Hkv + hk) * page_size + t % page_size) * D;
        double dot = 0.0;
        for (int d = 0; d < D; ++d) dot += bf16_to_double(qv[d]) * kv_value(ksrc, kv + d);
        s[t] = sm_scale * dot;
        if (s[t] > m) m = s[t];
      }
      double l = 0.0;
      for (int t = 0; t < len; ++t) l += exp(s[t] - m);
      for (int t = 0; t < len; ++t) {
        int64_t pid = page_table[(int64_t)b * max_pages + t / page_size];
        int64_t vv = ((pid * Hkv + hk) * page_size + t % page_size) * D;
        double pt = exp(s[t] - m) / l;
        if (p) p[t] = pt;
        for (int d = 0; d < D; ++d) o[d] += pt * kv_value(vsrc, vv + d);
      }
      lse[(int64_t)b * Hq + hq] = m + log(l);
    }
  }
  free(s);
  return 0;
}

int zfo_attention(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool,
                  int64_t num_pages, const int32_t* page_table, int max_pages,
                  const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int page_size,
                  double sm_scale, double* out, double* lse, double* p_out) {
  kv_source k = {k_pool, 0, 1.0}, v = {v_pool, 0, 1.0};
  return attention(q, &k, &v, num_pages, page_table, max_pages, seq_lens, B, Hq, Hkv, D, page_size, sm_scale,
                   out, lse, p_out);
}

/* The same attention over E4M3 pools (codes [P][Hkv][page_size][D], one
 * scale per pool): K and V values are decode(code) * scale (reading R8). */
int zfo_attention_fp8(const uint16_t* q, const uint8_t* k_codes, const uint8_t* v_codes, double k_scale,
                      double v_scale, int64_t num_pages, const int32_t* page_table, int max_pages,
                      const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int page_size, double sm_scale,
                      double* out, double* lse, double* p_out) {
  kv_source k = {k_codes, 1, k_scale}, v = {v_codes, 1, v_scale};
  return attention(q, &k, &v, num_pages, page_table, max_pages, seq_lens, B, Hq, Hkv, D, page_size, sm_scale,
                   out, lse, p_out);
}
