/* Every entry point of the C oracle run under AddressSanitizer and
 * UndefinedBehaviorSanitizer on exact-size heap buffers (worst-case sizes
 * where the output size depends on the data), so any read or write past a
 * buffer, any use of uninitialised sizes or any undefined arithmetic stops
 * the program.  Also checks the round trips, so the run is not vacuous. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

void zfo_block_stats(const uint16_t* w, int n, int* emin, int* emax);
int zfo_block_eligible(const uint16_t* w, int n);
int64_t zfo_pack_block(const uint16_t* w, int n, uint8_t* out, uint8_t* base_out, int* eligible_out);
void zfo_unpack_block(const uint8_t* in, int n, uint8_t base, int eligible, uint16_t* w);
int64_t zfo_compress_general(const uint16_t* src, int64_t n_values, int n, uint8_t* payload, int64_t* offs_bytes,
                             uint8_t* base, uint8_t* eligible);
void zfo_decompress_general(const uint8_t* payload, const int64_t* offs_bytes, const uint8_t* base,
                            const uint8_t* eligible, int n, int64_t i0, int64_t i1, uint16_t* dst);
int64_t zfo_compress(const uint16_t* src, int64_t n_values, uint8_t* payload, uint32_t* offs, uint8_t* base,
                     uint32_t* elig);
void zfo_decompress(const uint8_t* payload, const uint32_t* offs, const uint8_t* base, const uint32_t* elig,
                    int64_t i0, int64_t i1, uint16_t* dst);
int64_t zfo_pack_chunk(const uint16_t* src, int n_blocks, uint8_t* out);
int64_t zfo_compress_paged(const uint16_t* src, int64_t num_chunks, uint8_t* data, uint32_t* chunk_tab);
void zfo_decompress_paged(const uint8_t* data, const uint32_t* chunk_tab, int64_t num_chunks, int n_blocks,
                          uint16_t* dst);
double zfo_e4m3_decode(uint8_t c);
uint8_t zfo_e4m3_encode(double x);
void zfo_fp8_quantize(const uint16_t* w, int64_t n, float inv_scale, uint8_t* out);
void zfo_fp8_dequantize(const uint8_t* c, int64_t n, double scale, double* out);
int zfo_attention(const uint16_t* q, const uint16_t* k_pool, const uint16_t* v_pool, int64_t num_pages,
                  const int32_t* page_table, int max_pages, const int32_t* seq_lens, int B, int Hq, int Hkv, int D,
                  int page_size, double sm_scale, double* out, double* lse, double* p_out);
int zfo_attention_fp8(const uint16_t* q, const uint8_t* k_codes, const uint8_t* v_codes, double k_scale,
                      double v_scale, int64_t num_pages, const int32_t* page_table, int max_pages,
                      const int32_t* seq_lens, int B, int Hq, int Hkv, int D, int page_size, double sm_scale,
                      double* out, double* lse, double* p_out);

#define CHECK(c)                                               \
  do {                                                         \
    if (!(c)) {                                                \
      fprintf(stderr, "failed: %s (line %d)\n", #c, __LINE__); \
      exit(1);                                                 \
    }                                                          \
  } while (0)

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static uint32_t rnd(void) {  /* xorshift64* */
  rng_state ^= rng_state >> 12;
  rng_state ^= rng_state << 25;
  rng_state ^= rng_state >> 27;
  return (uint32_t)((rng_state * 0x2545F4914F6CDD1Dull) >> 32);
}

/* bf16 values around 1 with a few wide-spread blocks (every 5th block gets
 * one tiny and one huge value, so it is stored raw) */
static uint16_t* values(int64_t n) {
  uint16_t* v = (uint16_t*)malloc((size_t)n * sizeof *v);
  for (int64_t i = 0; i < n; ++i) v[i] = (uint16_t)(((rnd() & 1) << 15) | ((120 + rnd() % 12) << 7) | (rnd() & 0x7F));
  for (int64_t b = 0; b * 64 < n; b += 5) {
    v[b * 64] = (uint16_t)(200u << 7);
    v[b * 64 + 1] = (uint16_t)(30u << 7);
  }
  return v;
}

static void* zalloc(size_t bytes) { return calloc(bytes ? bytes : 1, 1); }

int main(void) {
  /* ---- canonical flat form, exact worst-case buffers */
  for (int64_t nb = 1; nb <= 70; nb += 23) {
    int64_t n = nb * 64;
    uint16_t* v = values(n);
    uint8_t* payload = (uint8_t*)zalloc((size_t)(2 * n));
    uint32_t* offs = (uint32_t*)zalloc((size_t)(nb + 1) * 4);
    uint8_t* base = (uint8_t*)zalloc((size_t)nb);
    uint32_t* elig = (uint32_t*)zalloc((size_t)((nb + 31) / 32) * 4);
    int64_t units = zfo_compress(v, n, payload, offs, base, elig);
    CHECK(units == (int64_t)offs[nb] && units * 16 <= 2 * n);
    uint16_t* back = (uint16_t*)zalloc((size_t)n * 2);
    zfo_decompress(payload, offs, base, elig, 0, nb, back);
    CHECK(memcmp(back, v, (size_t)n * 2) == 0);
    zfo_decompress(payload, offs, base, elig, nb - 1, nb, back);  /* last block alone */
    CHECK(memcmp(back, v + (nb - 1) * 64, 128) == 0);
    free(v), free(payload), free(offs), free(base), free(elig), free(back);
  }
  /* ---- general block sizes */
  for (int bs = 2; bs <= 64; bs *= 2) {
    int64_t n = (int64_t)bs * 37;
    uint16_t* v = values(n);
    uint8_t* payload = (uint8_t*)zalloc((size_t)(2 * n));
    int64_t* offs = (int64_t*)zalloc((size_t)(37 + 1) * 8);
    uint8_t* base = (uint8_t*)zalloc(37);
    uint8_t* el = (uint8_t*)zalloc(37);
    int64_t total = zfo_compress_general(v, n, bs, payload, offs, base, el);
    CHECK(total == offs[37] && total <= 2 * n);
    uint16_t* back = (uint16_t*)zalloc((size_t)n * 2);
    zfo_decompress_general(payload, offs, base, el, bs, 0, 37, back);
    CHECK(memcmp(back, v, (size_t)n * 2) == 0);
    free(v), free(payload), free(offs), free(base), free(el), free(back);
  }
  /* ---- paged form: partial chunks and whole pools */
  {
    uint16_t* v = values(2048 * 5);
    for (int k = 0; k <= 32; ++k) {
      uint8_t* out = (uint8_t*)zalloc(48 + (size_t)k * 128);
      int64_t bytes = zfo_pack_chunk(v, k, out);
      CHECK(bytes >= 48 && bytes <= 48 + (int64_t)k * 128);
      uint32_t tab[2] = {0, (uint32_t)(bytes / 16)};
      uint16_t* back = (uint16_t*)zalloc(2048 * 2);
      zfo_decompress_paged(out, tab, 1, k, back);
      CHECK(memcmp(back, v, (size_t)k * 128) == 0);
      free(out), free(back);
    }
    uint8_t* data = (uint8_t*)zalloc(5 * (48 + 4096));
    uint32_t* tab = (uint32_t*)zalloc(2 * 5 * 4);
    int64_t units = zfo_compress_paged(v, 5, data, tab);
    CHECK(units * 16 <= 5 * (48 + 4096));
    uint16_t* back = (uint16_t*)zalloc(2048 * 5 * 2);
    zfo_decompress_paged(data, tab, 5, 32, back);
    CHECK(memcmp(back, v, 2048 * 5 * 2) == 0);
    free(v), free(data), free(tab), free(back);
  }
  /* ---- E4M3 */
  for (int c = 0; c < 256; ++c) {
    double d = zfo_e4m3_decode((uint8_t)c);
    if (!isnan(d)) CHECK(zfo_e4m3_encode(d) == c || (d == 0.0 && (c & 0x7F) == 0));
  }
  {
    uint16_t* v = values(1024);
    uint8_t* codes = (uint8_t*)zalloc(1024);
    double* deq = (double*)zalloc(1024 * sizeof(double));
    zfo_fp8_quantize(v, 1024, 0.5f, codes);
    zfo_fp8_dequantize(codes, 1024, 2.0, deq);
    free(v), free(codes), free(deq);
  }
  /* ---- attention, ragged lengths including 0 and a full row */
  {
    const int B = 3, Hq = 4, Hkv = 2, D = 128, PS = 16, maxp = 3, P = 7;
    const int32_t lens[3] = {0, 37, 48};
    int32_t* sl = (int32_t*)zalloc(sizeof lens);
    memcpy(sl, lens, sizeof lens);
    int32_t* pt = (int32_t*)zalloc((size_t)B * maxp * 4);
    for (int i = 0; i < B * maxp; ++i) pt[i] = (int32_t)(rnd() % P);
    uint16_t* q = values((int64_t)B * Hq * D);
    uint16_t* k = values((int64_t)P * Hkv * PS * D);
    uint16_t* vv = values((int64_t)P * Hkv * PS * D);
    uint8_t* k8 = (uint8_t*)zalloc((size_t)P * Hkv * PS * D);
    uint8_t* v8 = (uint8_t*)zalloc((size_t)P * Hkv * PS * D);
    zfo_fp8_quantize(k, (int64_t)P * Hkv * PS * D, 1.0f / 64, k8);
    zfo_fp8_quantize(vv, (int64_t)P * Hkv * PS * D, 1.0f / 64, v8);
    double* out = (double*)zalloc((size_t)B * Hq * D * 8);
    double* lse = (double*)zalloc((size_t)B * Hq * 8);
    double* p = (double*)zalloc((size_t)B * Hq * maxp * PS * 8);
    CHECK(zfo_attention(q, k, vv, P, pt, maxp, sl, B, Hq, Hkv, D, PS, 0.088, out, lse, p) == 0);
    CHECK(isinf(lse[0]) && lse[0] < 0);
    for (int h = 0; h < Hq; ++h) {
      double s = 0;
      for (int t = 0; t < lens[2]; ++t) s += p[((int64_t)2 * Hq + h) * maxp * PS + t];
      CHECK(fabs(s - 1.0) < 1e-12);
    }
    CHECK(zfo_attention_fp8(q, k8, v8, 64.0, 64.0, P, pt, maxp, sl, B, Hq, Hkv, D, PS, 0.088, out, lse, p) == 0);
    pt[3] = P;  /* a bad page id in row 1 is rejected before anything is read */
    CHECK(zfo_attention(q, k, vv, P, pt, maxp, sl, B, Hq, Hkv, D, PS, 0.088, out, lse, NULL) == -1);
    free(sl), free(pt), free(q), free(k), free(vv), free(k8), free(v8), free(out), free(lse), free(p);
  }
  puts("ok");
  return 0;
}
