/* Exhaustive pin of the oracle's block codec at block size 2: every one of
 * the 2^32 pairs (w0, w1) of bf16 bit patterns is packed and unpacked with
 * the oracle (libzf_oracle.so) and checked against the definitions:
 *   eligible  <=> |e0 - e1| <= 15        (e = exponent field, bits 7..14)
 *   base      =   min(e0, e1)
 *   size      =   3 bytes (12 bits per value) if eligible, else 4
 *   unpack(pack(w0, w1)) == (w0, w1)      (lossless)
 * Threads split the range of w0.  Prints the number of failing pairs.
 * Usage: bruteforce_pairs [threads [w0_count]] (w0_count < 65536 checks only
 * the pairs whose first value is below it). */
#include <pthread.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>

int64_t zfo_pack_block(const uint16_t* w, int n, uint8_t* out, uint8_t* base_out, int* eligible_out);
void zfo_unpack_block(const uint8_t* in, int n, uint8_t base, int eligible, uint16_t* w);

typedef struct {
  uint32_t w0_lo, w0_hi;
  uint64_t failures;
} span;

static void* run(void* arg) {
  span* s = (span*)arg;
  uint64_t bad = 0;
  for (uint32_t a = s->w0_lo; a < s->w0_hi; ++a) {
    for (uint32_t b = 0; b < 65536; ++b) {
      uint16_t w[2] = {(uint16_t)a, (uint16_t)b};
      uint8_t out[8] = {0};
      uint8_t base = 0;
      int el = -1;
      int64_t size = zfo_pack_block(w, 2, out, &base, &el);
      int e0 = (int)((a >> 7) & 0xFF), e1 = (int)((b >> 7) & 0xFF);
      int want_el = abs(e0 - e1) <= 15;
      int want_base = e0 < e1 ? e0 : e1;
      uint16_t back[2] = {0, 0};
      zfo_unpack_block(out, 2, base, el, back);
      if (el != want_el || base != want_base || size != (want_el ? 3 : 4) || back[0] != w[0] ||
          back[1] != w[1])
        ++bad;
    }
  }
  s->failures = bad;
  return NULL;
}

int main(int argc, char** argv) {
  int threads = argc > 1 ? atoi(argv[1]) : 8;
  if (threads < 1) threads = 1;
  if (threads > 64) threads = 64;
  uint64_t w0_count = argc > 2 ? strtoull(argv[2], NULL, 10) : 65536;
  if (w0_count > 65536) w0_count = 65536;
  pthread_t tid[64];
  span spans[64];
  for (int t = 0; t < threads; ++t) {
    spans[t].w0_lo = (uint32_t)(w0_count * t / threads);
    spans[t].w0_hi = (uint32_t)(w0_count * (t + 1) / threads);
    spans[t].failures = 0;
    pthread_create(&tid[t], NULL, run, &spans[t]);
  }
  uint64_t total = 0;
  for (int t = 0; t < threads; ++t) {
    pthread_join(tid[t], NULL);
    total += spans[t].failures;
  }
  printf("%llu\n", (unsigned long long)total);
  return total != 0;
}
