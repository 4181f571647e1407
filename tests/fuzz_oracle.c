/* Host fuzz driver for the oracle, built with AddressSanitizer and
 * UndefinedBehaviorSanitizer by tests/test_oracle_fuzz.py (test
 * infrastructure; it checks the oracle, not the GPU library).
 *
 * Containers of every front-end (bf16 and f32 lossless, bf16 transform) are
 * damaged in every way the container must refuse (every single-byte change,
 * every truncation: the QATQ page's corrupt or truncated input rejected
 * before restore) and, separately, forged: a record changed and sealed again
 * with fresh CRCs, so that the stream parsers themselves meet malformed
 * headers, tables and payloads. The decoders must return a status and stay
 * inside their buffers (the sanitizers abort the run otherwise). The inputs
 * are drawn from a small xorshift generator of this file's own: only the
 * oracle sees them. */
#include <math.h>
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include "../oracle/kvco.h"

static uint64_t rng_state = 0x9E3779B97F4A7C15ull;
static uint64_t next_u64(void) {
  rng_state ^= rng_state << 13;
  rng_state ^= rng_state >> 7;
  rng_state ^= rng_state << 17;
  return rng_state;
}

static void put32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get32(const uint8_t* p) {
  return (uint32_t)p[0] | ((uint32_t)p[1] << 8) | ((uint32_t)p[2] << 16) | ((uint32_t)p[3] << 24);
}
static uint64_t get64(const uint8_t* p) { return (uint64_t)get32(p) | ((uint64_t)get32(p + 4) << 32); }

/* Recompute record i's CRC in the index and the header CRC (header[0, 60) and the index). */
static void reseal(uint8_t* c, uint32_t i) {
  uint32_t nr = get32(c + 36);
  const uint8_t* e = c + 64 + 16u * i;
  put32(c + 64 + 16u * i + 12, kvco_crc32(c + get64(e), get32(e + 8)));
  size_t hl = 60u + 16u * (size_t)nr;
  uint8_t* tmp = (uint8_t*)malloc(hl);
  memcpy(tmp, c, 60);
  memcpy(tmp + 60, c + 64, 16u * (size_t)nr);
  put32(c + 60, kvco_crc32(tmp, hl));
  free(tmp);
}

typedef int (*decode_fn)(const kvco_desc*, const uint8_t*, size_t, void*, size_t, uint64_t*);

static int dec_lossless(const kvco_desc* d, const uint8_t* s, size_t n, void* o, size_t cap, uint64_t* w) {
  return kvco_decode_lossless(d, s, n, o, cap, w);
}
static int dec_transform(const kvco_desc* d, const uint8_t* s, size_t n, void* o, size_t cap, uint64_t* w) {
  return kvco_decode_transform(d, s, n, (uint16_t*)o, cap, w);
}

/* Returns the number of failures (a damaged container accepted). */
static int fuzz(const char* name, const kvco_desc* d, const uint8_t* c, size_t len, size_t out_bytes,
                decode_fn dec, int forged_rounds) {
  int bad = 0;
  uint8_t* buf = (uint8_t*)malloc(len);
  uint8_t* out = (uint8_t*)malloc(out_bytes);
  uint64_t w = 0;
  if (dec(d, c, len, out, out_bytes, &w) != KVCO_OK) {
    printf("%s: clean container refused\n", name);
    bad++;
  }
  for (size_t pos = 0; pos < len; pos++) {  /* every single-byte change */
    memcpy(buf, c, len);
    buf[pos] ^= (uint8_t)(1u + next_u64() % 255u);
    if (dec(d, buf, len, out, out_bytes, &w) == KVCO_OK) {
      printf("%s: byte %zu changed, accepted\n", name, pos);
      bad++;
    }
  }
  for (size_t n = 0; n < len; n++)  /* every truncation, from a buffer of exactly n bytes */
    if (dec(d, c, n, out, out_bytes, &w) == KVCO_OK) {
      printf("%s: truncated to %zu, accepted\n", name, n);
      bad++;
    }
  uint32_t nr = get32(c + 36);
  int accepted = 0, refused = 0;
  for (int round = 0; round < forged_rounds; round++) {  /* forged records: the parsers decide */
    memcpy(buf, c, len);
    uint32_t i = (uint32_t)(next_u64() % nr);
    const uint8_t* e = c + 64 + 16u * i;
    uint64_t off = get64(e);
    uint32_t rl = get32(e + 8);
    int edits = 1 + (int)(next_u64() % 3);
    for (int k = 0; k < edits && rl; k++) {
      uint32_t p = (uint32_t)(next_u64() % (next_u64() % 2 ? (rl < 96 ? rl : 96) : rl));
      buf[off + p] = (uint8_t)next_u64();
    }
    reseal(buf, i);
    if (dec(d, buf, len, out, out_bytes, &w) == KVCO_OK) accepted++;
    else refused++;
  }
  for (int round = 0; round < 200; round++) {  /* garbage of random lengths */
    size_t n = (size_t)(next_u64() % (len + 1));
    for (size_t k = 0; k < n; k++) buf[k] = (uint8_t)next_u64();
    if (n >= 64 && next_u64() % 2) memcpy(buf, c, 64);  /* a valid-looking header */
    (void)dec(d, buf, n, out, out_bytes, &w);
  }
  printf("%s: %zu bytes, forged records accepted %d refused %d\n", name, len, accepted, refused);
  free(buf);
  free(out);
  return bad;
}

int main(void) {
  int bad = 0;
  /* bf16 lossless: 2 slices of 48 tokens x 128, chunks of 32 tokens (ragged tail) */
  {
    kvco_desc d;
    memset(&d, 0, sizeof d);
    d.dtype = KVCO_BF16; d.n_layers = 1; d.n_heads = 1; d.n_tokens = 48; d.head_dim = 128;
    d.values_per_chunk = 4096;
    size_t nv = 2u * 48u * 128u;
    uint16_t* x = (uint16_t*)malloc(nv * 2);
    for (size_t i = 0; i < nv; i++) x[i] = (uint16_t)(0x3F00u + (i % 128u) + (next_u64() % 7u));
    size_t cap = kvco_lossless_bound(&d, 2);
    uint8_t* c = (uint8_t*)malloc(cap);
    size_t len = kvco_encode_lossless(&d, 0, 2, x, c, cap);
    bad += fuzz("lossless bf16", &d, c, len, nv * 2, dec_lossless, 3000);
    free(x); free(c);
  }
  /* f32 lossless: 2 slices of 40 tokens x 64 */
  {
    kvco_desc d;
    memset(&d, 0, sizeof d);
    d.dtype = KVCO_F32; d.n_layers = 1; d.n_heads = 1; d.n_tokens = 40; d.head_dim = 64;
    d.values_per_chunk = 1024;
    size_t nv = 2u * 40u * 64u;
    float* x = (float*)malloc(nv * 4);
    for (size_t i = 0; i < nv; i++) x[i] = 1.0f + (float)(i % 64u) * 0.25f + (float)(next_u64() % 1000u) * 1e-4f;
    size_t cap = kvco_lossless_bound(&d, 2);
    uint8_t* c = (uint8_t*)malloc(cap);
    size_t len = kvco_encode_lossless(&d, 0, 2, x, c, cap);
    bad += fuzz("lossless f32", &d, c, len, nv * 4, dec_lossless, 3000);
    free(x); free(c);
  }
  /* bf16 transform: 2 slices of 200 tokens x 16, identity basis, widths 0..8 */
  {
    kvco_desc d;
    memset(&d, 0, sizeof d);
    d.dtype = KVCO_BF16; d.n_layers = 1; d.n_heads = 1; d.n_tokens = 200; d.head_dim = 16;
    d.values_per_chunk = 65536; d.n_sink = 4; d.n_recent = 16; d.block_tokens = 16; d.chunk_tokens = 64;
    d.max_bits = 8; d.rope_theta = 10000.0;
    float* q = (float*)calloc(2u * 16u * 16u, sizeof(float));
    uint8_t* wd = (uint8_t*)malloc(2u * 16u);
    for (uint32_t s = 0; s < 2; s++)
      for (uint32_t j = 0; j < 16; j++) {
        q[(s * 16u + j) * 16u + j] = 1.0f;
        wd[s * 16u + j] = (uint8_t)((j * 5u + s) % 9u);
      }
    d.bases = q;
    d.widths = wd;
    size_t nv = 2u * 200u * 16u;
    uint16_t* x = (uint16_t*)malloc(nv * 2);
    for (size_t i = 0; i < nv; i++) {
      float f = sinf((float)i * 0.01f) * 3.0f + (float)(next_u64() % 100u) * 0.01f;
      x[i] = kvco_f32_to_bf16(f);
    }
    size_t cap = kvco_transform_bound(&d, 2);
    uint8_t* c = (uint8_t*)malloc(cap);
    size_t len = kvco_encode_transform(&d, 0, 2, x, c, cap);
    bad += fuzz("transform bf16", &d, c, len, nv * 2, dec_transform, 3000);
    free(x); free(c); free(q); free(wd);
  }
  printf(bad ? "FAILURES %d\n" : "ok\n", bad);
  return bad ? 1 : 0;
}
