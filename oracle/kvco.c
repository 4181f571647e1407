/*
 * kvco — the CPU oracle for the KV codec (TEST INFRASTRUCTURE ONLY: loaded by
 * the tests, the smoke check and the benchmark's CPU-baseline leg, never by the
 * product path). Plain, slow, single-threaded C; no SIMD, no threads, no
 * blocking or reordering beyond what each definition states. It shares no code
 * with the GPU library: formats and constants are restated here from the
 * codec's written format rules.
 *
 * Page citations are by page title and section (see kvco.h for the list).
 */
#include "kvco.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define M_SCALE 4096u      /* rANS frequency total, 2^12 */
#define RANS_L 65536u      /* rANS lower bound, 2^16; 16-bit words */
#define MAX_LANES 128u
#define LANES_PER_GROUP 32u
#define MODE_RAW 0
#define MODE_CONST 1
#define MODE_RANS 2

/* ---------------------------------------------------------------------------
 * little-endian byte helpers
 * ------------------------------------------------------------------------- */
static void put16(uint8_t* p, uint32_t v) { p[0] = (uint8_t)v; p[1] = (uint8_t)(v >> 8); }
static void put32(uint8_t* p, uint32_t v) {
  for (int i = 0; i < 4; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static void put64(uint8_t* p, uint64_t v) {
  for (int i = 0; i < 8; i++) p[i] = (uint8_t)(v >> (8 * i));
}
static uint32_t get16(const uint8_t* p) { return (uint32_t)p[0] | ((uint32_t)p[1] << 8); }
static uint32_t get32(const uint8_t* p) {
  uint32_t v = 0;
  for (int i = 0; i < 4; i++) v |= (uint32_t)p[i] << (8 * i);
  return v;
}
static uint64_t get64(const uint8_t* p) {
  uint64_t v = 0;
  for (int i = 0; i < 8; i++) v |= (uint64_t)p[i] << (8 * i);
  return v;
}
static size_t pad16(size_t n) { return (n + 15u) & ~(size_t)15u; }

float kvco_bf16_to_f32(uint16_t h) {
  uint32_t x = (uint32_t)h << 16;
  float f;
  memcpy(&f, &x, 4);
  return f;
}

/* round-to-nearest-even fp32 -> bf16; NaN stays NaN (quiet bit set) */
uint16_t kvco_f32_to_bf16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((x >> 16) | 0x40u);
  uint32_t upper = x >> 16, lower = x & 0xffffu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) upper++;
  return (uint16_t)upper;
}

/* ---------------------------------------------------------------------------
 * CRC-32 (ISO-HDLC / zlib variant): reflected polynomial 0xEDB88320, initial
 * value and final xor 0xFFFFFFFF. One bit at a time.
 * [QATQ] "QATC v2 checksum validated": corrupt or truncated payloads are
 * refused before restore; [AT1] "What's proven": single-byte tamper refusal.
 * ------------------------------------------------------------------------- */
uint32_t kvco_crc32(const void* data, size_t n) {
  const uint8_t* p = (const uint8_t*)data;
  uint32_t crc = 0xffffffffu;
  for (size_t i = 0; i < n; i++) {
    crc ^= p[i];
    for (int b = 0; b < 8; b++) crc = (crc >> 1) ^ ((crc & 1u) ? 0xedb88320u : 0u);
  }
  return crc ^ 0xffffffffu;
}

/* ---------------------------------------------------------------------------
 * Frequency normalisation to a total of M = 4096 ([KVTC] "rANS Makes the Last
 * Mile Smaller": a table of symbol frequencies drives the coder). The pages fix
 * no rule; this codec's rule (largest-remainder apportionment):
 *   k = number of present symbols, n = total count;
 *   f_s = 1 + floor(c_s * (M - k) / n), r_s = c_s * (M - k) mod n  (c_s > 0);
 *   d = M - sum f_s (0 <= d < k);
 *   the d present symbols with the largest r_s get one more (ties: smaller s).
 * Returns k. k == 1 gives f = M for the one symbol (CONST streams use no table).
 * ------------------------------------------------------------------------- */
int kvco_normalize(const uint32_t count[256], uint16_t freq[256]) {
  uint64_t n = 0;
  uint32_t k = 0;
  for (int s = 0; s < 256; s++) {
    n += count[s];
    if (count[s]) k++;
    freq[s] = 0;
  }
  if (k == 0) return 0;
  if (k == 1) {
    for (int s = 0; s < 256; s++)
      if (count[s]) freq[s] = (uint16_t)M_SCALE;
    return 1;
  }
  uint64_t rem[256];
  int given[256];
  uint32_t sum = 0;
  for (int s = 0; s < 256; s++) {
    given[s] = 0;
    rem[s] = 0;
    if (!count[s]) continue;
    uint64_t q = (uint64_t)count[s] * (M_SCALE - k);
    freq[s] = (uint16_t)(1 + q / n);
    rem[s] = q % n;
    sum += freq[s];
  }
  uint32_t d = M_SCALE - sum;
  for (uint32_t i = 0; i < d; i++) {
    int best = -1;
    for (int s = 0; s < 256; s++) {
      if (!count[s] || given[s]) continue;
      if (best < 0 || rem[s] > rem[best]) best = s;
    }
    given[best] = 1;
    freq[best]++;
  }
  return (int)k;
}

/* ---------------------------------------------------------------------------
 * Interleaved rANS ([KVTC] "rANS Makes the Last Mile Smaller"). Standard rANS
 * (J. Duda, arXiv:1311.2540) with interleaved lanes (F. Giesen,
 * arXiv:1402.3392). Parameters are this codec's: 32-bit state, L = 2^16,
 * 16-bit words, M = 2^12.
 *   lanes N = min(128, max(1, floor(n / 512))); lane l owns the contiguous
 *   symbol range [start_l, start_l + len_l), len_l = floor(n/N) + (l < n mod N);
 *   groups of 32 lanes, one sub-stream per group.
 * The decoder defines the format: per step tau, lanes of the group ascending
 * (only those with tau < len_l): slot = x & 4095, s = symbol owning slot,
 * x = f_s * (x >> 12) + slot - cum_s, emit s, and if x < 2^16 read one word:
 * x = (x << 16) | word. Every lane must end at x == 2^16 with every word read.
 * ------------------------------------------------------------------------- */
static uint32_t lanes_for(uint32_t n) {
  uint32_t N = n / 512u;
  if (N < 1) N = 1;
  if (N > MAX_LANES) N = MAX_LANES;
  return N;
}

/* Side streams (the byte planes of a middle record's zero points and scales,
 * at most 2 * D * ct / B symbols) take one lane per 64 symbols, at most one
 * group: N = min(32, max(1, floor(n / 64))). This codec's reading: it keeps a
 * lane's serial chain at most 127 steps, a quarter of a code stream's. */
static uint32_t side_lanes_for(uint32_t n) {
  uint32_t N = n / 64u;
  if (N < 1) N = 1;
  if (N > LANES_PER_GROUP) N = LANES_PER_GROUP;
  return N;
}

static void lane_range(uint32_t n, uint32_t N, uint32_t l, uint32_t* start, uint32_t* len) {
  uint32_t base = n / N, extra = n % N;
  *len = base + (l < extra ? 1u : 0u);
  *start = l * base + (l < extra ? l : extra);
}

static void cum_from_freq(const uint16_t freq[256], uint32_t cum[256]) {
  uint32_t c = 0;
  for (int s = 0; s < 256; s++) {
    cum[s] = c;
    c += freq[s];
  }
}

/* Encode group g of a stream. Writes states then words to out; returns the
 * unpadded sub-stream byte length (4 * lanes + 2 * words). The encoder mirrors
 * the decoder: x starts at 2^16; steps in reverse (tau descending, lanes
 * descending); before coding s, if x >= f_s << 20 the low 16 bits of x are
 * prepended as a word and x >>= 16; then x = (x / f_s) * 4096 + x mod f_s + cum_s. */
static size_t rans_encode_group(const uint8_t* sym, uint32_t n, uint32_t N, uint32_t g,
                                const uint16_t freq[256], const uint32_t cum[256],
                                uint8_t* out) {
  uint32_t lo = g * LANES_PER_GROUP;
  uint32_t hi = lo + LANES_PER_GROUP < N ? lo + LANES_PER_GROUP : N;
  uint64_t x[LANES_PER_GROUP];
  uint32_t start[LANES_PER_GROUP] = {0}, len[LANES_PER_GROUP] = {0};
  size_t n_group_syms = 0;
  for (uint32_t l = lo; l < hi; l++) {
    lane_range(n, N, l, &start[l - lo], &len[l - lo]);
    x[l - lo] = RANS_L;
    n_group_syms += len[l - lo];
  }
  uint16_t* rev = (uint16_t*)malloc(sizeof(uint16_t) * (n_group_syms + 1));
  size_t W = 0;
  uint32_t maxlen = len[0];
  for (uint32_t tau = maxlen; tau-- > 0;) {
    for (uint32_t l = hi; l-- > lo;) {
      uint32_t i = l - lo;
      if (tau >= len[i]) continue;
      uint32_t s = sym[start[i] + tau];
      uint64_t f = freq[s];
      if (x[i] >= (f << 20)) {
        rev[W++] = (uint16_t)(x[i] & 0xffffu);
        x[i] >>= 16;
      }
      x[i] = ((x[i] / f) << 12) + (x[i] % f) + cum[s];
    }
  }
  uint8_t* p = out;
  for (uint32_t l = lo; l < hi; l++) {
    put32(p, (uint32_t)x[l - lo]);
    p += 4;
  }
  for (size_t w = W; w-- > 0;) {
    put16(p, rev[w]);
    p += 2;
  }
  free(rev);
  return (size_t)(p - out);
}

/* Decode group g from a sub-stream of sub_len bytes. Returns 0 on success. */
static int rans_decode_group(const uint8_t* sub, size_t sub_len, uint32_t n, uint32_t N,
                             uint32_t g, const uint16_t freq[256], const uint32_t cum[256],
                             uint8_t* sym) {
  uint32_t lo = g * LANES_PER_GROUP;
  uint32_t hi = lo + LANES_PER_GROUP < N ? lo + LANES_PER_GROUP : N;
  uint32_t lanes = hi - lo;
  if (sub_len < 4u * lanes || ((sub_len - 4u * lanes) & 1u)) return KVCO_CORRUPT;
  size_t W = (sub_len - 4u * lanes) / 2u;
  const uint8_t* words = sub + 4u * lanes;
  uint64_t x[LANES_PER_GROUP];
  uint32_t start[LANES_PER_GROUP], len[LANES_PER_GROUP];
  for (uint32_t l = lo; l < hi; l++) {
    lane_range(n, N, l, &start[l - lo], &len[l - lo]);
    x[l - lo] = get32(sub + 4u * (l - lo));
  }
  size_t pos = 0;
  uint32_t maxlen = len[0];
  for (uint32_t tau = 0; tau < maxlen; tau++) {
    for (uint32_t l = lo; l < hi; l++) {
      uint32_t i = l - lo;
      if (tau >= len[i]) continue;
      uint32_t slot = (uint32_t)(x[i] & (M_SCALE - 1u));
      int s = 0;
      while (s < 256 && !(freq[s] && cum[s] <= slot && slot < cum[s] + freq[s])) s++;
      if (s == 256) return KVCO_CORRUPT;
      sym[start[i] + tau] = (uint8_t)s;
      x[i] = (uint64_t)freq[s] * (x[i] >> 12) + slot - cum[s];
      if (x[i] < RANS_L) {
        if (pos >= W) return KVCO_CORRUPT;
        x[i] = (x[i] << 16) | get16(words + 2 * pos);
        pos++;
      }
    }
  }
  if (pos != W) return KVCO_CORRUPT;
  for (uint32_t i = 0; i < lanes; i++)
    if (x[i] != RANS_L) return KVCO_CORRUPT;
  return KVCO_OK;
}

/* ---------------------------------------------------------------------------
 * Stream record. One stream = n byte symbols; the record keeps whichever is
 * smallest: CONST (one distinct symbol), RANS if strictly smaller than RAW,
 * else RAW ([AT1] "KV & tensor mode": keep whichever is smaller, so never worse
 * than the fallback).
 *   header (16 bytes): u8 mode, u8 const symbol, u8 groups, u8 flags (bit 0: the
 *                      RANS symbols are lane deltas, see kvco_lane_delta; 0 otherwise),
 *                      u32 record bytes (multiple of 16, header included),
 *                      u32 n, u32 k (present symbols: RAW 0, CONST 1, RANS k)
 *   RAW:   n bytes, zero padded to 16
 *   CONST: nothing
 *   RANS:  32-byte presence bitmap (bit s&7 of byte s>>3), k u16 frequencies
 *          for present symbols ascending, zero pad to 16; G u32 sub-stream
 *          byte lengths (unpadded), zero pad to 16; each group's sub-stream
 *          (u32 states of its lanes ascending, u16 words) zero padded to 16.
 * ------------------------------------------------------------------------- */
size_t kvco_stream_bound(uint32_t n) { return 16u + pad16(n); }

static size_t stream_raw(const uint8_t* sym, uint32_t n, uint8_t* out) {
  size_t bytes = 16u + pad16(n);
  memset(out, 0, bytes);
  out[0] = MODE_RAW;
  put32(out + 4, (uint32_t)bytes);
  put32(out + 8, n);
  if (n) memcpy(out + 16, sym, n);
  return bytes;
}

/* Build the RANS record into out (capacity 2n + 4096); returns its size. */
static size_t stream_rans(const uint8_t* sym, uint32_t n, uint32_t N, const uint16_t freq[256],
                          uint32_t k, uint32_t flags, uint8_t* out, size_t* payload) {
  uint32_t cum[256];
  cum_from_freq(freq, cum);
  uint32_t G = (N + LANES_PER_GROUP - 1) / LANES_PER_GROUP;
  size_t p = 16;
  memset(out, 0, 16 + 32);
  for (int s = 0; s < 256; s++)
    if (freq[s]) out[p + (s >> 3)] |= (uint8_t)(1u << (s & 7));
  p += 32;
  for (int s = 0; s < 256; s++)
    if (freq[s]) {
      put16(out + p, freq[s]);
      p += 2;
    }
  while (p & 15u) out[p++] = 0;
  size_t lens_at = p;
  p += 4u * G;
  while (p & 15u) out[p++] = 0;
  *payload = 0;
  for (uint32_t g = 0; g < G; g++) {
    size_t sub = rans_encode_group(sym, n, N, g, freq, cum, out + p);
    put32(out + lens_at + 4u * g, (uint32_t)sub);
    *payload += sub;
    p += sub;
    while (p & 15u) out[p++] = 0;
  }
  out[0] = MODE_RANS;
  out[1] = 0;
  out[2] = (uint8_t)G;
  out[3] = (uint8_t)flags;
  put32(out + 4, (uint32_t)p);
  put32(out + 8, n);
  put32(out + 12, k);
  return p;
}

static int stream_table(const uint8_t* sym, uint32_t n, uint16_t freq[256]) {
  uint32_t count[256];
  memset(count, 0, sizeof count);
  for (uint32_t i = 0; i < n; i++) count[sym[i]]++;
  return kvco_normalize(count, freq);
}

/* Lane delta ([QATQ] "How it works": delta-XOR along tokens in channel-major
 * order). Reading: within each rANS lane's contiguous range of the stream, a
 * symbol is replaced by its XOR with the previous symbol of the same lane; the
 * lane's first symbol is kept. Undone lane by lane in order. */
static void lane_delta_n(const uint8_t* sym, uint32_t n, uint32_t N, uint8_t* out) {
  for (uint32_t l = 0; l < N; l++) {
    uint32_t start, len;
    lane_range(n, N, l, &start, &len);
    for (uint32_t i = 0; i < len; i++)
      out[start + i] = i ? (uint8_t)(sym[start + i] ^ sym[start + i - 1]) : sym[start];
  }
}

static void lane_undelta_n(uint8_t* sym, uint32_t n, uint32_t N) {
  for (uint32_t l = 0; l < N; l++) {
    uint32_t start, len;
    lane_range(n, N, l, &start, &len);
    for (uint32_t i = 1; i < len; i++) sym[start + i] ^= sym[start + i - 1];
  }
}

void kvco_lane_delta(const uint8_t* sym, uint32_t n, uint8_t* out) {
  if (n) lane_delta_n(sym, n, lanes_for(n), out);
}

void kvco_lane_undelta(uint8_t* sym, uint32_t n) {
  if (n) lane_undelta_n(sym, n, lanes_for(n));
}

/* One stream record of n symbols on N rANS lanes: CONST for a single symbol;
 * with allow_delta, a RANS record of the lane-delta symbols (flag byte 1) when
 * strictly smaller than both the plain RANS record and RAW; else plain RANS if
 * strictly smaller than RAW; else RAW. */
static size_t stream_encode_lanes(const uint8_t* sym, uint32_t n, uint32_t N, int allow_delta, uint8_t* out) {
  uint16_t freq[256], dfreq[256];
  int k = stream_table(sym, n, freq);
  if (k == 0) return stream_raw(sym, n, out);
  if (k == 1) {
    memset(out, 0, 16);
    out[0] = MODE_CONST;
    out[1] = sym[0];
    put32(out + 4, 16);
    put32(out + 8, n);
    put32(out + 12, 1);
    return 16;
  }
  size_t raw_bytes = 16u + pad16(n);
  uint8_t* tmp = (uint8_t*)malloc(2u * (size_t)n + 4096u);
  uint8_t* dtmp = (uint8_t*)malloc(2u * (size_t)n + 4096u);
  uint8_t* dsym = (uint8_t*)malloc(n);
  size_t payload;
  size_t rb = stream_rans(sym, n, N, freq, (uint32_t)k, 0, tmp, &payload);
  size_t rd = (size_t)-1;
  if (allow_delta) {
    lane_delta_n(sym, n, N, dsym);
    int kd = stream_table(dsym, n, dfreq);
    if (kd >= 2) rd = stream_rans(dsym, n, N, dfreq, (uint32_t)kd, 1, dtmp, &payload);
  }
  size_t out_bytes;
  if (rd < rb && rd < raw_bytes) {
    memcpy(out, dtmp, rd);
    out_bytes = rd;
  } else if (rb < raw_bytes) {
    memcpy(out, tmp, rb);
    out_bytes = rb;
  } else {
    out_bytes = stream_raw(sym, n, out);
  }
  free(tmp);
  free(dtmp);
  free(dsym);
  return out_bytes;
}

size_t kvco_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out) {
  return stream_encode_lanes(sym, n, lanes_for(n), 0, out);
}

/* Sum of the squared symbol counts (the number of ordered pairs of equal symbols). */
static uint64_t sq_counts(const uint8_t* sym, uint32_t n) {
  uint64_t c[256] = {0}, q = 0;
  for (uint32_t i = 0; i < n; i++) c[sym[i]]++;
  for (int s = 0; s < 256; s++) q += c[s] * c[s];
  return q;
}

/* Stream of a lossless chunk's byte plane with the lane-delta candidate. The
 * candidate is coded only when the lane deltas' counts are more concentrated
 * than the plane's own (sum of squared counts strictly larger) and their
 * collision entropy -log2(sum (c/n)^2) is below log2(181), about 7.5 bits
 * (181 sum c^2 > n^2): deltas of noise-like bytes cannot beat RAW by enough to
 * pay for coding them. Exact integer tests on the two histograms, so any
 * encoder takes the same decision before coding; the candidate is then kept
 * only where strictly the smallest record. */
size_t kvco_stream_encode_delta(const uint8_t* sym, uint32_t n, uint8_t* out) {
  uint32_t N = lanes_for(n);
  int allow = 0;
  if (n) {
    uint8_t* dsym = (uint8_t*)malloc(n);
    lane_delta_n(sym, n, N, dsym);
    uint64_t qd = sq_counts(dsym, n);
    allow = qd > sq_counts(sym, n) && 181u * qd > (uint64_t)n * n;
    free(dsym);
  }
  return stream_encode_lanes(sym, n, N, allow, out);
}

/* Side stream: the lane-delta choice on the side lane rule. */
size_t kvco_side_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out) {
  return stream_encode_lanes(sym, n, side_lanes_for(n), 1, out);
}

/* rANS payload (states + words, no header, table or padding) for n symbols,
 * whatever mode the record would pick; 0 if fewer than two distinct symbols. */
size_t kvco_rans_payload_bytes(const uint8_t* sym, uint32_t n) {
  uint16_t freq[256];
  int k = stream_table(sym, n, freq);
  if (k < 2) return 0;
  uint8_t* tmp = (uint8_t*)malloc(2u * (size_t)n + 4096u);
  size_t payload;
  stream_rans(sym, n, lanes_for(n), freq, (uint32_t)k, 0, tmp, &payload);
  free(tmp);
  return payload;
}

static int stream_decode(const uint8_t* rec, size_t avail, uint32_t n, uint8_t* sym, size_t* used,
                         int allow_delta, int side) {
  if (avail < 16) return KVCO_CORRUPT;
  uint32_t mode = rec[0], csym = rec[1], G = rec[2], flags = rec[3];
  uint32_t bytes = get32(rec + 4), rn = get32(rec + 8), k = get32(rec + 12);
  if (flags > (allow_delta && mode == MODE_RANS ? 1u : 0u) || rn != n || (bytes & 15u) ||
      bytes < 16 || bytes > avail)
    return KVCO_CORRUPT;
  *used = bytes;
  /* a side stream is never longer than RAW (the never-worse choice); a longer
   * one cannot come from the encoder and is refused */
  if (side && bytes > 16u + pad16(n)) return KVCO_CORRUPT;
  if (mode == MODE_RAW) {
    if (csym != 0 || G != 0 || k != 0 || bytes != 16u + pad16(n)) return KVCO_CORRUPT;
    if (n) memcpy(sym, rec + 16, n);
    return KVCO_OK;
  }
  if (mode == MODE_CONST) {
    if (G != 0 || k != 1 || bytes != 16) return KVCO_CORRUPT;
    memset(sym, (int)csym, n);
    return KVCO_OK;
  }
  if (mode != MODE_RANS || csym != 0 || n == 0) return KVCO_CORRUPT;
  uint32_t N = side ? side_lanes_for(n) : lanes_for(n);
  if (G != (N + LANES_PER_GROUP - 1) / LANES_PER_GROUP) return KVCO_CORRUPT;
  if (k < 2 || k > 256) return KVCO_CORRUPT;
  size_t p = 16;
  if (p + 32 > bytes) return KVCO_CORRUPT;
  uint16_t freq[256];
  uint32_t present = 0;
  for (int s = 0; s < 256; s++) present += (rec[p + (s >> 3)] >> (s & 7)) & 1u;
  if (present != k) return KVCO_CORRUPT;
  size_t fp = p + 32;
  if (pad16(fp + 2u * k) > bytes) return KVCO_CORRUPT;
  uint32_t total = 0;
  for (int s = 0; s < 256; s++) {
    freq[s] = 0;
    if ((rec[p + (s >> 3)] >> (s & 7)) & 1u) {
      freq[s] = (uint16_t)get16(rec + fp);
      fp += 2;
      if (freq[s] == 0) return KVCO_CORRUPT;
      total += freq[s];
    }
  }
  if (total != M_SCALE) return KVCO_CORRUPT;
  uint32_t cum[256];
  cum_from_freq(freq, cum);
  p = pad16(fp);
  size_t lens_at = p;
  p = pad16(p + 4u * G);
  if (p > bytes) return KVCO_CORRUPT;
  for (uint32_t g = 0; g < G; g++) {
    uint32_t sub = get32(rec + lens_at + 4u * g);
    if (sub > bytes || p + pad16(sub) > bytes) return KVCO_CORRUPT;
    int st = rans_decode_group(rec + p, sub, n, N, g, freq, cum, sym);
    if (st) return st;
    p += pad16(sub);
  }
  if (p != bytes) return KVCO_CORRUPT;
  if (flags) lane_undelta_n(sym, n, N);
  return KVCO_OK;
}

int kvco_stream_decode(const uint8_t* rec, size_t avail, uint32_t n, uint8_t* sym,
                       size_t* used) {
  return stream_decode(rec, avail, n, sym, used, 1, 0);
}

int kvco_side_stream_decode(const uint8_t* rec, size_t avail, uint32_t n, uint8_t* sym, size_t* used) {
  return stream_decode(rec, avail, n, sym, used, 1, 1);
}

/* ---------------------------------------------------------------------------
 * Container ([QATQ] "How it works" — QATC transport: bounded chunks with
 * ordered lengths and an aggregate checksum; "QATC v2 checksum validated").
 *   header (64 bytes): "KVC1", u16 version 1, u8 path, u8 dtype,
 *     u32 L, H, T, D, first_slice, n_slices, chunk_tokens, n_records,
 *     u64 total_bytes, u32 plan_crc, u16 n_sink, u16 n_recent, u16 block_tokens,
 *     u16 0, u32 header_crc = CRC32(header[0..60) || index)
 *   index: per record u64 offset, u32 length (multiple of 16), u32 CRC32(record)
 *   records: back to back from offset 64 + 16 * n_records.
 * ------------------------------------------------------------------------- */
#define HDR_BYTES 64u
#define IDX_ENTRY 16u

static int desc_ok(const kvco_desc* d) {
  if (!d) return 0;
  if (d->dtype != KVCO_BF16 && d->dtype != KVCO_FP16 && d->dtype != KVCO_F32) return 0;
  if (!d->n_layers || !d->n_heads || !d->n_tokens || !d->head_dim) return 0;
  return 1;
}

static uint32_t n_slices_total(const kvco_desc* d) { return d->n_layers * 2u * d->n_heads; }

static void write_header(uint8_t* h, int path, const kvco_desc* d, uint32_t first,
                         uint32_t n_slices, uint32_t chunk_tokens, uint32_t n_rec,
                         uint64_t total, uint32_t plan_crc) {
  memset(h, 0, HDR_BYTES);
  memcpy(h, "KVC1", 4);
  put16(h + 4, 1);
  h[6] = (uint8_t)path;
  h[7] = (uint8_t)d->dtype;
  put32(h + 8, d->n_layers);
  put32(h + 12, d->n_heads);
  put32(h + 16, d->n_tokens);
  put32(h + 20, d->head_dim);
  put32(h + 24, first);
  put32(h + 28, n_slices);
  put32(h + 32, chunk_tokens);
  put32(h + 36, n_rec);
  put64(h + 40, total);
  put32(h + 48, plan_crc);
  if (path == KVCO_TRANSFORM) {
    put16(h + 52, d->n_sink);
    put16(h + 54, d->n_recent);
    put16(h + 56, d->block_tokens);
  }
}

static uint32_t header_crc(const uint8_t* c, uint32_t n_rec) {
  size_t len = 60u + (size_t)IDX_ENTRY * n_rec;
  uint8_t* tmp = (uint8_t*)malloc(len);
  memcpy(tmp, c, 60);
  memcpy(tmp + 60, c + HDR_BYTES, (size_t)IDX_ENTRY * n_rec);
  uint32_t crc = kvco_crc32(tmp, len);
  free(tmp);
  return crc;
}

/* Validate header and index in the fixed order the codec documents.
 * expected_records(n_slices) gives the record count a valid header must have. */
typedef uint64_t (*records_fn)(const kvco_desc*, uint32_t);

static int check_container(const kvco_desc* d, int path, const uint8_t* src, size_t n,
                           records_fn expected_records, uint32_t expected_chunk_tokens,
                           uint32_t plan_crc, uint32_t* first, uint32_t* n_slices,
                           uint32_t* n_rec) {
  if (n < HDR_BYTES) return KVCO_TRUNCATED;
  if (memcmp(src, "KVC1", 4) != 0 || get16(src + 4) != 1) return KVCO_CORRUPT;
  uint64_t total = get64(src + 40);
  if (n < total) return KVCO_TRUNCATED;
  if (n > total) return KVCO_CORRUPT;
  uint32_t nr = get32(src + 36);
  if ((uint64_t)HDR_BYTES + (uint64_t)IDX_ENTRY * nr > total) return KVCO_CORRUPT;
  if (header_crc(src, nr) != get32(src + 60)) return KVCO_CORRUPT;
  if (src[6] != path || src[7] != d->dtype || get32(src + 8) != d->n_layers ||
      get32(src + 12) != d->n_heads || get32(src + 16) != d->n_tokens ||
      get32(src + 20) != d->head_dim || get32(src + 32) != expected_chunk_tokens)
    return KVCO_PLAN_MISMATCH;
  if (get16(src + 58) != 0) return KVCO_CORRUPT;
  if (path == KVCO_LOSSLESS) {
    if (get32(src + 48) != 0 || get16(src + 52) || get16(src + 54) || get16(src + 56))
      return KVCO_CORRUPT;
  } else {
    if (get16(src + 52) != d->n_sink || get16(src + 54) != d->n_recent ||
        get16(src + 56) != d->block_tokens || get32(src + 48) != plan_crc)
      return KVCO_PLAN_MISMATCH;
  }
  uint32_t f = get32(src + 24), ns = get32(src + 28);
  if ((uint64_t)f + ns > n_slices_total(d)) return KVCO_PLAN_MISMATCH;
  if (expected_records(d, ns) != nr) return KVCO_CORRUPT;
  uint64_t off = (uint64_t)HDR_BYTES + (uint64_t)IDX_ENTRY * nr;
  for (uint32_t i = 0; i < nr; i++) {
    const uint8_t* e = src + HDR_BYTES + (size_t)IDX_ENTRY * i;
    uint64_t o = get64(e);
    uint32_t len = get32(e + 8);
    if (o != off || (len & 15u) || off + len > total) return KVCO_CORRUPT;
    off += len;
  }
  if (off != total) return KVCO_CORRUPT;
  *first = f;
  *n_slices = ns;
  *n_rec = nr;
  return KVCO_OK;
}

/* ---------------------------------------------------------------------------
 * Lossless front-end ([AT1] "KV & tensor mode": token-major floats reordered to
 * channel-major and split into byte planes, keeping whichever is smaller;
 * [QATQ] "qatq encode": chunks of at most 65536 values, row width known).
 * Reading: the channel-major reorder is applied inside each chunk of
 * tc = floor(values_per_chunk / D) consecutive tokens of one slice (the last
 * chunk of a slice may be shorter). Plane p holds byte p (p = 0 low) of every
 * 16-bit value in channel-major order i = d * tc' + t.
 * ------------------------------------------------------------------------- */
static uint32_t lossless_tc(const kvco_desc* d) { return d->values_per_chunk / d->head_dim; }

/* Bytes per value, and so byte planes per chunk: 2 for bf16 / fp16, 4 for f32
 * ([QATQ] "f32, f16, and bf16"; [AT-1] "Works on fp32/fp16/bf16"). */
static uint32_t elem_bytes(const kvco_desc* d) { return d->dtype == KVCO_F32 ? 4u : 2u; }

static int lossless_ok(const kvco_desc* d) {
  return desc_ok(d) && d->values_per_chunk <= 65536u && d->values_per_chunk >= d->head_dim;
}

static uint64_t lossless_records(const kvco_desc* d, uint32_t n_slices) {
  uint32_t tc = lossless_tc(d);
  return (uint64_t)n_slices * ((d->n_tokens + tc - 1) / tc);
}

size_t kvco_lossless_bound(const kvco_desc* d, uint32_t n_slices) {
  if (!lossless_ok(d)) return 0;
  uint32_t tc = lossless_tc(d), T = d->n_tokens, D = d->head_dim, E = elem_bytes(d);
  size_t per_slice = 0;
  for (uint32_t t0 = 0; t0 < T; t0 += tc) {
    uint32_t tcc = T - t0 < tc ? T - t0 : tc;
    per_slice += E * (16u + pad16((size_t)tcc * D)) + IDX_ENTRY;
  }
  return HDR_BYTES + per_slice * n_slices;
}

/* Chunk record: for p = 0 .. E-1, the stream record of plane p (byte p of
 * every little-endian value, channel-major order inside the chunk). Every
 * plane takes the lane-delta candidate ([QATQ] "How it works", lossless
 * candidates: delta-XOR, native 16-bit adjacent-XOR, shape-aware strided-XOR).
 * In the channel-major chunk a value's stream predecessor is the previous
 * token of its channel, which is also the value one row (the row width, the
 * shape-aware stride) back in the token-major input; XOR is bytewise, so the
 * 16-bit XOR with that predecessor is the lane delta of each byte plane; a
 * plane codes it where its counts are concentrated enough (the gate of
 * kvco_stream_encode_delta) and keeps it where it is strictly the smallest. */
size_t kvco_encode_lossless(const kvco_desc* d, uint32_t first_slice, uint32_t n_slices,
                            const void* src, uint8_t* dst, size_t cap) {
  if (!lossless_ok(d) || (uint64_t)first_slice + n_slices > n_slices_total(d)) return 0;
  size_t bound = kvco_lossless_bound(d, n_slices);
  if (cap < bound) return 0;
  uint32_t tc = lossless_tc(d), T = d->n_tokens, D = d->head_dim, E = elem_bytes(d);
  const uint8_t* in = (const uint8_t*)src;
  uint32_t nr = (uint32_t)lossless_records(d, n_slices);
  uint8_t* pl = (uint8_t*)malloc((size_t)tc * D);
  size_t p = HDR_BYTES + (size_t)IDX_ENTRY * nr;
  uint32_t r = 0;
  for (uint32_t s = 0; s < n_slices; s++) {
    for (uint32_t t0 = 0; t0 < T; t0 += tc) {
      uint32_t tcc = T - t0 < tc ? T - t0 : tc;
      uint32_t n = tcc * D;
      size_t start = p;
      for (uint32_t b = 0; b < E; b++) {
        for (uint32_t dd = 0; dd < D; dd++)
          for (uint32_t t = 0; t < tcc; t++)
            pl[(size_t)dd * tcc + t] = in[(((size_t)s * T + t0 + t) * D + dd) * E + b];
        p += kvco_stream_encode_delta(pl, n, dst + p);
      }
      uint8_t* e = dst + HDR_BYTES + (size_t)IDX_ENTRY * r;
      put64(e, start);
      put32(e + 8, (uint32_t)(p - start));
      put32(e + 12, kvco_crc32(dst + start, p - start));
      r++;
    }
  }
  free(pl);
  write_header(dst, KVCO_LOSSLESS, d, first_slice, n_slices, tc, nr, p, 0);
  put32(dst + 60, header_crc(dst, nr));
  return p;
}

int kvco_decode_lossless(const kvco_desc* d, const uint8_t* src, size_t n, void* dst,
                         size_t cap, uint64_t* written) {
  if (!lossless_ok(d)) return KVCO_INVALID;
  uint32_t first, ns, nr;
  int st = check_container(d, KVCO_LOSSLESS, src, n, lossless_records, lossless_tc(d), 0,
                           &first, &ns, &nr);
  if (st) return st;
  uint32_t tc = lossless_tc(d), T = d->n_tokens, D = d->head_dim, E = elem_bytes(d);
  uint64_t out_bytes = (uint64_t)ns * T * D * E;
  if (out_bytes > cap) return KVCO_CAPACITY;
  uint8_t* out = (uint8_t*)dst;
  uint8_t* pl = (uint8_t*)malloc((size_t)tc * D);
  uint32_t r = 0;
  st = KVCO_OK;
  for (uint32_t s = 0; s < ns && !st; s++) {
    for (uint32_t t0 = 0; t0 < T && !st; t0 += tc, r++) {
      uint32_t tcc = T - t0 < tc ? T - t0 : tc;
      uint32_t nv = tcc * D;
      const uint8_t* e = src + HDR_BYTES + (size_t)IDX_ENTRY * r;
      const uint8_t* rec = src + get64(e);
      uint32_t len = get32(e + 8);
      if (kvco_crc32(rec, len) != get32(e + 12)) { st = KVCO_CORRUPT; break; }
      size_t off = 0;
      for (uint32_t b = 0; b < E && !st; b++) {
        size_t used = 0;
        st = kvco_stream_decode(rec + off, len - off, nv, pl, &used);
        if (st) break;
        off += used;
        for (uint32_t dd = 0; dd < D; dd++)
          for (uint32_t t = 0; t < tcc; t++)
            out[(((size_t)s * T + t0 + t) * D + dd) * E + b] = pl[(size_t)dd * tcc + t];
      }
      if (!st && off != len) st = KVCO_CORRUPT;
    }
  }
  free(pl);
  if (!st && written) *written = out_bytes;
  return st;
}

/* ---------------------------------------------------------------------------
 * Rotary position table and rotations ([KVTC] "Why RoPE Has to Be Reversed
 * First": undo the positional rotation on keys before the basis change).
 * Reading: half-split pairs (i, i + D/2), angle t * theta^(-2i/D); the table is
 * computed in fp64 and stored as fp32 cos, sin: cs[(t * D/2 + i) * 2 + {0,1}].
 * Rotations are fp32 with every product and sum rounded on its own (no fused
 * multiply-add):
 *   inverse: a' = fl(fl(a c) + fl(b s)), b' = fl(fl(b c) - fl(a s))
 *   forward: a' = fl(fl(a c) - fl(b s)), b' = fl(fl(a s) + fl(b c))
 * ------------------------------------------------------------------------- */
void kvco_rope_table(uint32_t T, uint32_t D, double theta, float* cs) {
  uint32_t half = D / 2;
  for (uint32_t t = 0; t < T; t++)
    for (uint32_t i = 0; i < half; i++) {
      double inv = pow(theta, -(2.0 * (double)i) / (double)D);
      double a = (double)t * inv;
      cs[((size_t)t * half + i) * 2] = (float)cos(a);
      cs[((size_t)t * half + i) * 2 + 1] = (float)sin(a);
    }
}

void kvco_rope_inverse(const float* cs_row, uint32_t D, float* x) {
  uint32_t half = D / 2;
  for (uint32_t i = 0; i < half; i++) {
    float a = x[i], b = x[i + half], c = cs_row[2 * i], s = cs_row[2 * i + 1];
    float ac = a * c, bs = b * s, bc = b * c, as = a * s;
    x[i] = ac + bs;
    x[i + half] = bc - as;
  }
}

void kvco_rope_forward(const float* cs_row, uint32_t D, float* x) {
  uint32_t half = D / 2;
  for (uint32_t i = 0; i < half; i++) {
    float a = x[i], b = x[i + half], c = cs_row[2 * i], s = cs_row[2 * i + 1];
    float ac = a * c, bs = b * s, as = a * s, bc = b * c;
    x[i] = ac - bs;
    x[i + half] = as + bc;
  }
}

/* ---------------------------------------------------------------------------
 * Greedy bit allocation ([KVTC] "Bit Budget Is Not Fair": greedy variants in the
 * fast path; the budget moves across layers). Units are every
 * (layer, K/V, head, component). Every unit starts at 0 bits; the budget
 * B = floor(avg_bits * U + 0.5) is spent one bit at a time on the unit with
 * the largest lambda * 4^-b (ties: lowest unit index), no unit above max_bits.
 * A binary max-heap keyed on (gain, -index) finds that unit.
 * ------------------------------------------------------------------------- */
typedef struct { double gain; uint64_t idx; } heap_item;

static int heap_before(const heap_item* a, const heap_item* b) {
  return a->gain > b->gain || (a->gain == b->gain && a->idx < b->idx);
}

static void heap_down(heap_item* h, size_t n, size_t i) {
  for (;;) {
    size_t l = 2 * i + 1, r = l + 1, m = i;
    if (l < n && heap_before(&h[l], &h[m])) m = l;
    if (r < n && heap_before(&h[r], &h[m])) m = r;
    if (m == i) return;
    heap_item t = h[i]; h[i] = h[m]; h[m] = t;
    i = m;
  }
}

int kvco_allocate(const double* lambda, uint64_t n_units, double avg_bits, uint32_t max_bits,
                  uint8_t* widths) {
  if (n_units == 0 || max_bits > 8 || !(avg_bits >= 0.0)) return KVCO_INVALID;
  double bd = floor(avg_bits * (double)n_units + 0.5);
  if (bd > (double)max_bits * (double)n_units) return KVCO_INVALID;
  uint64_t budget = (uint64_t)bd;
  for (uint64_t u = 0; u < n_units; u++)
    if (lambda[u] != lambda[u]) return KVCO_INVALID;
  heap_item* h = (heap_item*)malloc(sizeof(heap_item) * n_units);
  /* a variance below zero (eigenvalue round-off) carries no distortion */
  double* lam = (double*)malloc(sizeof(double) * n_units);
  for (uint64_t u = 0; u < n_units; u++) {
    lam[u] = lambda[u] > 0.0 ? lambda[u] : 0.0;
    widths[u] = 0;
    h[u].gain = lam[u];
    h[u].idx = u;
  }
  size_t n = n_units;
  for (size_t i = n / 2; i-- > 0;) heap_down(h, n, i);
  for (uint64_t k = 0; k < budget; k++) {
    uint64_t u = h[0].idx;
    widths[u]++;
    if (widths[u] < max_bits) {
      h[0].gain = ldexp(lam[u], -2 * (int)widths[u]);
    } else {
      h[0] = h[n - 1];
      n--;
    }
    heap_down(h, n, 0);
  }
  free(h);
  free(lam);
  return KVCO_OK;
}

/* CRC32 over the plan parameters that the bytes depend on: u32 dtype, L, H, T, D,
 * n_sink, n_recent, block_tokens, chunk_tokens, max_bits; u64 bits of theta;
 * the U widths; the bases as little-endian fp32; then, for a range mode other
 * than BLOCK, u32 ranges. */
uint32_t kvco_plan_crc(const kvco_desc* d) {
  uint64_t U = (uint64_t)n_slices_total(d) * d->head_dim;
  size_t len = 48 + U + U * d->head_dim * 4u + (d->ranges ? 4u : 0u);
  uint8_t* b = (uint8_t*)malloc(len);
  uint32_t v[10] = {d->dtype, d->n_layers, d->n_heads, d->n_tokens, d->head_dim,
                    d->n_sink, d->n_recent, d->block_tokens, d->chunk_tokens, d->max_bits};
  for (int i = 0; i < 10; i++) put32(b + 4 * i, v[i]);
  uint64_t tb;
  memcpy(&tb, &d->rope_theta, 8);
  put64(b + 40, tb);
  memcpy(b + 48, d->widths, U);
  for (uint64_t i = 0; i < U * d->head_dim; i++) {
    uint32_t fb;
    memcpy(&fb, &d->bases[i], 4);
    put32(b + 48 + U + 4 * i, fb);
  }
  if (d->ranges) put32(b + len - 4, d->ranges);  /* only a non-default range mode */
  uint32_t crc = kvco_crc32(b, len);
  free(b);
  return crc;
}

/* The plan CRC a container carries: the caller's precomputed value when set. */
static uint32_t plan_crc_of(const kvco_desc* d) {
  return d->plan_crc_set ? d->plan_crc : kvco_plan_crc(d);
}

/* ---------------------------------------------------------------------------
 * Transform coding ([KVTC] "How the Pipeline Works": sink tokens and a recent
 * window kept at full fidelity, the middle RoPE-undone, projected on a PCA basis,
 * quantised with scales, zero points and bit widths, then rANS coded;
 * [GAUGE] "Problem Statement and Overview": Z = G X per (layer, K/V, head) with
 * inverse G^T; "Compression Conditions": block-uniform ranges per token block).
 *   regions: sinks [0, s_end), middle [s_end, r_start), recent [r_start, T),
 *     s_end = min(n_sink, T), r_start = max(s_end, T - n_recent);
 *   per slice one raw record (sink then recent token rows, bf16 bytes, padded)
 *   then the middle in chunks of chunk_tokens tokens from s_end (last shorter);
 *   per token: x = fp32(bf16); keys: inverse rotation; y_j = (float) sum_k
 *     (double) Q[k][j] * (double) x_k, k ascending in fp64, rounded once;
 *   per component j with b_j > 0 and block of block_tokens tokens (aligned at
 *     the chunk start, last may be shorter): z = min y, s = fl(max - min) /
 *     (2^b - 1) in fp32 (0 if max == min);
 *     code = clamp(rint_even(fl(fl(y - z) / s)), 0, 2^b - 1), 0 if s == 0;
 *   record: the side information as four stream records, then for b = 1..8
 *     with m_b > 0 components one stream of m_b * tc codes (components
 *     ascending, each component's tokens in order) in the stream record format
 *     above. The side information is the sequence V of 2 * coded * nb fp32
 *     values: every z (for j ascending with b_j > 0, for each block), then
 *     every s in the same order; stream p (p = 0..3) holds byte p of each value
 *     of V, on the side lane rule, and may take the lane delta (no side streams
 *     when nothing is coded).
 *   decode: y^ = fmaf(code, s, z) (0 for b_j = 0); x^_k = (float) sum_j
 *     (double) Q[k][j] * (double) y^_j in fp64; keys: forward rotation;
 *     bf16 round-to-nearest-even.
 * ------------------------------------------------------------------------- */
static int transform_ok(const kvco_desc* d) {
  if (!desc_ok(d) || d->dtype != KVCO_BF16 || (d->head_dim & 1u)) return 0;
  if (!d->bases || !d->widths || d->max_bits > 8) return 0;
  if (!d->block_tokens || !d->chunk_tokens || d->chunk_tokens % d->block_tokens) return 0;
  if ((uint64_t)d->chunk_tokens * d->head_dim > 65536u) return 0;
  if (d->n_sink > 65535u || d->n_recent > 65535u || d->block_tokens > 65535u) return 0;
  if (!(d->rope_theta > 0.0)) return 0;
  if (d->ranges > KVCO_RANGES_KIVI) return 0;
  /* a KIVI-style chunk's (z, range) pairs, one per token, use the side buffers
   * of its D x (ct / B) (z, s) pairs */
  if (d->ranges == KVCO_RANGES_KIVI && d->head_dim < d->block_tokens) return 0;
  return 1;
}

/* Values of a KIVI-style plan take one range per token ([GAUGE] "Compression
 * Conditions": per-channel key ranges, per-token value ranges); keys keep the
 * per-component block ranges, which are per-channel ranges in the basis. */
static int kivi_values(const kvco_desc* d, uint32_t sidx) {
  return d->ranges == KVCO_RANGES_KIVI && ((sidx / d->n_heads) % 2u) == 1u;
}

/* Values of V, the side information of a middle record of tcc tokens: every
 * zero point, then every scale or range. */
static uint32_t side_values(const kvco_desc* d, uint32_t sidx, uint32_t coded, uint32_t tcc) {
  if (!coded) return 0;
  return kivi_values(d, sidx) ? 2u * tcc : 2u * coded * ((tcc + d->block_tokens - 1) / d->block_tokens);
}

static void regions(const kvco_desc* d, uint32_t* s_end, uint32_t* r_start) {
  uint32_t T = d->n_tokens;
  *s_end = d->n_sink < T ? d->n_sink : T;
  uint32_t rs = T > d->n_recent ? T - d->n_recent : 0;
  *r_start = rs > *s_end ? rs : *s_end;
}

static uint32_t n_mid_chunks(const kvco_desc* d) {
  uint32_t s_end, r_start;
  regions(d, &s_end, &r_start);
  return (r_start - s_end + d->chunk_tokens - 1) / d->chunk_tokens;
}

static uint64_t transform_records(const kvco_desc* d, uint32_t n_slices) {
  return (uint64_t)n_slices * (1u + n_mid_chunks(d));
}

static uint32_t count_width(const uint8_t* w, uint32_t D, uint32_t b) {
  uint32_t m = 0;
  for (uint32_t j = 0; j < D; j++) m += (w[j] == b);
  return m;
}

static size_t mid_record_bound(const kvco_desc* d, uint32_t sidx, uint32_t tcc) {
  const uint8_t* w = d->widths + (size_t)sidx * d->head_dim;
  uint32_t coded = d->head_dim - count_width(w, d->head_dim, 0);
  uint32_t nv = side_values(d, sidx, coded, tcc);
  size_t bytes = nv ? 4u * (16u + pad16((size_t)nv)) : 0u;  /* side streams at most RAW */
  for (uint32_t b = 1; b <= 8; b++) {
    uint32_t m = count_width(w, d->head_dim, b);
    if (m) bytes += 16u + pad16((size_t)m * tcc);
  }
  return bytes;
}

/* Bytes of the parser's scratch: a stream of codes (ct * D) or the four side
 * planes (8 * D * ct / B). */
static size_t parse_buf_bytes(const kvco_desc* d) {
  size_t a = (size_t)d->chunk_tokens * d->head_dim;
  size_t b = (size_t)8 * d->head_dim * (d->chunk_tokens / d->block_tokens);
  return a > b ? a : b;
}

/* Largest record bytes of one slice (raw record + middle records at most RAW). */
static size_t slice_bound(const kvco_desc* d, uint32_t sl) {
  uint32_t s_end, r_start, T = d->n_tokens, D = d->head_dim;
  regions(d, &s_end, &r_start);
  uint32_t nm = n_mid_chunks(d);
  size_t b = pad16((size_t)(s_end + T - r_start) * D * 2u);
  for (uint32_t c = 0; c < nm; c++) {
    uint32_t t0 = s_end + c * d->chunk_tokens;
    uint32_t tcc = r_start - t0 < d->chunk_tokens ? r_start - t0 : d->chunk_tokens;
    b += mid_record_bound(d, sl, tcc);
  }
  return b;
}

size_t kvco_transform_bound(const kvco_desc* d, uint32_t n_slices) {
  if (!transform_ok(d)) return 0;
  size_t max_slice = 0;
  for (uint32_t sl = 0; sl < n_slices_total(d); sl++) {
    size_t b = slice_bound(d, sl);
    if (b > max_slice) max_slice = b;
  }
  return HDR_BYTES + (size_t)n_slices * ((size_t)IDX_ENTRY * (1u + n_mid_chunks(d)) + max_slice);
}

/* The most bytes slices [first, first + n) can take (at most the bound above). */
static size_t transform_range_bound(const kvco_desc* d, uint32_t first, uint32_t n) {
  size_t b = HDR_BYTES + (size_t)n * IDX_ENTRY * (1u + n_mid_chunks(d));
  for (uint32_t sl = first; sl < first + n; sl++) b += slice_bound(d, sl);
  return b;
}

/* y_j = (float) sum_k (double) Q[k][j] * (double) x_k, k ascending, fp64 sum
 * rounded once ([GAUGE] "Problem Statement and Overview": Z = G X, here G = Q^T). */
void kvco_project(const float* Q, uint32_t D, const float* x, float* y) {
  for (uint32_t j = 0; j < D; j++) {
    double acc = 0.0;
    for (uint32_t k = 0; k < D; k++) acc += (double)Q[(size_t)k * D + j] * (double)x[k];
    y[j] = (float)acc;
  }
}

/* x_k = (float) sum_j (double) Q[k][j] * (double) y_j, j ascending (G^-1 = G^T). */
void kvco_unproject(const float* Q, uint32_t D, const float* y, float* x) {
  for (uint32_t k = 0; k < D; k++) {
    double acc = 0.0;
    for (uint32_t j = 0; j < D; j++) acc += (double)Q[(size_t)k * D + j] * (double)y[j];
    x[k] = (float)acc;
  }
}

static uint32_t quantize(float y, float z, float s, uint32_t levels, float* qpre) {
  if (s == 0.0f) {
    if (qpre) *qpre = 0.0f;
    return 0;
  }
  float dlt = y - z;
  float q = dlt / s;
  if (qpre) *qpre = q;
  float r = rintf(q);
  if (!(r > 0.0f)) return 0;
  if (r >= (float)levels) return levels;
  return (uint32_t)r;
}

/* Project and quantise one middle chunk. codes[j * ct + t]; qpre[t * D + j]
 * (optional); zs[(j * nbmax + blk) * 2 + {0: z, 1: s}], or for the values of a
 * KIVI-style plan zs[t * 2 + {0: z, 1: range}]. */
static void mid_chunk_quantize(const kvco_desc* d, uint32_t sidx, const uint16_t* xs,
                               const float* cs, uint32_t t0, uint32_t tcc, float* y,
                               uint8_t* codes, float* qpre, float* zs) {
  uint32_t D = d->head_dim, half = D / 2, H = d->n_heads, ct = d->chunk_tokens;
  uint32_t B = d->block_tokens, nbmax = ct / B;
  int is_key = ((sidx / H) % 2u) == 0;
  const float* Q = d->bases + (size_t)sidx * D * D;
  const uint8_t* w = d->widths + (size_t)sidx * D;
  float* x = (float*)malloc(sizeof(float) * D);
  for (uint32_t t = 0; t < tcc; t++) {
    uint32_t ta = t0 + t;
    for (uint32_t k = 0; k < D; k++) x[k] = kvco_bf16_to_f32(xs[(size_t)ta * D + k]);
    if (is_key) kvco_rope_inverse(cs + (size_t)ta * half * 2, D, x);
    kvco_project(Q, D, x, y + (size_t)t * D);
  }
  free(x);
  if (kivi_values(d, sidx)) {
    /* per token: z = min over the coded components (ascending), range =
     * fl(max - min); a component of width b uses s = fl(range / (2^b - 1)) */
    for (uint32_t t = 0; t < tcc; t++) {
      float mn = 0.0f, mx = 0.0f;
      int first = 1;
      for (uint32_t j = 0; j < D; j++) {
        if (!w[j]) continue;
        float v = y[(size_t)t * D + j];
        if (first) { mn = mx = v; first = 0; continue; }
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      float rng = mx - mn;
      for (uint32_t j = 0; j < D; j++) {
        uint32_t b = w[j];
        if (!b) {
          codes[(size_t)j * ct + t] = 0;
          if (qpre) qpre[(size_t)t * D + j] = 0.0f;
          continue;
        }
        uint32_t levels = (1u << b) - 1u;
        float sc = (mx == mn) ? 0.0f : rng / (float)levels;
        codes[(size_t)j * ct + t] =
            (uint8_t)quantize(y[(size_t)t * D + j], mn, sc, levels, qpre ? &qpre[(size_t)t * D + j] : NULL);
      }
      if (zs) {
        zs[(size_t)t * 2] = mn;
        zs[(size_t)t * 2 + 1] = first ? 0.0f : rng;
      }
    }
    return;
  }
  uint32_t nb = (tcc + B - 1) / B;
  for (uint32_t j = 0; j < D; j++) {
    uint32_t b = w[j];
    for (uint32_t blk = 0; blk < nb; blk++) {
      uint32_t lo = blk * B, hi = lo + B < tcc ? lo + B : tcc;
      if (b == 0) {
        for (uint32_t t = lo; t < hi; t++) {
          codes[(size_t)j * ct + t] = 0;
          if (qpre) qpre[(size_t)t * D + j] = 0.0f;
        }
        if (zs) zs[((size_t)j * nbmax + blk) * 2] = zs[((size_t)j * nbmax + blk) * 2 + 1] = 0.0f;
        continue;
      }
      uint32_t levels = (1u << b) - 1u;
      float mn = y[(size_t)lo * D + j], mx = mn;
      for (uint32_t t = lo + 1; t < hi; t++) {
        float v = y[(size_t)t * D + j];
        if (v < mn) mn = v;
        if (v > mx) mx = v;
      }
      float rng = mx - mn;
      float s = (mx == mn) ? 0.0f : rng / (float)levels;
      for (uint32_t t = lo; t < hi; t++)
        codes[(size_t)j * ct + t] = (uint8_t)quantize(
            y[(size_t)t * D + j], mn, s, levels, qpre ? &qpre[(size_t)t * D + j] : NULL);
      if (zs) {
        zs[((size_t)j * nbmax + blk) * 2] = mn;
        zs[((size_t)j * nbmax + blk) * 2 + 1] = s;
      }
    }
  }
}

size_t kvco_encode_transform(const kvco_desc* d, uint32_t first_slice, uint32_t n_slices,
                             const uint16_t* src, uint8_t* dst, size_t cap) {
  if (!transform_ok(d) || (uint64_t)first_slice + n_slices > n_slices_total(d)) return 0;
  if (cap < transform_range_bound(d, first_slice, n_slices)) return 0;
  uint32_t T = d->n_tokens, D = d->head_dim, half = D / 2, ct = d->chunk_tokens;
  uint32_t B = d->block_tokens, nbmax = ct / B;
  uint32_t s_end, r_start;
  regions(d, &s_end, &r_start);
  uint32_t nm = n_mid_chunks(d);
  uint32_t nr = n_slices * (1u + nm);
  float* cs = (float*)malloc(sizeof(float) * (size_t)T * half * 2);
  kvco_rope_table(T, D, d->rope_theta, cs);
  float* y = (float*)malloc(sizeof(float) * (size_t)ct * D);
  uint8_t* codes = (uint8_t*)malloc((size_t)ct * D);
  uint8_t* syms = (uint8_t*)malloc(parse_buf_bytes(d));
  float* zs = (float*)malloc(sizeof(float) * (size_t)D * nbmax * 2);
  uint8_t* side = (uint8_t*)malloc((size_t)4 * 2 * D * nbmax);  /* four byte planes of V */
  size_t p = HDR_BYTES + (size_t)IDX_ENTRY * nr;
  uint32_t r = 0;
  for (uint32_t s = 0; s < n_slices; s++) {
    uint32_t sidx = first_slice + s;
    const uint16_t* xs = src + (size_t)s * T * D;
    const uint8_t* w = d->widths + (size_t)sidx * D;
    /* raw record: sink rows then recent rows */
    size_t start = p;
    for (uint32_t t = 0; t < T; t++) {
      if (t >= s_end && t < r_start) continue;
      for (uint32_t k = 0; k < D; k++) {
        put16(dst + p, xs[(size_t)t * D + k]);
        p += 2;
      }
    }
    while (p & 15u) dst[p++] = 0;
    uint8_t* e = dst + HDR_BYTES + (size_t)IDX_ENTRY * r++;
    put64(e, start);
    put32(e + 8, (uint32_t)(p - start));
    put32(e + 12, kvco_crc32(dst + start, p - start));
    for (uint32_t c = 0; c < nm; c++) {
      uint32_t t0 = s_end + c * ct;
      uint32_t tcc = r_start - t0 < ct ? r_start - t0 : ct;
      uint32_t nb = (tcc + B - 1) / B;
      mid_chunk_quantize(d, sidx, xs, cs, t0, tcc, y, codes, NULL, zs);
      start = p;
      /* side information: V = every z, then every s (KIVI-style values: every
       * token's z, then every token's range), split into byte planes */
      uint32_t coded = D - count_width(w, D, 0), nv = side_values(d, sidx, coded, tcc), i = 0;
      for (uint32_t half_v = 0; half_v < 2 && nv; half_v++) {
        if (kivi_values(d, sidx)) {
          for (uint32_t t = 0; t < tcc; t++, i++) {
            uint32_t v;
            memcpy(&v, &zs[(size_t)t * 2 + half_v], 4);
            for (uint32_t q = 0; q < 4; q++) side[(size_t)q * nv + i] = (uint8_t)(v >> (8u * q));
          }
          continue;
        }
        for (uint32_t j = 0; j < D; j++) {
          if (!w[j]) continue;
          for (uint32_t blk = 0; blk < nb; blk++, i++) {
            uint32_t v;
            memcpy(&v, &zs[((size_t)j * nbmax + blk) * 2 + half_v], 4);
            for (uint32_t q = 0; q < 4; q++) side[(size_t)q * nv + i] = (uint8_t)(v >> (8u * q));
          }
        }
      }
      if (nv)
        for (uint32_t q = 0; q < 4; q++) p += kvco_side_stream_encode(side + (size_t)q * nv, nv, dst + p);
      for (uint32_t b = 1; b <= 8; b++) {
        uint32_t m = 0;
        for (uint32_t j = 0; j < D; j++) {
          if (w[j] != b) continue;
          memcpy(syms + (size_t)m * tcc, codes + (size_t)j * ct, tcc);
          m++;
        }
        if (m) p += kvco_stream_encode(syms, m * tcc, dst + p);
      }
      e = dst + HDR_BYTES + (size_t)IDX_ENTRY * r++;
      put64(e, start);
      put32(e + 8, (uint32_t)(p - start));
      put32(e + 12, kvco_crc32(dst + start, p - start));
    }
  }
  free(cs); free(y); free(codes); free(syms); free(zs); free(side);
  write_header(dst, KVCO_TRANSFORM, d, first_slice, n_slices, ct, nr, p, plan_crc_of(d));
  put32(dst + 60, header_crc(dst, nr));
  return p;
}

/* Parse one middle-chunk record into codes[j * ct + t] and zs. */
static int mid_chunk_parse(const kvco_desc* d, uint32_t sidx, const uint8_t* rec, uint32_t len,
                           uint32_t tcc, uint8_t* codes, float* zs, uint8_t* syms) {
  uint32_t D = d->head_dim, ct = d->chunk_tokens, B = d->block_tokens, nbmax = ct / B;
  const uint8_t* w = d->widths + (size_t)sidx * D;
  uint32_t nb = (tcc + B - 1) / B;
  uint32_t coded = D - count_width(w, D, 0), nv = side_values(d, sidx, coded, tcc);
  size_t p = 0;
  /* side streams: byte q of every value of V (the syms buffer holds ct * D >= 4 nv bytes) */
  for (uint32_t q = 0; q < 4 && nv; q++) {
    size_t used = 0;
    int st = stream_decode(rec + p, len - p, nv, syms + (size_t)q * nv, &used, 1, 1);
    if (st) return st;
    p += used;
  }
  uint32_t i = 0;
  for (uint32_t j = 0; j < D; j++) {
    for (uint32_t blk = 0; blk < nbmax; blk++)
      zs[((size_t)j * nbmax + blk) * 2] = zs[((size_t)j * nbmax + blk) * 2 + 1] = 0.0f;
    memset(codes + (size_t)j * ct, 0, ct);
  }
  for (uint32_t half_v = 0; half_v < 2 && nv; half_v++) {
    if (kivi_values(d, sidx)) {
      for (uint32_t t = 0; t < tcc; t++, i++) {
        uint32_t v = 0;
        for (uint32_t q = 0; q < 4; q++) v |= (uint32_t)syms[(size_t)q * nv + i] << (8u * q);
        memcpy(&zs[(size_t)t * 2 + half_v], &v, 4);
      }
      continue;
    }
    for (uint32_t j = 0; j < D; j++) {
      if (!w[j]) continue;
      for (uint32_t blk = 0; blk < nb; blk++, i++) {
        uint32_t v = 0;
        for (uint32_t q = 0; q < 4; q++) v |= (uint32_t)syms[(size_t)q * nv + i] << (8u * q);
        memcpy(&zs[((size_t)j * nbmax + blk) * 2 + half_v], &v, 4);
      }
    }
  }
  for (uint32_t b = 1; b <= 8; b++) {
    uint32_t m = count_width(w, D, b);
    if (!m) continue;
    size_t used = 0;
    int st = stream_decode(rec + p, len - p, m * tcc, syms, &used, 0, 0);  /* no lane delta here */
    if (st) return st;
    p += used;
    uint32_t mm = 0;
    for (uint32_t j = 0; j < D; j++) {
      if (w[j] != b) continue;
      for (uint32_t t = 0; t < tcc; t++) {
        uint8_t c = syms[(size_t)mm * tcc + t];
        if (c > (1u << b) - 1u) return KVCO_CORRUPT;
        codes[(size_t)j * ct + t] = c;
      }
      mm++;
    }
  }
  if (p != len) return KVCO_CORRUPT;
  return KVCO_OK;
}

int kvco_decode_transform(const kvco_desc* d, const uint8_t* src, size_t n, uint16_t* dst,
                          size_t cap, uint64_t* written) {
  if (!transform_ok(d)) return KVCO_INVALID;
  uint32_t first, ns, nr;
  int st = check_container(d, KVCO_TRANSFORM, src, n, transform_records, d->chunk_tokens,
                           plan_crc_of(d), &first, &ns, &nr);
  if (st) return st;
  uint32_t T = d->n_tokens, D = d->head_dim, half = D / 2, ct = d->chunk_tokens;
  uint32_t H = d->n_heads, B = d->block_tokens, nbmax = ct / B;
  uint64_t out_bytes = (uint64_t)ns * T * D * 2u;
  if (out_bytes > cap) return KVCO_CAPACITY;
  uint32_t s_end, r_start;
  regions(d, &s_end, &r_start);
  uint32_t nm = n_mid_chunks(d);
  size_t raw_len = pad16((size_t)(s_end + T - r_start) * D * 2u);
  float* cs = (float*)malloc(sizeof(float) * (size_t)T * half * 2);
  kvco_rope_table(T, D, d->rope_theta, cs);
  uint8_t* codes = (uint8_t*)malloc((size_t)ct * D);
  uint8_t* syms = (uint8_t*)malloc(parse_buf_bytes(d));
  float* zs = (float*)malloc(sizeof(float) * (size_t)D * nbmax * 2);
  float* yh = (float*)malloc(sizeof(float) * D);
  float* xh = (float*)malloc(sizeof(float) * D);
  uint32_t r = 0;
  for (uint32_t s = 0; s < ns && !st; s++) {
    uint32_t sidx = first + s;
    int is_key = ((sidx / H) % 2u) == 0;
    const float* Q = d->bases + (size_t)sidx * D * D;
    const uint8_t* w = d->widths + (size_t)sidx * D;
    uint16_t* xs = dst + (size_t)s * T * D;
    const uint8_t* e = src + HDR_BYTES + (size_t)IDX_ENTRY * r++;
    const uint8_t* rec = src + get64(e);
    uint32_t len = get32(e + 8);
    if (kvco_crc32(rec, len) != get32(e + 12) || len != raw_len) { st = KVCO_CORRUPT; break; }
    size_t p = 0;
    for (uint32_t t = 0; t < T; t++) {
      if (t >= s_end && t < r_start) continue;
      for (uint32_t k = 0; k < D; k++) {
        xs[(size_t)t * D + k] = (uint16_t)get16(rec + p);
        p += 2;
      }
    }
    for (uint32_t c = 0; c < nm && !st; c++) {
      uint32_t t0 = s_end + c * ct;
      uint32_t tcc = r_start - t0 < ct ? r_start - t0 : ct;
      e = src + HDR_BYTES + (size_t)IDX_ENTRY * r++;
      rec = src + get64(e);
      len = get32(e + 8);
      if (kvco_crc32(rec, len) != get32(e + 12)) { st = KVCO_CORRUPT; break; }
      st = mid_chunk_parse(d, sidx, rec, len, tcc, codes, zs, syms);
      if (st) break;
      const int kv = kivi_values(d, sidx);
      for (uint32_t t = 0; t < tcc; t++) {
        uint32_t blk = t / B;
        for (uint32_t j = 0; j < D; j++) {
          if (!w[j]) { yh[j] = 0.0f; continue; }
          float z, sc;
          if (kv) {  /* the token's zero point; its range in 2^b - 1 steps */
            float rng = zs[(size_t)t * 2 + 1];
            z = zs[(size_t)t * 2];
            sc = rng == 0.0f ? 0.0f : rng / (float)((1u << w[j]) - 1u);
          } else {
            z = zs[((size_t)j * nbmax + blk) * 2];
            sc = zs[((size_t)j * nbmax + blk) * 2 + 1];
          }
          yh[j] = fmaf((float)codes[(size_t)j * ct + t], sc, z);
        }
        kvco_unproject(Q, D, yh, xh);
        if (is_key) kvco_rope_forward(cs + (size_t)(t0 + t) * half * 2, D, xh);
        for (uint32_t k = 0; k < D; k++) xs[(size_t)(t0 + t) * D + k] = kvco_f32_to_bf16(xh[k]);
      }
    }
  }
  free(cs); free(codes); free(syms); free(zs); free(yh); free(xh);
  if (!st && written) *written = out_bytes;
  return st;
}

/* Test helper: the oracle's codes, pre-rounding quotients and side info for one
 * slice (global index). codes/qpre are [T][D] token-major (0 outside the middle
 * and for b = 0); zs is [n_mid][D][ct / B][2]. */
int kvco_transform_slice_codes(const kvco_desc* d, uint32_t slice, const uint16_t* src_slice,
                               uint8_t* codes, float* qpre, float* zs) {
  if (!transform_ok(d) || slice >= n_slices_total(d)) return KVCO_INVALID;
  uint32_t T = d->n_tokens, D = d->head_dim, half = D / 2, ct = d->chunk_tokens;
  uint32_t nbmax = ct / d->block_tokens;
  uint32_t s_end, r_start;
  regions(d, &s_end, &r_start);
  uint32_t nm = n_mid_chunks(d);
  float* cs = (float*)malloc(sizeof(float) * (size_t)T * half * 2);
  kvco_rope_table(T, D, d->rope_theta, cs);
  float* y = (float*)malloc(sizeof(float) * (size_t)ct * D);
  uint8_t* cc = (uint8_t*)malloc((size_t)ct * D);
  float* qq = (float*)malloc(sizeof(float) * (size_t)ct * D);
  memset(codes, 0, (size_t)T * D);
  memset(qpre, 0, sizeof(float) * (size_t)T * D);
  for (uint32_t c = 0; c < nm; c++) {
    uint32_t t0 = s_end + c * ct;
    uint32_t tcc = r_start - t0 < ct ? r_start - t0 : ct;
    mid_chunk_quantize(d, slice, src_slice, cs, t0, tcc, y, cc, qq,
                       zs + (size_t)c * D * nbmax * 2);
    for (uint32_t t = 0; t < tcc; t++)
      for (uint32_t j = 0; j < D; j++) {
        codes[(size_t)(t0 + t) * D + j] = cc[(size_t)j * ct + t];
        qpre[(size_t)(t0 + t) * D + j] = qq[(size_t)t * D + j];
      }
  }
  free(cs); free(y); free(cc); free(qq);
  return KVCO_OK;
}

/* Test helper: codes [tcc][D] token-major and side info [D][ct / B][2] of one
 * middle-chunk record of slice sidx (global index) holding tcc tokens. */
int kvco_record_codes(const kvco_desc* d, uint32_t sidx, const uint8_t* rec, uint32_t len,
                      uint32_t tcc, uint8_t* codes, float* zs) {
  if (!transform_ok(d) || sidx >= n_slices_total(d) || tcc == 0 || tcc > d->chunk_tokens)
    return KVCO_INVALID;
  uint32_t D = d->head_dim, ct = d->chunk_tokens;
  uint8_t* cc = (uint8_t*)malloc((size_t)ct * D);
  uint8_t* syms = (uint8_t*)malloc(parse_buf_bytes(d));
  int st = mid_chunk_parse(d, sidx, rec, len, tcc, cc, zs, syms);
  for (uint32_t t = 0; t < tcc && !st; t++)
    for (uint32_t j = 0; j < D; j++) codes[(size_t)t * D + j] = cc[(size_t)j * ct + t];
  free(cc);
  free(syms);
  return st;
}

/* Test helper: codes [n_slices][T][D] and side info [n_slices][n_mid][D][ct/B][2]
 * read back from a transform container (any producer), after full validation. */
int kvco_container_codes(const kvco_desc* d, const uint8_t* src, size_t n, uint32_t rec_unused,
                         uint8_t* codes, float* zs, uint32_t* n_slices_out) {
  (void)rec_unused;
  if (!transform_ok(d)) return KVCO_INVALID;
  uint32_t first, ns, nr;
  int st = check_container(d, KVCO_TRANSFORM, src, n, transform_records, d->chunk_tokens,
                           plan_crc_of(d), &first, &ns, &nr);
  if (st) return st;
  uint32_t T = d->n_tokens, D = d->head_dim, ct = d->chunk_tokens;
  uint32_t nbmax = ct / d->block_tokens;
  uint32_t s_end, r_start;
  regions(d, &s_end, &r_start);
  uint32_t nm = n_mid_chunks(d);
  uint8_t* cc = (uint8_t*)malloc((size_t)ct * D);
  uint8_t* syms = (uint8_t*)malloc(parse_buf_bytes(d));
  memset(codes, 0, (size_t)ns * T * D);
  uint32_t r = 0;
  for (uint32_t s = 0; s < ns && !st; s++) {
    r++; /* raw record */
    for (uint32_t c = 0; c < nm && !st; c++) {
      uint32_t t0 = s_end + c * ct;
      uint32_t tcc = r_start - t0 < ct ? r_start - t0 : ct;
      const uint8_t* e = src + HDR_BYTES + (size_t)IDX_ENTRY * r++;
      const uint8_t* rec = src + get64(e);
      uint32_t len = get32(e + 8);
      if (kvco_crc32(rec, len) != get32(e + 12)) { st = KVCO_CORRUPT; break; }
      st = mid_chunk_parse(d, first + s, rec, len, tcc, cc,
                           zs + ((size_t)s * nm + c) * D * nbmax * 2, syms);
      for (uint32_t t = 0; t < tcc && !st; t++)
        for (uint32_t j = 0; j < D; j++)
          codes[((size_t)s * T + t0 + t) * D + j] = cc[(size_t)j * ct + t];
    }
  }
  free(cc); free(syms);
  if (n_slices_out) *n_slices_out = ns;
  return st;
}

/* ---------------------------------------------------------------------------
 * PCA basis for the benchmark's and the tests' inputs ([GAUGE] "Compression
 * Conditions": PCA/KLT is the uncentered second-moment eigenbasis at the same
 * layer, K/V and head granularity; [KVTC] "How the Pipeline Works": PCA after
 * RoPE undo, fitted on calibration data).
 *   C = (1/n) sum_t x_t x_t^T in fp64 (keys after the fp32 inverse rotation at
 *   positions 0..n-1); eigenvectors by the cyclic Jacobi method (textbook,
 *   e.g. Golub & Van Loan, "Matrix Computations", symmetric Schur
 *   decomposition); eigenvalues descending (ties: lower original index); each
 *   column's largest-magnitude entry made positive; rounded to fp32.
 * ------------------------------------------------------------------------- */
int kvco_jacobi_eigen(const double* A, uint32_t n, double* V, double* w) {
  double* a = (double*)malloc(sizeof(double) * n * n);
  memcpy(a, A, sizeof(double) * n * n);
  for (uint32_t i = 0; i < n; i++)
    for (uint32_t j = 0; j < n; j++) V[(size_t)i * n + j] = (i == j) ? 1.0 : 0.0;
  double total = 0.0;
  for (size_t i = 0; i < (size_t)n * n; i++) total += a[i] * a[i];
  for (int sweep = 0; sweep < 100; sweep++) {
    double off = 0.0;
    for (uint32_t p = 0; p < n; p++)
      for (uint32_t q = p + 1; q < n; q++) off += a[(size_t)p * n + q] * a[(size_t)p * n + q];
    if (off <= 1e-30 * total) break;
    for (uint32_t p = 0; p < n; p++) {
      for (uint32_t q = p + 1; q < n; q++) {
        double apq = a[(size_t)p * n + q];
        if (apq == 0.0) continue;
        double tau = (a[(size_t)q * n + q] - a[(size_t)p * n + p]) / (2.0 * apq);
        double t = (tau >= 0.0 ? 1.0 : -1.0) / (fabs(tau) + sqrt(tau * tau + 1.0));
        double c = 1.0 / sqrt(t * t + 1.0), s = t * c;
        for (uint32_t k = 0; k < n; k++) {
          double akp = a[(size_t)k * n + p], akq = a[(size_t)k * n + q];
          a[(size_t)k * n + p] = c * akp - s * akq;
          a[(size_t)k * n + q] = s * akp + c * akq;
        }
        for (uint32_t k = 0; k < n; k++) {
          double apk = a[(size_t)p * n + k], aqk = a[(size_t)q * n + k];
          a[(size_t)p * n + k] = c * apk - s * aqk;
          a[(size_t)q * n + k] = s * apk + c * aqk;
        }
        for (uint32_t k = 0; k < n; k++) {
          double vkp = V[(size_t)k * n + p], vkq = V[(size_t)k * n + q];
          V[(size_t)k * n + p] = c * vkp - s * vkq;
          V[(size_t)k * n + q] = s * vkp + c * vkq;
        }
      }
    }
  }
  for (uint32_t i = 0; i < n; i++) w[i] = a[(size_t)i * n + i];
  free(a);
  return KVCO_OK;
}

/* Uncentered second moments C = (1/n) sum_t x_t x_t^T of the calibration
 * tokens (keys de-rotated), accumulated in fp64 over t ascending. */
static double* second_moments(const uint16_t* calib, uint32_t n_tok, uint32_t D, int is_key, double theta) {
  uint32_t half = D / 2;
  float* cs = (float*)malloc(sizeof(float) * (size_t)n_tok * half * 2);
  kvco_rope_table(n_tok, D, theta, cs);
  double* C = (double*)calloc((size_t)D * D, sizeof(double));
  float* x = (float*)malloc(sizeof(float) * D);
  for (uint32_t t = 0; t < n_tok; t++) {
    for (uint32_t k = 0; k < D; k++) x[k] = kvco_bf16_to_f32(calib[(size_t)t * D + k]);
    if (is_key) kvco_rope_inverse(cs + (size_t)t * half * 2, D, x);
    for (uint32_t a = 0; a < D; a++)
      for (uint32_t b = 0; b < D; b++) C[(size_t)a * D + b] += (double)x[a] * (double)x[b];
  }
  for (size_t i = 0; i < (size_t)D * D; i++) C[i] /= (double)n_tok;
  free(cs);
  free(x);
  return C;
}

int kvco_pca(const uint16_t* calib, uint32_t n_tok, uint32_t D, uint32_t dtype, int is_key,
             double theta, float* Q, double* lambda) {
  if (dtype != KVCO_BF16 || n_tok == 0 || D == 0 || (D & 1u)) return KVCO_INVALID;
  double* C = second_moments(calib, n_tok, D, is_key, theta);
  double* V = (double*)malloc(sizeof(double) * D * D);
  double* w = (double*)malloc(sizeof(double) * D);
  kvco_jacobi_eigen(C, D, V, w);
  uint32_t* order = (uint32_t*)malloc(sizeof(uint32_t) * D);
  int* used = (int*)calloc(D, sizeof(int));
  for (uint32_t j = 0; j < D; j++) {
    int best = -1;
    for (uint32_t i = 0; i < D; i++) {
      if (used[i]) continue;
      if (best < 0 || w[i] > w[best]) best = (int)i;
    }
    used[best] = 1;
    order[j] = (uint32_t)best;
  }
  for (uint32_t j = 0; j < D; j++) {
    uint32_t c = order[j];
    uint32_t arg = 0;
    for (uint32_t k = 1; k < D; k++)
      if (fabs(V[(size_t)k * D + c]) > fabs(V[(size_t)arg * D + c])) arg = k;
    double sign = V[(size_t)arg * D + c] < 0.0 ? -1.0 : 1.0;
    for (uint32_t k = 0; k < D; k++) Q[(size_t)k * D + j] = (float)(sign * V[(size_t)k * D + c]);
    lambda[j] = w[c];
  }
  free(C); free(V); free(w); free(order); free(used);
  return KVCO_OK;
}

/* ---------------------------------------------------------------------------
 * Calibration-free bases ([Codec-Gauge] "Compression Conditions": a coordinate
 * control run with Hadamard and DCT coordinates beside PCA/KLT; "Coordinate
 * Controls"). Reading: the orthonormal forms with columns as components, the
 * Hadamard matrix in Sylvester (natural) order, H[k][j] = (-1)^popcount(k & j)
 * / sqrt(D) for D a power of two, and the DCT-II, Q[k][j] = c_j cos(pi (2k + 1)
 * j / (2D)) with c_0 = sqrt(1/D), c_j = sqrt(2/D); both in fp64, rounded to
 * fp32. The bit allocation ranks components by variance; in a fixed basis that
 * is the calibration second moment of each coordinate, q_j^T C q_j.
 * ------------------------------------------------------------------------- */
int kvco_fixed_basis(uint32_t kind, uint32_t D, float* Q) {
  if (D == 0) return KVCO_INVALID;
  if (kind == KVCO_BASIS_HADAMARD) {
    if (D & (D - 1u)) return KVCO_INVALID;
    double inv = 1.0 / sqrt((double)D);
    for (uint32_t k = 0; k < D; k++)
      for (uint32_t j = 0; j < D; j++) {
        uint32_t v = k & j, odd = 0;
        while (v) {  /* parity of the common bits */
          odd ^= 1u;
          v &= v - 1u;
        }
        Q[(size_t)k * D + j] = (float)(odd ? -inv : inv);
      }
    return KVCO_OK;
  }
  if (kind == KVCO_BASIS_DCT) {
    for (uint32_t j = 0; j < D; j++) {
      double c = j == 0 ? sqrt(1.0 / (double)D) : sqrt(2.0 / (double)D);
      for (uint32_t k = 0; k < D; k++) {
        double ang = 3.141592653589793 * (double)((2u * k + 1u) * j) / (double)(2u * D);
        Q[(size_t)k * D + j] = (float)(c * cos(ang));
      }
    }
    return KVCO_OK;
  }
  return KVCO_INVALID;
}

/* lambda_j = sum_a Q[a][j] (sum_b C[a][b] Q[b][j]), a and b ascending, in fp64. */
int kvco_basis_variances(const uint16_t* calib, uint32_t n_tok, uint32_t D, uint32_t dtype, int is_key,
                         double theta, const float* Q, double* lambda) {
  if (dtype != KVCO_BF16 || n_tok == 0 || D == 0 || (D & 1u)) return KVCO_INVALID;
  double* C = second_moments(calib, n_tok, D, is_key, theta);
  for (uint32_t j = 0; j < D; j++) {
    double lam = 0.0;
    for (uint32_t a = 0; a < D; a++) {
      double s = 0.0;
      for (uint32_t b = 0; b < D; b++) s += C[(size_t)a * D + b] * (double)Q[(size_t)b * D + j];
      lam += (double)Q[(size_t)a * D + j] * s;
    }
    lambda[j] = lam;
  }
  free(C);
  return KVCO_OK;
}
