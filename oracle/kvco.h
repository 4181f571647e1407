/*
 * kvco — the CPU oracle for the KV codec.
 *
 * TEST INFRASTRUCTURE ONLY. This is a plain, slow, single-threaded C
 * restatement of what the codec computes, used to check the GPU library. Only
 * the tests, the smoke check and the benchmark's CPU-baseline leg may load it.
 * It shares no code, header, table or constant generator with the GPU library.
 *
 * Sources (web pages; cited by title and section):
 *   [QATQ]   "QATQ — lossless LLM memory compression" (qatq.org): "qatq encode",
 *            "QATC v2 checksum validated", "How it works".
 *   [AT1]    "AT-1 Memory" (tinyfiles.io/memory): "KV & tensor mode",
 *            "What's proven" (never-worse, tamper refusal).
 *   [GAUGE]  "Codec-Gauge: Learning Compression-Friendly Gauges for Transformer
 *            KV Caches": "Problem Statement and Overview", "Gauge
 *            Parameterization and Training", "Compression Conditions",
 *            "Evaluation Design".
 *   [KVTC]   "KVTC: The Open-Source KV Cache Codec That Treats LLM Memory Like
 *            Media": "How the Pipeline Works", "Why RoPE Has to Be Reversed
 *            First", "Bit Budget Is Not Fair", "rANS Makes the Last Mile Smaller".
 *
 * Parity status: every function here is pinned by tests against closed forms,
 * invariants, library routines or brute force. The frequency normalisation
 * rule, a definition of this codec, is pinned to hand-worked tables, to the
 * defining property of largest-remainder apportionment and to a restatement of
 * Hamilton's method in exact rationals; the cyclic Jacobi PCA to closed forms
 * and to numpy's symmetric eigensolver.
 */
#ifndef KVCO_H
#define KVCO_H
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

enum { KVCO_BF16 = 1, KVCO_FP16 = 2, KVCO_F32 = 3 };
enum { KVCO_LOSSLESS = 0, KVCO_TRANSFORM = 1 };
enum {
  KVCO_OK = 0, KVCO_INVALID = 1, KVCO_CAPACITY = 2, KVCO_CORRUPT = 3,
  KVCO_TRUNCATED = 4, KVCO_PLAN_MISMATCH = 5
};

typedef struct {
  uint32_t dtype;            /* KVCO_BF16, KVCO_FP16 or (lossless only) KVCO_F32 */
  uint32_t n_layers, n_heads, n_tokens, head_dim;
  uint32_t values_per_chunk; /* lossless chunk bound, 65536 */
  /* transform coding only */
  uint32_t n_sink, n_recent, block_tokens, chunk_tokens, max_bits;
  double rope_theta;
  const float* bases;        /* [L*2*H][D][D], Q[k*D + j], column j = component j */
  const uint8_t* widths;     /* [L*2*H][D] bits per component */
  /* optional: kvco_plan_crc(d) computed once by the caller (plan_crc_set = 1),
   * so that each transform call does not recompute it over all the bases;
   * 0 and 0 make every call compute it */
  uint32_t plan_crc, plan_crc_set;
  /* transform value ranges: KVCO_RANGES_BLOCK (per component and block of
   * tokens, keys and values) or KVCO_RANGES_KIVI (keys as BLOCK; values one
   * range per token over its coded components) */
  uint32_t ranges;
} kvco_desc;
enum { KVCO_RANGES_BLOCK = 0, KVCO_RANGES_KIVI = 1 };

uint32_t kvco_crc32(const void* p, size_t n);

int kvco_normalize(const uint32_t count[256], uint16_t freq[256]);

size_t kvco_stream_bound(uint32_t n);
size_t kvco_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out);
int kvco_stream_decode(const uint8_t* rec, size_t avail, uint32_t n, uint8_t* sym, size_t* used);
/* Lane-delta candidate (used for every byte plane of lossless chunks): coded
 * when the lane deltas' counts are more concentrated than the plane's (sum of
 * squared counts strictly larger) and their collision entropy is below
 * log2(181) bits (181 sum c^2 > n^2), then taken only if its RANS record is
 * strictly smaller than both the plain RANS record and RAW; the plain choice
 * otherwise. kvco_lane_delta / _undelta apply and undo the transform (XOR with
 * the previous symbol of the same rANS lane). */
size_t kvco_stream_encode_delta(const uint8_t* sym, uint32_t n, uint8_t* out);
void kvco_lane_delta(const uint8_t* sym, uint32_t n, uint8_t* out);
void kvco_lane_undelta(uint8_t* sym, uint32_t n);
size_t kvco_rans_payload_bytes(const uint8_t* sym, uint32_t n);
/* Side streams of a middle record (the byte planes of its zero points and
 * scales): the lane-delta choice on N = min(32, max(1, floor(n / 64))) lanes. */
size_t kvco_side_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out);
int kvco_side_stream_decode(const uint8_t* rec, size_t avail, uint32_t n, uint8_t* sym, size_t* used);

size_t kvco_lossless_bound(const kvco_desc* d, uint32_t n_slices);
/* src / dst: [n_slices][T][D] little-endian values of 2 bytes (bf16, fp16)
 * or 4 bytes (f32); cap in bytes. */
size_t kvco_encode_lossless(const kvco_desc* d, uint32_t first_slice, uint32_t n_slices,
                            const void* src, uint8_t* dst, size_t cap);
int kvco_decode_lossless(const kvco_desc* d, const uint8_t* src, size_t n, void* dst,
                         size_t cap, uint64_t* written);

void kvco_rope_table(uint32_t T, uint32_t D, double theta, float* cs);
void kvco_rope_inverse(const float* cs_row, uint32_t D, float* x);
void kvco_rope_forward(const float* cs_row, uint32_t D, float* x);

void kvco_project(const float* Q, uint32_t D, const float* x, float* y);
void kvco_unproject(const float* Q, uint32_t D, const float* y, float* x);

int kvco_allocate(const double* lambda, uint64_t n_units, double avg_bits, uint32_t max_bits,
                  uint8_t* widths);
uint32_t kvco_plan_crc(const kvco_desc* d);

size_t kvco_transform_bound(const kvco_desc* d, uint32_t n_slices);
size_t kvco_encode_transform(const kvco_desc* d, uint32_t first_slice, uint32_t n_slices,
                             const uint16_t* src, uint8_t* dst, size_t cap);
int kvco_decode_transform(const kvco_desc* d, const uint8_t* src, size_t n, uint16_t* dst,
                          size_t cap, uint64_t* written);
int kvco_transform_slice_codes(const kvco_desc* d, uint32_t slice, const uint16_t* src_slice,
                               uint8_t* codes, float* qpre, float* zs);
int kvco_record_codes(const kvco_desc* d, uint32_t sidx, const uint8_t* rec, uint32_t len,
                      uint32_t tcc, uint8_t* codes, float* zs);
int kvco_container_codes(const kvco_desc* d, const uint8_t* src, size_t n, uint32_t rec,
                         uint8_t* codes, float* zs, uint32_t* n_tokens);

int kvco_pca(const uint16_t* calib, uint32_t n_tok, uint32_t D, uint32_t dtype, int is_key,
             double theta, float* Q, double* lambda);
int kvco_jacobi_eigen(const double* A, uint32_t n, double* V, double* w);

/* Calibration-free bases and the component second moments in a given basis. */
enum { KVCO_BASIS_HADAMARD = 1, KVCO_BASIS_DCT = 2 };
int kvco_fixed_basis(uint32_t kind, uint32_t D, float* Q);
int kvco_basis_variances(const uint16_t* calib, uint32_t n_tok, uint32_t D, uint32_t dtype, int is_key,
                         double theta, const float* Q, double* lambda);

float kvco_bf16_to_f32(uint16_t h);
uint16_t kvco_f32_to_bf16(float f);

#ifdef __cplusplus
}
#endif
#endif
