/*
 * kvc.h — C ABI of the B200 KV-cache codec library (libkvc.so).
 *
 * The codec compresses an exported LLM KV cache laid out [L][2][H][T][D]
 * (layer, K = 0 / V = 1, KV head, token, channel; one [T][D] block is a
 * "slice", slice index (l * 2 + kv) * H + h), as in the Codec-Gauge page,
 * "Problem Statement and Overview" (K_l, V_l in R^{B x H_l x T x d_l}, B = 1).
 *
 * Two front-ends feed one entropy back-end and one container:
 *   lossless   — channel-major reorder of each chunk of floor(values_per_chunk
 *                / D) tokens, byte-plane split, and per plane the smallest of a
 *                constant, an rANS-coded or a raw record (AT-1 Memory page,
 *                "KV & tensor mode"; QATQ page, "qatq encode" and "How it works").
 *   transform  — sink and recent tokens kept raw, the middle RoPE-undone on
 *                keys, projected on a given per-(layer, K/V, head) orthonormal
 *                basis, and quantised per component at an allocated bit width
 *                with a scale and zero point per 64-token block (KVTC page, "How
 *                the Pipeline Works", "Why RoPE Has to Be Reversed First", "Bit
 *                Budget Is Not Fair"; Codec-Gauge page, "Compression Conditions").
 *                The fp32 zero points and scales of a record are themselves
 *                entropy coded: four byte-plane streams of all z, then all s.
 *   back-end   — chunked, 128-lane interleaved rANS with per-stream frequency
 *                tables (KVTC page, "rANS Makes the Last Mile Smaller").
 *   container  — 64-byte header, chunk-offset index with a CRC-32 per record,
 *                and a header CRC-32 over header and index; corrupt or truncated
 *                input is refused (QATQ page, "QATC v2 checksum validated").
 *
 * Conventions
 *   - Device pointers (d_*) are CUDA device memory owned by the caller, 16-byte
 *     aligned; host pointers (h_*) are ordinary host memory owned by the caller.
 *     The plan owns its own device copies of bases, widths and tables.
 *   - Calls that take a cudaStream_t are asynchronous on that stream; they
 *     launch kernels only (no allocation, no host synchronisation).
 *   - Two error channels: the return value reports what the host can see
 *     (bad arguments, too small buffers, launch failures); data-dependent
 *     results (bytes written, corrupt/truncated input, plan mismatch) are
 *     written by the device into *d_res once the stream reaches that point.
 *   - On a decode error the output contents are unspecified; read d_res first.
 *   - A plan is bound to the CUDA device that was current when it was made.
 */
#ifndef KVC_H
#define KVC_H

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define KVC_ABI_VERSION 2u

/* status codes (return values and kvc_result.status) */
enum {
  KVC_OK = 0,
  KVC_ERR_INVALID = 1,       /* bad argument or plan description */
  KVC_ERR_CAPACITY = 2,      /* destination or workspace too small */
  KVC_ERR_CORRUPT = 3,       /* checksum, structure or rANS end-state failure */
  KVC_ERR_TRUNCATED = 4,     /* container shorter than its header says */
  KVC_ERR_PLAN_MISMATCH = 5, /* container made with another shape or plan */
  KVC_ERR_TIMEOUT = 6,       /* a bounded device wait gave up */
  KVC_ERR_CUDA = 7,          /* CUDA runtime error on the host side */
  KVC_ERR_UNSUPPORTED = 8    /* valid request this build does not handle */
};

/* Value types: 16-bit bf16 / fp16 (two byte planes) and, lossless only, f32
 * (four byte planes; QATQ "qatq encode" and AT-1 "KV & tensor mode" code f32
 * tensors too). */
enum { KVC_DTYPE_BF16 = 1, KVC_DTYPE_FP16 = 2, KVC_DTYPE_F32 = 3 };
enum { KVC_PATH_LOSSLESS = 0, KVC_PATH_TRANSFORM = 1 };

/* Written by the device at the end of an encode or decode: status, and the
 * container bytes (encode) or decoded bytes (decode); 16 bytes. */
typedef struct {
  int32_t status;
  uint32_t reserved;
  uint64_t bytes;
} kvc_result;

typedef struct kvc_plan_s kvc_plan_t;

/* Plan description (host memory; copied by kvc_plan).
 *   abi_version       KVC_ABI_VERSION
 *   dtype             KVC_DTYPE_BF16, KVC_DTYPE_FP16 or KVC_DTYPE_F32 (f32:
 *                     lossless only; transform: bf16 only)
 *   n_layers, n_heads, n_tokens, head_dim   cache shape L, H, T, D
 *   values_per_chunk  lossless chunk bound (65536): chunks hold
 *                     floor(values_per_chunk / D) tokens, at most 65536 values
 *   n_sink, n_recent  transform: leading / trailing tokens kept raw
 *   block_tokens      transform: tokens per scale/zero-point block (64)
 *   chunk_tokens      transform: middle tokens per record (multiple of
 *                     block_tokens, at most 512)
 *   max_bits          transform: bit-width cap per component (<= 8)
 *   rope_theta        transform: rotary base; pairs (i, i + D/2), angle
 *                     t * theta^(-2i/D)
 *   avg_bits          transform: average code bits per middle value; the budget
 *                     floor(avg_bits * U + 0.5) over U = L*2*H*D components is
 *                     spent greedily, one bit at a time, on the component with
 *                     the largest eigenvalue * 4^-bits (ties: lowest index)
 *   bases             transform: host [L*2*H][D][D] fp32, element [k*D + j] is
 *                     channel k of component j; columns orthonormal
 *   eigvals           transform: host [L*2*H][D] component variances (used when
 *                     widths is NULL; negative values count as 0)
 *   widths            transform: optional host [L*2*H][D] bit widths that
 *                     replace the greedy allocation
 *   range_mode        transform: KVC_RANGES_BLOCK (0: a zero point and scale per
 *                     component and block of block_tokens tokens, keys and
 *                     values) or KVC_RANGES_KIVI (Codec-Gauge page, "Compression
 *                     Conditions": per-channel key ranges, per-token value
 *                     ranges: keys as BLOCK; each value token one zero point z
 *                     and range r over its coded components, a component of
 *                     width b quantised in steps r / (2^b - 1); needs D >=
 *                     block_tokens). Part of the plan CRC when not BLOCK.
 * For a lossless-only plan set bases, eigvals and widths to NULL. */
typedef struct {
  uint32_t abi_version;
  uint32_t dtype;
  uint32_t n_layers, n_heads, n_tokens, head_dim;
  uint32_t values_per_chunk;
  uint32_t n_sink, n_recent, block_tokens, chunk_tokens, max_bits;
  double rope_theta;
  double avg_bits;
  const float* bases;
  const double* eigvals;
  const uint8_t* widths;
  uint32_t range_mode;
  uint32_t reserved;
} kvc_plan_desc;
enum { KVC_RANGES_BLOCK = 0, KVC_RANGES_KIVI = 1 };

/* kvc_plan — the plan of a cache shape (KVTC page, "How the Pipeline Works":
 * the per-component bit widths, scales and zero points that reconstruction
 * needs; "Bit Budget Is Not Fair": widths spent unevenly; "Why RoPE Has to Be
 * Reversed First": the rotation undone before the basis).
 * Validates the description, allocates bit widths, builds the fp32 cos/sin
 * table (fp64-computed) and uploads the plan to the current device. Checks
 * each basis for orthonormality (max |Q^T Q - I| <= 1e-3).
 *   desc  host plan description (read only; copied)
 *   out   host out: the new library-owned plan, released by kvc_plan_destroy
 * Returns KVC_OK and *out, or KVC_ERR_INVALID (bad description), KVC_ERR_CUDA
 * (device allocation or copy failed) with *out = NULL and nothing allocated.
 * Blocking; call outside stream capture. kvc_plan_create is the same call
 * under its earlier name. */
int kvc_plan(const kvc_plan_desc* desc, kvc_plan_t** out);
int kvc_plan_create(const kvc_plan_desc* desc, kvc_plan_t** out);
/* Free the plan (device memory included). NULL is ignored. */
void kvc_plan_destroy(kvc_plan_t* plan);
/* Copy the plan's bit widths ([L*2*H][D]) to h_out (n bytes). */
int kvc_plan_widths(const kvc_plan_t* plan, uint8_t* h_out, size_t n);
/* CRC-32 identifying the transform plan; 0 for a lossless-only plan. */
uint32_t kvc_plan_crc(const kvc_plan_t* plan);

/* Upper bound of the container size for n_slices slices of the given path
 * (exact for incompressible input: the codec never exceeds it). 0 on error. */
size_t kvc_max_encoded_bytes(const kvc_plan_t* plan, int path, uint32_t n_slices);
/* Device workspace an encode of n_slices slices needs; for a decode, n_slices
 * is the most slices a container will hold (0: any container of the plan), and
 * a container with more slices than the workspace allows reports
 * KVC_ERR_CAPACITY in its result. */
size_t kvc_workspace_bytes(const kvc_plan_t* plan, int path, int decode, uint32_t n_slices);

/* kvc_encode_lossless — lossless coding of slices [first_slice, first_slice +
 * n_slices) of the cache (AT-1 Memory page, "KV & tensor mode": token-major
 * values reordered channel-major, split into byte planes, the smaller of coded
 * and plain kept; QATQ page, "qatq encode": chunks of at most 65536 values).
 *   d_src     device [n_slices][T][D] values (the selected slices only;
 *             16-bit, or 32-bit for an f32 plan), read only
 *   d_dst     device output, dst_cap bytes (>= kvc_max_encoded_bytes)
 *   d_ws      device workspace, ws_bytes (>= kvc_workspace_bytes(..., 0, n_slices))
 *   d_res     device kvc_result: status and container bytes
 * Returns KVC_OK when launched; KVC_ERR_INVALID / KVC_ERR_CAPACITY / KVC_ERR_CUDA
 * otherwise (then nothing was launched or the stream is in error). */
int kvc_encode_lossless(const kvc_plan_t* plan, uint32_t first_slice, uint32_t n_slices,
                        const void* d_src, void* d_dst, size_t dst_cap, void* d_ws,
                        size_t ws_bytes, kvc_result* d_res, cudaStream_t stream);

/* kvc_decode_lossless — restore the exact value bytes of a lossless container
 * (QATQ page, "QATC v2 checksum validated": corrupt or truncated payloads are
 * refused; AT-1 Memory page, "What's proven": byte-exact round trip, tamper
 * refusal).
 *   d_src/src_bytes  device container and its exact length in bytes
 *   d_dst/dst_cap    device output [n_slices][T][D] 16-bit values
 *   d_ws/ws_bytes    device workspace (>= kvc_workspace_bytes(..., 1, 0))
 *   d_res            device kvc_result: status (OK, CORRUPT, TRUNCATED,
 *                    PLAN_MISMATCH, CAPACITY) and decoded bytes
 * The header, the index and every record's CRC-32 are checked; a record that
 * fails leaves its output unspecified and sets the status of the lowest
 * failing record. */
int kvc_decode_lossless(const kvc_plan_t* plan, const void* d_src, size_t src_bytes, void* d_dst,
                        size_t dst_cap, void* d_ws, size_t ws_bytes, kvc_result* d_res,
                        cudaStream_t stream);

/* kvc_encode_transform — transform coding of slices [first_slice, first_slice
 * + n_slices) (KVTC page, "How the Pipeline Works": sinks and recent window
 * kept, RoPE undone, PCA projection, bit allocation, quantisation, entropy
 * coding; Codec-Gauge page, "Problem Statement and Overview": Z = G X with an
 * orthogonal G). Arguments, ownership and error channels as
 * kvc_encode_lossless. Needs a plan with bases; D = 128, bf16, 64-token
 * blocks, at most 512-token records (else KVC_ERR_UNSUPPORTED). */
int kvc_encode_transform(const kvc_plan_t* plan, uint32_t first_slice, uint32_t n_slices,
                         const void* d_src, void* d_dst, size_t dst_cap, void* d_ws,
                         size_t ws_bytes, kvc_result* d_res, cudaStream_t stream);
/* kvc_decode_transform — reconstruct a transform container (KVTC page, "How
 * the Pipeline Works": dequantise with the stored scales and zero points, and
 * reverse the process; Codec-Gauge page, "Problem Statement and Overview":
 * X^ = G^-1 Z^ with G^-1 = G^T): codes dequantised, projected back, keys
 * rotated forward, rounded to bf16. Arguments, ownership and error channels
 * as kvc_decode_lossless; the raw sink and recent rows come back bit-exact. */
int kvc_decode_transform(const kvc_plan_t* plan, const void* d_src, size_t src_bytes, void* d_dst,
                         size_t dst_cap, void* d_ws, size_t ws_bytes, kvc_result* d_res,
                         cudaStream_t stream);

/* Batches. Each frame is an independent container (for example one 64 MiB
 * layer-K or layer-V tensor of a long cache); a batch codes many frames with
 * one launch per kernel for every 64 frames, which keeps all SMs busy when a
 * single frame has too few chunks to fill the GPU.
 *   encode: src = device [n_slices][T][D] values of slices
 *           [first_slice, first_slice + n_slices); dst/dst_cap = container
 *           buffer (>= kvc_max_encoded_bytes for n_slices)
 *   decode: src/src_bytes = device container; dst/dst_cap = output values;
 *           first_slice and n_slices are ignored
 *   res:    device kvc_result of this frame
 * Frames in one call must not share dst buffers. */
typedef struct {
  uint32_t first_slice;
  uint32_t n_slices;
  const void* src;
  size_t src_bytes;
  void* dst;
  size_t dst_cap;
  kvc_result* res;
} kvc_frame;

/* Device workspace for a batch call of n_frames frames of at most
 * max_slices_per_frame slices each. Decoding a container with more slices
 * than max_slices_per_frame reports KVC_ERR_CAPACITY in its result. */
size_t kvc_batch_workspace_bytes(const kvc_plan_t* plan, int path, int decode, uint32_t n_frames,
                                 uint32_t max_slices_per_frame);
/* Encode or decode n_frames frames (host array h_frames) on one stream. Return
 * values and per-frame results as for the single-container calls. */
int kvc_encode_batch(const kvc_plan_t* plan, int path, const kvc_frame* h_frames, uint32_t n_frames,
                     void* d_ws, size_t ws_bytes, cudaStream_t stream);
int kvc_decode_batch(const kvc_plan_t* plan, int path, const kvc_frame* h_frames, uint32_t n_frames,
                     uint32_t max_slices_per_frame, void* d_ws, size_t ws_bytes, cudaStream_t stream);

/* Host-streamed coding (QATQ page, "Measured evidence": raw blocks streamed
 * through the codec in a live migration). A range of slices in host memory
 * is coded frame by frame, each frame of frame_slices slices (the last may be
 * shorter) an independent container; the H2D copies, the codec and the D2H
 * copies of consecutive frames overlap on three streams (the caller's stream
 * runs the codec; two copy streams and the ring's events are made by the
 * first such call on a plan and kept until kvc_plan_destroy) through a ring
 * of device slots in d_buf. The calls are blocking: they return when every
 * copy has landed. Host-streamed calls on one plan must not run at the same
 * time from several host threads (they share the plan's copy streams).
 * h_src, h_dst and h_results should be pinned (cudaHostAlloc or registered)
 * memory, else the copies do not overlap.
 *   kvc_stream_buffer_bytes: size of d_buf (device, 256-byte aligned) for
 *     frames of frame_slices slices.
 *   kvc_stream_encode_host: slices [first_slice, first_slice + n_slices) of
 *     h_src ([n_slices][T][D] values) into h_dst, containers back to back in
 *     frame order; h_frame_bytes[i] gets frame i's container size and
 *     h_results[i] its device result (n_frames = ceil(n_slices / frame_slices)
 *     entries each). KVC_ERR_CAPACITY if the containers outgrow dst_cap: the
 *     frames whose sizes were written are in place, the later entries of
 *     h_frame_bytes are not written.
 *   kvc_stream_decode_host: the n_frames containers back to back in h_src
 *     (sizes h_frame_bytes), as written by kvc_stream_encode_host for
 *     n_slices slices in frames of frame_slices, into h_dst ([n_slices][T][D]
 *     values, dst_cap bytes); h_results[i] gets frame i's status (a corrupt
 *     frame leaves its part of h_dst unspecified and the others decoded).
 * Return values report host-visible errors, as for the other calls. */
size_t kvc_stream_buffer_bytes(const kvc_plan_t* plan, int path, uint32_t frame_slices);
int kvc_stream_encode_host(const kvc_plan_t* plan, int path, uint32_t first_slice, uint32_t n_slices,
                           uint32_t frame_slices, const void* h_src, void* h_dst, size_t dst_cap,
                           uint64_t* h_frame_bytes, kvc_result* h_results, void* d_buf, size_t buf_bytes,
                           cudaStream_t stream);
int kvc_stream_decode_host(const kvc_plan_t* plan, int path, uint32_t n_slices, uint32_t frame_slices,
                           const void* h_src, const uint64_t* h_frame_bytes, void* h_dst, size_t dst_cap,
                           kvc_result* h_results, void* d_buf, size_t buf_bytes, cudaStream_t stream);

/* Human-readable name of a status code (static string). */
const char* kvc_status_string(int status);

/* Calibration (host, multithreaded): the uncentered second-moment eigenbasis of
 * each slice (Codec-Gauge page, "Compression Conditions": PCA/KLT at layer,
 * K/V and head granularity; KVTC page, "The Tradeoff Is Real": calibration).
 *   h_calib   host [L*2*H][n_calib][D] bf16 calibration tokens at positions
 *             0..n_calib-1; keys are de-rotated first
 *   h_bases   host out [L*2*H][D][D] fp32, columns sorted by eigenvalue
 *             descending, each column's largest-magnitude entry positive
 *   h_eigvals host out [L*2*H][D]
 * Shape and rope_theta come from desc (bases/eigvals/widths ignored). */
int kvc_calibrate_pca(const kvc_plan_desc* desc, const uint16_t* h_calib, uint32_t n_calib,
                      float* h_bases, double* h_eigvals, int n_threads);

/* Calibration-free bases (Codec-Gauge page, "Compression Conditions" and
 * "Coordinate Controls": Hadamard and DCT coordinates beside PCA/KLT), fp64
 * values rounded to fp32, element [k*D + j] = channel k of component j:
 *   KVC_BASIS_HADAMARD  Sylvester order, (-1)^popcount(k & j) / sqrt(D);
 *                       D must be a power of two
 *   KVC_BASIS_DCT       orthonormal DCT-II, c_j cos(pi (2k + 1) j / (2D)),
 *                       c_0 = sqrt(1/D), c_j = sqrt(2/D)
 * kvc_fixed_basis writes one [D][D] basis to h_basis (host). Returns
 * KVC_ERR_INVALID for another kind, a NULL pointer or D = 0. */
enum { KVC_BASIS_PCA = 0, KVC_BASIS_HADAMARD = 1, KVC_BASIS_DCT = 2 };
int kvc_fixed_basis(int kind, uint32_t D, float* h_basis);
/* kvc_calibrate_pca for kind KVC_BASIS_PCA; otherwise the fixed basis of that
 * kind for every slice (h_bases [L*2*H][D][D]) and, as h_eigvals, each
 * component's second moment over the slice's calibration tokens (keys
 * de-rotated): q_j^T C q_j with C = (1/n_calib) sum_t x_t x_t^T, fp64, sums over
 * tokens and then channels in ascending order. Host, multithreaded over slices. */
int kvc_calibrate_basis(const kvc_plan_desc* desc, int kind, const uint16_t* h_calib, uint32_t n_calib,
                        float* h_bases, double* h_eigvals, int n_threads);

/* Greedy bit allocation on its own (host): the widths kvc_plan_create would
 * assign. h_eigvals [n_units] (negative values count as 0), h_widths out
 * [n_units]; the budget is floor(avg_bits * n_units + 0.5) bits, each unit at
 * most max_bits (KVTC page, "Bit Budget Is Not Fair"). */
int kvc_allocate_bits(const double* h_eigvals, uint64_t n_units, double avg_bits, uint32_t max_bits,
                      uint8_t* h_widths);

/* Kernel timing. Between kvc_profile_begin and kvc_profile_end every kernel the
 * library launches is bracketed by CUDA events on its own stream.
 * kvc_profile_end waits for those events, fills out[0 .. *n_kernels) with one
 * entry per kernel name (launch count, summed device time in ms) and stops
 * recording. Host-side bookkeeping only; not for use under stream capture. */
typedef struct {
  char name[40];
  uint32_t launches;
  double total_ms;
} kvc_kernel_time;
int kvc_profile_begin(void);
int kvc_profile_end(kvc_kernel_time* out, int max_kernels, int* n_kernels);

/* Stage entry points (check the CRC and rANS stages on their own).
 * kvc_stage_crc32: CRC-32 of n bytes at d_src into *d_out (one block).
 * kvc_stage_stream_encode: one stream record of n (<= 65536) byte symbols at
 *   d_sym into d_out (capacity 16 + n rounded up to 16), using d_scratch
 *   (2n bytes); d_res gets the record bytes.
 * kvc_stage_stream_decode: decode the record at d_rec (rec_bytes) holding n
 *   symbols into d_sym; d_res gets the status and record bytes. */
int kvc_stage_crc32(const void* d_src, size_t n, uint32_t* d_out, cudaStream_t stream);
int kvc_stage_stream_encode(const uint8_t* d_sym, uint32_t n, uint8_t* d_out, void* d_scratch,
                            kvc_result* d_res, cudaStream_t stream);
int kvc_stage_stream_decode(const uint8_t* d_rec, uint32_t rec_bytes, uint32_t n, uint8_t* d_sym,
                            kvc_result* d_res, cudaStream_t stream);

/* kvc_stage_stream_encode_noalloc: kvc_stage_stream_encode without a caller
 * scratch buffer and without allocating anything. It is for callers that must
 * not allocate device memory at the point of the call: a serving loop that has
 * handed all device memory to a preallocated pool, code running inside an
 * allocator's out-of-memory handler (where allocating again would recurse), or
 * a latency-critical path that must not wait on an allocation. The scratch is
 * a fixed 128 KiB array inside the library, one per device, so n is limited to
 * 65536 symbols; larger n returns KVC_ERR_CAPACITY. The output bytes and
 * d_res are those of kvc_stage_stream_encode for the same symbols.
 * Every call looks up the array's device address on the current device
 * (cudaGetSymbolAddress, host side). The first call on a device, and the first
 * after a cudaDeviceReset, also loads the library's device code there, which
 * is when the array is reserved: make that first call before starting any
 * stream capture. Calls that overlap on
 * the device (on different streams, or from different host threads without
 * ordering) share the one array and race: order them. The container format
 * has no counterpart of this call; it only changes where the scratch lives. */
int kvc_stage_stream_encode_noalloc(const uint8_t* d_sym, uint32_t n, uint8_t* d_out,
                                    kvc_result* d_res, cudaStream_t stream);

#ifdef __cplusplus
}
#endif
#endif /* KVC_H */
