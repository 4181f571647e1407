// Host/device interface between the C-ABI layer and the kernels of the KV codec
// library. GPU-library only.
#pragma once
#include <algorithm>
#include <atomic>
#include <mutex>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

namespace kvc {

constexpr uint32_t kHeaderBytes = 64;        // container header
constexpr uint32_t kIndexEntry = 16;         // u64 offset, u32 length, u32 CRC-32
constexpr uint32_t kMaxChunkValues = 65536;  // values per lossless chunk at most

// Kernel timing: while profiling is on, a ProfRange around a launch records
// CUDA events before and after it on the launch stream.
bool prof_enabled();
void prof_record(const char* name, cudaStream_t st, bool end);
// A kernel's dynamic shared-memory limit, raised only when a launch needs
// more than the device already allows it (track: one per kernel, the largest
// size set on each of the first 64 devices). cudaFuncSetAttribute on every
// launch made concurrent calls from other host threads serialise. The limit
// only grows, under one process-wide lock, so first launches of one kernel
// with different sizes on several threads cannot leave it below a recorded
// size.
constexpr int kSmemAttrDevices = 64;
struct SmemAttr {
  std::atomic<int> set[kSmemAttrDevices];
};
inline std::mutex& smem_attr_lock() {
  static std::mutex m;
  return m;
}
inline cudaError_t smem_attr(SmemAttr& track, const void* kern, size_t bytes) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) dev = -1;
  const int need = int(bytes);
  const bool tracked = dev >= 0 && dev < kSmemAttrDevices;
  if (tracked && track.set[dev].load(std::memory_order_acquire) >= need) return cudaSuccess;
  std::lock_guard<std::mutex> lock(smem_attr_lock());
  const int target = tracked ? std::max(need, track.set[dev].load(std::memory_order_relaxed)) : need;
  const cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, target);
  if (e == cudaSuccess && tracked) track.set[dev].store(target, std::memory_order_release);
  return e;
}

struct ProfRange {
  const char* name;
  cudaStream_t st;
  bool on;
  ProfRange(const char* n, cudaStream_t s) : name(n), st(s), on(prof_enabled()) {
    if (on) prof_record(name, st, false);
  }
  ~ProfRange() {
    if (on) prof_record(name, st, true);
  }
};

// A group of up to kBatchMax frames (independent containers) coded by one
// launch per kernel; passed to kernels by value.
constexpr uint32_t kBatchMax = 64;
struct FrameDesc {
  const uint8_t* src;   // encode: values; decode: container
  uint8_t* dst;         // encode: container; decode: values
  void* res;            // kvc_result
  uint64_t src_bytes, dst_cap;
  uint32_t first_slice, n_slices;
};
struct FrameBatch {
  uint32_t n;
  uint32_t rec_base[kBatchMax + 1];  // encode: first global record of each frame
  FrameDesc f[kBatchMax];
};

// Decoder workspace: one DecodeState per frame of the group, then the batch
// state and the list of records the fast decoders deferred.
struct DecodeState {
  int status;                  // container-level status (header, index, capacity)
  uint32_t first_slice, n_slices, n_records;
  unsigned long long err_key;  // min over failing records of (record << 8) | status
  uint64_t out_bytes;
};
constexpr uint32_t kDecodeStateBytes = 256;
struct BatchDecodeState {
  uint32_t n_deferred;
};
inline __host__ __device__ DecodeState* decode_state(uint8_t* ws, uint32_t f) {
  return reinterpret_cast<DecodeState*>(ws + uint64_t(f) * kDecodeStateBytes);
}
inline __host__ __device__ BatchDecodeState* batch_state(uint8_t* ws) {
  return reinterpret_cast<BatchDecodeState*>(ws + uint64_t(kBatchMax) * kDecodeStateBytes);
}
inline __host__ __device__ unsigned long long* deferred_list(uint8_t* ws) {
  return reinterpret_cast<unsigned long long*>(ws + uint64_t(kBatchMax + 1) * kDecodeStateBytes);
}
constexpr uint64_t kDecodeWsFixed = uint64_t(kBatchMax + 1) * kDecodeStateBytes;

// Encoder workspace (device): per frame an EncodeState, per global record its
// length, CRC and container offset, then one slot per record.
struct EncodeState {
  int status;
  uint32_t n_records;
  uint64_t total_bytes;
};
struct EncodeLayout {
  EncodeState* state;   // [frames]
  uint32_t* rec_len;    // [records]
  uint32_t* rec_crc;
  uint64_t* rec_off;
  uint8_t* slots;
  uint64_t slot_bytes;
};

// What a valid container header must carry for this plan.
struct ContainerExpect {
  uint32_t path, dtype, L, H, T, D, chunk_tokens;
  uint32_t E;                  // bytes per value of the decoded output
  uint32_t n_sink, n_recent, block_tokens, plan_crc;
  uint32_t recs_per_slice;     // records per slice
  uint32_t max_slices;         // slices a container may hold in this call
};

// header fields common to the frames of a batch
struct HeaderFields {
  uint32_t path, dtype, L, H, T, D, chunk_tokens, recs_per_slice;
  uint32_t plan_crc, n_sink, n_recent, block_tokens;
};

cudaError_t launch_finalize(const HeaderFields& h, const FrameBatch& b, const EncodeLayout& ws,
                            cudaStream_t st);
cudaError_t launch_check_container(const FrameBatch& b, const ContainerExpect& e, uint8_t* ws,
                                   cudaStream_t st);
cudaError_t launch_decode_finish(const FrameBatch& b, uint8_t* ws, cudaStream_t st);

#ifdef __CUDACC__
// frame of global record g: largest f with rec_base[f] <= g
__device__ inline uint32_t frame_of(const uint32_t* base, uint32_t n, uint32_t g) {
  uint32_t lo = 0, hi = n - 1;
  while (lo < hi) {
    const uint32_t mid = (lo + hi + 1) >> 1;
    if (base[mid] <= g) lo = mid; else hi = mid - 1;
  }
  return lo;
}
#endif

// lossless
struct LosslessShape {
  uint32_t T, D, tc, cps;      // tokens, head_dim, chunk tokens, chunks per slice
  uint32_t E;                  // bytes per value (byte planes per chunk): 2, or 4 for f32
};
uint64_t lossless_slot_bytes(const LosslessShape& s);
cudaError_t launch_lossless_encode(const LosslessShape& s, const FrameBatch& b,
                                   const EncodeLayout& ws, cudaStream_t st);
cudaError_t launch_lossless_decode(const LosslessShape& s, const FrameBatch& b, uint8_t* ws,
                                   uint32_t max_records, cudaStream_t st);

// transform coding
struct TransformShape {
  uint32_t L, H, T, D, ct, block, n_sink, n_recent;
  uint32_t s_end, r_start, n_mid;   // regions and middle chunks per slice
  uint32_t kivi;                    // values take per-token ranges (KVC_RANGES_KIVI)
};
// Per-slice component order of the transform path (head_dim 128), computed on
// the host when the plan is made: the coded components (width >= 1) grouped by
// width b = 1..8, ascending index within a width; coded_idx is the rank of a
// coded component among all coded components in index order.
struct alignas(16) CompInfo {
  uint32_t width[128];
  uint32_t comp[128];       // components ordered by (width, index), widths >= 1
  uint32_t coded_idx[128];  // rank among coded components (width >= 1)
  uint32_t bstart[10], bcount[10];
  uint32_t n_coded;
};
// Per slice, the coded columns of Q (coded components in index order, "cc")
// for the encoder's tensor-core projection: J[k][cc] = rint(Q[k][j] 2^r), r =
// 29 - f, f = ilogb(max_k |Q[k][j]|), so |J| <= 2^30; the four bytes of J (two's
// complement, byte 0 the top one) are the planes of qdig, each 128 rows (cc) x
// 128 K bytes in the B-operand layout, zero past the coded columns.
struct alignas(16) QColInfo {
  int32_t f[128];   // ilogb(max_k |Q[k][j]|); kQColZero for an all-zero column
  float q1[128];    // an upper bound of sum_k |Q[k][j]|
};
constexpr int32_t kQColZero = -100000;
constexpr uint32_t kQDigPlane = 128u * 128u;         // bytes of one digit plane
constexpr uint32_t kQDigBytes = 4u * kQDigPlane;     // per slice
struct TransformPlanDev {
  const float* bases;      // [S][D][D], Q[k*D + j]
  const uint8_t* widths;   // [S][D]
  const float* rope;       // [T][D/2][2] cos, sin
  const uint8_t* qsplit;   // [S][hi, lo][128 x 256 B] Q as bf16 pieces, B-operand layout
  const CompInfo* comp;    // [S]
  const uint8_t* qdig;     // [S][4 planes][128 x 128 B] Q's digits (QColInfo)
  const QColInfo* qcol;    // [S]
  const float* qt;         // [S][D][D] Q transposed: qt[j*D + k] = Q[k][j]
};
constexpr uint32_t kQSplitBytes = 2u * 128u * 256u;  // per slice
// A record length at or above kRecLenError marks a record its encoder could not
// produce; its low byte is the status the frame reports.
constexpr uint32_t kRecLenError = 0xffffff00u;
uint64_t transform_slot_bytes(const TransformShape& s);
cudaError_t launch_transform_encode(const TransformShape& s, const TransformPlanDev& p,
                                    const FrameBatch& b, const EncodeLayout& ws, cudaStream_t st);
// Transform decode workspace beyond the common part, for `records` records:
// a status word and a code block of ct rows of 128 bytes per record.
uint64_t transform_decode_ws_extra(const TransformShape& s, uint64_t records);
cudaError_t launch_transform_decode(const TransformShape& s, const TransformPlanDev& p,
                                    const FrameBatch& b, uint8_t* ws, uint32_t max_records,
                                    cudaStream_t st);

// stage entry points
cudaError_t launch_stage_crc32(const uint8_t* src, uint64_t n, uint32_t* out, cudaStream_t st);
cudaError_t launch_stage_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out,
                                       uint16_t* scratch, void* res, cudaStream_t st);
cudaError_t launch_stage_stream_decode(const uint8_t* rec, uint32_t rec_bytes, uint32_t n,
                                       uint8_t* sym, void* res, cudaStream_t st);

}  // namespace kvc
