// Host/device interface between the C-ABI layer and the kernels of the KV codec
// library. GPU-library only.
#pragma once
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

// Decoder workspace (device): header/index verdict and the first failing record.
struct DecodeState {
  int status;                  // container-level status (header, index, capacity)
  uint32_t first_slice, n_slices, n_records;
  unsigned long long err_key;  // min over failing records of (record << 8) | status
  uint64_t out_bytes;
  uint32_t n_deferred;         // records the fast decoder left to the general one
  uint32_t reserved;
};
// the deferred-record list follows the state in the decode workspace
constexpr uint32_t kDecodeStateBytes = 256;
inline __host__ __device__ uint32_t* deferred_list(DecodeState* ds) {
  return reinterpret_cast<uint32_t*>(reinterpret_cast<uint8_t*>(ds) + kDecodeStateBytes);
}

// Encoder workspace header (device), followed by per-record arrays and slots.
struct EncodeState {
  int status;
  uint32_t n_records;
  uint64_t total_bytes;
};

// What a valid container header must carry for this plan.
struct ContainerExpect {
  uint32_t path, dtype, L, H, T, D, chunk_tokens;
  uint32_t n_sink, n_recent, block_tokens, plan_crc;
  uint32_t recs_per_slice;     // records per slice
  uint64_t dst_cap;            // decode output capacity in bytes
};

struct EncodeLayout {          // workspace carve-up for an encode call
  EncodeState* state;
  uint32_t* rec_len;
  uint32_t* rec_crc;
  uint64_t* rec_off;
  uint8_t* slots;
  uint64_t slot_bytes;
};

// header writer / record copier shared by both paths
struct HeaderFields {
  uint32_t path, dtype, L, H, T, D, first_slice, n_slices, chunk_tokens, n_records;
  uint32_t plan_crc, n_sink, n_recent, block_tokens;
};

cudaError_t launch_finalize(const HeaderFields& h, const EncodeLayout& ws, uint8_t* dst,
                            uint64_t dst_cap, void* res, cudaStream_t st);
cudaError_t launch_check_container(const uint8_t* src, uint64_t src_bytes,
                                   const ContainerExpect& e, DecodeState* ds, void* res,
                                   cudaStream_t st);
cudaError_t launch_decode_finish(DecodeState* ds, void* res, cudaStream_t st);

// lossless
struct LosslessShape {
  uint32_t T, D, tc, cps;      // tokens, head_dim, chunk tokens, chunks per slice
};
uint64_t lossless_slot_bytes(const LosslessShape& s);
cudaError_t launch_lossless_encode(const LosslessShape& s, const uint16_t* src, uint32_t n_slices,
                                   const EncodeLayout& ws, cudaStream_t st);
cudaError_t launch_lossless_decode(const LosslessShape& s, const uint8_t* src, uint16_t* dst,
                                   DecodeState* ds, uint32_t max_records, cudaStream_t st);

// transform coding
struct TransformShape {
  uint32_t L, H, T, D, ct, block, n_sink, n_recent;
  uint32_t s_end, r_start, n_mid;   // regions and middle chunks per slice
};
struct TransformPlanDev {
  const float* bases;      // [S][D][D], Q[k*D + j]
  const uint8_t* widths;   // [S][D]
  const float* rope;       // [T][D/2][2] cos, sin
  const uint8_t* qsplit;   // [S][hi, lo][128 x 256 B] Q as bf16 pieces, B-operand layout
};
constexpr uint32_t kQSplitBytes = 2u * 128u * 256u;  // per slice
uint64_t transform_slot_bytes(const TransformShape& s);
cudaError_t launch_transform_encode(const TransformShape& s, const TransformPlanDev& p,
                                    const uint16_t* src, uint32_t first_slice, uint32_t n_slices,
                                    const EncodeLayout& ws, cudaStream_t st);
cudaError_t launch_transform_decode(const TransformShape& s, const TransformPlanDev& p,
                                    const uint8_t* src, uint16_t* dst, DecodeState* ds,
                                    uint32_t max_records, cudaStream_t st);

// stage entry points
cudaError_t launch_stage_crc32(const uint8_t* src, uint64_t n, uint32_t* out, cudaStream_t st);
cudaError_t launch_stage_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out,
                                       uint16_t* scratch, void* res, cudaStream_t st);
cudaError_t launch_stage_stream_decode(const uint8_t* rec, uint32_t rec_bytes, uint32_t n,
                                       uint8_t* sym, void* res, cudaStream_t st);

}  // namespace kvc
