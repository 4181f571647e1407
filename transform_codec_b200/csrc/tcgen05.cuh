// Blackwell (sm_100a) tensor-core building blocks as inline PTX: tensor-memory
// allocation, shared-memory matrix descriptors for K-major operands with the
// 128-byte swizzle, instruction descriptors, single-thread MMA issue with
// mbarrier completion, and tensor-memory loads. GPU-library only.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

namespace kvc {
namespace tc {

__device__ inline uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---- tensor memory (one warp calls alloc / dealloc)
__device__ inline void tmem_alloc(uint32_t* slot, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(slot)),
               "r"(ncols)
               : "memory");
}
__device__ inline void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ inline void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ---- ordering between ordinary threads, the async proxy and tensor ops
__device__ inline void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ inline void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ inline void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// ---- mbarrier
__device__ inline void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
// Wait for the phase with the given parity; gives up after max_iter polls and
// returns false (the caller records an error instead of spinning forever).
__device__ inline bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t max_iter) {
  const uint32_t a = smem_addr(bar);
  for (uint32_t i = 0; i < max_iter; ++i) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done)
        : "r"(a), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
}

// ---- descriptors
// Shared-memory matrix descriptor, K-major operand in 128-byte-swizzled atoms of
// 8 rows x 128 bytes (1024-byte aligned atoms, consecutive 8-row groups 1024
// bytes apart): start address >> 4 in bits 0-13, leading byte offset (unused
// for this layout, 16 bytes) in 16-29, stride byte offset 1024 >> 4 in 32-45,
// descriptor version 1 in 46-47, swizzle mode 2 (128-byte) in 61-63.
__device__ inline uint64_t desc_sw128(uint32_t saddr) {
  return uint64_t((saddr >> 4) & 0x3fffu) | (uint64_t(1) << 16) | (uint64_t(1024 >> 4) << 32) |
         (uint64_t(1) << 46) | (uint64_t(2) << 61);
}

// Instruction descriptor: D format in bits 4-5, A and B formats in 7-9 and
// 10-12, K-major A and B (bits 15, 16 clear), N >> 3 in 17-22, M >> 4 in 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(uint32_t M, uint32_t N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((N >> 3) << 17) | ((M >> 4) << 24);
}

// 8-bit integer operands (each signed or unsigned), 32-bit integer accumulator
__host__ __device__ constexpr uint32_t idesc_i8_s32(uint32_t M, uint32_t N, bool a_signed, bool b_signed) {
  return (2u << 4) | ((a_signed ? 1u : 0u) << 7) | ((b_signed ? 1u : 0u) << 10) | ((N >> 3) << 17) |
         ((M >> 4) << 24);
}

// ---- MMA (one thread issues), D[M][N] (+)= A[M][K] * B[N][K]^T
__device__ inline void mma_bf16(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// integer bytes: K = 32 per instruction, exact s32 sums
__device__ inline void mma_i8(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n\t}"
      ::"r"(d_tmem), "l"(a), "l"(b), "r"(idesc), "r"(acc)
      : "memory");
}
// arrive on bar once every MMA issued so far by this thread has completed
__device__ inline void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   smem_addr(bar))
               : "memory");
}

// ---- tensor memory -> registers: warp w reads lanes 32 (w % 4) .. + 31, one
// row per thread, 16 consecutive 32-bit columns starting at taddr's column
__device__ inline void tmem_ld16(uint32_t taddr, uint32_t* r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ inline void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Byte offset of element (row, kbyte) of a K-major operand tile of `rows` rows
// stored as 128-byte-swizzled atoms; K is split into 128-byte blocks placed
// rows * 128 bytes apart.
__host__ __device__ inline uint32_t sw128_offset(uint32_t row, uint32_t kbyte, uint32_t rows) {
  const uint32_t kb = kbyte >> 7, in = kbyte & 127u;
  const uint32_t chunk = (in >> 4) ^ (row & 7u);
  return kb * rows * 128u + row * 128u + (chunk << 4) + (in & 15u);
}

}  // namespace tc
}  // namespace kvc
