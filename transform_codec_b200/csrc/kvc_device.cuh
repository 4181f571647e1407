// Device-side building blocks of the KV codec library (sm_100a).
//
// Container, stream-record and rANS parameters follow the codec's format
// rules (lossless front-end: AT-1 Memory page, "KV & tensor mode"; container:
// QATQ page, "How it works" and "QATC v2 checksum validated"; entropy stage:
// KVTC page, "rANS Makes the Last Mile Smaller"). This header is GPU-library
// only.
#pragma once
#include <cuda_runtime.h>
#include <stdint.h>

#include "kvc_internal.h"

namespace kvc {

// ---------------------------------------------------------------- format
constexpr uint32_t kProbScale = 4096;   // rANS frequency total (2^12)
constexpr uint32_t kProbBits = 12;
constexpr uint32_t kRansLow = 65536;    // rANS state lower bound (2^16), 16-bit words
constexpr uint32_t kMaxLanes = 128;
constexpr uint32_t kGroupLanes = 32;
constexpr uint32_t kModeRaw = 0, kModeConst = 1, kModeRans = 2;

// status codes (mirrors include/kvc.h)
constexpr int kOk = 0, kErrInvalid = 1, kErrCapacity = 2, kErrCorrupt = 3, kErrTruncated = 4,
              kErrPlanMismatch = 5, kErrTimeout = 6, kErrCuda = 7, kErrUnsupported = 8;

__host__ __device__ inline uint32_t pad16(uint32_t n) { return (n + 15u) & ~15u; }
__host__ __device__ inline uint64_t pad16_64(uint64_t n) { return (n + 15u) & ~uint64_t(15); }

// lanes of a stream of n symbols and the contiguous range lane l owns
__host__ __device__ inline uint32_t rans_lanes(uint32_t n) {
  uint32_t N = n / 512u;
  return N < 1u ? 1u : (N > kMaxLanes ? kMaxLanes : N);
}
__host__ __device__ inline void lane_range(uint32_t n, uint32_t N, uint32_t l, uint32_t& start,
                                           uint32_t& len) {
  uint32_t base = n / N, extra = n % N;
  len = base + (l < extra ? 1u : 0u);
  start = l * base + (l < extra ? l : extra);
}
// Whether stream index i starts a rANS lane (lanes of a stream of n symbols on N lanes).
__device__ inline bool lane_start(uint32_t i, uint32_t n, uint32_t N) {
  const uint32_t base = n / N, extra = n - base * N;
  const uint32_t big = extra * (base + 1u);
  return i < big ? (i % (base + 1u)) == 0u : ((i - big) % base) == 0u;
}

__host__ __device__ inline uint32_t rans_groups(uint32_t N) {
  return (N + kGroupLanes - 1) / kGroupLanes;
}

// little-endian unaligned accessors for byte pointers (global or shared)
__device__ inline uint32_t ld_u16(const uint8_t* p) { return uint32_t(p[0]) | (uint32_t(p[1]) << 8); }
__device__ inline uint32_t ld_u32(const uint8_t* p) {
  return uint32_t(p[0]) | (uint32_t(p[1]) << 8) | (uint32_t(p[2]) << 16) | (uint32_t(p[3]) << 24);
}
__device__ inline uint64_t ld_u64(const uint8_t* p) {
  return uint64_t(ld_u32(p)) | (uint64_t(ld_u32(p + 4)) << 32);
}
__device__ inline void st_u16(uint8_t* p, uint32_t v) {
  p[0] = uint8_t(v);
  p[1] = uint8_t(v >> 8);
}
__device__ inline void st_u32(uint8_t* p, uint32_t v) {
  p[0] = uint8_t(v); p[1] = uint8_t(v >> 8); p[2] = uint8_t(v >> 16); p[3] = uint8_t(v >> 24);
}
__device__ inline void st_u64(uint8_t* p, uint64_t v) {
  st_u32(p, uint32_t(v));
  st_u32(p + 4, uint32_t(v >> 32));
}

// ---------------------------------------------------------------- GF(2) / CRC-32
// Reflected CRC-32 (polynomial 0xEDB88320). A register value r stands for the
// polynomial sum_i bit_i(r) x^(31-i); one step r -> (r >> 1) ^ (r & 1 ? P : 0)
// multiplies by x modulo P. Appending n zero bytes to a zero-initialised CRC
// multiplies its register by x^(8n) mod P, which lets independently computed
// pieces be joined: crc(A || B) = crc(A) * x^(8|B|) + crc(B).
constexpr uint32_t kCrcPoly = 0xEDB88320u;

__host__ __device__ constexpr uint32_t gf2_times_x(uint32_t a) {
  return (a >> 1) ^ ((a & 1u) ? kCrcPoly : 0u);
}
// a * b mod P: Horner over a's coefficients from x^31 (bit 0) down to x^0 (bit 31)
__host__ __device__ constexpr uint32_t gf2_mul(uint32_t a, uint32_t b) {
  uint32_t acc = 0;
  for (int i = 0; i < 32; ++i) {
    acc = gf2_times_x(acc);
    if ((a >> i) & 1u) acc ^= b;
  }
  return acc;
}
// x^(8n) mod P by square and multiply (x^8 is bit 23)
__host__ __device__ constexpr uint32_t gf2_xpow8(uint64_t n) {
  uint32_t r = 0x80000000u, base = 0x00800000u;
  while (n) {
    if (n & 1u) r = gf2_mul(r, base);
    base = gf2_mul(base, base);
    n >>= 1;
  }
  return r;
}

// Block CRC: every thread owns a contiguous run of kCrcRun bytes per round;
// kCrcShift[l] = x^(8 * kCrcRun * 2^l) joins neighbouring runs in a tree and
// kCrcShift[log2(threads)] steps a thread's accumulator from round to round.
constexpr uint32_t kCrcRun = 256;
struct CrcShifts { uint32_t v[12]; };
constexpr CrcShifts make_crc_shifts() {
  CrcShifts s{};
  for (int l = 0; l < 12; ++l) s.v[l] = gf2_xpow8(uint64_t(kCrcRun) << l);
  return s;
}
__constant__ CrcShifts kCrcShift = make_crc_shifts();

// slice-by-4 tables in shared memory: t[0..255] one byte, t[256*k + b] byte b
// followed by k zero bytes
__device__ inline void crc_tables_init(uint32_t* t) {
  for (uint32_t b = threadIdx.x; b < 256; b += blockDim.x) {
    uint32_t c = b;
    for (int i = 0; i < 8; ++i) c = gf2_times_x(c);
    t[b] = c;
  }
  __syncthreads();
  for (uint32_t b = threadIdx.x; b < 256; b += blockDim.x) {
    uint32_t c = t[b];
    for (int k = 1; k < 4; ++k) {
      c = (c >> 8) ^ t[c & 0xffu];
      t[256 * k + b] = c;
    }
  }
  __syncthreads();
}

__device__ inline uint32_t crc_word(const uint32_t* t, uint32_t crc, uint32_t w) {
  crc ^= w;
  return t[768 + (crc & 0xffu)] ^ t[512 + ((crc >> 8) & 0xffu)] ^ t[256 + ((crc >> 16) & 0xffu)] ^
         t[crc >> 24];
}
__device__ inline uint32_t crc_byte(const uint32_t* t, uint32_t crc, uint32_t b) {
  return (crc >> 8) ^ t[(crc ^ b) & 0xffu];
}

// x^(8 kCrcRun d) mod P for d < 1024: the factor that carries the register of
// a run of kCrcRun bytes past d further runs.
struct CrcRunPow {
  uint32_t v[1024];
};
constexpr CrcRunPow make_crc_run_pow() {
  CrcRunPow t{};
  const uint32_t step = gf2_xpow8(kCrcRun);
  uint32_t p = 0x80000000u;
  for (int d = 0; d < 1024; ++d) {
    t.v[d] = p;
    p = gf2_mul(p, step);
  }
  return t;
}
__device__ const CrcRunPow kCrcRunPow = make_crc_run_pow();

// Join per-thread raw CRCs (thread order = message order, one run of kCrcRun
// bytes per thread) into thread 0's value: crc(A B) = crc(A) x^(8|B|) + crc(B),
// so each register is carried past the runs after it by one multiplication
// (in parallel; zero registers need none) and the products are summed by
// exclusive or. red must hold blockDim.x / 32 words.
__device__ inline uint32_t crc_block_join(uint32_t c, uint32_t* red) {
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  const uint32_t nwarps = blockDim.x >> 5;
  if (c) c = gf2_mul(c, __ldg(&kCrcRunPow.v[blockDim.x - 1u - threadIdx.x]));
  c = __reduce_xor_sync(0xffffffffu, c);
  __syncthreads();
  if (lane == 0) red[warp] = c;
  __syncthreads();
  uint32_t total = 0;
  if (threadIdx.x == 0)
    for (uint32_t w = 0; w < nwarps; ++w) total ^= red[w];
  __syncthreads();
  return total;  // valid in thread 0
}

__device__ inline int ilog2_u32(uint32_t v) { return 31 - __clz(v); }

// CRC-32 of len bytes at p (16-byte aligned, len a multiple of 16), computed by
// the whole block; result valid in thread 0. The message is padded in front
// with zero bytes to whole rounds (a zero-initialised CRC ignores leading
// zeros); the standard initial value is applied by complementing the first
// four message bytes, and the final xor at the end. A thread's run is loaded
// four 16-byte units at a time, so that its loads overlap. kReadOnly: the
// bytes are not written while the kernel runs, so the loads may allocate in L1
// (where the caller's later reads of the same record then find them).
template <bool kReadOnly = false>
__device__ inline uint32_t crc32_block_aligned(const uint8_t* p, uint32_t len, const uint32_t* t,
                                               uint32_t* red) {
  const uint32_t nthr = blockDim.x;
  const uint32_t round_bytes = nthr * kCrcRun;
  const uint32_t rounds = (len + round_bytes - 1) / round_bytes;
  const uint32_t pad = rounds * round_bytes - len;
  const uint32_t step = kCrcShift.v[ilog2_u32(nthr)];
  uint32_t acc = 0;
  for (uint32_t r = 0; r < rounds; ++r) {
    if (acc) acc = gf2_mul(acc, step);
    const int64_t run0 = int64_t(r) * round_bytes + int64_t(threadIdx.x) * kCrcRun - int64_t(pad);
    uint32_t c = 0;
    if (run0 + int64_t(kCrcRun) > 0) {  // runs wholly inside the padding leave c = 0
      for (uint32_t k = 0; k < kCrcRun; k += 64) {
        uint4 v[4];
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
          const int64_t off = run0 + k + 16u * i;
          const uint4* q = reinterpret_cast<const uint4*>(p + off);
          v[i] = off < 0 ? make_uint4(0, 0, 0, 0) : kReadOnly ? __ldg(q) : __ldcg(q);
        }
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
          const int64_t off = run0 + k + 16u * i;
          if (off < 0) continue;
          if (off == 0) v[i].x = ~v[i].x;
          c = crc_word(t, c, v[i].x);
          c = crc_word(t, c, v[i].y);
          c = crc_word(t, c, v[i].z);
          c = crc_word(t, c, v[i].w);
        }
      }
    }
    acc ^= c;
  }
  uint32_t total = crc_block_join(acc, red);
  return len ? (total ^ 0xffffffffu) : 0u;
}

// CRC-32 of a virtual message of len bytes whose byte i is fetch(i), any
// length; result valid in thread 0. The initial value 0xFFFFFFFF is applied by
// complementing the first four bytes (the register absorbs exactly the next 32
// message bits), or for shorter messages by adding 0xFFFFFFFF * x^(8 len).
template <class Fetch>
__device__ inline uint32_t crc32_block_bytes(Fetch fetch, uint64_t len, const uint32_t* t,
                                             uint32_t* red) {
  const uint32_t nthr = blockDim.x;
  const uint64_t round_bytes = uint64_t(nthr) * kCrcRun;
  const uint64_t rounds = (len + round_bytes - 1) / round_bytes;
  const uint64_t pad = rounds * round_bytes - len;
  const uint32_t step = kCrcShift.v[ilog2_u32(nthr)];
  uint32_t acc = 0;
  for (uint64_t r = 0; r < rounds; ++r) {
    if (acc) acc = gf2_mul(acc, step);
    int64_t run0 = int64_t(r * round_bytes) + int64_t(threadIdx.x) * kCrcRun - int64_t(pad);
    uint32_t c = 0;
    for (uint32_t k = 0; k < kCrcRun; ++k) {
      int64_t off = run0 + k;
      if (off < 0) continue;
      uint32_t b = fetch(uint64_t(off));
      if (off < 4 && len >= 4) b ^= 0xffu;
      c = crc_byte(t, c, b);
    }
    acc ^= c;
  }
  uint32_t total = crc_block_join(acc, red);
  if (len == 0) return 0u;
  // under four bytes the initial register is shifted through the message instead
  if (len < 4) total ^= gf2_mul(0xffffffffu, gf2_xpow8(len));
  return total ^ 0xffffffffu;
}

constexpr uint32_t kCrcRegionMaxUnits = 33;  // runs of at most 33 * 16 bytes: regions <= 67584 bytes

// Powers of x used to join CRC pieces: q[n][l] = x^(8 * 16n * 2^l) joins
// neighbouring runs of 16n bytes (l-th level of a tree); u[m] = x^(8 * 16m).
struct CrcPowTables {
  uint32_t q[34][8];
  uint32_t u[128];
};
constexpr CrcPowTables make_crc_pow_tables() {
  CrcPowTables t{};
  const uint32_t x16 = gf2_xpow8(16);
  uint32_t p = 0x80000000u;  // x^0
  for (int n = 0; n < 34; ++n) {
    uint32_t c = p;
    for (int l = 0; l < 8; ++l) {
      t.q[n][l] = c;
      c = gf2_mul(c, c);
    }
    p = gf2_mul(p, x16);
  }
  p = 0x80000000u;
  for (int m = 0; m < 128; ++m) {
    t.u[m] = p;
    p = gf2_mul(p, x16);
  }
  return t;
}
__constant__ CrcPowTables kCrcPow = make_crc_pow_tables();

// Per-thread powers for joining the registers of 128 consecutive runs of 16q
// bytes: the register of run t, multiplied by x^(8 * 16q * (127 - t)), is its
// share of the register of the concatenation, so the join is one multiply per
// thread and an exclusive-or reduction.
struct CrcLanePow {
  uint32_t v[kCrcRegionMaxUnits + 1][128];
};
constexpr CrcLanePow make_crc_lane_pow() {
  CrcLanePow t{};
  const uint32_t x16 = gf2_xpow8(16);
  uint32_t step = 0x80000000u;  // x^(8 * 16q)
  for (uint32_t q = 0; q <= kCrcRegionMaxUnits; ++q) {
    uint32_t p = 0x80000000u;
    for (int i = 127; i >= 0; --i) {
      t.v[q][i] = p;
      p = gf2_mul(p, step);
    }
    step = gf2_mul(step, x16);
  }
  return t;
}
__device__ const CrcLanePow kCrcLanePow = make_crc_lane_pow();

// Join the registers of 128 consecutive runs of 16q bytes (thread t holds run
// t, exactly 128 threads); result in thread 0.
__device__ inline uint32_t crc_join_lanes(uint32_t c, uint32_t q, uint32_t* red) {
  c = gf2_mul(c, __ldg(&kCrcLanePow.v[q][threadIdx.x]));
#pragma unroll
  for (uint32_t o = 16; o; o >>= 1) c ^= __shfl_xor_sync(0xffffffffu, c, o);
  __syncthreads();
  if ((threadIdx.x & 31u) == 0) red[threadIdx.x >> 5] = c;
  __syncthreads();
  return threadIdx.x == 0 ? red[0] ^ red[1] ^ red[2] ^ red[3] : 0u;
}

// ---------------------------------------------------------------- block helpers
// exclusive scan of one value per thread (blockDim.x <= 1024); tmp holds 32 words
__device__ inline uint32_t block_exclusive_scan(uint32_t v, uint32_t* tmp, uint32_t* total) {
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= uint32_t(o)) x += y;
  }
  __syncthreads();
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t nw = blockDim.x >> 5;
    uint32_t w = lane < nw ? tmp[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= uint32_t(o)) w += y;
    }
    if (lane < nw) tmp[lane] = w;
  }
  __syncthreads();
  uint32_t base = warp ? tmp[warp - 1] : 0u;
  if (total) *total = tmp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return base + x - v;
}

__device__ inline uint32_t block_sum(uint32_t v, uint32_t* tmp) {
  uint32_t total;
  block_exclusive_scan(v, tmp, &total);
  return total;
}


// ---------------------------------------------------------------- frequency tables
// Largest-remainder normalisation of a 256-bin histogram of n symbols to a
// total of 4096 (any power-of-two block of 64..1024 threads): f_s = 1 + floor(c_s (4096 - k) / n),
// the 4096 - sum f_s symbols with the largest remainders c_s (4096 - k) mod n
// (ties: smaller symbol) get one more. freq and rem are 256-word shared arrays.
// Returns k, the number of present symbols (block-uniform).
__device__ inline uint32_t block_normalize(const uint32_t* hist, uint32_t n, uint32_t* freq,
                                           uint32_t* rem, uint32_t* tmp) {
  // thread owns symbols [s0, s0 + per); blockDim.x is a power of two <= 1024
  const uint32_t per = blockDim.x >= 256 ? 1u : 256u / blockDim.x;
  const uint32_t s0 = threadIdx.x * per;
  uint32_t present = 0;
  for (uint32_t i = 0; i < per; ++i) present += (s0 + i < 256 && hist[s0 + i]) ? 1u : 0u;
  const uint32_t k = block_sum(present, tmp);
  uint32_t fsum = 0;
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t s = s0 + i;
    if (s >= 256) break;
    const uint32_t c = hist[s];
    uint32_t f = 0, r = 0;
    if (k >= 2 && c) {
      const uint32_t q = c * (kProbScale - k);  // < 2^28
      f = 1u + q / n;
      r = q % n;
    } else if (k == 1 && c) {
      f = kProbScale;
    }
    rem[s] = r;
    freq[s] = f;
    fsum += f;
  }
  const uint32_t sum = block_sum(fsum, tmp);  // synchronises: rem and freq complete
  const uint32_t d = k >= 2 ? kProbScale - sum : 0u;
  if (d) {
    // The d present symbols with the largest keys (r << 8) | (255 - s) (largest
    // remainder, ties to the smaller symbol; keys are distinct) get one more.
    // Radix select of the d-th largest key, one bit per round: P holds the key
    // bits fixed so far, need the rank still sought among keys with prefix P.
    uint32_t P = 0, need = d;
    for (int bit = 23; bit >= 0; --bit) {
      uint32_t cnt = 0;
      for (uint32_t i = 0; i < per; ++i) {
        const uint32_t s = s0 + i;
        const bool present = s < 256 && hist[s];
        const uint32_t key = present ? (rem[s] << 8) | (255u - s) : 0u;
        cnt += __syncthreads_count(present && (key >> bit) == ((P << 1) | 1u));
      }
      if (cnt >= need) P = (P << 1) | 1u;
      else {
        need -= cnt;
        P <<= 1;
      }
    }
    for (uint32_t i = 0; i < per; ++i) {
      const uint32_t s = s0 + i;
      if (s < 256 && hist[s] && ((rem[s] << 8) | (255u - s)) >= P) freq[s] += 1u;
    }
  }
  __syncthreads();
  return k;
}

// From freq[256] (sum 4096): fc[s] = f | cum << 16 and rcp[s] = floor((2^32-1)/f).
__device__ inline void block_enc_tables(const uint32_t* freq, uint32_t* fc, uint32_t* rcp,
                                        uint32_t* tmp) {
  const uint32_t per = blockDim.x >= 256 ? 1u : 256u / blockDim.x;
  const uint32_t s0 = threadIdx.x * per;
  uint32_t mine = 0;
  for (uint32_t i = 0; i < per; ++i) mine += s0 + i < 256 ? freq[s0 + i] : 0u;
  uint32_t cum = block_exclusive_scan(mine, tmp, nullptr);
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t s = s0 + i;
    if (s >= 256) break;
    const uint32_t f = freq[s];
    fc[s] = f | (cum << 16);
    rcp[s] = f ? 0xffffffffu / f : 0u;
    cum += f;
  }
  __syncthreads();
}

// Largest-remainder normalisation by one warp (the rule of block_normalize) of
// hist[0 .. A), A <= 256, n symbols: writes freq[0 .. 256) and the coding table
// tab[0 .. A) = {f | cum << 16, floor((2^32-1)/f)}; rem is not used (kept for
// the callers' layouts). Returns k. The d symbols that get one more are found
// by a radix select over the keys 1 << 24 | r << 8 | (255 - s) of the present
// symbols (absent: 0), held in registers: lane l keeps the keys of symbols
// l + 32 j. freq may alias hist: each lane reads a symbol's count before it
// writes that symbol's frequency.
__device__ inline uint32_t warp_normalize(const uint32_t* hist, uint32_t A, uint32_t n, uint32_t* freq,
                                          uint32_t* rem, uint2* tab) {
  (void)rem;
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t present = 0;
  for (uint32_t s = lane; s < A; s += 32u) present += hist[s] ? 1u : 0u;
  const uint32_t k = __reduce_add_sync(0xffffffffu, present);
  uint32_t fsum = 0, key[8];
#pragma unroll
  for (uint32_t j = 0; j < 8; ++j) {
    const uint32_t s = lane + 32u * j;
    const uint32_t c = s < A ? hist[s] : 0u;
    uint32_t f = 0, r = 0;
    if (k >= 2 && c) {
      const uint32_t q = c * (kProbScale - k);
      f = 1u + q / n;
      r = q % n;
    } else if (k == 1 && c) {
      f = kProbScale;
    }
    key[j] = c ? (1u << 24) | (r << 8) | (255u - s) : 0u;
    freq[s] = f;
    fsum += f;
  }
  const uint32_t sum = __reduce_add_sync(0xffffffffu, fsum);
  if (k >= 2 && sum < kProbScale) {
    // P: the key bits fixed so far (bit 24, presence, is 1); need: the rank
    // still sought among the keys that start with P
    uint32_t P = 1, need = kProbScale - sum;
    for (int bit = 23; bit >= 0; --bit) {
      uint32_t cnt = 0;
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j)
        if (32u * j < A) cnt += __popc(__ballot_sync(0xffffffffu, (key[j] >> bit) == ((P << 1) | 1u)));
      if (cnt >= need) P = (P << 1) | 1u;
      else {
        need -= cnt;
        P <<= 1;
      }
    }
#pragma unroll
    for (uint32_t j = 0; j < 8; ++j)
      if (key[j] >= P) freq[lane + 32u * j] += 1u;
  }
  __syncwarp();
  uint32_t carry = 0;
  for (uint32_t s0 = 0; s0 < A; s0 += 32u) {
    const uint32_t s = s0 + lane;
    const uint32_t f = s < A ? freq[s] : 0u;
    uint32_t incl = f;
#pragma unroll
    for (uint32_t o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (s < A) tab[s] = make_uint2(f | ((carry + incl - f) << 16), f ? 0xffffffffu / f : 0u);
    carry += __shfl_sync(0xffffffffu, incl, 31);
  }
  __syncwarp();
  return k;
}

// Decode table: lut[slot] = s | (slot - cum_s) << 8 | f_s << 20, and the
// symbols' cumulative starts in cum[257]. freq must be validated (sum 4096).
// The first slot of every present symbol is marked with s + 1; each warp then
// resolves its span of slots 32 at a time, a running maximum of the marks
// giving every slot its symbol.
__device__ inline void block_dec_lut(const uint32_t* freq, uint32_t* cum, uint32_t* lut,
                                     uint32_t* tmp) {
  const uint32_t per = blockDim.x >= 256 ? 1u : 256u / blockDim.x;
  const uint32_t s0 = threadIdx.x * per;
  uint32_t mine = 0;
  for (uint32_t i = 0; i < per; ++i) mine += s0 + i < 256 ? freq[s0 + i] : 0u;
  uint32_t c = block_exclusive_scan(mine, tmp, nullptr);
  for (uint32_t i = 0; i < per; ++i) {
    if (s0 + i >= 256) break;
    cum[s0 + i] = c;
    c += freq[s0 + i];
  }
  if (threadIdx.x == 0) cum[256] = kProbScale;
  for (uint32_t i = threadIdx.x; i < kProbScale / 4u; i += blockDim.x)
    reinterpret_cast<uint4*>(lut)[i] = make_uint4(0, 0, 0, 0);
  __syncthreads();
  for (uint32_t s = threadIdx.x; s < 256; s += blockDim.x)
    if (freq[s]) lut[cum[s]] = s + 1u;
  __syncthreads();
  const uint32_t nw = blockDim.x >> 5, warp = threadIdx.x >> 5, lane = threadIdx.x & 31u;
  const uint32_t span = kProbScale / nw, first = warp * span;
  // mark carried into the span: the last symbol starting before it (its start
  // is below `first`, and the largest such s has a nonzero frequency)
  uint32_t carry = 0;
  if (first) {
    uint32_t lo = 0, hi = 255;
    while (lo < hi) {
      const uint32_t mid = (lo + hi + 1) >> 1;
      if (cum[mid] < first) lo = mid; else hi = mid - 1;
    }
    carry = lo + 1u;
  }
#pragma unroll 4
  for (uint32_t b = 0; b < span; b += 32u) {
    const uint32_t slot = first + b + lane;
    uint32_t m = lut[slot];
#pragma unroll
    for (uint32_t o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, m, o);
      if (lane >= o) m = max(m, y);
    }
    m = max(m, carry);
    carry = __shfl_sync(0xffffffffu, m, 31);
    const uint32_t sym = m - 1u;
    lut[slot] = sym | ((slot - cum[sym]) << 8) | (freq[sym] << 20);
  }
  __syncthreads();
}

__device__ inline uint32_t lanemask_lt() {
  return (1u << (threadIdx.x & 31u)) - 1u;
}

// Warp-level rANS encode of group g of a stream of n symbols (all 32 lanes
// call). Steps run in reverse (tau descending); within a step, words of the
// lanes that renormalise are placed in ascending lane order in front of the
// words already written, exactly mirroring the decoder. Words go backwards into
// words[0, cap) ending at cap; returns the number of words; *x_out gets the
// lane's final state (to be stored as its initial state).
template <class SymFn>
__device__ inline uint32_t rans_encode_group(SymFn sym, uint32_t n, uint32_t N, uint32_t g,
                                             const uint32_t* fc, const uint32_t* rcp,
                                             uint16_t* words, uint32_t cap, uint32_t* x_out) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t l = g * kGroupLanes + lane;
  const bool live = l < N;
  uint32_t start = 0, len = 0, start0, maxlen;
  if (live) lane_range(n, N, l, start, len);
  lane_range(n, N, g * kGroupLanes, start0, maxlen);
  uint32_t x = kRansLow, pos = cap;
  const uint32_t lt = lanemask_lt();
  for (uint32_t tau = maxlen; tau-- > 0;) {
    const bool act = live && tau < len;
    uint32_t s = act ? sym(start + tau) : 0u;
    uint32_t e = fc[s], f = e & 0xffffu, cum = e >> 16;
    bool emit = act && x >= (f << 20);
    uint32_t mask = __ballot_sync(0xffffffffu, emit);
    pos -= __popc(mask);
    if (emit) {
      words[pos + __popc(mask & lt)] = uint16_t(x & 0xffffu);
      x >>= 16;
    }
    if (act) {
      uint32_t q = __umulhi(x, rcp[s]);
      uint32_t r = x - q * f;
      if (r >= f) { ++q; r -= f; }
      x = (q << kProbBits) + r + cum;
    }
  }
  *x_out = x;
  return cap - pos;
}

// rANS encode of group g of a stream of n symbols laid out as a strided 2-D
// byte array (all 32 lanes call): symbol i = col * tcc + t is the byte at
// col_base(col) + t * stride. The steps and word placement are those of
// rans_encode_group; each lane walks a byte pointer backwards (recomputing it
// only when it wraps to the previous column) and fetches its next symbol and
// that symbol's table entry tab[s] = {f | cum << 16, floor((2^32 - 1) / f)}
// one step ahead, so the loop's dependency chain is the state update alone.
// With kDelta the coded symbol is the lane delta: the byte XORed with the
// lane's previous byte (the one at the next smaller index), except for the
// lane's first symbol.
template <bool kDelta = false, class ColBase>
__device__ inline uint32_t rans_encode_strided(ColBase col_base, uint32_t stride, uint32_t tcc, uint32_t n,
                                               uint32_t N, uint32_t g, const uint2* tab, uint16_t* words,
                                               uint32_t cap, uint32_t* x_out) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t l = g * kGroupLanes + lane;
  const bool live = l < N;
  uint32_t start = 0, len = 0, start0, maxlen;
  if (live) lane_range(n, N, l, start, len);
  lane_range(n, N, g * kGroupLanes, start0, maxlen);
  const uint32_t lt = lanemask_lt();
  uint32_t col = 0, t = 0;
  const uint8_t* p = nullptr;
  uint32_t s = 0;
  // byte before the one at (col, t) in stream order (for the lane delta)
  auto prev_byte = [&](uint32_t c, uint32_t tt, const uint8_t* q) -> uint32_t {
    return tt ? uint32_t(q[-int64_t(stride)]) : uint32_t(col_base(c - 1u)[uint64_t(tcc - 1u) * stride]);
  };
  if (live) {
    const uint32_t last = start + len - 1u;
    col = last / tcc;
    t = last - col * tcc;
    p = col_base(col) + uint64_t(t) * stride;
    s = *p;
    if (kDelta && len > 1u) s ^= prev_byte(col, t, p);
  }
  uint2 e = tab[s];
  uint32_t x = kRansLow, pos = cap;
  for (uint32_t tau = maxlen; tau-- > 0;) {
    const bool act = live && tau < len;
    // the lane's next symbol (tau - 1 < len), without a branch: the pointer only
    // ever points into the lane's own range, so the load is always in bounds
    const bool adv = act && tau > 0u;
    const bool wrap = adv && t == 0u;
    if (wrap) {
      t = tcc;
      --col;
      p = col_base(col) + uint64_t(tcc) * stride;
    }
    t -= adv ? 1u : 0u;
    p -= adv ? stride : 0u;
    uint32_t ns = live ? uint32_t(*p) : 0u;
    if (kDelta) {
      if (adv && tau > 1u) ns ^= prev_byte(col, t, p);  // the next symbol is not the lane's first
      ns = adv ? ns : s;  // a lane waiting for its first step keeps its (delta) symbol
    }
    const uint2 ne = tab[ns];
    const uint32_t f = e.x & 0xffffu, cum = e.x >> 16;
    const bool emit = act && x >= (f << 20);
    const uint32_t mask = __ballot_sync(0xffffffffu, emit);
    pos -= __popc(mask);
    if (emit) words[pos + __popc(mask & lt)] = uint16_t(x & 0xffffu);
    const uint32_t xe = emit ? (x >> 16) : x;
    uint32_t q = __umulhi(xe, e.y);
    uint32_t r = xe - q * f;
    const bool over = r >= f;
    q += over ? 1u : 0u;
    r -= over ? f : 0u;
    x = act ? (q << kProbBits) + r + cum : xe;
    s = ns;
    e = ne;
  }
  *x_out = x;
  return cap - pos;
}

// Warp-level rANS decode of group g from its sub-stream (sub_len bytes, states
// then words; sub is 4-byte aligned). out(i, s) receives symbol i. Returns
// true when every lane ends at 2^16 and exactly all words were read.
template <class OutFn>
__device__ inline bool rans_decode_group(const uint8_t* sub, uint32_t sub_len, uint32_t n,
                                         uint32_t N, uint32_t g, const uint32_t* lut, OutFn out) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t l = g * kGroupLanes + lane;
  const uint32_t lanes_g = min(kGroupLanes, N - g * kGroupLanes);
  if (sub_len < 4u * lanes_g || ((sub_len - 4u * lanes_g) & 1u)) return false;
  const uint32_t W = (sub_len - 4u * lanes_g) >> 1;
  const uint16_t* w16 = reinterpret_cast<const uint16_t*>(sub + 4u * lanes_g);
  const bool live = lane < lanes_g;
  uint32_t start = 0, len = 0, start0, maxlen;
  if (live) lane_range(n, N, l, start, len);
  lane_range(n, N, g * kGroupLanes, start0, maxlen);
  uint32_t x = live ? reinterpret_cast<const uint32_t*>(sub)[lane] : kRansLow;
  uint32_t pos = 0;
  bool bad = false;
  const uint32_t lt = lanemask_lt();
  for (uint32_t tau = 0; tau < maxlen; ++tau) {
    const bool act = live && tau < len;
    if (act) {
      uint32_t e = lut[x & (kProbScale - 1u)];
      x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xfffu);
      out(start + tau, e & 0xffu);
    }
    bool need = act && x < kRansLow;
    uint32_t mask = __ballot_sync(0xffffffffu, need);
    if (need) {
      uint32_t idx = pos + __popc(mask & lt);
      if (idx < W) x = (x << 16) | w16[idx];
      else { bad = true; x = kRansLow; }
    }
    pos += __popc(mask);
  }
  bool ok = !bad && pos == W && (!live || x == kRansLow);
  return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- stream records
// header: u8 mode, u8 const symbol, u8 groups, u8 0, u32 record bytes, u32 n,
// u32 k; RAW: n bytes + pad; CONST: nothing; RANS: 32-byte bitmap, k u16
// frequencies + pad, G u32 sub-stream lengths + pad, padded sub-streams.
struct StreamInfo {
  uint32_t mode, sym, groups, bytes, k;
  uint32_t delta;  // 1: the RANS symbols are lane deltas (header byte 3)
  uint32_t sub_off[4], sub_len[4];
  int status;
};

__host__ __device__ inline uint32_t rans_record_bytes(uint32_t k, uint32_t G, const uint32_t* sub_len) {
  uint32_t b = 16u + 32u + pad16(2u * k) + pad16(4u * G);
  for (uint32_t g = 0; g < G; ++g) b += pad16(sub_len[g]);
  return b;
}

// Validate the stream record at rec (16-byte aligned, avail bytes left in the
// chunk record) for n symbols and, for RANS, load its frequency table into
// freq[256]. Block-cooperative; si is shared. Returns status (block-uniform).
__device__ inline int block_parse_stream(const uint8_t* rec, uint32_t avail, uint32_t n,
                                         StreamInfo* si, uint32_t* freq, uint32_t* tmp,
                                         bool allow_delta = true) {
  if (threadIdx.x == 0) {
    int st = kOk;
    if (avail < 16) st = kErrCorrupt;
    else {
      const uint4 hv = __ldg(reinterpret_cast<const uint4*>(rec));  // records are 16-byte aligned
      uint32_t mode = hv.x & 0xffu, csym = (hv.x >> 8) & 0xffu, G = (hv.x >> 16) & 0xffu;
      uint32_t bytes = hv.y, rn = hv.z, k = hv.w;
      const uint32_t b3 = hv.x >> 24;
      si->mode = mode; si->sym = csym; si->groups = G; si->bytes = bytes; si->k = k; si->delta = b3;
      if (b3 > (allow_delta && mode == kModeRans ? 1u : 0u) || rn != n || (bytes & 15u) || bytes < 16 ||
          bytes > avail)
        st = kErrCorrupt;
      else if (mode == kModeRaw) {
        if (csym || G || k || bytes != 16u + pad16(n)) st = kErrCorrupt;
      } else if (mode == kModeConst) {
        if (G || k != 1 || bytes != 16) st = kErrCorrupt;
      } else if (mode == kModeRans) {
        uint32_t N = rans_lanes(n);
        if (csym || n == 0 || G != rans_groups(N) || k < 2 || k > 256) st = kErrCorrupt;
        else {
          uint32_t p = pad16(48u + 2u * k);
          uint32_t lens_at = p;
          p = pad16(p + 4u * G);
          if (p > bytes) st = kErrCorrupt;
          uint32_t lens[4] = {0, 0, 0, 0};
          if (st == kOk) {  // G <= 4 lengths in one aligned 16-byte load
            const uint4 lv = __ldg(reinterpret_cast<const uint4*>(rec + lens_at));
            lens[0] = lv.x; lens[1] = lv.y; lens[2] = lv.z; lens[3] = lv.w;
          }
          for (uint32_t g = 0; g < G && st == kOk; ++g) {
            uint32_t sl = lens[g];
            if (sl > bytes || p + pad16(sl) > bytes) { st = kErrCorrupt; break; }
            si->sub_off[g] = p;
            si->sub_len[g] = sl;
            p += pad16(sl);
          }
          if (st == kOk && p != bytes) st = kErrCorrupt;
        }
      } else {
        st = kErrCorrupt;
      }
      si->status = st;
    }
    if (avail < 16) si->status = st;
  }
  __syncthreads();
  int st = si->status;
  if (st != kOk || si->mode != kModeRans) return st;
  // RANS table: presence bitmap + k u16 frequencies
  const uint32_t per = blockDim.x >= 256 ? 1u : 256u / blockDim.x;
  const uint32_t s0 = threadIdx.x * per;
  uint32_t mine = 0;
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t s = s0 + i;
    if (s < 256) mine += (rec[16 + (s >> 3)] >> (s & 7u)) & 1u;
  }
  uint32_t total_present;
  uint32_t idx = block_exclusive_scan(mine, tmp, &total_present);
  uint32_t bad = total_present != si->k;
  uint32_t fs = 0;
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t s = s0 + i;
    if (s >= 256) break;
    const uint32_t present = (rec[16 + (s >> 3)] >> (s & 7u)) & 1u;
    uint32_t f = 0;
    if (present && !bad) {
      f = ld_u16(rec + 48 + 2u * idx);
      ++idx;
      if (f == 0) bad = 1;
    }
    fs += f;
    freq[s] = f;
  }
  const uint32_t fsum = block_sum(fs, tmp);
  bad = __syncthreads_or(bad) || fsum != kProbScale;
  return bad ? kErrCorrupt : kOk;
}


// Sub-stream lengths and record size of a RANS stream whose groups produced
// W[g] words; returns the record bytes.
__device__ inline uint32_t rans_layout(uint32_t n, uint32_t k, const uint32_t* W, uint32_t* sub_len) {
  uint32_t N = rans_lanes(n), G = rans_groups(N);
  for (uint32_t g = 0; g < G; ++g) {
    uint32_t lanes_g = min(kGroupLanes, N - g * kGroupLanes);
    sub_len[g] = 4u * lanes_g + 2u * W[g];
  }
  return rans_record_bytes(k, G, sub_len);
}

// Write one stream record at rec (global, 16-byte aligned); all threads call.
//   RAW:   raw(i) gives symbol i
//   CONST: csym
//   RANS:  freq[256] table, states[l] final encoder states (shared), group g's
//          words at words[wbeg[g] .. wbeg[g] + W[g]) (global, written before a
//          __syncthreads), sub_len from rans_layout.
// Every padding byte is written as zero.
template <class RawFn>
__device__ inline void block_write_stream(uint8_t* rec, uint32_t mode, uint32_t n, uint32_t bytes,
                                          uint32_t csym, uint32_t k, const uint32_t* freq,
                                          const uint32_t* states, const uint16_t* words,
                                          const uint32_t* wbeg, const uint32_t* W,
                                          const uint32_t* sub_len, RawFn raw, uint32_t* tmp,
                                          uint32_t delta = 0) {
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  if (mode == kModeRaw || mode == kModeConst) {
    if (tid == 0) {
      *reinterpret_cast<uint4*>(rec) =
          make_uint4(mode | (mode == kModeConst ? (csym << 8) : 0u), bytes, n,
                     mode == kModeConst ? 1u : 0u);
    }
    if (mode == kModeRaw) {
      const uint32_t chunks = pad16(n) / 16u;
      for (uint32_t q = tid; q < chunks; q += nthr) {
        uint32_t w[4] = {0, 0, 0, 0};
        for (uint32_t b = 0; b < 16; ++b) {
          uint32_t i = q * 16u + b;
          uint32_t v = i < n ? raw(i) : 0u;
          w[b >> 2] |= v << (8 * (b & 3u));
        }
        *reinterpret_cast<uint4*>(rec + 16 + q * 16u) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    return;
  }
  // RANS
  const uint32_t N = rans_lanes(n), G = rans_groups(N);
  const uint32_t lane = tid & 31u, warp = tid >> 5;
  if (tid == 0) *reinterpret_cast<uint4*>(rec) = make_uint4(kModeRans | (G << 16) | (delta << 24), bytes, n, k);
  // bitmap word w (symbols 32w .. 32w+31) from a ballot of warp w % nwarps
  for (uint32_t w = warp; w < 8; w += nthr >> 5) {
    const uint32_t bits = __ballot_sync(0xffffffffu, freq[32 * w + lane] != 0u);
    if (lane == 0) reinterpret_cast<uint32_t*>(rec + 16)[w] = bits;
  }
  const uint32_t per = nthr >= 256 ? 1u : 256u / nthr;
  const uint32_t s0 = tid * per;
  uint32_t mine = 0;
  for (uint32_t i = 0; i < per; ++i) mine += (s0 + i < 256 && freq[s0 + i]) ? 1u : 0u;
  uint32_t idx = block_exclusive_scan(mine, tmp, nullptr);
  const uint32_t ftab_end = 48u + 2u * k, lens_at = pad16(ftab_end);
  for (uint32_t i = 0; i < per; ++i) {
    const uint32_t s = s0 + i;
    if (s < 256 && freq[s]) st_u16(rec + 48 + 2u * idx++, freq[s]);
  }
  if (tid < lens_at - ftab_end) rec[ftab_end + tid] = 0;
  const uint32_t lens_end = lens_at + 4u * G, sub0 = pad16(lens_end);
  if (tid < G) reinterpret_cast<uint32_t*>(rec + lens_at)[tid] = sub_len[tid];
  if (tid < sub0 - lens_end) rec[lens_end + tid] = 0;
  uint32_t off = sub0;
  for (uint32_t g = 0; g < G; ++g) {
    const uint32_t lanes_g = min(kGroupLanes, N - g * kGroupLanes);
    uint8_t* sub = rec + off;
    if (tid < lanes_g) reinterpret_cast<uint32_t*>(sub)[tid] = states[g * kGroupLanes + tid];
    uint16_t* w16 = reinterpret_cast<uint16_t*>(sub + 4u * lanes_g);
    const uint16_t* src = words + wbeg[g];
    for (uint32_t i = tid; i < W[g]; i += nthr) w16[i] = src[i];
    const uint32_t end = off + sub_len[g], padded = off + pad16(sub_len[g]);
    if (tid < padded - end) rec[end + tid] = 0;
    off = padded;
  }
}

}  // namespace kvc
