// Transform-coding kernels (sm_100a), KVTC-style (KVTC page, "How the Pipeline
// Works": sink tokens and a recent window kept exact, the middle RoPE-undone,
// projected on a per-head PCA basis, quantised with scales, zero points and bit
// widths, then rANS coded; Codec-Gauge page, "Problem Statement and Overview":
// Z = G X per (layer, K/V, head) with G^-1 = G^T, and "Compression Conditions":
// one range per token block).
//
// Numerics: keys are de-rotated in fp32 with every product and sum rounded on
// its own (__fmul_rn / __fadd_rn, no contraction) from an fp32 cos/sin table;
// the projection y_j = sum_k Q[k][j] x_k runs in fp64 with k ascending (each
// product of two fp32 values is exact in fp64, so every fused step equals a
// rounded add of the exact product) and is rounded to fp32 once; scale and
// zero point are fp32 with IEEE division; codes use round-half-even.
#include "kvc_device.cuh"
#include "kvc_internal.h"
#include "tcgen05.cuh"

namespace kvc {
namespace {

constexpr uint32_t kThreads = 256;
constexpr uint32_t kD = 128;        // head_dim handled by these kernels
constexpr uint32_t kTile = 64;      // tokens per tile = quantiser block
constexpr uint32_t kMaxCt = 512;    // max tokens per middle chunk
constexpr uint32_t kTcRows = 128;   // tokens per tensor-core tile (MMA M)
constexpr uint32_t kTcCols = 128;   // tensor-memory columns: one fp32 128 x 128 accumulator
// Polls of the tensor stage's wait for its own MMAs before the record is
// reported as KVC_ERR_TIMEOUT. A build with -DKVC_MMA_WAIT_POLLS=0
// makes that wait give up on purpose, so tests can check the timeout status;
// the drain wait that follows keeps its own long bound in every build.
#ifndef KVC_MMA_WAIT_POLLS
#define KVC_MMA_WAIT_POLLS (1u << 22)
#endif
constexpr uint32_t kMmaDrainPolls = 1u << 22;

__device__ inline float bf16_to_f32(uint32_t h) { return __uint_as_float(h << 16); }

// two fp32 values rounded to bf16 (nearest, ties to even) and packed, lo in bits 0-15
__device__ inline uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

__device__ inline uint32_t quantize(float y, float z, float s, uint32_t levels) {
  if (s == 0.0f) return 0u;
  float q = __fdiv_rn(__fsub_rn(y, z), s);
  float r = rintf(q);
  if (!(r > 0.0f)) return 0u;
  if (r >= float(levels)) return levels;
  return uint32_t(r);
}

// The plan's per-slice component order, copied into shared memory.
__device__ inline void load_comp_info(const CompInfo* src, CompInfo& dst) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
  uint4* d4 = reinterpret_cast<uint4*>(&dst);
  for (uint32_t i = threadIdx.x; i < sizeof(CompInfo) / 16u; i += blockDim.x) d4[i] = __ldg(s4 + i);
  __syncthreads();
}

struct Split {  // i -> (component slot, token) for i = slot * tcc + t
  uint32_t tcc, magic;
  __device__ Split(uint32_t t) : tcc(t), magic(0xffffffffu / t) {}
  __device__ inline void operator()(uint32_t i, uint32_t& a, uint32_t& t) const {
    a = __umulhi(i, magic);
    t = i - a * tcc;
    if (t >= tcc) { ++a; t -= tcc; }
  }
};

// ---------------------------------------------------------------------------
// Transform encode, part 1 (k_transform_project): the projection on the
// tensor cores, reproducing the oracle's y to the bit.
//
// The quantiser must see y[t][j] = fl32(acc), acc the fp64 sum over k
// ascending of Q[k][j] x_k (each product exact in fp64, one rounding per
// addition; x is the token after the keys' RoPE undo, in fp32). Per 128-token
// tile the kernel computes an estimate of acc with a rigorous bound, from exact
// integer products on the tensor cores:
//   X[t][k] = rint(x_k 2^s), s = 29 - e_t, e_t = ilogb(max_k |x_k|)   |X| <= 2^30
//   J[k][j] = rint(Q[k][j] 2^r), r = 29 - f_j (plan time, QColInfo)   |J| <= 2^30
// both as four bytes (two's complement; byte 0, the top one, signed, the others
// unsigned). tcgen05.mma kind::i8 sums the products of byte a of X and byte b
// of J over k exactly in s32; the ten pairs with a + b <= 3 add into four
// accumulators (level w = a + b: four times the coded components' columns of
// tensor memory), and
//   V = ((P0 2^8 + P1) 2^8 + P2) 2^8 + P3,   S~ = V 2^(24 - s - r)
// are exact in fp64. The six dropped pairs (a + b >= 4: unsigned bytes, 128
// terms of at most 255^2) add at most 128 255^2 (3 2^16 + 2 2^8 + 1) units of
// 2^(-s-r); rounding x and Q to X, J adds at most x1 2^(-r-1) + q1 2^(-s-1) +
// 96 2^(-s-r) (x1 >= sum_k |x_k|, q1 >= sum_k |Q[k][j]|); and the oracle's fp64
// chain is within 127 2^-53 sum_k |Q[k][j] x_k| <= 2^-46 x1 2^(f+1) of the exact
// sum. So |acc - S~| <= E, and |y - fl32(S~)| <= R = E + one fp32 ulp of the
// largest magnitude involved, with E taken per 64-token block and component at
// the block's largest e_t and x1.
//
// Where R leaves a decision open, the fp64 chain itself is run (exact_y):
//   - every token whose estimate lies within 2R of the block's smallest or
//     largest estimate: the true minimum and maximum are among them, and every
//     other token is strictly inside, so the sequential scan over the block
//     (exact values for these tokens, estimates for the rest) gives the
//     oracle's zero point and scale, -0 / +0 and ties included;
//   - every code whose interval [y~ - R, y~ + R] maps to two different codes
//     (the quantiser is monotone in y).
// Tokens whose x is all zero are exact (+0) without a chain.
//
// Layout: one CTA per SM (persistent, contiguous runs of middle records, so a
// slice's Q digits stay in shared memory across its records), 512 threads.
// Per tile: digits (thread: token t = tid / 4, channels 16g .. 16g+15 and
// their RoPE partners, g = tid % 4) -> 40 MMAs issued by one thread (four
// K-steps of 32 bytes x ten pairs) -> epilogue (warp w: tensor-memory lanes
// 32 (w % 4) .., column chunks w / 4 + 4i) writes y~ to y[cc][t] -> per-word
// phase (thread: block tid / 256, coded component (tid / 2) % 128, half tid % 2
// of the block = 32 tokens): bound, candidates, chains, zero point and scale,
// codes, counts. The side information (z, s per coded component and block)
// goes to the record area of the slot, the codes component-major to the code
// array, the symbol counts per width stream behind them.
constexpr uint32_t kCodesRow = kMaxCt;  // bytes per component row of the code array in the slot
constexpr uint32_t kTabPool = 512;     // sum over widths 1..8 of 2^b, rounded up
constexpr uint32_t kHistOffset = kCodesRow * kD;      // counts follow the codes in the slot
constexpr uint32_t kCodesArea = kHistOffset + 4u * kTabPool;
constexpr uint32_t kWordsArea = 2u * kD * kMaxCt + 64u;  // rANS word scratch: a word per symbol
// last count of a record whose projection gave up waiting for its MMAs (the
// entropy kernel then marks the record as failed)
constexpr uint32_t kHistTimeout = 0xffffffffu;

__device__ inline uint32_t tab_base(uint32_t b) { return (1u << b) - 2u; }  // 2 + 4 + ... + 2^(b-1)

// The tail of a middle record's slot: the rANS word scratch, then the code
// array (component-major: codes[j * kCodesRow + t] for component j, token t)
// and the symbol counts per width stream.
__device__ inline uint8_t* slot_codes(uint8_t* slot, uint64_t slot_bytes) { return slot + slot_bytes - kCodesArea; }
__device__ inline uint16_t* slot_words(uint8_t* slot, uint64_t slot_bytes) {
  return reinterpret_cast<uint16_t*>(slot + slot_bytes - kCodesArea - kWordsArea);
}

constexpr uint32_t kPThreads = 512;
constexpr uint32_t kPTok = 128;                  // tokens per tile (MMA M)
constexpr uint32_t kYStride = kPTok + 1u;        // y rows, one per coded component (odd stride)
constexpr int32_t kZeroTok = INT32_MIN;          // exponent of an all-zero token
constexpr uint32_t kChainList = 2048;            // chains per tile run by all threads; the rest by their word
constexpr double kDropUnits = 128.0 * 255.0 * 255.0 * (3.0 * 65536.0 + 2.0 * 256.0 + 1.0) + 96.0;

struct __align__(1024) PtSmem {
  uint8_t a[4][kQDigPlane];    // x digits of the tile (A operand): byte p of X, p = 0 the top byte
  uint8_t b[4][kQDigPlane];    // Q digits of the slice's coded columns (B operand)
  float y[kD * kYStride];      // y[cc][t]: fl32(S~), the exact y where a chain ran
  int32_t tok_e[kPTok];        // e_t, or kZeroTok
  float tok_x1[kPTok];         // x1 of the token (per-token ranges)
  int32_t kq_fmax;             // per-token ranges: the slice's largest coded column exponent
  float kq_q1max;              // and 1-norm bound
  int32_t blk_e[2][2];         // per tile parity and block: largest e_t (kZeroTok: all tokens zero)
  uint32_t blk_x1[2][2];       // largest x1 (bits of a non-negative float)
  uint32_t zero_tok[2][4];     // per 32-token word: tokens whose x is all zero
  uint32_t clist[kChainList];  // chains of the tile: token | coded component << 8
  uint32_t n_chain;
  uint32_t hist[kTabPool];     // symbol counts of the record per width stream
  uint32_t ccnt[8][kD];        // counts of symbols 0..7 per coded component
  uint32_t cidx[kD];           // coded component cc -> component j
  int32_t col_f[kD];
  float col_q1[kD];
  CompInfo ci;
  uint64_t bar;
  uint32_t tmem_base;
};
static_assert(sizeof(PtSmem) + 1024 <= 232448, "projection shared memory exceeds the per-block limit");

__device__ __forceinline__ double pow2d(int e) {  // 2^e, e clamped to the normal range
  e = max(-1022, min(1023, e));
  return __longlong_as_double(static_cast<long long>(1023 + e) << 52);
}

__device__ __forceinline__ float pow2f(int e) { return __int_as_float((127 + e) << 23); }  // -126 <= e <= 127

// The oracle's y of one token and component: xr the token's de-rotated x and
// qr = Q[0..127][j] (a row of the transposed basis), both fp32 in shared memory
// as 32 float4 chunks, chunk c stored at c ^ xs and c ^ qs: fp64 fused
// multiply-adds over k ascending (each fp32 x fp32 product is exact in fp64, so
// each step is the oracle's rounded addition), rounded to fp32 once.
__device__ __forceinline__ float exact_y_inl(const float4* xr, uint32_t xs, const float4* qr, uint32_t qs) {
  double acc = 0.0;
  float4 xn = xr[xs], qn = qr[qs];
#pragma unroll 4
  for (uint32_t c = 0; c < 32; ++c) {
    const float4 xv = xn, qv = qn;
    if (c + 1u < 32u) {
      xn = xr[(c + 1u) ^ xs];
      qn = qr[(c + 1u) ^ qs];
    }
    acc = fma(double(qv.x), double(xv.x), acc);
    acc = fma(double(qv.y), double(xv.y), acc);
    acc = fma(double(qv.z), double(xv.z), acc);
    acc = fma(double(qv.w), double(xv.w), acc);
  }
  return __double2float_rn(acc);
}
// the same as a call, for the rare paths
__device__ __noinline__ float exact_y(const float4* xr, uint32_t xs, const float4* qr, uint32_t qs) {
  return exact_y_inl(xr, xs, qr, qs);
}

__global__ void __launch_bounds__(kPThreads, 1)
k_transform_project(TransformShape sh, TransformPlanDev pl, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // the swizzled operand tiles need 1024-byte-aligned shared addresses
  const uint32_t pad = (1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u;
  PtSmem& S = *reinterpret_cast<PtSmem*>(smem_raw + pad);
  const uint32_t tid = threadIdx.x, warp = tid >> 5, lane = tid & 31u;
  const uint32_t rps = 1u + sh.n_mid;
  const uint32_t n_mid_total = (b.rec_base[b.n] / rps) * sh.n_mid;
  const uint32_t mbeg = uint32_t(uint64_t(blockIdx.x) * n_mid_total / gridDim.x);
  const uint32_t mend = uint32_t(uint64_t(blockIdx.x + 1u) * n_mid_total / gridDim.x);
  if (mbeg >= mend) return;
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, 512u);
    tc::tmem_relinquish();
  }
  if (tid == 0) tc::mbar_init(&S.bar, 1);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  uint32_t phase = 0;
  bool alive = true, drained = true;
  int32_t cur_slice = -1;
  // per-word roles: block blk2 of the tile, coded component wc, half hf
  const uint32_t blk2 = tid >> 8, wc = (tid >> 1) & 127u, hf = tid & 1u;
  // digit roles: token dt, channel quarter dg
  const uint32_t dt = tid >> 2, dg = tid & 3u;

  for (uint32_t m = mbeg; m < mend && alive; ++m) {
    const uint32_t gs = m / sh.n_mid, c = m % sh.n_mid;
    const uint32_t r = gs * rps + 1u + c;
    const uint32_t fr = frame_of(b.rec_base, b.n, r);
    const uint32_t ls = (r - b.rec_base[fr]) / rps;
    const uint16_t* src = reinterpret_cast<const uint16_t*>(b.f[fr].src);
    const uint32_t sidx = b.f[fr].first_slice + ls;
    const bool is_key = ((sidx / sh.H) & 1u) == 0;
    const bool kiv = sh.kivi && !is_key;  // values with per-token ranges
    const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
    const uint32_t nb = (tcc + kTile - 1) / kTile;
    const uint16_t* xs = src + uint64_t(ls) * sh.T * kD;
    uint8_t* rec = ws.slots + uint64_t(r) * ws.slot_bytes;
    uint8_t* codes = slot_codes(rec, ws.slot_bytes);

    if (int32_t(sidx) != cur_slice) {  // the slice's component order and Q digits
      cur_slice = int32_t(sidx);
      load_comp_info(pl.comp + sidx, S.ci);
      if (tid < kD) {
        if (S.ci.width[tid]) S.cidx[S.ci.coded_idx[tid]] = tid;
        S.col_f[tid] = pl.qcol[sidx].f[tid];
        S.col_q1[tid] = pl.qcol[sidx].q1[tid];
      }
      __syncthreads();
      if (tid < 32u) {  // the largest column exponent and 1-norm bound of the coded columns
        int32_t fm = kQColZero;
        float qm = 0.0f;
        for (uint32_t cc = tid; cc < S.ci.n_coded; cc += 32u) {
          fm = max(fm, S.col_f[cc]);
          qm = fmaxf(qm, S.col_q1[cc]);
        }
#pragma unroll
        for (uint32_t o = 16; o; o >>= 1) {
          fm = max(fm, __shfl_xor_sync(0xffffffffu, fm, o));
          qm = fmaxf(qm, __shfl_xor_sync(0xffffffffu, qm, o));
        }
        if (tid == 0) {
          S.kq_fmax = fm;
          S.kq_q1max = qm;
        }
      }
    }
    for (uint32_t i = tid; i < kTabPool; i += kPThreads) S.hist[i] = 0;
    for (uint32_t i = tid; i < 8u * kD; i += kPThreads) (&S.ccnt[0][0])[i] = 0;
    if (tid < 4u) {
      S.blk_e[tid >> 1][tid & 1u] = kZeroTok;
      S.blk_x1[tid >> 1][tid & 1u] = 0u;
    }
    if (tid < 8u) S.zero_tok[tid >> 2][tid & 3u] = 0u;
    if (tid == 0) S.n_chain = 0;
    const uint32_t nc = S.ci.n_coded;
    const uint32_t N = max(16u, (nc + 15u) & ~15u);
    {  // side-information padding of the record (its values are written below)
      const uint32_t side = nc ? 8u * (kiv ? tcc : nc * nb) : 0u;
      if (tid < pad16(side) - side) rec[side + tid] = 0;
    }
    __syncthreads();
    const bool wlive = wc < nc;
    const uint32_t wj = wlive ? S.cidx[wc] : 0u;
    const uint32_t levels = (1u << S.ci.width[wj]) - 1u;
    uint32_t cnt0 = 0u, cnt1 = 0u;  // counts of symbols 0..3 and 4..7 of this thread's codes, a byte each

    for (uint32_t tb = 0; tb < tcc && alive; tb += kPTok) {
      const uint32_t bl = min(kPTok, tcc - tb);
      const uint32_t par = (tb / kPTok) & 1u;
      if (tid < 2u) {  // the next tile's block statistics start empty
        S.blk_e[par ^ 1u][tid] = kZeroTok;
        S.blk_x1[par ^ 1u][tid] = 0u;
      } else if (tid < 6u) {
        S.zero_tok[par ^ 1u][tid - 2u] = 0u;
      }
      {  // the slice's Q digits (their space holds Q itself during the previous tile's chains)
        const char* g = reinterpret_cast<const char*>(pl.qdig + uint64_t(sidx) * kQDigBytes);
        const uint32_t d0 = tc::smem_addr(&S.b[0][0]);
#pragma unroll
        for (uint32_t u = 0; u < kQDigBytes / 16u / kPThreads; ++u) {
          const uint32_t i = tid + u * kPThreads;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d0 + 16u * i), "l"(g + 16u * i) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      // ---- digits of token dt, channels 16 dg .. + 15 and their partners
      float xa[16], xb[16];  // de-rotated x, kept for the chains (stored once the MMAs are done)
      {
        if (dt < bl) {
          const uint4* row = reinterpret_cast<const uint4*>(xs + uint64_t(t0 + tb + dt) * kD);
          const uint4 v[4] = {__ldg(row + 2u * dg), __ldg(row + 2u * dg + 1u), __ldg(row + 8u + 2u * dg),
                              __ldg(row + 8u + 2u * dg + 1u)};
#pragma unroll
          for (uint32_t h = 0; h < 2; ++h) {
            const uint32_t w[4] = {v[h].x, v[h].y, v[h].z, v[h].w}, u[4] = {v[2 + h].x, v[2 + h].y, v[2 + h].z, v[2 + h].w};
#pragma unroll
            for (uint32_t i = 0; i < 4; ++i) {
              xa[8 * h + 2 * i] = bf16_to_f32(w[i] & 0xffffu);
              xa[8 * h + 2 * i + 1] = bf16_to_f32(w[i] >> 16);
              xb[8 * h + 2 * i] = bf16_to_f32(u[i] & 0xffffu);
              xb[8 * h + 2 * i + 1] = bf16_to_f32(u[i] >> 16);
            }
          }
          if (is_key) {
            const float4* c4 = reinterpret_cast<const float4*>(pl.rope + (uint64_t(t0 + tb + dt) * (kD / 2) + 16u * dg) * 2u);
#pragma unroll
            for (uint32_t i = 0; i < 8; ++i) {
              const float4 k = __ldg(c4 + i);  // (cos, sin) of pairs 16 dg + 2i, + 2i + 1
              const float a0 = xa[2 * i], a1 = xa[2 * i + 1], b0 = xb[2 * i], b1 = xb[2 * i + 1];
              xa[2 * i] = __fadd_rn(__fmul_rn(a0, k.x), __fmul_rn(b0, k.y));
              xb[2 * i] = __fsub_rn(__fmul_rn(b0, k.x), __fmul_rn(a0, k.y));
              xa[2 * i + 1] = __fadd_rn(__fmul_rn(a1, k.z), __fmul_rn(b1, k.w));
              xb[2 * i + 1] = __fsub_rn(__fmul_rn(b1, k.z), __fmul_rn(a1, k.w));
            }
          }
        } else {
#pragma unroll
          for (uint32_t i = 0; i < 16; ++i) xa[i] = xb[i] = 0.0f;
        }
        float mx = 0.0f, x1 = 0.0f;
#pragma unroll
        for (uint32_t i = 0; i < 16; ++i) {
          mx = fmaxf(mx, fmaxf(fabsf(xa[i]), fabsf(xb[i])));
          x1 = __fadd_ru(x1, __fadd_ru(fabsf(xa[i]), fabsf(xb[i])));
        }
#pragma unroll
        for (uint32_t o = 1; o < 4; o <<= 1) {
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
          x1 = __fadd_ru(x1, __shfl_xor_sync(0xffffffffu, x1, o));
        }
        const int32_t e = mx > 0.0f ? ilogbf(mx) : kZeroTok;
        int32_t X[32];
        if (e == kZeroTok || e >= -98) {  // 2^(29 - e) is an fp32 number: x * 2^(29 - e) is exact
          const float sc = e == kZeroTok ? 0.0f : pow2f(29 - e);
#pragma unroll
          for (uint32_t i = 0; i < 16; ++i) {
            X[i] = __float2int_rn(__fmul_rn(xa[i], sc));
            X[16 + i] = __float2int_rn(__fmul_rn(xb[i], sc));
          }
        } else {  // tiny tokens
          const double sc = pow2d(29 - e);
#pragma unroll
          for (uint32_t i = 0; i < 16; ++i) {
            X[i] = __double2int_rn(double(xa[i]) * sc);
            X[16 + i] = __double2int_rn(double(xb[i]) * sc);
          }
        }
#pragma unroll
        for (uint32_t p = 0; p < 4; ++p) {
          const uint32_t sel = (3u - p) | ((7u - p) << 4);  // byte 3 - p of two words
#pragma unroll
          for (uint32_t h = 0; h < 2; ++h) {
            uint32_t wv[4];
#pragma unroll
            for (uint32_t q = 0; q < 4; ++q) {
              const int32_t* x4 = X + 16 * h + 4 * q;
              wv[q] = __byte_perm(__byte_perm(x4[0], x4[1], sel), __byte_perm(x4[2], x4[3], sel), 0x5410);
            }
            *reinterpret_cast<uint4*>(&S.a[p][0] + tc::sw128_offset(dt, 16u * (dg + 4u * h), kPTok)) =
                make_uint4(wv[0], wv[1], wv[2], wv[3]);
          }
        }
        if (dg == 0) {
          S.tok_e[dt] = e;
          S.tok_x1[dt] = x1;
          if (dt < bl) {
            if (e == kZeroTok) atomicOr(&S.zero_tok[par][dt >> 5], 1u << (dt & 31u));
            else {
              atomicMax(&S.blk_e[par][dt >> 6], e);
              atomicMax(&S.blk_x1[par][dt >> 6], __float_as_uint(x1));
            }
          }
        }
      }
      asm volatile("cp.async.wait_group 0;" ::: "memory");
      tc::fence_async_smem();
      tc::fence_before_sync();
      __syncthreads();
      // ---- ten digit pairs x four K-steps on the tensor cores
      if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t a0 = tc::smem_addr(&S.a[0][0]), b0 = tc::smem_addr(&S.b[0][0]);
#pragma unroll 1
        for (uint32_t ks = 0; ks < 4; ++ks) {
#pragma unroll
          for (uint32_t w = 0; w < 4; ++w) {
#pragma unroll
            for (uint32_t pa = 0; pa <= w; ++pa) {
              const uint32_t pb = w - pa;
              const uint64_t da = tc::desc_sw128(a0 + pa * kQDigPlane + ks * 32u);
              const uint64_t db = tc::desc_sw128(b0 + pb * kQDigPlane + ks * 32u);
              tc::mma_i8(tmem + w * N, da, db, tc::idesc_i8_s32(kPTok, N, pa == 0, pb == 0),
                         (ks > 0 || pa > 0) ? 1u : 0u);
            }
          }
        }
        tc::mma_commit(&S.bar);
      }
      // the issuing warp reconverges before it polls the barrier: a suspended poll
      // of its other lanes would otherwise hold back the issue
      __syncwarp();
      {  // while the MMAs run: the next 128 tokens' rows (and keys' cos/sin) toward L2
        const uint32_t tn = t0 + tb + kPTok + dt;
        if (tn < sh.r_start) {
          const char* pr = dg < 2u ? reinterpret_cast<const char*>(xs + uint64_t(tn) * kD) + 128u * dg
                                   : reinterpret_cast<const char*>(pl.rope + uint64_t(tn) * kD) + 256u * (dg - 2u);
          if (dg < 2u || is_key) {
            asm volatile("prefetch.global.L2 [%0];" ::"l"(pr));
            if (dg >= 2u) asm volatile("prefetch.global.L2 [%0];" ::"l"(pr + 128));
          }
        }
      }
      const bool done = tc::mbar_wait(&S.bar, phase, KVC_MMA_WAIT_POLLS);
      phase ^= 1u;
      if (!__syncthreads_and(done)) {
        // drain: the same completion again, with the long bound, so that the
        // accumulator is no longer written when the block frees it
        drained = __syncthreads_and(tc::mbar_wait(&S.bar, phase ^ 1u, kMmaDrainPolls));
        alive = false;
        break;
      }
      tc::fence_after_sync();
      {  // the Q digits are consumed: their space holds the coded rows of Q^T for the chains
        const char* g = reinterpret_cast<const char*>(pl.qt + uint64_t(sidx) * kD * kD);
        const uint32_t d0 = tc::smem_addr(&S.b[0][0]);
        for (uint32_t i = tid; i < nc * 32u; i += kPThreads) {
          const uint32_t cc = i >> 5, ch = i & 31u;
          asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(d0 + 512u * cc + 16u * (ch ^ (cc & 7u))),
                       "l"(g + 512u * S.cidx[cc] + 16u * ch) : "memory");
        }
        asm volatile("cp.async.commit_group;" ::: "memory");
      }
      {  // the x digits are consumed: their space holds x as fp32 rows for the chains
        float4* xp = reinterpret_cast<float4*>(&S.a[0][0]) + dt * 32u;
        const uint32_t sw = dt & 7u;
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
          xp[(4u * dg + i) ^ sw] = make_float4(xa[4 * i], xa[4 * i + 1], xa[4 * i + 2], xa[4 * i + 3]);
          xp[(16u + 4u * dg + i) ^ sw] = make_float4(xb[4 * i], xb[4 * i + 1], xb[4 * i + 2], xb[4 * i + 3]);
        }
      }
      // ---- epilogue: the estimates y~ = fl32(S~)
      {
        const uint32_t g4 = warp & 3u, tt = 32u * g4 + lane;
        const int32_t et = S.tok_e[tt];
        const bool tv = tt < bl;
        for (uint32_t cch = warp >> 2; cch < N / 16u; cch += 4u) {
          uint32_t p[4][16];
#pragma unroll
          for (uint32_t w = 0; w < 4; ++w) tc::tmem_ld16(tmem + ((32u * g4) << 16) + w * N + 16u * cch, p[w]);
          tc::tmem_wait_ld();
#pragma unroll
          for (uint32_t i = 0; i < 16; ++i) {
            const uint32_t cc = 16u * cch + i;
            if (tv && cc < nc) {
              // integers to fp32 by the magic constant 1.5 * 2^23 (exact below 2^22 in
              // magnitude: |P0| <= 2^19, |P1| < 2^22); P2 and P3 (below 2^24 and 2^25)
              // rounded down to multiples of 4 and 8 first; the levels combined with
              // fused multiply-adds: within 2^-22 |V~| + 2^11 of V
              const float f0 = __int_as_float(0x4b400000 + int32_t(p[0][i])) - 12582912.0f;
              const float f1 = __int_as_float(0x4b400000 + int32_t(p[1][i])) - 12582912.0f;
              const float f2 = (__int_as_float(0x4b400000 + (int32_t(p[2][i]) >> 2)) - 12582912.0f) * 4.0f;
              const float f3 = (__int_as_float(0x4b400000 + (int32_t(p[3][i]) >> 3)) - 12582912.0f) * 8.0f;
              const float v = __fmaf_rn(__fmaf_rn(__fmaf_rn(f0, 256.0f, f1), 256.0f, f2), 256.0f, f3);
              float yv = 0.0f;
              if (et != kZeroTok) {
                const int k = et + S.col_f[cc] - 34;
                yv = k >= -126 ? __fmul_rn(v, pow2f(min(k, 127))) : __fmul_rn(__fmul_rn(v, pow2f(k + 64)), 0x1p-64f);
              }
              S.y[cc * kYStride + tt] = yv;
            }
          }
        }
      }
      tc::fence_before_sync();
      __syncthreads();
      if (!kiv) {
      // ---- per word: bound, candidates, chains, zero point and scale, codes
      {
        const uint32_t w0 = blk2 * 64u + hf * 32u;  // first token of the word in the tile
        const uint32_t nv = bl > w0 ? min(32u, bl - w0) : 0u;
        const bool live = wlive && blk2 * 64u < bl;
        float* yr = S.y + wc * kYStride + w0;
        const int32_t em = S.blk_e[par][blk2];
        const float xm = __uint_as_float(S.blk_x1[par][blk2]);
        const uint32_t zmask = S.zero_tok[par][blk2 * 2u + hf];
        float mn = __int_as_float(0x7f800000), mx = __int_as_float(0xff800000);
        for (uint32_t i = 0; i < nv; ++i) {
          const float v = yr[i];
          mn = fminf(mn, v);
          mx = fmaxf(mx, v);
        }
        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
        const int32_t f = S.col_f[wc];
        const bool all_exact = em == kZeroTok || f == kQColZero;
        float R = 0.0f;
        uint32_t exact = zmask, cand = 0;
        const uint32_t vmask = nv == 32u ? 0xffffffffu : (1u << nv) - 1u;
        if (live) {
          if (all_exact) {
            exact = vmask;
          } else {
            double E = pow2d(em + f - 58) * kDropUnits + double(xm) * (pow2d(f - 30) + pow2d(f - 45)) +
                       double(S.col_q1[wc]) * pow2d(em - 30);
            // the estimates are within dl of S~ (fp32 combination of the levels)
            const double Ma = double(fmaxf(fabsf(mn), fabsf(mx)));
            const double dl = Ma * 0x1p-21 + pow2d(em + f - 22) + 0x1p-148;
            E *= 1.0 + 0x1p-40;
            const double M = Ma * (1.0 + 0x1p-21) + E + dl;
            const int lm = M > 0.0 ? ilogb(M) : -1000;
            R = __double2float_ru((E + dl + pow2d(max(lm - 23, -149))) * (1.0 + 0x1p-40));
            const float two = __fmul_ru(R, 2.0f);
            const float lo_thr = __fadd_ru(mn, two), hi_thr = __fsub_rd(mx, two);
            for (uint32_t i = 0; i < nv; ++i) {
              const float v = yr[i];
              if (v <= lo_thr || v >= hi_thr) cand |= 1u << i;
            }
            cand &= ~zmask;
          }
        }
        const float4* xp = reinterpret_cast<const float4*>(&S.a[0][0]) + w0 * 32u;
        const float4* qr = reinterpret_cast<const float4*>(&S.b[0][0]) + wc * 32u;
        {  // the candidates go to the tile's list; what does not fit stays with the word.
           // Every slot below min(n_chain, kChainList) is written by the thread that
           // reserved it, so the list holds no stale entry.
          const uint32_t n = __popc(cand);
          if (n) {
            const uint32_t base = atomicAdd(&S.n_chain, n);
            const uint32_t fit = base < kChainList ? min(n, kChainList - base) : 0u;
            for (uint32_t u = 0; u < fit; ++u) {
              const uint32_t i = __ffs(cand) - 1u;
              cand &= cand - 1u;
              S.clist[base + u] = (w0 + i) | (wc << 8);
              exact |= 1u << i;
            }
          }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");  // Q^T rows landed
        __syncthreads();
        {  // the listed chains, spread over all threads
          const uint32_t nl = min(S.n_chain, kChainList);
          for (uint32_t u = tid; u < nl; u += kPThreads) {
            const uint32_t e = S.clist[u], t = e & 0xffu, cc = e >> 8;
            S.y[cc * kYStride + t] = exact_y_inl(reinterpret_cast<const float4*>(&S.a[0][0]) + t * 32u, t & 7u,
                                                 reinterpret_cast<const float4*>(&S.b[0][0]) + cc * 32u, cc & 7u);
          }
        }
        __syncthreads();
        if (tid == 0) S.n_chain = 0;  // for the next tile (read again only after two barriers)
        while (cand) {  // chains that did not fit the list
          const uint32_t i = __ffs(cand) - 1u;
          cand &= cand - 1u;
          yr[i] = exact_y(xp + i * 32u, (w0 + i) & 7u, qr, wc & 7u);
          exact |= 1u << i;
        }
        // the oracle's scan over the block: exact values where they decide
        float z = __int_as_float(0x7f800000), zx = __int_as_float(0xff800000);
        for (uint32_t i = 0; i < nv; ++i) {
          const float v = yr[i];
          if (v < z) z = v;
          if (v > zx) zx = v;
        }
        {  // lower half first: the upper half's value wins only when strictly beyond
          const float pz = __shfl_xor_sync(0xffffffffu, z, 1), pzx = __shfl_xor_sync(0xffffffffu, zx, 1);
          if (hf == 0) {
            if (pz < z) z = pz;
            if (pzx > zx) zx = pzx;
          } else {
            z = z < pz ? z : pz;
            zx = zx > pzx ? zx : pzx;
          }
        }
        if (live) {
          const float s = (zx == z) ? 0.0f : __fdiv_rn(__fsub_rn(zx, z), float(levels));
          const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
          const bool exact_rs = !(rs < 0x1p126f);
          if (hf == 0) {
            uint32_t* zp = reinterpret_cast<uint32_t*>(rec + 8u * (wc * nb + tb / kTile + blk2));
            zp[0] = __float_as_uint(z);
            zp[1] = __float_as_uint(s);
          }
          // Codes. With qa = RN(RN(y~ - z) * RN(1/s)), the oracle's quotient for any y
          // in [y~ - R, y~ + R] is within R/s (1 + 2^-21) + |qa| 2^-21 of qa (R = 0
          // where y~ is exact); decisions change only at half-integers, so a larger
          // distance to the nearest one settles the code (rint by the magic
          // constant 1.5 * 2^23: |qa| is small). The rest is settled after the pass.
          const float mR = __fmul_ru(__fmul_ru(R, rs), 1.0f + 0x1p-19f);
          // symbols 0..7 in the packed counters, the rest (widths >= 4) by atomics
          auto count_code = [&](uint32_t q, int32_t sign = 1) {
            const uint32_t inc = uint32_t(sign) << (8u * (q & 3u));
            if (q < 4u) cnt0 += inc;
            else if (q < 8u) cnt1 += inc;
            else atomicAdd(&S.hist[levels - 1u + q], uint32_t(sign));  // tab_base(b) = 2^b - 2 = levels - 1
          };
          uint32_t word[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
          uint32_t unc = 0;
#pragma unroll
          for (uint32_t i = 0; i < 32; ++i) {
            const float v = yr[i];
            const float qa = __fmul_rn(__fsub_rn(v, z), rs);
            const float mg = __fadd_rn(qa, 12582912.0f);
            const int32_t iq = __float_as_int(mg) - 0x4b400000;
            const float d = __fsub_rn(0.5f, fabsf(__fsub_rn(qa, __fsub_rn(mg, 12582912.0f))));
            const float m = __fadd_ru(((exact >> i) & 1u) ? 0.0f : mR, __fmul_ru(fabsf(qa), 0x1p-19f));
            const uint32_t q = uint32_t(min(max(iq, 0), int32_t(levels)));
            word[i >> 2] |= q << (8u * (i & 3u));
            if (!(d > m)) unc |= 1u << i;
            if (i < nv) count_code(q);
          }
          unc = exact_rs ? vmask : (unc & vmask);
          while (unc) {  // the IEEE quotient at both ends, else the chain decides
            const uint32_t i = __ffs(unc) - 1u;
            unc &= unc - 1u;
            const float v = yr[i];
            uint32_t q;
            if ((exact >> i) & 1u) {
              q = quantize(v, z, s, levels);
            } else {
              const uint32_t q1 = quantize(__fsub_rd(v, R), z, s, levels);
              const uint32_t q2 = quantize(__fadd_ru(v, R), z, s, levels);
              q = q1 == q2 ? q1 : quantize(exact_y(xp + i * 32u, (w0 + i) & 7u, qr, wc & 7u), z, s, levels);
            }
            const uint32_t sh = 8u * (i & 3u);
#pragma unroll
            for (uint32_t j = 0; j < 8; ++j) {
              if (j == (i >> 2)) {
                const uint32_t old = (word[j] >> sh) & 0xffu;
                if (old != q) {
                  count_code(old, -1);
                  count_code(q);
                }
                word[j] = (word[j] & ~(0xffu << sh)) | (q << sh);
              }
            }
          }
#pragma unroll
          for (uint32_t j = 0; j < 8; ++j) {  // tokens past the tile's end code as 0
            const uint32_t vb = nv > 4u * j ? min(4u, nv - 4u * j) : 0u;
            if (vb < 4u) word[j] &= (1u << (8u * vb)) - 1u;
          }
          uint4* cd = reinterpret_cast<uint4*>(codes + uint64_t(wj) * kCodesRow + tb + w0);
          cd[0] = make_uint4(word[0], word[1], word[2], word[3]);
          cd[1] = make_uint4(word[4], word[5], word[6], word[7]);
        }
      }
      } else {
      // ---- values with per-token ranges (KIVI-style): thread t = tid / 4 takes
      // quarter q = tid % 4 of the coded components of token t; the four
      // quarters of a token are neighbouring lanes
      {
        const uint32_t t = tid >> 2, q = tid & 3u, nq = (nc + 3u) >> 2;
        const uint32_t c0 = min(nc, q * nq), c1 = min(nc, c0 + nq);
        const bool tv = t < bl;
        const int32_t et = S.tok_e[t];
        float mn = __int_as_float(0x7f800000), mx = __int_as_float(0xff800000);
        for (uint32_t cc = c0; cc < c1; ++cc) {
          const float v = S.y[cc * kYStride + t];
          mn = fminf(mn, v);
          mx = fmaxf(mx, v);
        }
#pragma unroll
        for (uint32_t o = 1; o < 4; o <<= 1) {
          mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, o));
          mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, o));
        }
        const uint32_t qmask = (c1 - c0) == 32u ? 0xffffffffu : (1u << (c1 - c0)) - 1u;
        uint32_t exact = 0, cand = 0;
        float R = 0.0f;
        if (tv && nc) {
          if (et == kZeroTok || S.kq_fmax == kQColZero) {
            exact = qmask;  // an all-zero token (or basis): every y is +0
          } else {
            // the bound at the slice's largest column exponent and 1-norm bound
            const int32_t f = S.kq_fmax;
            double E = pow2d(et + f - 58) * kDropUnits + double(S.tok_x1[t]) * (pow2d(f - 30) + pow2d(f - 45)) +
                       double(S.kq_q1max) * pow2d(et - 30);
            const double Ma = double(fmaxf(fabsf(mn), fabsf(mx)));
            const double dl = Ma * 0x1p-21 + pow2d(et + f - 22) + 0x1p-148;
            E *= 1.0 + 0x1p-40;
            const double M = Ma * (1.0 + 0x1p-21) + E + dl;
            const int lm = M > 0.0 ? ilogb(M) : -1000;
            R = __double2float_ru((E + dl + pow2d(max(lm - 23, -149))) * (1.0 + 0x1p-40));
            const float two = __fmul_ru(R, 2.0f);
            const float lo_thr = __fadd_ru(mn, two), hi_thr = __fsub_rd(mx, two);
            for (uint32_t cc = c0; cc < c1; ++cc) {
              const float v = S.y[cc * kYStride + t];
              if (v <= lo_thr || v >= hi_thr) cand |= 1u << (cc - c0);
            }
          }
        }
        {  // the candidates go to the tile's list (see the block path)
          const uint32_t n = __popc(cand);
          if (n) {
            const uint32_t base = atomicAdd(&S.n_chain, n);
            const uint32_t fit = base < kChainList ? min(n, kChainList - base) : 0u;
            for (uint32_t u = 0; u < fit; ++u) {
              const uint32_t i = __ffs(cand) - 1u;
              cand &= cand - 1u;
              S.clist[base + u] = t | ((c0 + i) << 8);
              exact |= 1u << i;
            }
          }
        }
        asm volatile("cp.async.wait_group 0;" ::: "memory");  // Q^T rows landed
        __syncthreads();
        {  // the listed chains, spread over all threads
          const uint32_t nl = min(S.n_chain, kChainList);
          for (uint32_t u = tid; u < nl; u += kPThreads) {
            const uint32_t e = S.clist[u], tt = e & 0xffu, cc = e >> 8;
            S.y[cc * kYStride + tt] = exact_y_inl(reinterpret_cast<const float4*>(&S.a[0][0]) + tt * 32u, tt & 7u,
                                                  reinterpret_cast<const float4*>(&S.b[0][0]) + cc * 32u, cc & 7u);
          }
        }
        __syncthreads();
        if (tid == 0) S.n_chain = 0;  // for the next tile (read again only after two barriers)
        const float4* xp = reinterpret_cast<const float4*>(&S.a[0][0]) + t * 32u;
        while (cand) {  // chains that did not fit the list
          const uint32_t i = __ffs(cand) - 1u;
          cand &= cand - 1u;
          const uint32_t cc = c0 + i;
          S.y[cc * kYStride + t] =
              exact_y(xp, t & 7u, reinterpret_cast<const float4*>(&S.b[0][0]) + cc * 32u, cc & 7u);
          exact |= 1u << i;
        }
        // the oracle's scan over the token's coded components, ascending
        float z = __int_as_float(0x7f800000), zx = __int_as_float(0xff800000);
        for (uint32_t cc = c0; cc < c1; ++cc) {
          const float v = S.y[cc * kYStride + t];
          if (v < z) z = v;
          if (v > zx) zx = v;
        }
#pragma unroll
        for (uint32_t o = 1; o < 4; o <<= 1) {  // lower quarters first
          const float pz = __shfl_xor_sync(0xffffffffu, z, o), pzx = __shfl_xor_sync(0xffffffffu, zx, o);
          if ((q & o) == 0) {
            if (pz < z) z = pz;
            if (pzx > zx) zx = pzx;
          } else {
            z = z < pz ? z : pz;
            zx = zx > pzx ? zx : pzx;
          }
        }
        if (tv && nc) {
          const float rng = __fsub_rn(zx, z);
          if (q == 0) {
            uint32_t* zp = reinterpret_cast<uint32_t*>(rec + 8u * (tb + t));
            zp[0] = __float_as_uint(z);
            zp[1] = __float_as_uint(zx == z ? 0.0f : rng);
          }
          for (uint32_t cc = c0; cc < c1; ++cc) {
            const uint32_t i = cc - c0, j = S.cidx[cc], bw = S.ci.width[j], levels = (1u << bw) - 1u;
            const float s = (zx == z) ? 0.0f : __fdiv_rn(rng, float(levels));
            const float rs = s == 0.0f ? 0.0f : __frcp_rn(s);
            const bool exact_rs = !(rs < 0x1p126f);
            const float v = S.y[cc * kYStride + t];
            uint32_t qv;
            bool done = false;
            if (!exact_rs) {  // the distance test of the block path, at this token's bound
              const float qa = __fmul_rn(__fsub_rn(v, z), rs);
              const float mg = __fadd_rn(qa, 12582912.0f);
              const int32_t iq = __float_as_int(mg) - 0x4b400000;
              const float d = __fsub_rn(0.5f, fabsf(__fsub_rn(qa, __fsub_rn(mg, 12582912.0f))));
              const float mR = ((exact >> i) & 1u) ? 0.0f : __fmul_ru(__fmul_ru(R, rs), 1.0f + 0x1p-19f);
              if (d > __fadd_ru(mR, __fmul_ru(fabsf(qa), 0x1p-19f))) {
                qv = uint32_t(min(max(iq, 0), int32_t(levels)));
                done = true;
              }
            }
            if (!done) {
              if ((exact >> i) & 1u) {
                qv = quantize(v, z, s, levels);
              } else {
                const uint32_t q1 = quantize(__fsub_rd(v, R), z, s, levels);
                const uint32_t q2 = quantize(__fadd_ru(v, R), z, s, levels);
                qv = q1 == q2 ? q1
                              : quantize(exact_y(xp, t & 7u, reinterpret_cast<const float4*>(&S.b[0][0]) + cc * 32u,
                                                 cc & 7u),
                                         z, s, levels);
              }
            }
            codes[uint64_t(j) * kCodesRow + tb + t] = uint8_t(qv);
            atomicAdd(&S.hist[levels - 1u + qv], 1u);  // tab_base(b) = 2^b - 2 = levels - 1
          }
        }
      }
      }
      __syncthreads();  // y and the token arrays are rewritten by the next tile
    }
    if (!alive) break;
    if (wlive) {
#pragma unroll
      for (uint32_t q = 0; q < 8; ++q) {
        const uint32_t n = ((q < 4u ? cnt0 : cnt1) >> (8u * (q & 3u))) & 0xffu;
        if (n) atomicAdd(&S.ccnt[q][wc], n);
      }
    }
    __syncthreads();
    // counts of symbols 0..7 summed over the components of each width
    if (tid < 64u) {
      const uint32_t bw = (tid >> 3) + 1u, q = tid & 7u;
      if (q < (1u << bw)) {
        uint32_t sum = 0;
        for (uint32_t cc = 0; cc < nc; ++cc)
          if (S.ci.width[S.cidx[cc]] == bw) sum += S.ccnt[q][cc];
        S.hist[tab_base(bw) + q] += sum;
      }
    }
    __syncthreads();
    for (uint32_t i = tid; i < kTabPool; i += kPThreads)
      reinterpret_cast<uint32_t*>(codes + kHistOffset)[i] = S.hist[i];
  }
  if (!alive) {  // this block's records from the one that timed out on are marked failed
    for (uint32_t m = mbeg; m < mend; ++m) {
      const uint32_t r = (m / sh.n_mid) * rps + 1u + m % sh.n_mid;
      uint8_t* codes = slot_codes(ws.slots + uint64_t(r) * ws.slot_bytes, ws.slot_bytes);
      if (tid == 0) reinterpret_cast<uint32_t*>(codes + kHistOffset)[kTabPool - 1u] = kHistTimeout;
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  // MMAs still pending after the drain's bound would write tensor memory
  // after it is freed (and handed to another block): the block then keeps its
  // allocation, and its records already carry the timeout status
  if (warp == 0 && drained) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, 512u);
  }
}

// ---------------------------------------------------------------------------
// Transform encode, part 1b (k_transform_side): one CTA per middle record. The
// projection leaves the record's side information raw at the start of the
// slot's record area: (z, s) of coded component cc and block blk at 8 (cc nb +
// blk). It becomes the sequence V = every z, then every s (components and
// blocks in order), and V's four byte planes become four stream records, the
// lane-delta candidate included (the rule of the lossless high plane: CONST
// for one symbol; the lane deltas' RANS record if strictly smaller than both
// the plain RANS record and RAW; else plain RANS if smaller than RAW; else
// RAW). Side streams take one lane per 64 symbols, at most 32 (one group), so
// a lane's chain is at most 127 steps. Warp v owns variant v (plane v / 2,
// its lane deltas when v is odd): histogram, then a bound on its RANS record
// from the empirical entropy; only a variant that could beat RAW is
// normalised and coded. The streams replace the raw values, and their total
// length goes to rec_len, where the entropy kernel finds the offset of its
// code streams.
constexpr uint32_t kSideMax = 2u * kD * (kMaxCt / kTile);  // values of V at most

__host__ __device__ inline uint32_t side_lanes(uint32_t n) {
  const uint32_t N = n / 64u;
  return N < 1u ? 1u : (N > kGroupLanes ? kGroupLanes : N);
}
// Bytes of a side stream's RANS record: header, bitmap, k frequencies, one
// group length, the N states and W words.
__host__ __device__ inline uint32_t side_rans_bytes(uint32_t k, uint32_t N, uint32_t W) {
  return 48u + pad16(2u * k) + 16u + pad16(4u * N + 2u * W);
}

struct __align__(16) SideSmem {
  uint8_t sym[4][kSideMax];   // byte plane q of V
  uint32_t hist[8][256];      // counts of variant v; its frequencies once normalised
  uint32_t rem[8][256];       // normalisation scratch
  uint2 tab[8][256];          // coding table of variant v: {f | cum << 16, floor((2^32 - 1) / f)}
  uint32_t states[8][kGroupLanes];
  uint32_t W[8], k[8], ran[8];
  uint32_t mode[4], bytes[4], var[4], off[5];
};
static_assert(sizeof(SideSmem) <= 232448 / 5, "side kernel should fit five blocks per SM");

// rANS chain of one side-stream variant by one warp (lanes l < N <= 32): lane
// l codes its range of plane sy (the lane deltas when delta), last symbol
// first, with the symbol and table entry of the next two steps fetched ahead.
// Words go backwards into words[0, cap); returns their count.
__device__ inline uint32_t side_chain(const uint8_t* sy, bool delta, uint32_t n, uint32_t N, const uint2* tab,
                                      uint16_t* words, uint32_t cap, uint32_t* x_out) {
  const uint32_t lane = threadIdx.x & 31u;
  const bool live = lane < N;
  uint32_t start = 0, len = 0, start0, maxlen;
  if (live) lane_range(n, N, lane, start, len);
  lane_range(n, N, 0u, start0, maxlen);
  auto sym_at = [&](int t) -> uint32_t {  // symbol of step t, 0 where the lane has none
    if (!live || t < 0 || uint32_t(t) >= len) return 0u;
    const uint32_t a = sy[start + t];
    return (delta && t > 0) ? (a ^ sy[start + t - 1]) : a;
  };
  uint32_t x = kRansLow, pos = cap;
  const uint32_t lt = lanemask_lt();
  uint2 e_next = tab[sym_at(int(maxlen) - 1)];
  uint32_t s_next = sym_at(int(maxlen) - 2);
#pragma unroll 1
  for (int tau = int(maxlen) - 1; tau >= 0; --tau) {
    const bool act = live && uint32_t(tau) < len;
    const uint2 e = e_next;
    e_next = tab[s_next];
    s_next = sym_at(tau - 2);
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
    x = act ? (q << kProbBits) + r + cum : x;
  }
  *x_out = x;
  return cap - pos;
}

// One side stream record at dst (global, 16-byte aligned), written by one warp
// with every padding byte zero: RAW (the plane), CONST (its one symbol) or RANS
// (frequencies freq[256], one group: N states, then W words).
__device__ inline void warp_write_side(uint8_t* dst, uint32_t mode, uint32_t bytes, uint32_t n, uint32_t k,
                                       const uint8_t* sy, const uint32_t* freq, const uint32_t* states,
                                       const uint16_t* words, uint32_t W, uint32_t N, uint32_t delta) {
  const uint32_t lane = threadIdx.x & 31u;
  for (uint32_t i = lane; i < bytes / 16u; i += 32u) reinterpret_cast<uint4*>(dst)[i] = make_uint4(0, 0, 0, 0);
  __syncwarp();
  if (mode == kModeConst) {
    if (lane == 0) *reinterpret_cast<uint4*>(dst) = make_uint4(kModeConst | (uint32_t(sy[0]) << 8), 16u, n, 1u);
    return;
  }
  if (mode == kModeRaw) {
    if (lane == 0) *reinterpret_cast<uint4*>(dst) = make_uint4(kModeRaw, bytes, n, 0u);
    for (uint32_t i = lane; i < n; i += 32u) dst[16u + i] = sy[i];
    return;
  }
  if (lane == 0) *reinterpret_cast<uint4*>(dst) = make_uint4(kModeRans | (1u << 16) | (delta << 24), bytes, n, k);
#pragma unroll
  for (uint32_t w = 0; w < 8; ++w) {
    const uint32_t bits = __ballot_sync(0xffffffffu, freq[32u * w + lane] != 0u);
    if (lane == 0) reinterpret_cast<uint32_t*>(dst + 16)[w] = bits;
  }
  uint32_t f[8], cnt = 0;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    f[i] = freq[8u * lane + i];
    cnt += f[i] ? 1u : 0u;
  }
  uint32_t incl = cnt;
#pragma unroll
  for (uint32_t o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t idx = incl - cnt;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i)
    if (f[i]) st_u16(dst + 48u + 2u * idx++, f[i]);
  const uint32_t lens_at = pad16(48u + 2u * k), sub = lens_at + 16u;
  if (lane == 0) *reinterpret_cast<uint32_t*>(dst + lens_at) = 4u * N + 2u * W;
  if (lane < N) reinterpret_cast<uint32_t*>(dst + sub)[lane] = states[lane];
  uint16_t* w16 = reinterpret_cast<uint16_t*>(dst + sub + 4u * N);
  for (uint32_t i = lane; i < W; i += 32u) w16[i] = words[i];
}

__global__ void __launch_bounds__(kThreads)
k_transform_side(TransformShape sh, TransformPlanDev pl, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  SideSmem& S = *reinterpret_cast<SideSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t warp = tid >> 5, lane = tid & 31u;
  const uint32_t rps = 1u + sh.n_mid;
  const uint32_t gs = blockIdx.x / sh.n_mid, c = blockIdx.x % sh.n_mid;
  const uint32_t r = gs * rps + 1u + c;
  const uint32_t fr = frame_of(b.rec_base, b.n, r);
  const uint32_t ls = (r - b.rec_base[fr]) / rps;
  const uint32_t sidx = b.f[fr].first_slice + ls;
  const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
  const uint32_t nb = (tcc + kTile - 1) / kTile;
  uint8_t* rec = ws.slots + uint64_t(r) * ws.slot_bytes;
  uint16_t* scratch = slot_words(rec, ws.slot_bytes);  // variant v's words end at (v + 1) * kSideMax
  // pairs of the record: one per coded component and block, or one per token
  // for values with per-token ranges
  const uint32_t n_coded = __ldg(&pl.comp[sidx].n_coded);
  const bool kiv = sh.kivi && ((sidx / sh.H) & 1u) == 1u;
  const uint32_t half = n_coded ? (kiv ? tcc : n_coded * nb) : 0u, n = 2u * half;
  if (n == 0) {  // nothing coded: no side streams
    if (tid == 0) ws.rec_len[r] = 0;
    return;
  }
  for (uint32_t i = tid; i < 8u * 256u; i += nthr) (&S.hist[0][0])[i] = 0;
  for (uint32_t i = tid; i < half; i += nthr) {
    const uint2 v = *reinterpret_cast<const uint2*>(rec + 8u * i);  // (z, s) of pair i
#pragma unroll
    for (uint32_t q = 0; q < 4; ++q) {
      S.sym[q][i] = uint8_t(v.x >> (8u * q));
      S.sym[q][half + i] = uint8_t(v.y >> (8u * q));
    }
  }
  __syncthreads();  // the raw values are in shared memory; the records may overwrite them
  const uint32_t N = side_lanes(n), raw_b = 16u + pad16(n);
  {
    const uint32_t v = warp, q = v >> 1;
    const bool delta = (v & 1u) != 0;
    const uint8_t* sy = S.sym[q];
    uint32_t* h = S.hist[v];
    // histogram: lanes holding the same symbol add once
    const uint32_t base = n / N, extra = n - base * N, big = extra * (base + 1u);
    for (uint32_t i0 = 0; i0 < n; i0 += 32u) {
      const uint32_t i = i0 + lane;
      uint32_t s = 256u + lane;  // past the end: a key no other lane holds
      if (i < n) {
        s = sy[i];
        if (delta) {
          const bool first = i < big ? (i % (base + 1u)) == 0u : ((i - big) % base) == 0u;
          if (!first) s ^= sy[i - 1];
        }
      }
      const uint32_t same = __match_any_sync(0xffffffffu, s);
      if (s < 256u && lane == uint32_t(__ffs(same) - 1)) atomicAdd(&h[s], uint32_t(__popc(same)));
    }
    __syncwarp();
    // Could its RANS record be smaller than RAW? Every coding step adds at least
    // log2(M / f_s) - log2(16/15) bits to the state and every word at most
    // 16 + log2(16/15), the final states hold at most 32 - 16 bits each beyond
    // their start, and sum_s c_s log2(M / f_s) >= n H for the empirical entropy
    // H (Gibbs), so W >= (n H - n log2(16/15) - 16 N) / (16 + log2(16/15)).
    uint32_t present = 0;
    float bits = 0.0f;
    const float lgn = log2f(float(n));
    for (uint32_t s = lane; s < 256u; s += 32u) {
      const uint32_t cs = h[s];
      if (cs) {
        ++present;
        bits += float(cs) * (lgn - log2f(float(cs)));
      }
    }
    const uint32_t k = __reduce_add_sync(0xffffffffu, present);
#pragma unroll
    for (uint32_t o = 16; o; o >>= 1) bits += __shfl_xor_sync(0xffffffffu, bits, o);
    const float slack = 0.0932f;  // > log2(16/15)
    const float w_lb = (bits * 0.9999f - 2.0f - slack * float(n) - 16.0f * float(N)) / (16.0f + slack);
    const float rec_lb = float(48u + pad16(2u * k) + 16u + 4u * N) + 2.0f * fmaxf(w_lb, 0.0f);
    const bool run = k >= 2 && rec_lb < float(raw_b);
    if (lane == 0) {
      S.k[v] = k;
      S.ran[v] = run ? 1u : 0u;
    }
    if (run) {
      warp_normalize(h, 256u, n, h, S.rem[v], S.tab[v]);  // frequencies replace the counts
      uint32_t x;
      const uint32_t Wv = side_chain(sy, delta, n, N, S.tab[v], scratch + v * kSideMax, kSideMax, &x);
      if (lane < N) S.states[v][lane] = x;
      if (lane == 0) S.W[v] = Wv;
    }
  }
  __syncthreads();
  if (tid == 0) {  // per plane: CONST; lane-delta RANS if strictly smaller than plain RANS and RAW; RANS; RAW
    uint32_t off = 0;
    for (uint32_t q = 0; q < 4; ++q) {
      const uint32_t vp = 2u * q, vd = vp + 1u;
      uint32_t mode = kModeRaw, bytes = raw_b, var = vp;
      if (S.k[vp] == 1) {
        mode = kModeConst;
        bytes = 16;
      } else {
        const uint32_t rb = S.ran[vp] ? side_rans_bytes(S.k[vp], N, S.W[vp]) : 0xffffffffu;
        const uint32_t rd = S.ran[vd] ? side_rans_bytes(S.k[vd], N, S.W[vd]) : 0xffffffffu;
        if (rd < rb && rd < raw_b) {
          mode = kModeRans; bytes = rd; var = vd;
        } else if (rb < raw_b) {
          mode = kModeRans; bytes = rb;
        }
      }
      S.mode[q] = mode; S.bytes[q] = bytes; S.var[q] = var; S.off[q] = off;
      off += bytes;
    }
    S.off[4] = off;
  }
  __syncthreads();
  if (warp < 4) {
    const uint32_t q = warp, v = S.var[q];
    const uint32_t Wv = S.mode[q] == kModeRans ? S.W[v] : 0u;
    warp_write_side(rec + S.off[q], S.mode[q], S.bytes[q], n, S.k[v], S.sym[q], S.hist[v], S.states[v],
                    scratch + (v + 1u) * kSideMax - Wv, Wv, N, v & 1u);
  }
  if (tid == 0) ws.rec_len[r] = S.off[4];
}

// ---------------------------------------------------------------------------
// Transform encode, part 2 (k_transform_entropy): one CTA per middle record,
// several per SM (no codes in shared memory). Warp w owns the stream of width
// b = w + 1: it normalises the stream's counts and builds its coding tables.
// The rANS groups of all streams then run side by side, reading the codes from
// the slot: in a full chunk every lane is one component, whose 512 codes are
// one row, read 16 at a time into registers, and the groups are packed into
// warps (warp_pack_groups); otherwise one warp per (stream, group), symbol by
// symbol. The record is then laid out and its streams written one warp each.

// A rANS group of a record's width stream, placed in a warp: lanes base ..
// base + lanes - 1 of the warp code it (the decoder gives it ring_words refill
// words at ring_off of the block's ring area).
struct PackEntry {
  uint16_t sw, gg, base, lanes, ring_off, ring_words;
};
// At most 11 groups: sum over widths of ceil(lanes / 32) with at most 128
// lanes in all is at most 128 / 32 + 8 * 31 / 32 < 12.
constexpr uint32_t kMaxGroupsRec = 12;

// Packing of a record's rANS groups into warps, by one warp: the groups of
// every width stream sw with bit sw - 1 of rans set (one per 32 of its lanes),
// first fit into warps of 32 lanes, larger groups first (ties in stream
// order). With at most 128 lanes in groups of at most 32 this never needs more
// than eight warps: a group of at most 16 lanes opens a new warp only when
// every open warp holds more than 16, and groups of more than 16 lanes number
// at most 7. Each group gets a ring of 16 words per lane rounded up to a power
// of two (4096 words at most in all). Entries are listed by warp: warp w's are
// pk[first[w] .. first[w + 1]). Lane i handles group i; the eight fills live
// in every lane's registers.
__device__ inline void warp_pack_groups(const CompInfo& ci, uint32_t rans, uint32_t tcc, PackEntry* pk,
                                        uint32_t* first) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t sw = 0, gg = 0, L = 0, ng = 0;
  for (uint32_t b = 1; b <= 8; ++b) {
    const uint32_t m = ci.bcount[b];
    if (!m || !((rans >> (b - 1)) & 1u)) continue;
    const uint32_t N = rans_lanes(m * tcc), G = rans_groups(N);
    if (lane >= ng && lane < ng + G) {
      sw = b;
      gg = lane - ng;
      L = min(kGroupLanes, N - gg * kGroupLanes);
    }
    ng += G;
  }
  const bool item = lane < ng;
  uint32_t rank = 0;  // position in the order: larger groups first, ties in stream order
  for (uint32_t j = 0; j < ng; ++j) {
    const uint32_t Lj = __shfl_sync(0xffffffffu, L, j);
    rank += (Lj > L || (Lj == L && j < lane)) ? 1u : 0u;
  }
  uint32_t fill[8] = {0, 0, 0, 0, 0, 0, 0, 0};
  uint32_t bin = 0, base = 0, my_roff = 0, my_rw = 0, roff = 0;
  for (uint32_t r = 0; r < ng; ++r) {
    const uint32_t src = __ffs(__ballot_sync(0xffffffffu, item && rank == r)) - 1u;
    const uint32_t Lr = __shfl_sync(0xffffffffu, L, src);
    uint32_t bb = 7u;
#pragma unroll
    for (int q = 6; q >= 0; --q)
      if (fill[q] + Lr <= kGroupLanes) bb = uint32_t(q);
    uint32_t at = 0;
#pragma unroll
    for (uint32_t q = 0; q < 8; ++q) {
      if (q == bb) {
        at = fill[q];
        fill[q] += Lr;
      }
    }
    const uint32_t rw = Lr > 1u ? 16u << (32 - __clz(Lr - 1u)) : 16u;
    if (lane == src) {
      bin = bb;
      base = at;
      my_roff = roff;
      my_rw = rw;
    }
    roff += rw;
  }
  uint32_t f[9];  // first entry of each warp
#pragma unroll
  for (uint32_t w = 0; w < 9; ++w) f[w] = __popc(__ballot_sync(0xffffffffu, item && bin < w));
  const uint32_t same = __match_any_sync(0xffffffffu, item ? bin : 0xffu);
  uint32_t fb = 0;
#pragma unroll
  for (uint32_t w = 0; w < 8; ++w)
    if (w == bin) fb = f[w];
  if (item) {
    PackEntry e;
    e.sw = uint16_t(sw);
    e.gg = uint16_t(gg);
    e.base = uint16_t(base);
    e.lanes = uint16_t(L);
    e.ring_off = uint16_t(my_roff);
    e.ring_words = uint16_t(my_rw);
    pk[fb + __popc(same & lanemask_lt())] = e;
  }
#pragma unroll
  for (uint32_t w = 0; w < 9; ++w)
    if (lane == w) first[w] = f[w];
  __syncwarp();
}

struct __align__(16) EntSmem {
  uint32_t freq[8][256];                 // per width stream, zero past its alphabet
  uint2 tab[kTabPool];                   // per symbol of each width stream: {f | cum << 16, 1/f}
  uint32_t rem[kTabPool], hist[kTabPool];
  uint32_t states[8][kMaxLanes];
  uint32_t W[8][4], wbeg[8][4], sub_len[8][4];
  uint32_t k[8], mode[8], bytes[8], off[9];
  uint32_t crc_t[1024];
  uint32_t tmp[32], red[32];
  CompInfo ci;
  PackEntry pk[kMaxGroupsRec];           // the record's rANS groups, by warp (first pk_first[w])
  uint32_t pk_first[9];
};

// rANS encode of one group (warp-synchronous) of a stream in which lane l
// (live lanes only) codes the 512 symbols row[0 .. 512) of its own row, last
// symbol first. The row is read as 16-byte vectors, two ahead of use. Words go
// to words[.. cap), filled downwards; returns their count and the final state.
__device__ inline uint32_t rans_encode_rows(const uint8_t* row, bool live, const uint2* tab, uint16_t* words,
                                            uint32_t cap, uint32_t* x_out) {
  const uint32_t lt = lanemask_lt();
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  uint4 cur = live ? __ldcg(r4 + 31) : z4, nxt = live ? __ldcg(r4 + 30) : z4;
  uint32_t x = kRansLow, pos = cap;
#pragma unroll 1
  for (int c = 31; c >= 0; --c) {
    const uint4 nn = (live && c >= 2) ? __ldcg(r4 + (c - 2)) : z4;
    const uint32_t w[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
    for (int i = 15; i >= 0; --i) {
      const uint2 e = tab[(w[i >> 2] >> (8 * (i & 3))) & 0xffu];
      const uint32_t f = e.x & 0xffffu, cum = e.x >> 16;
      const bool emit = live && x >= (f << 20);
      const uint32_t mask = __ballot_sync(0xffffffffu, emit);
      pos -= __popc(mask);
      if (emit) words[pos + __popc(mask & lt)] = uint16_t(x & 0xffffu);
      const uint32_t xe = emit ? (x >> 16) : x;
      uint32_t q = __umulhi(xe, e.y);
      uint32_t r = xe - q * f;
      const bool over = r >= f;
      q += over ? 1u : 0u;
      r -= over ? f : 0u;
      x = live ? (q << kProbBits) + r + cum : x;
    }
    cur = nxt;
    nxt = nn;
  }
  *x_out = x;
  return cap - pos;
}

// A width stream's record (RAW, CONST or RANS; the layout of
// block_write_stream) written by one warp, so that the streams of a record are
// written side by side. raw(i) gives symbol i for RAW.
template <class RawFn>
__device__ inline void warp_write_stream(uint8_t* rec, uint32_t mode, uint32_t n, uint32_t bytes, uint32_t csym,
                                         uint32_t k, const uint32_t* freq, const uint32_t* states,
                                         const uint16_t* words, const uint32_t* wbeg, const uint32_t* W,
                                         const uint32_t* sub_len, RawFn raw) {
  const uint32_t lane = threadIdx.x & 31u;
  if (mode == kModeRaw || mode == kModeConst) {
    if (lane == 0)
      *reinterpret_cast<uint4*>(rec) =
          make_uint4(mode | (mode == kModeConst ? (csym << 8) : 0u), bytes, n, mode == kModeConst ? 1u : 0u);
    if (mode == kModeRaw) {
      for (uint32_t q = lane; q < pad16(n) / 16u; q += 32u) {
        uint32_t w[4] = {0, 0, 0, 0};
        for (uint32_t b = 0; b < 16; ++b) {
          const uint32_t i = q * 16u + b;
          w[b >> 2] |= (i < n ? raw(i) : 0u) << (8 * (b & 3u));
        }
        *reinterpret_cast<uint4*>(rec + 16 + q * 16u) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncwarp();
    return;
  }
  const uint32_t N = rans_lanes(n), G = rans_groups(N);
  if (lane == 0) *reinterpret_cast<uint4*>(rec) = make_uint4(kModeRans | (G << 16), bytes, n, k);
#pragma unroll
  for (uint32_t w = 0; w < 8; ++w) {  // presence bitmap, 32 symbols per word
    const uint32_t bits = __ballot_sync(0xffffffffu, freq[32 * w + lane] != 0u);
    if (lane == 0) reinterpret_cast<uint32_t*>(rec + 16)[w] = bits;
  }
  uint32_t cnt = 0;  // lane covers symbols 8 lane .. 8 lane + 7
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) cnt += freq[8 * lane + i] != 0u ? 1u : 0u;
  uint32_t incl = cnt;
#pragma unroll
  for (uint32_t o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t idx = incl - cnt;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    const uint32_t f = freq[8 * lane + i];
    if (f) st_u16(rec + 48 + 2u * idx++, f);
  }
  const uint32_t ftab_end = 48u + 2u * k, lens_at = pad16(ftab_end);
  if (lane < lens_at - ftab_end) rec[ftab_end + lane] = 0;
  const uint32_t lens_end = lens_at + 4u * G, sub0 = pad16(lens_end);
  if (lane < G) reinterpret_cast<uint32_t*>(rec + lens_at)[lane] = sub_len[lane];
  if (lane < sub0 - lens_end) rec[lens_end + lane] = 0;
  uint32_t off = sub0;
  for (uint32_t g = 0; g < G; ++g) {
    const uint32_t lanes_g = min(kGroupLanes, N - g * kGroupLanes);
    uint8_t* sub = rec + off;
    if (lane < lanes_g) reinterpret_cast<uint32_t*>(sub)[lane] = states[g * kGroupLanes + lane];
    uint16_t* w16 = reinterpret_cast<uint16_t*>(sub + 4u * lanes_g);
    const uint16_t* src = words + wbeg[g];
    const uint32_t Wg = W[g];
#pragma unroll 4
    for (uint32_t i = lane; i < Wg; i += 32u) w16[i] = src[i];
    const uint32_t end = off + sub_len[g], padded = off + pad16(sub_len[g]);
    if (lane < padded - end) rec[end + lane] = 0;
    off = padded;
  }
  __syncwarp();
}

// The same for the groups packed into one warp: the lanes of a group (mask gm)
// order its words and share its position; returns the group's word count.
__device__ inline uint32_t rans_encode_rows_packed(const uint8_t* row, bool live, const uint2* tab, uint16_t* words,
                                                   uint32_t cap, uint32_t gm, uint32_t* x_out) {
  const uint32_t lt = lanemask_lt();
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
  const uint4 z4 = make_uint4(0, 0, 0, 0);
  uint4 cur = live ? __ldcg(r4 + 31) : z4, nxt = live ? __ldcg(r4 + 30) : z4;
  uint32_t x = kRansLow, pos = cap;
#pragma unroll 1
  for (int c = 31; c >= 0; --c) {
    const uint4 nn = (live && c >= 2) ? __ldcg(r4 + (c - 2)) : z4;
    const uint32_t w[4] = {cur.x, cur.y, cur.z, cur.w};
#pragma unroll
    for (int i = 15; i >= 0; --i) {
      const uint2 e = tab[(w[i >> 2] >> (8 * (i & 3))) & 0xffu];
      const uint32_t f = e.x & 0xffffu, cum = e.x >> 16;
      const bool emit = live && x >= (f << 20);
      const uint32_t mask = __ballot_sync(0xffffffffu, emit) & gm;
      pos -= __popc(mask);
      if (emit) words[pos + __popc(mask & lt)] = uint16_t(x & 0xffffu);
      const uint32_t xe = emit ? (x >> 16) : x;
      uint32_t q = __umulhi(xe, e.y);
      uint32_t r = xe - q * f;
      const bool over = r >= f;
      q += over ? 1u : 0u;
      r -= over ? f : 0u;
      x = live ? (q << kProbBits) + r + cum : x;
    }
    cur = nxt;
    nxt = nn;
  }
  *x_out = x;
  return cap - pos;
}

__global__ void __launch_bounds__(kThreads, 5)
k_transform_entropy(TransformShape sh, TransformPlanDev pl, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  EntSmem& S = *reinterpret_cast<EntSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t warp = tid >> 5, lane = tid & 31u;
  const uint32_t rps = 1u + sh.n_mid;
  const uint32_t gs = blockIdx.x / sh.n_mid, c = blockIdx.x % sh.n_mid;
  const uint32_t r = gs * rps + 1u + c;
  const uint32_t fr = frame_of(b.rec_base, b.n, r);
  const uint32_t ls = (r - b.rec_base[fr]) / rps;
  const uint32_t sidx = b.f[fr].first_slice + ls;
  const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
  uint8_t* rec = ws.slots + uint64_t(r) * ws.slot_bytes;
  const uint8_t* codes_g = slot_codes(rec, ws.slot_bytes);
  uint16_t* scratch = slot_words(rec, ws.slot_bytes);

  const uint32_t side_len = __ldcg(&ws.rec_len[r]);  // written by k_transform_side
  crc_tables_init(S.crc_t);
  load_comp_info(pl.comp + sidx, S.ci);
  for (uint32_t i = tid; i < kTabPool; i += nthr)
    S.hist[i] = __ldcg(reinterpret_cast<const uint32_t*>(codes_g + kHistOffset) + i);
  __syncthreads();
  if (S.hist[kTabPool - 1u] == kHistTimeout) {  // the projection gave up on this record
    if (tid == 0) {
      ws.rec_len[r] = kRecLenError | uint32_t(kErrTimeout);
      ws.rec_crc[r] = 0;
    }
    return;
  }

  const Split split(tcc);
  // ---- per-stream tables from the counts: warp w takes width b = w + 1. In
  // a full chunk the record's rANS groups are packed into warps meanwhile, by
  // a warp with no table to build (warp 0 after its table when every width has
  // one), from the counts: a stream is rANS coded when it holds two symbols
  {
    const uint32_t bw = warp + 1u, m = S.ci.bcount[bw];
    if (m) {
      const uint32_t k = warp_normalize(S.hist + tab_base(bw), 1u << bw, m * tcc, S.freq[warp],
                                        S.rem + tab_base(bw), S.tab + tab_base(bw));
      if (lane == 0) S.k[warp] = k;
    }
    uint32_t present = 0;
    for (uint32_t b = 1; b <= 8; ++b) present |= S.ci.bcount[b] ? 1u << (b - 1) : 0u;
    const uint32_t pw = present == 0xffu ? 0u : 31u - __clz(~present & 0xffu);
    if (tcc == kMaxCt && warp == pw) {
      uint32_t rans = 0;
      for (uint32_t b = 1; b <= 8; ++b) {
        if (!S.ci.bcount[b]) continue;
        uint32_t c = 0;
        for (uint32_t i = lane; i < (1u << b); i += 32u) c += S.hist[tab_base(b) + i] != 0u ? 1u : 0u;
        if (__reduce_add_sync(0xffffffffu, c) >= 2u) rans |= 1u << (b - 1);
      }
      warp_pack_groups(S.ci, rans, tcc, S.pk, S.pk_first);
    }
  }
  __syncthreads();
  if (tcc == kMaxCt) {
    // ---- full chunk (lane l of a stream: component l, all 512 tokens): the
    // rANS groups packed into warps
    const uint32_t e0 = S.pk_first[warp], e1 = S.pk_first[warp + 1];
    if (e1 > e0) {
      int me = -1;
      for (uint32_t i = e0; i < e1; ++i)
        if (lane >= S.pk[i].base && lane < S.pk[i].base + S.pk[i].lanes) me = int(i);
      const bool live = me >= 0;
      const PackEntry pe = S.pk[live ? me : e0];
      const uint32_t bw = pe.sw, g = pe.gg, li = lane - pe.base;
      const uint32_t m = S.ci.bcount[bw], n = m * tcc, base = S.ci.bstart[bw];
      const uint32_t N = rans_lanes(n), G = rans_groups(N);
      uint32_t b0, len0, b1 = n, len1;
      lane_range(n, N, g * kGroupLanes, b0, len0);
      if (g + 1 < G) lane_range(n, N, (g + 1) * kGroupLanes, b1, len1);
      const uint32_t wbase = base * tcc;  // word scratch of this stream: one word per symbol
      const uint32_t l = g * kGroupLanes + li;
      const uint32_t gm = live ? (pe.lanes == 32u ? 0xffffffffu : ((1u << pe.lanes) - 1u) << pe.base) : 0u;
      uint32_t x;
      const uint32_t Wg = rans_encode_rows_packed(codes_g + uint64_t(live ? S.ci.comp[base + l] : 0u) * kCodesRow, live,
                                                  S.tab + tab_base(bw), scratch + wbase + b0, b1 - b0, gm, &x);
      if (live) S.states[bw - 1][l] = x;
      if (live && li == 0) {
        S.W[bw - 1][g] = Wg;
        S.wbeg[bw - 1][g] = wbase + b1 - Wg;
      }
    }
  } else {
  // ---- rANS groups of every stream, one warp per (stream, group)
  {
    uint32_t pair = 0;
    for (uint32_t bw = 1; bw <= 8; ++bw) {
      const uint32_t m = S.ci.bcount[bw];
      if (!m || S.k[bw - 1] < 2) continue;
      const uint32_t n = m * tcc, base = S.ci.bstart[bw];
      const uint32_t N = rans_lanes(n), G = rans_groups(N);
      const uint32_t wbase = base * tcc;  // word scratch of this stream: one word per symbol
      for (uint32_t g = 0; g < G; ++g, ++pair) {
        if (pair % (nthr >> 5) != warp) continue;
        uint32_t b0, len0, b1 = n, len1;
        lane_range(n, N, g * kGroupLanes, b0, len0);
        if (g + 1 < G) lane_range(n, N, (g + 1) * kGroupLanes, b1, len1);
        uint32_t x, Wg;
        const uint32_t* comp = S.ci.comp + base;
        if (tcc == kMaxCt) {  // lane l: component l, all 512 tokens
          const uint32_t l = g * kGroupLanes + lane;
          const bool live = l < N;
          Wg = rans_encode_rows(codes_g + uint64_t(live ? comp[l] : 0u) * kCodesRow, live, S.tab + tab_base(bw),
                                scratch + wbase + b0, b1 - b0, &x);
        } else {
          Wg = rans_encode_strided([comp, codes_g](uint32_t col) { return codes_g + uint64_t(comp[col]) * kCodesRow; },
                                   1u, tcc, n, N, g, S.tab + tab_base(bw), scratch + wbase + b0, b1 - b0, &x);
        }
        if (g * kGroupLanes + lane < N) S.states[bw - 1][g * kGroupLanes + lane] = x;
        if (lane == 0) {
          S.W[bw - 1][g] = Wg;
          S.wbeg[bw - 1][g] = wbase + b1 - Wg;
        }
      }
    }
  }
  }
  __syncthreads();
  // ---- layout: modes and record offsets
  if (tid == 0) {
    uint32_t off = side_len;  // the side streams come first
    for (uint32_t bw = 1; bw <= 8; ++bw) {
      S.off[bw - 1] = off;
      const uint32_t m = S.ci.bcount[bw];
      if (!m) continue;
      const uint32_t n = m * tcc, k = S.k[bw - 1], raw_b = 16u + pad16(n);
      uint32_t mode, bytes;
      if (k == 1) { mode = kModeConst; bytes = 16; }
      else {
        const uint32_t rb = rans_layout(n, k, S.W[bw - 1], S.sub_len[bw - 1]);
        if (rb < raw_b) { mode = kModeRans; bytes = rb; }
        else { mode = kModeRaw; bytes = raw_b; }
      }
      S.mode[bw - 1] = mode;
      S.bytes[bw - 1] = bytes;
      off += bytes;
    }
    S.off[8] = off;
  }
  __syncthreads();
  {  // warp w writes the stream of width w + 1, all streams side by side
    const uint32_t bw = warp + 1u, m = S.ci.bcount[bw];
    if (m) {
      const uint32_t n = m * tcc, base = S.ci.bstart[bw];
      auto sym = [&](uint32_t i) -> uint32_t {
        uint32_t a, t;
        split(i, a, t);
        return uint32_t(codes_g[uint64_t(S.ci.comp[base + a]) * kCodesRow + t]);
      };
      warp_write_stream(rec + S.off[bw - 1], S.mode[bw - 1], n, S.bytes[bw - 1], sym(0), S.k[bw - 1],
                        S.freq[bw - 1], S.states[bw - 1], scratch, S.wbeg[bw - 1], S.W[bw - 1], S.sub_len[bw - 1],
                        sym);
    }
  }
  __syncthreads();
  const uint32_t len = S.off[8];
  const uint32_t crc = crc32_block_aligned(rec, len, S.crc_t, S.red);
  if (tid == 0) {
    ws.rec_len[r] = len;
    ws.rec_crc[r] = crc;
  }
}


// Raw record of each slice: sink rows, then recent rows, bf16 bytes, padded.
__global__ void __launch_bounds__(kThreads)
k_transform_encode_raw(TransformShape sh, FrameBatch b, EncodeLayout ws) {
  __shared__ uint32_t crc_t[1024];
  __shared__ uint32_t red[32];
  const uint32_t tid = threadIdx.x;
  const uint32_t rps = 1u + sh.n_mid;
  const uint32_t r = blockIdx.x * rps;  // record of the batch
  const uint32_t fr = frame_of(b.rec_base, b.n, r);
  const uint32_t ls = (r - b.rec_base[fr]) / rps;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(b.f[fr].src);
  uint8_t* rec = ws.slots + uint64_t(r) * ws.slot_bytes;
  const uint32_t n_rows = sh.s_end + (sh.T - sh.r_start);
  const uint32_t bytes = n_rows * kD * 2u, len = pad16(bytes);
  const uint16_t* xs = src + uint64_t(ls) * sh.T * kD;
  crc_tables_init(crc_t);
  const uint32_t per_row = kD * 2u / 16u;
  for (uint32_t q = tid; q < n_rows * per_row; q += blockDim.x) {
    uint32_t row = q / per_row, part = q % per_row;
    uint32_t t = row < sh.s_end ? row : sh.r_start + (row - sh.s_end);
    reinterpret_cast<uint4*>(rec)[q] = __ldg(reinterpret_cast<const uint4*>(xs + uint64_t(t) * kD) + part);
  }
  __syncthreads();
  uint32_t crc = crc32_block_aligned(rec, len, crc_t, red);
  if (tid == 0) {
    ws.rec_len[r] = len;
    ws.rec_crc[r] = crc;
  }
}

// ---------------------------------------------------------------------------
// Transform decoder, in two stages.
//
// Entropy stage (k_transform_decode_codes): blocks of 8 warps, four per SM,
// each taking records in turn. A raw record is copied to its rows. A middle
// record is checked (CRC, stream walk, stream headers, side information) and
// its codes are decoded into the record's code block in the workspace,
// codes[t * 128 + j] for token t of the chunk and component j; the record's
// status word tells the tensor stage whether to use the block. A width
// stream's decode table is one byte per slot (its symbol) and f << 16 | cum
// per symbol: 5 KiB instead of a word per slot, so the tables of all eight
// streams of a record and the refill rings fit a quarter of an SM. The
// record's rANS groups are packed into warps (warp_pack_groups).
//
// Tensor stage (k_transform_decode): dequantisation, the inverse projection
// on the tensor cores and the RoPE epilogue of every middle record whose
// status is OK, reading its code block.
constexpr uint32_t kCodeRow = kD;  // bytes of a code block's token row

struct CodeBlocks {
  uint32_t* status;  // per record of the batch: kOk when the code block is complete
  uint8_t* codes;    // per record of the batch: ct token rows of kCodeRow bytes
  float2* zs;        // per record of the batch: (z, s) of coded component cc, block blk at cc * (ct / kTile) + blk
};
__device__ inline CodeBlocks code_blocks(uint8_t* ws, uint32_t max_records, uint32_t ct) {
  uint8_t* p = ws + kDecodeWsFixed + ((8ull * max_records + 255u) & ~255ull);
  CodeBlocks c;
  c.status = reinterpret_cast<uint32_t*>(p);
  c.codes = p + ((4ull * max_records + 255u) & ~255ull);
  c.zs = reinterpret_cast<float2*>(c.codes + uint64_t(max_records) * ct * kCodeRow);
  return c;
}

constexpr uint32_t kRingWords = 512;              // refill ring of one warp

struct __align__(16) DecEntSmem {
  uint8_t lut[8][kProbScale];  // per width stream: symbol of each slot
  alignas(16) uint16_t ring[kThreads / 32][kRingWords];  // refill rings of the packed rANS groups (cp.async targets)
  uint32_t crc_t[1024];        // CRC tables; after the record's CRC, the side streams' f << 16 | cum tables
  uint32_t freq[8][256];               // per width stream; f << 16 | cum after the table build
  uint32_t tmp[32], red[32];
  StreamInfo si[8];
  uint32_t str_off[8];                 // stream record offsets within the record, by width - 1
  CompInfo ci;
  uint32_t base[kBatchMax + 1];
  uint32_t crc_ok, bad, walk_ok, side_ok;
  uint32_t side_off[5];                // the side stream records' offsets in the record
  StreamInfo side_si[4];               // the side streams (their f << 16 | cum tables overlay crc_t)
  PackEntry pk[kMaxGroupsRec];         // the record's rANS groups, by warp (first pk_first[w])
  uint32_t pk_first[9];
};
static_assert(sizeof(DecEntSmem{}.crc_t) == 4u * 256u * sizeof(uint32_t), "four side tables overlay the CRC table");

// Decode table of one rANS stream built by one warp: freq[256] (validated, sum
// 4096) becomes freq[s] = f_s << 16 | cum_s, and lut[slot] the symbol whose
// range [cum_s, cum_s + f_s) holds slot: each present symbol's first slot is
// marked with the symbol, and a running maximum over the slots (unmarked slots
// are 0, which before the first mark is symbol 0's range) fills the rest,
// four slots per lane and step.
__device__ inline void warp_dec_lut8(uint32_t* freq, uint8_t* lut) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t f[8], mine = 0;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    f[i] = freq[8u * lane + i];
    mine += f[i];
  }
  uint32_t incl = mine;
#pragma unroll
  for (uint32_t o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t cum = incl - mine;
  uint32_t* lut32 = reinterpret_cast<uint32_t*>(lut);
  for (uint32_t i = lane; i < kProbScale / 16u; i += 32u) reinterpret_cast<uint4*>(lut)[i] = make_uint4(0, 0, 0, 0);
  __syncwarp();
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    const uint32_t s = 8u * lane + i;
    if (f[i]) lut[cum] = uint8_t(s);
    freq[s] = (f[i] << 16) | cum;
    cum += f[i];
  }
  __syncwarp();
  uint32_t carry = 0;
#pragma unroll 2
  for (uint32_t w0 = 0; w0 < kProbScale / 4u; w0 += 32u) {
    const uint32_t w = lut32[w0 + lane];
    const uint32_t m0 = w & 0xffu, m1 = max(m0, (w >> 8) & 0xffu);
    const uint32_t m2 = max(m1, (w >> 16) & 0xffu), m3 = max(m2, w >> 24);
    uint32_t x = m3;
#pragma unroll
    for (uint32_t o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
      if (lane >= o) x = max(x, y);
    }
    uint32_t before = __shfl_up_sync(0xffffffffu, x, 1);
    before = max(lane ? before : 0u, carry);
    lut32[w0 + lane] = max(m0, before) | (max(m1, before) << 8) | (max(m2, before) << 16) | (max(m3, before) << 24);
    carry = max(carry, __shfl_sync(0xffffffffu, x, 31));
  }
  __syncwarp();
}

// rANS decode of the groups packed into one warp (entries pe[0 .. ne - 1]).
// Group g of width stream sw holds lanes g * 32 .. of the stream's N lanes (n
// symbols); symbol i = a * tcc + t of the stream is written to codes[t * 128 +
// comp[a]] (codes in global memory). Each lane decodes its group's lane; the
// group's lanes of the ballot (mask gm) order its refill words. A group's
// sub-stream (sl bytes, 16-byte aligned) holds its lanes' states, then the
// refill words; its 16-byte units, from the one holding the first word on, are
// copied by cp.async into the group's ring of ring_words 16-bit positions
// counted from the sub-stream's start (the words begin at position 2 * lanes):
// at every stage of 8 steps (at most 8 words per lane consumed, half the ring)
// the warp waits for all its copies, then requests units up to ring_words
// positions past the unit holding the group's next word. The words of a stage
// were thus requested a stage earlier, and a unit's ring slot is reused only
// once every word in it has been consumed. Lanes outside every group idle.
// Returns false (on every lane) when a group's sub-stream cannot hold its
// states, a symbol exceeds its width's levels, a lane reads past its
// sub-stream, or the final states and word counts do not match.
template <bool kFull, class Smem>
__device__ inline bool decode_codes_packed(Smem& S, const PackEntry* pe, uint32_t ne, const uint8_t* rec,
                                           uint8_t* codes, uint32_t tcc) {
  const uint32_t lane = threadIdx.x & 31u;
  const uint32_t lt = lanemask_lt();
  int me = -1;
  for (uint32_t i = 0; i < ne; ++i)
    if (lane >= pe[i].base && lane < pe[i].base + pe[i].lanes) me = int(i);
  bool live = me >= 0, ok = true;
  uint32_t sw = 1, gg = 0, li = 0, lanes_g = 1, rw = 16, roff = 0;
  if (live) {
    sw = pe[me].sw;
    gg = pe[me].gg;
    li = lane - pe[me].base;
    lanes_g = pe[me].lanes;
    rw = pe[me].ring_words;
    roff = pe[me].ring_off;
  }
  const uint32_t m = live ? S.ci.bcount[sw] : 1u, n = m * tcc, N = rans_lanes(n), levels = (1u << sw) - 1u;
  const uint32_t sl = live ? S.si[sw - 1].sub_len[gg] : 0u;
  const uint8_t* sub = live ? rec + S.str_off[sw - 1] + S.si[sw - 1].sub_off[gg] : rec;
  if (live && (sl < 4u * lanes_g || ((sl - 4u * lanes_g) & 1u))) {
    ok = false;
    live = false;
  }
  const uint32_t W = live ? (sl - 4u * lanes_g) >> 1 : 0u, w0 = 2u * lanes_g;
  uint32_t start = 0, len = 0, start0 = 0, gmax = 0;
  if (live) {
    lane_range(n, N, gg * kGroupLanes + li, start, len);
    lane_range(n, N, gg * kGroupLanes, start0, gmax);
  }
  const uint32_t wmax = __reduce_max_sync(0xffffffffu, live ? gmax : 0u);
  const uint32_t gm = live ? (lanes_g == 32u ? 0xffffffffu : ((1u << lanes_g) - 1u) << pe[me].base) : 0u;
  const uint8_t* lut = &S.lut[live ? sw - 1 : 0][0];
  const uint32_t* fc = &S.freq[live ? sw - 1 : 0][0];
  const uint16_t* ring = &S.ring[0][0] + roff;
  const uint32_t ring_saddr = static_cast<uint32_t>(__cvta_generic_to_shared(ring)), runits = rw >> 3;
  uint32_t x = live ? reinterpret_cast<const uint32_t*>(sub)[li] : kRansLow;
  uint32_t a = start / tcc, t = start - a * tcc;
  const uint32_t* comp = S.ci.comp + S.ci.bstart[sw];
  uint32_t j = (live && len && a < m) ? comp[a] : 0u;
  uint8_t* cp = codes + uint64_t(t) * kCodeRow + j;  // this lane's next code
  uint32_t left = tcc - t;                          // steps until the lane moves to the next component
  uint32_t rp = w0, orv = 0;                        // ring position of the group's next word; OR of the symbols
  const uint32_t n_units = (sl + 15u) >> 4;
  uint32_t loaded = w0 >> 3;  // units wholly inside the states are never needed
  auto request = [&]() {
    if (live) {
      const uint32_t target = min(n_units, (rp >> 3) + runits);
      for (uint32_t u = loaded + li; u < target; u += lanes_g)
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ring_saddr + ((u & (runits - 1u)) << 4)),
                     "l"(sub + (uint64_t(u) << 4))
                     : "memory");
      loaded = max(loaded, target);
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  };
  request();
  for (uint32_t tau0 = 0; tau0 < wmax; tau0 += 8u) {
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();
    request();
#pragma unroll
    for (uint32_t k = 0; k < 8; ++k) {
      const bool act = live && tau0 + k < len;
      if (act) {
        const uint32_t slot = x & (kProbScale - 1u);
        const uint32_t sym = lut[slot];
        const uint32_t e = fc[sym];
        x = (e >> 16) * (x >> kProbBits) + slot - (e & 0xffffu);
        orv |= sym;
        *cp = uint8_t(sym);
        cp += kCodeRow;
        if constexpr (!kFull) {  // a full chunk's lane is one component: it never moves on
          if (--left == 0u) {
            ++a;
            cp = codes + (a < m ? comp[a] : 0u);
            left = tcc;
          }
        }
      }
      const bool need = act && x < kRansLow;
      const uint32_t mask = __ballot_sync(0xffffffffu, need) & gm;
      const uint32_t w = ring[(rp + __popc(mask & lt)) & (rw - 1u)];
      if (need) x = (x << 16) | w;
      rp += __popc(mask);
    }
  }
  asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();
  ok = ok && (!live || ((orv & ~levels) == 0u && rp - w0 == W && x == kRansLow));
  return __all_sync(0xffffffffu, ok);
}

// Check the side stream record at rec (16-byte aligned, avail bytes: exactly
// its own length from the header walk) for n symbols on N lanes (one group)
// and, for RANS, load its frequencies into freq[256]. Warp-cooperative; lane
// 0 fills si; returns the status on every lane.
__device__ inline int warp_parse_side(const uint8_t* rec, uint32_t avail, uint32_t n, uint32_t N, StreamInfo& si,
                                      uint32_t* freq) {
  const uint32_t lane = threadIdx.x & 31u;
  if (avail < 16u) return kErrCorrupt;
  const uint4 hv = __ldg(reinterpret_cast<const uint4*>(rec));
  const uint32_t mode = hv.x & 0xffu, csym = (hv.x >> 8) & 0xffu, G = (hv.x >> 16) & 0xffu, b3 = hv.x >> 24;
  const uint32_t bytes = hv.y, rn = hv.z, k = hv.w;
  bool bad = b3 > (mode == kModeRans ? 1u : 0u) || rn != n || (bytes & 15u) || bytes < 16u || bytes != avail;
  uint32_t sub_off = 0, sub_len = 0;
  if (!bad) {
    if (mode == kModeRaw) bad = csym || G || k || bytes != 16u + pad16(n);
    else if (mode == kModeConst) bad = G || k != 1u || bytes != 16u;
    else if (mode == kModeRans) {
      bad = csym || n == 0 || G != 1u || k < 2u || k > 256u;
      if (!bad) {
        const uint32_t lens_at = pad16(48u + 2u * k);
        sub_off = lens_at + 16u;
        bad = sub_off > bytes;
        if (!bad) {
          sub_len = ld_u32(rec + lens_at);
          bad = sub_len > bytes || sub_off + pad16(sub_len) != bytes;
        }
      }
    } else {
      bad = true;
    }
  }
  if (lane == 0) {
    si.mode = mode; si.sym = csym; si.groups = G; si.bytes = bytes; si.k = k; si.delta = b3;
    si.sub_off[0] = sub_off; si.sub_len[0] = sub_len;
  }
  if (bad || mode != kModeRans) {
    __syncwarp();
    return bad ? kErrCorrupt : kOk;
  }
  // presence bitmap byte `lane` covers symbols 8 lane .. 8 lane + 7
  const uint32_t bm = rec[16u + lane];
  const uint32_t cnt = __popc(bm);
  uint32_t incl = cnt;
#pragma unroll
  for (uint32_t o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
  uint32_t idx = incl - cnt, fs = 0;
  bool zero = false;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    uint32_t f = 0;
    if (total == k && ((bm >> i) & 1u)) {
      f = ld_u16(rec + 48u + 2u * idx++);
      zero |= f == 0;
    }
    freq[8u * lane + i] = f;
    fs += f;
  }
  fs = __reduce_add_sync(0xffffffffu, fs);
  bad = total != k || __any_sync(0xffffffffu, zero) || fs != kProbScale;
  __syncwarp();
  return bad ? kErrCorrupt : kOk;
}

// Check the width stream record at rec (16-byte aligned, avail bytes from its
// offset to the end of the record) for n symbols under the code streams' lane
// rule, with the checks of block_parse_stream (no lane-delta flag), and for
// RANS load its frequencies into freq[256]. Warp-cooperative; lane 0 fills si;
// returns the status on every lane.
__device__ inline int warp_parse_stream(const uint8_t* rec, uint32_t avail, uint32_t n, StreamInfo& si,
                                        uint32_t* freq) {
  const uint32_t lane = threadIdx.x & 31u;
  if (avail < 16u) {
    if (lane == 0) si.status = kErrCorrupt;
    __syncwarp();
    return kErrCorrupt;
  }
  const uint4 hv = __ldg(reinterpret_cast<const uint4*>(rec));
  const uint32_t mode = hv.x & 0xffu, csym = (hv.x >> 8) & 0xffu, G = (hv.x >> 16) & 0xffu, b3 = hv.x >> 24;
  const uint32_t bytes = hv.y, rn = hv.z, k = hv.w;
  bool bad = b3 != 0u || rn != n || (bytes & 15u) || bytes < 16u || bytes > avail;
  uint32_t offs[4] = {0, 0, 0, 0}, lens[4] = {0, 0, 0, 0};
  if (!bad) {
    if (mode == kModeRaw) {
      bad = csym || G || k || bytes != 16u + pad16(n);
    } else if (mode == kModeConst) {
      bad = G || k != 1u || bytes != 16u;
    } else if (mode == kModeRans) {
      bad = csym || n == 0 || G != rans_groups(rans_lanes(n)) || k < 2u || k > 256u;
      if (!bad) {
        const uint32_t lens_at = pad16(48u + 2u * k);
        uint32_t p = pad16(lens_at + 4u * G);
        bad = p > bytes;
        if (!bad) {  // G <= 4 lengths in one aligned 16-byte load
          const uint4 lv = __ldg(reinterpret_cast<const uint4*>(rec + lens_at));
          lens[0] = lv.x; lens[1] = lv.y; lens[2] = lv.z; lens[3] = lv.w;
#pragma unroll
          for (uint32_t g = 0; g < 4; ++g) {
            if (g >= G || bad) continue;
            if (lens[g] > bytes || p + pad16(lens[g]) > bytes) {
              bad = true;
            } else {
              offs[g] = p;
              p += pad16(lens[g]);
            }
          }
          bad = bad || p != bytes;
        }
      }
    } else {
      bad = true;
    }
  }
  if (lane == 0) {
    si.mode = mode; si.sym = csym; si.groups = G; si.bytes = bytes; si.k = k; si.delta = 0;
#pragma unroll
    for (uint32_t g = 0; g < 4; ++g) {
      si.sub_off[g] = offs[g];
      si.sub_len[g] = g < G ? lens[g] : 0u;
    }
  }
  if (!bad && mode == kModeRans) {
    // presence bitmap byte `lane` covers symbols 8 lane .. 8 lane + 7
    const uint32_t bm = rec[16u + lane];
    const uint32_t cnt = __popc(bm);
    uint32_t incl = cnt;
#pragma unroll
    for (uint32_t o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    const uint32_t total = __shfl_sync(0xffffffffu, incl, 31);
    uint32_t idx = incl - cnt, fs = 0;
    bool zero = false;
#pragma unroll
    for (uint32_t i = 0; i < 8; ++i) {
      uint32_t f = 0;
      if (total == k && ((bm >> i) & 1u)) {
        f = ld_u16(rec + 48u + 2u * idx++);
        zero |= f == 0;
      }
      freq[8u * lane + i] = f;
      fs += f;
    }
    fs = __reduce_add_sync(0xffffffffu, fs);
    bad = total != k || __any_sync(0xffffffffu, zero) || fs != kProbScale;
  }
  if (lane == 0) si.status = bad ? kErrCorrupt : kOk;
  __syncwarp();
  return bad ? kErrCorrupt : kOk;
}

// rANS decode of a side stream's single group by one warp (lanes l < N <= 32,
// the side lane rule) straight from the record (sl bytes at sub, 4-byte
// aligned), with no per-slot table: the symbol of a slot is the largest s with
// cum_s <= slot in fc[256] = f << 16 | cum (absent symbols carry the next
// present symbol's cum, so the search lands on the present one), found in
// eight steps. dm = 0xff undoes lane deltas; out(i, byte) takes value i's byte.
// Returns false (on every lane) when a lane reads past the words or the final
// states and word count do not match.
template <class Out>
__device__ inline bool side_decode_search(const uint8_t* sub, uint32_t sl, uint32_t n, const uint32_t* fc,
                                          uint32_t dm, Out out) {
  const uint32_t lane = threadIdx.x & 31u, N = side_lanes(n);
  if (sl < 4u * N || ((sl - 4u * N) & 1u)) return false;
  const uint32_t W = (sl - 4u * N) >> 1;
  const bool live = lane < N;
  uint32_t start = 0, len = 0, start0, maxlen;
  if (live) lane_range(n, N, lane, start, len);
  lane_range(n, N, 0u, start0, maxlen);
  const uint16_t* words = reinterpret_cast<const uint16_t*>(sub + 4u * N);
  uint32_t x = live ? __ldg(reinterpret_cast<const uint32_t*>(sub) + lane) : kRansLow;
  uint32_t pos = 0, prev = 0, over = 0;
  const uint32_t lt = lanemask_lt();
  for (uint32_t tau = 0; tau < maxlen; ++tau) {
    const bool act = live && tau < len;
    if (act) {
      const uint32_t slot = x & (kProbScale - 1u);
      uint32_t sym = 0;
#pragma unroll
      for (uint32_t step = 128u; step; step >>= 1)
        if ((fc[sym + step] & 0xffffu) <= slot) sym += step;
      const uint32_t e = fc[sym];
      x = (e >> 16) * (x >> kProbBits) + slot - (e & 0xffffu);
      prev = sym ^ (prev & dm);
      out(start + tau, prev);
    }
    const bool need = act && x < kRansLow;
    const uint32_t mask = __ballot_sync(0xffffffffu, need);
    const uint32_t idx = pos + __popc(mask & lt);
    if (need) {
      over |= idx >= W ? 1u : 0u;
      x = (x << 16) | (idx < W ? uint32_t(__ldg(words + idx)) : 0u);  // never past the sub-stream
    }
    pos += __popc(mask);
  }
  const bool ok = !over && pos == W && (!live || x == kRansLow);
  return __all_sync(0xffffffffu, ok);
}

// A stream's frequencies freq[256] (validated, sum 4096) become f << 16 | cum
// in place, by one warp.
__device__ inline void warp_fc_table(uint32_t* freq) {
  const uint32_t lane = threadIdx.x & 31u;
  uint32_t f[8], mine = 0;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    f[i] = freq[8u * lane + i];
    mine += f[i];
  }
  uint32_t incl = mine;
#pragma unroll
  for (uint32_t o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  uint32_t cum = incl - mine;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    freq[8u * lane + i] = (f[i] << 16) | cum;
    cum += f[i];
  }
  __syncwarp();
}

static_assert(sizeof(DecEntSmem) + 1024 <= 233472 / 4, "entropy stage should fit four blocks per SM");
static_assert(offsetof(DecEntSmem, ring) % 16 == 0 && offsetof(DecEntSmem, lut) % 4 == 0,
              "refill rings take 16-byte copies; the side streams' table reads 4-byte words");

__global__ void __launch_bounds__(kThreads, 4)
k_transform_decode_codes(TransformShape sh, TransformPlanDev pl, FrameBatch b, uint8_t* ws,
                         uint32_t max_records) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  DecEntSmem& S = *reinterpret_cast<DecEntSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t warp = tid >> 5, lane = tid & 31u;
  if (tid == 0) {  // records of the batch: prefix over frames that passed the header check
    uint32_t acc = 0;
    for (uint32_t f = 0; f < b.n; ++f) {
      S.base[f] = acc;
      const DecodeState* d = decode_state(ws, f);
      acc += d->status == kOk ? d->n_records : 0u;
    }
    S.base[b.n] = acc;
  }
  __syncthreads();
  const uint32_t nrec = S.base[b.n];
  if (blockIdx.x >= nrec) return;
  const CodeBlocks cb = code_blocks(ws, max_records, sh.ct);
  crc_tables_init(S.crc_t);
  const uint32_t rps = 1u + sh.n_mid;
  for (uint32_t g = blockIdx.x; g < nrec; g += gridDim.x) {
    __syncthreads();
    const uint32_t fr = frame_of(S.base, b.n, g), r = g - S.base[fr];
    const uint8_t* src = b.f[fr].src;
    uint16_t* dst = reinterpret_cast<uint16_t*>(b.f[fr].dst);
    DecodeState* ds = decode_state(ws, fr);
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint64_t off0 = ld_u64(e);
    const uint32_t len = ld_u32(e + 8), want = ld_u32(e + 12);
    const uint8_t* rec = src + off0;
    const uint32_t ls = r / rps, kind = r % rps;
    const uint32_t sidx = ds->first_slice + ls;
    if (g != blockIdx.x) crc_tables_init(S.crc_t);  // the previous record's side tables overlaid it
    uint32_t got = crc32_block_aligned<true>(rec, len, S.crc_t, S.red);
    if (tid == 0) S.crc_ok = (got == want);
    __syncthreads();
    int st = S.crc_ok ? kOk : kErrCorrupt;
    if (kind == 0) {
      uint16_t* xs = dst + uint64_t(ls) * sh.T * kD;
      const uint32_t n_rows = sh.s_end + (sh.T - sh.r_start);
      if (st == kOk && len != pad16(n_rows * kD * 2u)) st = kErrCorrupt;
      if (st != kOk) {
        if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
        continue;
      }
      const uint32_t per_row = kD * 2u / 16u;
      for (uint32_t q = tid; q < n_rows * per_row; q += nthr) {
        uint32_t row = q / per_row, part = q % per_row;
        uint32_t t = row < sh.s_end ? row : sh.r_start + (row - sh.s_end);
        reinterpret_cast<uint4*>(xs + uint64_t(t) * kD)[part] = reinterpret_cast<const uint4*>(rec)[q];
      }
      continue;
    }
    const uint32_t c = kind - 1;
    const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
    const uint32_t nb = (tcc + kTile - 1) / kTile;
    load_comp_info(pl.comp + sidx, S.ci);
    // Stream headers. One thread walks the side streams' headers (side
    // information: four byte-plane streams of V = every z, then every s) and
    // then the width streams' for their offsets. Warp q < 4 then checks side
    // stream q and turns its frequencies into a f << 16 | cum table over the
    // CRC table (rebuilt for the next record), while warps 4-7 check width
    // streams 5-8; warps 0-3 then check width streams 1-4. The side streams are
    // decoded later, beside the width streams, by warps without a rANS group.
    const bool kiv = sh.kivi && ((sidx / sh.H) & 1u) == 1u;  // values with per-token ranges
    const uint32_t half = S.ci.n_coded ? (kiv ? tcc : S.ci.n_coded * nb) : 0u, nv = 2u * half;
    if (tid == 0) {
      uint32_t o = 0, ok = st == kOk ? 1u : 0u;
      for (uint32_t q = 0; q < 4u && nv && ok; ++q) {
        S.side_off[q] = o;
        if (o + 16u > len) { ok = 0; break; }
        const uint32_t bytes = ld_u32(rec + o + 4);
        if (bytes < 16u || (bytes & 15u) || bytes > len - o || bytes > 16u + pad16(nv)) { ok = 0; break; }
        o += bytes;
      }
      S.side_off[4] = nv ? o : 0u;
      for (uint32_t bw = 1; bw <= 8 && ok; ++bw) {
        if (!S.ci.bcount[bw]) continue;
        S.str_off[bw - 1] = o;
        if (o + 16u > len) { ok = 0; break; }
        const uint32_t bytes = ld_u32(rec + o + 4);
        if (bytes < 16u || (bytes & 15u) || bytes > len - o) { ok = 0; break; }
        o += bytes;
      }
      S.walk_ok = ok && o == len;
      S.bad = 0;
    }
    __syncthreads();
    if (st == kOk && !S.walk_ok) st = kErrCorrupt;
    if (st == kOk) {
      bool okw = true;
      if (warp < 4 && nv) {
        const uint32_t q = warp, o = S.side_off[q];
        uint32_t* fcq = S.crc_t + 256u * q;
        okw = warp_parse_side(rec + o, S.side_off[q + 1] - o, nv, side_lanes(nv), S.side_si[q], fcq) == kOk;
        if (okw && S.side_si[q].mode == kModeRans) warp_fc_table(fcq);
      } else if (warp >= 4 && S.ci.bcount[warp + 1]) {
        const uint32_t o = S.str_off[warp];
        okw = warp_parse_stream(rec + o, len - o, S.ci.bcount[warp + 1] * tcc, S.si[warp], S.freq[warp]) == kOk;
      }
      if (!__syncthreads_and(okw)) st = kErrCorrupt;
    }
    if (st == kOk) {
      bool okw = true;
      if (warp < 4 && S.ci.bcount[warp + 1]) {
        const uint32_t o = S.str_off[warp];
        okw = warp_parse_stream(rec + o, len - o, S.ci.bcount[warp + 1] * tcc, S.si[warp], S.freq[warp]) == kOk;
      }
      if (!__syncthreads_and(okw)) st = kErrCorrupt;
    }
    if (st != kOk) {
      if (tid == 0) {
        atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
        cb.status[g] = uint32_t(st);
      }
      continue;
    }
    uint8_t* codes = cb.codes + uint64_t(g) * sh.ct * kCodeRow;
    // RAW and CONST streams: every thread writes codes
    {
      const Split split(tcc);
      for (uint32_t bw = 1; bw <= 8; ++bw) {
        const uint32_t m = S.ci.bcount[bw];
        const uint32_t mode = S.si[bw - 1].mode;
        if (!m || mode == kModeRans) continue;
        const uint32_t n = m * tcc, base = S.ci.bstart[bw], levels = (1u << bw) - 1u;
        const uint8_t* raw = rec + S.str_off[bw - 1] + 16u;
        const uint32_t csym = S.si[bw - 1].sym;
        uint32_t bad = 0;
        for (uint32_t i = tid; i < n; i += nthr) {
          uint32_t a, t;
          split(i, a, t);
          const uint32_t sy = mode == kModeRaw ? uint32_t(raw[i]) : csym;
          bad |= uint32_t(sy > levels);
          codes[t * kCodeRow + S.ci.comp[base + a]] = uint8_t(sy);
        }
        if (bad) S.bad = 1;
      }
    }
    // rANS streams: warp w builds the table of width w + 1 while another warp
    // packs the record's groups into warps (warp_pack_groups), each with its
    // own refill ring; then each warp decodes its groups side by side
    uint32_t rans = 0;  // width streams with rANS groups
    for (uint32_t sw = 1; sw <= 8; ++sw)
      if (S.ci.bcount[sw] && S.si[sw - 1].mode == kModeRans) rans |= 1u << (sw - 1);
    if ((rans >> warp) & 1u) warp_dec_lut8(S.freq[warp], S.lut[warp]);
    // the packing runs in a warp that builds no table (the highest such warp;
    // warp 0 after its table when every width has one)
    const uint32_t pw = rans == 0xffu ? 0u : 31u - __clz(~rans & 0xffu);
    if (warp == pw) warp_pack_groups(S.ci, rans, tcc, S.pk, S.pk_first);
    __syncthreads();
    if (S.pk_first[warp + 1] > S.pk_first[warp]) {
      const PackEntry* pe = S.pk + S.pk_first[warp];
      const uint32_t ne = S.pk_first[warp + 1] - S.pk_first[warp];
      const bool ok = tcc == kMaxCt ? decode_codes_packed<true>(S, pe, ne, rec, codes, tcc)
                                    : decode_codes_packed<false>(S, pe, ne, rec, codes, tcc);
      if (!ok && lane == 0) S.bad = 1;
    }
    if (nv && warp >= 4) {
      // side stream q = 7 - warp (warps that hold no rANS group unless a record
      // fills more than four): byte q of each value of V goes straight into the
      // record's (z, s) pairs; value i < half is a zero point, the rest scales
      // (ranges), in the order of V
      const uint32_t q = 7u - warp, o = S.side_off[q];
      const StreamInfo& si = S.side_si[q];
      uint8_t* zb = reinterpret_cast<uint8_t*>(cb.zs + uint64_t(g) * kD * (sh.ct / kTile));
      const uint32_t bstride = sh.ct / kTile;
      auto out = [&](uint32_t i, uint32_t v) {
        const uint32_t hi = i >= half ? 1u : 0u, j = i - hi * half;
        const uint32_t pair = kiv ? j : (j / nb) * bstride + (j % nb);
        zb[8u * pair + 4u * hi + q] = uint8_t(v);
      };
      bool ok = true;
      if (si.mode == kModeRaw) {
        for (uint32_t i = lane; i < nv; i += 32u) out(i, __ldg(rec + o + 16u + i));
      } else if (si.mode == kModeConst) {
        for (uint32_t i = lane; i < nv; i += 32u) out(i, si.sym);
      } else {
        ok = side_decode_search(rec + o + si.sub_off[0], si.sub_len[0], nv, S.crc_t + 256u * q,
                                si.delta ? 0xffu : 0u, out);
      }
      if (!ok && lane == 0) S.bad = 1;
    }
    __syncthreads();
    if (tid == 0) {
      if (S.bad) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrCorrupt));
      cb.status[g] = S.bad ? uint32_t(kErrCorrupt) : uint32_t(kOk);
    }
  }
}

// Tensor stage shared memory: the operand tiles (each 128-byte-swizzled tile
// on a 1024-byte boundary), the record's scales and zero points.
struct __align__(1024) DecSmem {
  struct {
    uint8_t a_hi[kTcRows * 256];  // y^ as bf16 pieces, A operand [token][component]
    uint8_t a_lo[kTcRows * 256];
    uint8_t b_hi[kD * 256];       // Q as bf16 pieces, B operand [channel][component]
    uint8_t b_lo[kD * 256];
  } tc;
  // scale and zero point (s, z) of component j in block blk at zsT[j % 8][blk][j / 8]:
  // the 16 threads that share a token read 16 consecutive entries
  float2 zsT[8][kMaxCt / kTile][kD / 8];
  // values with per-token ranges: each token's zero point, and its range in
  // 2^b - 1 steps for each width b
  float kz[kMaxCt];
  float ks[kMaxCt][8];
  CompInfo ci;
  uint64_t bar;
  uint32_t base[kBatchMax + 1];
  uint32_t tmem_base;
};

static_assert(sizeof(DecSmem) + 1024 <= 232448, "decoder shared memory exceeds the per-block limit");
static_assert(sizeof(EntSmem) + 1024 <= 233472 / 5, "entropy kernel should fit five blocks per SM");

constexpr uint32_t kTThreads = 512;  // tensor stage: 16 warps, four per tensor-memory lane quarter

__global__ void __launch_bounds__(kTThreads, 1)
k_transform_decode(TransformShape sh, TransformPlanDev pl, FrameBatch b, uint8_t* ws, uint32_t max_records) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  // the swizzled operand tiles need 1024-byte-aligned shared addresses
  const uint32_t pad = (1024u - (tc::smem_addr(smem_raw) & 1023u)) & 1023u;
  DecSmem& S = *reinterpret_cast<DecSmem*>(smem_raw + pad);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t warp = tid >> 5, lane = tid & 31u;
  if (tid == 0) {  // records of the batch: prefix over frames that passed the header check
    uint32_t acc = 0;
    for (uint32_t f = 0; f < b.n; ++f) {
      S.base[f] = acc;
      const DecodeState* d = decode_state(ws, f);
      acc += d->status == kOk ? d->n_records : 0u;
    }
    S.base[b.n] = acc;
  }
  __syncthreads();
  const uint32_t nrec = S.base[b.n];
  const uint32_t per = (nrec + gridDim.x - 1) / gridDim.x;
  const uint32_t rbeg = blockIdx.x * per, rend = min(nrec, rbeg + per);
  if (rbeg >= rend) return;
  const CodeBlocks cb = code_blocks(ws, max_records, sh.ct);
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, kTcCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) tc::mbar_init(&S.bar, 1);
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  uint32_t phase = 0;
  bool alive = true, drained = true;
  const uint32_t rps = 1u + sh.n_mid;
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcRows, kD);
  uint32_t cur_sidx = 0xffffffffu;  // slice whose component order and Q pieces are loaded
  for (uint32_t g = rbeg; g < rend && alive; ++g) {
    const uint32_t fr = frame_of(S.base, b.n, g), r = g - S.base[fr];
    const uint32_t ls = r / rps, kind = r % rps;
    if (kind == 0 || cb.status[g] != uint32_t(kOk)) continue;  // raw record, or one the entropy stage refused
    __syncthreads();
    const uint8_t* src = b.f[fr].src;
    uint16_t* dst = reinterpret_cast<uint16_t*>(b.f[fr].dst);
    DecodeState* ds = decode_state(ws, fr);
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint8_t* rec = src + ld_u64(e);
    const uint32_t sidx = ds->first_slice + ls;
    const bool is_key = ((sidx / sh.H) & 1u) == 0;
    uint16_t* xs = dst + uint64_t(ls) * sh.T * kD;
    const uint32_t c = kind - 1;
    const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
    const uint32_t nb = (tcc + kTile - 1) / kTile;
    const uint8_t* codes = cb.codes + uint64_t(g) * sh.ct * kCodeRow;
    if (sidx != cur_sidx) {
      load_comp_info(pl.comp + sidx, S.ci);
      // the B operand: Q of this slice as bf16 pieces (b_hi and b_lo are contiguous)
      const uint4* q4 = reinterpret_cast<const uint4*>(pl.qsplit + uint64_t(sidx) * kQSplitBytes);
      uint4* b4 = reinterpret_cast<uint4*>(S.tc.b_hi);
      for (uint32_t i = tid; i < kQSplitBytes / 16u; i += nthr) b4[i] = __ldg(q4 + i);
      cur_sidx = sidx;
    }
    // this thread's A-operand components j0 .. j0 + 7 and which of them are coded
    const uint32_t j0 = 8u * (tid & 15u);
    const bool kiv = sh.kivi && !is_key;  // values with per-token ranges
    uint32_t wmask = 0, wpack = 0;  // coded components; their widths - 1, 4 bits each
#pragma unroll
    for (uint32_t i = 0; i < 8; ++i) {
      const uint32_t bw = S.ci.width[j0 + i];
      wmask |= bw ? (1u << i) : 0u;
      wpack |= (bw ? bw - 1u : 0u) << (4u * i);
    }
    if (kiv) {  // each token's zero point and range, decoded from the side streams by the entropy stage
      const float2* p64 = cb.zs + uint64_t(g) * kD * (sh.ct / kTile);
      for (uint32_t t = tid; t < tcc; t += nthr) {
        const float2 zr = __ldg(p64 + t);
        S.kz[t] = zr.x;
#pragma unroll
        for (uint32_t bw = 1; bw <= 8; ++bw)
          if (S.ci.bcount[bw]) S.ks[t][bw - 1] = zr.y == 0.0f ? 0.0f : __fdiv_rn(zr.y, float((1u << bw) - 1u));
      }
    } else if (tid < kD && S.ci.width[tid]) {  // all of the component's (z, s) pairs are loaded before any is stored
      // decoded from the record's side streams by the entropy stage
      const float2* p64 = cb.zs + (uint64_t(g) * kD + S.ci.coded_idx[tid]) * (sh.ct / kTile);
      float2 zs[kMaxCt / kTile];
#pragma unroll
      for (uint32_t blk = 0; blk < kMaxCt / kTile; ++blk) zs[blk] = blk < nb ? __ldg(p64 + blk) : make_float2(0.f, 0.f);
#pragma unroll
      for (uint32_t blk = 0; blk < kMaxCt / kTile; ++blk)
        if (blk < nb) S.zsT[tid & 7u][blk][tid >> 3] = zs[blk];
    }
    // inverse projection on the tensor cores, 128 tokens at a time:
    // x^[t][k] = sum_j y^[t][j] Q[k][j] with y^ and Q split into bf16 hi + lo
    // pieces (hi*hi + hi*lo + lo*hi, fp32 accumulation in tensor memory).
    // Item k of this thread: token tt = tid / 16 + 32 k, components j0 .. j0 + 7
    // (the same for all its items) -> one 16-byte chunk of each piece. A tile's
    // codes are loaded while the previous tile's products run (the first tile's
    // here), so that their latency overlaps the tensor cores and the epilogue.
    constexpr uint32_t kItems = kTcRows * (kD / 8u) / kTThreads;
    static_assert(kItems == 4 && kTcRows == 2 * kTile, "item k lies in the tile's block k / 2");
    uint2 cw8[kItems];
    auto load_codes = [&](uint32_t tb) {
      const uint32_t n = min(kTcRows, tcc - tb);
#pragma unroll
      for (uint32_t k = 0; k < kItems; ++k) {
        const uint32_t tt = (tid >> 4) + 32u * k;
        cw8[k] = tt < n ? __ldcg(reinterpret_cast<const uint2*>(codes + (tb + tt) * kCodeRow + j0)) : make_uint2(0, 0);
      }
    };
    load_codes(0);
    for (uint32_t t_base = 0; t_base < tcc; t_base += kTcRows) {
      const uint32_t bl = min(kTcRows, tcc - t_base);
      __syncthreads();
      // the scales and zero points of the tile's two blocks come from shared memory once
      float2 zr[2][8];
#pragma unroll
      for (uint32_t b2 = 0; b2 < 2; ++b2)
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) zr[b2][i] = S.zsT[i][t_base / kTile + b2][tid & 15u];
#pragma unroll
      for (uint32_t k = 0; k < kItems; ++k) {
        const uint32_t tt = (tid >> 4) + 32u * k;
        float v[8];
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) v[i] = 0.0f;
        if (tt < bl) {
          const uint32_t c4[2] = {cw8[k].x, cw8[k].y};
#pragma unroll
          for (uint32_t i = 0; i < 8; ++i) {
            float2 zs = zr[k >> 1][i];
            if (kiv) zs = make_float2(S.kz[t_base + tt], S.ks[t_base + tt][(wpack >> (4u * i)) & 15u]);
            const float y = __fmaf_rn(float((c4[i >> 2] >> (8u * (i & 3u))) & 0xffu), zs.y, zs.x);
            v[i] = (wmask >> i) & 1u ? y : 0.0f;
          }
        }
        uint32_t h[4], l[4];
#pragma unroll
        for (uint32_t i = 0; i < 4; ++i) {
          h[i] = pack_bf16x2(v[2 * i], v[2 * i + 1]);
          l[i] = pack_bf16x2(__fsub_rn(v[2 * i], bf16_to_f32(h[i] & 0xffffu)),
                             __fsub_rn(v[2 * i + 1], bf16_to_f32(h[i] >> 16)));
        }
        const uint32_t o = tc::sw128_offset(tt, 2u * j0, kTcRows);
        *reinterpret_cast<uint4*>(S.tc.a_hi + o) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4*>(S.tc.a_lo + o) = make_uint4(l[0], l[1], l[2], l[3]);
      }
      tc::fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t ah = tc::smem_addr(S.tc.a_hi), al = tc::smem_addr(S.tc.a_lo);
        const uint32_t bh = tc::smem_addr(S.tc.b_hi), bo = tc::smem_addr(S.tc.b_lo);
        uint32_t acc = 0;
        for (uint32_t ks = 0; ks < kD / 16u; ++ks) {  // K = 16 components per MMA
          const uint32_t koff = (ks >> 2) * (kTcRows * 128u) + (ks & 3u) * 32u;
          const uint32_t kboff = (ks >> 2) * (kD * 128u) + (ks & 3u) * 32u;
          tc::mma_bf16(tmem, tc::desc_sw128(ah + koff), tc::desc_sw128(bh + kboff), idesc, acc);
          acc = 1;
          tc::mma_bf16(tmem, tc::desc_sw128(ah + koff), tc::desc_sw128(bo + kboff), idesc, 1);
          tc::mma_bf16(tmem, tc::desc_sw128(al + koff), tc::desc_sw128(bh + kboff), idesc, 1);
        }
        tc::mma_commit(&S.bar);
      }
      __syncwarp();  // the issuing warp reconverges before its lanes poll the barrier
      // while the MMAs run: this thread's RoPE pairs for the epilogue (warp w:
      // token rows 32 (w % 4) .., channel pairs 16 (w / 4) .. + 16) and the next
      // tile's codes
      float4 rp[8];
      {
        const uint32_t ptt = (warp & 3u) * 32u + lane;
        const float4* cs4 = reinterpret_cast<const float4*>(pl.rope + (uint64_t(t0 + t_base + ptt) * (kD / 2) + (warp >> 2) * 16u) * 2u);
        const bool rl = is_key && ptt < bl;
#pragma unroll
        for (uint32_t i = 0; i < 8; ++i) rp[i] = rl ? __ldg(cs4 + i) : make_float4(0.f, 0.f, 0.f, 0.f);
      }
      if (t_base + kTcRows < tcc) load_codes(t_base + kTcRows);
      const bool done = tc::mbar_wait(&S.bar, phase, KVC_MMA_WAIT_POLLS);
      phase ^= 1u;
      if (!__syncthreads_and(done)) {
        if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrTimeout));
        // drain: the same completion again, with the long bound, so that the
        // accumulator is no longer written when the block frees it
        drained = __syncthreads_and(tc::mbar_wait(&S.bar, phase ^ 1u, kMmaDrainPolls));
        alive = false;
        break;
      }
      tc::fence_after_sync();
      // epilogue: warp w reads token rows 32 (w % 4) .., channel sixteenth w / 4:
      // channels [16q, 16q + 16) and their RoPE partners [16q + 64, 16q + 80)
      {
        const uint32_t sub = warp & 3u, q = warp >> 2;
        const uint32_t tt = sub * 32u + lane;
        const uint32_t c0 = q * 16u;
        uint32_t va[16], vb[16];
        const uint32_t ta = tmem + ((sub * 32u) << 16);
        tc::tmem_ld16(ta + c0, va);
        tc::tmem_ld16(ta + c0 + 64u, vb);
        tc::tmem_wait_ld();
        if (tt < bl) {
          const uint32_t t = t0 + t_base + tt;
          uint32_t pa[8], pb[8];
#pragma unroll
          for (uint32_t i = 0; i < 16; i += 2) {
            float a0 = __uint_as_float(va[i]), b0 = __uint_as_float(vb[i]);
            float a1 = __uint_as_float(va[i + 1]), b1 = __uint_as_float(vb[i + 1]);
            if (is_key) {
              const float4 kk = rp[i >> 1];  // (cos, sin) of pairs i, i + 1
              const float2 k0 = make_float2(kk.x, kk.y), k1 = make_float2(kk.z, kk.w);
              const float na0 = __fsub_rn(__fmul_rn(a0, k0.x), __fmul_rn(b0, k0.y));
              const float nb0 = __fadd_rn(__fmul_rn(a0, k0.y), __fmul_rn(b0, k0.x));
              const float na1 = __fsub_rn(__fmul_rn(a1, k1.x), __fmul_rn(b1, k1.y));
              const float nb1 = __fadd_rn(__fmul_rn(a1, k1.y), __fmul_rn(b1, k1.x));
              a0 = na0; b0 = nb0; a1 = na1; b1 = nb1;
            }
            pa[i >> 1] = pack_bf16x2(a0, a1);
            pb[i >> 1] = pack_bf16x2(b0, b1);
          }
          uint4* ra = reinterpret_cast<uint4*>(xs + uint64_t(t) * kD + c0);
          uint4* rb = reinterpret_cast<uint4*>(xs + uint64_t(t) * kD + c0 + 64u);
          ra[0] = make_uint4(pa[0], pa[1], pa[2], pa[3]);
          ra[1] = make_uint4(pa[4], pa[5], pa[6], pa[7]);
          rb[0] = make_uint4(pb[0], pb[1], pb[2], pb[3]);
          rb[1] = make_uint4(pb[4], pb[5], pb[6], pb[7]);
        }
      }
      tc::fence_before_sync();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  // MMAs still pending after the drain's bound would write tensor memory
  // after it is freed (and handed to another block): the block then keeps its
  // allocation, and the record already carries the timeout status
  if (warp == 0 && drained) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tmem, kTcCols);
  }
}

int g_num_sms = 0;
int num_sms() {
  if (!g_num_sms) {
    int dev = 0;
    cudaGetDevice(&dev);
    cudaDeviceGetAttribute(&g_num_sms, cudaDevAttrMultiProcessorCount, dev);
    if (g_num_sms <= 0) g_num_sms = 148;
  }
  return g_num_sms;
}

}  // namespace

uint64_t transform_slot_bytes(const TransformShape& s) {
  // largest record: side info + up to 8 streams of the codes, or the raw rows
  uint64_t mid = 4u * (16u + pad16_64(kSideMax)) + 8u * 16u + pad16_64(uint64_t(kD) * kMaxCt);
  uint64_t raw = pad16_64(uint64_t(s.s_end + (s.T - s.r_start)) * kD * 2u);
  uint64_t b = (mid > raw ? mid : raw) + kWordsArea + kCodesArea;
  return (b + 255u) & ~uint64_t(255);
}

cudaError_t launch_transform_encode(const TransformShape& s, const TransformPlanDev& p,
                                    const FrameBatch& b, const EncodeLayout& ws, cudaStream_t st) {
  const uint32_t n_slices = b.rec_base[b.n] / (1u + s.n_mid);
  if (n_slices == 0) return cudaSuccess;
  {
    ProfRange pr_("transform_encode_raw", st);
    k_transform_encode_raw<<<n_slices, kThreads, 0, st>>>(s, b, ws);
  }
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess || s.n_mid == 0) return e;
  const uint32_t grid = n_slices * s.n_mid;
  const size_t psmem = sizeof(PtSmem) + 1024;
  static SmemAttr attr_p, attr_e, attr_s;
  e = smem_attr(attr_p, reinterpret_cast<const void*>(k_transform_project), psmem);
  if (e != cudaSuccess) return e;
  e = smem_attr(attr_e, reinterpret_cast<const void*>(k_transform_entropy), sizeof(EntSmem));
  if (e != cudaSuccess) return e;
  e = smem_attr(attr_s, reinterpret_cast<const void*>(k_transform_side), sizeof(SideSmem));
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("transform_project", st);
    k_transform_project<<<min(grid, uint32_t(num_sms())), kPThreads, psmem, st>>>(s, p, b, ws);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("transform_side", st);
    k_transform_side<<<grid, kThreads, sizeof(SideSmem), st>>>(s, p, b, ws);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("transform_entropy", st);
    k_transform_entropy<<<grid, kThreads, sizeof(EntSmem), st>>>(s, p, b, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_transform_decode(const TransformShape& s, const TransformPlanDev& p,
                                    const FrameBatch& b, uint8_t* ws, uint32_t max_records,
                                    cudaStream_t st) {
  if (max_records == 0 || b.n == 0) return cudaSuccess;
  static int ent_blocks_per_sm = 0;
  const size_t esmem = sizeof(DecEntSmem);
  static SmemAttr attr_c, attr_t;
  cudaError_t e = smem_attr(attr_c, reinterpret_cast<const void*>(k_transform_decode_codes), esmem);
  if (e != cudaSuccess) return e;
  if (!ent_blocks_per_sm) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&ent_blocks_per_sm, k_transform_decode_codes, kThreads, esmem);
    if (e != cudaSuccess || ent_blocks_per_sm < 1) ent_blocks_per_sm = 1;
  }
  {
    ProfRange pr_("transform_decode_codes", st);
    const uint32_t grid = min(max_records, uint32_t(num_sms() * ent_blocks_per_sm));
    k_transform_decode_codes<<<grid, kThreads, esmem, st>>>(s, p, b, ws, max_records);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  size_t smem = sizeof(DecSmem) + 1024;
  e = smem_attr(attr_t, reinterpret_cast<const void*>(k_transform_decode), smem);
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("transform_decode", st);
    const uint32_t grid = min(max_records, uint32_t(num_sms()));
    k_transform_decode<<<grid, kTThreads, smem, st>>>(s, p, b, ws, max_records);
  }
  return cudaGetLastError();
}

uint64_t transform_decode_ws_extra(const TransformShape& s, uint64_t records) {
  return ((4u * records + 255u) & ~uint64_t(255)) + records * uint64_t(s.ct) * kCodeRow +
         records * uint64_t(kD) * (s.ct / kTile) * sizeof(float2);
}

}  // namespace kvc
