// Lossless front-end kernels (sm_100a): per chunk of tc tokens x D channels,
// channel-major byte planes (p = 0 low byte, p = 1 high byte), each plane one
// stream record that keeps the smallest of CONST / RANS / RAW (AT-1 Memory
// page, "KV & tensor mode": channel-major reorder, byte planes, keep whichever
// is smaller; QATQ page, "qatq encode": bounded chunks, known row width).
#include <type_traits>
#include "kvc_device.cuh"
#include "tcgen05.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr uint32_t kThreads = 256;  // 8 warps: plane p = warp / 4, group = warp % 4

// Encode: persistent CTAs of 16 warps, a chunk at a time. Warp w codes variant
// v = w / 4: plane 0 (v = 0), plane 1 (v = 1), plane 1's lane deltas (v = 2)
// and plane 0's lane deltas (v = 3), warp % 4 being the rANS group; all 16
// share the histograms, the writes and the CRC.
constexpr uint32_t kEncThreads = 512;
constexpr uint32_t kEncVars = 4;
// rec_len of a full chunk the fast encoder leaves to the general one
constexpr uint32_t kRecLenDefer = kRecLenError | 0xfeu;
__host__ __device__ constexpr uint32_t var_plane(uint32_t v) { return (v == 1u || v == 2u) ? 1u : 0u; }

// Sum of the squared counts of a 256-bin histogram, by one warp (all lanes get
// it). A plane's lane-delta candidate is coded only when its deltas' sum qd is
// strictly larger than the plane's own and 181 qd > n^2 (delta_gate): their
// counts are more concentrated, with a collision entropy under log2(181) bits.
__device__ inline unsigned long long warp_sq_counts(const uint32_t* h) {
  const uint32_t lane = threadIdx.x & 31u;
  unsigned long long q = 0;
#pragma unroll
  for (uint32_t i = 0; i < 8; ++i) {
    const unsigned long long c = h[lane + 32u * i];
    q += c * c;
  }
#pragma unroll
  for (uint32_t o = 16; o; o >>= 1) q += __shfl_xor_sync(0xffffffffu, q, o);
  return q;
}
__device__ inline bool delta_gate(unsigned long long qd, unsigned long long qp, uint32_t n) {
  return qd > qp && 181ull * qd > uint64_t(n) * n;
}

struct __align__(16) EncSmem {
  uint32_t crc_t[1024];
  uint32_t hist[kEncVars][256];
  uint32_t freq[kEncVars][256];
  uint32_t rem[256];
  uint32_t fc[kEncVars][256];
  uint32_t rcp[kEncVars][256];
  uint2 tab[kEncVars][256];      // {f | cum << 16, 1/f} per variant
  uint32_t states[kEncVars][kMaxLanes];
  uint32_t tmp[32], red[32];
  uint32_t k[kEncVars], mode[2], bytes[2], csym[2], var[2];
  uint32_t W[kEncVars][4], wbeg[kEncVars][4], sub_len[kEncVars][4];
  unsigned long long sq[kEncVars];
  uint32_t take;
};

struct __align__(16) DecSmem {
  uint32_t crc_t[1024];
  uint32_t freq[2][256];
  uint32_t cum[2][260];
  uint32_t lut[2][kProbScale];
  uint32_t tmp[32], red[32];
  StreamInfo si[2];
  uint32_t crc_ok;
};

// i -> (d, t) for channel-major index i = d * tcc + t
struct ChanMajor {
  uint32_t tcc, magic;
  __device__ ChanMajor(uint32_t tcc_) : tcc(tcc_), magic(0xffffffffu / tcc_) {}
  __device__ inline void split(uint32_t i, uint32_t& d, uint32_t& t) const {
    d = __umulhi(i, magic);
    t = i - d * tcc;
    if (t >= tcc) { ++d; t -= tcc; }
  }
};

// sel = 0: every record; sel = 1: the ragged last chunk of each slice and the
// full chunks the fast encoder deferred (rec_len kRecLenDefer).
__global__ void __launch_bounds__(kEncThreads)
k_lossless_encode(LosslessShape sh, FrameBatch b, EncodeLayout ws, uint32_t sel) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  EncSmem& S = *reinterpret_cast<EncSmem*>(smem_raw);
  uint16_t* vals = reinterpret_cast<uint16_t*>(smem_raw + sizeof(EncSmem));
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t nrec = b.rec_base[b.n];
  const bool ragged_tail = sh.T % sh.tc != 0;
  crc_tables_init(S.crc_t);
  for (uint32_t gr = blockIdx.x; gr < nrec; gr += gridDim.x) {
  __syncthreads();
  if (tid == 0)
    S.take = sel == 0u || (ragged_tail && (gr - b.rec_base[frame_of(b.rec_base, b.n, gr)]) % sh.cps == sh.cps - 1u) ||
             ws.rec_len[gr] == kRecLenDefer;
  __syncthreads();
  if (!S.take) continue;
  const uint32_t fr = frame_of(b.rec_base, b.n, gr);
  const uint32_t r = gr - b.rec_base[fr];
  const uint16_t* src = reinterpret_cast<const uint16_t*>(b.f[fr].src);
  const uint32_t slice = r / sh.cps, c = r % sh.cps;
  const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0), D = sh.D, n = tcc * D;
  const uint32_t n_max = sh.tc * D;
  const uint16_t* g = src + (uint64_t(slice) * sh.T + t0) * D;

  for (uint32_t i = tid; i < kEncVars * 256u; i += nthr) (&S.hist[0][0])[i] = 0;
  if ((reinterpret_cast<uintptr_t>(g) & 15u) == 0 && (n & 7u) == 0) {
    const uint4* g4 = reinterpret_cast<const uint4*>(g);
    uint4* v4 = reinterpret_cast<uint4*>(vals);
    for (uint32_t q = tid; q < n / 8u; q += nthr) v4[q] = __ldg(g4 + q);
  } else {
    for (uint32_t i = tid; i < n; i += nthr) vals[i] = g[i];
  }
  __syncthreads();
  const uint32_t N = rans_lanes(n), G = rans_groups(N);
  {
    // histograms; stream index of value (t, d) is d * tcc + t, its predecessor in
    // stream order is (t - 1, d), or (tcc - 1, d - 1) at t = 0
    for (uint32_t i = tid; i < n; i += nthr) {
      const uint32_t v = vals[i];
      atomicAdd(&S.hist[0][v & 0xffu], 1u);
      atomicAdd(&S.hist[1][v >> 8], 1u);
      const uint32_t t = i / D, d = i - t * D, si = d * tcc + t;
      uint32_t dv = v;  // the 16-bit XOR with the predecessor: both planes' lane deltas
      if (!lane_start(si, n, N)) dv ^= t ? vals[i - D] : vals[(tcc - 1u) * D + d - 1u];
      atomicAdd(&S.hist[2][dv >> 8], 1u);
      atomicAdd(&S.hist[3][dv & 0xffu], 1u);
    }
  }
  __syncthreads();
  {
    const uint32_t warp = tid >> 5;
    if (warp < kEncVars) {
      const unsigned long long q = warp_sq_counts(S.hist[warp]);
      if ((tid & 31u) == 0) S.sq[warp] = q;
    }
  }
  for (uint32_t v = 0; v < kEncVars; ++v) {
    uint32_t k = block_normalize(S.hist[v], n, S.freq[v], S.rem, S.tmp);
    if (tid == 0) S.k[v] = k;
    block_enc_tables(S.freq[v], S.fc[v], S.rcp[v], S.tmp);
    for (uint32_t i = tid; i < 256; i += nthr) S.tab[v][i] = make_uint2(S.fc[v][i], S.rcp[v][i]);
  }
  __syncthreads();

  const ChanMajor cm(tcc);
  uint8_t* slot = ws.slots + uint64_t(gr) * ws.slot_bytes;
  const uint32_t rec_area = 2u * (16u + pad16(n_max));
  uint16_t* scratch0 = reinterpret_cast<uint16_t*>(slot + rec_area);
  {
    const uint32_t warp = tid >> 5, lane = tid & 31u;
    const uint32_t v = warp >> 2, gg = warp & 3u;
    // variant 2 (3): plane 1's (0's) lane deltas, coded where their counts are more concentrated
    const bool gated = v < 2u || delta_gate(S.sq[v], S.sq[var_plane(v)], n);
    if (v < kEncVars && S.k[v] >= 2 && gg < G && gated) {
      uint32_t b0, len0, b1 = n, len1;
      lane_range(n, N, gg * kGroupLanes, b0, len0);
      if (gg + 1 < G) lane_range(n, N, (gg + 1) * kGroupLanes, b1, len1);
      // symbol i of plane p: byte p of the value of channel d = i / tcc, token t = i % tcc
      const uint8_t* v8 = reinterpret_cast<const uint8_t*>(vals) + var_plane(v);
      uint16_t* scratch = scratch0 + uint64_t(v) * (n_max + 32u);
      uint32_t x, Wg;
      if (v < 2)
        Wg = rans_encode_strided([v8](uint32_t d) { return v8 + 2u * d; }, 2u * D, tcc, n, N, gg, S.tab[v],
                                 scratch + b0, b1 - b0, &x);
      else
        Wg = rans_encode_strided<true>([v8](uint32_t d) { return v8 + 2u * d; }, 2u * D, tcc, n, N, gg,
                                       S.tab[v], scratch + b0, b1 - b0, &x);
      uint32_t l = gg * kGroupLanes + lane;
      if (l < N) S.states[v][l] = x;
      if (lane == 0) {
        S.W[v][gg] = Wg;
        S.wbeg[v][gg] = b0 + (b1 - b0) - Wg;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    // per plane: CONST for one symbol; else the smallest of RANS (plain), RANS of
    // the plane's lane deltas (only if strictly smaller than both others) and RAW
    const uint32_t raw_b = 16u + pad16(n);
    for (uint32_t p = 0; p < 2; ++p) {
      const uint32_t k = S.k[p], vd = p ? 2u : 3u;
      const uint32_t v0 = vals[0];
      S.csym[p] = p ? (v0 >> 8) : (v0 & 0xffu);
      S.var[p] = p;
      if (k == 1) { S.mode[p] = kModeConst; S.bytes[p] = 16; continue; }
      if (k < 2) { S.mode[p] = kModeRaw; S.bytes[p] = raw_b; continue; }
      const uint32_t rb = rans_layout(n, k, S.W[p], S.sub_len[p]);
      uint32_t rd = 0xffffffffu;
      if (S.k[vd] >= 2 && delta_gate(S.sq[vd], S.sq[p], n)) rd = rans_layout(n, S.k[vd], S.W[vd], S.sub_len[vd]);
      if (rd < rb && rd < raw_b) { S.mode[p] = kModeRans; S.bytes[p] = rd; S.var[p] = vd; }
      else if (rb < raw_b) { S.mode[p] = kModeRans; S.bytes[p] = rb; }
      else { S.mode[p] = kModeRaw; S.bytes[p] = raw_b; }
    }
  }
  __syncthreads();
  uint8_t* rec = slot;
  uint32_t off = 0;
  for (uint32_t p = 0; p < 2; ++p) {
    auto raw = [&](uint32_t i) -> uint32_t {
      uint32_t d, t;
      cm.split(i, d, t);
      uint32_t v = vals[t * D + d];
      return p ? (v >> 8) : (v & 0xffu);
    };
    const uint32_t v = S.var[p];
    if (S.mode[p] == kModeRaw && (tcc & 15u) == 0) {
      // raw plane: thread writes 16 tokens of one channel, neighbouring threads neighbouring channels
      if (tid == 0) *reinterpret_cast<uint4*>(rec + off) = make_uint4(kModeRaw, S.bytes[p], n, 0u);
      const uint8_t* v8 = reinterpret_cast<const uint8_t*>(vals) + p;
      for (uint32_t idx = tid; idx < n / 16u; idx += nthr) {
        const uint32_t d = idx % D, tq = 16u * (idx / D);
        uint32_t w[4] = {0, 0, 0, 0};
#pragma unroll
        for (uint32_t k = 0; k < 16; ++k) w[k >> 2] |= uint32_t(v8[2u * ((tq + k) * D + d)]) << (8u * (k & 3u));
        *reinterpret_cast<uint4*>(rec + off + 16u + d * tcc + tq) = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      block_write_stream(rec + off, S.mode[p], n, S.bytes[p], S.csym[p], S.k[v], S.freq[v], S.states[v],
                         scratch0 + uint64_t(v) * (n_max + 32u), S.wbeg[v], S.W[v], S.sub_len[v], raw, S.tmp,
                         v >= 2u ? 1u : 0u);
    }
    off += S.bytes[p];
  }
  __syncthreads();
  uint32_t crc = crc32_block_aligned(rec, off, S.crc_t, S.red);
  if (tid == 0) {
    ws.rec_len[gr] = off;
    ws.rec_crc[gr] = crc;
  }
  }
}

// General decoder: any chunk shape and any plane modes; stages both planes in
// shared memory (one CTA per SM). Runs the records the fast decoder deferred.
__global__ void __launch_bounds__(kThreads)
k_lossless_decode(LosslessShape sh, FrameBatch b, uint8_t* ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  DecSmem& S = *reinterpret_cast<DecSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t D = sh.D, n_max = sh.tc * D;
  uint8_t* planes[2] = {smem_raw + sizeof(DecSmem), smem_raw + sizeof(DecSmem) + pad16(n_max)};
  const uint32_t n_todo = batch_state(ws)->n_deferred;
  if (blockIdx.x >= n_todo) return;
  const unsigned long long* todo = deferred_list(ws);
  crc_tables_init(S.crc_t);
  for (uint32_t i = blockIdx.x; i < n_todo; i += gridDim.x) {
    __syncthreads();
    const uint32_t fr = uint32_t(todo[i] >> 32), r = uint32_t(todo[i]);
    const uint8_t* src = b.f[fr].src;
    uint16_t* dst = reinterpret_cast<uint16_t*>(b.f[fr].dst);
    DecodeState* ds = decode_state(ws, fr);
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint64_t off = ld_u64(e);
    const uint32_t len = ld_u32(e + 8), want = ld_u32(e + 12);
    const uint8_t* rec = src + off;
    const uint32_t slice = r / sh.cps, c = r % sh.cps;
    const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0), n = tcc * D;
    uint32_t got = crc32_block_aligned<true>(rec, len, S.crc_t, S.red);
    if (tid == 0) S.crc_ok = (got == want);
    __syncthreads();
    int st = S.crc_ok ? kOk : kErrCorrupt;
    if (st == kOk) st = block_parse_stream(rec, len, n, &S.si[0], S.freq[0], S.tmp);
    uint32_t b0 = 0;
    if (st == kOk) {
      b0 = S.si[0].bytes;
      st = block_parse_stream(rec + b0, len - b0, n, &S.si[1], S.freq[1], S.tmp);
      if (st == kOk && b0 + S.si[1].bytes != len) st = kErrCorrupt;
    }
    if (st != kOk) {
      if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
      continue;
    }
    const uint8_t* recp[2] = {rec, rec + b0};
    for (uint32_t p = 0; p < 2; ++p) {
      const uint32_t mode = S.si[p].mode;
      if (mode == kModeRans) {
        block_dec_lut(S.freq[p], S.cum[p], S.lut[p], S.tmp);
      } else if (mode == kModeRaw) {
        const uint4* s4 = reinterpret_cast<const uint4*>(recp[p] + 16);
        uint4* d4 = reinterpret_cast<uint4*>(planes[p]);
        for (uint32_t q = tid; q < n / 16u; q += nthr) d4[q] = s4[q];
        for (uint32_t i = (n & ~15u) + tid; i < n; i += nthr) planes[p][i] = recp[p][16 + i];
      } else {
        const uint8_t v = uint8_t(S.si[p].sym);
        for (uint32_t i = tid; i < n; i += nthr) planes[p][i] = v;
      }
    }
    __syncthreads();
    bool ok = true;
    {
      const uint32_t warp = tid >> 5, p = warp >> 2, gg = warp & 3u;
      const uint32_t N = rans_lanes(n), G = rans_groups(N);
      if (S.si[p].mode == kModeRans && gg < G) {
        uint8_t* pl = planes[p];
        // a lane-delta record: each lane's outputs are the running XOR of its symbols
        const uint32_t dm = S.si[p].delta ? 0xffu : 0u;
        uint32_t prev = 0;
        ok = rans_decode_group(recp[p] + S.si[p].sub_off[gg], S.si[p].sub_len[gg], n, N, gg, S.lut[p],
                               [&](uint32_t i, uint32_t s) {
                                 prev = s ^ (prev & dm);
                                 pl[i] = uint8_t(prev);
                               });
      }
    }
    if (!__syncthreads_and(ok)) {
      if (tid == 0)
        atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrCorrupt));
      continue;
    }
    uint16_t* out = dst + (uint64_t(slice) * sh.T + t0) * D;
    if ((D & 7u) == 0 && (reinterpret_cast<uintptr_t>(out) & 15u) == 0) {
      const uint32_t per_row = D / 8u;
      for (uint32_t q = tid; q < tcc * per_row; q += nthr) {
        uint32_t t = q / per_row, d0 = (q - t * per_row) * 8u;
        uint32_t w[4];
        for (uint32_t e2 = 0; e2 < 4; ++e2) {
          uint32_t i0 = (d0 + 2 * e2) * tcc + t, i1 = i0 + tcc;
          uint32_t v0 = planes[0][i0] | (uint32_t(planes[1][i0]) << 8);
          uint32_t v1 = planes[0][i1] | (uint32_t(planes[1][i1]) << 8);
          w[e2] = v0 | (v1 << 16);
        }
        reinterpret_cast<uint4*>(out)[q] = make_uint4(w[0], w[1], w[2], w[3]);
      }
    } else {
      for (uint32_t q = tid; q < n; q += nthr) {
        uint32_t t = q / D, d = q - t * D;
        uint32_t i = d * tcc + t;
        out[q] = uint16_t(planes[0][i] | (uint32_t(planes[1][i]) << 8));
      }
    }
  }
}


// ---------------------------------------------------------------------------
// Fast encoder for full chunks of D = 128 or 64 channels (tc * D = 65536
// values, 16-byte aligned input). 128 threads; thread l is rANS lane l of all
// three variants (lane l: channel l / LPC, tokens (l % LPC) * 512 .. + 512,
// LPC = 128 / D; warp w = rANS group w). Only tables and a small refill ring
// live in shared memory, so several chunks share an SM. Phases:
//  1. histograms of plane 0, plane 1 and plane 1's lane deltas in one pass.
//     Plane 1 and the deltas are counted by runs of equal high bytes along
//     tokens: a delta is zero exactly while a run goes on, so the hot bins see
//     one atomic per run instead of one per value;
//  2. the three frequency tables, one warp each;
//  3. each thread runs its lane's three rANS chains side by side, reading
//     token rows that cp.async stages into a three-slot ring per warp;
//  4. the smallest choice per plane, by the general encoder's rule;
//  5. each thread assembles a contiguous run of the record's 16-byte units
//     (prefix and states from shared memory, words from the scratch, a RAW
//     payload transposed through a shared tile) and folds it into its CRC
//     register; the registers are joined with powers of x.
constexpr uint32_t kFencThreads = 128;
constexpr uint32_t kFencStage = 16;                     // rANS steps per ring stage
constexpr uint32_t kFencSlots = 3;                      // ring slots: 2 stages in flight
constexpr uint32_t kFencRowBytes = 64;                  // one token row of a warp's 32 lanes
constexpr uint32_t kFencSlotBytes = kFencStage * kFencRowBytes;
constexpr uint32_t kGroupWords = kGroupLanes * 512u;    // scratch words of one (variant, group)
constexpr uint32_t kVarWords = kMaxChunkValues + 32u;   // scratch words of one variant
constexpr uint32_t kRecArea = 2u * (16u + kMaxChunkValues);
constexpr uint32_t kXRawPayload = gf2_xpow8(kMaxChunkValues);  // joins a RAW header to its payload

struct __align__(16) FencSmem {
  uint32_t freq[3][256];
  uint2 tab[3][256];
  uint32_t states[3][kMaxLanes];
  union {
    struct {
      uint32_t hist[4][256];                            // plane 0, plane 1, their lane deltas (1, 0)
      uint32_t rem[3][256];
    } h;                                                // phases 1-2
    uint8_t ring[kFencThreads / 32][kFencSlots][kFencSlotBytes];  // phase 3
    struct {
      uint32_t crc_t[1024];
      uint4 tile[256];                                  // RAW planes
    } a;                                                // phase 5
  } u;
  uint4 prefix[2][36];  // RANS record prefix: header, bitmap, frequencies, lengths (<= 576 B)
  uint32_t tmp[32], red[32];
  uint32_t k[3], W[3][4], sub_len[2][4], subst[2][5];
  uint32_t mode[2], bytes[2], var[2], csym[2], pbytes[2], crc[2];
  uint32_t gate[2];  // the lane deltas of plane p are more concentrated than the plane
};

__device__ __forceinline__ uint32_t crc_unit(const uint32_t* t, uint32_t c, uint4 v) {
  c = crc_word(t, c, v.x);
  c = crc_word(t, c, v.y);
  c = crc_word(t, c, v.z);
  return crc_word(t, c, v.w);
}

// One rANS encode step of a warp's 32 lanes (all active): renormalise into the
// group's word area (ascending lanes at ascending addresses), then encode sym.
__device__ __forceinline__ void fenc_step(const uint2* tab, uint32_t sym, uint32_t& x, uint32_t& pos,
                                          uint16_t* words, uint32_t lt) {
  const uint2 e = tab[sym];
  const uint32_t f = e.x & 0xffffu, cum = e.x >> 16;
  const bool emit = x >= (f << 20);
  const uint32_t mask = __ballot_sync(0xffffffffu, emit);
  pos -= __popc(mask);
  if (emit) words[pos + __popc(mask & lt)] = uint16_t(x & 0xffffu);
  const uint32_t xe = emit ? (x >> 16) : x;
  uint32_t q = __umulhi(xe, e.y);
  uint32_t r = xe - q * f;
  const bool over = r >= f;
  q += over ? 1u : 0u;
  r -= over ? f : 0u;
  x = (q << kProbBits) + r + cum;
}

__device__ __forceinline__ uint32_t lds_u16(const uint8_t* p) {
  return *reinterpret_cast<const uint16_t*>(p);
}

template <uint32_t D>
__global__ void __launch_bounds__(kFencThreads, 9)
k_lossless_encode_fast(LosslessShape sh, FrameBatch b, EncodeLayout ws) {
  constexpr uint32_t TCC = kMaxChunkValues / D, LPC = 128u / D;
  constexpr uint32_t CB = D / 8u;                       // 16-byte column blocks of a token row
  constexpr uint32_t SEGLEN = TCC / (kFencThreads / CB);  // tokens per histogram segment (64)
  constexpr uint32_t n = kMaxChunkValues;
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FencSmem& S = *reinterpret_cast<FencSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, lane = tid & 31u, warp = tid >> 5;
  const uint32_t gr = blockIdx.x;  // record of the batch
  const uint32_t fr = frame_of(b.rec_base, b.n, gr), r = gr - b.rec_base[fr];
  const uint32_t slice = r / sh.cps, t0 = (r % sh.cps) * sh.tc;
  if (sh.T - t0 < TCC) return;  // ragged last chunk: the general encoder's
  const uint16_t* g = reinterpret_cast<const uint16_t*>(b.f[fr].src) + (uint64_t(slice) * sh.T + t0) * D;
  const uint4* g4 = reinterpret_cast<const uint4*>(g);

  for (uint32_t i = tid; i < 4u * 256u; i += kFencThreads) (&S.u.h.hist[0][0])[i] = 0;
  __syncthreads();
  {
    // thread: column block cb (8 channels), tokens [tb, tb + SEGLEN); cur[j] and
    // lo[j] are the previous token's high and low bytes (0 before a lane's first
    // token, which makes its delta the byte itself), run[j] the count of equal
    // high bytes so far
    const uint32_t cb = tid % CB, tb = (tid / CB) * SEGLEN;
    const uint4* col = g4 + cb;
    uint32_t cur[8], lo[8], run[8], zeros = 0, zlo = 0;
    if (tb % 512u == 0) {
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j) cur[j] = lo[j] = 0;
    } else {
      const uint4 w = __ldg(col + uint64_t(tb - 1u) * CB);
      const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j) {
        cur[j] = (wv[j >> 1] >> (16u * (j & 1u) + 8u)) & 0xffu;
        lo[j] = (wv[j >> 1] >> (16u * (j & 1u))) & 0xffu;
      }
    }
#pragma unroll
    for (uint32_t j = 0; j < 8; ++j) run[j] = 0;
#pragma unroll 1
    for (uint32_t t = tb; t < tb + SEGLEN; t += 4) {
      uint4 rows[4];
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) rows[i] = __ldg(col + uint64_t(t + i) * CB);
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) {
        const uint32_t wv[4] = {rows[i].x, rows[i].y, rows[i].z, rows[i].w};
#pragma unroll
        for (uint32_t j = 0; j < 8; ++j) {
          const uint32_t v = wv[j >> 1] >> (16u * (j & 1u));
          const uint32_t lb = v & 0xffu, dl = lb ^ lo[j];
          atomicAdd(&S.u.h.hist[0][lb], 1u);
          if (dl) atomicAdd(&S.u.h.hist[3][dl], 1u);
          else ++zlo;
          lo[j] = lb;
          const uint32_t hb = (v >> 8) & 0xffu;
          if (hb == cur[j]) {
            ++run[j];
            ++zeros;
          } else {
            if (run[j]) atomicAdd(&S.u.h.hist[1][cur[j]], run[j]);
            atomicAdd(&S.u.h.hist[2][hb ^ cur[j]], 1u);
            cur[j] = hb;
            run[j] = 1;
          }
        }
      }
    }
#pragma unroll
    for (uint32_t j = 0; j < 8; ++j)
      if (run[j]) atomicAdd(&S.u.h.hist[1][cur[j]], run[j]);
    if (zeros) atomicAdd(&S.u.h.hist[2][0], zeros);
    if (zlo) atomicAdd(&S.u.h.hist[3][0], zlo);
  }
  __syncthreads();
  if (warp < 3) {  // warp v: the table of variant v
    const uint32_t k = warp_normalize(S.u.h.hist[warp], 256u, n, S.freq[warp], S.u.h.rem[warp], S.tab[warp]);
    if (lane == 0) S.k[warp] = k;
  } else {  // warp 3: the lane-delta gates of both planes
    const unsigned long long q0 = warp_sq_counts(S.u.h.hist[0]), q1 = warp_sq_counts(S.u.h.hist[1]);
    const unsigned long long q2 = warp_sq_counts(S.u.h.hist[2]), q3 = warp_sq_counts(S.u.h.hist[3]);
    if (lane == 0) {
      S.gate[0] = delta_gate(q3, q0, n) ? 1u : 0u;
      S.gate[1] = delta_gate(q2, q1, n) ? 1u : 0u;
    }
  }
  __syncthreads();
  if (S.gate[0] && S.k[0] >= 2u) {  // plane 0 codes its lane deltas too: the general encoder's chunk
    if (tid == 0) ws.rec_len[gr] = kRecLenDefer;
    return;
  }
  const bool en0 = S.k[0] >= 2, en1 = S.k[1] >= 2, en2 = en1 && S.k[2] >= 2 && S.gate[1];
  uint8_t* slot = ws.slots + uint64_t(gr) * ws.slot_bytes;
  uint16_t* scratch0 = reinterpret_cast<uint16_t*>(slot + kRecArea);
  {
    // ring stage s holds lane steps tau = 16 s .. 16 s + 15; unit u = 4 j + q of
    // a stage is 16 bytes of token row j: D = 128: channels 32 w + 8 q .. + 7 of
    // token tau; D = 64: channels 16 w + 8 (q & 1) .. + 7 of token (q >> 1) * 512 + tau
    uint16_t* sc0 = scratch0 + warp * kGroupWords;
    uint16_t* sc1 = sc0 + kVarWords;
    uint16_t* sc2 = sc1 + kVarWords;
    const uint8_t* ring = &S.u.ring[warp][0][0];
    const uint32_t ring_saddr = tc::smem_addr(ring);
    const uint32_t loff = LPC == 1 ? 2u * lane : (lane & 1u) * 32u + (lane >> 1) * 2u;
    auto issue = [&](uint32_t s) {
#pragma unroll
      for (uint32_t i = 0; i < 2; ++i) {
        const uint32_t u = lane + 32u * i, j = u >> 2, q = u & 3u;
        const uint32_t row = (LPC == 1 ? 0u : (q >> 1) * 512u) + s * kFencStage + j;
        const uint32_t c0 = LPC == 1 ? 32u * warp + 8u * q : 16u * warp + 8u * (q & 1u);
        const uint16_t* src = g + uint64_t(row) * D + c0;
        const uint32_t dst = ring_saddr + (s % kFencSlots) * kFencSlotBytes + 16u * u;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
      }
      asm volatile("cp.async.commit_group;" ::: "memory");
    };
    const uint32_t lt = lanemask_lt();
    uint32_t x0 = kRansLow, x1 = kRansLow, x2 = kRansLow;
    uint32_t p0 = kGroupWords, p1 = kGroupWords, p2 = kGroupWords;
    constexpr uint32_t kStages = 512u / kFencStage;
    issue(kStages - 1);
    issue(kStages - 2);
    // the chains a chunk codes are fixed before the loop: one instance of the
    // loop per combination, so that no step branches on them
    auto chains = [&](auto E0, auto E1, auto E2) {
      constexpr bool e0 = decltype(E0)::value, e1 = decltype(E1)::value, e2 = decltype(E2)::value;
      uint32_t vcur = 0;
#pragma unroll 1
      for (int s = int(kStages) - 1; s >= 0; --s) {
        __syncwarp();  // every lane is done with the slot the next copy overwrites
        if (s >= 2) issue(uint32_t(s) - 2u);
        else asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 1;" ::: "memory");  // stages s and s - 1 landed
        __syncwarp();
        const uint8_t* cur = ring + (uint32_t(s) % kFencSlots) * kFencSlotBytes + loff;
        const uint8_t* prv = ring + ((uint32_t(s) + kFencSlots - 1u) % kFencSlots) * kFencSlotBytes + loff;
        if (s == int(kStages) - 1) vcur = lds_u16(cur + (kFencStage - 1u) * kFencRowBytes);
#pragma unroll 4
        for (int j = int(kFencStage) - 1; j >= 0; --j) {
          // the value one step earlier in the lane (0 before the lane's first)
          const uint32_t vprev = j ? lds_u16(cur + uint32_t(j - 1) * kFencRowBytes)
                                   : (s ? lds_u16(prv + (kFencStage - 1u) * kFencRowBytes) : 0u);
          const uint32_t hb = vcur >> 8;
          if constexpr (e0) fenc_step(S.tab[0], vcur & 0xffu, x0, p0, sc0, lt);
          if constexpr (e1) fenc_step(S.tab[1], hb, x1, p1, sc1, lt);
          if constexpr (e2) fenc_step(S.tab[2], hb ^ (vprev >> 8), x2, p2, sc2, lt);
          vcur = vprev;
        }
      }
    };
    using T1 = std::true_type;
    using F0 = std::false_type;
    if (en2) {  // en2 implies en1
      if (en0) chains(T1{}, T1{}, T1{});
      else chains(F0{}, T1{}, T1{});
    } else if (en1) {
      if (en0) chains(T1{}, T1{}, F0{});
      else chains(F0{}, T1{}, F0{});
    } else {
      if (en0) chains(T1{}, F0{}, F0{});
      else chains(F0{}, F0{}, F0{});
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
    S.states[0][tid] = x0;
    S.states[1][tid] = x1;
    S.states[2][tid] = x2;
    if (lane == 0) {
      S.W[0][warp] = kGroupWords - p0;
      S.W[1][warp] = kGroupWords - p1;
      S.W[2][warp] = kGroupWords - p2;
    }
  }
  __syncthreads();
  if (tid == 0) {
    // per plane: CONST for one symbol; else the smallest of RANS (plain), RANS of
    // the lane deltas (plane 1, only if strictly smaller than both others) and RAW
    const uint32_t raw_b = 16u + n, v0 = g[0];
    for (uint32_t p = 0; p < 2; ++p) {
      const uint32_t k = S.k[p];
      S.csym[p] = p ? (v0 >> 8) : (v0 & 0xffu);
      S.var[p] = p;
      if (k == 1) {
        S.mode[p] = kModeConst;
        S.bytes[p] = 16;
        continue;
      }
      const uint32_t rb = rans_layout(n, k, S.W[p], S.sub_len[p]);
      uint32_t rd = 0xffffffffu, dl[4];
      if (p == 1 && S.k[2] >= 2 && S.gate[1]) rd = rans_layout(n, S.k[2], S.W[2], dl);
      if (rd < rb && rd < raw_b) {
        S.mode[p] = kModeRans;
        S.bytes[p] = rd;
        S.var[p] = 2;
        for (uint32_t q = 0; q < 4; ++q) S.sub_len[p][q] = dl[q];
      } else if (rb < raw_b) {
        S.mode[p] = kModeRans;
        S.bytes[p] = rb;
      } else {
        S.mode[p] = kModeRaw;
        S.bytes[p] = raw_b;
      }
      if (S.mode[p] == kModeRans) {
        const uint32_t pb = pad16(48u + 2u * S.k[S.var[p]]) + 16u;
        S.pbytes[p] = pb;
        uint32_t o = pb;
        for (uint32_t q = 0; q < 4; ++q) {
          S.subst[p][q] = o;
          o += pad16(S.sub_len[p][q]);
        }
        S.subst[p][4] = o;
      }
    }
  }
  for (uint32_t i = tid; i < 2u * 36u; i += kFencThreads) (&S.prefix[0][0])[i] = make_uint4(0, 0, 0, 0);
  crc_tables_init(S.u.a.crc_t);  // synchronises
  // RANS prefixes: header, presence bitmap, frequencies of present symbols, sub-stream lengths
  for (uint32_t p = 0; p < 2; ++p) {
    if (S.mode[p] != kModeRans) continue;
    const uint32_t v = S.var[p], k = S.k[v];
    uint8_t* pf = reinterpret_cast<uint8_t*>(S.prefix[p]);
    const uint32_t* fq = S.freq[v];
    if (tid == 0)
      *reinterpret_cast<uint4*>(pf) = make_uint4(kModeRans | (4u << 16) | ((v == 2 ? 1u : 0u) << 24), S.bytes[p], n, k);
    for (uint32_t wd = warp; wd < 8; wd += kFencThreads / 32u) {
      const uint32_t bits = __ballot_sync(0xffffffffu, fq[32u * wd + lane] != 0u);
      if (lane == 0) reinterpret_cast<uint32_t*>(pf + 16)[wd] = bits;
    }
    const uint32_t s0 = 2u * tid, f0 = fq[s0], f1 = fq[s0 + 1u];
    uint32_t idx = block_exclusive_scan((f0 ? 1u : 0u) + (f1 ? 1u : 0u), S.tmp, nullptr);
    uint16_t* fl = reinterpret_cast<uint16_t*>(pf + 48);
    if (f0) fl[idx++] = uint16_t(f0);
    if (f1) fl[idx] = uint16_t(f1);
    if (tid < 4) reinterpret_cast<uint32_t*>(pf + S.pbytes[p] - 16u)[tid] = S.sub_len[p][tid];
  }
  __syncthreads();
  uint8_t* rec = slot;
  uint32_t off = 0;
  for (uint32_t p = 0; p < 2; ++p) {
    const uint32_t mode = S.mode[p], bytes = S.bytes[p];
    uint8_t* out = rec + off;
    uint32_t creg = 0;  // CRC register of this plane's stream record (thread 0 after the join)
    if (mode == kModeConst) {
      if (tid == 0) {
        uint4 h = make_uint4(kModeConst | (S.csym[p] << 8), 16u, n, 1u);
        *reinterpret_cast<uint4*>(out) = h;
        if (p == 0) h.x = ~h.x;
        creg = crc_unit(S.u.a.crc_t, 0u, h);
      }
    } else if (mode == kModeRaw) {
      // payload unit 1 + 32 t + i: 16 tokens (block i) of thread t's lane range,
      // i.e. channel t / LPC, tokens (t % LPC) * 512 + 16 i .. + 15; the tile holds
      // those 16 token rows of every lane (both halves for D = 64)
      uint32_t hreg = 0;
      if (tid == 0) {
        uint4 h = make_uint4(kModeRaw, bytes, n, 0u);
        *reinterpret_cast<uint4*>(out) = h;
        if (p == 0) h.x = ~h.x;
        hreg = crc_unit(S.u.a.crc_t, 0u, h);
      }
      auto tile_src = [&](uint32_t i, uint32_t m) -> const uint4* {
        return LPC == 1 ? g4 + (16u * i) * CB + m
                        : g4 + uint64_t((m >> 7) * 512u + 16u * i) * CB + (m & 127u);
      };
      uint4 nx0 = __ldcg(tile_src(0, tid)), nx1 = __ldcg(tile_src(0, tid + 128u));
      const uint8_t* tb = reinterpret_cast<const uint8_t*>(S.u.a.tile) + p +
                          (LPC == 1 ? 2u * tid : (tid & 1u) * 2048u + 2u * (tid >> 1));
      constexpr uint32_t RS = 2u * D;  // tile row stride
#pragma unroll 1
      for (uint32_t i = 0; i < 32; ++i) {
        __syncthreads();
        S.u.a.tile[tid] = nx0;
        S.u.a.tile[tid + 128u] = nx1;
        __syncthreads();
        if (i + 1 < 32) {
          nx0 = __ldcg(tile_src(i + 1, tid));
          nx1 = __ldcg(tile_src(i + 1, tid + 128u));
        }
        uint32_t w[4];
#pragma unroll
        for (uint32_t e = 0; e < 4; ++e)
          w[e] = uint32_t(tb[(4u * e) * RS]) | (uint32_t(tb[(4u * e + 1u) * RS]) << 8) |
                 (uint32_t(tb[(4u * e + 2u) * RS]) << 16) | (uint32_t(tb[(4u * e + 3u) * RS]) << 24);
        const uint4 val = make_uint4(w[0], w[1], w[2], w[3]);
        *reinterpret_cast<uint4*>(out + 16u * (1u + 32u * tid + i)) = val;
        creg = crc_unit(S.u.a.crc_t, creg, val);
      }
      creg = crc_join_lanes(creg, 32u, S.red);
      if (tid == 0) creg = gf2_mul(hreg, kXRawPayload) ^ creg;
    } else {
      // RANS: thread t owns units [t q, t q + q) of the record right-aligned in
      // 128 q units (leading zero units leave a zero register unchanged)
      const uint32_t v = S.var[p], U = bytes >> 4, q = (U + 127u) >> 7, z = 128u * q - U;
      const uint16_t* scv = scratch0 + v * kVarWords;
      for (uint32_t i = 0; i < q; ++i) {
        const int32_t u = int32_t(tid * q + i) - int32_t(z);
        if (u < 0) continue;
        const uint32_t o = 16u * uint32_t(u);
        uint4 val;
        if (o < S.pbytes[p]) {
          val = S.prefix[p][u];
        } else {
          uint32_t gg = 0;
          while (gg < 3 && o >= S.subst[p][gg + 1]) ++gg;
          const uint32_t ro = o - S.subst[p][gg];
          if (ro < 4u * kGroupLanes) {
            val = *reinterpret_cast<const uint4*>(&S.states[v][kGroupLanes * gg + (ro >> 2)]);
          } else {
            const uint32_t wi = (ro - 4u * kGroupLanes) >> 1, Wg = S.W[v][gg];
            const uint16_t* src = scv + gg * kGroupWords + (kGroupWords - Wg);
            uint32_t w[4];
#pragma unroll
            for (uint32_t e = 0; e < 4; ++e) {
              const uint32_t i0 = wi + 2u * e;
              const uint32_t lo = i0 < Wg ? uint32_t(src[i0]) : 0u;
              const uint32_t hi = i0 + 1u < Wg ? uint32_t(src[i0 + 1u]) : 0u;
              w[e] = lo | (hi << 16);
            }
            val = make_uint4(w[0], w[1], w[2], w[3]);
          }
        }
        *reinterpret_cast<uint4*>(out + o) = val;
        if (p == 0 && u == 0) val.x = ~val.x;
        creg = crc_unit(S.u.a.crc_t, creg, val);
      }
      creg = crc_join_lanes(creg, q, S.red);
    }
    if (tid == 0) S.crc[p] = creg;
    off += bytes;
  }
  if (tid == 0) {
    const uint32_t c = gf2_mul(S.crc[0], gf2_xpow8(S.bytes[1])) ^ S.crc[1];
    ws.rec_len[gr] = off;
    ws.rec_crc[gr] = c ^ 0xffffffffu;
  }
}

// ---------------------------------------------------------------------------
// Fast decoder for full chunks of D = 128 or 64 channels (tc * D = 65536
// values): every stream then has 128 lanes of 512 symbols and lane l's symbol
// tau sits at channel-major index l * 512 + tau in both planes, i.e. channel
// l / lpc, token (l % lpc) * 512 + tau with lpc = 128 / D. Thread l owns lane l
// of both planes (warp w = rANS group w), decodes token-synchronously, merges
// the other plane's raw bytes from registers and stores the values straight
// to the token-major output, two channels per 32-bit store after one exchange
// between neighbouring channels. Records with two rANS planes or other shapes
// are deferred to the general decoder.
//
// The record's CRC is checked without a second pass over the raw plane: each
// lane folds its own 512 raw bytes into a CRC register as it consumes them, a
// short pre-pass covers the other stream record, and the pieces are joined
// with powers of x (crc(A || B) = crc(A) * x^(8|B|) + crc(B)). The output of a
// record that fails the check is unspecified, as for every decode error.
constexpr uint32_t kFastThreads = 128;
constexpr uint32_t kRawStream = 16u + kMaxChunkValues;  // bytes of a full-chunk RAW stream record

struct __align__(16) FastSmem {
  uint32_t crc_t[1024];
  uint32_t lut[kProbScale];
  union {
    uint16_t ring[kFastThreads / 32][1024];  // per-group window of rANS refill words
    uint32_t cum[260];                       // table build scratch; the build ends before any refill
  };
  uint32_t freq[2][256];
  uint32_t tmp[32], red[32];
  StreamInfo si[2];
  uint32_t base[kBatchMax + 1];
};

// One rANS lane of a 32-lane group (warp-synchronous). Refill words come from
// the group's window in shared memory (word i at ring[i % 1024]). A lane whose
// index runs past the sub-stream reads a stale word, but then the group's word
// count ends above the sub-stream's and the final check rejects the record.
struct LaneRans {
  uint32_t x, pos, W;
  const uint16_t* ring;
  __device__ __forceinline__ uint32_t step(const uint32_t* lut, uint32_t lt) {
    const uint32_t e = lut[x & (kProbScale - 1u)];
    x = (e >> 20) * (x >> kProbBits) + ((e >> 8) & 0xfffu);
    const bool need = x < kRansLow;
    const uint32_t mask = __ballot_sync(0xffffffffu, need);
    const uint32_t w = ring[(pos + __popc(mask & lt)) & 1023u];
    x = need ? ((x << 16) | w) : x;
    pos += __popc(mask);
    return e;  // symbol in the low byte
  }
};

// The refill window of one group: 16-byte units of the sub-stream's words are
// copied asynchronously into a 1024-word ring. At every stage (8 decode steps,
// at most 256 words consumed) the group waits for all but the newest copy
// group, then requests units up to 1024 words past the unit holding `pos`, so
// a unit is only overwritten once every word in it has been consumed and the
// words of the coming stage were requested at least one stage earlier. Units
// past the last word stay inside the record: sub-streams are padded to 16
// bytes and start 16-byte aligned.
struct RefillWindow {
  const uint8_t* units;  // first refill word, 16-byte aligned
  uint32_t n_units, loaded, ring_saddr;
  __device__ __forceinline__ void request(uint32_t pos, uint32_t lane) {
    const uint32_t target = min(n_units, (pos >> 3) + 128u);
    for (uint32_t u = loaded + lane; u < target; u += 32u)
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(ring_saddr + ((u & 127u) << 4)),
                   "l"(units + (uint64_t(u) << 4))
                   : "memory");
    asm volatile("cp.async.commit_group;" ::: "memory");
    loaded = max(loaded, target);
  }
  __device__ __forceinline__ void settle() {  // all but the newest group landed, visible to the warp
    asm volatile("cp.async.wait_group 1;" ::: "memory");
    __syncwarp();
  }
};

// Value of step j (low 16 bits; the high half is don't-care) from the two
// planes' bytes: a RAW plane gives byte j % 4 of its word r, a rANS plane the
// low byte of the table entry, a CONST plane its symbol.
template <uint32_t M0, uint32_t M1>
__device__ __forceinline__ uint32_t merge_planes(uint32_t j, uint32_t a, uint32_t b) {
  constexpr bool raw0 = M0 == kModeRaw, raw1 = M1 == kModeRaw;
  const uint32_t s0 = raw0 ? (j & 3u) : 0u;
  const uint32_t s1 = raw1 ? 4u + (j & 3u) : 4u;
  return __byte_perm(a, b, s0 | (s1 << 4));
}

// CRC register of this thread's run of the pre-pass region (the record bytes
// the tiles do not see: everything but the RAW payloads). Thread t owns a run
// of q 16-byte units, q = ceil(len / 2048), right-aligned (leading zero units,
// which leave a zero register unchanged; comp complements the record's first
// four bytes, the standard CRC's initial value) or left-aligned (trailing zero
// units, processed: the result is then multiplied by x^(8 * (2048q - len))).
// It runs before the tiles, four loads ahead, so that none of its state is
// live during the decode loop.
struct PreRun {
  const uint8_t* p;
  uint32_t len, q;
  int32_t run0;
  bool left, comp;
  uint32_t c;
  __device__ __forceinline__ void run(const uint8_t* base, uint32_t n, bool left_aligned, bool comp_first,
                                      const uint32_t* t) {
    p = base;
    len = n;
    q = (n + 2047u) >> 11;
    left = left_aligned;
    comp = comp_first;
    run0 = int32_t(threadIdx.x * 16u * q) - (left ? 0 : int32_t(128u * 16u * q - n));
    c = 0;
    for (uint32_t u0 = 0; u0 < q; u0 += 4u) {
      uint4 v[4];
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) {
        const int32_t off = run0 + int32_t(16u * (u0 + i));
        const bool in = u0 + i < q && off >= 0 && uint32_t(off) < len;
        v[i] = in ? __ldcg(reinterpret_cast<const uint4*>(p + off)) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (uint32_t i = 0; i < 4; ++i) {
        const int32_t off = run0 + int32_t(16u * (u0 + i));
        if (u0 + i < q && (left || off >= 0)) {
          if (comp && off == 0) v[i].x = ~v[i].x;
          c = crc_word(t, c, v[i].x);
          c = crc_word(t, c, v[i].y);
          c = crc_word(t, c, v[i].z);
          c = crc_word(t, c, v[i].w);
        }
      }
    }
  }
};

// Decode the 16 tiles of 32 steps of one record. crc0 / crc1 return the CRC
// register of this lane's 512 bytes of plane 0 / 1 when that plane is RAW.
template <uint32_t M0, uint32_t M1, uint32_t D>
__device__ inline bool fast_tiles(FastSmem& S, const uint8_t* const recp[2], uint16_t* out,
                                  uint32_t& crc0, uint32_t& crc1) {
  constexpr uint32_t LPC = 128u / D;  // lanes per channel
  constexpr bool kRaw0 = M0 == kModeRaw, kRaw1 = M1 == kModeRaw;
  constexpr bool kRans = (M0 == kModeRans || M1 == kModeRans);
  constexpr uint32_t RP = (M0 == kModeRans) ? 0u : 1u;  // the rANS plane, if any
  const uint32_t l = threadIdx.x, lane = l & 31u, g = l >> 5;
  const uint32_t lt = lanemask_lt();
  // Lane l decodes channel ch = l / LPC of tokens (l % LPC) * 512 + j and
  // stores each value as it comes: the warp's 32 lanes write 64 contiguous
  // bytes of a token row (two rows for D = 64), whole 32-byte sectors.
  const uint32_t ch = l / LPC;
  uint16_t* o16 = out + uint64_t(l % LPC) * 512u * D + ch;
  LaneRans rs{kRansLow, 0, 0, S.ring[g]};
  RefillWindow win{nullptr, 0, 0, tc::smem_addr(S.ring[g])};
  const uint8_t* raw0 = recp[0] + 16 + l * 512u;
  const uint8_t* raw1 = recp[1] + 16 + l * 512u;
  const uint32_t c0 = S.si[0].sym, c1 = S.si[1].sym;
  bool live = true;
  if (kRans) {
    const StreamInfo& si = S.si[RP];
    const uint8_t* sub = recp[RP] + si.sub_off[g];
    const uint32_t sl = si.sub_len[g];
    if (sl < 128u || (sl & 1u)) live = false;
    else {
      rs.x = reinterpret_cast<const uint32_t*>(sub)[lane];
      rs.W = (sl - 128u) >> 1;
      win.units = sub + 128;
      win.n_units = (rs.W + 7u) >> 3;
    }
    if (!__all_sync(0xffffffffu, live)) return false;
    win.request(0, lane);
    asm volatile("cp.async.commit_group;" ::: "memory");  // empty group: the first settle waits for the window
  }
  // lane deltas: each decoded symbol is XORed with the lane's previous output
  const uint32_t dm = (kRans && S.si[RP].delta) ? 0xffu : 0u;
  uint32_t prev = 0;
  uint4 n0a = make_uint4(0, 0, 0, 0), n0b = n0a, n1a = n0a, n1b = n0a;  // next tile's raw bytes
  if (kRaw0) { n0a = __ldcg(reinterpret_cast<const uint4*>(raw0)); n0b = __ldcg(reinterpret_cast<const uint4*>(raw0 + 16)); }
  if (kRaw1) { n1a = __ldcg(reinterpret_cast<const uint4*>(raw1)); n1b = __ldcg(reinterpret_cast<const uint4*>(raw1 + 16)); }
  uint32_t k0 = 0, k1 = 0;  // CRC registers of the raw runs
#pragma unroll 1
  for (uint32_t k = 0; k < 16; ++k) {
    uint32_t r0[8], r1[8];
    if (kRaw0) {
      r0[0] = n0a.x; r0[1] = n0a.y; r0[2] = n0a.z; r0[3] = n0a.w;
      r0[4] = n0b.x; r0[5] = n0b.y; r0[6] = n0b.z; r0[7] = n0b.w;
      if (k + 1 < 16) {
        n0a = __ldcg(reinterpret_cast<const uint4*>(raw0 + 32u * (k + 1)));
        n0b = __ldcg(reinterpret_cast<const uint4*>(raw0 + 32u * (k + 1) + 16u));
      }
    }
    if (kRaw1) {
      r1[0] = n1a.x; r1[1] = n1a.y; r1[2] = n1a.z; r1[3] = n1a.w;
      r1[4] = n1b.x; r1[5] = n1b.y; r1[6] = n1b.z; r1[7] = n1b.w;
      if (k + 1 < 16) {
        n1a = __ldcg(reinterpret_cast<const uint4*>(raw1 + 32u * (k + 1)));
        n1b = __ldcg(reinterpret_cast<const uint4*>(raw1 + 32u * (k + 1) + 16u));
      }
    }
    uint16_t* o = o16 + (k * 32u) * D;
    // four stages of 8 steps, unrolled so that raw word indices and output
    // offsets are constants; stage st consumes raw words 2 st and 2 st + 1
#pragma unroll
    for (uint32_t st = 0; st < 4; ++st) {
      if (kRans) {
        win.settle();
        win.request(rs.pos, lane);
      }
#pragma unroll
      for (uint32_t j = 0; j < 8; ++j) {
        const uint32_t jj = 8u * st + j;
        uint32_t e = 0u;
        if (kRans) {
          e = rs.step(S.lut, lt) ^ (prev & dm);
          prev = e;
        }
        const uint32_t a = kRaw0 ? r0[jj >> 2] : (M0 == kModeRans ? e : c0);
        const uint32_t b = kRaw1 ? r1[jj >> 2] : (M1 == kModeRans ? e : c1);
        o[jj * D] = uint16_t(merge_planes<M0, M1>(jj, a, b));
      }
      if (kRaw0) k0 = crc_word(S.crc_t, crc_word(S.crc_t, k0, r0[2 * st]), r0[2 * st + 1]);
      if (kRaw1) k1 = crc_word(S.crc_t, crc_word(S.crc_t, k1, r1[2 * st]), r1[2 * st + 1]);
    }
  }
  crc0 = k0;
  crc1 = k1;
  if (kRans) asm volatile("cp.async.wait_group 0;" ::: "memory");  // no copy outlives the record
  return !kRans || (rs.pos == rs.W && rs.x == kRansLow);
}

template <uint32_t D>
__device__ inline bool fast_dispatch(FastSmem& S, const uint8_t* const recp[2], uint16_t* out,
                                     uint32_t m0, uint32_t m1, uint32_t& crc0, uint32_t& crc1) {
  if (m0 == kModeRaw && m1 == kModeRans) return fast_tiles<kModeRaw, kModeRans, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeRaw && m1 == kModeRaw) return fast_tiles<kModeRaw, kModeRaw, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeRaw && m1 == kModeConst) return fast_tiles<kModeRaw, kModeConst, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeRans && m1 == kModeRaw) return fast_tiles<kModeRans, kModeRaw, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeRans && m1 == kModeConst) return fast_tiles<kModeRans, kModeConst, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeConst && m1 == kModeRans) return fast_tiles<kModeConst, kModeRans, D>(S, recp, out, crc0, crc1);
  if (m0 == kModeConst && m1 == kModeRaw) return fast_tiles<kModeConst, kModeRaw, D>(S, recp, out, crc0, crc1);
  return fast_tiles<kModeConst, kModeConst, D>(S, recp, out, crc0, crc1);
}

// CRC register of a 16-byte stream header; comp complements its first four
// bytes (the record's initial value when the header opens the record)
__device__ inline uint32_t crc_header16(const uint32_t* t, const uint8_t* h, bool comp) {
  uint4 v = __ldcg(reinterpret_cast<const uint4*>(h));
  if (comp) v.x = ~v.x;
  uint32_t c = crc_word(t, 0u, v.x);
  c = crc_word(t, c, v.y);
  c = crc_word(t, c, v.z);
  return crc_word(t, c, v.w);
}

__global__ void __launch_bounds__(kFastThreads, 6)
k_lossless_decode_fast(LosslessShape sh, FrameBatch b, uint8_t* ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FastSmem& S = *reinterpret_cast<FastSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x;
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
  const uint32_t D = sh.D;
  const bool shape_ok = (D * sh.tc == kMaxChunkValues) && (D == 128u || D == 64u);
  crc_tables_init(S.crc_t);
  for (uint32_t g = blockIdx.x; g < nrec; g += gridDim.x) {
    __syncthreads();
    const uint32_t fr = frame_of(S.base, b.n, g), r = g - S.base[fr];
    const uint8_t* src = b.f[fr].src;
    uint16_t* dst = reinterpret_cast<uint16_t*>(b.f[fr].dst);
    DecodeState* ds = decode_state(ws, fr);
    const uint32_t slice = r / sh.cps, c = r % sh.cps;
    const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0);
    bool defer = !shape_ok || tcc != sh.tc;
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint64_t off = ld_u64(e);
    const uint32_t len = ld_u32(e + 8), want = ld_u32(e + 12);
    const uint8_t* rec = src + off;
    int st = kOk;
    if (!defer && len > 2u * kRawStream) defer = true;  // cannot be a valid full-chunk record
    uint32_t b0 = 0, b1 = 0;
    if (!defer) {
      const uint32_t n = kMaxChunkValues;
      st = block_parse_stream(rec, len, n, &S.si[0], S.freq[0], S.tmp);
      if (st == kOk) {
        b0 = S.si[0].bytes;
        st = block_parse_stream(rec + b0, len - b0, n, &S.si[1], S.freq[1], S.tmp);
        b1 = S.si[1].bytes;
        if (st == kOk && b0 + b1 != len) st = kErrCorrupt;
      }
      if (st == kOk) {
        const uint32_t m0 = S.si[0].mode, m1 = S.si[1].mode;
        if (m0 == kModeRans && m1 == kModeRans) defer = true;
        // the pre-pass region must fit one round of runs
        const uint32_t pre = m0 != kModeRaw && m1 != kModeRaw ? len : m0 != kModeRaw ? b0 : m1 != kModeRaw ? b1 : 0u;
        if (pre > 2048u * kCrcRegionMaxUnits) defer = true;
      }
    }
    if (defer) {
      if (tid == 0)
        deferred_list(ws)[atomicAdd(&batch_state(ws)->n_deferred, 1u)] =
            (static_cast<unsigned long long>(fr) << 32) | r;
      continue;
    }
    if (st != kOk) {
      if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
      continue;
    }
    const uint32_t m0 = S.si[0].mode, m1 = S.si[1].mode;
    const bool raw0 = m0 == kModeRaw, raw1 = m1 == kModeRaw;
    // CRC pre-pass region: the bytes the tiles do not see. The whole record when
    // neither plane is RAW, else the other stream record (left-aligned when it
    // follows the RAW stream, so that no shift by its runtime length is needed)
    PreRun pre;
    if (!raw0 && !raw1) pre.run(rec, len, false, true, S.crc_t);
    else if (raw0 && !raw1) pre.run(rec + b0, b1, true, false, S.crc_t);
    else if (!raw0 && raw1) pre.run(rec, b0, false, true, S.crc_t);
    else pre.run(rec, 0, false, false, S.crc_t);
    if (m0 == kModeRans) block_dec_lut(S.freq[0], S.cum, S.lut, S.tmp);
    else if (m1 == kModeRans) block_dec_lut(S.freq[1], S.cum, S.lut, S.tmp);
    const uint8_t* recp[2] = {rec, rec + b0};
    uint16_t* out = dst + (uint64_t(slice) * sh.T + t0) * D;
    uint32_t cr0 = 0, cr1 = 0;
    bool ok = D == 128u ? fast_dispatch<128>(S, recp, out, m0, m1, cr0, cr1)
                        : fast_dispatch<64>(S, recp, out, m0, m1, cr0, cr1);
    const uint32_t prc = !(raw0 && raw1) ? crc_join_lanes(pre.c, pre.q, S.red) : 0u;
    const uint32_t p0 = raw0 ? crc_join_lanes(cr0, 32u, S.red) : 0u;  // 512-byte lane runs
    const uint32_t p1 = raw1 ? crc_join_lanes(cr1, 32u, S.red) : 0u;
    if (tid == 0) {
      const uint32_t x64k = kCrcPow.q[32][7], x16 = kCrcPow.u[1];  // x^(8 * 65536), x^(8 * 16)
      const uint32_t xraw = gf2_mul(x64k, x16);                     // x^(8 * full RAW stream record)
      const uint32_t fin = want ^ 0xffffffffu;
      uint32_t lhs = prc, rhs = fin;
      if (raw0 && !raw1) {
        // register(H0' P0) * x^(8 * 2048q) + pre == register(record') * x^(8 * pad)
        const uint32_t q = (b1 + 2047u) >> 11, pad = 2048u * q - b1;
        const uint32_t hp = gf2_mul(crc_header16(S.crc_t, rec, true), x64k) ^ p0;
        lhs = gf2_mul(hp, kCrcPow.q[q][7]) ^ prc;
        rhs = gf2_mul(fin, kCrcPow.u[pad >> 4]);
      } else if (!raw0 && raw1) {
        lhs = gf2_mul(prc, xraw) ^ gf2_mul(crc_header16(S.crc_t, rec + b0, false), x64k) ^ p1;
      } else if (raw0 && raw1) {
        const uint32_t hp = gf2_mul(crc_header16(S.crc_t, rec, true), x64k) ^ p0;
        lhs = gf2_mul(hp, xraw) ^ gf2_mul(crc_header16(S.crc_t, rec + b0, false), x64k) ^ p1;
      }
      ok = ok && lhs == rhs;
    }
    if (!__syncthreads_and(ok) && tid == 0)
      atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrCorrupt));
  }
}

// ---------------------------------------------------------------------------
// Wide values (f32: four byte planes; QATQ and AT-1 code f32 tensors too).
// Encode: one CTA per chunk, 512 threads. The planes are coded one after
// another through one shared plane buffer of the chunk's size: plane p is
// gathered channel-major from the chunk (which stays in L2 across the
// planes), counted with its lane deltas, its tables built, coded by one warp per
// (variant, rANS group), and its stream record written at the record's
// running offset by the never-worse rule. The record's CRC follows.
struct __align__(16) WideEncSmem {
  uint32_t crc_t[1024];
  uint32_t hist[2][256], freq[2][256], rem[256], fc[2][256], rcp[2][256];
  uint32_t states[2][kMaxLanes];
  uint32_t tmp[32], red[32];
  uint32_t k[2], W[2][4], wbeg[2][4], sub_len[2][4];
  uint32_t mode, bytes, var, off, gate;
};

template <uint32_t E>
__global__ void __launch_bounds__(kEncThreads)
k_lossless_encode_wide(LosslessShape sh, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  WideEncSmem& S = *reinterpret_cast<WideEncSmem*>(smem_raw);
  uint8_t* pl = smem_raw + sizeof(WideEncSmem);  // one plane of the chunk, channel-major
  const uint32_t tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5, lane = tid & 31u;
  const uint32_t gr = blockIdx.x;
  const uint32_t fr = frame_of(b.rec_base, b.n, gr), r = gr - b.rec_base[fr];
  const uint32_t slice = r / sh.cps, c = r % sh.cps;
  const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0), D = sh.D, n = tcc * D;
  const uint32_t n_max = sh.tc * D;
  const uint8_t* g = b.f[fr].src + (uint64_t(slice) * sh.T + t0) * D * E;
  uint8_t* rec = ws.slots + uint64_t(gr) * ws.slot_bytes;
  uint16_t* scratch0 = reinterpret_cast<uint16_t*>(rec + E * (16u + pad16(n_max)));
  const uint32_t N = rans_lanes(n), G = rans_groups(N), raw_b = 16u + pad16(n);
  crc_tables_init(S.crc_t);
  if (tid == 0) S.off = 0;
  for (uint32_t p = 0; p < E; ++p) {
    uint32_t nvar = 2u;  // the plane and its lane deltas
    for (uint32_t i = tid; i < 2u * 256u; i += nthr) (&S.hist[0][0])[i] = 0;
    for (uint32_t q = tid; q < n; q += nthr) {
      const uint32_t t = q / D, d = q - t * D;
      pl[d * tcc + t] = g[uint64_t(q) * E + p];
    }
    __syncthreads();
    for (uint32_t i = tid; i < n; i += nthr) {
      const uint32_t v = pl[i];
      atomicAdd(&S.hist[0][v], 1u);
      atomicAdd(&S.hist[1][lane_start(i, n, N) ? v : (v ^ pl[i - 1])], 1u);
    }
    __syncthreads();
    if (warp == 0) {  // the lane deltas are coded where their counts are more concentrated
      const unsigned long long q0 = warp_sq_counts(S.hist[0]), q1 = warp_sq_counts(S.hist[1]);
      if (lane == 0) S.gate = delta_gate(q1, q0, n) ? 1u : 0u;
    }
    __syncthreads();
    nvar = S.gate ? 2u : 1u;
    for (uint32_t v = 0; v < nvar; ++v) {
      const uint32_t k = block_normalize(S.hist[v], n, S.freq[v], S.rem, S.tmp);
      if (tid == 0) S.k[v] = k;
      block_enc_tables(S.freq[v], S.fc[v], S.rcp[v], S.tmp);
    }
    __syncthreads();
    {
      const uint32_t v = warp >> 2, gg = warp & 3u;
      if (v < nvar && S.k[v] >= 2 && gg < G) {
        uint32_t b0, len0, b1 = n, len1;
        lane_range(n, N, gg * kGroupLanes, b0, len0);
        if (gg + 1 < G) lane_range(n, N, (gg + 1) * kGroupLanes, b1, len1);
        uint16_t* scratch = scratch0 + uint64_t(v) * (n_max + 32u);
        uint32_t x, Wg;
        if (v == 0)
          Wg = rans_encode_group([pl](uint32_t i) -> uint32_t { return pl[i]; }, n, N, gg, S.fc[0], S.rcp[0],
                                 scratch + b0, b1 - b0, &x);
        else
          Wg = rans_encode_group(
              [pl, n, N](uint32_t i) -> uint32_t {
                return lane_start(i, n, N) ? uint32_t(pl[i]) : uint32_t(pl[i] ^ pl[i - 1]);
              },
              n, N, gg, S.fc[1], S.rcp[1], scratch + b0, b1 - b0, &x);
        const uint32_t l = gg * kGroupLanes + lane;
        if (l < N) S.states[v][l] = x;
        if (lane == 0) {
          S.W[v][gg] = Wg;
          S.wbeg[v][gg] = b0 + (b1 - b0) - Wg;
        }
      }
    }
    __syncthreads();
    if (tid == 0) {  // CONST; lane-delta RANS if strictly smaller than plain RANS and RAW; RANS; RAW
      const uint32_t k = S.k[0];
      uint32_t mode = kModeRaw, bytes = raw_b, var = 0;
      if (k == 1) {
        mode = kModeConst;
        bytes = 16;
      } else if (k >= 2) {
        const uint32_t rb = rans_layout(n, k, S.W[0], S.sub_len[0]);
        const uint32_t rd = nvar == 2u && S.k[1] >= 2 ? rans_layout(n, S.k[1], S.W[1], S.sub_len[1]) : 0xffffffffu;
        if (rd < rb && rd < raw_b) {
          mode = kModeRans; bytes = rd; var = 1;
        } else if (rb < raw_b) {
          mode = kModeRans; bytes = rb;
        }
      }
      S.mode = mode; S.bytes = bytes; S.var = var;
    }
    __syncthreads();
    const uint32_t v = S.var;
    block_write_stream(rec + S.off, S.mode, n, S.bytes, uint32_t(pl[0]), S.k[v], S.freq[v], S.states[v],
                       scratch0 + uint64_t(v) * (n_max + 32u), S.wbeg[v], S.W[v], S.sub_len[v],
                       [pl](uint32_t i) -> uint32_t { return pl[i]; }, S.tmp, v);
    __syncthreads();
    if (tid == 0) S.off += S.bytes;
    __syncthreads();
  }
  const uint32_t len = S.off;
  const uint32_t crc = crc32_block_aligned(rec, len, S.crc_t, S.red);
  if (tid == 0) {
    ws.rec_len[gr] = len;
    ws.rec_crc[gr] = crc;
  }
}

// Decode of wide values: persistent CTAs of 256 threads over the batch's
// records. Per record the CRC, then per plane: its stream record checked, a
// RANS table built, the plane decoded into shared memory (one warp per rANS
// group, lane deltas undone per lane) and written as byte p of every value of
// the chunk; the stream records must fill the record exactly.
struct __align__(16) WideDecSmem {
  uint32_t crc_t[1024];
  uint32_t freq[256], cum[260], lut[kProbScale];
  uint32_t tmp[32], red[32];
  StreamInfo si;
  uint32_t crc_ok;
  uint32_t base[kBatchMax + 1];
};

template <uint32_t E>
__global__ void __launch_bounds__(kThreads)
k_lossless_decode_wide(LosslessShape sh, FrameBatch b, uint8_t* ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  WideDecSmem& S = *reinterpret_cast<WideDecSmem*>(smem_raw);
  uint8_t* pl = smem_raw + sizeof(WideDecSmem);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x, warp = tid >> 5;
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
  const uint32_t nrec = S.base[b.n], D = sh.D;
  if (blockIdx.x >= nrec) return;
  crc_tables_init(S.crc_t);
  for (uint32_t g = blockIdx.x; g < nrec; g += gridDim.x) {
    __syncthreads();
    const uint32_t fr = frame_of(S.base, b.n, g), r = g - S.base[fr];
    const uint8_t* src = b.f[fr].src;
    DecodeState* ds = decode_state(ws, fr);
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint64_t roff = ld_u64(e);
    const uint32_t len = ld_u32(e + 8), want = ld_u32(e + 12);
    const uint8_t* rec = src + roff;
    const uint32_t slice = r / sh.cps, c = r % sh.cps;
    const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0), n = tcc * D;
    uint8_t* out = b.f[fr].dst + (uint64_t(slice) * sh.T + t0) * D * E;
    const uint32_t got = crc32_block_aligned<true>(rec, len, S.crc_t, S.red);
    if (tid == 0) S.crc_ok = (got == want);
    __syncthreads();
    int st = S.crc_ok ? kOk : kErrCorrupt;
    const uint32_t N = rans_lanes(n), G = rans_groups(N);
    uint32_t off = 0;
    for (uint32_t p = 0; p < E && st == kOk; ++p) {
      st = block_parse_stream(rec + off, len - off, n, &S.si, S.freq, S.tmp);
      if (st != kOk) break;
      const StreamInfo si = S.si;
      if (si.mode == kModeRans) {
        block_dec_lut(S.freq, S.cum, S.lut, S.tmp);
      } else if (si.mode == kModeRaw) {
        for (uint32_t i = tid; i < n; i += nthr) pl[i] = rec[off + 16u + i];
      } else {
        for (uint32_t i = tid; i < n; i += nthr) pl[i] = uint8_t(si.sym);
      }
      __syncthreads();
      bool ok = true;
      if (si.mode == kModeRans && warp < G) {
        const uint32_t dm = si.delta ? 0xffu : 0u;
        uint32_t prev = 0;
        ok = rans_decode_group(rec + off + si.sub_off[warp], si.sub_len[warp], n, N, warp, S.lut,
                               [&](uint32_t i, uint32_t s) {
                                 prev = s ^ (prev & dm);
                                 pl[i] = uint8_t(prev);
                               });
      }
      if (!__syncthreads_and(ok)) {
        st = kErrCorrupt;
        break;
      }
      for (uint32_t q = tid; q < n; q += nthr) {
        const uint32_t t = q / D, d = q - t * D;
        out[uint64_t(q) * E + p] = pl[d * tcc + t];
      }
      off += si.bytes;
      __syncthreads();  // the plane buffer and the stream info are reused
    }
    if (st == kOk && off != len) st = kErrCorrupt;
    if (st != kOk && tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
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

uint64_t lossless_slot_bytes(const LosslessShape& s) {
  const uint64_t n_max = uint64_t(s.tc) * s.D;
  // the record (a stream per byte plane, each at most RAW), then the word
  // scratch of the variants coded side by side: four for 16-bit values (each
  // plane and its lane deltas), two for wide values (one plane at a time and
  // its lane deltas)
  uint64_t b = s.E * (16u + pad16_64(n_max)) + (s.E == 4u ? 2u : kEncVars) * (2u * n_max + 64u);
  return (b + 255u) & ~uint64_t(255);
}

cudaError_t launch_lossless_encode(const LosslessShape& s, const FrameBatch& b,
                                   const EncodeLayout& ws, cudaStream_t st) {
  const uint32_t nrec = b.rec_base[b.n];
  if (nrec == 0) return cudaSuccess;
  if (s.E == 4u) {  // f32: the plane-at-a-time encoder for every chunk
    const size_t smem = sizeof(WideEncSmem) + pad16(s.tc * s.D);
    static SmemAttr attr;
    cudaError_t e = smem_attr(attr, reinterpret_cast<const void*>(k_lossless_encode_wide<4>), smem);
    if (e != cudaSuccess) return e;
    ProfRange pr_("lossless_encode_wide", st);
    k_lossless_encode_wide<4><<<nrec, kEncThreads, smem, st>>>(s, b, ws);
    return cudaGetLastError();
  }
  // full chunks of 65536 values with D = 128 or 64 and 16-byte aligned input go
  // to the fast encoder; the general one takes the rest (with the fast one, only
  // the ragged last chunk of each slice)
  bool fast = s.tc * s.D == kMaxChunkValues && (s.D == 128u || s.D == 64u);
  for (uint32_t f = 0; f < b.n; ++f)
    if (reinterpret_cast<uintptr_t>(b.f[f].src) & 15u) fast = false;
  cudaError_t e;
  if (fast) {
    const size_t fsmem = sizeof(FencSmem);
    auto kern = s.D == 128u ? k_lossless_encode_fast<128> : k_lossless_encode_fast<64>;
    static SmemAttr attr128, attr64;
    e = smem_attr(s.D == 128u ? attr128 : attr64, reinterpret_cast<const void*>(kern), fsmem);
    if (e != cudaSuccess) return e;
    {
      ProfRange pr_("lossless_encode", st);
      kern<<<nrec, kFencThreads, fsmem, st>>>(s, b, ws);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // the general encoder: every record, or (after the fast one) the ragged last
  // chunks and the chunks it deferred
  size_t smem = sizeof(EncSmem) + pad16(s.tc * s.D * 2u);
  static SmemAttr attr_gen;
  e = smem_attr(attr_gen, reinterpret_cast<const void*>(k_lossless_encode), smem);
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_(fast ? "lossless_encode_tail" : "lossless_encode", st);
    k_lossless_encode<<<min(nrec, uint32_t(num_sms())), kEncThreads, smem, st>>>(s, b, ws, fast ? 1u : 0u);
  }
  return cudaGetLastError();
}

cudaError_t launch_lossless_decode(const LosslessShape& s, const FrameBatch& b, uint8_t* ws,
                                   uint32_t max_records, cudaStream_t st) {
  if (max_records == 0 || b.n == 0) return cudaSuccess;
  if (s.E == 4u) {  // f32: the plane-at-a-time decoder for every record
    const size_t smem = sizeof(WideDecSmem) + pad16(s.tc * s.D);
    static SmemAttr attr;
    cudaError_t e = smem_attr(attr, reinterpret_cast<const void*>(k_lossless_decode_wide<4>), smem);
    if (e != cudaSuccess) return e;
    ProfRange pr_("lossless_decode_wide", st);
    const uint32_t grid = min(max_records, uint32_t(num_sms() * 2));
    k_lossless_decode_wide<4><<<grid, kThreads, smem, st>>>(s, b, ws);
    return cudaGetLastError();
  }
  static int fast_blocks_per_sm = 0;
  const size_t fsmem = sizeof(FastSmem);
  static SmemAttr attr_fast;
  cudaError_t e = smem_attr(attr_fast, reinterpret_cast<const void*>(k_lossless_decode_fast), fsmem);
  if (e != cudaSuccess) return e;
  if (!fast_blocks_per_sm) {
    e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&fast_blocks_per_sm, k_lossless_decode_fast,
                                                      kFastThreads, fsmem);
    if (e != cudaSuccess || fast_blocks_per_sm < 1) fast_blocks_per_sm = 1;
  }
  {
    ProfRange pr_("lossless_decode", st);
    uint32_t grid = min(max_records, uint32_t(num_sms() * fast_blocks_per_sm));
    k_lossless_decode_fast<<<grid, kFastThreads, fsmem, st>>>(s, b, ws);
  }
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const size_t smem = sizeof(DecSmem) + 2u * pad16(s.tc * s.D);
  static SmemAttr attr_gen;
  e = smem_attr(attr_gen, reinterpret_cast<const void*>(k_lossless_decode), smem);
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("lossless_decode_general", st);
    uint32_t grid = min(max_records, uint32_t(num_sms()));
    k_lossless_decode<<<grid, kThreads, smem, st>>>(s, b, ws);
  }
  return cudaGetLastError();
}

}  // namespace kvc
