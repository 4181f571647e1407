// Lossless front-end kernels (sm_100a): per chunk of tc tokens x D channels,
// channel-major byte planes (p = 0 low byte, p = 1 high byte), each plane one
// stream record that keeps the smallest of CONST / RANS / RAW (AT-1 Memory
// page, "KV & tensor mode": channel-major reorder, byte planes, keep whichever
// is smaller; QATQ page, "qatq encode": bounded chunks, known row width).
#include "kvc_device.cuh"
#include "tcgen05.cuh"
#include "kvc_internal.h"

namespace kvc {
namespace {

constexpr uint32_t kThreads = 256;  // 8 warps: plane p = warp / 4, group = warp % 4

struct __align__(16) EncSmem {
  uint32_t crc_t[1024];
  uint32_t hist[2][256];
  uint32_t freq[2][256];
  uint32_t rem[256];
  uint32_t fc[2][256];
  uint32_t rcp[2][256];
  uint32_t states[2][kMaxLanes];
  uint32_t tmp[32], red[32];
  uint32_t k[2], mode[2], bytes[2], csym[2];
  uint32_t W[2][4], wbeg[2][4], sub_len[2][4];
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

__global__ void __launch_bounds__(kThreads)
k_lossless_encode(LosslessShape sh, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  EncSmem& S = *reinterpret_cast<EncSmem*>(smem_raw);
  uint16_t* vals = reinterpret_cast<uint16_t*>(smem_raw + sizeof(EncSmem));
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t gr = blockIdx.x;  // record of the batch
  const uint32_t fr = frame_of(b.rec_base, b.n, gr);
  const uint32_t r = gr - b.rec_base[fr];
  const uint16_t* src = reinterpret_cast<const uint16_t*>(b.f[fr].src);
  const uint32_t slice = r / sh.cps, c = r % sh.cps;
  const uint32_t t0 = c * sh.tc, tcc = min(sh.tc, sh.T - t0), D = sh.D, n = tcc * D;
  const uint32_t n_max = sh.tc * D;
  const uint16_t* g = src + (uint64_t(slice) * sh.T + t0) * D;

  crc_tables_init(S.crc_t);
  for (uint32_t i = tid; i < 512; i += nthr) (&S.hist[0][0])[i] = 0;
  if ((reinterpret_cast<uintptr_t>(g) & 15u) == 0 && (n & 7u) == 0) {
    const uint4* g4 = reinterpret_cast<const uint4*>(g);
    uint4* v4 = reinterpret_cast<uint4*>(vals);
    for (uint32_t q = tid; q < n / 8u; q += nthr) v4[q] = __ldg(g4 + q);
  } else {
    for (uint32_t i = tid; i < n; i += nthr) vals[i] = g[i];
  }
  __syncthreads();
  for (uint32_t i = tid; i < n; i += nthr) {
    uint32_t v = vals[i];
    atomicAdd(&S.hist[0][v & 0xffu], 1u);
    atomicAdd(&S.hist[1][v >> 8], 1u);
  }
  __syncthreads();
  for (uint32_t p = 0; p < 2; ++p) {
    uint32_t k = block_normalize(S.hist[p], n, S.freq[p], S.rem, S.tmp);
    if (tid == 0) S.k[p] = k;
    block_enc_tables(S.freq[p], S.fc[p], S.rcp[p], S.tmp);
  }

  const ChanMajor cm(tcc);
  const uint32_t N = rans_lanes(n), G = rans_groups(N);
  uint8_t* slot = ws.slots + uint64_t(gr) * ws.slot_bytes;
  const uint32_t rec_area = 2u * (16u + pad16(n_max));
  uint16_t* scratch[2] = {reinterpret_cast<uint16_t*>(slot + rec_area),
                          reinterpret_cast<uint16_t*>(slot + rec_area + 2u * n_max + 64u)};
  {
    const uint32_t warp = tid >> 5, lane = tid & 31u;
    const uint32_t p = warp >> 2, gg = warp & 3u;
    if (S.k[p] >= 2 && gg < G) {
      uint32_t b0, len0, b1 = n, len1;
      lane_range(n, N, gg * kGroupLanes, b0, len0);
      if (gg + 1 < G) lane_range(n, N, (gg + 1) * kGroupLanes, b1, len1);
      auto sym = [&](uint32_t i) -> uint32_t {
        uint32_t d, t;
        cm.split(i, d, t);
        uint32_t v = vals[t * D + d];
        return p ? (v >> 8) : (v & 0xffu);
      };
      uint32_t x;
      uint32_t Wg = rans_encode_group(sym, n, N, gg, S.fc[p], S.rcp[p], scratch[p] + b0, b1 - b0, &x);
      uint32_t l = gg * kGroupLanes + lane;
      if (l < N) S.states[p][l] = x;
      if (lane == 0) {
        S.W[p][gg] = Wg;
        S.wbeg[p][gg] = b0 + (b1 - b0) - Wg;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    for (uint32_t p = 0; p < 2; ++p) {
      uint32_t k = S.k[p], raw_b = 16u + pad16(n);
      uint32_t v0 = vals[0];
      S.csym[p] = p ? (v0 >> 8) : (v0 & 0xffu);
      if (k == 1) { S.mode[p] = kModeConst; S.bytes[p] = 16; }
      else if (k >= 2) {
        uint32_t rb = rans_layout(n, k, S.W[p], S.sub_len[p]);
        if (rb < raw_b) { S.mode[p] = kModeRans; S.bytes[p] = rb; }
        else { S.mode[p] = kModeRaw; S.bytes[p] = raw_b; }
      } else { S.mode[p] = kModeRaw; S.bytes[p] = raw_b; }
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
    block_write_stream(rec + off, S.mode[p], n, S.bytes[p], S.csym[p], S.k[p], S.freq[p],
                       S.states[p], scratch[p], S.wbeg[p], S.W[p], S.sub_len[p], raw, S.tmp);
    off += S.bytes[p];
  }
  __syncthreads();
  uint32_t crc = crc32_block_aligned(rec, off, S.crc_t, S.red);
  if (tid == 0) {
    ws.rec_len[gr] = off;
    ws.rec_crc[gr] = crc;
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
    uint32_t got = crc32_block_aligned(rec, len, S.crc_t, S.red);
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
        ok = rans_decode_group(recp[p] + S.si[p].sub_off[gg], S.si[p].sub_len[gg], n, N, gg,
                               S.lut[p], [&](uint32_t i, uint32_t s) { pl[i] = uint8_t(s); });
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
// Fast decoder for full chunks (D * tc = 65536 values, tc a multiple of 512):
// then every stream has 128 lanes of 512 symbols and lane l's symbol tau sits at
// channel-major index l * 512 + tau in both planes, i.e. channel l / lpc, token
// (l % lpc) * 512 + tau with lpc = tc / 512. Thread l owns lane l of both planes
// (warp w = rANS group w), decodes token-synchronously, merges the other
// plane's raw bytes from registers and writes 32-token tiles of token-major
// rows through shared memory. Records with two rANS planes or other shapes are
// deferred to the general decoder.
constexpr uint32_t kFastThreads = 128;

struct __align__(16) FastSmem {
  uint32_t crc_t[1024];
  uint32_t lut[kProbScale];
  uint16_t tile[32 * 128];
  uint32_t freq[2][256];
  uint32_t cum[260];
  uint32_t tmp[32], red[32];
  StreamInfo si[2];
  uint16_t ring[kFastThreads / 32][1024];  // per-group window of rANS refill words
  CrcJoin join;
  uint32_t base[kBatchMax + 1];
  uint32_t crc_ok;
};

// One rANS lane of a 32-lane group (warp-synchronous). Refill words come from
// the group's window in shared memory (word i at ring[i % 1024]); a lane whose
// index runs past the sub-stream marks the record bad and its state is junk.
struct LaneRans {
  uint32_t x, pos, W;
  const uint16_t* ring;
  uint32_t bad;
  __device__ __forceinline__ uint32_t step(const uint32_t* lut, uint32_t lt) {
    const uint32_t e = lut[x & (kProbScale - 1u)];
    x = ((e >> 12) & 0xfffu) * (x >> kProbBits) + (e & 0xfffu);
    const bool need = x < kRansLow;
    const uint32_t mask = __ballot_sync(0xffffffffu, need);
    const uint32_t idx = pos + __popc(mask & lt);
    const uint32_t w = ring[idx & 1023u];
    x = need ? ((x << 16) | w) : x;
    bad |= uint32_t(need && idx >= W);
    pos += __popc(mask);
    return e >> 24;
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

// value of step j: byte (j % 4) of raw word r (plane 0) and decoded symbol (plane 1),
// or the other way round, merged into one 16-bit value
__device__ __forceinline__ uint32_t merge_raw_lo(uint32_t r, uint32_t j, uint32_t hi) {
  return __byte_perm(r, hi, (j & 3u) | 0x40u);  // byte0 = r.byte(j%4), byte1 = hi.byte0
}
__device__ __forceinline__ uint32_t merge_raw_hi(uint32_t r, uint32_t j, uint32_t lo) {
  return __byte_perm(lo, r, 0u | ((4u + (j & 3u)) << 4));  // byte0 = lo.byte0, byte1 = r.byte(j%4)
}

template <uint32_t M0, uint32_t M1, uint32_t D>
__device__ inline bool fast_tiles(FastSmem& S, const uint8_t* const recp[2], uint16_t* out) {
  constexpr uint32_t LPC = 128u / D;  // lanes per channel
  const uint32_t l = threadIdx.x, lane = l & 31u, g = l >> 5;
  const uint32_t lt = lanemask_lt();
  const uint32_t tbase = (l % LPC) * 32u * D + (l / LPC);
  uint16_t* tile = S.tile + tbase;
  LaneRans rs{kRansLow, 0, 0, S.ring[g], 0};
  RefillWindow win{nullptr, 0, 0, tc::smem_addr(S.ring[g])};
  const uint8_t* raw0 = recp[0] + 16 + l * 512u;
  const uint8_t* raw1 = recp[1] + 16 + l * 512u;
  const uint32_t c0 = S.si[0].sym, c1 = S.si[1].sym;
  constexpr bool kRans = (M0 == kModeRans || M1 == kModeRans);
  constexpr uint32_t RP = (M0 == kModeRans) ? 0u : 1u;  // the rANS plane, if any
  if (kRans) {
    const StreamInfo& si = S.si[RP];
    const uint8_t* sub = recp[RP] + si.sub_off[g];
    const uint32_t sl = si.sub_len[g];
    if (sl < 128u || (sl & 1u)) rs.bad = 1;
    else {
      rs.x = reinterpret_cast<const uint32_t*>(sub)[lane];
      rs.W = (sl - 128u) >> 1;
      win.units = sub + 128;
      win.n_units = (rs.W + 7u) >> 3;
    }
  }
  const bool live = __all_sync(0xffffffffu, rs.bad == 0);
  uint4 n0a = make_uint4(0, 0, 0, 0), n0b = n0a, n1a = n0a, n1b = n0a;  // next tile's raw bytes
  if (M0 == kModeRaw) { n0a = __ldcs(reinterpret_cast<const uint4*>(raw0)); n0b = __ldcs(reinterpret_cast<const uint4*>(raw0 + 16)); }
  if (M1 == kModeRaw) { n1a = __ldcs(reinterpret_cast<const uint4*>(raw1)); n1b = __ldcs(reinterpret_cast<const uint4*>(raw1 + 16)); }
  if (kRans && !live) return false;
  if (kRans) {
    win.request(0, lane);
    asm volatile("cp.async.commit_group;" ::: "memory");  // empty group: the first settle waits for the window
  }
  for (uint32_t k = 0; k < 16; ++k) {
    uint32_t r0[8], r1[8];
    if (M0 == kModeRaw) {
      r0[0] = n0a.x; r0[1] = n0a.y; r0[2] = n0a.z; r0[3] = n0a.w;
      r0[4] = n0b.x; r0[5] = n0b.y; r0[6] = n0b.z; r0[7] = n0b.w;
      if (k + 1 < 16) {
        n0a = __ldcs(reinterpret_cast<const uint4*>(raw0 + 32u * (k + 1)));
        n0b = __ldcs(reinterpret_cast<const uint4*>(raw0 + 32u * (k + 1) + 16u));
      }
    }
    if (M1 == kModeRaw) {
      r1[0] = n1a.x; r1[1] = n1a.y; r1[2] = n1a.z; r1[3] = n1a.w;
      r1[4] = n1b.x; r1[5] = n1b.y; r1[6] = n1b.z; r1[7] = n1b.w;
      if (k + 1 < 16) {
        n1a = __ldcs(reinterpret_cast<const uint4*>(raw1 + 32u * (k + 1)));
        n1b = __ldcs(reinterpret_cast<const uint4*>(raw1 + 32u * (k + 1) + 16u));
      }
    }
#pragma unroll
    for (uint32_t j = 0; j < 32; ++j) {
      if (kRans && (j & 7u) == 0) {
        win.settle();
        win.request(rs.pos, lane);
      }
      uint32_t v;
      if (M0 == kModeRaw && M1 == kModeRans) v = merge_raw_lo(r0[j >> 2], j, rs.step(S.lut, lt));
      else if (M0 == kModeRans && M1 == kModeRaw) v = merge_raw_hi(r1[j >> 2], j, rs.step(S.lut, lt));
      else if (M0 == kModeRaw && M1 == kModeRaw) v = __byte_perm(r0[j >> 2], r1[j >> 2], (j & 3u) | ((4u + (j & 3u)) << 4));
      else if (M0 == kModeRaw && M1 == kModeConst) v = merge_raw_lo(r0[j >> 2], j, c1);
      else if (M0 == kModeConst && M1 == kModeRaw) v = merge_raw_hi(r1[j >> 2], j, c0);
      else if (M0 == kModeRans && M1 == kModeConst) v = rs.step(S.lut, lt) | (c1 << 8);
      else if (M0 == kModeConst && M1 == kModeRans) v = c0 | (rs.step(S.lut, lt) << 8);
      else v = c0 | (c1 << 8);
      tile[j * D] = uint16_t(v);
    }
    __syncthreads();
    // tile = LPC blocks of 32 token rows x D channels, each contiguous in the output
    constexpr uint32_t per_block = 4u * D;  // uint4 per block
#pragma unroll
    for (uint32_t i = 0; i < 4; ++i) {
      const uint32_t q = l + i * kFastThreads;
      const uint32_t sblk = q / per_block, w = q % per_block;
      uint4* o = reinterpret_cast<uint4*>(out + (uint64_t(sblk) * 512u + 32u * k) * D);
      o[w] = reinterpret_cast<const uint4*>(S.tile)[q];
    }
    __syncthreads();
  }
  if (kRans) asm volatile("cp.async.wait_group 0;" ::: "memory");  // no copy outlives the record
  bool ok = rs.bad == 0;
  if (kRans) ok = ok && rs.pos == rs.W && rs.x == kRansLow;
  return ok;
}

template <uint32_t D>
__device__ inline bool fast_dispatch(FastSmem& S, const uint8_t* const recp[2], uint16_t* out,
                                     uint32_t m0, uint32_t m1) {
  if (m0 == kModeRaw && m1 == kModeRans) return fast_tiles<kModeRaw, kModeRans, D>(S, recp, out);
  if (m0 == kModeRaw && m1 == kModeRaw) return fast_tiles<kModeRaw, kModeRaw, D>(S, recp, out);
  if (m0 == kModeRaw && m1 == kModeConst) return fast_tiles<kModeRaw, kModeConst, D>(S, recp, out);
  if (m0 == kModeRans && m1 == kModeRaw) return fast_tiles<kModeRans, kModeRaw, D>(S, recp, out);
  if (m0 == kModeRans && m1 == kModeConst) return fast_tiles<kModeRans, kModeConst, D>(S, recp, out);
  if (m0 == kModeConst && m1 == kModeRans) return fast_tiles<kModeConst, kModeRans, D>(S, recp, out);
  if (m0 == kModeConst && m1 == kModeRaw) return fast_tiles<kModeConst, kModeRaw, D>(S, recp, out);
  return fast_tiles<kModeConst, kModeConst, D>(S, recp, out);
}

__global__ void __launch_bounds__(kFastThreads)
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
  crc_join_init(&S.join);
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
    if (!defer && len > kCrcOneRound) {  // cannot be a valid full-chunk record; let the general decoder report it
      defer = true;
    }
    if (!defer) {
      uint32_t got = crc32_block_128(rec, len, S.crc_t, &S.join, S.red);
      if (tid == 0) S.crc_ok = (got == want);
      __syncthreads();
      st = S.crc_ok ? kOk : kErrCorrupt;
      const uint32_t n = kMaxChunkValues;
      if (st == kOk) st = block_parse_stream(rec, len, n, &S.si[0], S.freq[0], S.tmp);
      if (st == kOk) {
        const uint32_t b0 = S.si[0].bytes;
        st = block_parse_stream(rec + b0, len - b0, n, &S.si[1], S.freq[1], S.tmp);
        if (st == kOk && b0 + S.si[1].bytes != len) st = kErrCorrupt;
      }
      if (st == kOk && S.si[0].mode == kModeRans && S.si[1].mode == kModeRans) defer = true;
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
    if (m0 == kModeRans) block_dec_lut(S.freq[0], S.cum, S.lut, S.tmp);
    else if (m1 == kModeRans) block_dec_lut(S.freq[1], S.cum, S.lut, S.tmp);
    const uint8_t* recp[2] = {rec, rec + S.si[0].bytes};
    uint16_t* out = dst + (uint64_t(slice) * sh.T + t0) * D;
    const bool ok = D == 128u ? fast_dispatch<128>(S, recp, out, m0, m1)
                              : fast_dispatch<64>(S, recp, out, m0, m1);
    if (!__syncthreads_and(ok) && tid == 0)
      atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrCorrupt));
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
  uint64_t b = 2u * (16u + pad16_64(n_max)) + 2u * (2u * n_max + 64u);
  return (b + 255u) & ~uint64_t(255);
}

cudaError_t launch_lossless_encode(const LosslessShape& s, const FrameBatch& b,
                                   const EncodeLayout& ws, cudaStream_t st) {
  const uint32_t nrec = b.rec_base[b.n];
  if (nrec == 0) return cudaSuccess;
  size_t smem = sizeof(EncSmem) + pad16(s.tc * s.D * 2u);
  cudaError_t e = cudaFuncSetAttribute(k_lossless_encode, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       int(smem));
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("lossless_encode", st);
    k_lossless_encode<<<nrec, kThreads, smem, st>>>(s, b, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_lossless_decode(const LosslessShape& s, const FrameBatch& b, uint8_t* ws,
                                   uint32_t max_records, cudaStream_t st) {
  if (max_records == 0 || b.n == 0) return cudaSuccess;
  static int fast_blocks_per_sm = 0;
  const size_t fsmem = sizeof(FastSmem);
  cudaError_t e = cudaFuncSetAttribute(k_lossless_decode_fast,
                                       cudaFuncAttributeMaxDynamicSharedMemorySize, int(fsmem));
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
  e = cudaFuncSetAttribute(k_lossless_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("lossless_decode_general", st);
    uint32_t grid = min(max_records, uint32_t(num_sms()));
    k_lossless_decode<<<grid, kThreads, smem, st>>>(s, b, ws);
  }
  return cudaGetLastError();
}

}  // namespace kvc
