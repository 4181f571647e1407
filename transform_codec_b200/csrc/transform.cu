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

__device__ inline float bf16_to_f32(uint32_t h) { return __uint_as_float(h << 16); }
__device__ inline uint32_t f32_to_bf16_rne(float f) {
  uint32_t x = __float_as_uint(f);
  if ((x & 0x7fffffffu) > 0x7f800000u) return ((x >> 16) | 0x40u) & 0xffffu;
  uint32_t upper = x >> 16, lower = x & 0xffffu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) ++upper;
  return upper & 0xffffu;
}

__device__ inline uint32_t quantize(float y, float z, float s, uint32_t levels) {
  if (s == 0.0f) return 0u;
  float q = __fdiv_rn(__fsub_rn(y, z), s);
  float r = rintf(q);
  if (!(r > 0.0f)) return 0u;
  if (r >= float(levels)) return levels;
  return uint32_t(r);
}

struct __align__(16) CompInfo {
  uint32_t width[kD];
  uint32_t comp[kD];        // components ordered by (width, index), widths >= 1
  uint32_t coded_idx[kD];   // rank among coded components (width >= 1)
  uint32_t bstart[10], bcount[10];
  uint32_t n_coded;
};

// widths of slice sidx -> component order per bit width (needs blockDim >= 128)
__device__ inline void build_comp_info(const uint8_t* widths, CompInfo& ci, uint32_t* tmp) {
  const uint32_t j = threadIdx.x;
  const uint32_t w = j < kD ? widths[j] : 0u;
  if (j < kD) ci.width[j] = w;
  uint32_t tot;
  uint32_t ci_idx = block_exclusive_scan(j < kD && w > 0 ? 1u : 0u, tmp, &tot);
  if (j < kD) ci.coded_idx[j] = ci_idx;
  if (j == 0) ci.n_coded = tot;
  uint32_t base = 0;
  for (uint32_t b = 1; b <= 8; ++b) {
    uint32_t flag = (j < kD && w == b) ? 1u : 0u;
    uint32_t cnt;
    uint32_t ex = block_exclusive_scan(flag, tmp, &cnt);
    if (flag) ci.comp[base + ex] = j;
    if (j == 0) { ci.bstart[b] = base; ci.bcount[b] = cnt; }
    base += cnt;
  }
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

struct __align__(16) EncSmem {
  float Q[kD * kD];            // Q[k][j]
  float xy[kTile * kD];        // x' then y, [token][k or j]
  uint8_t codes[kD * kMaxCt];  // [j][t]
  float zs[kD][kMaxCt / kTile][2];
  uint32_t crc_t[1024];
  uint32_t hist[256], freq[256], rem[256], fc[256], rcp[256];
  uint32_t states[kMaxLanes];
  uint32_t tmp[32], red[32];
  uint32_t W[4], wbeg[4], sub_len[4];
  uint32_t k, mode, bytes, off;
  CompInfo ci;
};

__global__ void __launch_bounds__(kThreads)
k_transform_encode_mid(TransformShape sh, TransformPlanDev pl, FrameBatch b, EncodeLayout ws) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  EncSmem& S = *reinterpret_cast<EncSmem*>(smem_raw);
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t rps = 1u + sh.n_mid;
  const uint32_t gs = blockIdx.x / sh.n_mid, c = blockIdx.x % sh.n_mid;  // slice of the batch
  const uint32_t r = gs * rps + 1u + c;                                   // record of the batch
  const uint32_t fr = frame_of(b.rec_base, b.n, r);
  const uint32_t ls = (r - b.rec_base[fr]) / rps;
  const uint16_t* src = reinterpret_cast<const uint16_t*>(b.f[fr].src);
  const uint32_t sidx = b.f[fr].first_slice + ls;
  const bool is_key = ((sidx / sh.H) & 1u) == 0;
  const uint32_t t0 = sh.s_end + c * sh.ct, tcc = min(sh.ct, sh.r_start - t0);
  const uint32_t nb = (tcc + kTile - 1) / kTile;
  const uint16_t* xs = src + uint64_t(ls) * sh.T * kD;

  crc_tables_init(S.crc_t);
  {
    const uint4* q4 = reinterpret_cast<const uint4*>(pl.bases + uint64_t(sidx) * kD * kD);
    uint4* d4 = reinterpret_cast<uint4*>(S.Q);
    for (uint32_t i = tid; i < kD * kD / 4; i += nthr) d4[i] = __ldg(q4 + i);
  }
  build_comp_info(pl.widths + uint64_t(sidx) * kD, S.ci, S.tmp);

  const uint32_t tg = tid >> 4, jg = tid & 15u;  // projection tile: tokens 4tg.., comps 8jg..
  for (uint32_t blk = 0; blk < nb; ++blk) {
    const uint32_t bl = min(kTile, tcc - blk * kTile);
    const uint32_t tb = t0 + blk * kTile;
    for (uint32_t idx = tid; idx < kTile * (kD / 2); idx += nthr) {
      const uint32_t tt = idx / (kD / 2), i = idx % (kD / 2);
      float a = 0.0f, b = 0.0f;
      if (tt < bl) {
        const uint16_t* row = xs + uint64_t(tb + tt) * kD;
        a = bf16_to_f32(row[i]);
        b = bf16_to_f32(row[i + kD / 2]);
        if (is_key) {
          const float2 cs = reinterpret_cast<const float2*>(pl.rope)[uint64_t(tb + tt) * (kD / 2) + i];
          float na = __fadd_rn(__fmul_rn(a, cs.x), __fmul_rn(b, cs.y));
          float nb2 = __fsub_rn(__fmul_rn(b, cs.x), __fmul_rn(a, cs.y));
          a = na;
          b = nb2;
        }
      }
      S.xy[tt * kD + i] = a;
      S.xy[tt * kD + i + kD / 2] = b;
    }
    __syncthreads();
    double acc[4][8];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) acc[a][b] = 0.0;
    for (uint32_t k = 0; k < kD; ++k) {
      const float4 q0 = *reinterpret_cast<const float4*>(&S.Q[k * kD + jg * 8]);
      const float4 q1 = *reinterpret_cast<const float4*>(&S.Q[k * kD + jg * 8 + 4]);
      const double qv[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
#pragma unroll
      for (int a = 0; a < 4; ++a) {
        const double xv = S.xy[(tg * 4 + a) * kD + k];
#pragma unroll
        for (int b = 0; b < 8; ++b) acc[a][b] = fma(qv[b], xv, acc[a][b]);
      }
    }
    __syncthreads();
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 8; ++b) S.xy[(tg * 4 + a) * kD + jg * 8 + b] = __double2float_rn(acc[a][b]);
    __syncthreads();
    if (tid < kD) {
      const uint32_t j = tid, w = S.ci.width[j];
      if (w) {
        float mn = S.xy[j], mx = mn;
        for (uint32_t tt = 1; tt < bl; ++tt) {
          float v = S.xy[tt * kD + j];
          if (v < mn) mn = v;
          if (v > mx) mx = v;
        }
        const uint32_t levels = (1u << w) - 1u;
        const float s = (mx == mn) ? 0.0f : __fdiv_rn(__fsub_rn(mx, mn), float(levels));
        for (uint32_t tt = 0; tt < bl; ++tt)
          S.codes[j * kMaxCt + blk * kTile + tt] = uint8_t(quantize(S.xy[tt * kD + j], mn, s, levels));
        S.zs[j][blk][0] = mn;
        S.zs[j][blk][1] = s;
      }
    }
    __syncthreads();
  }

  // record: side info, then one stream per present bit width
  uint8_t* rec = ws.slots + uint64_t(r) * ws.slot_bytes;
  uint16_t* scratch = reinterpret_cast<uint16_t*>(rec + ws.slot_bytes - (2u * kD * kMaxCt + 64u));
  const uint32_t side = 8u * S.ci.n_coded * nb;
  if (tid < kD && S.ci.width[tid]) {
    uint32_t* p32 = reinterpret_cast<uint32_t*>(rec + 8u * S.ci.coded_idx[tid] * nb);
    for (uint32_t blk = 0; blk < nb; ++blk) {
      p32[2 * blk] = __float_as_uint(S.zs[tid][blk][0]);
      p32[2 * blk + 1] = __float_as_uint(S.zs[tid][blk][1]);
    }
  }
  if (tid < pad16(side) - side) rec[side + tid] = 0;
  uint32_t off = pad16(side);
  const Split split(tcc);
  for (uint32_t b = 1; b <= 8; ++b) {
    const uint32_t m = S.ci.bcount[b];
    if (!m) continue;
    const uint32_t n = m * tcc, base = S.ci.bstart[b];
    auto sym = [&](uint32_t i) -> uint32_t {
      uint32_t a, t;
      split(i, a, t);
      return S.codes[S.ci.comp[base + a] * kMaxCt + t];
    };
    __syncthreads();
    for (uint32_t i = tid; i < 256; i += nthr) S.hist[i] = 0;
    __syncthreads();
    for (uint32_t i = tid; i < n; i += nthr) atomicAdd(&S.hist[sym(i)], 1u);
    __syncthreads();
    const uint32_t k = block_normalize(S.hist, n, S.freq, S.rem, S.tmp);
    block_enc_tables(S.freq, S.fc, S.rcp, S.tmp);
    const uint32_t N = rans_lanes(n), G = rans_groups(N);
    const uint32_t warp = tid >> 5, lane = tid & 31u;
    if (k >= 2 && warp < G) {
      uint32_t b0, len0, b1 = n, len1;
      lane_range(n, N, warp * kGroupLanes, b0, len0);
      if (warp + 1 < G) lane_range(n, N, (warp + 1) * kGroupLanes, b1, len1);
      uint32_t x;
      uint32_t Wg = rans_encode_group(sym, n, N, warp, S.fc, S.rcp, scratch + b0, b1 - b0, &x);
      if (warp * kGroupLanes + lane < N) S.states[warp * kGroupLanes + lane] = x;
      if (lane == 0) { S.W[warp] = Wg; S.wbeg[warp] = b1 - Wg; }
    }
    __syncthreads();
    if (tid == 0) {
      const uint32_t raw_b = 16u + pad16(n);
      if (k == 1) { S.mode = kModeConst; S.bytes = 16; }
      else {
        uint32_t rb = rans_layout(n, k, S.W, S.sub_len);
        if (rb < raw_b) { S.mode = kModeRans; S.bytes = rb; }
        else { S.mode = kModeRaw; S.bytes = raw_b; }
      }
      S.k = k;
    }
    __syncthreads();
    block_write_stream(rec + off, S.mode, n, S.bytes, sym(0), S.k, S.freq, S.states, scratch,
                       S.wbeg, S.W, S.sub_len, sym, S.tmp);
    off += S.bytes;
  }
  __syncthreads();
  uint32_t crc = crc32_block_aligned(rec, off, S.crc_t, S.red);
  if (tid == 0) {
    ws.rec_len[r] = off;
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

// Decoder shared memory. Operand tiles come first so each 128-byte-swizzled
// tile starts on a 1024-byte boundary.
struct __align__(1024) DecSmem {
  uint8_t a_hi[kTcRows * 256];   // y^ as bf16 pieces, A operand [token][component]
  uint8_t a_lo[kTcRows * 256];
  uint8_t b_hi[kD * 256];        // Q as bf16 pieces, B operand [channel][component]
  uint8_t b_lo[kD * 256];
  uint8_t codes[kD * kMaxCt];    // [j][t]
  float zs[kD][kMaxCt / kTile][2];
  uint32_t crc_t[1024];
  uint32_t freq[256], cum[260], lut[kProbScale];
  uint32_t tmp[32], red[32];
  StreamInfo si;
  CompInfo ci;
  uint64_t bar;
  uint32_t base[kBatchMax + 1];
  uint32_t tmem_base;
  uint32_t crc_ok, cur_slice, bad;
};

static_assert(sizeof(DecSmem) + 1024 <= 232448, "decoder shared memory exceeds the per-block limit");

__global__ void __launch_bounds__(kThreads)
k_transform_decode(TransformShape sh, TransformPlanDev pl, FrameBatch b, uint8_t* ws) {
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
  crc_tables_init(S.crc_t);
  if (warp == 0) {
    tc::tmem_alloc(&S.tmem_base, kTcCols);
    tc::tmem_relinquish();
  }
  if (tid == 0) {
    S.cur_slice = 0xffffffffu;
    tc::mbar_init(&S.bar, 1);
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tmem = S.tmem_base;
  uint32_t phase = 0;
  bool alive = true;
  const uint32_t rps = 1u + sh.n_mid;
  constexpr uint32_t idesc = tc::idesc_bf16_f32(kTcRows, kD);
  for (uint32_t g = rbeg; g < rend && alive; ++g) {
    __syncthreads();
    const uint32_t fr = frame_of(S.base, b.n, g), r = g - S.base[fr];
    const uint8_t* src = b.f[fr].src;
    uint16_t* dst = reinterpret_cast<uint16_t*>(b.f[fr].dst);
    DecodeState* ds = decode_state(ws, fr);
    const uint32_t first = ds->first_slice;
    const uint8_t* e = src + kHeaderBytes + uint64_t(kIndexEntry) * r;
    const uint64_t off0 = ld_u64(e);
    const uint32_t len = ld_u32(e + 8), want = ld_u32(e + 12);
    const uint8_t* rec = src + off0;
    const uint32_t ls = r / rps, kind = r % rps;
    const uint32_t sidx = first + ls;
    const bool is_key = ((sidx / sh.H) & 1u) == 0;
    uint16_t* xs = dst + uint64_t(ls) * sh.T * kD;
    uint32_t got = crc32_block_aligned(rec, len, S.crc_t, S.red);
    if (tid == 0) S.crc_ok = (got == want);
    __syncthreads();
    int st = S.crc_ok ? kOk : kErrCorrupt;
    if (kind == 0) {
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
    if (S.cur_slice != sidx) {
      __syncthreads();
      const uint4* q4 = reinterpret_cast<const uint4*>(pl.qsplit + uint64_t(sidx) * kQSplitBytes);
      uint4* b4 = reinterpret_cast<uint4*>(S.b_hi);  // b_hi and b_lo are contiguous
      for (uint32_t i = tid; i < kQSplitBytes / 16u; i += nthr) b4[i] = __ldg(q4 + i);
      build_comp_info(pl.widths + uint64_t(sidx) * kD, S.ci, S.tmp);
      if (tid == 0) S.cur_slice = sidx;
      __syncthreads();
    }
    const uint32_t side = 8u * S.ci.n_coded * nb;
    if (st == kOk && pad16(side) > len) st = kErrCorrupt;
    if (st == kOk) {
      if (tid < kD && S.ci.width[tid]) {
        const uint32_t* p32 = reinterpret_cast<const uint32_t*>(rec + 8u * S.ci.coded_idx[tid] * nb);
        for (uint32_t blk = 0; blk < nb; ++blk) {
          S.zs[tid][blk][0] = __uint_as_float(p32[2 * blk]);
          S.zs[tid][blk][1] = __uint_as_float(p32[2 * blk + 1]);
        }
      }
      if (tid == 0) S.bad = 0;
    }
    uint32_t off = pad16(side);
    const Split split(tcc);
    for (uint32_t b = 1; b <= 8 && st == kOk; ++b) {
      const uint32_t m = S.ci.bcount[b];
      if (!m) continue;
      const uint32_t n = m * tcc, base = S.ci.bstart[b], levels = (1u << b) - 1u;
      __syncthreads();
      st = block_parse_stream(rec + off, len - off, n, &S.si, S.freq, S.tmp);
      if (st != kOk) break;
      auto put = [&](uint32_t i, uint32_t sy) {
        uint32_t a, t;
        split(i, a, t);
        if (sy > levels) S.bad = 1;
        S.codes[S.ci.comp[base + a] * kMaxCt + t] = uint8_t(sy);
      };
      bool ok = true;
      if (S.si.mode == kModeRaw) {
        for (uint32_t i = tid; i < n; i += nthr) put(i, rec[off + 16 + i]);
      } else if (S.si.mode == kModeConst) {
        for (uint32_t i = tid; i < n; i += nthr) put(i, S.si.sym);
      } else {
        block_dec_lut(S.freq, S.cum, S.lut, S.tmp);
        const uint32_t N = rans_lanes(n), G = rans_groups(N);
        if (warp < G)
          ok = rans_decode_group(rec + off + S.si.sub_off[warp], S.si.sub_len[warp], n, N, warp,
                                 S.lut, put);
      }
      ok = __syncthreads_and(ok);
      if (!ok || S.bad) st = kErrCorrupt;
      off += S.si.bytes;
    }
    if (st == kOk && off != len) st = kErrCorrupt;
    if (st != kOk) {
      if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(st));
      continue;
    }
    // inverse projection on the tensor cores, 128 tokens at a time:
    // x^[t][k] = sum_j y^[t][j] Q[k][j] with y^ and Q split into bf16 hi + lo
    // pieces (hi*hi + hi*lo + lo*hi, fp32 accumulation in tensor memory)
    for (uint32_t t_base = 0; t_base < tcc; t_base += kTcRows) {
      const uint32_t bl = min(kTcRows, tcc - t_base);
      __syncthreads();
      for (uint32_t idx = tid; idx < kTcRows * kD; idx += nthr) {
        const uint32_t tt = idx >> 7, j = idx & (kD - 1u);
        float v = 0.0f;
        if (tt < bl && S.ci.width[j]) {
          const uint32_t t = t_base + tt, blk = t / kTile;
          v = __fmaf_rn(float(S.codes[j * kMaxCt + t]), S.zs[j][blk][1], S.zs[j][blk][0]);
        }
        const uint32_t h = f32_to_bf16_rne(v);
        const uint32_t l = f32_to_bf16_rne(__fsub_rn(v, bf16_to_f32(h)));
        const uint32_t o = tc::sw128_offset(tt, 2u * j, kTcRows);
        *reinterpret_cast<uint16_t*>(S.a_hi + o) = uint16_t(h);
        *reinterpret_cast<uint16_t*>(S.a_lo + o) = uint16_t(l);
      }
      tc::fence_async_smem();
      __syncthreads();
      if (tid == 0) {
        tc::fence_after_sync();
        const uint32_t ah = tc::smem_addr(S.a_hi), al = tc::smem_addr(S.a_lo);
        const uint32_t bh = tc::smem_addr(S.b_hi), bo = tc::smem_addr(S.b_lo);
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
      const bool done = tc::mbar_wait(&S.bar, phase, 1u << 22);
      phase ^= 1u;
      if (!__syncthreads_and(done)) {
        if (tid == 0) atomicMin(&ds->err_key, (static_cast<unsigned long long>(r) << 8) | unsigned(kErrTimeout));
        tc::mbar_wait(&S.bar, phase ^ 1u, 1u << 22);
        alive = false;
        break;
      }
      tc::fence_after_sync();
      // epilogue: warp w reads token rows 32 (w % 4) .., channel quarter (w / 4):
      // channels [32q, 32q + 32) and their RoPE partners [32q + 64, 32q + 96)
      {
        const uint32_t sub = warp & 3u, q = warp >> 2;
        const uint32_t tt = sub * 32u + lane;
        const uint32_t c0 = q * 32u;
        uint32_t va[32], vb[32];
        const uint32_t ta = tmem + ((sub * 32u) << 16);
        tc::tmem_ld16(ta + c0, va);
        tc::tmem_ld16(ta + c0 + 16u, va + 16);
        tc::tmem_ld16(ta + c0 + 64u, vb);
        tc::tmem_ld16(ta + c0 + 80u, vb + 16);
        tc::tmem_wait_ld();
        if (tt < bl) {
          const uint32_t t = t0 + t_base + tt;
          const float2* cs = reinterpret_cast<const float2*>(pl.rope) + uint64_t(t) * (kD / 2) + c0;
          uint32_t pa[16], pb[16];
#pragma unroll
          for (uint32_t i = 0; i < 32; i += 2) {
            float a0 = __uint_as_float(va[i]), b0 = __uint_as_float(vb[i]);
            float a1 = __uint_as_float(va[i + 1]), b1 = __uint_as_float(vb[i + 1]);
            if (is_key) {
              const float2 k0 = cs[i], k1 = cs[i + 1];
              const float na0 = __fsub_rn(__fmul_rn(a0, k0.x), __fmul_rn(b0, k0.y));
              const float nb0 = __fadd_rn(__fmul_rn(a0, k0.y), __fmul_rn(b0, k0.x));
              const float na1 = __fsub_rn(__fmul_rn(a1, k1.x), __fmul_rn(b1, k1.y));
              const float nb1 = __fadd_rn(__fmul_rn(a1, k1.y), __fmul_rn(b1, k1.x));
              a0 = na0; b0 = nb0; a1 = na1; b1 = nb1;
            }
            pa[i >> 1] = f32_to_bf16_rne(a0) | (f32_to_bf16_rne(a1) << 16);
            pb[i >> 1] = f32_to_bf16_rne(b0) | (f32_to_bf16_rne(b1) << 16);
          }
          uint4* ra = reinterpret_cast<uint4*>(xs + uint64_t(t) * kD + c0);
          uint4* rb = reinterpret_cast<uint4*>(xs + uint64_t(t) * kD + c0 + 64u);
#pragma unroll
          for (uint32_t v = 0; v < 4; ++v) {
            ra[v] = make_uint4(pa[4 * v], pa[4 * v + 1], pa[4 * v + 2], pa[4 * v + 3]);
            rb[v] = make_uint4(pb[4 * v], pb[4 * v + 1], pb[4 * v + 2], pb[4 * v + 3]);
          }
        }
      }
      tc::fence_before_sync();
    }
  }
  tc::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
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
  uint64_t mid = pad16_64(8ull * kD * (kMaxCt / kTile)) + 8u * 16u + pad16_64(uint64_t(kD) * kMaxCt);
  uint64_t raw = pad16_64(uint64_t(s.s_end + (s.T - s.r_start)) * kD * 2u);
  uint64_t b = (mid > raw ? mid : raw) + 2ull * kD * kMaxCt + 64u;
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
  size_t smem = sizeof(EncSmem);
  e = cudaFuncSetAttribute(k_transform_encode_mid, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  {
    ProfRange pr_("transform_encode_mid", st);
    k_transform_encode_mid<<<n_slices * s.n_mid, kThreads, smem, st>>>(s, p, b, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_transform_decode(const TransformShape& s, const TransformPlanDev& p,
                                    const FrameBatch& b, uint8_t* ws, uint32_t max_records,
                                    cudaStream_t st) {
  if (max_records == 0 || b.n == 0) return cudaSuccess;
  size_t smem = sizeof(DecSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k_transform_decode, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
  if (e != cudaSuccess) return e;
  uint32_t grid = min(max_records, uint32_t(num_sms()));
  {
    ProfRange pr_("transform_decode", st);
    k_transform_decode<<<grid, kThreads, smem, st>>>(s, p, b, ws);
  }
  return cudaGetLastError();
}

}  // namespace kvc
