// Container kernels (sm_100a): header + chunk index writer with the aggregate
// header CRC, record placement, and the decoder's header/index validation
// (QATQ page, "How it works": bounded chunks with ordered lengths and an
// aggregate checksum; "QATC v2 checksum validated": corrupt or truncated
// payloads are refused before restore). Also the stage kernels used to check
// the CRC and rANS stages on their own.

#include "kvc.h"
#include "kvc_device.cuh"
#include "kvc_internal.h"

namespace kvc {

struct Result {
  int32_t status;
  uint32_t pad;
  uint64_t bytes;
};

namespace {

constexpr uint32_t kBig = 1024;  // threads of the single-block container kernels

__device__ inline uint64_t block_exclusive_scan64(uint64_t v, uint64_t* tmp, uint64_t* total) {
  const uint32_t lane = threadIdx.x & 31u, warp = threadIdx.x >> 5;
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= uint32_t(o)) x += y;
  }
  __syncthreads();
  if (lane == 31) tmp[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t nw = blockDim.x >> 5;
    uint64_t w = lane < nw ? tmp[lane] : 0ull;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      uint64_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= uint32_t(o)) w += y;
    }
    if (lane < nw) tmp[lane] = w;
  }
  __syncthreads();
  uint64_t base = warp ? tmp[warp - 1] : 0ull;
  *total = tmp[(blockDim.x >> 5) - 1];
  __syncthreads();
  return base + x - v;
}

// One CTA per frame: offsets from the frame's record lengths, the index, the
// header and its CRC; the frame's result.
__global__ void __launch_bounds__(kBig)
k_finalize(HeaderFields h, FrameBatch b, EncodeLayout ws) {
  __shared__ uint32_t crc_t[1024];
  __shared__ uint32_t red[32];
  __shared__ uint64_t tmp64[32];
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t f = blockIdx.x;
  const FrameDesc& fd = b.f[f];
  const uint32_t g0 = b.rec_base[f], nr = b.rec_base[f + 1] - g0;
  uint8_t* dst = fd.dst;
  Result* res = static_cast<Result*>(fd.res);
  EncodeState* es = ws.state + f;
  __shared__ int kerr;
  if (tid == 0) kerr = 0;
  crc_tables_init(crc_t);
  const uint32_t per = (nr + nthr - 1) / nthr;
  const uint32_t beg = min(nr, tid * per), end = min(nr, beg + per);
  uint64_t mine = 0;
  for (uint32_t i = beg; i < end; ++i) {
    const uint32_t len = ws.rec_len[g0 + i];
    if (len >= kRecLenError) atomicMax(&kerr, int(len & 0xffu));
    mine += len;
  }
  __syncthreads();
  if (kerr) {  // a record its encoder could not produce: the frame reports its status
    if (tid == 0) {
      es->status = kerr;
      es->total_bytes = 0;
      res->status = kerr;
      res->bytes = 0;
    }
    return;
  }
  uint64_t sum_all;
  uint64_t pre = block_exclusive_scan64(mine, tmp64, &sum_all);
  const uint64_t first = uint64_t(kHeaderBytes) + uint64_t(kIndexEntry) * nr;
  const uint64_t total = first + sum_all;
  if (total > fd.dst_cap) {
    if (tid == 0) {
      es->status = kErrCapacity;
      es->total_bytes = total;
      res->status = kErrCapacity;
      res->bytes = total;
    }
    return;
  }
  uint64_t off = first + pre;
  for (uint32_t i = beg; i < end; ++i) {
    ws.rec_off[g0 + i] = off;
    uint32_t len = ws.rec_len[g0 + i];
    uint4 ent = make_uint4(uint32_t(off), uint32_t(off >> 32), len, ws.rec_crc[g0 + i]);
    *reinterpret_cast<uint4*>(dst + kHeaderBytes + uint64_t(kIndexEntry) * i) = ent;
    off += len;
  }
  if (tid == 0) {
    uint32_t* w = reinterpret_cast<uint32_t*>(dst);
    w[0] = 0x3143564bu;  // "KVC1"
    w[1] = 1u | (h.path << 16) | (h.dtype << 24);
    w[2] = h.L; w[3] = h.H; w[4] = h.T; w[5] = h.D;
    w[6] = fd.first_slice; w[7] = fd.n_slices; w[8] = h.chunk_tokens; w[9] = nr;
    w[10] = uint32_t(total); w[11] = uint32_t(total >> 32);
    w[12] = h.plan_crc;
    w[13] = h.n_sink | (h.n_recent << 16);
    w[14] = h.block_tokens;
  }
  __syncthreads();
  const uint8_t* cdst = dst;
  uint32_t hcrc = crc32_block_bytes(
      [cdst](uint64_t i) -> uint32_t { return i < 60 ? cdst[i] : cdst[kHeaderBytes + (i - 60)]; },
      60ull + uint64_t(kIndexEntry) * nr, crc_t, red);
  if (tid == 0) {
    reinterpret_cast<uint32_t*>(dst)[15] = hcrc;
    es->status = kOk;
    es->n_records = nr;
    es->total_bytes = total;
    res->status = kOk;
    res->bytes = total;
  }
}

__global__ void k_copy_records(FrameBatch b, EncodeLayout ws) {
  const uint32_t total = b.rec_base[b.n];
  for (uint32_t g = blockIdx.x; g < total; g += gridDim.x) {
    const uint32_t f = frame_of(b.rec_base, b.n, g);
    if (ws.state[f].status != kOk) continue;
    const uint4* s = reinterpret_cast<const uint4*>(ws.slots + uint64_t(g) * ws.slot_bytes);
    uint4* d = reinterpret_cast<uint4*>(b.f[f].dst + ws.rec_off[g]);
    const uint32_t q = ws.rec_len[g] / 16u;
    for (uint32_t i = threadIdx.x; i < q; i += blockDim.x) d[i] = s[i];
  }
}

// One CTA per frame: validate the header and index in the codec's fixed order.
__global__ void __launch_bounds__(kBig)
k_check_container(FrameBatch b, ContainerExpect e, uint8_t* ws) {
  __shared__ uint32_t crc_t[1024];
  __shared__ uint32_t red[32];
  __shared__ int st_s;
  __shared__ uint32_t nr_s, first_s, ns_s;
  const uint32_t tid = threadIdx.x, nthr = blockDim.x;
  const uint32_t f = blockIdx.x;
  const uint8_t* src = b.f[f].src;
  const uint64_t src_bytes = b.f[f].src_bytes;
  DecodeState* ds = decode_state(ws, f);
  Result* res = static_cast<Result*>(b.f[f].res);
  crc_tables_init(crc_t);
  if (tid == 0) {
    int st = kOk;
    uint32_t nr = 0;
    if (src_bytes < kHeaderBytes) st = kErrTruncated;
    else if (ld_u32(src) != 0x3143564bu || ld_u16(src + 4) != 1u) st = kErrCorrupt;
    else {
      uint64_t total = ld_u64(src + 40);
      if (src_bytes < total) st = kErrTruncated;
      else if (src_bytes > total) st = kErrCorrupt;
      else {
        nr = ld_u32(src + 36);
        if (uint64_t(kHeaderBytes) + uint64_t(kIndexEntry) * nr > total) st = kErrCorrupt;
      }
    }
    st_s = st;
    nr_s = nr;
    first_s = 0;
    ns_s = 0;
  }
  __syncthreads();
  uint64_t total = 0;
  if (st_s == kOk) {
    const uint32_t nr = nr_s;
    total = ld_u64(src + 40);
    uint32_t hcrc = crc32_block_bytes(
        [src](uint64_t i) -> uint32_t { return i < 60 ? src[i] : src[kHeaderBytes + (i - 60)]; },
        60ull + uint64_t(kIndexEntry) * nr, crc_t, red);
    if (tid == 0) {
      int st = kOk;
      uint32_t first = ld_u32(src + 24), ns = ld_u32(src + 28);
      if (hcrc != ld_u32(src + 60)) st = kErrCorrupt;
      else if (src[6] != e.path || src[7] != e.dtype || ld_u32(src + 8) != e.L ||
               ld_u32(src + 12) != e.H || ld_u32(src + 16) != e.T || ld_u32(src + 20) != e.D ||
               ld_u32(src + 32) != e.chunk_tokens)
        st = kErrPlanMismatch;
      else if (ld_u16(src + 58) != 0) st = kErrCorrupt;
      else if (e.path == 0) {
        if (ld_u32(src + 48) || ld_u16(src + 52) || ld_u16(src + 54) || ld_u16(src + 56))
          st = kErrCorrupt;
      } else if (ld_u16(src + 52) != e.n_sink || ld_u16(src + 54) != e.n_recent ||
                 ld_u16(src + 56) != e.block_tokens || ld_u32(src + 48) != e.plan_crc) {
        st = kErrPlanMismatch;
      }
      if (st == kOk && uint64_t(first) + ns > uint64_t(e.L) * 2u * e.H) st = kErrPlanMismatch;
      if (st == kOk && uint64_t(ns) * e.recs_per_slice != nr) st = kErrCorrupt;
      st_s = st;
      first_s = first;
      ns_s = ns;
    }
    __syncthreads();
    if (st_s == kOk) {
      const uint64_t start = uint64_t(kHeaderBytes) + uint64_t(kIndexEntry) * nr;
      int bad = 0;
      for (uint32_t i = tid; i < nr; i += nthr) {
        const uint8_t* en = src + kHeaderBytes + uint64_t(kIndexEntry) * i;
        uint64_t o = ld_u64(en);
        uint32_t len = ld_u32(en + 8);
        if (len & 15u) bad = 1;
        if (i == 0 && o != start) bad = 1;
        if (i + 1 < nr && ld_u64(en + kIndexEntry) != o + len) bad = 1;
        if (i + 1 == nr && o + len != total) bad = 1;
      }
      if (nr == 0 && start != total) bad = 1;
      bad = __syncthreads_or(bad);
      if (tid == 0) {
        int st = bad ? kErrCorrupt : kOk;
        if (st == kOk && (uint64_t(ns_s) * e.T * e.D * e.E > b.f[f].dst_cap || ns_s > e.max_slices))
          st = kErrCapacity;
        st_s = st;
      }
    }
  }
  __syncthreads();
  if (tid == 0) {
    int st = st_s;
    ds->status = st;
    ds->first_slice = st == kOk ? first_s : 0;
    ds->n_slices = st == kOk ? ns_s : 0;
    ds->n_records = st == kOk ? nr_s : 0;
    ds->err_key = ~0ull;
    ds->out_bytes = st == kOk ? uint64_t(ns_s) * e.T * e.D * e.E : 0;
    if (f == 0) batch_state(ws)->n_deferred = 0;
    res->status = st;
    res->bytes = 0;
  }
}

__global__ void k_decode_finish(FrameBatch b, uint8_t* ws) {
  const uint32_t f = threadIdx.x;
  if (f >= b.n) return;
  const DecodeState* ds = decode_state(ws, f);
  Result* res = static_cast<Result*>(b.f[f].res);
  int st = ds->status;
  if (st == kOk && ds->err_key != ~0ull) st = int(ds->err_key & 0xffu);
  res->status = st;
  res->bytes = st == kOk ? ds->out_bytes : 0;
}

// ------------------------------------------------------------------ stage kernels
__global__ void __launch_bounds__(kBig) k_stage_crc32(const uint8_t* src, uint64_t n, uint32_t* out) {
  __shared__ uint32_t crc_t[1024];
  __shared__ uint32_t red[32];
  crc_tables_init(crc_t);
  uint32_t c = crc32_block_bytes([src](uint64_t i) -> uint32_t { return src[i]; }, n, crc_t, red);
  if (threadIdx.x == 0) *out = c;
}

struct __align__(16) StageSmem {
  uint32_t hist[256], freq[256], rem[256], fc[256], rcp[256], cum[260];
  uint32_t lut[kProbScale];
  uint32_t states[kMaxLanes];
  uint32_t tmp[32];
  uint32_t W[4], wbeg[4], sub_len[4];
  uint32_t k, mode, bytes;
  StreamInfo si;
};

__global__ void __launch_bounds__(256)
k_stage_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out, uint16_t* scratch, Result* res) {
  __shared__ StageSmem S;
  const uint32_t tid = threadIdx.x;
  for (uint32_t i = tid; i < 256; i += blockDim.x) S.hist[i] = 0;
  __syncthreads();
  for (uint32_t i = tid; i < n; i += blockDim.x) atomicAdd(&S.hist[sym[i]], 1u);
  __syncthreads();
  uint32_t k = block_normalize(S.hist, n, S.freq, S.rem, S.tmp);
  block_enc_tables(S.freq, S.fc, S.rcp, S.tmp);
  const uint32_t N = rans_lanes(n), G = rans_groups(N);
  const uint32_t warp = tid >> 5, lane = tid & 31u;
  if (k >= 2 && warp < G) {
    uint32_t b0, len0, b1 = n, len1;
    lane_range(n, N, warp * kGroupLanes, b0, len0);
    if (warp + 1 < G) lane_range(n, N, (warp + 1) * kGroupLanes, b1, len1);
    uint32_t x;
    uint32_t Wg = rans_encode_group([sym](uint32_t i) -> uint32_t { return sym[i]; }, n, N, warp,
                                    S.fc, S.rcp, scratch + b0, b1 - b0, &x);
    if (warp * kGroupLanes + lane < N) S.states[warp * kGroupLanes + lane] = x;
    if (lane == 0) { S.W[warp] = Wg; S.wbeg[warp] = b1 - Wg; }
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t raw_b = 16u + pad16(n);
    if (k == 1) { S.mode = kModeConst; S.bytes = 16; }
    else if (k >= 2) {
      uint32_t rb = rans_layout(n, k, S.W, S.sub_len);
      if (rb < raw_b) { S.mode = kModeRans; S.bytes = rb; }
      else { S.mode = kModeRaw; S.bytes = raw_b; }
    } else { S.mode = kModeRaw; S.bytes = raw_b; }
    S.k = k;
  }
  __syncthreads();
  block_write_stream(out, S.mode, n, S.bytes, n ? uint32_t(sym[0]) : 0u, S.k, S.freq, S.states,
                     scratch, S.wbeg, S.W, S.sub_len,
                     [sym](uint32_t i) -> uint32_t { return sym[i]; }, S.tmp);
  if (tid == 0) { res->status = kOk; res->bytes = S.bytes; }
}

__global__ void __launch_bounds__(256)
k_stage_stream_decode(const uint8_t* rec, uint32_t rec_bytes, uint32_t n, uint8_t* sym, Result* res) {
  __shared__ StageSmem S;
  const uint32_t tid = threadIdx.x;
  int st = block_parse_stream(rec, rec_bytes, n, &S.si, S.freq, S.tmp);
  bool ok = st == kOk;
  if (ok) {
    if (S.si.mode == kModeRaw) {
      for (uint32_t i = tid; i < n; i += blockDim.x) sym[i] = rec[16 + i];
    } else if (S.si.mode == kModeConst) {
      for (uint32_t i = tid; i < n; i += blockDim.x) sym[i] = uint8_t(S.si.sym);
    } else {
      block_dec_lut(S.freq, S.cum, S.lut, S.tmp);
      const uint32_t N = rans_lanes(n), G = rans_groups(N), warp = tid >> 5;
      bool okw = true;
      const uint32_t dm = S.si.delta ? 0xffu : 0u;  // lane deltas: running XOR per lane
      uint32_t prev = 0;
      if (warp < G)
        okw = rans_decode_group(rec + S.si.sub_off[warp], S.si.sub_len[warp], n, N, warp, S.lut,
                                [&](uint32_t i, uint32_t s) {
                                  prev = s ^ (prev & dm);
                                  sym[i] = uint8_t(prev);
                                });
      ok = __syncthreads_and(okw);
    }
  }
  if (tid == 0) {
    res->status = ok ? kOk : kErrCorrupt;
    res->bytes = ok ? S.si.bytes : 0;
  }
}

}  // namespace

cudaError_t launch_finalize(const HeaderFields& h, const FrameBatch& b, const EncodeLayout& ws,
                            cudaStream_t st) {
  if (b.n == 0) return cudaSuccess;
  {
    ProfRange pr_("finalize", st);
    k_finalize<<<b.n, kBig, 0, st>>>(h, b, ws);
  }
  cudaError_t e = cudaGetLastError();
  const uint32_t total = b.rec_base[b.n];
  if (e != cudaSuccess || total == 0) return e;
  {
    ProfRange pr_("copy_records", st);
    k_copy_records<<<min(total, 148u * 8u), 256, 0, st>>>(b, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_check_container(const FrameBatch& b, const ContainerExpect& e, uint8_t* ws,
                                   cudaStream_t st) {
  if (b.n == 0) return cudaSuccess;
  {
    ProfRange pr_("check_container", st);
    k_check_container<<<b.n, kBig, 0, st>>>(b, e, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode_finish(const FrameBatch& b, uint8_t* ws, cudaStream_t st) {
  if (b.n == 0) return cudaSuccess;
  {
    ProfRange pr_("decode_finish", st);
    k_decode_finish<<<1, kBatchMax, 0, st>>>(b, ws);
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_crc32(const uint8_t* src, uint64_t n, uint32_t* out, cudaStream_t st) {
  {
    ProfRange pr_("stage_crc32", st);
    k_stage_crc32<<<1, kBig, 0, st>>>(src, n, out);
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_stream_encode(const uint8_t* sym, uint32_t n, uint8_t* out,
                                       uint16_t* scratch, void* res, cudaStream_t st) {
  {
    ProfRange pr_("stage_stream_encode", st);
    k_stage_stream_encode<<<1, 256, 0, st>>>(sym, n, out, scratch, static_cast<Result*>(res));
  }
  return cudaGetLastError();
}

cudaError_t launch_stage_stream_decode(const uint8_t* rec, uint32_t rec_bytes, uint32_t n,
                                       uint8_t* sym, void* res, cudaStream_t st) {
  {
    ProfRange pr_("stage_stream_decode", st);
    k_stage_stream_decode<<<1, 256, 0, st>>>(rec, rec_bytes, n, sym, static_cast<Result*>(res));
  }
  return cudaGetLastError();
}

}  // namespace kvc

// ------------------------------------------------------------ no-alloc stage encode
// Word scratch of kvc_stage_stream_encode_noalloc: the rANS encoder emits at
// most one 16-bit word per symbol, so kMaxChunkValues words (128 KiB) cover the
// largest stream. The encoder writes every scratch word it later reads, so the
// array needs no clearing between calls.
static __device__ __align__(256) uint16_t g_noalloc_scratch[kvc::kMaxChunkValues];

namespace {
// Device address of the scratch array in the current context. It is looked up
// on every call: the lookup is host-side and allocates nothing once the
// library's device code is loaded, and a cached address would go stale after
// a cudaDeviceReset or under another context made current on the same device.
uint16_t* noalloc_scratch(int* status) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || !p) {
    *status = KVC_ERR_CUDA;
    return nullptr;
  }
  *status = KVC_OK;
  return static_cast<uint16_t*>(p);
}
}  // namespace

extern "C" int kvc_stage_stream_encode_noalloc(const uint8_t* d_sym, uint32_t n, uint8_t* d_out,
                                               kvc_result* d_res, cudaStream_t stream) {
  if (n > kvc::kMaxChunkValues) return KVC_ERR_CAPACITY;
  if (n == 0 || !d_sym || !d_out || !d_res || (reinterpret_cast<uintptr_t>(d_out) & 15u))
    return KVC_ERR_INVALID;
  int status = KVC_OK;
  uint16_t* scratch = noalloc_scratch(&status);
  if (!scratch) return status;
  return kvc::launch_stage_stream_encode(d_sym, n, d_out, scratch, d_res, stream) == cudaSuccess
             ? KVC_OK
             : KVC_ERR_CUDA;
}
