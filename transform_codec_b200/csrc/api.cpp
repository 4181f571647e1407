// Host side of the KV codec library: plans, workspace sizing and the C ABI
// declared in include/kvc.h. Kernels live in the .cu files of this directory.
#include "kvc.h"

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>
#include <thread>
#include <vector>

#include "kvc_internal.h"

using namespace kvc;

namespace {

inline uint64_t pad16u(uint64_t n) { return (n + 15u) & ~uint64_t(15); }
inline uint64_t pad256u(uint64_t n) { return (n + 255u) & ~uint64_t(255); }

// Table-driven CRC-32 (reflected 0xEDB88320, init/xorout 0xFFFFFFFF).
struct HostCrc {
  uint32_t t[256];
  HostCrc() {
    for (uint32_t b = 0; b < 256; ++b) {
      uint32_t c = b;
      for (int i = 0; i < 8; ++i) c = (c >> 1) ^ ((c & 1u) ? 0xEDB88320u : 0u);
      t[b] = c;
    }
  }
  uint32_t update(uint32_t crc, const void* p, size_t n) const {
    const uint8_t* b = static_cast<const uint8_t*>(p);
    for (size_t i = 0; i < n; ++i) crc = (crc >> 8) ^ t[(crc ^ b[i]) & 0xffu];
    return crc;
  }
};
const HostCrc& host_crc() {
  static HostCrc c;
  return c;
}

int n_workers(int want) {
  if (want > 0) return want;
  unsigned h = std::thread::hardware_concurrency();
  return h ? int(h) : 4;
}

template <class F>
void parallel_for(uint32_t n, int threads, F f) {
  threads = std::max(1, std::min<int>(threads, int(n)));
  std::atomic<uint32_t> next{0};
  std::vector<std::thread> pool;
  for (int i = 0; i < threads; ++i)
    pool.emplace_back([&] {
      for (uint32_t k; (k = next.fetch_add(1)) < n;) f(k);
    });
  for (auto& th : pool) th.join();
}

}  // namespace

struct kvc_plan_s {
  kvc_plan_desc d{};
  int device = 0;
  uint32_t S = 0;                 // slices L*2*H
  bool transform = false;
  LosslessShape ls{};
  TransformShape ts{};
  uint32_t plan_crc = 0;
  std::vector<uint8_t> widths;    // [S][D]
  uint64_t max_slice_bytes = 0;   // transform: largest per-slice record bytes
  float* d_bases = nullptr;
  uint8_t* d_widths = nullptr;
  float* d_rope = nullptr;
  uint8_t* d_qsplit = nullptr;
  CompInfo* d_comp = nullptr;
  uint8_t* d_qdig = nullptr;
  QColInfo* d_qcol = nullptr;
  float* d_qt = nullptr;
  // host-streamed calls: two copy streams and the ring's events, made by the
  // first such call and kept until the plan is destroyed
  cudaStream_t copy_in = nullptr, copy_out = nullptr;
  cudaEvent_t ring_ev[3][3] = {};   // [in, coded, out][slot]
};

namespace {

// Greedy allocation as a selection: every (component u, level b < max_bits)
// increment has gain lambda_u * 4^-b; taking them one at a time by largest gain
// (ties: lowest component) equals sorting all increments by (gain desc, u asc,
// b asc) and keeping the first B, because each component's gains fall with b.
bool allocate_widths(const double* lam, uint64_t U, double avg_bits, uint32_t max_bits,
                     std::vector<uint8_t>& w) {
  double bd = std::floor(avg_bits * double(U) + 0.5);
  if (!(avg_bits >= 0.0) || bd > double(max_bits) * double(U)) return false;
  uint64_t B = uint64_t(bd);
  struct Cand { double g; uint32_t u; uint32_t b; };
  std::vector<Cand> c;
  c.reserve(U * max_bits);
  for (uint64_t u = 0; u < U; ++u) {
    if (std::isnan(lam[u])) return false;
    double l = lam[u] > 0.0 ? lam[u] : 0.0;
    for (uint32_t b = 0; b < max_bits; ++b) c.push_back({std::ldexp(l, -2 * int(b)), uint32_t(u), b});
  }
  auto before = [](const Cand& a, const Cand& b) {
    if (a.g != b.g) return a.g > b.g;
    if (a.u != b.u) return a.u < b.u;
    return a.b < b.b;
  };
  if (B < c.size()) std::nth_element(c.begin(), c.begin() + B, c.end(), before);
  w.assign(U, 0);
  for (uint64_t i = 0; i < B; ++i) w[c[i].u]++;
  return true;
}

void regions(const kvc_plan_desc& d, uint32_t& s_end, uint32_t& r_start) {
  s_end = std::min(d.n_sink, d.n_tokens);
  uint32_t rs = d.n_tokens > d.n_recent ? d.n_tokens - d.n_recent : 0;
  r_start = std::max(rs, s_end);
}

uint64_t mid_record_bound(const uint8_t* w, uint32_t D, uint32_t tcc, uint32_t block, bool kivi_values) {
  uint32_t nb = (tcc + block - 1) / block, coded = 0, m[9] = {0};
  for (uint32_t j = 0; j < D; ++j) {
    coded += w[j] > 0;
    m[w[j]]++;
  }
  // side information: four byte-plane streams of 2 * coded * nb values (per-token
  // value ranges: 2 * tcc), each at most RAW
  const uint64_t nv = kivi_values ? 2ull * tcc : 2ull * coded * nb;
  uint64_t b = coded ? 4ull * (16 + pad16u(nv)) : 0ull;
  for (uint32_t k = 1; k <= 8; ++k)
    if (m[k]) b += 16 + pad16u(uint64_t(m[k]) * tcc);
  return b;
}

void rope_table(uint32_t T, uint32_t D, double theta, std::vector<float>& cs) {
  const uint32_t half = D / 2;
  cs.resize(size_t(T) * half * 2);
  for (uint32_t t = 0; t < T; ++t)
    for (uint32_t i = 0; i < half; ++i) {
      double inv = std::pow(theta, -(2.0 * double(i)) / double(D));
      double a = double(t) * inv;
      cs[(size_t(t) * half + i) * 2] = float(std::cos(a));
      cs[(size_t(t) * half + i) * 2 + 1] = float(std::sin(a));
    }
}

uint32_t compute_plan_crc(const kvc_plan_desc& d, const std::vector<uint8_t>& widths, uint32_t S) {
  const HostCrc& h = host_crc();
  uint8_t head[48];
  uint32_t v[10] = {d.dtype, d.n_layers, d.n_heads, d.n_tokens, d.head_dim,
                    d.n_sink, d.n_recent, d.block_tokens, d.chunk_tokens, d.max_bits};
  for (int i = 0; i < 10; ++i)
    for (int b = 0; b < 4; ++b) head[4 * i + b] = uint8_t(v[i] >> (8 * b));
  uint64_t tb;
  std::memcpy(&tb, &d.rope_theta, 8);
  for (int b = 0; b < 8; ++b) head[40 + b] = uint8_t(tb >> (8 * b));
  uint32_t crc = 0xffffffffu;
  crc = h.update(crc, head, sizeof head);
  crc = h.update(crc, widths.data(), widths.size());
  const size_t nb = size_t(S) * d.head_dim * d.head_dim;
  std::vector<uint8_t> le(nb * 4);
  for (size_t i = 0; i < nb; ++i) {
    uint32_t x;
    std::memcpy(&x, &d.bases[i], 4);
    for (int b = 0; b < 4; ++b) le[4 * i + b] = uint8_t(x >> (8 * b));
  }
  crc = h.update(crc, le.data(), le.size());
  if (d.range_mode) {  // only a non-default range mode
    uint8_t rm[4];
    for (int b = 0; b < 4; ++b) rm[b] = uint8_t(d.range_mode >> (8 * b));
    crc = h.update(crc, rm, 4);
  }
  return crc ^ 0xffffffffu;
}

// max |Q^T Q - I| over every slice's basis, fp64
bool bases_orthonormal(const float* bases, uint32_t S, uint32_t D, double tol) {
  std::atomic<bool> ok{true};
  parallel_for(S, n_workers(0), [&](uint32_t s) {
    const float* Q = bases + size_t(s) * D * D;
    for (uint32_t a = 0; a < D && ok; ++a)
      for (uint32_t b = a; b < D; ++b) {
        double acc = 0.0;
        for (uint32_t k = 0; k < D; ++k) acc += double(Q[size_t(k) * D + a]) * double(Q[size_t(k) * D + b]);
        if (std::fabs(acc - (a == b ? 1.0 : 0.0)) > tol || std::isnan(acc)) { ok = false; break; }
      }
  });
  return ok;
}

uint16_t bf16_rne(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  if ((x & 0x7fffffffu) > 0x7f800000u) return uint16_t((x >> 16) | 0x40u);
  uint32_t upper = x >> 16, lower = x & 0xffffu;
  if (lower > 0x8000u || (lower == 0x8000u && (upper & 1u))) ++upper;
  return uint16_t(upper);
}

// Byte offset of element (row, kbyte) in a K-major operand of `rows` rows stored
// in 128-byte-swizzled atoms (the tensor cores' layout: 16-byte chunk c of row r
// sits at chunk c ^ (r mod 8)), K split into 128-byte blocks rows*128 bytes apart.
uint32_t sw128_offset_host(uint32_t row, uint32_t kbyte, uint32_t rows) {
  const uint32_t kb = kbyte >> 7, in = kbyte & 127u;
  const uint32_t chunk = (in >> 4) ^ (row & 7u);
  return kb * rows * 128u + row * 128u + (chunk << 4) + (in & 15u);
}

// Per slice, Q as two bf16 pieces (hi = rne(Q), lo = rne(Q - hi)) laid out as the
// B operand of D[token][k] = sum_j y[token][j] * Q[k][j]: row k, K index j.
// Component order of one slice from its 128 widths (see CompInfo).
void comp_info(const uint8_t* widths, CompInfo& ci) {
  ci = CompInfo{};
  uint32_t coded = 0;
  for (uint32_t j = 0; j < 128; ++j) {
    ci.width[j] = widths[j];
    ci.coded_idx[j] = coded;
    if (widths[j]) ++coded;
  }
  ci.n_coded = coded;
  uint32_t base = 0;
  for (uint32_t b = 1; b <= 8; ++b) {
    ci.bstart[b] = base;
    for (uint32_t j = 0; j < 128; ++j)
      if (widths[j] == b) ci.comp[base++] = j;
    ci.bcount[b] = base - ci.bstart[b];
  }
}

void split_bases(const float* bases, uint32_t S, std::vector<uint8_t>& out) {
  const uint32_t D = 128;
  out.assign(size_t(S) * kQSplitBytes, 0);
  for (uint32_t s = 0; s < S; ++s) {
    uint8_t* hi = out.data() + size_t(s) * kQSplitBytes;
    uint8_t* lo = hi + kQSplitBytes / 2;
    const float* Q = bases + size_t(s) * D * D;
    for (uint32_t k = 0; k < D; ++k)
      for (uint32_t j = 0; j < D; ++j) {
        const float q = Q[size_t(k) * D + j];
        const uint16_t h = bf16_rne(q);
        uint32_t hb = uint32_t(h) << 16;
        float hf;
        std::memcpy(&hf, &hb, 4);
        const uint16_t l = bf16_rne(q - hf);
        const uint32_t off = sw128_offset_host(k, 2 * j, D);
        std::memcpy(hi + off, &h, 2);
        std::memcpy(lo + off, &l, 2);
      }
  }
}

// Per slice, the coded columns of Q as the B operand of the encoder's exact
// tensor-core projection (see QColInfo): integer J = rint(Q 2^(29 - f)) as four
// byte planes (byte 0 the signed top byte), row cc, K index k; and Q
// transposed (fp32) for the fp64 chains that settle open decisions.
void digit_bases(const float* bases, const uint8_t* widths, uint32_t S, std::vector<uint8_t>& dig,
                 std::vector<QColInfo>& col, std::vector<float>& qt) {
  const uint32_t D = 128;
  dig.assign(size_t(S) * kQDigBytes, 0);
  col.assign(S, QColInfo{});
  qt.assign(size_t(S) * D * D, 0.0f);
  for (uint32_t s = 0; s < S; ++s) {
    const float* Q = bases + size_t(s) * D * D;
    uint8_t* planes = dig.data() + size_t(s) * kQDigBytes;
    for (uint32_t j = 0; j < D; ++j)
      for (uint32_t k = 0; k < D; ++k) qt[(size_t(s) * D + j) * D + k] = Q[size_t(k) * D + j];
    uint32_t cc = 0;
    for (uint32_t j = 0; j < D; ++j) {
      if (!widths[size_t(s) * D + j]) continue;
      double m = 0.0, l1 = 0.0;
      for (uint32_t k = 0; k < D; ++k) {
        const double q = std::fabs(double(Q[size_t(k) * D + j]));
        m = std::max(m, q);
        l1 += q;
      }
      // l1 is within 128 * 2^-53 relative of the exact sum; the margin makes
      // the stored value an upper bound
      float q1 = float(l1 * (1.0 + 0x1p-40));
      if (double(q1) < l1 * (1.0 + 0x1p-40)) q1 = std::nextafter(q1, INFINITY);
      col[s].q1[cc] = q1;
      if (m == 0.0) {
        col[s].f[cc] = kQColZero;
      } else {
        const int f = std::ilogb(m);
        col[s].f[cc] = f;
        for (uint32_t k = 0; k < D; ++k) {
          const int64_t J = int64_t(std::nearbyint(std::ldexp(double(Q[size_t(k) * D + j]), 29 - f)));
          const uint32_t u = uint32_t(int32_t(J));
          for (uint32_t p = 0; p < 4; ++p)
            planes[p * kQDigPlane + sw128_offset_host(cc, k, D)] = uint8_t(u >> (24 - 8 * p));
        }
      }
      ++cc;
    }
  }
}

void free_plan(kvc_plan_s* p) {
  if (!p) return;
  if (p->d_bases) cudaFree(p->d_bases);
  if (p->d_widths) cudaFree(p->d_widths);
  if (p->d_rope) cudaFree(p->d_rope);
  if (p->d_qsplit) cudaFree(p->d_qsplit);
  if (p->d_comp) cudaFree(p->d_comp);
  if (p->d_qdig) cudaFree(p->d_qdig);
  if (p->d_qcol) cudaFree(p->d_qcol);
  if (p->d_qt) cudaFree(p->d_qt);
  if (p->copy_in) cudaStreamSynchronize(p->copy_in);
  if (p->copy_out) cudaStreamSynchronize(p->copy_out);
  for (auto& row : p->ring_ev)
    for (cudaEvent_t e : row)
      if (e) cudaEventDestroy(e);
  if (p->copy_in) cudaStreamDestroy(p->copy_in);
  if (p->copy_out) cudaStreamDestroy(p->copy_out);
  delete p;
}

}  // namespace

extern "C" int kvc_plan(const kvc_plan_desc* desc, kvc_plan_t** out) {
  if (!desc || !out) return KVC_ERR_INVALID;
  *out = nullptr;
  const kvc_plan_desc& d = *desc;
  if (d.abi_version != KVC_ABI_VERSION) return KVC_ERR_INVALID;
  if (d.dtype != KVC_DTYPE_BF16 && d.dtype != KVC_DTYPE_FP16 && d.dtype != KVC_DTYPE_F32) return KVC_ERR_INVALID;
  if (!d.n_layers || !d.n_heads || !d.n_tokens || !d.head_dim) return KVC_ERR_INVALID;
  if (uint64_t(d.n_layers) * 2u * d.n_heads > 0x7fffffffu) return KVC_ERR_INVALID;
  if (d.values_per_chunk < d.head_dim || d.values_per_chunk > kMaxChunkValues) return KVC_ERR_INVALID;
  if (d.range_mode > KVC_RANGES_KIVI || d.reserved) return KVC_ERR_INVALID;
  auto* p = new kvc_plan_s();
  p->d = d;
  p->d.bases = nullptr;
  p->d.eigvals = nullptr;
  p->d.widths = nullptr;
  p->S = d.n_layers * 2u * d.n_heads;
  cudaGetDevice(&p->device);
  p->ls.T = d.n_tokens;
  p->ls.D = d.head_dim;
  p->ls.tc = d.values_per_chunk / d.head_dim;
  p->ls.cps = (d.n_tokens + p->ls.tc - 1) / p->ls.tc;
  p->ls.E = d.dtype == KVC_DTYPE_F32 ? 4u : 2u;
  if (d.bases) {
    int st = KVC_OK;
    if (d.dtype != KVC_DTYPE_BF16 || (d.head_dim & 1u) || d.max_bits > 8 || !(d.rope_theta > 0.0) ||
        !d.block_tokens || !d.chunk_tokens || d.chunk_tokens % d.block_tokens ||
        d.n_sink > 65535u || d.n_recent > 65535u || d.block_tokens > 65535u ||
        (!d.eigvals && !d.widths) || (d.range_mode == KVC_RANGES_KIVI && d.head_dim < d.block_tokens))
      st = KVC_ERR_INVALID;
    else if (d.head_dim != 128 || d.block_tokens != 64 || d.chunk_tokens > 512)
      st = KVC_ERR_UNSUPPORTED;
    else if (!bases_orthonormal(d.bases, p->S, d.head_dim, 1e-3))
      st = KVC_ERR_INVALID;
    const uint64_t U = uint64_t(p->S) * d.head_dim;
    if (st == KVC_OK) {
      if (d.widths) {
        p->widths.assign(d.widths, d.widths + U);
        for (uint8_t w : p->widths)
          if (w > d.max_bits) st = KVC_ERR_INVALID;
      } else if (!allocate_widths(d.eigvals, U, d.avg_bits, d.max_bits, p->widths)) {
        st = KVC_ERR_INVALID;
      }
    }
    if (st != KVC_OK) {
      free_plan(p);
      return st;
    }
    p->transform = true;
    TransformShape& ts = p->ts;
    ts.L = d.n_layers; ts.H = d.n_heads; ts.T = d.n_tokens; ts.D = d.head_dim;
    ts.ct = d.chunk_tokens; ts.block = d.block_tokens; ts.n_sink = d.n_sink; ts.n_recent = d.n_recent;
    ts.kivi = d.range_mode == KVC_RANGES_KIVI ? 1u : 0u;
    regions(d, ts.s_end, ts.r_start);
    ts.n_mid = (ts.r_start - ts.s_end + ts.ct - 1) / ts.ct;
    const uint64_t raw = pad16u(uint64_t(ts.s_end + ts.T - ts.r_start) * ts.D * 2u);
    for (uint32_t s = 0; s < p->S; ++s) {
      uint64_t b = raw;
      for (uint32_t c = 0; c < ts.n_mid; ++c) {
        uint32_t t0 = ts.s_end + c * ts.ct, tcc = std::min(ts.ct, ts.r_start - t0);
        b += mid_record_bound(p->widths.data() + size_t(s) * ts.D, ts.D, tcc, ts.block,
                              ts.kivi && ((s / ts.H) & 1u) == 1u);
      }
      p->max_slice_bytes = std::max(p->max_slice_bytes, b);
    }
    p->plan_crc = compute_plan_crc(d, p->widths, p->S);
    std::vector<float> cs;
    rope_table(d.n_tokens, d.head_dim, d.rope_theta, cs);
    std::vector<uint8_t> qs;
    split_bases(d.bases, p->S, qs);
    std::vector<CompInfo> ci(p->S);
    for (uint32_t s = 0; s < p->S; ++s) comp_info(p->widths.data() + size_t(s) * 128u, ci[s]);
    std::vector<uint8_t> qd;
    std::vector<QColInfo> qc;
    std::vector<float> qt;
    digit_bases(d.bases, p->widths.data(), p->S, qd, qc, qt);
    const size_t nb = size_t(p->S) * d.head_dim * d.head_dim * sizeof(float);
    bool ok = cudaMalloc(&p->d_bases, nb) == cudaSuccess &&
              cudaMalloc(&p->d_widths, p->widths.size()) == cudaSuccess &&
              cudaMalloc(&p->d_rope, cs.size() * sizeof(float)) == cudaSuccess &&
              cudaMemcpy(p->d_bases, d.bases, nb, cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMemcpy(p->d_widths, p->widths.data(), p->widths.size(), cudaMemcpyHostToDevice) ==
                  cudaSuccess &&
              cudaMemcpy(p->d_rope, cs.data(), cs.size() * sizeof(float), cudaMemcpyHostToDevice) ==
                  cudaSuccess &&
              cudaMalloc(&p->d_qsplit, qs.size()) == cudaSuccess &&
              cudaMemcpy(p->d_qsplit, qs.data(), qs.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&p->d_comp, ci.size() * sizeof(CompInfo)) == cudaSuccess &&
              cudaMemcpy(p->d_comp, ci.data(), ci.size() * sizeof(CompInfo), cudaMemcpyHostToDevice) ==
                  cudaSuccess &&
              cudaMalloc(&p->d_qdig, qd.size()) == cudaSuccess &&
              cudaMemcpy(p->d_qdig, qd.data(), qd.size(), cudaMemcpyHostToDevice) == cudaSuccess &&
              cudaMalloc(&p->d_qcol, qc.size() * sizeof(QColInfo)) == cudaSuccess &&
              cudaMemcpy(p->d_qcol, qc.data(), qc.size() * sizeof(QColInfo), cudaMemcpyHostToDevice) ==
                  cudaSuccess &&
              cudaMalloc(&p->d_qt, qt.size() * sizeof(float)) == cudaSuccess &&
              cudaMemcpy(p->d_qt, qt.data(), qt.size() * sizeof(float), cudaMemcpyHostToDevice) == cudaSuccess;
    if (!ok) {
      free_plan(p);
      return KVC_ERR_CUDA;
    }
  }
  *out = p;
  return KVC_OK;
}

extern "C" int kvc_plan_create(const kvc_plan_desc* desc, kvc_plan_t** out) { return kvc_plan(desc, out); }

extern "C" void kvc_plan_destroy(kvc_plan_t* plan) { free_plan(plan); }

extern "C" int kvc_plan_widths(const kvc_plan_t* plan, uint8_t* h_out, size_t n) {
  if (!plan || !h_out || n < plan->widths.size()) return KVC_ERR_INVALID;
  std::memcpy(h_out, plan->widths.data(), plan->widths.size());
  return KVC_OK;
}

extern "C" uint32_t kvc_plan_crc(const kvc_plan_t* plan) { return plan ? plan->plan_crc : 0u; }

// ------------------------------------------------------------------ sizing
namespace {

uint32_t records_per_slice(const kvc_plan_s* p, int path) {
  return path == KVC_PATH_LOSSLESS ? p->ls.cps : 1u + p->ts.n_mid;
}

uint64_t slot_bytes(const kvc_plan_s* p, int path) {
  return path == KVC_PATH_LOSSLESS ? lossless_slot_bytes(p->ls) : transform_slot_bytes(p->ts);
}

bool path_ok(const kvc_plan_s* p, int path) {
  return p && (path == KVC_PATH_LOSSLESS || (path == KVC_PATH_TRANSFORM && p->transform));
}

// encode workspace for `frames` frames holding `recs` records in total
uint64_t encode_ws_for(const kvc_plan_s* p, int path, uint64_t recs) {
  return pad256u(sizeof(EncodeState) * kBatchMax) + pad256u(recs * 4) * 2 + pad256u(recs * 8) +
         recs * slot_bytes(p, path);
}

EncodeLayout encode_layout(const kvc_plan_s* p, int path, uint64_t recs, void* ws) {
  uint8_t* b = static_cast<uint8_t*>(ws);
  EncodeLayout L;
  L.state = reinterpret_cast<EncodeState*>(b);
  b += pad256u(sizeof(EncodeState) * kBatchMax);
  L.rec_len = reinterpret_cast<uint32_t*>(b);
  b += pad256u(recs * 4);
  L.rec_crc = reinterpret_cast<uint32_t*>(b);
  b += pad256u(recs * 4);
  L.rec_off = reinterpret_cast<uint64_t*>(b);
  b += pad256u(recs * 8);
  L.slots = b;
  L.slot_bytes = slot_bytes(p, path);
  return L;
}

uint64_t decode_ws_for(const kvc_plan_s* p, int path, uint32_t frames, uint32_t max_slices) {
  const uint64_t f = std::min<uint32_t>(frames, kBatchMax);
  const uint64_t recs = f * max_slices * records_per_slice(p, path);
  return kDecodeWsFixed + pad256u(8ull * recs) +
         (path == KVC_PATH_TRANSFORM ? transform_decode_ws_extra(p->ts, recs) : 0u);
}

bool aligned16(const void* ptr) { return (reinterpret_cast<uintptr_t>(ptr) & 15u) == 0; }

int cuda_status(cudaError_t e) { return e == cudaSuccess ? KVC_OK : KVC_ERR_CUDA; }

int check_plan_device(const kvc_plan_s* p) {
  int dev = 0;
  cudaGetDevice(&dev);
  return dev == p->device ? KVC_OK : KVC_ERR_INVALID;
}

HeaderFields header_fields(const kvc_plan_s* p, int path) {
  HeaderFields h{};
  h.path = uint32_t(path);
  h.dtype = p->d.dtype;
  h.L = p->d.n_layers; h.H = p->d.n_heads; h.T = p->d.n_tokens; h.D = p->d.head_dim;
  h.recs_per_slice = records_per_slice(p, path);
  if (path == KVC_PATH_LOSSLESS) {
    h.chunk_tokens = p->ls.tc;
  } else {
    h.chunk_tokens = p->ts.ct;
    h.plan_crc = p->plan_crc;
    h.n_sink = p->d.n_sink;
    h.n_recent = p->d.n_recent;
    h.block_tokens = p->d.block_tokens;
  }
  return h;
}

int encode_frames(const kvc_plan_s* plan, int path, const kvc_frame* fr, uint32_t n, void* d_ws,
                  size_t ws_bytes, cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  if ((n && !fr) || !d_ws || !aligned16(d_ws)) return KVC_ERR_INVALID;
  int st = check_plan_device(plan);
  if (st) return st;
  const uint32_t rps = records_per_slice(plan, path);
  for (uint32_t i = 0; i < n; ++i) {
    const kvc_frame& f = fr[i];
    if (uint64_t(f.first_slice) + f.n_slices > plan->S || !f.dst || !f.res) return KVC_ERR_INVALID;
    if ((f.n_slices && !f.src) || !aligned16(f.src) || !aligned16(f.dst) || !aligned16(f.res))
      return KVC_ERR_INVALID;
    if (f.dst_cap < kvc_max_encoded_bytes(plan, path, f.n_slices)) return KVC_ERR_CAPACITY;
  }
  const HeaderFields h = header_fields(plan, path);
  uint32_t i = 0;
  while (i < n) {  // groups of frames whose records fit the workspace
    FrameBatch b{};
    uint64_t recs = 0;
    while (i < n && b.n < kBatchMax) {
      const uint64_t r = uint64_t(fr[i].n_slices) * rps;
      if (encode_ws_for(plan, path, recs + r) > ws_bytes) break;
      FrameDesc& d = b.f[b.n];
      d.src = static_cast<const uint8_t*>(fr[i].src);
      d.dst = static_cast<uint8_t*>(fr[i].dst);
      d.res = fr[i].res;
      d.dst_cap = fr[i].dst_cap;
      d.first_slice = fr[i].first_slice;
      d.n_slices = fr[i].n_slices;
      b.rec_base[b.n] = uint32_t(recs);
      recs += r;
      ++b.n;
      ++i;
    }
    if (b.n == 0) return KVC_ERR_CAPACITY;
    b.rec_base[b.n] = uint32_t(recs);
    const EncodeLayout L = encode_layout(plan, path, recs, d_ws);
    cudaError_t e;
    if (path == KVC_PATH_LOSSLESS) {
      e = launch_lossless_encode(plan->ls, b, L, stream);
    } else {
      TransformPlanDev pd{plan->d_bases, plan->d_widths, plan->d_rope, plan->d_qsplit, plan->d_comp,
                          plan->d_qdig, plan->d_qcol, plan->d_qt};
      e = launch_transform_encode(plan->ts, pd, b, L, stream);
    }
    if (e != cudaSuccess) return KVC_ERR_CUDA;
    e = launch_finalize(h, b, L, stream);
    if (e != cudaSuccess) return KVC_ERR_CUDA;
  }
  return KVC_OK;
}

int decode_frames(const kvc_plan_s* plan, int path, const kvc_frame* fr, uint32_t n,
                  uint32_t max_slices, void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  if ((n && !fr) || !d_ws || !aligned16(d_ws)) return KVC_ERR_INVALID;
  if (max_slices == 0 || max_slices > plan->S) max_slices = plan->S;
  if (ws_bytes < decode_ws_for(plan, path, n, max_slices)) return KVC_ERR_CAPACITY;
  int st = check_plan_device(plan);
  if (st) return st;
  for (uint32_t i = 0; i < n; ++i) {
    const kvc_frame& f = fr[i];
    if (!f.src || !f.res || (f.dst_cap && !f.dst) || !aligned16(f.src) || !aligned16(f.dst) ||
        !aligned16(f.res))
      return KVC_ERR_INVALID;
  }
  ContainerExpect ex{};
  ex.path = uint32_t(path);
  ex.dtype = plan->d.dtype;
  ex.L = plan->d.n_layers; ex.H = plan->d.n_heads; ex.T = plan->d.n_tokens; ex.D = plan->d.head_dim;
  ex.recs_per_slice = records_per_slice(plan, path);
  ex.max_slices = max_slices;
  ex.E = path == KVC_PATH_LOSSLESS ? plan->ls.E : 2u;
  if (path == KVC_PATH_LOSSLESS) {
    ex.chunk_tokens = plan->ls.tc;
  } else {
    ex.chunk_tokens = plan->ts.ct;
    ex.n_sink = plan->d.n_sink;
    ex.n_recent = plan->d.n_recent;
    ex.block_tokens = plan->d.block_tokens;
    ex.plan_crc = plan->plan_crc;
  }
  uint8_t* ws = static_cast<uint8_t*>(d_ws);
  for (uint32_t i = 0; i < n; i += kBatchMax) {
    FrameBatch b{};
    b.n = std::min<uint32_t>(kBatchMax, n - i);
    for (uint32_t k = 0; k < b.n; ++k) {
      FrameDesc& d = b.f[k];
      d.src = static_cast<const uint8_t*>(fr[i + k].src);
      d.src_bytes = fr[i + k].src_bytes;
      d.dst = static_cast<uint8_t*>(fr[i + k].dst);
      d.dst_cap = fr[i + k].dst_cap;
      d.res = fr[i + k].res;
    }
    cudaError_t e = launch_check_container(b, ex, ws, stream);
    if (e != cudaSuccess) return KVC_ERR_CUDA;
    const uint64_t max_rec64 = uint64_t(b.n) * max_slices * ex.recs_per_slice;
    const uint32_t max_rec = uint32_t(std::min<uint64_t>(max_rec64, 0xffffffffu));
    if (path == KVC_PATH_LOSSLESS) {
      e = launch_lossless_decode(plan->ls, b, ws, max_rec, stream);
    } else {
      TransformPlanDev pd{plan->d_bases, plan->d_widths, plan->d_rope, plan->d_qsplit, plan->d_comp,
                          plan->d_qdig, plan->d_qcol, plan->d_qt};
      e = launch_transform_decode(plan->ts, pd, b, ws, max_rec, stream);
    }
    if (e != cudaSuccess) return KVC_ERR_CUDA;
    e = launch_decode_finish(b, ws, stream);
    if (e != cudaSuccess) return KVC_ERR_CUDA;
  }
  return KVC_OK;
}

int encode_common(const kvc_plan_t* plan, int path, uint32_t first_slice, uint32_t n_slices,
                  const void* d_src, void* d_dst, size_t dst_cap, void* d_ws, size_t ws_bytes,
                  kvc_result* d_res, cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  if (ws_bytes < encode_ws_for(plan, path, uint64_t(n_slices) * records_per_slice(plan, path)))
    return KVC_ERR_CAPACITY;
  kvc_frame f{first_slice, n_slices, d_src, 0, d_dst, dst_cap, d_res};
  return encode_frames(plan, path, &f, 1, d_ws, ws_bytes, stream);
}

int decode_common(const kvc_plan_t* plan, int path, const void* d_src, size_t src_bytes, void* d_dst,
                  size_t dst_cap, void* d_ws, size_t ws_bytes, kvc_result* d_res,
                  cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  // the workspace bounds the slices a container may hold in this call
  uint32_t ms = plan->S;
  while (ms > 0 && decode_ws_for(plan, path, 1, ms) > ws_bytes) {
    const uint64_t per = std::max<uint64_t>(1u, (decode_ws_for(plan, path, 1, ms) - ws_bytes) /
                                                    (decode_ws_for(plan, path, 1, 1) - kDecodeWsFixed));
    ms = per >= ms ? 0u : ms - uint32_t(per);
  }
  if (ms == 0) return KVC_ERR_CAPACITY;
  kvc_frame f{0, 0, d_src, src_bytes, d_dst, dst_cap, d_res};
  return decode_frames(plan, path, &f, 1, ms, d_ws, ws_bytes, stream);
}

}  // namespace

extern "C" size_t kvc_max_encoded_bytes(const kvc_plan_t* plan, int path, uint32_t n_slices) {
  if (!path_ok(plan, path)) return 0;
  if (path == KVC_PATH_LOSSLESS) {
    const LosslessShape& s = plan->ls;
    uint64_t per = 0;
    for (uint32_t t0 = 0; t0 < s.T; t0 += s.tc) {
      uint32_t tcc = std::min(s.tc, s.T - t0);
      per += kIndexEntry + s.E * (16u + pad16u(uint64_t(tcc) * s.D));
    }
    return size_t(kHeaderBytes + per * n_slices);
  }
  return size_t(kHeaderBytes +
                uint64_t(n_slices) * (uint64_t(kIndexEntry) * (1u + plan->ts.n_mid) + plan->max_slice_bytes));
}

extern "C" size_t kvc_workspace_bytes(const kvc_plan_t* plan, int path, int decode, uint32_t n_slices) {
  if (!path_ok(plan, path)) return 0;
  if (decode) return size_t(decode_ws_for(plan, path, 1, n_slices ? n_slices : plan->S));
  return size_t(encode_ws_for(plan, path, uint64_t(n_slices) * records_per_slice(plan, path)));
}

extern "C" size_t kvc_batch_workspace_bytes(const kvc_plan_t* plan, int path, int decode,
                                            uint32_t n_frames, uint32_t max_slices_per_frame) {
  if (!path_ok(plan, path)) return 0;
  const uint32_t ms = max_slices_per_frame ? max_slices_per_frame : plan->S;
  if (decode) return size_t(decode_ws_for(plan, path, n_frames, ms));
  const uint64_t f = std::min<uint32_t>(std::max<uint32_t>(n_frames, 1u), kBatchMax);
  return size_t(encode_ws_for(plan, path, f * ms * records_per_slice(plan, path)));
}

extern "C" int kvc_encode_batch(const kvc_plan_t* plan, int path, const kvc_frame* h_frames,
                                uint32_t n_frames, void* d_ws, size_t ws_bytes, cudaStream_t stream) {
  return encode_frames(plan, path, h_frames, n_frames, d_ws, ws_bytes, stream);
}

extern "C" int kvc_decode_batch(const kvc_plan_t* plan, int path, const kvc_frame* h_frames,
                                uint32_t n_frames, uint32_t max_slices_per_frame, void* d_ws,
                                size_t ws_bytes, cudaStream_t stream) {
  return decode_frames(plan, path, h_frames, n_frames, max_slices_per_frame, d_ws, ws_bytes, stream);
}

extern "C" int kvc_encode_lossless(const kvc_plan_t* plan, uint32_t first_slice, uint32_t n_slices,
                                   const void* d_src, void* d_dst, size_t dst_cap, void* d_ws,
                                   size_t ws_bytes, kvc_result* d_res, cudaStream_t stream) {
  return encode_common(plan, KVC_PATH_LOSSLESS, first_slice, n_slices, d_src, d_dst, dst_cap, d_ws,
                       ws_bytes, d_res, stream);
}

extern "C" int kvc_decode_lossless(const kvc_plan_t* plan, const void* d_src, size_t src_bytes,
                                   void* d_dst, size_t dst_cap, void* d_ws, size_t ws_bytes,
                                   kvc_result* d_res, cudaStream_t stream) {
  return decode_common(plan, KVC_PATH_LOSSLESS, d_src, src_bytes, d_dst, dst_cap, d_ws, ws_bytes,
                       d_res, stream);
}

extern "C" int kvc_encode_transform(const kvc_plan_t* plan, uint32_t first_slice, uint32_t n_slices,
                                    const void* d_src, void* d_dst, size_t dst_cap, void* d_ws,
                                    size_t ws_bytes, kvc_result* d_res, cudaStream_t stream) {
  return encode_common(plan, KVC_PATH_TRANSFORM, first_slice, n_slices, d_src, d_dst, dst_cap, d_ws,
                       ws_bytes, d_res, stream);
}

extern "C" int kvc_decode_transform(const kvc_plan_t* plan, const void* d_src, size_t src_bytes,
                                    void* d_dst, size_t dst_cap, void* d_ws, size_t ws_bytes,
                                    kvc_result* d_res, cudaStream_t stream) {
  return decode_common(plan, KVC_PATH_TRANSFORM, d_src, src_bytes, d_dst, dst_cap, d_ws, ws_bytes,
                       d_res, stream);
}

extern "C" int kvc_allocate_bits(const double* h_eigvals, uint64_t n_units, double avg_bits,
                                 uint32_t max_bits, uint8_t* h_widths) {
  if (!h_eigvals || !h_widths || !n_units || max_bits > 8) return KVC_ERR_INVALID;
  std::vector<uint8_t> w;
  if (!allocate_widths(h_eigvals, n_units, avg_bits, max_bits, w)) return KVC_ERR_INVALID;
  std::memcpy(h_widths, w.data(), w.size());
  return KVC_OK;
}

// ------------------------------------------------------------------ kernel timing
namespace {

struct ProfState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;
  size_t used = 0;
  struct Rec { const char* name; cudaEvent_t a, b; };
  std::vector<Rec> recs;
  cudaEvent_t pending = nullptr;
  const char* pending_name = nullptr;
};
ProfState& prof() {
  static ProfState p;
  return p;
}
cudaEvent_t prof_event(ProfState& p) {
  if (p.used == p.pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    p.pool.push_back(e);
  }
  return p.pool[p.used++];
}

}  // namespace

namespace kvc {
bool prof_enabled() { return prof().on; }
void prof_record(const char* name, cudaStream_t st, bool end) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  if (!p.on) return;
  cudaEvent_t e = prof_event(p);
  if (!e) return;
  cudaEventRecord(e, st);
  if (!end) {
    p.pending = e;
    p.pending_name = name;
  } else if (p.pending) {
    p.recs.push_back({name, p.pending, e});
    p.pending = nullptr;
  }
}
}  // namespace kvc

extern "C" int kvc_profile_begin(void) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = true;
  p.used = 0;
  p.recs.clear();
  p.pending = nullptr;
  return KVC_OK;
}

extern "C" int kvc_profile_end(kvc_kernel_time* out, int max_kernels, int* n_kernels) {
  ProfState& p = prof();
  std::lock_guard<std::mutex> g(p.mu);
  p.on = false;
  std::vector<std::string> names;
  std::vector<kvc_kernel_time> agg;
  int st = KVC_OK;
  for (auto& r : p.recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      st = KVC_ERR_CUDA;
      continue;
    }
    size_t k = 0;
    while (k < names.size() && names[k] != r.name) ++k;
    if (k == names.size()) {
      names.push_back(r.name);
      kvc_kernel_time t{};
      std::strncpy(t.name, r.name, sizeof t.name - 1);
      agg.push_back(t);
    }
    agg[k].launches++;
    agg[k].total_ms += ms;
  }
  p.recs.clear();
  p.used = 0;
  int n = std::min<int>(int(agg.size()), max_kernels);
  for (int i = 0; i < n; ++i) out[i] = agg[i];
  if (n_kernels) *n_kernels = n;
  return st;
}

// ------------------------------------------------------------------ host-streamed coding
namespace {

constexpr uint32_t kStreamSlots = 3;  // depth of the device ring

uint32_t value_bytes(const kvc_plan_s* p, int path) { return path == KVC_PATH_LOSSLESS ? p->ls.E : 2u; }

struct StreamRing {
  uint64_t raw_bytes = 0, cont_bytes = 0, slot_bytes = 0, ws_bytes = 0;
};

// Per slot: a raw frame, a container of frame_slices slices and a result;
// then one workspace shared by the frames (they are coded one after another).
StreamRing stream_ring(const kvc_plan_s* p, int path, uint32_t fs) {
  StreamRing r;
  r.raw_bytes = pad256u(uint64_t(fs) * p->d.n_tokens * p->d.head_dim * value_bytes(p, path));
  r.cont_bytes = pad256u(kvc_max_encoded_bytes(p, path, fs));
  r.slot_bytes = r.raw_bytes + r.cont_bytes + 256u;
  r.ws_bytes = pad256u(std::max(encode_ws_for(p, path, uint64_t(fs) * records_per_slice(p, path)),
                                decode_ws_for(p, path, 1, fs)));
  return r;
}

// The plan's two copy streams and the ring's events, made on first use.
struct StreamCall {
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t *ev_in = nullptr, *ev_coded = nullptr, *ev_out = nullptr;
  bool ok = true;
  explicit StreamCall(kvc_plan_s* p) {
    if (!p->copy_in) ok = cudaStreamCreateWithFlags(&p->copy_in, cudaStreamNonBlocking) == cudaSuccess;
    if (ok && !p->copy_out) ok = cudaStreamCreateWithFlags(&p->copy_out, cudaStreamNonBlocking) == cudaSuccess;
    for (auto& row : p->ring_ev)
      for (cudaEvent_t& e : row)
        if (ok && !e) ok = cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    in = p->copy_in;
    out = p->copy_out;
    ev_in = p->ring_ev[0];
    ev_coded = p->ring_ev[1];
    ev_out = p->ring_ev[2];
  }
};

}  // namespace

extern "C" size_t kvc_stream_buffer_bytes(const kvc_plan_t* plan, int path, uint32_t frame_slices) {
  if (!path_ok(plan, path) || frame_slices == 0 || frame_slices > plan->S) return 0;
  const StreamRing r = stream_ring(plan, path, frame_slices);
  return size_t(kStreamSlots * r.slot_bytes + r.ws_bytes);
}

extern "C" int kvc_stream_encode_host(const kvc_plan_t* plan, int path, uint32_t first_slice, uint32_t n_slices,
                                      uint32_t frame_slices, const void* h_src, void* h_dst, size_t dst_cap,
                                      uint64_t* h_frame_bytes, kvc_result* h_results, void* d_buf,
                                      size_t buf_bytes, cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  if (frame_slices == 0 || frame_slices > plan->S || uint64_t(first_slice) + n_slices > plan->S || !d_buf ||
      (reinterpret_cast<uintptr_t>(d_buf) & 255u) ||
      (n_slices && (!h_src || !h_dst || !h_frame_bytes || !h_results)))
    return KVC_ERR_INVALID;
  int st = check_plan_device(plan);
  if (st) return st;
  const StreamRing R = stream_ring(plan, path, frame_slices);
  if (buf_bytes < kStreamSlots * R.slot_bytes + R.ws_bytes) return KVC_ERR_CAPACITY;
  if (n_slices == 0) return KVC_OK;
  StreamCall sc(const_cast<kvc_plan_s*>(plan));
  if (!sc.ok) return KVC_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(d_buf);
  auto raw = [&](uint32_t k) { return base + k * R.slot_bytes; };
  auto cont = [&](uint32_t k) { return raw(k) + R.raw_bytes; };
  auto res = [&](uint32_t k) { return reinterpret_cast<kvc_result*>(cont(k) + R.cont_bytes); };
  uint8_t* ws = base + kStreamSlots * R.slot_bytes;
  const uint64_t slice_bytes = uint64_t(plan->d.n_tokens) * plan->d.head_dim * value_bytes(plan, path);
  const uint32_t nf = (n_slices + frame_slices - 1) / frame_slices;
  const uint8_t* src = static_cast<const uint8_t*>(h_src);
  uint8_t* dst = static_cast<uint8_t*>(h_dst);
  uint64_t dst_off = 0;
  int ret = KVC_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && ret == KVC_OK) ret = KVC_ERR_CUDA;
  };
  // Frame g's container goes out once its encode has reported the size; the
  // host asks two frames after issuing it, so the copy engines never idle on it.
  auto drain = [&](uint32_t g) {
    const uint32_t k = g % kStreamSlots;
    ck(cudaEventSynchronize(sc.ev_coded[k]));
    uint64_t n = ret == KVC_OK && h_results[g].status == KVC_OK ? h_results[g].bytes : 0u;
    if (n > R.cont_bytes && ret == KVC_OK) ret = KVC_ERR_CUDA;  // a size no encode can report
    if (n > R.cont_bytes || dst_off + n > dst_cap) {
      if (ret == KVC_OK) ret = KVC_ERR_CAPACITY;
      n = 0;
    }
    h_frame_bytes[g] = n;
    ck(cudaStreamWaitEvent(sc.out, sc.ev_coded[k], 0));
    if (n) ck(cudaMemcpyAsync(dst + dst_off, cont(k), n, cudaMemcpyDeviceToHost, sc.out));
    ck(cudaEventRecord(sc.ev_out[k], sc.out));
    dst_off += n;
  };
  for (uint32_t f = 0; f < nf && ret == KVC_OK; ++f) {
    const uint32_t k = f % kStreamSlots, s0 = f * frame_slices, ns = std::min(frame_slices, n_slices - s0);
    if (f >= kStreamSlots) ck(cudaStreamWaitEvent(sc.in, sc.ev_coded[k], 0));  // frame f - 3 read the slot
    ck(cudaMemcpyAsync(raw(k), src + s0 * slice_bytes, ns * slice_bytes, cudaMemcpyHostToDevice, sc.in));
    ck(cudaEventRecord(sc.ev_in[k], sc.in));
    if (f + 1 >= kStreamSlots) drain(f + 1 - kStreamSlots);
    ck(cudaStreamWaitEvent(stream, sc.ev_in[k], 0));
    if (f >= kStreamSlots) ck(cudaStreamWaitEvent(stream, sc.ev_out[k], 0));  // its container is out
    if (ret != KVC_OK) break;
    const kvc_frame fr{first_slice + s0, ns, raw(k), 0, cont(k), size_t(R.cont_bytes), res(k)};
    const int e = encode_frames(plan, path, &fr, 1, ws, size_t(R.ws_bytes), stream);
    if (e != KVC_OK) ret = e;
    ck(cudaMemcpyAsync(&h_results[f], res(k), sizeof(kvc_result), cudaMemcpyDeviceToHost, stream));
    ck(cudaEventRecord(sc.ev_coded[k], stream));
  }
  for (uint32_t g = nf + 1 > kStreamSlots ? nf + 1 - kStreamSlots : 0u; g < nf && ret == KVC_OK; ++g) drain(g);
  ck(cudaStreamSynchronize(sc.in));
  ck(cudaStreamSynchronize(stream));
  ck(cudaStreamSynchronize(sc.out));
  return ret;
}

extern "C" int kvc_stream_decode_host(const kvc_plan_t* plan, int path, uint32_t n_slices, uint32_t frame_slices,
                                      const void* h_src, const uint64_t* h_frame_bytes, void* h_dst,
                                      size_t dst_cap, kvc_result* h_results, void* d_buf, size_t buf_bytes,
                                      cudaStream_t stream) {
  if (!path_ok(plan, path)) return plan ? KVC_ERR_UNSUPPORTED : KVC_ERR_INVALID;
  if (frame_slices == 0 || frame_slices > plan->S || n_slices > plan->S || !d_buf ||
      (reinterpret_cast<uintptr_t>(d_buf) & 255u) ||
      (n_slices && (!h_src || !h_dst || !h_frame_bytes || !h_results)))
    return KVC_ERR_INVALID;
  int st = check_plan_device(plan);
  if (st) return st;
  const StreamRing R = stream_ring(plan, path, frame_slices);
  if (buf_bytes < kStreamSlots * R.slot_bytes + R.ws_bytes) return KVC_ERR_CAPACITY;
  const uint64_t slice_bytes = uint64_t(plan->d.n_tokens) * plan->d.head_dim * value_bytes(plan, path);
  if (dst_cap < n_slices * slice_bytes) return KVC_ERR_CAPACITY;
  if (n_slices == 0) return KVC_OK;
  StreamCall sc(const_cast<kvc_plan_s*>(plan));
  if (!sc.ok) return KVC_ERR_CUDA;
  uint8_t* base = static_cast<uint8_t*>(d_buf);
  auto raw = [&](uint32_t k) { return base + k * R.slot_bytes; };
  auto cont = [&](uint32_t k) { return raw(k) + R.raw_bytes; };
  auto res = [&](uint32_t k) { return reinterpret_cast<kvc_result*>(cont(k) + R.cont_bytes); };
  uint8_t* ws = base + kStreamSlots * R.slot_bytes;
  const uint32_t nf = (n_slices + frame_slices - 1) / frame_slices;
  const uint8_t* src = static_cast<const uint8_t*>(h_src);
  uint8_t* dst = static_cast<uint8_t*>(h_dst);
  uint64_t src_off = 0;
  int ret = KVC_OK;
  auto ck = [&](cudaError_t e) {
    if (e != cudaSuccess && ret == KVC_OK) ret = KVC_ERR_CUDA;
  };
  for (uint32_t f = 0; f < nf && ret == KVC_OK; ++f) {
    const uint32_t k = f % kStreamSlots, s0 = f * frame_slices, ns = std::min(frame_slices, n_slices - s0);
    const uint64_t nb = h_frame_bytes[f];
    if (nb > R.cont_bytes) {  // longer than any container of frame_slices slices
      h_results[f].status = KVC_ERR_CORRUPT;
      h_results[f].bytes = 0;
      src_off += nb;
      continue;
    }
    if (f >= kStreamSlots) ck(cudaStreamWaitEvent(sc.in, sc.ev_coded[k], 0));  // frame f - 3 read the slot
    if (nb) ck(cudaMemcpyAsync(cont(k), src + src_off, nb, cudaMemcpyHostToDevice, sc.in));
    ck(cudaEventRecord(sc.ev_in[k], sc.in));
    ck(cudaStreamWaitEvent(stream, sc.ev_in[k], 0));
    if (f >= kStreamSlots) ck(cudaStreamWaitEvent(stream, sc.ev_out[k], 0));  // its values are out
    if (ret != KVC_OK) break;
    const kvc_frame fr{0, 0, cont(k), size_t(nb), raw(k), size_t(ns * slice_bytes), res(k)};
    const int e = decode_frames(plan, path, &fr, 1, frame_slices, ws, size_t(R.ws_bytes), stream);
    if (e != KVC_OK) ret = e;
    ck(cudaMemcpyAsync(&h_results[f], res(k), sizeof(kvc_result), cudaMemcpyDeviceToHost, stream));
    ck(cudaEventRecord(sc.ev_coded[k], stream));
    ck(cudaStreamWaitEvent(sc.out, sc.ev_coded[k], 0));
    ck(cudaMemcpyAsync(dst + s0 * slice_bytes, raw(k), ns * slice_bytes, cudaMemcpyDeviceToHost, sc.out));
    ck(cudaEventRecord(sc.ev_out[k], sc.out));
    src_off += nb;
  }
  ck(cudaStreamSynchronize(sc.in));
  ck(cudaStreamSynchronize(stream));
  ck(cudaStreamSynchronize(sc.out));
  return ret;
}

extern "C" const char* kvc_status_string(int status) {
  switch (status) {
    case KVC_OK: return "ok";
    case KVC_ERR_INVALID: return "invalid argument";
    case KVC_ERR_CAPACITY: return "capacity too small";
    case KVC_ERR_CORRUPT: return "corrupt input";
    case KVC_ERR_TRUNCATED: return "truncated input";
    case KVC_ERR_PLAN_MISMATCH: return "plan mismatch";
    case KVC_ERR_TIMEOUT: return "device wait timed out";
    case KVC_ERR_CUDA: return "CUDA error";
    case KVC_ERR_UNSUPPORTED: return "unsupported";
    default: return "unknown status";
  }
}

extern "C" int kvc_stage_crc32(const void* d_src, size_t n, uint32_t* d_out, cudaStream_t stream) {
  if ((n && !d_src) || !d_out) return KVC_ERR_INVALID;
  return cuda_status(launch_stage_crc32(static_cast<const uint8_t*>(d_src), n, d_out, stream));
}

extern "C" int kvc_stage_stream_encode(const uint8_t* d_sym, uint32_t n, uint8_t* d_out,
                                       void* d_scratch, kvc_result* d_res, cudaStream_t stream) {
  if (n == 0 || n > kMaxChunkValues || !d_sym || !d_out || !d_scratch || !d_res ||
      !aligned16(d_out) || (reinterpret_cast<uintptr_t>(d_scratch) & 1u))
    return KVC_ERR_INVALID;
  return cuda_status(launch_stage_stream_encode(d_sym, n, d_out, static_cast<uint16_t*>(d_scratch),
                                                d_res, stream));
}

extern "C" int kvc_stage_stream_decode(const uint8_t* d_rec, uint32_t rec_bytes, uint32_t n,
                                       uint8_t* d_sym, kvc_result* d_res, cudaStream_t stream) {
  if (n == 0 || n > kMaxChunkValues || !d_rec || !d_sym || !d_res || !aligned16(d_rec))
    return KVC_ERR_INVALID;
  return cuda_status(launch_stage_stream_decode(d_rec, rec_bytes, n, d_sym, d_res, stream));
}

// ------------------------------------------------------------------ calibration
namespace {

// Symmetric eigen-decomposition (Golub & Van Loan, "Matrix Computations",
// symmetric QR algorithm): Householder reflections bring A to tridiagonal form
// T = V^T A V, then implicit QR steps with the Wilkinson shift, each a chase of
// Givens rotations down the unreduced block, diagonalise T while V collects the
// rotations. Dense storage (n is a head dimension). a (n x n, row-major) is
// replaced by the eigenvectors (columns); w gets the eigenvalues.
void sym_eigen(std::vector<double>& a, int n, std::vector<double>& w) {
  std::vector<double> T = a, V(size_t(n) * n, 0.0), v(n), p(n), q(n);
  auto at = [n](std::vector<double>& m, int i, int j) -> double& { return m[size_t(i) * n + j]; };
  for (int i = 0; i < n; ++i) at(V, i, i) = 1.0;
  for (int k = 0; k + 2 < n; ++k) {
    double norm2 = 0.0;
    for (int i = k + 1; i < n; ++i) norm2 += at(T, i, k) * at(T, i, k);
    const double alpha = std::sqrt(norm2);
    if (alpha == 0.0) continue;
    const double x0 = at(T, k + 1, k);
    const double target = x0 >= 0.0 ? -alpha : alpha;  // T[k+1][k] after the reflection
    std::fill(v.begin(), v.end(), 0.0);
    v[k + 1] = x0 - target;
    for (int i = k + 2; i < n; ++i) v[i] = at(T, i, k);
    double vv = 0.0;
    for (int i = k + 1; i < n; ++i) vv += v[i] * v[i];
    if (vv == 0.0) continue;
    const double beta = 2.0 / vv;
    // T <- H T H with H = I - beta v v^T: T -= v q^T + q v^T, q = p - (beta p.v / 2) v, p = beta T v
    double pv = 0.0;
    for (int i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int j = k + 1; j < n; ++j) acc += at(T, i, j) * v[j];
      p[i] = beta * acc;
      pv += p[i] * v[i];
    }
    const double half = 0.5 * beta * pv;
    for (int i = 0; i < n; ++i) q[i] = p[i] - half * v[i];
    for (int i = 0; i < n; ++i)
      for (int j = 0; j < n; ++j) at(T, i, j) -= v[i] * q[j] + q[i] * v[j];
    // V <- V H
    for (int i = 0; i < n; ++i) {
      double acc = 0.0;
      for (int j = k + 1; j < n; ++j) acc += at(V, i, j) * v[j];
      acc *= beta;
      for (int j = k + 1; j < n; ++j) at(V, i, j) -= acc * v[j];
    }
  }
  for (int i = 0; i < n; ++i)
    for (int j = 0; j < n; ++j)
      if (j < i - 1 || j > i + 1) at(T, i, j) = 0.0;
  auto negligible = [&](int i) {  // T[i][i-1]
    return std::fabs(at(T, i, i - 1)) <= 1e-15 * (std::fabs(at(T, i, i)) + std::fabs(at(T, i - 1, i - 1)));
  };
  int hi = n - 1;
  for (int guard = 0; hi > 0 && guard < 64 * n; ++guard) {
    if (negligible(hi)) {
      at(T, hi, hi - 1) = at(T, hi - 1, hi) = 0.0;
      --hi;
      continue;
    }
    int lo = hi - 1;
    while (lo > 0 && !negligible(lo)) --lo;
    if (lo > 0) at(T, lo, lo - 1) = at(T, lo - 1, lo) = 0.0;
    const double ta = at(T, hi - 1, hi - 1), tb = at(T, hi, hi - 1), tc = at(T, hi, hi);
    const double delta = 0.5 * (ta - tc);
    const double mu = tc - tb * tb / (delta + (delta >= 0.0 ? 1.0 : -1.0) * std::hypot(delta, tb));
    double x = at(T, lo, lo) - mu, z = at(T, lo + 1, lo);
    for (int k = lo; k < hi; ++k) {
      const double r = std::hypot(x, z);
      const double c = r == 0.0 ? 1.0 : x / r, s = r == 0.0 ? 0.0 : -z / r;
      // rows k, k+1 then columns k, k+1 of T (block lo..hi); columns of V
      for (int j = lo; j <= hi; ++j) {
        const double u0 = at(T, k, j), u1 = at(T, k + 1, j);
        at(T, k, j) = c * u0 - s * u1;
        at(T, k + 1, j) = s * u0 + c * u1;
      }
      for (int i = lo; i <= hi; ++i) {
        const double u0 = at(T, i, k), u1 = at(T, i, k + 1);
        at(T, i, k) = c * u0 - s * u1;
        at(T, i, k + 1) = s * u0 + c * u1;
      }
      for (int i = 0; i < n; ++i) {
        const double u0 = at(V, i, k), u1 = at(V, i, k + 1);
        at(V, i, k) = c * u0 - s * u1;
        at(V, i, k + 1) = s * u0 + c * u1;
      }
      if (k + 1 < hi) {
        x = at(T, k + 1, k);
        z = at(T, k + 2, k);
      }
    }
  }
  w.resize(n);
  for (int i = 0; i < n; ++i) w[i] = at(T, i, i);
  a = V;
}

}  // namespace

namespace {
// Uncentered second moments C = (1/n) sum_t x_t x_t^T of slice s's calibration
// tokens (keys de-rotated with the fp32 table cs), fp64, t ascending.
void calib_moments(const kvc_plan_desc& d, uint32_t s, const uint16_t* h_calib, uint32_t n_calib,
                   const std::vector<float>& cs, std::vector<double>& C) {
  const uint32_t D = d.head_dim, half = D / 2;
  const bool key = ((s / d.n_heads) & 1u) == 0;
  C.assign(size_t(D) * D, 0.0);
  std::vector<float> x(D);
  const uint16_t* xs = h_calib + size_t(s) * n_calib * D;
  for (uint32_t t = 0; t < n_calib; ++t) {
    for (uint32_t k = 0; k < D; ++k) {
      uint32_t bits = uint32_t(xs[size_t(t) * D + k]) << 16;
      std::memcpy(&x[k], &bits, 4);
    }
    if (key) {
      const float* row = cs.data() + size_t(t) * half * 2;
      for (uint32_t i = 0; i < half; ++i) {
        volatile float a = x[i], b = x[i + half], c = row[2 * i], sn = row[2 * i + 1];
        volatile float ac = a * c, bs = b * sn, bc = b * c, as = a * sn;
        x[i] = ac + bs;
        x[i + half] = bc - as;
      }
    }
    for (uint32_t a = 0; a < D; ++a) {
      const double xa = x[a];
      double* Ca = C.data() + size_t(a) * D;
      for (uint32_t b = 0; b <= a; ++b) Ca[b] += xa * double(x[b]);
    }
  }
  for (uint32_t a = 0; a < D; ++a)
    for (uint32_t b = 0; b <= a; ++b) {
      double v = C[size_t(a) * D + b] / double(n_calib);
      C[size_t(a) * D + b] = v;
      C[size_t(b) * D + a] = v;
    }
}

bool calib_desc_ok(const kvc_plan_desc& d) {
  return d.dtype == KVC_DTYPE_BF16 && d.head_dim && !(d.head_dim & 1u) && d.rope_theta > 0.0 && d.n_layers &&
         d.n_heads;
}
}  // namespace

extern "C" int kvc_calibrate_pca(const kvc_plan_desc* desc, const uint16_t* h_calib, uint32_t n_calib,
                                 float* h_bases, double* h_eigvals, int n_threads) {
  if (!desc || !h_calib || !h_bases || !h_eigvals || !n_calib) return KVC_ERR_INVALID;
  const kvc_plan_desc& d = *desc;
  if (!calib_desc_ok(d)) return KVC_ERR_INVALID;
  const uint32_t D = d.head_dim, S = d.n_layers * 2u * d.n_heads;
  std::vector<float> cs;
  rope_table(n_calib, D, d.rope_theta, cs);
  parallel_for(S, n_workers(n_threads), [&](uint32_t s) {
    std::vector<double> C;
    calib_moments(d, s, h_calib, n_calib, cs, C);
    std::vector<double> w;
    sym_eigen(C, int(D), w);
    std::vector<uint32_t> order(D);
    for (uint32_t j = 0; j < D; ++j) order[j] = j;
    std::stable_sort(order.begin(), order.end(), [&](uint32_t a, uint32_t b) { return w[a] > w[b]; });
    float* Q = h_bases + size_t(s) * D * D;
    for (uint32_t j = 0; j < D; ++j) {
      const uint32_t c = order[j];
      uint32_t arg = 0;
      for (uint32_t k = 1; k < D; ++k)
        if (std::fabs(C[size_t(k) * D + c]) > std::fabs(C[size_t(arg) * D + c])) arg = k;
      const double sign = C[size_t(arg) * D + c] < 0.0 ? -1.0 : 1.0;
      for (uint32_t k = 0; k < D; ++k) Q[size_t(k) * D + j] = float(sign * C[size_t(k) * D + c]);
      h_eigvals[size_t(s) * D + j] = w[c];
    }
  });
  return KVC_OK;
}

extern "C" int kvc_fixed_basis(int kind, uint32_t D, float* h_basis) {
  if (!h_basis || !D) return KVC_ERR_INVALID;
  if (kind == KVC_BASIS_HADAMARD) {
    if (D & (D - 1u)) return KVC_ERR_INVALID;
    const double inv = 1.0 / std::sqrt(double(D));
    for (uint32_t k = 0; k < D; ++k)
      for (uint32_t j = 0; j < D; ++j)
        h_basis[size_t(k) * D + j] = float((__builtin_popcount(k & j) & 1) ? -inv : inv);
    return KVC_OK;
  }
  if (kind == KVC_BASIS_DCT) {
    const double pi = 3.141592653589793;
    for (uint32_t j = 0; j < D; ++j) {
      const double c = j == 0 ? std::sqrt(1.0 / double(D)) : std::sqrt(2.0 / double(D));
      for (uint32_t k = 0; k < D; ++k) {
        const double ang = pi * double((2u * k + 1u) * j) / double(2u * D);
        h_basis[size_t(k) * D + j] = float(c * std::cos(ang));
      }
    }
    return KVC_OK;
  }
  return KVC_ERR_INVALID;
}

extern "C" int kvc_calibrate_basis(const kvc_plan_desc* desc, int kind, const uint16_t* h_calib,
                                   uint32_t n_calib, float* h_bases, double* h_eigvals, int n_threads) {
  if (kind == KVC_BASIS_PCA) return kvc_calibrate_pca(desc, h_calib, n_calib, h_bases, h_eigvals, n_threads);
  if (!desc || !h_calib || !h_bases || !h_eigvals || !n_calib) return KVC_ERR_INVALID;
  const kvc_plan_desc& d = *desc;
  if (!calib_desc_ok(d)) return KVC_ERR_INVALID;
  const uint32_t D = d.head_dim, S = d.n_layers * 2u * d.n_heads;
  std::vector<float> Q(size_t(D) * D);
  const int st = kvc_fixed_basis(kind, D, Q.data());
  if (st != KVC_OK) return st;
  std::vector<float> cs;
  rope_table(n_calib, D, d.rope_theta, cs);
  parallel_for(S, n_workers(n_threads), [&](uint32_t s) {
    std::vector<double> C;
    calib_moments(d, s, h_calib, n_calib, cs, C);
    std::memcpy(h_bases + size_t(s) * D * D, Q.data(), sizeof(float) * D * D);
    for (uint32_t j = 0; j < D; ++j) {  // q_j^T C q_j, a and b ascending
      double lam = 0.0;
      for (uint32_t a = 0; a < D; ++a) {
        double acc = 0.0;
        for (uint32_t b = 0; b < D; ++b) acc += C[size_t(a) * D + b] * double(Q[size_t(b) * D + j]);
        lam += double(Q[size_t(a) * D + j]) * acc;
      }
      h_eigvals[size_t(s) * D + j] = lam;
    }
  });
  return KVC_OK;
}
