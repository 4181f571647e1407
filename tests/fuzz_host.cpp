// Host fuzz driver for the library's host-side code, built with
// AddressSanitizer and UndefinedBehaviorSanitizer by tests/test_host_fuzz.py
// (api.cpp compiled here with the sanitizers; the device objects are linked as
// built). It calls only entry points that run on the host: plan validation
// and sizing, the greedy bit allocation, the calibration solvers (PCA by
// Householder tridiagonalisation and QR, the fixed Hadamard / DCT-II bases
// and their variances), with valid, extreme and invalid arguments. Plans that
// need a device fail cleanly when there is none. Every call must return a
// status and stay inside its buffers.
#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <vector>

#include "kvc.h"

static uint64_t rs = 0x243F6A8885A308D3ull;
static uint64_t rnd() {
  rs ^= rs << 13;
  rs ^= rs >> 7;
  rs ^= rs << 17;
  return rs;
}
static double unit() { return double(rnd() >> 11) * (1.0 / 9007199254740992.0); }
static uint16_t bf16(float f) {
  uint32_t x;
  std::memcpy(&x, &f, 4);
  return uint16_t((x + 0x7fffu + ((x >> 16) & 1u)) >> 16);
}

static kvc_plan_desc base_desc(uint32_t dtype, uint32_t L, uint32_t H, uint32_t T, uint32_t D) {
  kvc_plan_desc d;
  std::memset(&d, 0, sizeof d);
  d.abi_version = KVC_ABI_VERSION;
  d.dtype = dtype;
  d.n_layers = L; d.n_heads = H; d.n_tokens = T; d.head_dim = D;
  d.values_per_chunk = 65536; d.n_sink = 4; d.n_recent = 128; d.block_tokens = 64; d.chunk_tokens = 512;
  d.max_bits = 8; d.rope_theta = 10000.0; d.avg_bits = 2.0;
  return d;
}

int main() {
  int calls = 0;
  // allocation: random, tied, zero and slightly negative variances; every budget edge
  for (int trial = 0; trial < 300; ++trial) {
    const uint64_t U = 1 + rnd() % 3000;
    std::vector<double> lam(U);
    for (auto& l : lam) l = std::exp((unit() - 0.5) * 12.0);
    if (trial % 3 == 0) for (uint64_t i = 0; i < U / 4; ++i) lam[rnd() % U] = 1.0;
    if (trial % 5 == 1) for (uint64_t i = 0; i < U / 5; ++i) lam[rnd() % U] = (rnd() & 1) ? 0.0 : -1e-17;
    std::vector<uint8_t> w(U);
    const uint32_t mb = uint32_t(rnd() % 10);
    const double avg = (trial % 7 == 0) ? double(mb) + 0.5 : unit() * 9.0;
    kvc_allocate_bits(lam.data(), U, avg, mb, w.data());
    ++calls;
  }
  // fixed bases, valid and invalid sizes and kinds
  for (uint32_t D : {0u, 1u, 2u, 6u, 8u, 64u, 96u, 128u, 256u}) {
    std::vector<float> q(size_t(D) * D + 1);
    for (int kind : {-1, 0, 1, 2, 3}) {
      kvc_fixed_basis(kind, D, q.data());
      ++calls;
    }
  }
  // calibration: PCA and fixed bases on random, constant and degenerate draws
  for (uint32_t D : {8u, 16u, 128u}) {
    for (uint32_t n_calib : {0u, 1u, 7u, 64u}) {
      kvc_plan_desc d = base_desc(KVC_DTYPE_BF16, 1, 1, 256, D);
      const uint32_t S = 2;
      std::vector<uint16_t> cal(size_t(S) * n_calib * D + 1);
      const int pattern = int(rnd() % 3);
      for (auto& v : cal) v = pattern == 0 ? bf16(float(unit() * 4 - 2)) : pattern == 1 ? bf16(1.5f) : uint16_t(0);
      std::vector<float> bases(size_t(S) * D * D);
      std::vector<double> ev(size_t(S) * D);
      for (int kind : {int(KVC_BASIS_PCA), int(KVC_BASIS_HADAMARD), int(KVC_BASIS_DCT), 7}) {
        kvc_calibrate_basis(&d, kind, cal.data(), n_calib, bases.data(), ev.data(), 2);
        ++calls;
      }
      kvc_calibrate_pca(&d, cal.data(), n_calib, bases.data(), ev.data(), 1);
      ++calls;
    }
  }
  // plans: lossless shapes (valid and invalid), sizes; transform plans whose
  // upload fails without a device after their host work
  for (int trial = 0; trial < 200; ++trial) {
    const uint32_t dtype = uint32_t(rnd() % 5);
    const uint32_t D = uint32_t(rnd() % 3 == 0 ? 128 : 1 + rnd() % 200);
    kvc_plan_desc d = base_desc(dtype, uint32_t(rnd() % 4), uint32_t(1 + rnd() % 3), uint32_t(rnd() % 5000), D);
    d.values_per_chunk = uint32_t(rnd() % 3 == 0 ? 65536 : rnd() % 70000);
    kvc_plan_t* p = nullptr;
    if (kvc_plan_create(&d, &p) == KVC_OK && p) {
      for (int path : {0, 1, 2}) {
        kvc_max_encoded_bytes(p, path, uint32_t(rnd() % 9));
        kvc_workspace_bytes(p, path, int(rnd() & 1), uint32_t(rnd() % 9));
        kvc_batch_workspace_bytes(p, path, int(rnd() & 1), uint32_t(rnd() % 70), uint32_t(rnd() % 9));
        kvc_stream_buffer_bytes(p, path, uint32_t(rnd() % 9));
      }
      kvc_plan_destroy(p);
    }
    ++calls;
  }
  for (int trial = 0; trial < 40; ++trial) {
    const uint32_t D = trial % 4 == 0 ? 64 : 128;
    kvc_plan_desc d = base_desc(KVC_DTYPE_BF16, 1, 1, uint32_t(100 + rnd() % 900), D);
    const uint32_t S = 2;
    std::vector<float> q(size_t(S) * D * D, 0.0f);
    for (uint32_t s = 0; s < S; ++s)
      for (uint32_t j = 0; j < D; ++j) q[(size_t(s) * D + j) * D + j] = trial % 5 == 3 ? 2.0f : 1.0f;
    std::vector<double> ev(size_t(S) * D);
    for (auto& e : ev) e = unit();
    std::vector<uint8_t> w(size_t(S) * D);
    for (auto& x : w) x = uint8_t(rnd() % 10);
    d.bases = q.data();
    if (trial & 1) d.widths = w.data(); else d.eigvals = ev.data();
    d.avg_bits = unit() * 8.0;
    d.block_tokens = trial % 7 == 0 ? 48 : 64;
    kvc_plan_t* p = nullptr;
    if (kvc_plan_create(&d, &p) == KVC_OK && p) kvc_plan_destroy(p);
    ++calls;
  }
  for (int s = -2; s < 12; ++s) kvc_status_string(s);
  std::printf("%d calls\nok\n", calls);
  return 0;
}
