/*
 * kvgen — seeded synthetic KV-cache generator.
 *
 * This module only makes inputs. It holds none of the codec's arithmetic and is
 * shared, as a pure input source, by the CPU oracle and by the GPU codec's tests
 * and benchmark.
 *
 * Workload model (stands in for the exported caches the pages measure, which are
 * not available here):
 *   cache layout [L][2][H][T][D] (K = 0, V = 1), one "slice" = one [T][D] block,
 *   slice index = (l * 2 + kv) * H + h.
 *   per channel (l, kv, h, d):  mu ~ N(0,1), sigma = exp(0.5 * N(0,1))
 *   per token:  z_0 = e_0,  z_t = rho * z_{t-1} + sqrt(1 - rho^2) * e_t,
 *               x = mu + sigma * z                              (fp64)
 *   keys only:  rotary position encoding at position t, half-split pairs
 *               (i, i + D/2), angle t * theta^(-2i/D)          (fp64)
 *   stored:     fp64 -> fp32 -> bf16 or fp16, each step round-to-nearest-even.
 *
 * Random numbers: SplitMix64's output mixer (Steele, Lea & Flood, OOPSLA 2014)
 * used as a counter-based generator over a hashed key, then the Box-Muller
 * transform in fp64. Keys: (seed, 0, l, kv, h, d) channel parameters,
 * (seed, 1, l, kv, h, d) data noise, (seed, 2, ...) calibration noise,
 * (seed, 3) the uniform random control block.
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <unistd.h>

#define KVGEN_BF16 1
#define KVGEN_FP16 2
#define KVGEN_F32 3   /* 4-byte IEEE single: the fp64 value rounded to nearest */

static uint64_t mix64(uint64_t z) {
  z += 0x9e3779b97f4a7c15ULL;
  z = (z ^ (z >> 30)) * 0xbf58476d1ce4e5b9ULL;
  z = (z ^ (z >> 27)) * 0x94d049bb133111ebULL;
  return z ^ (z >> 31);
}

static uint64_t chain(uint64_t h, uint64_t v) { return mix64(h ^ mix64(v)); }

static uint64_t channel_key(uint64_t seed, uint64_t stream, uint64_t l, uint64_t kv,
                            uint64_t h, uint64_t d) {
  uint64_t k = mix64(seed);
  k = chain(k, stream);
  k = chain(k, l);
  k = chain(k, kv);
  k = chain(k, h);
  k = chain(k, d);
  return k;
}

/* uniform in (0, 1] with 53 random bits */
static double unif(uint64_t r) { return (double)((r >> 11) + 1) * 0x1.0p-53; }

/* two standard normals from counter pair (2p, 2p+1) of a key */
static void normal_pair(uint64_t key, uint64_t p, double* n0, double* n1) {
  double u1 = unif(mix64(key + 2 * p));
  double u2 = unif(mix64(key + 2 * p + 1));
  double r = sqrt(-2.0 * log(u1));
  double a = 6.283185307179586476925286766559 * u2;
  *n0 = r * cos(a);
  *n1 = r * sin(a);
}

static uint16_t f32_to_bf16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  if ((x & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((x >> 16) | 0x40u);
  uint32_t lsb = (x >> 16) & 1u;
  x += 0x7fffu + lsb;
  return (uint16_t)(x >> 16);
}

static uint16_t f32_to_f16(float f) {
  uint32_t x;
  memcpy(&x, &f, 4);
  uint32_t sign = (x >> 16) & 0x8000u;
  uint32_t ax = x & 0x7fffffffu;
  if (ax >= 0x7f800000u) return (uint16_t)(sign | 0x7c00u | (ax > 0x7f800000u ? 0x200u : 0u));
  if (ax >= 0x477ff000u) return (uint16_t)(sign | 0x7c00u);
  if (ax < 0x38800000u) {
    float af;
    memcpy(&af, &ax, 4);
    float m = rintf(af * 16777216.0f);
    return (uint16_t)(sign | (uint32_t)m);
  }
  uint32_t e = (ax >> 23) - 127u + 15u;
  uint32_t mant = ax & 0x7fffffu;
  uint32_t hv = (e << 10) | (mant >> 13);
  uint32_t rem = mant & 0x1fffu;
  if (rem > 0x1000u || (rem == 0x1000u && (hv & 1u))) hv++;
  return (uint16_t)(sign | hv);
}

static uint16_t to_dtype(double v, int dtype) {
  float f = (float)v;
  return dtype == KVGEN_FP16 ? f32_to_f16(f) : f32_to_bf16(f);
}

typedef struct {
  uint64_t seed;
  uint32_t L, H, T, D;
  int dtype;
  double rho, theta;
  uint32_t first_slice, n_slices;
  uint64_t noise_stream; /* 1 = data, 2 = calibration */
  void* out;             /* [n_slices][T][D] 16-bit values, or 32-bit for F32 */
  const double* cs;      /* [T][D/2][2] cos, sin (keys) */
  uint32_t next;         /* work counter */
  pthread_mutex_t mu;
} gen_job;

static void gen_slice(gen_job* J, uint32_t local) {
  uint32_t sidx = J->first_slice + local;
  uint32_t h = sidx % J->H;
  uint32_t kv = (sidx / J->H) % 2;
  uint32_t l = sidx / (2 * J->H);
  uint32_t D = J->D, T = J->T, half = D / 2;
  double* mu = (double*)malloc(sizeof(double) * D);
  double* sg = (double*)malloc(sizeof(double) * D);
  double* z = (double*)malloc(sizeof(double) * D);
  double* nz = (double*)malloc(sizeof(double) * D * 2);
  uint64_t* nkey = (uint64_t*)malloc(sizeof(uint64_t) * D);
  double* row = (double*)malloc(sizeof(double) * D);
  double a = J->rho, b = sqrt(1.0 - J->rho * J->rho);
  for (uint32_t d = 0; d < D; d++) {
    double n0, n1;
    normal_pair(channel_key(J->seed, 0, l, kv, h, d), 0, &n0, &n1);
    mu[d] = n0;
    sg[d] = exp(0.5 * n1);
    nkey[d] = channel_key(J->seed, J->noise_stream, l, kv, h, d);
  }
  uint16_t* out = J->dtype == KVGEN_F32 ? NULL : (uint16_t*)J->out + (size_t)local * T * D;
  uint32_t* out32 = J->dtype == KVGEN_F32 ? (uint32_t*)J->out + (size_t)local * T * D : NULL;
  for (uint32_t t = 0; t < T; t++) {
    for (uint32_t d = 0; d < D; d++) {
      double e;
      if ((t & 1u) == 0) {
        normal_pair(nkey[d], t >> 1, &nz[2 * d], &nz[2 * d + 1]);
        e = nz[2 * d];
      } else {
        e = nz[2 * d + 1];
      }
      z[d] = (t == 0) ? e : a * z[d] + b * e;
      row[d] = mu[d] + sg[d] * z[d];
    }
    if (kv == 0) {
      const double* c = J->cs + (size_t)t * half * 2;
      for (uint32_t i = 0; i < half; i++) {
        double x0 = row[i], x1 = row[i + half];
        double co = c[2 * i], si = c[2 * i + 1];
        row[i] = x0 * co - x1 * si;
        row[i + half] = x0 * si + x1 * co;
      }
    }
    if (out32) {
      for (uint32_t d = 0; d < D; d++) {
        float f = (float)row[d];
        memcpy(&out32[(size_t)t * D + d], &f, 4);
      }
    } else {
      for (uint32_t d = 0; d < D; d++) out[(size_t)t * D + d] = to_dtype(row[d], J->dtype);
    }
  }
  free(mu); free(sg); free(z); free(nz); free(nkey); free(row);
}

static void* gen_worker(void* arg) {
  gen_job* J = (gen_job*)arg;
  for (;;) {
    pthread_mutex_lock(&J->mu);
    uint32_t i = J->next++;
    pthread_mutex_unlock(&J->mu);
    if (i >= J->n_slices) break;
    gen_slice(J, i);
  }
  return NULL;
}

static int run_gen(gen_job* J, int n_threads) {
  uint32_t half = J->D / 2;
  double* cs = (double*)malloc(sizeof(double) * (size_t)J->T * half * 2);
  if (!cs) return -1;
  for (uint32_t t = 0; t < J->T; t++)
    for (uint32_t i = 0; i < half; i++) {
      double ang = (double)t * pow(J->theta, -2.0 * (double)i / (double)J->D);
      cs[((size_t)t * half + i) * 2] = cos(ang);
      cs[((size_t)t * half + i) * 2 + 1] = sin(ang);
    }
  J->cs = cs;
  J->next = 0;
  pthread_mutex_init(&J->mu, NULL);
  if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (n_threads < 1) n_threads = 1;
  if ((uint32_t)n_threads > J->n_slices) n_threads = (int)(J->n_slices ? J->n_slices : 1);
  pthread_t* th = (pthread_t*)malloc(sizeof(pthread_t) * n_threads);
  for (int i = 0; i < n_threads; i++) pthread_create(&th[i], NULL, gen_worker, J);
  for (int i = 0; i < n_threads; i++) pthread_join(th[i], NULL);
  free(th);
  pthread_mutex_destroy(&J->mu);
  free(cs);
  return 0;
}

/* Slices [first_slice, first_slice + n_slices) of the [L][2][H][T][D] cache. */
int kvgen_slices(uint64_t seed, uint32_t L, uint32_t H, uint32_t T, uint32_t D, int dtype,
                 double rho, double theta, uint32_t first_slice, uint32_t n_slices,
                 int n_threads, void* out) {
  if (D == 0 || (D & 1u) || first_slice + n_slices > L * 2 * H) return -1;
  gen_job J;
  memset(&J, 0, sizeof J);
  J.seed = seed; J.L = L; J.H = H; J.T = T; J.D = D; J.dtype = dtype;
  J.rho = rho; J.theta = theta; J.first_slice = first_slice; J.n_slices = n_slices;
  J.noise_stream = 1; J.out = out;
  return run_gen(&J, n_threads);
}

/* Calibration draw: same channel parameters, separate noise stream, n_calib
 * tokens at positions 0..n_calib-1, every slice. Output [L*2*H][n_calib][D]. */
int kvgen_calibration(uint64_t seed, uint32_t L, uint32_t H, uint32_t n_calib, uint32_t D,
                      int dtype, double rho, double theta, int n_threads, void* out) {
  if (D == 0 || (D & 1u)) return -1;
  gen_job J;
  memset(&J, 0, sizeof J);
  J.seed = seed; J.L = L; J.H = H; J.T = n_calib; J.D = D; J.dtype = dtype;
  J.rho = rho; J.theta = theta; J.first_slice = 0; J.n_slices = L * 2 * H;
  J.noise_stream = 2; J.out = out;
  return run_gen(&J, n_threads);
}

/* Uniform random bytes (control block), key (seed, 3). */
void kvgen_random_bytes(uint64_t seed, uint64_t n, uint8_t* out) {
  uint64_t key = chain(mix64(seed), 3);
  for (uint64_t i = 0; i < n; i += 8) {
    uint64_t r = mix64(key + (i >> 3));
    for (uint64_t j = 0; j < 8 && i + j < n; j++) out[i + j] = (uint8_t)(r >> (8 * j));
  }
}
