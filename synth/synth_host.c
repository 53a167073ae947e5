/*
 * synth_host.c - CPU implementation of the seeded input generator.
 * The recipe is stated in synth.h; synth_device.cu implements the same
 * recipe on the GPU and must produce identical bits.
 */
#include "synth.h"

#include <pthread.h>
#include <string.h>
#include <unistd.h>

/* Philox4x32-10 (Salmon et al., SC'11): multipliers, Weyl key increments. */
#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

static inline void philox_block(uint32_t c[4], uint32_t k0, uint32_t k1) {
  for (int round = 0; round < 10; ++round) {
    const uint64_t p0 = (uint64_t)PHILOX_M0 * c[0];
    const uint64_t p1 = (uint64_t)PHILOX_M1 * c[2];
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c[1] ^ k0;
    const uint32_t n2 = hi0 ^ c[3] ^ k1;
    c[0] = n0; c[1] = lo1; c[2] = n2; c[3] = lo0;
    k0 += PHILOX_W0; k1 += PHILOX_W1;
  }
}

void synth_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]) {
  uint32_t c[4] = {ctr[0], ctr[1], ctr[2], ctr[3]};
  philox_block(c, key[0], key[1]);
  memcpy(out, c, sizeof(c));
}

static inline void draw(uint64_t seed, uint32_t tid, uint64_t i, uint32_t r[4]) {
  r[0] = (uint32_t)i; r[1] = (uint32_t)(i >> 32); r[2] = tid; r[3] = SYNTH_CTR_TAG;
  philox_block(r, (uint32_t)seed, (uint32_t)(seed >> 32));
}

/* Irwin-Hall (n = 4) value, exact up to the final double multiply. */
static inline double centred_value(uint64_t seed, uint32_t tid, uint64_t i, double scale) {
  uint32_t r[4];
  draw(seed, tid, i, r);
  const int64_t s = (int64_t)r[0] + (int64_t)r[1] + (int64_t)r[2] + (int64_t)r[3];
  const int64_t c = s - 2 * (int64_t)0xFFFFFFFFu;
  return (double)c * scale;
}

static inline double value_scale(double std) { return std * 0x1.bb67ae8584caap+0 * 0x1p-32; }

/* Round a double straight to bf16 (nearest, ties to even).  Values are
   inside the float normal range by construction of the recipe. */
static inline uint16_t bf16_from_double(double x) {
  uint64_t b;
  memcpy(&b, &x, sizeof(b));
  const uint32_t sign = (uint32_t)(b >> 63);
  const uint64_t mag = b & 0x7FFFFFFFFFFFFFFFull;
  if (mag == 0) return (uint16_t)(sign << 15);
  const int e = (int)(mag >> 52) - 1023;
  if (e < -126) return (uint16_t)(sign << 15);
  const uint64_t mant = mag & ((1ull << 52) - 1);
  uint32_t v = ((uint32_t)(e + 127) << 7) | (uint32_t)(mant >> 45);
  const uint64_t rem = mant & ((1ull << 45) - 1), half = 1ull << 44;
  if (rem > half || (rem == half && (v & 1u))) v += 1u;
  return (uint16_t)((sign << 15) | v);
}

typedef struct {
  int kind; /* 0 bf16, 1 f32 */
  void* dst;
  int64_t row0, rows, cols, stride_r, stride_c;
  uint64_t seed;
  uint32_t tid;
  double scale;
  int64_t begin, end; /* flat element range */
} job_t;

static void* run_job(void* arg) {
  const job_t* j = (const job_t*)arg;
  for (int64_t i = j->begin; i < j->end; ++i) {
    if (j->kind == 0) {
      const int64_t r = i / j->cols, c = i % j->cols;
      const double x = centred_value(j->seed, j->tid, (uint64_t)(i + j->row0 * j->cols), j->scale);
      ((uint16_t*)j->dst)[r * j->stride_r + c * j->stride_c] = bf16_from_double(x);
    } else {
      ((float*)j->dst)[i] = (float)centred_value(j->seed, j->tid, (uint64_t)i, j->scale);
    }
  }
  return NULL;
}

static int run_parallel(job_t proto, int64_t n, int n_threads) {
  if (n <= 0) return 0;
  if (n_threads <= 0) n_threads = (int)sysconf(_SC_NPROCESSORS_ONLN);
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > n / 4096 + 1) n_threads = (int)(n / 4096 + 1);
  pthread_t th[256];
  int created[256];
  job_t jobs[256];
  for (int t = 0; t < n_threads; ++t) {
    jobs[t] = proto;
    jobs[t].begin = n * t / n_threads;
    jobs[t].end = n * (t + 1) / n_threads;
    created[t] = 0;
    if (t < n_threads - 1 && pthread_create(&th[t], NULL, run_job, &jobs[t]) == 0) {
      created[t] = 1;
    } else {
      run_job(&jobs[t]); /* the last chunk (or a failed spawn) runs on this thread */
    }
  }
  for (int t = 0; t < n_threads; ++t)
    if (created[t]) pthread_join(th[t], NULL);
  return 0;
}

int synth_fill_bf16_host(uint16_t* dst, int64_t row0, int64_t rows, int64_t cols,
                         int64_t stride_r, int64_t stride_c, uint64_t seed, uint32_t tid,
                         double std, int n_threads) {
  if (!dst || row0 < 0 || rows < 0 || cols <= 0) return 1;
  job_t p = {0, dst, row0, rows, cols, stride_r, stride_c, seed, tid, value_scale(std), 0, 0};
  return run_parallel(p, rows * cols, n_threads);
}

int synth_fill_f32_host(float* dst, int64_t n, uint64_t seed, uint32_t tid, double std,
                        int n_threads) {
  if (!dst || n < 0) return 1;
  job_t p = {1, dst, 0, n, 1, 1, 0, seed, tid, value_scale(std), 0, 0};
  return run_parallel(p, n, n_threads);
}

int synth_fill_tokens_host(int32_t* dst, int64_t n, uint64_t seed, uint32_t tid, int32_t V) {
  if (!dst || n < 0 || V <= 0) return 1;
  for (int64_t i = 0; i < n; ++i) {
    uint32_t r[4];
    draw(seed, tid, (uint64_t)i, r);
    dst[i] = (int32_t)(((uint64_t)r[0] * (uint64_t)(uint32_t)V) >> 32);
  }
  return 0;
}
