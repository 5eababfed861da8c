/*
 * Host build of the seeded synthetic-input generator (see gen_core.h).
 * Fills contiguous [B, L, Hx, d] tensors for one denoising step; this is the
 * only source of the inputs the CPU oracle reads.
 */
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include "gen_core.h"

void synth_philox(const uint32_t ctr[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
  syn_u32x4 c;
  memcpy(c.v, ctr, sizeof(c.v));
  syn_u32x4 r = syn_philox4x32_10(c, k0, k1);
  memcpy(out, r.v, sizeof(r.v));
}

/* One fp64 normal deviate, exposed for distribution tests. */
double synth_normal(uint64_t elem, uint32_t step, uint32_t tensor, uint64_t seed, double unit) {
  return syn_normal(elem, step, tensor, (uint32_t)seed, (uint32_t)(seed >> 32), unit);
}

typedef struct {
  void* out;
  int dtype; /* 0 = bf16 bits, 1 = fp32 */
  int B, L, Hx, d, bs;
  uint32_t step, tensor;
  uint64_t seed;
  double unit, noise;
  const double* sharp;   /* [Hx] or NULL (1.0) */
  const double* dir;     /* [B, Hx, d] or NULL */
  const uint8_t* plant;  /* [B, Hx, L/bs] or NULL */
  double amp;
  int64_t row0, row1; /* rows of B*L */
} fill_job;

static void* fill_worker(void* arg) {
  fill_job* j = (fill_job*)arg;
  uint32_t k0 = (uint32_t)j->seed, k1 = (uint32_t)(j->seed >> 32);
  int nb = j->L / j->bs;
  for (int64_t row = j->row0; row < j->row1; ++row) {
    int b = (int)(row / j->L);
    int t = (int)(row % j->L);
    for (int h = 0; h < j->Hx; ++h) {
      double sharp = j->sharp ? j->sharp[h] : 1.0;
      int planted = 0;
      if (j->plant && j->dir) planted = j->plant[((int64_t)b * j->Hx + h) * nb + t / j->bs] != 0;
      for (int c = 0; c < j->d; ++c) {
        uint64_t elem = (((uint64_t)row * j->Hx + h) * j->d) + c;
        double shift = planted ? j->amp * j->dir[((int64_t)b * j->Hx + h) * j->d + c] : 0.0;
        double x = syn_value(elem, j->step, j->tensor, k0, k1, j->unit, j->noise, sharp, shift);
        float f = (float)x;
        if (j->dtype == 1)
          ((float*)j->out)[elem] = f;
        else
          ((uint16_t*)j->out)[elem] = syn_f32_to_bf16(f);
      }
    }
  }
  return NULL;
}

/* Fill one step tensor.  Returns 0 on success, -1 on bad arguments. */
int synth_fill(void* out, int dtype, int B, int L, int Hx, int d, int bs, uint32_t step,
               uint32_t tensor, uint64_t seed, double unit, double noise, const double* sharp,
               const double* dir, const uint8_t* plant, double amp, int nthreads) {
  if (!out || B <= 0 || L <= 0 || Hx <= 0 || d <= 0 || bs <= 0 || L % bs) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  int64_t rows = (int64_t)B * L;
  pthread_t th[256];
  fill_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    fill_job j = {out, dtype, B, L, Hx, d, bs, step, tensor, seed, unit, noise,
                  sharp, dir, plant, amp, rows * i / nthreads, rows * (i + 1) / nthreads};
    jobs[i] = j;
    pthread_create(&th[i], NULL, fill_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  return 0;
}

typedef struct {
  int64_t* sums;
  int B, L, H, d;
  uint64_t seed;
  int h0, h1;
} qsum_job;

static void* qsum_worker(void* arg) {
  qsum_job* j = (qsum_job*)arg;
  uint32_t k0 = (uint32_t)j->seed, k1 = (uint32_t)(j->seed >> 32);
  for (int b = 0; b < j->B; ++b)
    for (int h = j->h0; h < j->h1; ++h)
      for (int c = 0; c < j->d; ++c) {
        int64_t s = 0;
        for (int t = 0; t < j->L; ++t) {
          uint64_t elem = ((((uint64_t)b * j->L + t) * j->H + h) * j->d) + c;
          s += syn_ih_int(elem, SYN_STEP_BASE, SYN_T_Q, k0, k1);
        }
        j->sums[((int64_t)b * j->H + h) * j->d + c] = s;
      }
  return NULL;
}

/* Exact integer sums over tokens of the base query draws: sums[B, H, d].
 * The planted-key direction of each KV head is derived from these. */
int synth_qsum(int64_t* sums, int B, int L, int H, int d, uint64_t seed, int nthreads) {
  if (!sums || B <= 0 || L <= 0 || H <= 0 || d <= 0) return -1;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > H) nthreads = H;
  if (nthreads > 256) nthreads = 256;
  pthread_t th[256];
  qsum_job jobs[256];
  for (int i = 0; i < nthreads; ++i) {
    qsum_job j = {sums, B, L, H, d, seed, H * i / nthreads, H * (i + 1) / nthreads};
    jobs[i] = j;
    pthread_create(&th[i], NULL, qsum_worker, &jobs[i]);
  }
  for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
  return 0;
}
