/*
 * Host implementation of the seeded input generator (formulas in gen_core.h).
 * Threads split a contiguous index range; every element depends only on its
 * index, so the result is independent of the thread count.
 */
#include <math.h>
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>

#include "gen_core.h"

uint64_t gen_stream_key(uint64_t seed, uint64_t stream) { return gen_key_of(seed, stream); }

float gen_normal_scale(double sigma) { return (float)(sigma / (65536.0 * sqrt(8.0 / 3.0))); }

typedef struct {
  uint64_t key, first;
  size_t lo, hi;
  float scale;
  void* out;
  int kind; /* 0 normal bf16, 1 normal f32, 2 uniform f32 */
} gen_job;

static void* gen_worker(void* p) {
  gen_job* j = (gen_job*)p;
  for (size_t i = j->lo; i < j->hi; ++i) {
    uint64_t idx = j->first + (uint64_t)i;
    if (j->kind == 0)
      ((uint16_t*)j->out)[i] = gen_f32_to_bf16(gen_normal_f32(j->key, idx, j->scale));
    else if (j->kind == 1)
      ((float*)j->out)[i] = gen_normal_f32(j->key, idx, j->scale);
    else
      ((float*)j->out)[i] = gen_uniform01(j->key, idx);
  }
  return NULL;
}

static void gen_run(uint64_t key, uint64_t first, size_t count, float scale, void* out, int kind,
                    int nthreads) {
  enum { MAXT = 256 };
  if (nthreads < 1) nthreads = 1;
  if (nthreads > MAXT) nthreads = MAXT;
  if ((size_t)nthreads > count / 65536 + 1) nthreads = (int)(count / 65536 + 1);
  gen_job jobs[MAXT];
  pthread_t tid[MAXT];
  int spawned[MAXT];
  size_t per = (count + (size_t)nthreads - 1) / (size_t)nthreads;
  for (int t = 0; t < nthreads; ++t) {
    size_t lo = (size_t)t * per, hi = lo + per;
    if (lo > count) lo = count;
    if (hi > count) hi = count;
    jobs[t] = (gen_job){key, first, lo, hi, scale, out, kind};
    spawned[t] = 0;
    /* the last slice, or one whose thread could not be started, runs here */
    if (t < nthreads - 1 && pthread_create(&tid[t], NULL, gen_worker, &jobs[t]) == 0)
      spawned[t] = 1;
    else
      gen_worker(&jobs[t]);
  }
  for (int t = 0; t < nthreads; ++t)
    if (spawned[t]) pthread_join(tid[t], NULL);
}

void gen_normal_bf16_host(uint64_t key, uint64_t first, size_t count, float scale, uint16_t* out,
                          int nthreads) {
  gen_run(key, first, count, scale, out, 0, nthreads);
}

void gen_normal_f32_host(uint64_t key, uint64_t first, size_t count, float scale, float* out,
                         int nthreads) {
  gen_run(key, first, count, scale, out, 1, nthreads);
}

void gen_uniform_f32_host(uint64_t key, uint64_t first, size_t count, float* out, int nthreads) {
  gen_run(key, first, count, 0.0f, out, 2, nthreads);
}

uint64_t gen_draw_u64(uint64_t key, uint64_t i) { return gen_draw(key, i); }
