/*
 * Host side of the seeded input generator (see gen_core.h for the
 * definitions).  Fills contiguous counter ranges of a stream, split over
 * POSIX threads.  Test and benchmark plumbing only.
 */
#include <pthread.h>
#include <stddef.h>
#include <stdint.h>

#include "gen_core.h"

typedef struct {
  int kind;
  uint64_t state;
  uint64_t start;
  uint64_t begin, end; /* offsets into the output */
  double a, b;
  int as_bf16;
  void* out;
} gen_job;

static void* gen_worker(void* arg) {
  gen_job* j = (gen_job*)arg;
  if (j->as_bf16) {
    uint16_t* o = (uint16_t*)j->out;
    for (uint64_t i = j->begin; i < j->end; ++i)
      o[i] = gen_f32_to_bf16(gen_value_f32(j->kind, j->state, j->start + i, j->a, j->b));
  } else {
    float* o = (float*)j->out;
    for (uint64_t i = j->begin; i < j->end; ++i)
      o[i] = gen_value_f32(j->kind, j->state, j->start + i, j->a, j->b);
  }
  return NULL;
}

/* Fill out[0..count) with elements start..start+count-1 of stream `stream`.
   kind: 0 normal (a = mean, b = std), 1 uniform on [a, b).
   as_bf16: 1 -> out is uint16_t bf16 bits (RNE from the float32 value), 0 -> float32.
   Returns 0, or -1 on a bad argument. */
int gen_fill(uint64_t seed, uint64_t stream, uint64_t start, uint64_t count, int kind, double a,
             double b, int as_bf16, void* out, int threads) {
  if ((count && !out) || (kind != GEN_NORMAL && kind != GEN_UNIFORM)) return -1;
  if (threads < 1) threads = 1;
  if (threads > 256) threads = 256;
  if ((uint64_t)threads > count / 65536 + 1) threads = (int)(count / 65536 + 1);
  uint64_t state = gen_stream_state(seed, stream);
  gen_job jobs[256];
  pthread_t tids[256];
  int created[256];
  uint64_t per = (count + (uint64_t)threads - 1) / (uint64_t)threads;
  for (int t = 0; t < threads; ++t) {
    gen_job* j = &jobs[t];
    j->kind = kind;
    j->state = state;
    j->start = start;
    j->begin = per * (uint64_t)t;
    j->end = j->begin + per < count ? j->begin + per : count;
    j->a = a;
    j->b = b;
    j->as_bf16 = as_bf16;
    j->out = out;
    created[t] = 0;
    if (j->begin >= j->end) continue;
    if (t < threads - 1 && pthread_create(&tids[t], NULL, gen_worker, j) == 0)
      created[t] = 1;
    else
      gen_worker(j);
  }
  for (int t = 0; t < threads; ++t)
    if (created[t]) pthread_join(tids[t], NULL);
  return 0;
}

/* Raw 64-bit draw number `ctr` of stream `stream` (for integer samples such as lengths and row picks). */
uint64_t gen_draw_u64(uint64_t seed, uint64_t stream, uint64_t ctr) {
  return gen_draw(gen_stream_state(seed, stream), ctr);
}

/* One float32 value, for spot checks. */
float gen_value_one(uint64_t seed, uint64_t stream, uint64_t idx, int kind, double a, double b) {
  return gen_value_f32(kind, gen_stream_state(seed, stream), idx, a, b);
}
