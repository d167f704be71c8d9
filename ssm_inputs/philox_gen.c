/*
 * philox_gen.c -- seeded, counter-based synthetic input generator.
 *
 * Shared by the tests, the benchmark and the smoke check to build the same
 * input bytes for the CUDA path and the CPU oracle. It holds none of the
 * selective-scan arithmetic: only random numbers and their rounding to the
 * storage type.
 *
 * Generator: Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel Random
 * Numbers: As Easy as 1, 2, 3", SC'11), key = (seed lo, seed hi) and
 * counter = (index lo, index hi, stream id, 0) for element `index` of the
 * tensor with stream id `stream`. Each counter block gives one value:
 *   u1 = 1 - U53(w0, w1)   in (0, 1]
 *   u2 =     U53(w2, w3)   in [0, 1)
 *   normal  = mean + sigma * sqrt(-2 ln u1) * cos(2 pi u2)      (Box-Muller)
 *   uniform = lo + (hi - lo) * u2
 * where U53(a, b) = ((a >> 5) * 2^26 + (b >> 6)) * 2^-53.
 * Values are rounded to binary32 (round to nearest even) and, for bf16, on
 * from binary32 to bf16 (round to nearest even on the upper 16 bits).
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <string.h>

#define PHILOX_M0 0xD2511F53u
#define PHILOX_M1 0xCD9E8D57u
#define PHILOX_W0 0x9E3779B9u
#define PHILOX_W1 0xBB67AE85u

void philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)PHILOX_M0 * c0;
    const uint64_t p1 = (uint64_t)PHILOX_M1 * c2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    c0 = hi1 ^ c1 ^ k0;
    c1 = lo1;
    c2 = hi0 ^ c3 ^ k1;
    c3 = lo0;
    k0 += PHILOX_W0;
    k1 += PHILOX_W1;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

static double u53(uint32_t a, uint32_t b) {
  return ((double)(a >> 5) * 67108864.0 + (double)(b >> 6)) * (1.0 / 9007199254740992.0);
}

static uint16_t f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  u += 0x7FFFu + ((u >> 16) & 1u);
  return (uint16_t)(u >> 16);
}

enum { KIND_NORMAL = 0, KIND_UNIFORM = 1 };
enum { OUT_F64 = 0, OUT_F32 = 1, OUT_BF16 = 2 };

typedef struct {
  uint64_t seed, stream, offset;
  int64_t lo_i, hi_i;
  int kind, out_type;
  double a, b; /* normal: mean, sigma; uniform: lo, hi */
  void* out;
} gen_job;

static void* gen_worker(void* arg) {
  const gen_job* j = (const gen_job*)arg;
  const uint32_t key[2] = {(uint32_t)j->seed, (uint32_t)(j->seed >> 32)};
  for (int64_t i = j->lo_i; i < j->hi_i; ++i) {
    const uint64_t idx = j->offset + (uint64_t)i;
    const uint32_t ctr[4] = {(uint32_t)idx, (uint32_t)(idx >> 32), (uint32_t)j->stream, 0u};
    uint32_t w[4];
    philox4x32_10(ctr, key, w);
    double v;
    if (j->kind == KIND_NORMAL) {
      const double u1 = 1.0 - u53(w[0], w[1]);
      const double u2 = u53(w[2], w[3]);
      v = j->a + j->b * sqrt(-2.0 * log(u1)) * cos(6.283185307179586 * u2);
    } else {
      v = j->a + (j->b - j->a) * u53(w[2], w[3]);
    }
    if (j->out_type == OUT_F64) {
      ((double*)j->out)[i] = v;
    } else if (j->out_type == OUT_F32) {
      ((float*)j->out)[i] = (float)v;
    } else {
      ((uint16_t*)j->out)[i] = f32_to_bf16_rne((float)v);
    }
  }
  return NULL;
}

/* Fill out[0..count) with values for elements offset..offset+count of
 * stream `stream`. Returns 0. */
int ssm_gen_fill(uint64_t seed, uint64_t stream, uint64_t offset, int64_t count, int kind,
                 double a, double b, int out_type, void* out, int nthreads) {
  if (count <= 0) return 0;
  if (nthreads < 1) nthreads = 1;
  if (nthreads > 256) nthreads = 256;
  if (count < 65536) nthreads = 1;
  gen_job jobs[256];
  pthread_t tid[256];
  int ok[256];
  for (int w = 0; w < nthreads; ++w) {
    jobs[w].seed = seed; jobs[w].stream = stream; jobs[w].offset = offset;
    jobs[w].lo_i = count * w / nthreads; jobs[w].hi_i = count * (w + 1) / nthreads;
    jobs[w].kind = kind; jobs[w].out_type = out_type; jobs[w].a = a; jobs[w].b = b;
    jobs[w].out = out;
    ok[w] = nthreads > 1 && pthread_create(&tid[w], NULL, gen_worker, &jobs[w]) == 0;
    if (!ok[w]) gen_worker(&jobs[w]);
  }
  for (int w = 0; w < nthreads; ++w)
    if (ok[w]) pthread_join(tid[w], NULL);
  return 0;
}
