/* fastgen.c -- CPU implementation of the seeded bf16 generator in synth/__init__.py
 * (same SplitMix64 counter hash, same inverse-CDF table lookup), multithreaded.
 * Input-generation code only: it holds none of the attention arithmetic. */
#include <pthread.h>
#include <stdint.h>

#define GAMMA 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

typedef struct {
  uint64_t key;
  int64_t start, count;
  const int64_t* thr;
  int64_t n_thr;
  const int16_t* val;
  int16_t* out;
} job_t;

static void* run(void* arg) {
  job_t* J = (job_t*)arg;
  for (int64_t i = 0; i < J->count; ++i) {
    const uint64_t z = mix64(J->key + GAMMA + (uint64_t)(J->start + i) * GAMMA);
    const int64_t u = (int64_t)(z >> 32);
    /* number of thresholds <= u */
    int64_t lo = 0, hi = J->n_thr;
    while (lo < hi) {
      const int64_t mid = (lo + hi) >> 1;
      if (J->thr[mid] <= u) lo = mid + 1; else hi = mid;
    }
    J->out[i] = J->val[lo];
  }
  return 0;
}

int fastgen_normal_bf16(uint64_t key, int64_t start, int64_t count, const int64_t* thr, int64_t n_thr,
                        const int16_t* val, int16_t* out, int n_threads) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 64) n_threads = 64;
  if (count < 65536) n_threads = 1;
  job_t jobs[64];
  pthread_t tid[64];
  for (int t = 0; t < n_threads; ++t) {
    const int64_t a = count * t / n_threads, b = count * (t + 1) / n_threads;
    jobs[t] = (job_t){key, start + a, b - a, thr, n_thr, val, out + a};
  }
  if (n_threads == 1) {
    run(&jobs[0]);
    return 0;
  }
  for (int t = 0; t < n_threads; ++t) pthread_create(&tid[t], 0, run, &jobs[t]);
  for (int t = 0; t < n_threads; ++t) pthread_join(tid[t], 0);
  return 0;
}
