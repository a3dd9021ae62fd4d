/*
 * oracle.c -- fp64 CPU reference (test infrastructure only; see oracle.h for
 * the passages each function follows and the readings taken).
 *
 * Nothing here is blocked, fused or reordered beyond the definitions: each
 * output row is computed on its own with an explicit window test, a first pass
 * for the scores and their maximum, and a second pass for the weights and the
 * weighted sum of values. Threads only split independent (row, head) outputs.
 */
#include "oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdlib.h>
#include <string.h>

static double bf16_to_double(uint16_t b) {
  uint32_t u = ((uint32_t)b) << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return (double)f;
}

/* eq.(1): the first key position a query at position i may attend. */
static int64_t window_lo(int64_t i, int64_t window) {
  if (window <= 0) return 0; /* full causal attention */
  int64_t lo = i - window + 1;
  return lo > 0 ? lo : 0;
}

/* eq.(2): M_ij = 1 iff j in W(i). */
static int in_window(int64_t i, int64_t j, int64_t window) {
  return j <= i && j >= window_lo(i, window);
}

int64_t orc_mask_count(int64_t n, int64_t window) {
  int64_t c = 0;
  for (int64_t i = 0; i < n; ++i)
    for (int64_t j = 0; j < n; ++j) c += in_window(i, j, window);
  return c;
}

typedef struct {
  const uint16_t* q;
  const int64_t* q_pos;
  int64_t n_rows;
  int n_q_heads;
  const uint16_t* k;   /* bf16 keys and values, or ... */
  const uint16_t* v;
  const double* k64;   /* ... fp64 ones (dequantized FP8 cache entries) when these are set */
  const double* v64;
  int64_t key_base, n_keys;
  int n_kv_heads, head_dim;
  int64_t window;
  double* out;
  int64_t first, last; /* (row, head) work items [first, last) */
  int status;
} attn_job;

/* Element e of key/value row `row` (relative to key_base) of KV head g. */
static double kv_at(const uint16_t* b16, const double* f64, int64_t row, int n_kv_heads, int g, int d, int e) {
  const size_t idx = ((size_t)row * n_kv_heads + g) * d + e;
  return f64 ? f64[idx] : bf16_to_double(b16[idx]);
}

static void* attn_worker(void* arg) {
  attn_job* J = (attn_job*)arg;
  const int d = J->head_dim;
  const int group = J->n_q_heads / J->n_kv_heads;
  const double scale = 1.0 / sqrt((double)d); /* eq.(3): 1/sqrt(d_k) */
  double* qd = (double*)malloc(sizeof(double) * (size_t)d);
  double* s = NULL;
  int64_t s_cap = 0;
  for (int64_t w = J->first; w < J->last; ++w) {
    const int64_t r = w / J->n_q_heads;
    const int h = (int)(w % J->n_q_heads);
    const int g = h / group; /* GQA: query head h reads KV head floor(h / G) */
    const int64_t i = J->q_pos[r];
    const int64_t lo = window_lo(i, J->window);
    if (i < 0 || lo < J->key_base || i >= J->key_base + J->n_keys) {
      J->status = -1;
      break;
    }
    const int64_t cnt = i - lo + 1;
    if (cnt > s_cap) {
      free(s);
      s_cap = cnt;
      s = (double*)malloc(sizeof(double) * (size_t)s_cap);
    }
    const uint16_t* qrow = J->q + ((size_t)r * J->n_q_heads + h) * d;
    for (int e = 0; e < d; ++e) qd[e] = bf16_to_double(qrow[e]);
    /* pass 1: masked scaled scores over W(i) (eq.(3)); entries outside W(i)
       are -inf and contribute exp(-inf) = 0 to eq.(4), so they are not visited */
    double mx = -INFINITY;
    for (int64_t j = lo; j <= i; ++j) {
      if (!in_window(i, j, J->window)) continue;
      double dot = 0.0;
      for (int e = 0; e < d; ++e) dot += qd[e] * kv_at(J->k, J->k64, j - J->key_base, J->n_kv_heads, g, d, e);
      s[j - lo] = dot * scale;
      if (s[j - lo] > mx) mx = s[j - lo];
    }
    /* pass 2: eq.(4) softmax weights (shifted by the row maximum, which cancels
       between numerator and denominator) and eq.(5) the weighted sum of values */
    double* o = J->out + ((size_t)r * J->n_q_heads + h) * d;
    for (int e = 0; e < d; ++e) o[e] = 0.0;
    double denom = 0.0;
    for (int64_t j = lo; j <= i; ++j) {
      const double p = exp(s[j - lo] - mx);
      denom += p;
      for (int e = 0; e < d; ++e) o[e] += p * kv_at(J->v, J->v64, j - J->key_base, J->n_kv_heads, g, d, e);
    }
    for (int e = 0; e < d; ++e) o[e] /= denom;
  }
  free(qd);
  free(s);
  return NULL;
}

static int attention_any(const uint16_t* q, const int64_t* q_pos, int64_t n_rows, int n_q_heads,
                         const uint16_t* k, const uint16_t* v, const double* k64, const double* v64,
                         int64_t key_base, int64_t n_keys, int n_kv_heads, int head_dim, int64_t window,
                         double* out, int n_threads) {
  if (n_rows < 0 || n_q_heads <= 0 || n_kv_heads <= 0 || head_dim <= 0 || window < 0) return -1;
  if (n_q_heads % n_kv_heads != 0) return -1;
  if (n_rows == 0) return 0;
  const int64_t items = n_rows * (int64_t)n_q_heads;
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > items) n_threads = (int)items;
  attn_job jobs[256];
  pthread_t tids[256];
  for (int t = 0; t < n_threads; ++t) {
    attn_job* J = &jobs[t];
    J->q = q; J->q_pos = q_pos; J->n_rows = n_rows; J->n_q_heads = n_q_heads;
    J->k = k; J->v = v; J->k64 = k64; J->v64 = v64; J->key_base = key_base; J->n_keys = n_keys;
    J->n_kv_heads = n_kv_heads; J->head_dim = head_dim; J->window = window; J->out = out;
    J->first = items * t / n_threads;
    J->last = items * (t + 1) / n_threads;
    J->status = 0;
  }
  if (n_threads == 1) {
    attn_worker(&jobs[0]);
  } else {
    for (int t = 0; t < n_threads; ++t) pthread_create(&tids[t], NULL, attn_worker, &jobs[t]);
    for (int t = 0; t < n_threads; ++t) pthread_join(tids[t], NULL);
  }
  for (int t = 0; t < n_threads; ++t)
    if (jobs[t].status) return -1;
  return 0;
}

int orc_attention(const uint16_t* q, const int64_t* q_pos, int64_t n_rows, int n_q_heads,
                  const uint16_t* k, const uint16_t* v, int64_t key_base, int64_t n_keys,
                  int n_kv_heads, int head_dim, int64_t window, double* out, int n_threads) {
  return attention_any(q, q_pos, n_rows, n_q_heads, k, v, NULL, NULL, key_base, n_keys, n_kv_heads, head_dim,
                       window, out, n_threads);
}

int orc_attention_kv64(const uint16_t* q, const int64_t* q_pos, int64_t n_rows, int n_q_heads,
                       const double* k, const double* v, int64_t key_base, int64_t n_keys,
                       int n_kv_heads, int head_dim, int64_t window, double* out, int n_threads) {
  return attention_any(q, q_pos, n_rows, n_q_heads, NULL, NULL, k, v, key_base, n_keys, n_kv_heads, head_dim,
                       window, out, n_threads);
}

/* OCP 8-bit floating point, E4M3: sign bit, 4 exponent bits with bias 7, 3 mantissa bits; no
   infinities; S.1111.111 is NaN; exponent field 0 holds the subnormals 0.mmm * 2^-6. */
double orc_e4m3_decode(uint8_t code) {
  const int sign = code >> 7, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  const double mag = e == 0 ? ldexp((double)m / 8.0, -6) : ldexp(1.0 + (double)m / 8.0, e - 7);
  return sign ? -mag : mag;
}

/* Nearest E4M3 value, ties to the even mantissa; magnitudes of 448 and above give +-448 (the
   largest finite value) instead of NaN; NaN gives 0x7F. Zero keeps its sign. */
uint8_t orc_e4m3_encode(double x) {
  if (isnan(x)) return 0x7F;
  const uint8_t sign = signbit(x) ? 0x80 : 0x00;
  const double a = fabs(x);
  if (a >= 448.0) return sign | 0x7E;
  if (a == 0.0) return sign;
  int e2;
  frexp(a, &e2); /* a in [2^(e2-1), 2^e2) */
  int ee = e2 - 1;
  if (ee < -6) ee = -6; /* below 2^-6 the spacing stays 2^-9 (subnormals) */
  const double step = ldexp(1.0, ee - 3);
  const double n = a / step; /* exact: a scaled by a power of two */
  double k = floor(n);
  const double frac = n - k;
  if (frac > 0.5 || (frac == 0.5 && fmod(k, 2.0) != 0.0)) k += 1.0;
  int ki = (int)k; /* 0 .. 16 */
  if (ki == 0) return sign;
  if (ee == -6 && ki < 8) return sign | (uint8_t)ki; /* subnormal */
  if (ki == 16) {
    ee += 1;
    ki = 8;
  }
  return sign | (uint8_t)(((ee + 7) << 3) | (ki - 8));
}

int orc_e4m3_quantize(const uint16_t* x, int64_t n, float scale, uint8_t* out) {
  if (n < 0 || !(scale > 0.0f)) return -1;
  const float inv = 1.0f / scale; /* fp32 reciprocal, then an fp32 product per element */
  for (int64_t i = 0; i < n; ++i) {
    const float v = (float)bf16_to_double(x[i]) * inv;
    out[i] = orc_e4m3_encode((double)v);
  }
  return 0;
}

static int slot_valid(const uint32_t* valid_row, int64_t slot) {
  return (valid_row[slot / 32] >> (slot % 32)) & 1u;
}

int orc_window_safe_len(const int64_t* m, const int64_t* cached, const uint32_t* valid,
                        int32_t window, int64_t n_req, int64_t* out) {
  if (window < 1 || n_req < 0) return -1;
  const int64_t W = window;
  const int64_t words = (W + 31) / 32;
  for (int64_t r = 0; r < n_req; ++r) {
    const int64_t M = m[r], C = cached[r];
    if (M < 0 || C < 0) return -1;
    const uint32_t* vr = valid + r * words;
    const int64_t ring_lo = C - W > 0 ? C - W : 0; /* the ring holds [max(0,C-W), C-1] */
    int64_t best = 0;                                /* safe(0) always holds */
    for (int64_t L = M; L >= 1; --L) {
      const int64_t tail_lo = L - W > 0 ? L - W : 0;
      int ok = 1;
      for (int64_t p = tail_lo; p <= L - 1 && ok; ++p) {
        const int resident = p >= ring_lo && p < C && slot_valid(vr, p % W);
        if (!resident) ok = 0;
      }
      if (ok) {
        best = L;
        break;
      }
    }
    out[r] = best;
  }
  return 0;
}

int orc_ring_trace(int64_t n_appended, int64_t w, int64_t* slot_pos) {
  if (w < 1 || n_appended < 0) return -1;
  for (int64_t s = 0; s < w; ++s) slot_pos[s] = -1;
  for (int64_t t = 0; t < n_appended; ++t) slot_pos[t % w] = t; /* eq.(7) */
  return 0;
}

int64_t orc_kv_bytes(int64_t layers, int64_t kv_heads, int64_t tokens, int64_t head_dim,
                     int64_t elem_bytes) {
  return 2 * layers * kv_heads * tokens * head_dim * elem_bytes;
}

double orc_hybrid_kv_ratio(int64_t n_swa, int64_t n_full, int64_t window, int64_t n_tokens) {
  const double num = (double)n_swa * (double)window + (double)n_full * (double)n_tokens;
  const double den = (double)(n_swa + n_full) * (double)n_tokens;
  return num / den;
}
