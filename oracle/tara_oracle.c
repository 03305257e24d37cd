/*
 * tara_oracle.c -- plain fp64 CPU oracle of the TARA-biased joint attention forward pass.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the benchmark's CPU-baseline leg
 * may build, load or call this file.  It shares no source with the CUDA path.
 *
 * What it computes, for each requested query row (b, h, i), in double precision on the inputs
 * widened exactly from their stored type:
 *
 *   s_j = (sum_k Q[b,h,i,k] * K[b,h,j,k]) * scale                   for every key j
 *     scale = 1/sqrt(head_dim) unless given ("TARA: Native Temporal Alignment for MiniMax H3
 *     References", "The temporal rule", the score line)
 *   if token i is TARGET and token j is GUIDE   (same section: only output-video queries to
 *                                                the selected motion video's keys change)
 *     dt  = |t_i - t_j|
 *     s_j = s_j - min(strength * (max(dt - window, 0) / falloff)^2, cap)
 *   if token i is TARGET and token j is PICTURE p ("BFS H3 Reference Attention Binding
 *                                                (Experimental)", "The exact rule")
 *     s_j = s_j + m_i * ln(gain_p)
 *           + sum over extra bindings k of m_k,i * ln(gain_k,p)   ("Common issues":
 *                                                chained bindings combine their log gains)
 *   M = max_j s_j,  l = sum_j exp(s_j - M),  LSE_i = M + ln l,
 *   O_i = sum_j exp(s_j - M) * V[b,h,j,:] / l
 *
 * The dense logit row is formed explicitly, one row at a time; no blocking, no fusion.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#ifdef _OPENMP
#include <omp.h>
#endif

enum { ROLE_TEXT = 0, ROLE_PICTURE = 1, ROLE_TARGET = 2, ROLE_GUIDE = 3 };
enum { IN_BF16 = 0, IN_FP16 = 1, IN_FP32 = 2, IN_FP64 = 3 };

/* Exact widening of one stored element to double. */
static double widen(const void* base, int dtype, int64_t idx) {
  if (dtype == IN_FP64) return ((const double*)base)[idx];
  if (dtype == IN_FP32) return (double)((const float*)base)[idx];
  uint16_t h = ((const uint16_t*)base)[idx];
  if (dtype == IN_BF16) {
    /* bf16 is the top half of an IEEE binary32 */
    uint32_t w = (uint32_t)h << 16;
    float f;
    memcpy(&f, &w, 4);
    return (double)f;
  }
  /* IEEE binary16: 1 sign, 5 exponent (bias 15), 10 fraction bits */
  int sign = (h >> 15) & 1, e = (h >> 10) & 31, frac = h & 1023;
  double v;
  if (e == 0) v = ldexp((double)frac, -24);
  else if (e == 31) v = frac ? NAN : INFINITY;
  else v = ldexp((double)(1024 + frac), e - 25);
  return sign ? -v : v;
}

/* The temporal penalty of one (target query, guide key) edge, as written on the page. */
double oracle_penalty(double dt, double window, double falloff, double strength, double cap) {
  double x = dt - window;
  if (x < 0.0) x = 0.0;
  x = x / falloff;
  double p = strength * x * x;
  return p < cap ? p : cap;
}

/* Extra reference bindings beyond the first ("BFS H3 Reference Attention Binding
 * (Experimental)", "Common issues": two subjects are two chained binding nodes, and
 * overlapping masks combine their log gains).  Binding k has its own 9 gains and its own mask
 * weight per token (m_extra + k * m_len, offset to the branch like m). */
typedef struct {
  int n;                  /* extra bindings, 0..3 */
  const double* gains;    /* n x 9 */
  const float* m;         /* n arrays of m_len floats */
  int64_t m_len;
} oracle_bindings;

/* Bias of the edge (query token i, key token j); meta arrays already offset to the branch. */
double oracle_bias(int64_t i, int64_t j, const uint8_t* seg, const float* time_s,
                   const uint8_t* pic, const float* m, double window, double falloff,
                   double strength, double cap, const double* gain9,
                   const oracle_bindings* extra, int64_t mo) {
  if (seg[i] != ROLE_TARGET) return 0.0;
  if (seg[j] == ROLE_GUIDE) {
    double dt = fabs((double)time_s[i] - (double)time_s[j]);
    return -oracle_penalty(dt, window, falloff, strength, cap);
  }
  if (seg[j] == ROLE_PICTURE) {
    int p = pic[j];
    if (p < 1 || p > 9) return 0.0;
    double b = (double)m[i] * log(gain9[p - 1]);
    for (int k = 0; extra && k < extra->n; ++k)
      b += (double)extra->m[k * extra->m_len + mo + i] * log(extra->gains[9 * k + p - 1]);
    return b;
  }
  return 0.0;
}

/*
 * rows:   n_rows triples (b, h, i), int64.
 * O_out:  n_rows x D doubles.  LSE_out: n_rows doubles.
 * meta_batch_stride: 0 = one metadata set for all branches, else the offset of branch b.
 * Returns 0, or -1 on a bad argument / allocation failure.
 */
int oracle_attention_rows(const void* Q, const void* K, const void* V, int dtype,
                          int64_t B, int64_t H, int64_t N, int64_t D,
                          const uint8_t* seg, const float* time_s, const uint8_t* pic,
                          const float* m, int64_t meta_batch_stride,
                          double window, double falloff, double strength, double cap,
                          const double* gain9, double scale,
                          const int64_t* rows, int64_t n_rows,
                          double* O_out, double* LSE_out, int n_threads,
                          int n_extra, const double* extra_gains, const float* extra_m,
                          int64_t m_len) {
  if (!Q || !K || !V || !seg || !time_s || !pic || !m || !gain9 || !rows || !O_out || !LSE_out)
    return -1;
  if (B < 1 || H < 1 || N < 1 || D < 1 || n_rows < 0) return -1;
  if (n_extra < 0 || n_extra > 3 || (n_extra > 0 && (!extra_gains || !extra_m))) return -1;
  if (scale == 0.0) scale = 1.0 / sqrt((double)D);
  const oracle_bindings extra = {n_extra, extra_gains, extra_m, m_len};
  int failed = 0;
#ifdef _OPENMP
  if (n_threads > 0) omp_set_num_threads(n_threads);
#pragma omp parallel
#endif
  {
    double* s = (double*)malloc(sizeof(double) * (size_t)N);
    double* q = (double*)malloc(sizeof(double) * (size_t)D);
    double* o = (double*)malloc(sizeof(double) * (size_t)D);
    if (!s || !q || !o) {
#ifdef _OPENMP
#pragma omp atomic write
#endif
      failed = 1;
    } else {
#ifdef _OPENMP
#pragma omp for schedule(dynamic, 1)
#endif
      for (int64_t r = 0; r < n_rows; ++r) {
        int64_t b = rows[3 * r], h = rows[3 * r + 1], i = rows[3 * r + 2];
        if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= N) {
          LSE_out[r] = NAN;
          for (int64_t k = 0; k < D; ++k) O_out[r * D + k] = NAN;
          continue;
        }
        int64_t head = (b * H + h) * N * D;
        const int64_t mo = meta_batch_stride * b;
        for (int64_t k = 0; k < D; ++k) q[k] = widen(Q, dtype, head + i * D + k);
        /* dense logit row */
        double M = -INFINITY;
        for (int64_t j = 0; j < N; ++j) {
          double dot = 0.0;
          for (int64_t k = 0; k < D; ++k) dot += q[k] * widen(K, dtype, head + j * D + k);
          double sj = dot * scale + oracle_bias(i, j, seg + mo, time_s + mo, pic + mo, m + mo,
                                                window, falloff, strength, cap, gain9, &extra, mo);
          s[j] = sj;
          if (sj > M) M = sj;
        }
        /* softmax and weighted sum of V */
        double l = 0.0;
        for (int64_t k = 0; k < D; ++k) o[k] = 0.0;
        for (int64_t j = 0; j < N; ++j) {
          double w = exp(s[j] - M);
          l += w;
          for (int64_t k = 0; k < D; ++k) o[k] += w * widen(V, dtype, head + j * D + k);
        }
        for (int64_t k = 0; k < D; ++k) O_out[r * D + k] = o[k] / l;
        LSE_out[r] = M + log(l);
      }
    }
    free(s);
    free(q);
    free(o);
  }
  return failed ? -1 : 0;
}

/* The dense logit row s_j (j = 0..N-1) of query (b, h, i), exactly as oracle_attention_rows
 * forms it.  out: N doubles.  Returns 0, or -1 on a bad argument. */
int oracle_logit_row(const void* Q, const void* K, int dtype, int64_t B, int64_t H, int64_t N,
                     int64_t D, const uint8_t* seg, const float* time_s, const uint8_t* pic,
                     const float* m, int64_t meta_batch_stride, double window, double falloff,
                     double strength, double cap, const double* gain9, double scale,
                     int64_t b, int64_t h, int64_t i, double* out, int n_extra,
                     const double* extra_gains, const float* extra_m, int64_t m_len) {
  if (!Q || !K || !seg || !time_s || !pic || !m || !gain9 || !out) return -1;
  if (n_extra < 0 || n_extra > 3 || (n_extra > 0 && (!extra_gains || !extra_m))) return -1;
  const oracle_bindings extra = {n_extra, extra_gains, extra_m, m_len};
  if (b < 0 || b >= B || h < 0 || h >= H || i < 0 || i >= N || D < 1) return -1;
  if (scale == 0.0) scale = 1.0 / sqrt((double)D);
  int64_t head = (b * H + h) * N * D;
  const int64_t mo = meta_batch_stride * b;
  for (int64_t j = 0; j < N; ++j) {
    double dot = 0.0;
    for (int64_t k = 0; k < D; ++k)
      dot += widen(Q, dtype, head + i * D + k) * widen(K, dtype, head + j * D + k);
    out[j] = dot * scale + oracle_bias(i, j, seg + mo, time_s + mo, pic + mo, m + mo, window,
                                       falloff, strength, cap, gain9, &extra, mo);
  }
  return 0;
}

/* Number of threads the OpenMP runtime would use for oracle_attention_rows. */
int oracle_max_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}
