/*
 * dq_oracle.c -- plain, slow, scalar CPU oracle for the D-Quant hot path.
 *
 * TEST INFRASTRUCTURE ONLY: loaded by tests/, __graft_entry__.smoke() and the
 * cpu_baseline / reference legs of bench.py. It shares no code with the
 * product library. Build: gcc -std=c11 -O2 -ffp-contract=off -fPIC -shared.
 * (-ffp-contract=off keeps every fp32 product and sum separately rounded;
 * the encoder's fp32 steps below are the format's definition.)
 *
 * Sources (see dq_oracle.h for the page titles):
 *   [news] "Why Fixed Width Is a Ceiling": after rotation and normalisation
 *          KV values are close to a normal distribution; entropy coding gives
 *          frequent symbols short codes.
 *   [news] "Drift: Bending Variable Back to Fixed": fixed-size byte container
 *          per token; rANS; drift of a few symbols from high-cost to nearby
 *          lower-cost symbols until the length fits; no symbol moves more than
 *          one reconstruction level; 8 levels for keys and 6 for values at a
 *          2.26-bit budget; probability model derived analytically.
 *   [abstract] drift turns each token's entropy-coded representation into a
 *          fixed-size bitstream for regular access and parallel dequantisation.
 * Textbook sources for steps the pages leave open:
 *   J. Max, "Quantizing for minimum distortion", IRE Trans. IT-6 (1960).
 *   P. A. Chou, T. Lookabaugh, R. M. Gray, "Entropy-constrained vector
 *     quantization", IEEE Trans. ASSP 37 (1989) -- scalar case (ECSQ).
 *   J. Duda, "Asymmetric numeral systems" (2013, arXiv:1311.2540); F. Giesen's
 *     public rANS notes (byte-wise renormalisation).
 *   J. J. Sylvester (1867) Hadamard construction; G. Steele, D. Lea,
 *     C. Flood, "Fast splittable pseudorandom number generators" (2014) for
 *     splitmix64.
 */
#include "dq_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define SQRT_D_F32 11.3137084989847604f /* fl32(sqrt(128)) */

/* ------------------------------------------------------------------ */
/* Normal distribution helpers (fp64, tail-accurate via erfc).        */
/* ------------------------------------------------------------------ */
static double norm_pdf(double t) {
  if (isinf(t)) return 0.0;
  return exp(-0.5 * t * t) / sqrt(2.0 * M_PI);
}
static double norm_cdf(double t) { /* P(u <= t) */
  if (t == INFINITY) return 1.0;
  if (t == -INFINITY) return 0.0;
  return 0.5 * erfc(-t / sqrt(2.0));
}
static double norm_sf(double t) { /* P(u > t) */
  if (t == INFINITY) return 0.0;
  if (t == -INFINITY) return 1.0;
  return 0.5 * erfc(t / sqrt(2.0));
}
/* Probability and centroid of the cell [a, b] under N(0,1).
 * Returns 0 if the cell has no mass in fp64. */
static int cell(double a, double b, double *p, double *centroid) {
  double m = (a >= 0.0) ? (norm_sf(a) - norm_sf(b)) : (norm_cdf(b) - norm_cdf(a));
  if (!(m > 0.0)) return 0;
  *p = m;
  *centroid = (norm_pdf(a) - norm_pdf(b)) / m; /* E[u | a < u <= b] */
  return 1;
}
/* All n cells for interior thresholds t[0..n-2]. */
static int cells(int n, const double *t, double *p, double *y) {
  for (int i = 0; i < n; ++i) {
    double a = (i == 0) ? -INFINITY : t[i - 1];
    double b = (i == n - 1) ? INFINITY : t[i];
    if (!cell(a, b, &p[i], &y[i])) return 0;
  }
  return 1;
}
static void mirror_odd(int n, double *v) { /* v[i] <- (v[i] - v[n-1-i]) / 2 */
  double w[DQO_MAX_LEVELS];
  for (int i = 0; i < n; ++i) w[i] = 0.5 * (v[i] - v[n - 1 - i]);
  memcpy(v, w, sizeof(double) * (size_t)n);
}

double dqo_entropy(int n, const double *p) {
  double h = 0.0;
  for (int i = 0; i < n; ++i)
    if (p[i] > 0.0) h -= p[i] * log2(p[i]);
  return h;
}

/* T2. Lloyd-Max quantiser for N(0,1) (Max 1960): thresholds at midpoints,
 * levels at cell centroids, iterated from levels uniform on [-2, 2] until no
 * level moves by 1e-13. */
int dqo_lloyd_max(int n, double *y, double *t, double *p, int *iters) {
  if (n < 2 || n > DQO_MAX_LEVELS) return -1;
  double yn[DQO_MAX_LEVELS];
  for (int i = 0; i < n; ++i) y[i] = -2.0 + 4.0 * (double)i / (double)(n - 1);
  int it = 0;
  for (; it < 100000; ++it) {
    for (int i = 0; i < n - 1; ++i) t[i] = 0.5 * (y[i] + y[i + 1]);
    if (!cells(n, t, p, yn)) return -2;
    mirror_odd(n, yn);
    double d = 0.0;
    for (int i = 0; i < n; ++i) d = fmax(d, fabs(yn[i] - y[i]));
    memcpy(y, yn, sizeof(double) * (size_t)n);
    if (d < 1e-13) break;
  }
  for (int i = 0; i < n - 1; ++i) t[i] = 0.5 * (y[i] + y[i + 1]);
  if (!cells(n, t, p, yn)) return -2;
  if (iters) *iters = it;
  return 0;
}

/* T3. Entropy-constrained scalar quantiser (Chou-Lookabaugh-Gray, scalar
 * case) at multiplier lambda, started from y_init. One pass: code lengths
 * l_i = -log2 p_i; thresholds where the Lagrangian costs (u-y)^2 + lambda*l
 * of neighbouring cells are equal,
 *   t_i = (y_i + y_{i+1})/2 + lambda (l_{i+1} - l_i) / (2 (y_{i+1} - y_i));
 * then levels at the new cells' centroids. Thresholds and levels are made
 * exactly odd-symmetric each pass. Returns -3 when a cell empties or the
 * thresholds cross (the design has collapsed at this lambda). */
int dqo_ecsq(int n, double lambda, const double *y_init, double *y, double *t,
             double *p, int *iters) {
  if (n < 2 || n > DQO_MAX_LEVELS) return -1;
  double yn[DQO_MAX_LEVELS], l[DQO_MAX_LEVELS], tt[DQO_MAX_LEVELS];
  memcpy(y, y_init, sizeof(double) * (size_t)n);
  for (int i = 0; i < n - 1; ++i) t[i] = 0.5 * (y[i] + y[i + 1]);
  if (!cells(n, t, p, yn)) return -3;
  int it = 0;
  for (; it < 200000; ++it) {
    for (int i = 0; i < n; ++i) l[i] = -log2(p[i]);
    for (int i = 0; i < n - 1; ++i)
      tt[i] = 0.5 * (y[i] + y[i + 1]) +
              lambda * (l[i + 1] - l[i]) / (2.0 * (y[i + 1] - y[i]));
    for (int i = 0; i < n - 1; ++i) t[i] = 0.5 * (tt[i] - tt[n - 2 - i]);
    for (int i = 0; i + 1 < n - 1; ++i)
      if (!(t[i] < t[i + 1])) return -3;
    if (!cells(n, t, p, yn)) return -3;
    mirror_odd(n, yn);
    double d = 0.0;
    for (int i = 0; i < n; ++i) d = fmax(d, fabs(yn[i] - y[i]));
    memcpy(y, yn, sizeof(double) * (size_t)n);
    if (d < 1e-13) break;
  }
  if (iters) *iters = it;
  return 0;
}

/* T4. Integer frequencies summing to M = 4096, odd-symmetric. On the upper
 * half (symbols n/2..n-1, target 2048): f = max(1, floor(4096 p)); the
 * shortfall goes one unit at a time to the symbol with the largest
 * 4096 p - f (ties: the lower index); an overshoot is taken one unit at a
 * time from the largest f above 1 (ties: the lower index). Then mirrored. */
int dqo_int_freqs(int n, const double *p, uint32_t *freq) {
  if (n < 2 || (n & 1) || n > DQO_MAX_LEVELS) return -1;
  int h = n / 2;
  long f[DQO_MAX_LEVELS];
  long sum = 0;
  for (int j = 0; j < h; ++j) {
    double target = 4096.0 * p[h + j];
    long v = (long)floor(target);
    if (v < 1) v = 1;
    f[j] = v;
    sum += v;
  }
  long rem = 2048 - sum;
  while (rem > 0) {
    int best = 0;
    double bestr = 4096.0 * p[h] - (double)f[0];
    for (int j = 1; j < h; ++j) {
      double r = 4096.0 * p[h + j] - (double)f[j];
      if (r > bestr) { bestr = r; best = j; }
    }
    f[best] += 1;
    rem -= 1;
  }
  while (rem < 0) {
    int best = -1;
    for (int j = 0; j < h; ++j)
      if (f[j] > 1 && (best < 0 || f[j] > f[best])) best = j;
    if (best < 0) return -2;
    f[best] -= 1;
    rem += 1;
  }
  for (int j = 0; j < h; ++j) {
    freq[h + j] = (uint32_t)f[j];
    freq[h - 1 - j] = (uint32_t)f[j];
  }
  return 0;
}

/* T1. Container size from a bits-per-value budget: round half up of
 * bits * 128 / 8 (2.26 -> 36 B, 1.96 -> 31 B, 3.0 -> 48 B). */
int dqo_container_bytes(double bits_per_value) {
  return (int)floor(bits_per_value * (double)DQO_D / 8.0 + 0.5);
}

/* T1-T5 for one stream. Target rate r = (8P - 24)/128 + rate_offset bits per
 * value, where P = C - 2 and 24 bits are the final-state flush. If the
 * Lloyd-Max design already meets r it is used (lambda = 0); otherwise lambda
 * is found by 60 bisection steps on [0, 1] so that H(p(lambda)) = r, a
 * collapsed design counting as "entropy too low". */
int dqo_build_stream(int n_levels, int container_bytes, double rate_offset,
                     dqo_stream *out) {
  int n = n_levels;
  if (n < 2 || (n & 1) || n > DQO_MAX_LEVELS) return -1;
  if (container_bytes < DQO_HEADER_BYTES + 1 || container_bytes > 4096) return -1;
  memset(out, 0, sizeof(*out));
  out->n_levels = n;
  out->container_bytes = container_bytes;
  out->payload_bytes = container_bytes - 2;
  double r = (8.0 * (double)out->payload_bytes - 24.0) / (double)DQO_D + rate_offset;
  out->rate = r;

  double ylm[DQO_MAX_LEVELS], tlm[DQO_MAX_LEVELS], plm[DQO_MAX_LEVELS];
  if (dqo_lloyd_max(n, ylm, tlm, plm, NULL) != 0) return -2;
  if (dqo_entropy(n, plm) <= r) {
    memcpy(out->y, ylm, sizeof(ylm));
    memcpy(out->t, tlm, sizeof(tlm));
    memcpy(out->p, plm, sizeof(plm));
    out->lambda = 0.0;
    out->is_lloyd_max = 1;
  } else {
    double y[DQO_MAX_LEVELS], t[DQO_MAX_LEVELS], p[DQO_MAX_LEVELS];
    double lo = 0.0, hi = 1.0;
    for (int k = 0; k < 60; ++k) {
      double mid = 0.5 * (lo + hi);
      int rc = dqo_ecsq(n, mid, ylm, y, t, p, NULL);
      if (rc == 0 && dqo_entropy(n, p) > r)
        lo = mid;
      else
        hi = mid;
    }
    if (lo == 0.0) return -3; /* no lambda in (0, 1] reaches r */
    if (dqo_ecsq(n, lo, ylm, y, t, p, NULL) != 0) return -3;
    memcpy(out->y, y, sizeof(y));
    memcpy(out->t, t, sizeof(t));
    memcpy(out->p, p, sizeof(p));
    out->lambda = lo;
    out->is_lloyd_max = 0;
  }
  out->entropy = dqo_entropy(n, out->p);
  double m = 1.0;
  for (int i = 0; i < n; ++i) m -= out->p[i] * out->y[i] * out->y[i];
  out->mse = m;

  if (dqo_int_freqs(n, out->p, out->freq) != 0) return -4;
  out->cum[0] = 0;
  for (int s = 0; s < n; ++s) out->cum[s + 1] = out->cum[s] + out->freq[s];
  if (out->cum[n] != DQO_M) return -4;
  for (int s = 0; s < n; ++s) {
    out->yf[s] = (float)out->y[s];
    out->cost[s] = (float)(12.0 - log2((double)out->freq[s]));
  }
  for (int i = 0; i < n - 1; ++i) out->tf[i] = (float)out->t[i];

  /* The overflow fallback (every symbol at the innermost level of its side)
   * must always fit: bytes <= 3 + floor(128 (l_inner + 0.09) / 8) + 1. */
  double l_in = 12.0 - log2((double)out->freq[n / 2]);
  int worst = 3 + (int)floor((double)DQO_D * (l_in + 0.09) / 8.0) + 1;
  if (worst > out->payload_bytes) return -5;
  return 0;
}

/* ------------------------------------------------------------------ */
/* splitmix64 and the per-head rotation signs                         */
/* ------------------------------------------------------------------ */
uint64_t dqo_splitmix64_next(uint64_t *state) {
  uint64_t z = (*state += 0x9E3779B97F4A7C15ull);
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

/* T6 (reading; the pages name no seed): KV head h takes outputs 2h and 2h+1
 * of one splitmix64 stream seeded with `seed`; coordinate i reads bit
 * (i mod 64) of output 2h + i/64, and a set bit means sign -1. */
void dqo_signs(uint64_t seed, int head, int8_t *signs) {
  uint64_t st = seed, w0 = 0, w1 = 0;
  for (int k = 0; k <= 2 * head + 1; ++k) {
    uint64_t w = dqo_splitmix64_next(&st);
    if (k == 2 * head) w0 = w;
    if (k == 2 * head + 1) w1 = w;
  }
  for (int i = 0; i < DQO_D; ++i) {
    uint64_t bit = (i < 64) ? (w0 >> i) & 1u : (w1 >> (i - 64)) & 1u;
    signs[i] = bit ? (int8_t)-1 : (int8_t)1;
  }
}

/* ------------------------------------------------------------------ */
/* Number formats                                                     */
/* ------------------------------------------------------------------ */
/* IEEE 754 binary32 -> binary16, round to nearest, ties to even. */
uint16_t dqo_f32_to_f16_rn(float v) {
  uint32_t b;
  memcpy(&b, &v, sizeof(b));
  uint32_t sign = (b >> 16) & 0x8000u;
  uint32_t exp = (b >> 23) & 0xFFu;
  uint32_t man = b & 0x7FFFFFu;
  if (exp == 0xFFu) return (uint16_t)(sign | 0x7C00u | (man ? 0x200u : 0u));
  int e = (int)exp - 127 + 15;
  if (e >= 31) return (uint16_t)(sign | 0x7C00u);
  if (e <= 0) {
    uint32_t m = (exp == 0) ? man : (man | 0x800000u);
    int s = 14 - e; /* value = m * 2^(e-14) half-subnormal units */
    if (exp == 0 || s >= 26) return (uint16_t)sign;
    uint32_t k = m >> s;
    uint32_t rem = m & ((1u << s) - 1u);
    uint32_t half = 1u << (s - 1);
    if (rem > half || (rem == half && (k & 1u))) k += 1u;
    return (uint16_t)(sign | k);
  }
  uint32_t h = sign | ((uint32_t)e << 10) | (man >> 13);
  uint32_t rem = man & 0x1FFFu;
  if (rem > 0x1000u || (rem == 0x1000u && (h & 1u))) h += 1u;
  return (uint16_t)h;
}

float dqo_f16_to_f32(uint16_t h) {
  uint32_t sign = ((uint32_t)h & 0x8000u) << 16;
  uint32_t exp = ((uint32_t)h >> 10) & 0x1Fu;
  uint32_t man = (uint32_t)h & 0x3FFu;
  float v;
  if (exp == 0) {
    v = (float)man * 5.9604644775390625e-08f; /* 2^-24, exact */
    uint32_t b;
    memcpy(&b, &v, 4);
    b |= sign;
    memcpy(&v, &b, 4);
    return v;
  }
  uint32_t b = sign | ((exp == 31 ? 0xFFu : exp - 15 + 127) << 23) | (man << 13);
  memcpy(&v, &b, 4);
  return v;
}

float dqo_bf16_to_f32(uint16_t x) {
  uint32_t b = (uint32_t)x << 16;
  float v;
  memcpy(&v, &b, 4);
  return v;
}

/* ------------------------------------------------------------------ */
/* Encode (append) path                                               */
/* ------------------------------------------------------------------ */
/* E2. Unnormalised Walsh-Hadamard transform in Sylvester order, fp32:
 * stages h = 1, 2, 4, ..., n/2, butterfly (a, b) -> (a + b, a - b). */
void dqo_wht_f32(float *z, int n) {
  for (int h = 1; h < n; h *= 2)
    for (int j = 0; j < n; j += 2 * h)
      for (int k = j; k < j + h; ++k) {
        float a = z[k], b = z[k + h];
        z[k] = a + b;
        z[k + h] = a - b;
      }
}

/* E1-E3 ([news] "Why Fixed Width Is a Ceiling": rotation and normalisation
 * make the coordinates close to N(0,1)). a = s * x; z = H a; the squared
 * norm is summed in a fixed tree (32 partial sums
 * ((z_l^2 + z_{l+32}^2) + (z_{l+64}^2 + z_{l+96}^2)), then pairs at xor
 * offsets 16, 8, 4, 2, 1); r = sqrt(ss); u = z * (fl(sqrt 128) / r); the
 * stored norm is fp16(min(r / fl(sqrt 128), 65504)) = ||x||. A vector with a
 * non-finite input or a non-finite sum of squares is treated as zero
 * (u = 0, norm 0) and the function returns 1; r == 0 or a non-finite scale
 * also gives u = 0. */
int dqo_rotate_normalize(const float *x, const int8_t *signs, float *u,
                         uint16_t *norm16) {
  float z[DQO_D];
  int nonfinite = 0;
  for (int i = 0; i < DQO_D; ++i) {
    if (!isfinite(x[i])) nonfinite = 1;
    z[i] = (signs[i] < 0) ? -x[i] : x[i];
  }
  if (nonfinite) {
    memset(u, 0, sizeof(float) * DQO_D);
    *norm16 = 0;
    return 1;
  }
  dqo_wht_f32(z, DQO_D);
  float part[32], next[32];
  for (int l = 0; l < 32; ++l) {
    float a = z[l] * z[l];
    float b = z[l + 32] * z[l + 32];
    float c = z[l + 64] * z[l + 64];
    float d = z[l + 96] * z[l + 96];
    part[l] = (a + b) + (c + d);
  }
  for (int off = 16; off >= 1; off /= 2) {
    for (int l = 0; l < 32; ++l) next[l] = part[l] + part[l ^ off];
    memcpy(part, next, sizeof(part));
  }
  float ss = part[0];
  if (!isfinite(ss)) {
    memset(u, 0, sizeof(float) * DQO_D);
    *norm16 = 0;
    return 1;
  }
  float r = sqrtf(ss);
  float sigma = (r == 0.0f) ? 0.0f : SQRT_D_F32 / r;
  if (r == 0.0f || !isfinite(sigma)) {
    memset(u, 0, sizeof(float) * DQO_D);
  } else {
    for (int i = 0; i < DQO_D; ++i) u[i] = z[i] * sigma;
  }
  float nv = r / SQRT_D_F32;
  if (nv > 65504.0f) nv = 65504.0f;
  *norm16 = dqo_f32_to_f16_rn(nv);
  return 0;
}

/* E4. Symbol = number of fp32 thresholds t_j <= u (a tie goes up). */
void dqo_quantize(const dqo_stream *st, const float *u, int n, uint8_t *q) {
  for (int i = 0; i < n; ++i) {
    int c = 0;
    for (int j = 0; j < st->n_levels - 1; ++j)
      if (st->tf[j] <= u[i]) c += 1;
    q[i] = (uint8_t)c;
  }
}

/* E5 (rANS, [news] "Drift..."; parameters are a reading: 32-bit state,
 * L = 2^16, byte-wise renormalisation, M = 2^12). Symbols are coded last to
 * first from x = L: while x >= 4096 f push the low byte and shift; then
 * x = (x / f) * 4096 + (x mod f) + c. The output is the final state as 3
 * little-endian bytes followed by the pushed bytes, last pushed first.
 * Returns the length 3 + #pushed; writes `out` only when length <= cap. */
int dqo_rans_encode(const dqo_stream *st, const uint8_t *q, int n,
                    uint8_t *out, int cap) {
  uint8_t *stack = (uint8_t *)malloc((size_t)2 * (size_t)n + 8);
  if (!stack) return -1;
  uint32_t x = DQO_L;
  int np = 0;
  for (int i = n - 1; i >= 0; --i) {
    uint32_t f = st->freq[q[i]];
    uint32_t c = st->cum[q[i]];
    uint32_t xmax = ((DQO_L >> DQO_PROB_BITS) << 8) * f;
    while (x >= xmax) {
      stack[np++] = (uint8_t)(x & 0xFFu);
      x >>= 8;
    }
    x = (x / f) * DQO_M + (x % f) + c;
  }
  int len = 3 + np;
  if (out && len <= cap) {
    out[0] = (uint8_t)(x & 0xFFu);
    out[1] = (uint8_t)((x >> 8) & 0xFFu);
    out[2] = (uint8_t)((x >> 16) & 0xFFu);
    for (int k = 0; k < np; ++k) out[3 + k] = stack[np - 1 - k];
  }
  free(stack);
  return len;
}

/* E6 drift ([news] "Drift: Bending Variable Back to Fixed": when a stream is
 * over budget, a few symbols drift from high-cost symbols to nearby
 * lower-cost ones until it fits; none moves more than one level). Greedy
 * reading: while the coded length exceeds `budget`, among symbols not yet
 * moved and neighbours j = q +- 1 with cost[j] < cost[q], pick the least
 *   key = ((u - y_j)^2 - (u - y_q)^2) / (cost[q] - cost[j])   (fp32)
 * (added squared error per bit saved); ties to the lowest i, then the lower
 * j. Move it, mark it, re-encode. If no candidate is left and it still does
 * not fit (reading; the pages are silent), every symbol goes to the
 * innermost level of its side and *fallback is set. Returns the length. */
int dqo_drift_fit(const dqo_stream *st, const float *u, uint8_t *q, int n,
                  int budget, int *moves, uint8_t *moved_mask, int *fallback) {
  uint8_t *moved = (uint8_t *)calloc((size_t)n, 1);
  if (!moved) return -1;
  int len = dqo_rans_encode(st, q, n, NULL, 0);
  int nm = 0;
  *fallback = 0;
  while (len > budget) {
    int bi = -1, bj = -1;
    float bkey = 0.0f;
    for (int i = 0; i < n; ++i) {
      if (moved[i]) continue;
      int s = q[i];
      for (int dj = -1; dj <= 1; dj += 2) {
        int j = s + dj;
        if (j < 0 || j >= st->n_levels) continue;
        if (!(st->cost[j] < st->cost[s])) continue;
        float dn = u[i] - st->yf[j];
        float d0 = u[i] - st->yf[s];
        float en = dn * dn;
        float e0 = d0 * d0;
        float num = en - e0;
        float den = st->cost[s] - st->cost[j];
        float key = num / den;
        if (bi < 0 || key < bkey) {
          bi = i;
          bj = j;
          bkey = key;
        }
      }
    }
    if (bi < 0) break;
    q[bi] = (uint8_t)bj;
    moved[bi] = 1;
    nm += 1;
    len = dqo_rans_encode(st, q, n, NULL, 0);
  }
  if (len > budget) {
    int h = st->n_levels / 2;
    for (int i = 0; i < n; ++i) q[i] = (uint8_t)((q[i] >= h) ? h : h - 1);
    len = dqo_rans_encode(st, q, n, NULL, 0);
    *fallback = 1;
  }
  if (moved_mask) memcpy(moved_mask, moved, (size_t)n);
  free(moved);
  *moves = nm;
  return len;
}

/* E1-E7 for one 128-dim vector. Container (reading): bytes [0,1] fp16 norm
 * little-endian, [2,4] final rANS state little-endian, then the pushed bytes,
 * then zero padding to C. Returns 0, or -1 if even the fallback did not fit. */
int dqo_encode_vector(const dqo_stream *st, const int8_t *signs,
                      const float *x, uint8_t *container, uint8_t *q_out,
                      dqo_stats *stats) {
  float u[DQO_D];
  uint16_t nh = 0;
  int nf = dqo_rotate_normalize(x, signs, u, &nh);
  uint8_t q[DQO_D];
  dqo_quantize(st, u, DQO_D, q);
  int moves = 0, fb = 0;
  int len = dqo_drift_fit(st, u, q, DQO_D, st->payload_bytes, &moves, NULL, &fb);
  memset(container, 0, (size_t)st->container_bytes);
  container[0] = (uint8_t)(nh & 0xFFu);
  container[1] = (uint8_t)(nh >> 8);
  if (stats) {
    stats->nonfinite_inputs += (uint64_t)nf;
    stats->syms_drifted += (uint64_t)moves;
    stats->cont_drifted += (moves > 0) ? 1u : 0u;
    stats->overflow_fallbacks += (uint64_t)fb;
  }
  if (q_out) memcpy(q_out, q, DQO_D);
  if (len < 0 || len > st->payload_bytes) return -1;
  dqo_rans_encode(st, q, DQO_D, container + 2, st->payload_bytes);
  return 0;
}

/* Rate-distortion fill (drift mode 1). [news] "So What": once entropy
 * coding sits in the KV path, the rate-distortion toolbox of video coding
 * carries over. Reading: a container's unused bytes are spent on accuracy,
 * the mirror image of drift. A candidate is a symbol i whose nearest level j
 * (least (u_i - y_j)^2 in fp32, ties to the lower level) is one level from
 * its current symbol q[i] and at most one level from the quantiser's symbol
 * q0[i], with dD = (u_i - y_j)^2 - (u_i - y_q)^2 < 0 and
 * dR = cost[j] - cost[q] > 0 (fp32). Candidates are taken in order of
 * key = dD / dR (fp32; ties to the lower i); each is kept if the re-encoded
 * stream still fits `budget`, else undone. Returns the final length;
 * *ups = candidates kept. */
int dqo_rd_fill(const dqo_stream *st, const float *u, const uint8_t *q0,
                uint8_t *q, int n, int budget, int *ups) {
  int len = dqo_rans_encode(st, q, n, NULL, 0);
  *ups = 0;
  if (len > budget) return len;
  int ci[DQO_D], cj[DQO_D];
  float ck[DQO_D];
  int nc = 0;
  for (int i = 0; i < n && i < DQO_D; ++i) {
    int j = 0;
    float best = 0.0f;
    for (int l = 0; l < st->n_levels; ++l) {
      float d = u[i] - st->yf[l];
      float e = d * d;
      if (l == 0 || e < best) {
        best = e;
        j = l;
      }
    }
    int s = q[i];
    if (j == s || abs(j - s) != 1 || abs(j - (int)q0[i]) > 1) continue;
    float dj = u[i] - st->yf[j];
    float ds = u[i] - st->yf[s];
    float dd = dj * dj - ds * ds;
    float dr = st->cost[j] - st->cost[s];
    if (!(dd < 0.0f) || !(dr > 0.0f)) continue;
    float key = dd / dr;
    /* insertion in (key, i) order */
    int k = nc++;
    while (k > 0 && (ck[k - 1] > key)) {
      ck[k] = ck[k - 1];
      ci[k] = ci[k - 1];
      cj[k] = cj[k - 1];
      --k;
    }
    ck[k] = key;
    ci[k] = i;
    cj[k] = j;
  }
  for (int k = 0; k < nc; ++k) {
    uint8_t old = q[ci[k]];
    q[ci[k]] = (uint8_t)cj[k];
    int l2 = dqo_rans_encode(st, q, n, NULL, 0);
    if (l2 > budget) {
      q[ci[k]] = old;
    } else {
      len = l2;
      *ups += 1;
    }
  }
  return len;
}

/* E1-E7 with the drift mode: 0 = drift only (dqo_encode_vector), 1 = drift
 * then the rate-distortion fill (skipped after a fallback). */
int dqo_encode_vector_mode(const dqo_stream *st, const int8_t *signs,
                           const float *x, uint8_t *container, uint8_t *q_out,
                           dqo_stats *stats, int drift_mode) {
  if (drift_mode == 0) return dqo_encode_vector(st, signs, x, container, q_out, stats);
  float u[DQO_D];
  uint16_t nh = 0;
  int nf = dqo_rotate_normalize(x, signs, u, &nh);
  uint8_t q0[DQO_D], q[DQO_D];
  dqo_quantize(st, u, DQO_D, q0);
  memcpy(q, q0, DQO_D);
  int moves = 0, fb = 0, ups = 0;
  int len = dqo_drift_fit(st, u, q, DQO_D, st->payload_bytes, &moves, NULL, &fb);
  if (!fb && len <= st->payload_bytes) len = dqo_rd_fill(st, u, q0, q, DQO_D, st->payload_bytes, &ups);
  memset(container, 0, (size_t)st->container_bytes);
  container[0] = (uint8_t)(nh & 0xFFu);
  container[1] = (uint8_t)(nh >> 8);
  if (stats) {
    stats->nonfinite_inputs += (uint64_t)nf;
    stats->syms_drifted += (uint64_t)moves;
    stats->cont_drifted += (moves > 0) ? 1u : 0u;
    stats->overflow_fallbacks += (uint64_t)fb;
    stats->syms_filled += (uint64_t)ups;
  }
  if (q_out) memcpy(q_out, q, DQO_D);
  if (len < 0 || len > st->payload_bytes) return -1;
  dqo_rans_encode(st, q, DQO_D, container + 2, st->payload_bytes);
  return 0;
}

/* ------------------------------------------------------------------ */
/* Decode                                                             */
/* ------------------------------------------------------------------ */
/* rANS decode of n symbols from buf[0..len): x from the 3 state bytes; per
 * symbol slot = x mod 4096, s with cum[s] <= slot < cum[s+1],
 * x = f_s (x >> 12) + slot - cum[s], then bytes are shifted in while x < L.
 * Status: 0 ok, 1 initial state below L, 2 read past the end,
 * 3 final state != L. */
int dqo_rans_decode(const dqo_stream *st, const uint8_t *buf, int len,
                    uint8_t *q, int n, uint32_t *x_final, int *consumed) {
  if (len < 3) return 2;
  uint32_t x = (uint32_t)buf[0] | ((uint32_t)buf[1] << 8) | ((uint32_t)buf[2] << 16);
  int pos = 3;
  if (x < DQO_L) {
    if (x_final) *x_final = x;
    if (consumed) *consumed = pos;
    return 1;
  }
  for (int i = 0; i < n; ++i) {
    uint32_t slot = x & (DQO_M - 1u);
    int s = 0;
    while (!(slot < st->cum[s + 1])) s += 1;
    q[i] = (uint8_t)s;
    x = st->freq[s] * (x >> DQO_PROB_BITS) + slot - st->cum[s];
    while (x < DQO_L) {
      if (pos >= len) {
        if (x_final) *x_final = x;
        if (consumed) *consumed = pos;
        return 2;
      }
      x = (x << 8) | (uint32_t)buf[pos++];
    }
  }
  if (x_final) *x_final = x;
  if (consumed) *consumed = pos;
  return (x == DQO_L) ? 0 : 3;
}

/* Container decode; status 4 = non-zero padding after the coded bytes. */
int dqo_decode_container(const dqo_stream *st, const uint8_t *container,
                         uint8_t *q, uint16_t *norm16) {
  *norm16 = (uint16_t)(container[0] | (container[1] << 8));
  memset(q, 0, DQO_D);
  int consumed = 0;
  uint32_t xf = 0;
  int rc = dqo_rans_decode(st, container + 2, st->payload_bytes, q, DQO_D, &xf,
                           &consumed);
  if (rc != 0) return rc;
  for (int k = 2 + consumed; k < st->container_bytes; ++k)
    if (container[k] != 0) return 4;
  return 0;
}

/* ------------------------------------------------------------------ */
/* Batch helpers                                                      */
/* ------------------------------------------------------------------ */
int dqo_encode_batch(const dqo_stream *st, const int8_t *signs_per_head,
                     const float *x, const int32_t *head_of, int64_t n_vec,
                     uint8_t *containers, uint8_t *syms, dqo_stats *stats) {
  int bad = 0;
  for (int64_t v = 0; v < n_vec; ++v) {
    const int8_t *sg = signs_per_head + (int64_t)head_of[v] * DQO_D;
    int rc = dqo_encode_vector(st, sg, x + v * DQO_D,
                               containers + v * st->container_bytes,
                               syms ? syms + v * DQO_D : NULL, stats);
    if (rc != 0) bad += 1;
  }
  return bad;
}

int dqo_encode_batch_mode(const dqo_stream *st, const int8_t *signs_per_head,
                          const float *x, const int32_t *head_of, int64_t n_vec,
                          uint8_t *containers, uint8_t *syms, dqo_stats *stats,
                          int drift_mode) {
  int bad = 0;
  for (int64_t v = 0; v < n_vec; ++v) {
    const int8_t *sg = signs_per_head + (int64_t)head_of[v] * DQO_D;
    int rc = dqo_encode_vector_mode(st, sg, x + v * DQO_D, containers + v * st->container_bytes,
                                    syms ? syms + v * DQO_D : NULL, stats, drift_mode);
    if (rc != 0) bad += 1;
  }
  return bad;
}

int64_t dqo_decode_batch(const dqo_stream *st, const uint8_t *containers,
                         int64_t n_vec, uint8_t *syms, uint16_t *norm16,
                         int32_t *status) {
  int64_t bad = 0;
  for (int64_t v = 0; v < n_vec; ++v) {
    int rc = dqo_decode_container(st, containers + v * st->container_bytes,
                                  syms + v * DQO_D, norm16 + v);
    if (status) status[v] = rc;
    if (rc != 0) bad += 1;
  }
  return bad;
}
