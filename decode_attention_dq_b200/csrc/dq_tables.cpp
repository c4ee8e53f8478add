// dq_tables.cpp -- host design of the analytic D-Quant tables (T1-T6).
//
// [news] "D-Quant: Entropy Coding Meets KV Cache at 2.26 Bits", section
// "Drift: Bending Variable Back to Fixed", 3rd paragraph: after rotation and
// normalisation the KV coordinates are close enough to N(0,1) that the
// probability model comes from the analytic form, with no calibration data;
// keys use 8 levels and values 6 at 2.26 bits. [news] "Why Fixed Width Is a
// Ceiling": entropy coding fits more levels into the same average budget.
//
// Level design (the pages leave it open): the entropy-constrained scalar
// quantiser (Chou, Lookabaugh & Gray 1989, scalar case) for N(0,1) whose
// entropy equals the container's rate, which is the Lloyd-Max quantiser
// (Max 1960) when that one already fits.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "dq_internal.h"

namespace dqi {
namespace {

constexpr double kInvSqrt2Pi = 0.39894228040143267794;
constexpr double kInvSqrt2 = 0.70710678118654752440;

// Standard normal density and the probability mass of (a, b].
double pdf(double t) { return std::isinf(t) ? 0.0 : kInvSqrt2Pi * std::exp(-0.5 * t * t); }

double mass(double a, double b) {
  // Upper tail Q(t) = erfc(t/sqrt2)/2, lower tail Phi(t) = erfc(-t/sqrt2)/2;
  // use whichever keeps the difference well conditioned.
  auto Q = [](double t) { return t == INFINITY ? 0.0 : (t == -INFINITY ? 1.0 : 0.5 * std::erfc(t * kInvSqrt2)); };
  auto P = [](double t) { return t == INFINITY ? 1.0 : (t == -INFINITY ? 0.0 : 0.5 * std::erfc(-t * kInvSqrt2)); };
  if (a >= 0.0) return Q(a) - Q(b);
  if (b <= 0.0) return P(b) - P(a);
  return 1.0 - Q(b) - P(a);
}

struct Quantizer {
  int n = 0;
  double y[kMaxLevels] = {};  // levels
  double t[kMaxLevels] = {};  // n-1 thresholds
  double p[kMaxLevels] = {};  // cell masses

  // Masses and centroids of the cells bounded by t; false if a cell is empty.
  bool centroids(double *cy) {
    for (int i = 0; i < n; ++i) {
      double a = i ? t[i - 1] : -INFINITY;
      double b = (i < n - 1) ? t[i] : INFINITY;
      double m = mass(a, b);
      if (!(m > 0.0) || !std::isfinite(m)) return false;
      p[i] = m;
      cy[i] = (pdf(a) - pdf(b)) / m;
    }
    return true;
  }
  static void make_odd(double *v, int len) {
    double w[kMaxLevels];
    for (int i = 0; i < len; ++i) w[i] = 0.5 * (v[i] - v[len - 1 - i]);
    std::memcpy(v, w, sizeof(double) * len);
  }
  double entropy() const {
    double h = 0.0;
    for (int i = 0; i < n; ++i) h += (p[i] > 0.0) ? -p[i] * std::log2(p[i]) : 0.0;
    return h;
  }
};

// Lloyd-Max: midpoint thresholds, centroid levels, to a fixed point.
bool lloyd_max(int n, Quantizer *q) {
  q->n = n;
  for (int i = 0; i < n; ++i) q->y[i] = 1.5 * (2.0 * i - (n - 1)) / (n - 1);
  double ny[kMaxLevels];
  for (int iter = 0; iter < 200000; ++iter) {
    for (int i = 0; i + 1 < n; ++i) q->t[i] = 0.5 * (q->y[i] + q->y[i + 1]);
    if (!q->centroids(ny)) return false;
    Quantizer::make_odd(ny, n);
    double delta = 0.0;
    for (int i = 0; i < n; ++i) delta = std::max(delta, std::abs(ny[i] - q->y[i]));
    std::memcpy(q->y, ny, sizeof(double) * n);
    if (delta < 1e-14) break;
  }
  for (int i = 0; i + 1 < n; ++i) q->t[i] = 0.5 * (q->y[i] + q->y[i + 1]);
  return q->centroids(ny);
}

// ECSQ at multiplier lambda from the Lloyd-Max start: thresholds where the
// neighbouring costs (u - y)^2 + lambda * (-log2 p) are equal, levels at the
// centroids; false when the design collapses (a cell empties or thresholds
// cross).
bool ecsq(const Quantizer &start, double lambda, Quantizer *q) {
  *q = start;
  const int n = q->n;
  double len[kMaxLevels], tt[kMaxLevels], ny[kMaxLevels];
  for (int i = 0; i + 1 < n; ++i) q->t[i] = 0.5 * (q->y[i] + q->y[i + 1]);
  if (!q->centroids(ny)) return false;
  for (int iter = 0; iter < 200000; ++iter) {
    for (int i = 0; i < n; ++i) len[i] = -std::log2(q->p[i]);
    for (int i = 0; i + 1 < n; ++i) {
      double gap = q->y[i + 1] - q->y[i];
      tt[i] = 0.5 * (q->y[i] + q->y[i + 1]) + lambda * (len[i + 1] - len[i]) / (2.0 * gap);
    }
    Quantizer::make_odd(tt, n - 1);
    for (int i = 0; i + 1 < n; ++i) q->t[i] = tt[i];
    for (int i = 0; i + 2 < n; ++i)
      if (!(q->t[i] < q->t[i + 1])) return false;
    if (!q->centroids(ny)) return false;
    Quantizer::make_odd(ny, n);
    double delta = 0.0;
    for (int i = 0; i < n; ++i) delta = std::max(delta, std::abs(ny[i] - q->y[i]));
    std::memcpy(q->y, ny, sizeof(double) * n);
    if (delta < 1e-14) break;
  }
  return true;
}

// Largest-remainder rounding of the upper half to 2048 with a floor of 1,
// one unit at a time (ties to the lower index), mirrored.
bool integer_freqs(const Quantizer &q, uint32_t *freq) {
  const int n = q.n, h = n / 2;
  long f[kMaxLevels];
  long total = 0;
  for (int j = 0; j < h; ++j) {
    f[j] = std::max(1L, static_cast<long>(std::floor(4096.0 * q.p[h + j])));
    total += f[j];
  }
  for (; total < 2048; ++total) {
    int pick = -1;
    double best = 0.0;
    for (int j = 0; j < h; ++j) {
      double residual = 4096.0 * q.p[h + j] - static_cast<double>(f[j]);
      if (pick < 0 || residual > best) { pick = j; best = residual; }
    }
    ++f[pick];
  }
  for (; total > 2048; --total) {
    int pick = -1;
    for (int j = 0; j < h; ++j)
      if (f[j] > 1 && (pick < 0 || f[j] > f[pick])) pick = j;
    if (pick < 0) return false;
    --f[pick];
  }
  for (int j = 0; j < h; ++j) freq[h + j] = freq[h - 1 - j] = static_cast<uint32_t>(f[j]);
  return true;
}

}  // namespace

int container_bytes_for(double bits_per_value) {
  return static_cast<int>(std::floor(bits_per_value * kD / 8.0 + 0.5));
}

int design_stream(int n_levels, int container_bytes, double rate_offset,
                  StreamDesign *out) {
  if (n_levels < 2 || n_levels > kMaxLevels || (n_levels & 1)) return DQ_ERR_CONFIG;
  if (container_bytes < kHeaderBytes + 1 || container_bytes > kMaxContainer) return DQ_ERR_BUDGET;
  StreamDesign d;
  d.n_levels = n_levels;
  d.container_bytes = container_bytes;
  d.payload_bytes = container_bytes - 2;
  // 24 of the payload bits hold the flushed 3-byte rANS state.
  d.rate = (8.0 * d.payload_bytes - 24.0) / kD + rate_offset;

  Quantizer lm, chosen;
  if (!lloyd_max(n_levels, &lm)) return DQ_ERR_CONFIG;
  if (lm.entropy() <= d.rate) {
    chosen = lm;
    d.lloyd_max = true;
    d.lambda = 0.0;
  } else {
    double lo = 0.0, hi = 1.0;
    Quantizer trial;
    for (int step = 0; step < 64; ++step) {
      const double mid = 0.5 * (lo + hi);
      const bool above = ecsq(lm, mid, &trial) && trial.entropy() > d.rate;
      (above ? lo : hi) = mid;
    }
    if (lo <= 0.0 || !ecsq(lm, lo, &chosen)) return DQ_ERR_BUDGET;
    d.lloyd_max = false;
    d.lambda = lo;
  }
  d.entropy = chosen.entropy();
  double second_moment = 0.0;
  for (int i = 0; i < n_levels; ++i) second_moment += chosen.p[i] * chosen.y[i] * chosen.y[i];
  d.mse = 1.0 - second_moment;
  std::memcpy(d.y, chosen.y, sizeof(d.y));
  std::memcpy(d.t, chosen.t, sizeof(d.t));
  std::memcpy(d.p, chosen.p, sizeof(d.p));
  if (!integer_freqs(chosen, d.freq)) return DQ_ERR_BUDGET;
  d.cum[0] = 0;
  for (int s = 0; s < n_levels; ++s) d.cum[s + 1] = d.cum[s] + d.freq[s];
  if (d.cum[n_levels] != kM) return DQ_ERR_BUDGET;
  for (int s = 0; s < n_levels; ++s) {
    d.levels[s] = static_cast<float>(d.y[s]);
    d.cost[s] = static_cast<float>(12.0 - std::log2(static_cast<double>(d.freq[s])));
  }
  for (int i = 0; i < kMaxLevels; ++i)
    d.thresholds[i] = (i < n_levels - 1) ? static_cast<float>(d.t[i]) : INFINITY;
  // The overflow fallback (every symbol at the innermost level of its side)
  // must always fit; bound its coded length conservatively.
  const double inner_bits = 12.0 - std::log2(static_cast<double>(d.freq[n_levels / 2]));
  const int worst = 3 + static_cast<int>(std::floor(kD * (inner_bits + 0.09) / 8.0)) + 1;
  if (worst > d.payload_bytes) return DQ_ERR_BUDGET;
  *out = d;
  return DQ_OK;
}

// Rotation signs: one splitmix64 stream from `seed`; KV head h uses outputs
// 2h and 2h+1, coordinate i reads bit i%64 of output 2h + i/64, set = -1.
void rotation_signs(uint64_t seed, int n_heads, int8_t *out) {
  uint64_t state = seed;
  auto next = [&state]() {
    state += 0x9E3779B97F4A7C15ull;
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  };
  for (int h = 0; h < n_heads; ++h) {
    const uint64_t words[2] = {next(), next()};
    for (int i = 0; i < kD; ++i)
      out[h * kD + i] = ((words[i >> 6] >> (i & 63)) & 1u) ? int8_t(-1) : int8_t(1);
  }
}

}  // namespace dqi
