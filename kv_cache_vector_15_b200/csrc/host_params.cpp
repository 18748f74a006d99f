// Host-side derivation of TurboQuant's fixed parameters (no CUDA calls).
//
//  * D, the Rademacher diagonal of R = H_d D / sqrt(d)
//      [0h-n0.github.io "ICLR 2026論文解説: TurboQuant", section "Step 1: PolarQuant"];
//  * S, the m x d Gaussian QJL projection
//      [Qiita TurboQuant explainer, section "Stage 2: QJL"];
//  * the (b-1)-bit Lloyd-Max codebook for one rotated coordinate
//      [Qiita explainer, "Stage 1: PolarQuant", Lloyd-Max step; ai.spot.hk
//       "Google TurboQuant", section "隨機旋轉與Beta分佈"].
//
// Random numbers: SplitMix64 (Steele, Lea & Flood 2014) used as a counter
// generator, output(seed, stream, i) = finalizer(seed + (stream*2^40 + i + 1) *
// 0x9E3779B97F4A7C15).  D_i = +1 iff bit 0 of stream-0 output i is clear.
// S_{j,i} = sqrt(-2 ln u1) cos(2 pi u2) with u = top 53 bits * 2^-53 of
// stream-1 outputs 2(j d + i) and 2(j d + i) + 1, u1 = 1 - u in (0, 1],
// rounded once (nearest, ties to even) to IEEE binary16.
//
// Codebook: the coordinate of a uniform unit vector in R^d has density
// f_d(x) = (1 - x^2)^k / (2 G_k(1)), k = (d-3)/2, with G_k(x) = int_0^x (1-t^2)^k dt.
// For even d, k is a half-integer and G_k follows from the integration-by-parts
// recurrence  G_k(x) = (x (1-x^2)^k + 2k G_{k-1}(x)) / (2k + 1)  started at
// G_{1/2}(x) = (x sqrt(1-x^2) + asin x) / 2.  The recurrence multiplies the
// carried error by 2k/(2k+1) < 1 at every step, so it is stable.  First
// moments have the closed form int_a^b x (1-x^2)^k dx =
// ((1-a^2)^(k+1) - (1-b^2)^(k+1)) / (2(k+1)).  Lloyd's iteration
// (thresholds = midpoints, centroids = conditional means) runs on the
// positive half of the symmetric codebook until it stops improving.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {

static constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

static inline uint64_t splitmix64(uint64_t seed, uint64_t counter) {
  uint64_t z = seed + (counter + 1) * kGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

static inline uint64_t stream_counter(uint64_t stream, uint64_t i) { return (stream << 40) + i; }

// Round a double once to binary16 (nearest, ties to even).  |v| < 65504.
uint16_t double_to_half_bits(double v) {
  uint16_t sign = std::signbit(v) ? 0x8000 : 0;
  double a = std::fabs(v);
  if (a == 0.0) return sign;
  int e2;
  std::frexp(a, &e2);          // a = f 2^e2, f in [0.5, 1)
  int e = e2 - 1;              // a in [2^e, 2^(e+1))
  if (e < -14) {               // subnormal: multiples of 2^-24
    double q = std::nearbyint(std::ldexp(a, 24));   // exact scaling; default rounding is to-even
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(q));   // q == 1024 is the smallest normal
  }
  double q = std::nearbyint(std::ldexp(a, 10 - e)); // in [1024, 2048]
  if (q >= 2048.0) { q = 1024.0; e += 1; }
  return static_cast<uint16_t>(sign | static_cast<uint16_t>((e + 15) << 10) |
                               static_cast<uint16_t>(static_cast<int>(q) - 1024));
}

void rademacher(int d, uint64_t seed, int8_t* D) {
  for (int i = 0; i < d; ++i) D[i] = (splitmix64(seed, stream_counter(0, i)) & 1ull) ? -1 : 1;
}

void gaussian_projection_half(int m, int d, uint64_t seed, uint16_t* S_bits) {
  const double two_pi = 6.283185307179586476925286766559;
  const uint64_t n = static_cast<uint64_t>(m) * static_cast<uint64_t>(d);
  for (uint64_t e = 0; e < n; ++e) {
    uint64_t w1 = splitmix64(seed, stream_counter(1, 2 * e));
    uint64_t w2 = splitmix64(seed, stream_counter(1, 2 * e + 1));
    double u1 = 1.0 - static_cast<double>(w1 >> 11) * 0x1.0p-53;
    double u2 = static_cast<double>(w2 >> 11) * 0x1.0p-53;
    double g = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
    S_bits[e] = double_to_half_bits(g);
  }
}

// ---- codebook -----------------------------------------------------------

namespace {

struct CoordLaw {
  int d;
  double k;       // (d - 3) / 2, a half-integer
  double total;   // G_k(1)

  explicit CoordLaw(int d_) : d(d_), k((d_ - 3) / 2.0) { total = G(1.0); }

  // G_k(x) for 0 <= x <= 1 by the upward recurrence from k = 1/2.
  double G(double x) const {
    double w = 1.0 - x * x;
    if (w < 0) w = 0;
    double pw = std::sqrt(w);                            // (1 - x^2)^(1/2)
    double g = 0.5 * (x * pw + std::asin(x));            // G_{1/2}(x)
    for (double kk = 1.5; kk <= k + 0.25; kk += 1.0) {
      pw *= w;                                           // (1 - x^2)^kk
      g = (x * pw + 2.0 * kk * g) / (2.0 * kk + 1.0);
    }
    return g;
  }
  // P(a < X <= b) for 0 <= a <= b <= 1
  double mass(double a, double b) const { return (G(b) - G(a)) / (2.0 * total); }
  // int_a^b x f_d(x) dx
  double moment(double a, double b) const {
    double e = k + 1.0;
    return (std::pow(1.0 - a * a, e) - std::pow(1.0 - b * b, e)) / (2.0 * e) / (2.0 * total);
  }
};

}  // namespace

// Lloyd-Max levels (ascending) and midpoint thresholds, fp64.
void lloyd_max(int d, int bits_mse, std::vector<double>& centroids, std::vector<double>& thresholds) {
  const int L = 1 << bits_mse, h = L / 2;
  CoordLaw law(d);
  std::vector<double> p(h), np(h), edges(h + 1);
  for (int j = 0; j < h; ++j) p[j] = (j + 0.5) * (3.0 / h) / std::sqrt(static_cast<double>(d));
  double best = INFINITY;
  int since_best = 0;
  for (int it = 0; it < 200000; ++it) {
    edges[0] = 0.0;
    for (int j = 1; j < h; ++j) edges[j] = 0.5 * (p[j - 1] + p[j]);
    edges[h] = 1.0;
    double delta = 0.0;
    for (int j = 0; j < h; ++j) {
      np[j] = law.moment(edges[j], edges[j + 1]) / law.mass(edges[j], edges[j + 1]);
      delta = std::fmax(delta, std::fabs(np[j] - p[j]));
    }
    p.swap(np);
    if (delta < best) { best = delta; since_best = 0; } else { ++since_best; }
    if (delta <= 1e-15 * p[h - 1] || since_best >= 200) break;
  }
  centroids.resize(L);
  thresholds.resize(L - 1);
  for (int j = 0; j < h; ++j) { centroids[h + j] = p[j]; centroids[h - 1 - j] = -p[j]; }
  for (int j = 0; j < L - 1; ++j) thresholds[j] = 0.5 * (centroids[j] + centroids[j + 1]);
  thresholds[h - 1] = 0.0;
}

}  // namespace tq

// --------------------------------------------------------------------------
extern "C" tq_status tq_host_params(int d, int b, int m, uint64_t seed, float* centroids, float* thresholds,
                                    int8_t* D, uint16_t* S_bits) {
  tq_status st = tq::check_dims(d, b, m);
  if (st != TQ_OK) return st;
  d = tq::padded_dim(d);                      // parameters of the padded dimension
  if (centroids || thresholds) {
    std::vector<double> c, t;
    tq::lloyd_max(d, b - 1, c, t);
    if (centroids)
      for (size_t i = 0; i < c.size(); ++i) centroids[i] = static_cast<float>(c[i]);
    if (thresholds)
      for (size_t i = 0; i < t.size(); ++i) thresholds[i] = static_cast<float>(t[i]);
  }
  if (D) tq::rademacher(d, seed, D);
  if (S_bits) tq::gaussian_projection_half(m, d, seed, S_bits);
  return TQ_OK;
}
