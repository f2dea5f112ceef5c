// NF4 level table ("QLoRA: Efficient Finetuning of Quantized LLMs", crackai.dev,
// How It Works 1: levels at quantiles of the normal distribution, each bin holding
// equal probability mass; "QLoRA", ozercemkelahmet.com, How it works -- Why
// NormalFloat).  Asymmetric halves with one exact zero, normalised to [-1, 1]:
//   positive: Phi^-1(p) at 9 evenly spaced p in [0.5, P_MAX], first dropped;
//   negative: -Phi^-1(p) at 8 evenly spaced p in [0.5, P_MAX], first dropped;
//   P_MAX = ((1 - 1/32) + (1 - 1/30)) / 2; all divided by Phi^-1(P_MAX).
#include "nf4_table.hpp"

#include <algorithm>
#include <cmath>
#include <limits>

namespace qlora {
namespace {

double phi(double z) { return 0.5 * std::erfc(-z / std::sqrt(2.0)); }

// Inverse standard normal CDF: Newton's method on Phi(x) - p, kept inside a
// shrinking bracket (bisection step whenever Newton would leave it).
double phi_inv(double p) {
  double lo = -40.0, hi = 40.0, x = 0.0;
  const double inv_sqrt_2pi = 0.3989422804014327;
  for (int it = 0; it < 400; ++it) {
    const double f = phi(x) - p;
    if (f < 0) lo = x; else hi = x;
    const double d = inv_sqrt_2pi * std::exp(-0.5 * x * x);
    double xn = (d > 0) ? x - f / d : 0.5 * (lo + hi);
    if (!(xn > lo && xn < hi)) xn = 0.5 * (lo + hi);
    if (xn == x || hi - lo <= 0) break;
    x = xn;
  }
  return x;
}

float round_down_f32(double m) {
  float t = static_cast<float>(m);
  if (static_cast<double>(t) > m) t = std::nextafter(t, -std::numeric_limits<float>::infinity());
  return t;
}

Nf4Tables build() {
  Nf4Tables T{};
  const double p_max = 0.5 * ((1.0 - 1.0 / 32.0) + (1.0 - 1.0 / 30.0));
  const double zmax = phi_inv(p_max);
  double v[16];
  int k = 0;
  for (int i = 7; i >= 1; --i) v[k++] = -phi_inv(0.5 + i * ((p_max - 0.5) / 7.0));
  v[k++] = 0.0;
  for (int i = 1; i <= 8; ++i) v[k++] = (i == 8) ? zmax : phi_inv(0.5 + i * ((p_max - 0.5) / 8.0));
  v[0] = -zmax;
  std::sort(v, v + 16);
  bool ok = true;
  for (int i = 0; i < 16; ++i) T.levels[i] = static_cast<float>(v[i] / zmax);
  T.levels[0] = -1.0f;
  T.levels[7] = 0.0f;
  T.levels[15] = 1.0f;
  for (int i = 0; i + 1 < 16; ++i) {
    if (!(T.levels[i] < T.levels[i + 1])) ok = false;
    // exact midpoint of two floats, rounded toward -inf: "xn > T" is then the
    // same decision as "xn is strictly closer to the upper level".
    const double mid = 0.5 * (static_cast<double>(T.levels[i]) + static_cast<double>(T.levels[i + 1]));
    T.thresholds[i] = round_down_f32(mid);
  }
  // Bin table for the quantizer: bin j (stored at (j - 32) mod 128) covers
  // 32*xn in [j-32.5, j-31.5].
  for (int j = 0; j < kQuantBins; ++j) {
    T.bins[j].t = 2.0f;
    T.bins[j].c = 0;
  }
  for (int j = 0; j <= 64; ++j) {
    const double lo = (j - 32 - 0.5) / 32.0, hi = (j - 32 + 0.5) / 32.0;
    int below = 0, inside = 0;
    float tin = 2.0f;
    for (int i = 0; i < 15; ++i) {
      const double t = T.thresholds[i];
      if (t < lo) ++below;
      else if (t <= hi) {
        ++inside;
        tin = T.thresholds[i];
        if (t == lo || t == hi) ok = false;  // never sits on a bin edge
      }
    }
    if (inside > 1) ok = false;
    const int slot = (j - 32) & (kQuantBins - 1);
    T.bins[slot].t = tin;
    T.bins[slot].c = below;
  }
  for (int k = 0; k < 128; ++k) {
    volatile float m = 1.0f + static_cast<float>(k) / 128.0f;
    T.rcp[k] = 1.0f / m;  // IEEE single division: RN32(1/m)
  }
  T.ok = ok;
  return T;
}

}  // namespace

const Nf4Tables &nf4_tables() {
  static const Nf4Tables t = build();
  return t;
}

}  // namespace qlora
