// The library's own binary16 centroid table: the 16-level Lloyd-Max quantiser of N(0,1)
// (the compact tier's fixed 16-entry table, "Context beyond VRAM", section "What I
// built"), solved on the host when the library loads.
//
// Method (J. Max, "Quantizing for Minimum Distortion", 1960, the sequential
// construction): by symmetry the middle boundary is 0.  Guess the first positive level
// y_8.  Each next boundary x_{j+1} is the point where the mean of N(0,1) over
// (x_j, x_{j+1}) equals y_j (found by bisection), and the next level is its mirror
// y_{j+1} = 2 x_{j+1} - y_j (the midpoint condition).  The guess is right when the last
// level equals the mean of the upper tail beyond x_15; bisection on y_8 finds it.  The
// positive levels are mirrored, and every level is rounded to binary16 with round to
// nearest even.
#include <cmath>
#include <cstdint>
#include <mutex>

#include "akv_internal.cuh"

namespace akv {
namespace {

using real = long double;

real upper_tail(real x) { return 0.5L * std::erfc(x / std::sqrt(2.0L)); }
real pdf(real x) { return std::exp(-0.5L * x * x) / std::sqrt(2.0L * 3.141592653589793238462643383279502884L); }

// mean of N(0,1) over (a, b), 0 <= a < b <= inf
real cell_mean(real a, real b) {
  const real mass = upper_tail(a) - (std::isinf(b) ? 0.0L : upper_tail(b));
  return (pdf(a) - (std::isinf(b) ? 0.0L : pdf(b))) / mass;
}

// Walk the construction from level y8.  Returns +1 when the guess is too large (a cell
// cannot reach its level, or the last level exceeds the tail mean), -1 when too small.
int walk(real y8, real* levels) {
  real x = 0.0L, y = y8;
  for (int j = 0; j < 8; ++j) {
    levels[j] = y;
    if (j == 7) return (y > cell_mean(x, INFINITY)) ? 1 : -1;
    if (y >= cell_mean(x, INFINITY)) return 1;
    real lo = x, hi = x + 1.0L;
    while (cell_mean(x, hi) < y) hi = x + 2.0L * (hi - x);
    for (int it = 0; it < 200; ++it) {
      real mid = 0.5L * (lo + hi);
      if (cell_mean(x, mid) < y) lo = mid; else hi = mid;
    }
    const real xn = 0.5L * (lo + hi);
    y = 2.0L * xn - y;
    x = xn;
  }
  return 1;
}

uint16_t to_binary16_rne(double v) {
  // finite positive or negative v, |v| within the binary16 normal range here
  uint16_t sign = 0;
  if (std::signbit(v)) { sign = 0x8000; v = -v; }
  if (v == 0.0) return sign;
  int e;
  std::frexp(v, &e);          // v = m * 2^e, m in [0.5, 1)
  int E = e - 1;              // v = 1.f * 2^E
  if (E < -14) {              // subnormal: multiples of 2^-24
    double q = std::nearbyint(std::ldexp(v, 24));
    return (uint16_t)(sign | (uint16_t)q);
  }
  double q = std::nearbyint(std::ldexp(v, 10 - E));  // in [1024, 2048]
  if (q == 2048.0) { q = 1024.0; ++E; }
  if (E > 15) return (uint16_t)(sign | 0x7c00);
  return (uint16_t)(sign | (uint16_t)((E + 15) << 10) | (uint16_t)(q - 1024.0));
}

double binary16_value(uint16_t h) {
  const int e = (h >> 10) & 0x1f, f = h & 0x3ff;
  double v = (e == 0) ? std::ldexp((double)f, -24) : std::ldexp((double)(1024 + f), e - 25);
  return (h & 0x8000) ? -v : v;
}

struct Table {
  uint16_t f16[16];
  double bound[15];
};

Table solve() {
  real lo = 0.01L, hi = 0.5L, levels[8];
  for (int it = 0; it < 200; ++it) {
    real mid = 0.5L * (lo + hi);
    if (walk(mid, levels) > 0) hi = mid; else lo = mid;
  }
  walk(0.5L * (lo + hi), levels);
  Table t;
  for (int j = 0; j < 8; ++j) {
    const uint16_t h = to_binary16_rne((double)levels[j]);
    t.f16[8 + j] = h;
    t.f16[7 - j] = (uint16_t)(h | 0x8000);
  }
  for (int j = 0; j < 15; ++j) t.bound[j] = (binary16_value(t.f16[j]) + binary16_value(t.f16[j + 1])) / 2.0;
  return t;
}

const Table& table() {
  static std::once_flag once;
  static Table t;
  std::call_once(once, [] { t = solve(); });
  return t;
}

}  // namespace

const uint16_t* centroid_table_f16() { return table().f16; }
const double* centroid_boundaries() { return table().bound; }

}  // namespace akv
