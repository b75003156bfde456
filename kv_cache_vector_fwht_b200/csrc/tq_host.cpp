// Host-side set-up of a TurboQuant quantizer: the Lloyd-Max Gaussian codebook, the seeded
// rotation signs and the seeded QJL projection S_rot (tqlite README: codebook.py,
// rotation.py "Hadamard x random signs", per-layer seeds; Implementing TurboQuant (part 5):
// QJL sign(S @ residual) with a Gaussian S).
//
// Random numbers: SplitMix64 (Steele, Lea & Flood, OOPSLA 2014): draw k of a stream seeded
// with z0 is mix(z0 + (k+1) * 0x9E3779B97F4A7C15). Stream `tag` of quantizer seed s is
// seeded with s ^ (tag << 56): tag 1 rotation signs, 2 S_rot, 3 outlier-group signs,
// 4 normal-group signs. A sign is -1 when bit 63 of its draw is set. S_rot entry k
// (row-major) is Box-Muller of draws 2k, 2k+1 -- sqrt(-2 ln u1) cos(2 pi u2) with
// u1 = ((a >> 11) + 1) 2^-53, u2 = (b >> 11) 2^-53 -- rounded to fp16 (nearest even).
#include <algorithm>
#include <cmath>
#include <cstring>
#include <vector>

#include "tq_internal.h"

namespace tq {
namespace {

constexpr uint64_t kGamma = 0x9E3779B97F4A7C15ull;

uint64_t splitmix_draw(uint64_t stream_seed, uint64_t k) {
  uint64_t z = stream_seed + (k + 1) * kGamma;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

uint64_t stream_of(uint64_t seed, uint64_t tag) { return seed ^ (tag << 56); }

int storage_width(int bits) { return bits == 1 ? 1 : (bits == 2 ? 2 : 4); }

// Lloyd-Max quantizer of N(0,1) with 2^bits levels: iterate the positive half (centroid =
// conditional mean of the cell, edge = midpoint of neighbouring centroids) until the
// largest change is below 1e-14, then mirror; the middle edge is exactly 0.
void lloyd_max(int bits, double* cent, double* thr) {
  const int levels = 1 << bits, half = levels / 2;
  const double inv_sqrt2 = 1.0 / std::sqrt(2.0);
  const double inv_sqrt2pi = 1.0 / std::sqrt(2.0 * M_PI);
  auto density = [&](double x) { return std::exp(-0.5 * x * x) * inv_sqrt2pi; };
  auto tail = [&](double x) { return 0.5 * std::erfc(x * inv_sqrt2); };
  std::vector<double> c(half), e(half), nc(half);
  for (int k = 0; k < half; ++k) c[k] = (k + 0.5) * 3.0 / half;
  for (int it = 0; it < 100000; ++it) {
    e[0] = 0.0;
    for (int k = 1; k < half; ++k) e[k] = 0.5 * (c[k - 1] + c[k]);
    double worst = 0.0;
    for (int k = 0; k < half; ++k) {
      const double lo = e[k];
      double v;
      if (k + 1 < half) {
        const double hi = e[k + 1];
        v = (density(lo) - density(hi)) / (tail(lo) - tail(hi));
      } else {
        v = density(lo) / tail(lo);
      }
      nc[k] = v;
      worst = std::max(worst, std::fabs(v - c[k]));
    }
    c.swap(nc);
    if (worst < 1e-14) break;
  }
  for (int k = 0; k < half; ++k) {
    cent[half + k] = c[k];
    cent[half - 1 - k] = -c[k];
  }
  for (int k = 0; k + 1 < levels; ++k) thr[k] = 0.5 * (cent[k] + cent[k + 1]);
  thr[half - 1] = 0.0;
}

}  // namespace

uint16_t float_to_half_bits_rn(double x) {
  // Round a double to the nearest binary16, ties to even (overflow to infinity).
  uint64_t b;
  std::memcpy(&b, &x, 8);
  const uint16_t sign = static_cast<uint16_t>((b >> 48) & 0x8000);
  const double a = std::fabs(x);
  if (std::isnan(x)) return static_cast<uint16_t>(sign | 0x7E00);
  if (a >= 65520.0) return static_cast<uint16_t>(sign | 0x7C00);
  if (a < std::ldexp(1.0, -14)) {
    // subnormal: units of 2^-24, rint is ties-to-even in the default rounding mode
    const double units = std::nearbyint(std::ldexp(a, 24));
    return static_cast<uint16_t>(sign | static_cast<uint16_t>(units));
  }
  int e;
  const double m = std::frexp(a, &e);            // a = m * 2^e, m in [0.5, 1)
  double sig = std::nearbyint(std::ldexp(m, 11)); // 11 significant bits
  if (sig >= 2048.0) { sig /= 2.0; e += 1; }
  const int exp16 = e - 1 + 15;
  if (exp16 >= 31) return static_cast<uint16_t>(sign | 0x7C00);
  return static_cast<uint16_t>(sign | (exp16 << 10) | (static_cast<int>(sig) - 1024));
}

tq_status build_host_tables(int d, int bits, int mode, uint64_t seed, const int32_t* outliers,
                            int n_outlier, HostTables* t, tq_key_layout_t* lay) {
  if (!t || !lay) return TQ_EINVAL;
  if (d < 2 || (d & (d - 1))) return TQ_EINVAL;
  if (d != kD) return TQ_EUNSUPPORTED;
  std::memset(t, 0, sizeof(*t));
  std::memset(lay, 0, sizeof(*lay));
  lay->d = d;
  lay->bits = bits;
  lay->mode = mode;
  if (mode == TQ_MODE_MSE || mode == TQ_MODE_PROD) {
    const int mse_bits = mode == TQ_MODE_MSE ? bits : bits - 1;
    if (mode == TQ_MODE_MSE && (bits < 1 || bits > 4)) return TQ_EUNSUPPORTED;
    if (mode == TQ_MODE_PROD && (bits < 2 || bits > 4)) return TQ_EUNSUPPORTED;
    if (outliers || n_outlier) return TQ_EINVAL;
    lloyd_max(mse_bits, t->cent[0], t->thr[0]);
    const uint64_t ss = stream_of(seed, 1);
    for (int j = 0; j < d; ++j) {
      t->signs[j] = (splitmix_draw(ss, j) >> 63) ? -1 : 1;
      t->chan[j] = j;
    }
    lay->idx_bytes = d * storage_width(mse_bits) / 8;
    lay->n_norms = mode == TQ_MODE_PROD ? 2 : 1;
    lay->sign_bytes = mode == TQ_MODE_PROD ? d / 8 : 0;
    if (mode == TQ_MODE_PROD) {
      const uint64_t gs = stream_of(seed, 2);
      const double two_pi = 2.0 * M_PI;
      const double unit = std::ldexp(1.0, -53);
      for (int k = 0; k < d * d; ++k) {
        const uint64_t a = splitmix_draw(gs, 2 * static_cast<uint64_t>(k));
        const uint64_t b = splitmix_draw(gs, 2 * static_cast<uint64_t>(k) + 1);
        const double u1 = static_cast<double>((a >> 11) + 1) * unit;
        const double u2 = static_cast<double>(b >> 11) * unit;
        const double z = std::sqrt(-2.0 * std::log(u1)) * std::cos(two_pi * u2);
        t->s_rot[k] = float_to_half_bits_rn(z);
      }
    }
  } else if (mode == TQ_MODE_GROUPED) {
    if (bits < 1 || bits > 3) return TQ_EUNSUPPORTED;
    if (!outliers || n_outlier != 32) return TQ_EINVAL;
    std::vector<int32_t> o(outliers, outliers + 32);
    std::sort(o.begin(), o.end());
    for (int i = 0; i < 32; ++i) {
      if (o[i] < 0 || o[i] >= d || (i && o[i] == o[i - 1])) return TQ_EINVAL;
    }
    std::vector<char> is_out(d, 0);
    for (int c : o) is_out[c] = 1;
    int n = 0;
    for (int i = 0; i < 32; ++i) t->chan[n++] = o[i];
    for (int c = 0; c < d; ++c)
      if (!is_out[c]) t->chan[n++] = c;
    lloyd_max(bits + 1, t->cent[0], t->thr[0]);
    lloyd_max(bits, t->cent[1], t->thr[1]);
    const uint64_t so = stream_of(seed, 3), sn = stream_of(seed, 4);
    for (int j = 0; j < 32; ++j) t->signs[j] = (splitmix_draw(so, j) >> 63) ? -1 : 1;
    for (int j = 0; j < 96; ++j) t->signs[32 + j] = (splitmix_draw(sn, j) >> 63) ? -1 : 1;
    lay->idx_bytes = (32 * storage_width(bits + 1) + 96 * storage_width(bits)) / 8;
    lay->n_norms = 2;
    lay->sign_bytes = 0;
  } else {
    return TQ_EINVAL;
  }
  lay->bytes_per_key = lay->idx_bytes + lay->sign_bytes + 2 * lay->n_norms;
  return TQ_OK;
}

}  // namespace tq
