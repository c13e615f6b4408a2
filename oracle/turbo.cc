// CPU oracle: the turbo value-cache rows (turbo2 / turbo3 / turbo4) and the
// turbo3_qjl key rows.  TEST INFRASTRUCTURE ONLY (see oracle.h).
//
// "Benchmark TurboQuant en Apple Silicon", section "¿Qué es TurboQuant?",
// outlines the method: a random rotation by a Walsh-Hadamard transform that
// makes the coordinates Gaussian, an optimal scalar quantizer, and QJL to keep
// inner products, at 3 bits per value, about 5x smaller than fp16; its FAQ
// ("¿Qué formato TurboQuant debería usar?") puts values at 2 to 3 bits.  The
// format fixes a per-vector L2 norm, a +-1 sign vector drawn from a seed, an
// orthonormal Hadamard transform of size head_dim and a fixed Lloyd-Max
// codebook for N(0, 1/head_dim).  Everything finer is a reading:
//   1. signs: splitmix64 (Steele, Lea & Flood 2014; Vigna) seeded with the
//      64-bit seed; output i gives s_i = -1 when its top bit is set;
//   2. v = s * x (exact);
//   3. n2 = sum of fl(v_i^2) by the strided pairwise tree (stride d/2 .. 1);
//      norm = sqrtf(n2);
//   4. w = unnormalised fast Walsh-Hadamard transform of v, stages h = 1, 2,
//      .., d/2, butterfly (a, b) -> (a + b, a - b), in binary32;
//   5. g_i = fl(w_i * fl(1/norm)) (0 when norm == 0): g = sqrt(d) H D x/|x|,
//      so the unit-variance thresholds give the N(0, 1/d) codebook;
//   6. code_i = #{k : g_i > tau_k}, tau_k the binary32 midpoints of the
//      2^b-level Lloyd-Max quantizer of N(0,1);
//   7. code i in bits b*i .. b*i+b-1 of a little-endian bit stream;
//   8. stored norm fp16(min(norm, 65504)).
// Dequantization (binary64): x_hat = (norm_h / d) * s * H_un * c[code], with
// H_un built by the Sylvester recursion.
//
// turbo3_qjl (the page's third part, read after the published QJL /
// TurboQuant constructions): the 2-bit row above, then the residual in the
// rotated unit domain e = g - c32[code], its projection u = P e summed left
// to right in binary32 (P the caller's [d][d] matrix), sign bits z_i = [u_i <
// 0], and gamma = fp16(min(fl(fl(norm * sqrtf(tree sum of e_i^2)) *
// fl32(1/sqrt d)), 65504)).  Since x = (norm/d) D H_un g, sign(P e) =
// sign(S r) for r the residual of x and S = P H_un D / sqrt(d), which has
// i.i.d. N(0,1) entries when P has: this is QJL of r.  Decoded key:
// x_hat = (norm_h/d) D H_un c[code] + sqrt(pi/2)/d * gamma_h * S^T (1 - 2z).

#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "oracle_internal.h"

namespace orc {

int turbo_bits(int32_t type) {
  switch (type) {
    case kTurbo2: return 2;
    case kTurbo3: return 3;
    case kTurbo4: return 4;
    case kTurbo3Qjl: return 2;
  }
  return 0;
}

static bool turbo_dim(int32_t d) { return pow2(d) && d >= 8 && d <= 4096; }

static double phi(double x) { return std::exp(-0.5 * x * x) / std::sqrt(2.0 * M_PI); }
static double upper_tail(double x) { return 0.5 * std::erfc(x / std::sqrt(2.0)); }  // P(Z > x)

// the n-level quantizer, solved once per process and level count (the rows
// below use it many times; the iteration is the same every time)
static bool lloyd_cached(int n, std::vector<double>& lv, std::vector<double>& th) {
  static std::mutex mu;
  static std::map<int, std::pair<std::vector<double>, std::vector<double>>> solved;
  std::lock_guard<std::mutex> lock(mu);
  auto it = solved.find(n);
  if (it == solved.end()) {
    std::vector<double> l(n), t(n - 1);
    if (orc_lloyd_max_gaussian(n, l.data(), t.data()) < 0) return false;
    it = solved.emplace(n, std::make_pair(l, t)).first;
  }
  lv = it->second.first;
  th = it->second.second;
  return true;
}

// binary32 thresholds and levels of the 2^bits-level quantizer
static bool codebook_f32(int bits, std::vector<float>& levels, std::vector<float>& thresholds) {
  const int n = 1 << bits;
  std::vector<double> lv, th;
  if (!lloyd_cached(n, lv, th)) return false;
  levels.resize(n);
  thresholds.resize(n - 1);
  for (int k = 0; k < n; ++k) levels[k] = (float)lv[k];
  for (int k = 0; k < n - 1; ++k) thresholds[k] = (float)th[k];
  return true;
}

static std::vector<float> sign_vector(uint64_t seed, int32_t d) {
  std::vector<float> s(d);
  orc_signs(seed, d, s.data());
  return s;
}

// steps 1-5 of one row: the binary32 norm and g
static float rotate_row(const uint16_t* xh, int32_t d, const std::vector<float>& s, float* g) {
  std::vector<float> v(d), sq(d);
  for (int i = 0; i < d; ++i) {
    v[i] = h2f(xh[i]) * s[i];
    sq[i] = v[i] * v[i];
  }
  float n2;
  orc_tree_sum_f32(sq.data(), 1, d, &n2);
  const float norm = std::sqrt(n2);  // binary32 square root, correctly rounded
  orc_fwht_f32(v.data(), 1, d, g);
  const float r = norm > 0.0f ? 1.0f / norm : 0.0f;
  for (int i = 0; i < d; ++i) g[i] = g[i] * r;
  return norm;
}

static uint8_t code_of(float g, const std::vector<float>& tau) {
  uint8_t c = 0;
  for (float t : tau) c += g > t ? 1 : 0;
  return c;
}

static uint16_t norm_to_f16(float v) { return f2h(std::fmin(v, 65504.0f)); }

// binary64 Sylvester matrix, cached per call site by the caller
static std::vector<double> sylvester(int32_t d) {
  std::vector<double> h((size_t)d * d);
  orc_sylvester(d, h.data());
  return h;
}

// out_i = (scale_over_d * s_i) * sum_k H[i][k] y_k
static void rotate_back(const std::vector<double>& h, const std::vector<float>& s, const double* y, int32_t d,
                        double scale_over_d, double* out) {
  for (int i = 0; i < d; ++i) {
    double acc = 0.0;
    for (int k = 0; k < d; ++k) acc += h[(size_t)i * d + k] * y[k];
    out[i] = (scale_over_d * (double)s[i]) * acc;
  }
}

}  // namespace orc

using namespace orc;

extern "C" {

void orc_splitmix64(uint64_t seed, int64_t n, uint64_t* out) {
  uint64_t state = seed;
  for (int64_t i = 0; i < n; ++i) {
    state += 0x9E3779B97F4A7C15ull;  // golden-ratio increment, then two xor-shift-multiply rounds
    uint64_t z = state;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    out[i] = z ^ (z >> 31);
  }
}

int orc_signs(uint64_t seed, int32_t d, float* out) {
  if (d <= 0) return -1;
  std::vector<uint64_t> z(d);
  orc_splitmix64(seed, d, z.data());
  for (int i = 0; i < d; ++i) out[i] = (z[i] >> 63) ? -1.0f : 1.0f;
  return 0;
}

int orc_sylvester(int32_t d, double* out) {
  if (!pow2(d)) return -1;
  // H_1 = [1]; H_2n = [[H_n, H_n], [H_n, -H_n]]
  out[0] = 1.0;
  for (int n = 1; n < d; n *= 2) {
    for (int i = n - 1; i >= 0; --i)
      for (int j = n - 1; j >= 0; --j) {
        const double v = out[(size_t)i * n + j];  // H_n, stored with row stride n
        out[(size_t)i * 2 * n + j] = v;
        out[(size_t)i * 2 * n + j + n] = v;
        out[(size_t)(i + n) * 2 * n + j] = v;
        out[(size_t)(i + n) * 2 * n + j + n] = -v;
      }
  }
  return 0;
}

int orc_fwht_f32(const float* v, int64_t n, int32_t d, float* out) {
  if (!pow2(d)) return -1;
  for (int64_t r = 0; r < n; ++r) {
    float* w = out + r * d;
    if (w != v + r * d) std::memcpy(w, v + r * d, sizeof(float) * d);
    for (int h = 1; h < d; h *= 2)
      for (int i0 = 0; i0 < d; i0 += 2 * h)
        for (int i = i0; i < i0 + h; ++i) {
          const float a = w[i], b = w[i + h];
          w[i] = a + b;
          w[i + h] = a - b;
        }
  }
  return 0;
}

int orc_tree_sum_f32(const float* a, int64_t n, int32_t d, float* out) {
  if (!pow2(d)) return -1;
  std::vector<float> t(d);
  for (int64_t r = 0; r < n; ++r) {
    std::memcpy(t.data(), a + r * d, sizeof(float) * d);
    for (int h = d / 2; h >= 1; h /= 2)
      for (int i = 0; i < h; ++i) t[i] = t[i] + t[i + h];
    out[r] = t[0];
  }
  return 0;
}

int orc_lloyd_max_gaussian(int32_t n_levels, double* levels, double* thresholds) {
  // Lloyd's iteration on the positive half (the middle threshold is 0 and the
  // quantizer is mirrored exactly): thresholds are the midpoints of adjacent
  // levels, and each level is the mean of N(0,1) on its cell,
  // E[Z | a < Z < b] = (phi(a) - phi(b)) / (P(Z > a) - P(Z > b)).
  if (n_levels < 2 || n_levels % 2 || n_levels > 256) return -1;
  const int m = n_levels / 2;
  std::vector<double> pos(m), nw(m), t(m + 1);
  for (int k = 0; k < m; ++k) pos[k] = (k + 0.5) * 3.0 / m;  // start spread over [0, 3]
  const double tol = 1e-15;
  for (int it = 1; it <= 400000; ++it) {
    t[0] = 0.0;
    for (int k = 0; k + 1 < m; ++k) t[k + 1] = (pos[k] + pos[k + 1]) / 2.0;
    double delta = 0.0;
    for (int k = 0; k < m; ++k) {
      const double a = t[k];
      const bool last = k == m - 1;  // cell [t_k, +inf)
      const double pb = last ? 0.0 : phi(t[k + 1]);
      const double qb = last ? 0.0 : upper_tail(t[k + 1]);
      nw[k] = (phi(a) - pb) / (upper_tail(a) - qb);
      delta = std::fmax(delta, std::fabs(nw[k] - pos[k]));
    }
    pos = nw;
    if (delta < tol) {
      for (int k = 0; k < m; ++k) {
        levels[m - 1 - k] = -pos[k];
        levels[m + k] = pos[k];
      }
      for (int k = 0; k + 1 < n_levels; ++k) thresholds[k] = (levels[k] + levels[k + 1]) / 2.0;
      return it;
    }
  }
  return -1;
}

int orc_turbo_quantize_indices(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, int32_t bits,
                               uint16_t* norm, uint8_t* idx) {
  if (!turbo_dim(d) || bits < 2 || bits > 4) return -1;
  std::vector<float> lv, tau;
  if (!codebook_f32(bits, lv, tau)) return -1;
  const std::vector<float> s = sign_vector(seed, d);
  std::vector<float> g(d);
  for (int64_t r = 0; r < n; ++r) {
    const float nr = rotate_row(x + r * d, d, s, g.data());
    for (int i = 0; i < d; ++i) idx[r * d + i] = code_of(g[i], tau);
    norm[r] = norm_to_f16(nr);
  }
  return 0;
}

int orc_turbo_pack(const uint8_t* idx, int64_t n, int32_t d, int32_t bits, uint8_t* out) {
  if (bits < 1 || bits > 8 || ((int64_t)bits * d) % 8) return -1;
  const int64_t nb = (int64_t)bits * d / 8;
  std::memset(out, 0, (size_t)(n * nb));
  for (int64_t r = 0; r < n; ++r)
    for (int i = 0; i < d; ++i)
      for (int j = 0; j < bits; ++j) {
        const int64_t p = (int64_t)bits * i + j;
        out[r * nb + p / 8] |= (uint8_t)(((idx[r * d + i] >> j) & 1) << (p % 8));
      }
  return 0;
}

int orc_turbo_unpack(const uint8_t* codes, int64_t n, int32_t d, int32_t bits, uint8_t* idx) {
  if (bits < 1 || bits > 8 || ((int64_t)bits * d) % 8) return -1;
  const int64_t nb = (int64_t)bits * d / 8;
  for (int64_t r = 0; r < n; ++r)
    for (int i = 0; i < d; ++i) {
      uint8_t v = 0;
      for (int j = 0; j < bits; ++j) {
        const int64_t p = (int64_t)bits * i + j;
        v |= (uint8_t)(((codes[r * nb + p / 8] >> (p % 8)) & 1) << j);
      }
      idx[r * d + i] = v;
    }
  return 0;
}

int orc_turbo_quantize(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, int32_t bits, uint16_t* norm,
                       uint8_t* codes) {
  std::vector<uint8_t> idx((size_t)(n * d));
  if (orc_turbo_quantize_indices(x, n, d, seed, bits, norm, idx.data())) return -1;
  return orc_turbo_pack(idx.data(), n, d, bits, codes);
}

int orc_turbo_dequantize(const uint16_t* norm, const uint8_t* codes, int64_t n, int32_t d, uint64_t seed,
                         int32_t bits, double* out) {
  if (!turbo_dim(d) || bits < 2 || bits > 4) return -1;
  std::vector<double> lv, th;
  if (!lloyd_cached(1 << bits, lv, th)) return -1;
  const std::vector<double> h = sylvester(d);
  const std::vector<float> s = sign_vector(seed, d);
  std::vector<uint8_t> idx(d);
  std::vector<double> y(d);
  const int64_t nb = (int64_t)bits * d / 8;
  for (int64_t r = 0; r < n; ++r) {
    orc_turbo_unpack(codes + r * nb, 1, d, bits, idx.data());
    for (int k = 0; k < d; ++k) y[k] = lv[idx[k]];
    rotate_back(h, s, y.data(), d, (double)h2f(norm[r]) / d, out + r * d);
  }
  return 0;
}

int orc_qjl_residual(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, float* norm, uint8_t* idx,
                     float* e) {
  if (!turbo_dim(d)) return -1;
  std::vector<float> lv, tau;
  if (!codebook_f32(2, lv, tau)) return -1;
  const std::vector<float> s = sign_vector(seed, d);
  std::vector<float> g(d);
  for (int64_t r = 0; r < n; ++r) {
    norm[r] = rotate_row(x + r * d, d, s, g.data());
    for (int i = 0; i < d; ++i) {
      const uint8_t c = code_of(g[i], tau);
      idx[r * d + i] = c;
      e[r * d + i] = g[i] - lv[c];
    }
  }
  return 0;
}

int orc_qjl_project(const float* P, const float* e, int64_t n, int32_t d, float* u) {
  if (d <= 0) return -1;
  for (int64_t r = 0; r < n; ++r)
    for (int i = 0; i < d; ++i) {
      float acc = 0.0f;
      for (int j = 0; j < d; ++j) acc = acc + P[(size_t)i * d + j] * e[r * d + j];
      u[r * d + i] = acc;
    }
  return 0;
}

int orc_qjl_quantize_parts(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, const float* P,
                           uint16_t* norm, uint16_t* gamma, uint8_t* idx, uint8_t* z) {
  if (!turbo_dim(d) || P == nullptr) return -1;
  std::vector<float> nr(n), e((size_t)(n * d)), u((size_t)(n * d)), sq(d);
  if (orc_qjl_residual(x, n, d, seed, nr.data(), idx, e.data())) return -1;
  orc_qjl_project(P, e.data(), n, d, u.data());
  const float kappa = (float)(1.0 / std::sqrt((double)d));
  for (int64_t r = 0; r < n; ++r) {
    for (int i = 0; i < d; ++i) {
      z[r * d + i] = u[r * d + i] < 0.0f ? 1 : 0;
      sq[i] = e[r * d + i] * e[r * d + i];
    }
    float eps2;
    orc_tree_sum_f32(sq.data(), 1, d, &eps2);
    const float eps = std::sqrt(eps2);
    gamma[r] = norm_to_f16((nr[r] * eps) * kappa);
    norm[r] = norm_to_f16(nr[r]);
  }
  return 0;
}

int orc_qjl_quantize(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, const float* P, uint16_t* scales,
                     uint8_t* codes) {
  if (!turbo_dim(d) || P == nullptr) return -1;
  std::vector<uint16_t> nm(n), gm(n);
  std::vector<uint8_t> idx((size_t)(n * d)), z((size_t)(n * d));
  if (orc_qjl_quantize_parts(x, n, d, seed, P, nm.data(), gm.data(), idx.data(), z.data())) return -1;
  const int64_t cb = 3 * (int64_t)d / 8, ib = d / 4;
  for (int64_t r = 0; r < n; ++r) {
    orc_turbo_pack(idx.data() + r * d, 1, d, 2, codes + r * cb);
    orc_turbo_pack(z.data() + r * d, 1, d, 1, codes + r * cb + ib);
    scales[2 * r] = nm[r];
    scales[2 * r + 1] = gm[r];
  }
  return 0;
}

int orc_qjl_dequantize(const uint16_t* scales, const uint8_t* codes, int64_t n, int32_t d, uint64_t seed,
                       const float* P, double* out) {
  if (!turbo_dim(d) || P == nullptr) return -1;
  std::vector<double> lv, th;
  if (!lloyd_cached(4, lv, th)) return -1;
  const std::vector<double> h = sylvester(d);
  const std::vector<float> s = sign_vector(seed, d);
  const int64_t cb = 3 * (int64_t)d / 8, ib = d / 4;
  std::vector<uint8_t> idx(d), z(d);
  std::vector<double> y(d), mse(d), t(d), rot(d);
  const double c = std::sqrt(M_PI / 2.0) / d;
  for (int64_t r = 0; r < n; ++r) {
    orc_turbo_unpack(codes + r * cb, 1, d, 2, idx.data());
    orc_turbo_unpack(codes + r * cb + ib, 1, d, 1, z.data());
    for (int k = 0; k < d; ++k) y[k] = lv[idx[k]];
    rotate_back(h, s, y.data(), d, (double)h2f(scales[2 * r]) / d, mse.data());
    // S^T z~ = D H_un P^T z~ / sqrt(d), z~ = 1 - 2z
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int i = 0; i < d; ++i) acc += (1.0 - 2.0 * z[i]) * (double)P[(size_t)i * d + j];
      t[j] = acc;
    }
    const double gam = (double)h2f(scales[2 * r + 1]);
    for (int i = 0; i < d; ++i) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += h[(size_t)i * d + k] * t[k];
      const double stz = (double)s[i] * acc / std::sqrt((double)d);
      out[r * d + i] = mse[i] + c * gam * stz;
    }
  }
  return 0;
}

int orc_qjl_projection_matrix(uint64_t seed, const float* P, int32_t d, double* out) {
  if (!turbo_dim(d) || P == nullptr) return -1;
  const std::vector<double> h = sylvester(d);
  const std::vector<float> s = sign_vector(seed, d);
  const double rs = std::sqrt((double)d);
  for (int i = 0; i < d; ++i)
    for (int j = 0; j < d; ++j) {
      double acc = 0.0;
      for (int k = 0; k < d; ++k) acc += (double)P[(size_t)i * d + k] * h[(size_t)k * d + j];
      out[(size_t)i * d + j] = acc * (double)s[j] / rs;
    }
  return 0;
}

}  // extern "C"
