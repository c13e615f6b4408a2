// CPU oracle: decode attention over a dequantized KV cache, in binary64.
// TEST INFRASTRUCTURE ONLY (see oracle.h).
//
// "llama.cpp für Geschwindigkeit und Speicher optimieren", section "Flash
// Attention": flash attention computes attention tile by tile in on-chip
// memory and is mathematically the same as standard attention, not an
// approximation.  A split-KV decode (partials per context slice, then a
// combine) therefore reaches exactly the plain definition in exact
// arithmetic, and the oracle is that definition:
//   s_t = scale * <q_h, k_hat_{g,t}>,  M = max_t s_t,  p_t = exp(s_t - M),
//   o_h = sum_t p_t v_hat_{g,t} / sum_t p_t,
// for every batch row b and query head h, with g = floor(h / G) the KV head
// of h's group, G = n_q / n_kv (consecutive grouping: the pages do not say
// which grouping; this is the common one), over every cached row, no mask.

#include <atomic>
#include <cmath>
#include <thread>
#include <vector>

#include "oracle_internal.h"

namespace orc {

// o = sum_t p_t v_t / sum_t p_t for one query row against T rows
static void attend(const double* q, const double* k, const double* v, int64_t T, int32_t D, double scale,
                   double* out, std::vector<double>& s) {
  s.resize((size_t)T);
  double M = -INFINITY;
  for (int64_t t = 0; t < T; ++t) {
    double dot = 0.0;
    for (int j = 0; j < D; ++j) dot += q[j] * k[t * D + j];
    s[t] = scale * dot;
    M = std::fmax(M, s[t]);
  }
  double l = 0.0;
  for (int j = 0; j < D; ++j) out[j] = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    const double p = std::exp(s[t] - M);
    l += p;
    for (int j = 0; j < D; ++j) out[j] += p * v[t * D + j];
  }
  for (int j = 0; j < D; ++j) out[j] /= l;
}

// runs work(i) for i = 0 .. n-1 over `threads` threads (items claimed in order)
template <class F>
static void parallel_for(int64_t n, int32_t threads, F work) {
  if (threads <= 0) threads = (int32_t)std::max(1u, std::thread::hardware_concurrency());
  if (threads == 1 || n <= 1) {
    for (int64_t i = 0; i < n; ++i) work(i);
    return;
  }
  std::atomic<int64_t> next{0};
  std::vector<std::thread> pool;
  const int64_t nt = std::min<int64_t>(threads, n);
  for (int64_t t = 0; t < nt; ++t)
    pool.emplace_back([&] {
      for (int64_t i = next++; i < n; i = next++) work(i);
    });
  for (auto& th : pool) th.join();
}

// n consecutive stored rows (codes + fp16 scale slots of their format) -> binary64 values
static int dequantize_rows(int32_t type, const uint8_t* codes, const uint16_t* sc, int64_t n, int32_t D,
                           uint64_t seed, const float* P, double* out) {
  switch (type) {
    case kF16: orc_dequantize_f16(reinterpret_cast<const uint16_t*>(codes), n * D, out); return 0;
    case kQ8_0: return orc_dequantize_q8_0(sc, reinterpret_cast<const int8_t*>(codes), n, D, out);
    case kQ4_0: return orc_dequantize_q4_0(sc, codes, n, D, out);
    case kQ5_0: {
      // a row's scale slots: the d/32 block scales, then each block's qh word
      // as two fp16 slots, low half first
      const int nb = D / kQK;
      std::vector<uint32_t> qh(nb);
      for (int64_t r = 0; r < n; ++r) {
        const uint16_t* s = sc + r * 3 * nb;
        for (int i = 0; i < nb; ++i) qh[i] = (uint32_t)s[nb + 2 * i] | ((uint32_t)s[nb + 2 * i + 1] << 16);
        if (orc_dequantize_q5_0(s, codes + r * (D / 2), qh.data(), 1, D, out + r * D)) return -1;
      }
      return 0;
    }
    case kTurbo2:
    case kTurbo3:
    case kTurbo4: return orc_turbo_dequantize(sc, codes, n, D, seed, turbo_bits(type), out);
    case kTurbo3Qjl: return orc_qjl_dequantize(sc, codes, n, D, seed, P, out);
  }
  return -1;
}

}  // namespace orc

using namespace orc;

extern "C" {

int orc_decode_attention(const double* q, const double* k, const double* v, int32_t B, int32_t n_q, int32_t n_kv,
                         int64_t T, int32_t D, double scale, double* out, int32_t n_threads) {
  if (B <= 0 || n_kv <= 0 || n_q % n_kv || T <= 0 || D <= 0) return -1;
  const int32_t G = n_q / n_kv;
  parallel_for((int64_t)B * n_q, n_threads, [&](int64_t i) {
    std::vector<double> s;
    const int64_t b = i / n_q, h = i % n_q, g = h / G;
    const double* kb = k + (b * n_kv + g) * T * D;
    const double* vb = v + (b * n_kv + g) * T * D;
    attend(q + i * D, kb, vb, T, D, scale, out + i * D, s);
  });
  return 0;
}

int orc_softmax_weights(const double* q, const double* k, int64_t T, int32_t D, double scale, double* w) {
  if (T <= 0 || D <= 0) return -1;
  double M = -INFINITY;
  for (int64_t t = 0; t < T; ++t) {
    double dot = 0.0;
    for (int j = 0; j < D; ++j) dot += q[j] * k[t * D + j];
    w[t] = scale * dot;
    M = std::fmax(M, w[t]);
  }
  double l = 0.0;
  for (int64_t t = 0; t < T; ++t) {
    w[t] = std::exp(w[t] - M);
    l += w[t];
  }
  for (int64_t t = 0; t < T; ++t) w[t] /= l;
  return 0;
}

int orc_partials(const double* q, const double* k, const double* v, int32_t D, double scale,
                 const int64_t* bounds, int32_t n_slices, double* m, double* l, double* acc) {
  if (n_slices <= 0 || D <= 0) return -1;
  for (int s = 0; s < n_slices; ++s) {
    const int64_t a = bounds[s], e = bounds[s + 1];
    if (e <= a) return -1;
    std::vector<double> sc((size_t)(e - a));
    double M = -INFINITY;
    for (int64_t t = a; t < e; ++t) {
      double dot = 0.0;
      for (int j = 0; j < D; ++j) dot += q[j] * k[t * D + j];
      sc[t - a] = scale * dot;
      M = std::fmax(M, sc[t - a]);
    }
    double ls = 0.0;
    double* as = acc + (int64_t)s * D;
    for (int j = 0; j < D; ++j) as[j] = 0.0;
    for (int64_t t = a; t < e; ++t) {
      const double p = std::exp(sc[t - a] - M);
      ls += p;
      for (int j = 0; j < D; ++j) as[j] += p * v[t * D + j];
    }
    m[s] = M;
    l[s] = ls;
  }
  return 0;
}

int orc_combine(const double* m, const double* l, const double* acc, int32_t n_slices, int32_t D, double* out) {
  if (n_slices <= 0 || D <= 0) return -1;
  double M = -INFINITY;
  for (int s = 0; s < n_slices; ++s) M = std::fmax(M, m[s]);
  double den = 0.0;
  for (int j = 0; j < D; ++j) out[j] = 0.0;
  for (int s = 0; s < n_slices; ++s) {
    const double w = std::exp(m[s] - M);
    den += w * l[s];
    for (int j = 0; j < D; ++j) out[j] += w * acc[(int64_t)s * D + j];
  }
  for (int j = 0; j < D; ++j) out[j] /= den;
  return 0;
}

int orc_decode_cache(int32_t k_type, int32_t v_type, int32_t B, int32_t n_q, int32_t n_kv, int64_t T, int32_t D,
                     const uint8_t* k_codes, const uint16_t* k_scales, const uint8_t* v_codes,
                     const uint16_t* v_scales, uint64_t seed, const float* P, const uint16_t* q, double scale,
                     double* out, int32_t n_threads) {
  if (!valid_row(k_type, D) || !valid_row(v_type, D) || B <= 0 || n_kv <= 0 || n_q % n_kv || T <= 0) return -1;
  if (k_type == kTurbo3Qjl && P == nullptr) return -1;
  const int64_t kcb = code_bytes(k_type, D), kns = n_scales(k_type, D);
  const int64_t vcb = code_bytes(v_type, D), vns = n_scales(v_type, D);
  const int32_t G = n_q / n_kv;
  const int64_t chunk = 256;  // rows per dequantization work item
  const int64_t n_chunks = (T + chunk - 1) / chunk;
  std::vector<double> kh((size_t)(n_kv * T * D)), vh((size_t)(n_kv * T * D)), qd((size_t)n_q * D);
  std::atomic<int> bad{0};
  for (int32_t b = 0; b < B; ++b) {
    parallel_for(n_kv * n_chunks, n_threads, [&](int64_t i) {
      const int64_t g = i / n_chunks, t0 = (i % n_chunks) * chunk, t1 = std::min(T, t0 + chunk);
      const int64_t plane = (int64_t)b * n_kv + g;
      const int64_t row = plane * T + t0;
      if (dequantize_rows(k_type, k_codes + row * kcb, k_scales + row * kns, t1 - t0, D, seed, P,
                          kh.data() + (g * T + t0) * D) ||
          dequantize_rows(v_type, v_codes + row * vcb, v_scales + row * vns, t1 - t0, D, seed, P,
                          vh.data() + (g * T + t0) * D))
        bad = 1;
    });
    orc_f16_to_f64(q + (int64_t)b * n_q * D, (int64_t)n_q * D, qd.data());
    parallel_for(n_q, n_threads, [&](int64_t h) {
      std::vector<double> s;
      const int64_t g = h / G;
      attend(qd.data() + h * D, kh.data() + g * T * D, vh.data() + g * T * D, T, D, scale,
             out + ((int64_t)b * n_q + h) * D, s);
    });
  }
  return bad ? -1 : 0;
}

int32_t orc_hardware_threads(void) { return (int32_t)std::max(1u, std::thread::hardware_concurrency()); }

}  // extern "C"
