// CPU oracle: the 32-element block cache formats q8_0, q4_0 and q5_0, and the
// f16 row.  TEST INFRASTRUCTURE ONLY (see oracle.h).
//
// The pages name the cache types and their cost per element ("llama.cpp für
// Geschwindigkeit und Speicher optimieren", section "KV-Cache-Präzision": f16
// 2 bytes, q8_0 1 byte, q4_0 0.5 bytes per element) and print cache sizes that
// only a 34-byte q8_0 block and an 18-byte q4_0 block per 32 elements
// reproduce ("KVSplit ...", "Vergleich der Speicherersparnis"; the llama.cpp
// issue "Eval bug: Metal fails mixed quantized KV ...", "Relevant output").
// The arithmetic inside a block is the format definition:
//   q8_0  amax = max |x_j|; d = amax / 127; q_j = round-half-away(x_j / d)
//   q4_0  m = the x_j of largest |x_j|; d = m / -8;
//         q_j = min(15, trunc(x_j * (1/d) + 8.5)); j -> low nibble of byte j,
//         j + 16 -> its high nibble
//   q5_0  q4_0 widened by one bit (-16, 16.5, 31); bit 4 of q_j is bit j of
//         a 32-bit word qh (a comment in the llama.cpp issue runs q5_0 caches;
//         no page prints its arithmetic)
// Readings where the definition is silent: the binary32 d (not its fp16
// image) quantizes; q8_0 divides each element by d (IEEE divide), q4_0 and
// q5_0 multiply by the binary32 reciprocal and add in a second rounding (no
// fused multiply-add); d == 0 gives q8_0 codes 0 and q4_0 / q5_0 codes 8 / 16;
// ties in |x_j| (also +a against -a) go to the lowest index j.
// Every quantizer widens its fp16 input to binary32 exactly and rounds once
// per operation (built with -ffp-contract=off, no fast-math).

#include <cmath>
#include <cstring>

#include "oracle_internal.h"

namespace orc {

float h2f(uint16_t h) {
  _Float16 v;
  std::memcpy(&v, &h, 2);
  return (float)v;
}

uint16_t f2h(float f) {
  _Float16 v = (_Float16)f;  // IEEE binary32 -> binary16, round to nearest even
  uint16_t h;
  std::memcpy(&h, &v, 2);
  return h;
}

int64_t code_bytes(int32_t type, int32_t d) {
  switch (type) {
    case kF16: return 2 * (int64_t)d;
    case kQ8_0: return d;
    case kQ4_0:
    case kQ5_0: return d / 2;
    case kTurbo2: return 2 * (int64_t)d / 8;
    case kTurbo3: return 3 * (int64_t)d / 8;
    case kTurbo4: return 4 * (int64_t)d / 8;
    case kTurbo3Qjl: return 3 * (int64_t)d / 8;
  }
  return 0;
}

int64_t n_scales(int32_t type, int32_t d) {
  switch (type) {
    case kF16: return 0;
    case kQ8_0:
    case kQ4_0: return d / 32;
    case kQ5_0: return 3 * (int64_t)d / 32;  // d/32 scales, then d/32 qh words as two slots each
    case kTurbo2:
    case kTurbo3:
    case kTurbo4: return 1;
    case kTurbo3Qjl: return 2;
  }
  return 0;
}

bool is_turbo(int32_t type) { return type == kTurbo2 || type == kTurbo3 || type == kTurbo4 || type == kTurbo3Qjl; }

bool valid_row(int32_t type, int32_t d) {
  if (type < 0 || type > kTurbo3Qjl || d <= 0) return false;
  if (is_turbo(type)) return pow2(d) && d >= 8 && d <= 4096;
  return d % 32 == 0;
}

// index of the element of largest |x| in a block of 32 (lowest on ties)
static int argmax_abs(const float* x) {
  int j = 0;
  for (int i = 1; i < kQK; ++i)
    if (std::fabs(x[i]) > std::fabs(x[j])) j = i;
  return j;
}

// q4_0 / q5_0 codes of one block: d = m / -half, q = min(top, trunc(fl(fl(x * fl(1/d)) + half + 0.5)))
static void quantize_offset_block(const uint16_t* xh, float half, int top, uint16_t* scale, uint8_t* codes) {
  float x[kQK];
  for (int j = 0; j < kQK; ++j) x[j] = h2f(xh[j]);
  const float m = x[argmax_abs(x)];
  const float d = m / -half;
  const float id = d != 0.0f ? 1.0f / d : 0.0f;
  const float bias = half + 0.5f;
  for (int j = 0; j < kQK; ++j) {
    const float p = x[j] * id;  // first rounding
    const float t = p + bias;   // second rounding; t >= 0.5
    const int q = (int)t;       // truncation
    codes[j] = (uint8_t)(q < top ? q : top);
  }
  *scale = f2h(d);
}

}  // namespace orc

using namespace orc;

extern "C" {

void orc_f32_to_f16(const float* x, int64_t n, uint16_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = f2h(x[i]);
}

void orc_f16_to_f64(const uint16_t* x, int64_t n, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = (double)h2f(x[i]);
}

int64_t orc_row_bytes(int32_t type, int32_t d) {
  if (!valid_row(type, d)) return 0;
  return code_bytes(type, d) + 2 * n_scales(type, d);
}

int orc_quantize_q8_0(const uint16_t* xh, int64_t n, int32_t d, uint16_t* scale, int8_t* qs) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) {
    float x[kQK];
    float amax = 0.0f;
    for (int j = 0; j < kQK; ++j) {
      x[j] = h2f(xh[b * kQK + j]);
      amax = std::fmax(amax, std::fabs(x[j]));
    }
    const float dd = amax / 127.0f;  // IEEE binary32 divide
    for (int j = 0; j < kQK; ++j) qs[b * kQK + j] = dd != 0.0f ? (int8_t)std::roundf(x[j] / dd) : (int8_t)0;
    scale[b] = f2h(dd);
  }
  return 0;
}

int orc_quantize_q4_0_codes(const uint16_t* xh, int64_t n, int32_t d, uint16_t* scale, uint8_t* codes) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) quantize_offset_block(xh + b * kQK, 8.0f, 15, scale + b, codes + b * kQK);
  return 0;
}

int orc_quantize_q5_0_codes(const uint16_t* xh, int64_t n, int32_t d, uint16_t* scale, uint8_t* codes) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) quantize_offset_block(xh + b * kQK, 16.0f, 31, scale + b, codes + b * kQK);
  return 0;
}

int orc_pack_q4_0(const uint8_t* codes, int64_t n, int32_t d, uint8_t* packed) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b)
    for (int j = 0; j < 16; ++j)
      packed[b * 16 + j] = (uint8_t)((codes[b * kQK + j] & 15) | ((codes[b * kQK + j + 16] & 15) << 4));
  return 0;
}

int orc_unpack_q4_0(const uint8_t* packed, int64_t n, int32_t d, uint8_t* codes) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b)
    for (int j = 0; j < 16; ++j) {
      codes[b * kQK + j] = packed[b * 16 + j] & 15;
      codes[b * kQK + j + 16] = packed[b * 16 + j] >> 4;
    }
  return 0;
}

int orc_pack_q5_0(const uint8_t* codes, int64_t n, int32_t d, uint8_t* qs, uint32_t* qh) {
  if (orc_pack_q4_0(codes, n, d, qs)) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) {
    uint32_t w = 0;
    for (int j = 0; j < kQK; ++j) w |= (uint32_t)((codes[b * kQK + j] >> 4) & 1) << j;
    qh[b] = w;
  }
  return 0;
}

int orc_unpack_q5_0(const uint8_t* qs, const uint32_t* qh, int64_t n, int32_t d, uint8_t* codes) {
  if (orc_unpack_q4_0(qs, n, d, codes)) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b)
    for (int j = 0; j < kQK; ++j) codes[b * kQK + j] |= (uint8_t)(((qh[b] >> j) & 1) << 4);
  return 0;
}

int orc_dequantize_q8_0(const uint16_t* scale, const int8_t* qs, int64_t n, int32_t d, double* out) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) {
    const double s = (double)h2f(scale[b]);
    for (int j = 0; j < kQK; ++j) out[b * kQK + j] = s * (double)qs[b * kQK + j];
  }
  return 0;
}

int orc_dequantize_q4_0(const uint16_t* scale, const uint8_t* packed, int64_t n, int32_t d, double* out) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) {
    const double s = (double)h2f(scale[b]);
    for (int j = 0; j < 16; ++j) {
      const uint8_t byte = packed[b * 16 + j];
      out[b * kQK + j] = s * ((double)(byte & 15) - 8.0);
      out[b * kQK + j + 16] = s * ((double)(byte >> 4) - 8.0);
    }
  }
  return 0;
}

int orc_dequantize_q5_0(const uint16_t* scale, const uint8_t* qs, const uint32_t* qh, int64_t n, int32_t d,
                        double* out) {
  if (d <= 0 || d % kQK) return -1;
  const int64_t nb = n * (d / kQK);
  for (int64_t b = 0; b < nb; ++b) {
    const double s = (double)h2f(scale[b]);
    for (int j = 0; j < 16; ++j) {
      const uint8_t byte = qs[b * 16 + j];
      const int lo = (byte & 15) | (int)(((qh[b] >> j) & 1) << 4);
      const int hi = (byte >> 4) | (int)(((qh[b] >> (j + 16)) & 1) << 4);
      out[b * kQK + j] = s * ((double)lo - 16.0);
      out[b * kQK + j + 16] = s * ((double)hi - 16.0);
    }
  }
  return 0;
}

void orc_dequantize_f16(const uint16_t* x, int64_t n, double* out) { orc_f16_to_f64(x, n, out); }

}  // extern "C"
