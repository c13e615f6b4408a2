// Helpers shared by the oracle's translation units.  TEST INFRASTRUCTURE ONLY
// (see oracle.h).
#pragma once

#include <cstdint>

#include "oracle.h"

namespace orc {

constexpr int kQK = 32;  // elements per block of q8_0 / q4_0 / q5_0

// type codes, as in oracle.h
constexpr int32_t kF16 = 0, kQ8_0 = 1, kQ4_0 = 2, kTurbo3 = 3, kTurbo2 = 4, kTurbo4 = 5, kQ5_0 = 6,
                  kTurbo3Qjl = 7;

inline bool pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

float h2f(uint16_t h);   // binary16 bits -> binary32 (exact)
uint16_t f2h(float f);   // binary32 -> binary16 bits, round to nearest even

int64_t code_bytes(int32_t type, int32_t d);  // code bytes of one row
int64_t n_scales(int32_t type, int32_t d);    // fp16 slots of one row's scale part
bool is_turbo(int32_t type);
bool valid_row(int32_t type, int32_t d);
int turbo_bits(int32_t type);                 // 2, 3, 4 (turbo3_qjl: its 2-bit stage)

}  // namespace orc
