// Quantize-on-append row bodies: fp16 K/V rows -> f16 / q8_0 / q4_0 / turbo3
// cache rows.  Used by the append kernel and by the fused decode step.
//
// The cache types are those of "llama.cpp für Geschwindigkeit und Speicher
// optimieren" (section "KV-Cache-Präzision") and, for turbo3, of "Benchmark
// TurboQuant en Apple Silicon" (section "¿Qué es TurboQuant?": random
// Walsh-Hadamard rotation, optimal scalar quantizer, 3 bits per value).  The
// arithmetic inside a block is the format definition in include/kvq.h.
//
// Every floating-point step that decides a stored bit uses an explicitly
// rounded intrinsic (__fdiv_rn, __fmul_rn, __fadd_rn, __fsqrt_rn, __frcp_rn):
// nvcc would otherwise contract a*b+c into an FMA and change the codes.
//
// Work mapping (gtid = the thread's index in the flat work of one call; whole
// warps share a gtid range aligned to 32): q8_0 / q4_0 give each 32-element
// block to 8 consecutive threads holding 4 contiguous elements each (one 8-byte
// load per thread; the block max is a 3-step xor-shuffle reduction inside the 8
// lanes).  turbo3 gives each row to one warp, D/32 contiguous elements per lane;
// the Walsh-Hadamard butterflies run in registers for strides below D/32 and
// as xor-shuffles above.  Threads past the work still take part in the
// shuffles and then return.
#pragma once

#include "kvq_internal.h"

namespace kvq {
namespace rows {

__device__ __forceinline__ void load4_f16(const __half* src, float x[4]) {
  uint2 raw = __ldg(reinterpret_cast<const uint2*>(src));
  __half2 a = *reinterpret_cast<__half2*>(&raw.x);
  __half2 b = *reinterpret_cast<__half2*>(&raw.y);
  x[0] = __low2float(a);
  x[1] = __high2float(a);
  x[2] = __low2float(b);
  x[3] = __high2float(b);
}

// Destination row index of flat input row `row` = ((b * n_tok + t) * H + h).
__device__ __forceinline__ int64_t dst_row(const AppendParams& p, int64_t row) {
  int64_t h = row % p.H;
  int64_t t = (row / p.H) % p.n_tok;
  int64_t b = row / ((int64_t)p.H * p.n_tok);
  return (b * p.H + h) * p.dst.T + p.pos + t;
}

// q8_0: d = amax/127; q = roundf(x / d) (IEEE divide per element); d == 0 -> 0.
__device__ __forceinline__ void append_q8_0(const AppendParams& p, int64_t gtid, int64_t gend) {
  const int nb = p.D / kBlock;
  const int64_t gblk = gtid >> 3;
  const int sub = (int)(gtid & 7);
  const bool active = gtid < gend;
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) load4_f16(p.src + gblk * kBlock + sub * 4, x);
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (!active) return;
  const float d = __fdiv_rn(amax, 127.0f);
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int q = 0;
    if (d != 0.0f) q = (int)roundf(__fdiv_rn(x[i], d));
    packed |= (uint32_t)(q & 0xFF) << (8 * i);
  }
  const int64_t row = gblk / nb;
  const int blk = (int)(gblk % nb);
  const int64_t r = dst_row(p, row);
  *reinterpret_cast<uint32_t*>(p.dst.codes + r * p.dst.code_bytes + blk * kBlock + sub * 4) = packed;
  if (sub == 0) p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// q4_0: m = signed max-magnitude element (lowest index on ties); d = m / -8;
// q = min(15, trunc(fl(fl(x * fl(1/d)) + 8.5))); byte j = q_j | q_{j+16} << 4.
__device__ __forceinline__ void append_q4_0(const AppendParams& p, int64_t gtid, int64_t gend) {
  const int nb = p.D / kBlock;
  const int64_t gblk = gtid >> 3;
  const int sub = (int)(gtid & 7);
  const bool active = gtid < gend;
  float x[4] = {0.f, 0.f, 0.f, 0.f};
  if (active) load4_f16(p.src + gblk * kBlock + sub * 4, x);
  // local best: largest |x|, first index on ties
  float bm = x[0];
  int bi = sub * 4;
#pragma unroll
  for (int i = 1; i < 4; ++i)
    if (fabsf(x[i]) > fabsf(bm)) { bm = x[i]; bi = sub * 4 + i; }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) {
    const float om = __shfl_xor_sync(0xffffffffu, bm, o);
    const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
    const float a = fabsf(bm), b = fabsf(om);
    if (b > a || (b == a && oi < bi)) { bm = om; bi = oi; }
  }
  const float d = __fdiv_rn(bm, -8.0f);
  const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
  uint32_t nib = 0;  // 4 codes, one per byte
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float t = __fadd_rn(__fmul_rn(x[i], id), 8.5f);
    const int q = min(15, __float2int_rz(t));
    nib |= (uint32_t)q << (8 * i);
  }
  // lanes 0-3 of the group hold elements 0..15, lanes 4-7 elements 16..31
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, nib, 4);
  if (!active || sub >= 4) return;
  const uint32_t bytes = nib | (hi << 4);
  const int64_t row = gblk / nb;
  const int blk = (int)(gblk % nb);
  const int64_t r = dst_row(p, row);
  *reinterpret_cast<uint32_t*>(p.dst.codes + r * p.dst.code_bytes + blk * 16 + sub * 4) = bytes;
  if (sub == 0) p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// f16: copy rows, 16 bytes per thread.
__device__ __forceinline__ void append_f16(const AppendParams& p, int64_t gtid, int64_t gend) {
  const int per_row = p.D / 8;  // 16-byte chunks per row
  const int64_t i = gtid;
  if (i >= gend) return;
  const int64_t row = i / per_row;
  const int c = (int)(i % per_row);
  const uint4 v = __ldg(reinterpret_cast<const uint4*>(p.src + row * p.D) + c);
  const int64_t r = dst_row(p, row);
  reinterpret_cast<uint4*>(p.dst.codes + r * p.dst.code_bytes)[c] = v;
}

// turbo3: one warp per row, E = D/32 contiguous elements per lane.
template <int E>
__device__ __forceinline__ void append_turbo3(const AppendParams& p, int64_t gtid, int64_t gend) {
  constexpr int D = 32 * E;
  const int64_t row = gtid >> 5;
  const int lane = (int)(gtid & 31);
  if (gtid >= gend) return;  // whole warps exit together (gend is a multiple of 32)
  const __half* src = p.src + row * D + lane * E;
  float v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    const float x = __half2float(src[e]);
    v[e] = ((p.t3.sign_bits[i >> 5] >> (i & 31)) & 1u) ? -x : x;
  }
  // |v|^2 by the strided pairwise tree a[i] += a[i+h], h = D/2 ... 1
  float a[E];
#pragma unroll
  for (int e = 0; e < E; ++e) a[e] = __fmul_rn(v[e], v[e]);
#pragma unroll
  for (int h = D / 2; h >= E; h >>= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] = __fadd_rn(a[e], __shfl_xor_sync(0xffffffffu, a[e], h / E));
  }
#pragma unroll
  for (int h = E / 2; h >= 1; h >>= 1) {
#pragma unroll
    for (int e = 0; e < h; ++e) a[e] = __fadd_rn(a[e], a[e + h]);
  }
  const float norm = __fsqrt_rn(__shfl_sync(0xffffffffu, a[0], 0));
  // unnormalised fast Walsh-Hadamard transform, strides h = 1, 2, ..., D/2
#pragma unroll
  for (int h = 1; h < E; h <<= 1) {
#pragma unroll
    for (int e = 0; e < E; ++e) {
      if ((e & h) == 0) {
        const float x0 = v[e], x1 = v[e + h];
        v[e] = __fadd_rn(x0, x1);
        v[e + h] = __fsub_rn(x0, x1);
      }
    }
  }
#pragma unroll
  for (int h = E; h < D; h <<= 1) {
    const int lm = h / E;
    const bool upper = (lane & lm) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], lm);
      v[e] = upper ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
    }
  }
  const float r = norm > 0.0f ? __frcp_rn(norm) : 0.0f;
  uint32_t bits = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float g = __fmul_rn(v[e], r);
    int c = 0;
#pragma unroll
    for (int k = 0; k < 7; ++k) c += (g > p.t3.tau[k]) ? 1 : 0;
    bits |= (uint32_t)c << (3 * e);
  }
  // 8 consecutive elements -> 3 bytes; a group of 8/E lanes holds them
  constexpr int L = (E >= 8) ? 1 : 8 / E;
  uint32_t word = bits;
#pragma unroll
  for (int j = 1; j < L; ++j) {
    const uint32_t o = __shfl_down_sync(0xffffffffu, bits, j);
    word |= o << (3 * E * j);
  }
  const int64_t r_dst = dst_row(p, row);
  uint8_t* codes = p.dst.codes + r_dst * p.dst.code_bytes;
  if (E >= 8) {
#pragma unroll
    for (int g8 = 0; g8 < E / 8; ++g8) {
      const uint32_t w = (bits >> (24 * g8)) & 0xFFFFFFu;  // E == 8: one group
      const int byte0 = 3 * ((lane * E) / 8 + g8);
      codes[byte0 + 0] = (uint8_t)(w & 0xFF);
      codes[byte0 + 1] = (uint8_t)((w >> 8) & 0xFF);
      codes[byte0 + 2] = (uint8_t)((w >> 16) & 0xFF);
    }
  } else if ((lane % L) == 0) {
    const int byte0 = 3 * ((lane * E) / 8);
    codes[byte0 + 0] = (uint8_t)(word & 0xFF);
    codes[byte0 + 1] = (uint8_t)((word >> 8) & 0xFF);
    codes[byte0 + 2] = (uint8_t)((word >> 16) & 0xFF);
  }
  if (lane == 0) p.dst.scales[r_dst] = __float2half_rn(fminf(norm, 65504.0f));
}

// Thread gtid of the flat work of one call's rows of a tensor of `type`;
// threads at or past gend do no work (but still take part in shuffles).
__device__ __forceinline__ void append_any(int32_t type, const AppendParams& p, int64_t gtid, int64_t gend) {
  switch (type) {
    case KVQ_F16: append_f16(p, gtid, gend); break;
    case KVQ_Q8_0: append_q8_0(p, gtid, gend); break;
    case KVQ_Q4_0: append_q4_0(p, gtid, gend); break;
    case KVQ_TURBO3:
      switch (p.D) {
        case 32: append_turbo3<1>(p, gtid, gend); break;
        case 64: append_turbo3<2>(p, gtid, gend); break;
        case 128: append_turbo3<4>(p, gtid, gend); break;
        case 256: append_turbo3<8>(p, gtid, gend); break;
      }
      break;
  }
}

// Threads one row of a tensor of `type` and head dim d needs.
__host__ __device__ constexpr int row_threads(int32_t type, int d) {
  return type == KVQ_F16 ? d / 8 : type == KVQ_TURBO3 ? 32 : (d / kBlock) * 8;
}

}  // namespace rows
}  // namespace kvq
