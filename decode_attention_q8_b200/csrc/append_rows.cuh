// Quantize-on-append row bodies: fp16 K/V rows -> f16 / q8_0 / q4_0 / q5_0 /
// turbo cache rows.  Used by the append kernel and by the fused decode step.
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
// lanes).  Loading (load_raw) and quantizing (finish) are separate steps, so a
// thread can have several loads in flight.  A turbo row takes one warp, D/32
// contiguous elements per lane; in the bulk append the turbo types other than
// turbo3_qjl take D/16 lanes, 16 contiguous elements each (append_turbo_wide).  The
// Walsh-Hadamard butterflies run in registers for strides below the elements
// per lane and as xor-shuffles above.  Threads past the work still take part in
// the shuffles and then return.
#pragma once

#include "kvq_internal.h"

namespace kvq {
namespace rows {

// The fp16 input bytes thread gtid of a call's flat work needs (zero past
// gend): q8_0 / q4_0 4 elements (8 bytes), f16 8 elements (16 bytes), turbo3
// D/32 elements.  Work item gtid's elements start at element 4, 8 or D/32 times
// gtid of the call's [rows][D] input.
template <int TYPE, int E>
__device__ __forceinline__ uint4 load_raw(const AppendParams& p, int64_t gtid, int64_t gend) {
  uint4 r = make_uint4(0u, 0u, 0u, 0u);
  if (gtid >= gend) return r;
  if constexpr (TYPE == KVQ_Q8_0 || TYPE == KVQ_Q4_0 || TYPE == KVQ_Q5_0) {
    const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.src + gtid * 4));
    r.x = v.x;
    r.y = v.y;
  } else if constexpr (TYPE == KVQ_F16) {
    r = __ldg(reinterpret_cast<const uint4*>(p.src + gtid * 8));
  } else {  // turbo types
    if constexpr (E == 8) {
      r = __ldg(reinterpret_cast<const uint4*>(p.src + gtid * 8));
    } else if constexpr (E == 4) {
      const uint2 v = __ldg(reinterpret_cast<const uint2*>(p.src + gtid * 4));
      r.x = v.x;
      r.y = v.y;
    } else if constexpr (E == 2) {
      r.x = __ldg(reinterpret_cast<const unsigned int*>(p.src + gtid * 2));
    } else {
      r.x = __ldg(reinterpret_cast<const unsigned short*>(p.src + gtid));
    }
  }
  return r;
}

// Packed binary32 pairs (low word: the first element), each lane rounded to
// nearest.  Used only where a stored bit does not hang on the last rounding
// step: q8_0's tie test falls back to the exact divide near a tie.  (q4_0's
// truncation, packed the same way, changed a nibble against the oracle, so it
// keeps the scalar intrinsics.)
__device__ __forceinline__ unsigned long long pack_f32x2(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void unpack_f32x2(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long sub_f32x2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long add_f32x2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long mul_f32x2(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ float raw_elem(const uint4& r, int i) {  // fp16 element i of r as float
  const uint32_t w = i < 2 ? r.x : i < 4 ? r.y : i < 6 ? r.z : r.w;
  const uint16_t h = (uint16_t)(w >> (16 * (i & 1)));
  return __half2float(__ushort_as_half(h));
}

// Destination row index of flat input row `row` = ((b * n_tok + t) * H + h),
// or -1 when batch row b's length (per-sequence lengths) is out of range or
// its page id (paged pool) is not a page of the pool.
// 32-bit division when the call's rows fit (the 64-bit one is a long routine).
__device__ __forceinline__ int64_t dst_row(const AppendParams& p, int64_t row) {
  int64_t h, t, b;
  if ((int64_t)p.B * p.n_tok * p.H <= 0xffffffffll) {
    const uint64_t r32 = (uint64_t)(uint32_t)row;
    const uint64_t bt = p.h_mul ? __umul64hi(r32, p.h_mul) : r32;
    h = (int64_t)(r32 - bt * (uint64_t)p.H);
    b = (int64_t)(p.t_mul ? __umul64hi(bt, p.t_mul) : bt);
    t = (int64_t)bt - b * p.n_tok;
  } else {
    h = row % p.H;
    t = (row / p.H) % p.n_tok;
    b = row / ((int64_t)p.H * p.n_tok);
  }
  int64_t pos = p.pos;
  if (p.lens != nullptr) {
    const int64_t len = p.lens[b];
    if (len < p.n_tok || len > p.len_max) return -1;
    pos = len - p.n_tok;
  }
  const int64_t lr = pos + t;  // logical row of sequence b
  if (p.block_table != nullptr) {
    const int64_t pg = p.block_table[b * p.max_pages + (lr >> p.log2_page)];
    if (pg < 0 || pg >= p.n_pages) return -1;
    return (pg * p.H + h) * p.dst.T + (lr & ((1ll << p.log2_page) - 1));
  }
  return (b * p.H + h) * p.dst.T + lr;
}

// log2 of the 32-element blocks per row (head_dim is 32 times a power of two)
__device__ __forceinline__ int log2_blocks(const AppendParams& p) { return 31 - __clz(p.D / kBlock); }

// q8_0: d = amax/127; q = roundf(x / d) (IEEE divide per element); d == 0 -> 0.
__device__ __forceinline__ void append_q8_0(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw) {
  const int nb = p.D / kBlock;
  const int64_t gblk = gtid >> 3;
  const int sub = (int)(gtid & 7);
  const bool active = gtid < gend;
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = raw_elem(raw, i);  // zeros past gend
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  if (!active) return;
  const float d = __fdiv_rn(amax, 127.0f);
  // q = roundf of the IEEE quotient x / d.  x * fl(1/d) is within 2^-15 of that
  // quotient (|x / d| <= 127, two roundings of 2^-24 relative), so it rounds to
  // the same integer unless it lies within 2^-14 of a half-integer; only then
  // is the exact divide taken.  Away from a tie round-to-nearest is roundf.
  const float rd = d != 0.0f ? __frcp_rn(d) : 0.0f;
  uint32_t packed = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    int q = 0;
    if (d != 0.0f) {
      const float t = __fmul_rn(x[i], rd);
      const float a = fabsf(t);
      if (fabsf(a - floorf(a) - 0.5f) > 6.103515625e-05f)  // 2^-14
        q = __float2int_rn(t);
      else
        q = (int)roundf(__fdiv_rn(x[i], d));
    }
    packed |= (uint32_t)(q & 0xFF) << (8 * i);
  }
  const int64_t row = gblk >> log2_blocks(p);
  const int blk = (int)(gblk & (nb - 1));
  const int64_t r = dst_row(p, row);
  if (r < 0) return;
  *reinterpret_cast<uint32_t*>(p.dst.codes + r * p.dst.code_bytes + blk * kBlock + sub * 4) = packed;
  if (sub == 0) p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// q4_0: m = signed max-magnitude element (lowest index on ties); d = m / -8;
// q = min(15, trunc(fl(fl(x * fl(1/d)) + 8.5))); byte j = q_j | q_{j+16} << 4.
__device__ __forceinline__ void append_q4_0(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw) {
  const int nb = p.D / kBlock;
  const int64_t gblk = gtid >> 3;
  const int sub = (int)(gtid & 7);
  const bool active = gtid < gend;
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = raw_elem(raw, i);  // zeros past gend
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
  const int64_t row = gblk >> log2_blocks(p);
  const int blk = (int)(gblk & (nb - 1));
  const int64_t r = dst_row(p, row);
  if (r < 0) return;
  *reinterpret_cast<uint32_t*>(p.dst.codes + r * p.dst.code_bytes + blk * 16 + sub * 4) = bytes;
  if (sub == 0) p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// q5_0: q4_0 widened by one bit: d = m / -16; q = min(31, trunc(fl(fl(x * fl(1/d))
// + 16.5))); the low nibbles as q4_0's, bit 4 of element j in bit j of qh, which
// sits in the scale plane after the row's block scales (two fp16 slots).
__device__ __forceinline__ void append_q5_0(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw) {
  const int nb = p.D / kBlock;
  const int64_t gblk = gtid >> 3;
  const int sub = (int)(gtid & 7);
  const bool active = gtid < gend;
  float x[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) x[i] = raw_elem(raw, i);  // zeros past gend
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
  const float d = __fdiv_rn(bm, -16.0f);
  const float id = (d != 0.0f) ? __frcp_rn(d) : 0.0f;
  uint32_t nib = 0, h = 0;  // 4 low nibbles, one per byte; their fifth bits
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float t = __fadd_rn(__fmul_rn(x[i], id), 16.5f);
    const int q = min(31, __float2int_rz(t));
    nib |= (uint32_t)(q & 15) << (8 * i);
    h |= (uint32_t)(q >> 4) << i;
  }
  const uint32_t hi = __shfl_xor_sync(0xffffffffu, nib, 4);
  uint32_t qh = h << (4 * sub);  // elements 4 sub .. 4 sub + 3
#pragma unroll
  for (int o = 1; o < 8; o <<= 1) qh |= __shfl_xor_sync(0xffffffffu, qh, o);
  if (!active || sub >= 4) return;
  const uint32_t bytes = nib | (hi << 4);
  const int64_t row = gblk >> log2_blocks(p);
  const int blk = (int)(gblk & (nb - 1));
  const int64_t r = dst_row(p, row);
  if (r < 0) return;
  *reinterpret_cast<uint32_t*>(p.dst.codes + r * p.dst.code_bytes + blk * 16 + sub * 4) = bytes;
  if (sub == 0) {
    __half* sc = p.dst.scales + r * p.dst.n_scales;
    sc[blk] = __float2half_rn(d);
    sc[nb + 2 * blk] = __ushort_as_half((unsigned short)(qh & 0xFFFF));
    sc[nb + 2 * blk + 1] = __ushort_as_half((unsigned short)(qh >> 16));
  }
}

// ---- Bulk mapping for q8_0 / q4_0: one thread per 32-element block ----------
// The 8-lane bodies above keep the latency of one row low (the fused decode
// step appends one row per KV head).  Many rows at once are bound by
// instruction issue instead, so the bulk append gives a whole block to one
// thread: four 16-byte loads, no shuffles, and the block's scale, divide and
// index math paid once per 32 elements.  The arithmetic is the same as above,
// so the stored bytes are identical.

struct BlockRaw {
  uint4 w[4];  // the block's 32 fp16 inputs, two per word
};

// Block gblk of the call's [rows][D] input (zeros past nblk).
__device__ __forceinline__ BlockRaw load_block(const AppendParams& p, int64_t gblk, int64_t nblk) {
  BlockRaw r;
  if (gblk < nblk) {
    const uint4* src = reinterpret_cast<const uint4*>(p.src + gblk * kBlock);
#pragma unroll
    for (int j = 0; j < 4; ++j) r.w[j] = __ldg(src + j);
  } else {
#pragma unroll
    for (int j = 0; j < 4; ++j) r.w[j] = make_uint4(0u, 0u, 0u, 0u);
  }
  return r;
}

__device__ __forceinline__ float block_elem(const BlockRaw& r, int i) {  // element i (0..31) as float
  const uint4& v = r.w[i >> 3];
  const int k = (i >> 1) & 3;
  const uint32_t w = k == 0 ? v.x : k == 1 ? v.y : k == 2 ? v.z : v.w;
  return __half2float(__ushort_as_half((uint16_t)(w >> (16 * (i & 1)))));
}

__device__ __forceinline__ __half2 block_pair(const BlockRaw& r, int k) {  // elements 2k, 2k+1
  const uint4& v = r.w[k >> 2];
  const int c = k & 3;
  const uint32_t w = c == 0 ? v.x : c == 1 ? v.y : c == 2 ? v.z : v.w;
  return *reinterpret_cast<const __half2*>(&w);
}

// Where block gblk's row lands in the cache (-1: not written), and the block's
// index in its row.
__device__ __forceinline__ void block_dst(const AppendParams& p, int64_t gblk, int64_t& r, int& blk) {
  const int lb = log2_blocks(p);
  r = dst_row(p, gblk >> lb);
  blk = (int)(gblk & ((1 << lb) - 1));
}

// q8_0 of one block (same definition as append_q8_0).  Rounding without the
// conversion pipe: s = fl(t + 1.5 * 2^23) holds t rounded to an integer (ties
// to even) in its low mantissa bits, so its low byte is the two's-complement
// code and s - 1.5 * 2^23 is that integer as a float.  Away from a tie this is
// roundf; if any t of the block lies within 2^-14 of a half-integer, the whole
// block takes the exact divide instead.
__device__ __forceinline__ void q8_0_block(const AppendParams& p, int64_t gblk, const BlockRaw& raw) {
  constexpr float kMagic = 12582912.0f;  // 1.5 * 2^23
  __half2 m2 = __habs2(block_pair(raw, 0));
#pragma unroll
  for (int k = 1; k < 16; ++k) m2 = __hmax2(m2, __habs2(block_pair(raw, k)));
  const float amax = fmaxf(__low2float(m2), __high2float(m2));  // max of fp16 values: exact
  const float d = __fdiv_rn(amax, 127.0f);
  const float rd = d != 0.0f ? __frcp_rn(d) : 0.0f;
  uint32_t code[8];
  bool near = false;
  const unsigned long long rd2 = pack_f32x2(rd, rd), mg2 = pack_f32x2(kMagic, kMagic);
#pragma unroll
  for (int w = 0; w < 8; ++w) {
    float s4[4];
#pragma unroll
    for (int i = 0; i < 4; i += 2) {  // two elements per packed operation
      const unsigned long long t2 = mul_f32x2(pack_f32x2(block_elem(raw, 4 * w + i), block_elem(raw, 4 * w + i + 1)), rd2);
      const unsigned long long s2 = add_f32x2(t2, mg2);
      float e0, e1;
      unpack_f32x2(sub_f32x2(t2, sub_f32x2(s2, mg2)), e0, e1);
      near |= fabsf(e0) >= 0.49993896484375f || fabsf(e1) >= 0.49993896484375f;  // 0.5 - 2^-14
      unpack_f32x2(s2, s4[i], s4[i + 1]);
    }
    code[w] = __byte_perm(__byte_perm(__float_as_uint(s4[0]), __float_as_uint(s4[1]), 0x0040),
                          __byte_perm(__float_as_uint(s4[2]), __float_as_uint(s4[3]), 0x0040), 0x5410);
  }
  if (near) {  // rare: some quotient is close to a tie
#pragma unroll
    for (int w = 0; w < 8; ++w) {
      uint32_t b = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i)
        b |= (uint32_t)((int)roundf(__fdiv_rn(block_elem(raw, 4 * w + i), d)) & 0xFF) << (8 * i);
      code[w] = b;
    }
  }
  int64_t r;
  int blk;
  block_dst(p, gblk, r, blk);
  if (r < 0) return;
  uint4* dst = reinterpret_cast<uint4*>(p.dst.codes + r * p.dst.code_bytes + blk * kBlock);
  dst[0] = make_uint4(code[0], code[1], code[2], code[3]);
  dst[1] = make_uint4(code[4], code[5], code[6], code[7]);
  p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// q4_0 of one block (same definition as append_q4_0).
__device__ __forceinline__ void q4_0_block(const AppendParams& p, int64_t gblk, const BlockRaw& raw) {
  float bm = block_elem(raw, 0);
#pragma unroll
  for (int i = 1; i < kBlock; ++i) {
    const float x = block_elem(raw, i);
    if (fabsf(x) > fabsf(bm)) bm = x;  // strictly larger: the first index wins ties
  }
  const float d = __fdiv_rn(bm, -8.0f);
  const float id = d != 0.0f ? __frcp_rn(d) : 0.0f;
  uint32_t q[kBlock];
#pragma unroll
  for (int i = 0; i < kBlock; ++i)
    q[i] = (uint32_t)min(15, __float2int_rz(__fadd_rn(__fmul_rn(block_elem(raw, i), id), 8.5f)));
  uint32_t word[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {  // byte j = q_j | q_{j+16} << 4
    uint32_t b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = q[4 * w + i] | (q[4 * w + i + 16] << 4);
    word[w] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  }
  int64_t r;
  int blk;
  block_dst(p, gblk, r, blk);
  if (r < 0) return;
  *reinterpret_cast<uint4*>(p.dst.codes + r * p.dst.code_bytes + blk * (kBlock / 2)) =
      make_uint4(word[0], word[1], word[2], word[3]);
  p.dst.scales[r * p.dst.n_scales + blk] = __float2half_rn(d);
}

// q5_0 of one block (same definition as append_q5_0).
__device__ __forceinline__ void q5_0_block(const AppendParams& p, int64_t gblk, const BlockRaw& raw) {
  float bm = block_elem(raw, 0);
#pragma unroll
  for (int i = 1; i < kBlock; ++i) {
    const float x = block_elem(raw, i);
    if (fabsf(x) > fabsf(bm)) bm = x;  // strictly larger: the first index wins ties
  }
  const float d = __fdiv_rn(bm, -16.0f);
  const float id = d != 0.0f ? __frcp_rn(d) : 0.0f;
  uint32_t q[kBlock];
  uint32_t qh = 0;
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    q[i] = (uint32_t)min(31, __float2int_rz(__fadd_rn(__fmul_rn(block_elem(raw, i), id), 16.5f)));
    qh |= (q[i] >> 4) << i;
  }
  uint32_t word[4];
#pragma unroll
  for (int w = 0; w < 4; ++w) {  // byte j = low nibbles of q_j and q_{j+16}
    uint32_t b[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) b[i] = (q[4 * w + i] & 15) | ((q[4 * w + i + 16] & 15) << 4);
    word[w] = __byte_perm(__byte_perm(b[0], b[1], 0x0040), __byte_perm(b[2], b[3], 0x0040), 0x5410);
  }
  int64_t r;
  int blk;
  block_dst(p, gblk, r, blk);
  if (r < 0) return;
  *reinterpret_cast<uint4*>(p.dst.codes + r * p.dst.code_bytes + blk * (kBlock / 2)) =
      make_uint4(word[0], word[1], word[2], word[3]);
  const int nb = p.D / kBlock;
  __half* sc = p.dst.scales + r * p.dst.n_scales;
  sc[blk] = __float2half_rn(d);
  sc[nb + 2 * blk] = __ushort_as_half((unsigned short)(qh & 0xFFFF));
  sc[nb + 2 * blk + 1] = __ushort_as_half((unsigned short)(qh >> 16));
}

// f16: copy rows, 16 bytes per thread.
__device__ __forceinline__ void append_f16(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw) {
  const int per_row = p.D / 8;  // 16-byte chunks per row (a power of two)
  const int64_t i = gtid;
  if (i >= gend) return;
  const int64_t row = i >> (31 - __clz(per_row));
  const int c = (int)(i & (per_row - 1));
  const int64_t r = dst_row(p, row);
  if (r < 0) return;
  reinterpret_cast<uint4*>(p.dst.codes + r * p.dst.code_bytes)[c] = raw;
}

// turbo (BITS = 2, 3 or 4 bits per value): one warp per row, E = D/32
// contiguous elements per lane.  QJL (turbo3_qjl, BITS = 2): after the level
// codes, the residual e = g - c[code] of each element, its norm by the same
// tree, and the sign bits of u = P e; lane l computes u_i of its own rows
// i = l*E .. l*E+E-1, taking e_j (j = 0 .. D-1 in order) from its owner lane.
// P comes from pt, a transposed copy in shared memory (pt[j*D + i] = P[i][j]:
// the warp reads one contiguous line per j), or, when pt is null, from global
// memory row by row.
// Code of g: the number of thresholds below it, #{k : g > tau[k]} (the
// thresholds ascend), found by binary search: at 2 and 3 bits each step
// compares against one threshold chosen by the bits decided so far (three or two
// compares and a few selects instead of seven or three compares and adds; a NaN
// fails every compare and gets code 0, as with the count).  4 bits: the count.
// Used by the bulk body; the one-warp body (also inlined into the fused decode
// step) keeps the plain count, which measured faster there.
template <int BITS>
__device__ __forceinline__ int turbo_code(float g, const float* tau) {
  if constexpr (BITS == 3) {
    const bool b2 = g > tau[3];
    const bool b1 = g > (b2 ? tau[5] : tau[1]);
    const float t0 = b2 ? (b1 ? tau[6] : tau[4]) : (b1 ? tau[2] : tau[0]);
    const bool b0 = g > t0;
    return (b2 ? 4 : 0) + (b1 ? 2 : 0) + (b0 ? 1 : 0);
  } else if constexpr (BITS == 2) {
    const bool b1 = g > tau[1];
    const bool b0 = g > (b1 ? tau[2] : tau[0]);
    return (b1 ? 2 : 0) + (b0 ? 1 : 0);
  } else {
    int c = 0;
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) c += g > tau[k] ? 1 : 0;
    return c;
  }
}

template <int BITS, int E, bool QJL = false>
__device__ __forceinline__ void append_turbo(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw,
                                             const float* pt) {
  constexpr int D = 32 * E;
  const int64_t row = gtid >> 5;
  const int lane = (int)(gtid & 31);
  if (gtid >= gend) return;  // whole warps exit together (gend is a multiple of 32)
  float v[E];
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const int i = lane * E + e;
    const float x = raw_elem(raw, e);
    v[e] = ((p.tq.sign_bits[i >> 5] >> (i & 31)) & 1u) ? -x : x;
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
  float res[E];  // QJL: residuals in the rotated unit domain
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float g = __fmul_rn(v[e], r);
    int c = 0;
    float lv = p.tq.levels[0];  // levels[c] (thresholds ascend), without a dynamic index
#pragma unroll
    for (int k = 0; k < (1 << BITS) - 1; ++k) {
      const bool up = g > p.tq.tau[k];
      c += up ? 1 : 0;
      if (QJL) lv = up ? p.tq.levels[k + 1] : lv;
    }
    bits |= (uint32_t)c << (BITS * e);
    res[e] = QJL ? __fsub_rn(g, lv) : 0.0f;
  }
  float gamma = 0.0f;
  uint32_t zbits = 0;
  if constexpr (QJL) {
#pragma unroll
    for (int e = 0; e < E; ++e) a[e] = __fmul_rn(res[e], res[e]);
#pragma unroll
    for (int h = D / 2; h >= E; h >>= 1) {
#pragma unroll
      for (int e = 0; e < E; ++e) a[e] = __fadd_rn(a[e], __shfl_xor_sync(0xffffffffu, a[e], h / E));
    }
#pragma unroll
    for (int h = E / 2; h >= 1; h >>= 1) {
#pragma unroll
      for (int e = 0; e < E; ++e) a[e] = __fadd_rn(a[e], a[e + h]);
    }
    const float eps = __fsqrt_rn(__shfl_sync(0xffffffffu, a[0], 0));
    gamma = __fmul_rn(__fmul_rn(norm, eps), qjl_rsqrt_d(p.tq));
    float u[E];
#pragma unroll
    for (int e = 0; e < E; ++e) u[e] = 0.0f;
    if (pt != nullptr) {
#pragma unroll 2
      for (int jl = 0; jl < 32; ++jl) {
#pragma unroll
        for (int e2 = 0; e2 < E; ++e2) {
          const float ej = __shfl_sync(0xffffffffu, res[e2], jl);
          const float* col = pt + (jl * E + e2) * D + lane * E;  // P[lane*E .. lane*E+E-1][j]
          float pv[E];
          if constexpr (E % 4 == 0) {
#pragma unroll
            for (int k4 = 0; k4 < E; k4 += 4) {
              const float4 f = *reinterpret_cast<const float4*>(col + k4);
              pv[k4] = f.x;
              pv[k4 + 1] = f.y;
              pv[k4 + 2] = f.z;
              pv[k4 + 3] = f.w;
            }
          } else if constexpr (E == 2) {
            const float2 f = *reinterpret_cast<const float2*>(col);
            pv[0] = f.x;
            pv[1] = f.y;
          } else {
            pv[0] = col[0];
          }
#pragma unroll
          for (int e = 0; e < E; ++e) u[e] = __fadd_rn(u[e], __fmul_rn(pv[e], ej));
        }
      }
    }
    const float* prow = qjl_proj(p.tq) + (size_t)(lane * E) * D;  // row lane*E of P
#pragma unroll 4
    for (int jl = 0; jl < (pt == nullptr ? 32 : 0); ++jl) {  // e_j of j = jl*E .. jl*E+E-1, held by lane jl
      float ej[E];
#pragma unroll
      for (int e2 = 0; e2 < E; ++e2) ej[e2] = __shfl_sync(0xffffffffu, res[e2], jl);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        float pv[E];
        const float* src = prow + (size_t)e * D + jl * E;
        if constexpr (E % 4 == 0) {
#pragma unroll
          for (int k4 = 0; k4 < E; k4 += 4) {
            const float4 f = __ldg(reinterpret_cast<const float4*>(src + k4));
            pv[k4] = f.x;
            pv[k4 + 1] = f.y;
            pv[k4 + 2] = f.z;
            pv[k4 + 3] = f.w;
          }
        } else if constexpr (E == 2) {
          const float2 f = __ldg(reinterpret_cast<const float2*>(src));
          pv[0] = f.x;
          pv[1] = f.y;
        } else {
          pv[0] = __ldg(src);
        }
#pragma unroll
        for (int e2 = 0; e2 < E; ++e2) u[e] = __fadd_rn(u[e], __fmul_rn(pv[e2], ej[e2]));
      }
    }
#pragma unroll
    for (int e = 0; e < E; ++e) zbits |= (u[e] < 0.0f ? 1u : 0u) << e;
  }
  // The lane's LB = BITS*E bits start at bit LB*lane of the row; a group of L
  // lanes (the fewest whose bits make whole bytes, at most 32) is stored by
  // its first lane.
  constexpr int LB = BITS * E;
  constexpr int L = LB % 8 == 0 ? 1 : LB % 4 == 0 ? 2 : LB % 2 == 0 ? 4 : 8;
  uint32_t word = bits;
#pragma unroll
  for (int j = 1; j < L; ++j) {
    const uint32_t o = __shfl_down_sync(0xffffffffu, bits, j);
    word |= o << (LB * j);
  }
  // QJL sign bits: E per lane, the same grouping at one bit per value
  constexpr int LZ = E % 8 == 0 ? 1 : E % 4 == 0 ? 2 : E % 2 == 0 ? 4 : 8;
  uint32_t zword = zbits;
  if constexpr (QJL) {
#pragma unroll
    for (int j = 1; j < LZ; ++j) {
      const uint32_t o = __shfl_down_sync(0xffffffffu, zbits, j);
      zword |= o << (E * j);
    }
  }
  const int64_t r_dst = dst_row(p, row);
  if (r_dst < 0) return;  // after the last shuffle
  uint8_t* codes = p.dst.codes + r_dst * p.dst.code_bytes;
  if ((lane % L) == 0) {
    const int byte0 = LB * lane / 8;
#pragma unroll
    for (int i = 0; i < L * LB / 8; ++i) codes[byte0 + i] = (uint8_t)((word >> (8 * i)) & 0xFF);
  }
  if constexpr (QJL) {
    if ((lane % LZ) == 0) {
      const int byte0 = BITS * D / 8 + E * lane / 8;
#pragma unroll
      for (int i = 0; i < LZ * E / 8; ++i) codes[byte0 + i] = (uint8_t)((zword >> (8 * i)) & 0xFF);
    }
    if (lane == 0) {
      p.dst.scales[2 * r_dst] = __float2half_rn(fminf(norm, 65504.0f));
      p.dst.scales[2 * r_dst + 1] = __float2half_rn(fminf(gamma, 65504.0f));
    }
  } else {
    if (lane == 0) p.dst.scales[r_dst] = __float2half_rn(fminf(norm, 65504.0f));
  }
}

// Bulk append of turbo rows other than turbo3_qjl: D/16 lanes per row, 16
// contiguous elements per lane (a row's lanes are an aligned group of the warp,
// 32/(D/16) rows per warp).  The same operations in the same order as append_turbo -- the
// norm's pairwise tree, each butterfly of the transform, the quantizer -- so the
// stored bytes are the same; fewer levels cross lanes (log2(D/16) instead of
// log2(32)), the per-row index work is shared by 32/(D/16) rows, and each lane
// stores its own 2*BITS code bytes.
constexpr int kWideElems = 16;
struct Raw32 {
  uint4 a, b;  // 16 fp16 elements
};
__device__ __forceinline__ Raw32 load_wide(const AppendParams& p, int64_t gtid, int64_t gend) {
  Raw32 r{make_uint4(0u, 0u, 0u, 0u), make_uint4(0u, 0u, 0u, 0u)};
  if (gtid >= gend) return r;
  const uint4* src = reinterpret_cast<const uint4*>(p.src + gtid * kWideElems);
  r.a = __ldg(src);
  r.b = __ldg(src + 1);
  return r;
}
__device__ __forceinline__ float wide_elem(const Raw32& r, int i) {  // fp16 element i (0..15) as float
  return raw_elem(i < 8 ? r.a : r.b, i & 7);
}

template <int BITS, int D>
__device__ __forceinline__ void append_turbo_wide(const AppendParams& p, int64_t gtid, int64_t gend, const Raw32& raw) {
  constexpr int LPR = D / kWideElems;  // lanes per row
  constexpr int E = kWideElems;
  const int lr = (int)(gtid & (LPR - 1));  // lane within the row (groups are aligned)
  const int64_t row = gtid / LPR;
  float v[E];
  const int i0 = lr * E;  // the lane's first element; its 16 sign bits lie in one word
  const uint32_t sw = p.tq.sign_bits[i0 >> 5] >> (i0 & 31);
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float x = wide_elem(raw, e);
    v[e] = ((sw >> e) & 1u) ? -x : x;
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
  const float norm = __fsqrt_rn(__shfl_sync(0xffffffffu, a[0], 0, LPR));
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
    const bool upper = (lr & lm) != 0;
#pragma unroll
    for (int e = 0; e < E; ++e) {
      const float o = __shfl_xor_sync(0xffffffffu, v[e], lm);
      v[e] = upper ? __fsub_rn(o, v[e]) : __fadd_rn(v[e], o);
    }
  }
  const float r = norm > 0.0f ? __frcp_rn(norm) : 0.0f;
  unsigned long long bits = 0;
#pragma unroll
  for (int e = 0; e < E; ++e) {
    const float g = __fmul_rn(v[e], r);
    const int c = turbo_code<BITS>(g, p.tq.tau);
    bits |= (unsigned long long)c << (BITS * e);
  }
  if (gtid >= gend) return;  // after the last shuffle
  const int64_t r_dst = dst_row(p, row);
  if (r_dst < 0) return;
  // the lane's codes: bits [16 * BITS * lr, 16 * BITS * (lr + 1)) of the row
  uint8_t* codes = p.dst.codes + r_dst * p.dst.code_bytes + lr * 2 * BITS;
  if constexpr (BITS % 2 == 0) {
#pragma unroll
    for (int k = 0; k < BITS / 2; ++k) reinterpret_cast<uint32_t*>(codes)[k] = (uint32_t)(bits >> (32 * k));
  } else {
#pragma unroll
    for (int k = 0; k < BITS; ++k) reinterpret_cast<uint16_t*>(codes)[k] = (uint16_t)(bits >> (16 * k));
  }
  if (lr == 0) p.dst.scales[r_dst] = __float2half_rn(fminf(norm, 65504.0f));
}

// Quantize and store work item gtid from its loaded bytes (every lane of the
// warp calls this: the bodies shuffle; items at or past gend store nothing).
template <int TYPE, int E>
__device__ __forceinline__ void finish(const AppendParams& p, int64_t gtid, int64_t gend, const uint4& raw,
                                       const float* pt = nullptr) {
  if constexpr (TYPE == KVQ_Q8_0) append_q8_0(p, gtid, gend, raw);
  else if constexpr (TYPE == KVQ_Q4_0) append_q4_0(p, gtid, gend, raw);
  else if constexpr (TYPE == KVQ_Q5_0) append_q5_0(p, gtid, gend, raw);
  else if constexpr (TYPE == KVQ_F16) append_f16(p, gtid, gend, raw);
  else append_turbo<turbo_bits(TYPE), E, is_qjl(TYPE)>(p, gtid, gend, raw, pt);
}

template <int TYPE, int E>
__device__ __forceinline__ void append_one(const AppendParams& p, int64_t gtid, int64_t gend) {
  finish<TYPE, E>(p, gtid, gend, load_raw<TYPE, E>(p, gtid, gend));
}

// Thread gtid of the flat work of one call's rows of a tensor of `type`;
// threads at or past gend do no work (but still take part in shuffles).
template <int TYPE>
__device__ __forceinline__ void append_turbo_any(const AppendParams& p, int64_t gtid, int64_t gend) {
  switch (p.D) {
    case 32: append_one<TYPE, 1>(p, gtid, gend); break;
    case 64: append_one<TYPE, 2>(p, gtid, gend); break;
    case 128: append_one<TYPE, 4>(p, gtid, gend); break;
    case 256: append_one<TYPE, 8>(p, gtid, gend); break;
  }
}

__device__ __forceinline__ void append_any(int32_t type, const AppendParams& p, int64_t gtid, int64_t gend) {
  switch (type) {
    case KVQ_F16: append_one<KVQ_F16, 0>(p, gtid, gend); break;
    case KVQ_Q8_0: append_one<KVQ_Q8_0, 0>(p, gtid, gend); break;
    case KVQ_Q4_0: append_one<KVQ_Q4_0, 0>(p, gtid, gend); break;
    case KVQ_Q5_0: append_one<KVQ_Q5_0, 0>(p, gtid, gend); break;
    case KVQ_TURBO2: append_turbo_any<KVQ_TURBO2>(p, gtid, gend); break;
    case KVQ_TURBO3: append_turbo_any<KVQ_TURBO3>(p, gtid, gend); break;
    case KVQ_TURBO4: append_turbo_any<KVQ_TURBO4>(p, gtid, gend); break;
    case KVQ_TURBO3_QJL: append_turbo_any<KVQ_TURBO3_QJL>(p, gtid, gend); break;
  }
}

// Threads one row of a tensor of `type` and head dim d needs.
// (append_one, append_any: a turbo row on one warp.)
__host__ __device__ constexpr int row_threads(int32_t type, int d) {
  return type == KVQ_F16 ? d / 8 : is_turbo(type) ? 32 : (d / kBlock) * 8;
}
// Threads one row needs in the bulk append: turbo rows other than turbo3_qjl
// take D/16 lanes there (append_turbo_wide).  The fused decode step appends its
// one row per head with row_threads: the wide body's registers would weigh on the
// decode kernel's own.
__host__ __device__ constexpr int bulk_row_threads(int32_t type, int d) {
  return is_turbo(type) && !is_qjl(type) ? d / kWideElems : row_threads(type, d);
}

}  // namespace rows
}  // namespace kvq
