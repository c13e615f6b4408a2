// Internal declarations shared by the libkvq translation units (host + device).
#pragma once

#include <atomic>
#include <cstdint>
#include <cstring>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "kvq.h"

namespace kvq {

constexpr int kBlock = 32;          // elements per q8_0 / q4_0 block
constexpr int kMaxHeadDim = 256;
constexpr int kRowAlign = 16;       // rows per plane are a multiple of this
constexpr int kMaxSplits = 4096;
constexpr int kSplitAlign = 32;     // split chunks are whole 32-row tiles (a tile never
                                    // crosses a page of a paged pool)

// Device view of one cache tensor (K or V) of one layer.
struct Plane {
  uint8_t* codes;      // [B][H][T][code_bytes]
  __half* scales;      // [B][H][T][n_scales]
  int64_t T;           // rows per (batch, head) plane
  int32_t code_bytes;
  int32_t n_scales;
};

// Turbo formats: bits of a row's level codes (2, 3 or 4), else 0.  turbo3_qjl
// rows hold 2-bit level codes and, after them, one QJL sign bit per value.
__host__ __device__ constexpr int turbo_bits(int32_t t) {
  return t == KVQ_TURBO2 || t == KVQ_TURBO3_QJL ? 2 : t == KVQ_TURBO3 ? 3 : t == KVQ_TURBO4 ? 4 : 0;
}
__host__ __device__ constexpr bool is_turbo(int32_t t) { return turbo_bits(t) != 0; }
__host__ __device__ constexpr bool is_qjl(int32_t t) { return t == KVQ_TURBO3_QJL; }

// A turbo type's codebook (2^b levels, 2^b - 1 thresholds) and sign bits.
// turbo3_qjl uses 4 levels and 3 thresholds; the last three threshold slots
// carry its QJL projection P ([D][D] fp32, row-major; the address as two
// 32-bit words, low first) and fl(1/sqrt(D)), so the struct (and with it every
// kernel's parameter block) keeps one layout for all types.
struct TurboConsts {
  float levels[16];
  float tau[15];
  uint32_t sign_bits[kMaxHeadDim / 32];  // bit i set -> s_i = -1
};
constexpr int kQjlSlot = 12;  // tau[12], tau[13]: P's address; tau[14]: fl(1/sqrt(D))
__host__ __device__ inline const float* qjl_proj(const TurboConsts& t) {
  uint32_t lo, hi;
  memcpy(&lo, &t.tau[kQjlSlot], 4);
  memcpy(&hi, &t.tau[kQjlSlot + 1], 4);
  return reinterpret_cast<const float*>(((uint64_t)hi << 32) | lo);
}
__host__ __device__ inline float qjl_rsqrt_d(const TurboConsts& t) { return t.tau[kQjlSlot + 2]; }

struct AppendParams {
  const __half* src;   // [B][n_tok][H][D]
  Plane dst;
  int32_t B, H, D, n_tok;
  int64_t pos;
  // Per-sequence lengths (device int32 [B], or null: every row at pos): batch
  // row b's tokens land at lens[b] - n_tok .. lens[b] - 1; a row whose length
  // lies outside [n_tok, len_max] is not written.
  const int32_t* lens;
  int64_t len_max;
  // Paged pool (block_table null: contiguous): logical row r of batch row b is
  // row r & (2^log2_page - 1) of page block_table[b * max_pages + (r >> log2_page)];
  // dst then describes the pool (B = pages, T = page rows).  A page id outside
  // [0, n_pages) is not written.
  const int32_t* block_table;
  int32_t max_pages, log2_page;
  int64_t n_pages;
  // n / H and n / n_tok for 32-bit n as the high half of n * mul (mul = 0: divisor 1)
  uint64_t h_mul, t_mul;
  TurboConsts tq;
};

// Multiplier for exact division of any 32-bit n by d (d >= 1): n / d equals the
// high 64 bits of n * (floor((2^64 - 1) / d) + 1), since the added n / 2^64 per
// unit of error stays below 1 / d; 0 stands for d = 1.
inline uint64_t div_multiplier(uint64_t d) { return d <= 1 ? 0 : ~0ull / d + 1; }

struct DecodeParams {
  Plane k, v;
  const __half* q;     // [B][n_q][D]
  float* ws_m;         // [B][n_q][S]
  float* ws_l;
  float* ws_acc;       // [B][n_q][S][D]
  int32_t B, n_q, n_kv, G, D, S;
  int64_t ctx, chunk;
  // Per-sequence lengths (device int32 [B], or null: every row attends ctx
  // rows): batch row b attends rows [0, ctx_lens[b]) in S chunks of its own;
  // ctx is then the bound, and a length outside [1, ctx] attends nothing.
  const int32_t* ctx_lens;
  // Paged pool (block_table null: contiguous): as in AppendParams; k and v
  // describe the pools (T = page rows), and the tensor maps span n_pages * n_kv
  // planes.  A page id outside [0, n_pages) makes the split's partials NaN.
  const int32_t* block_table;
  int32_t max_pages, log2_page;
  int64_t n_pages;
  float qscale;        // softmax_scale * log2(e)
  TurboConsts tq;      // V sign bits and codebook (turbo values)
  TurboConsts tqk;     // K sign bits and codebook (turbo keys)
  // Fused decode step (kvq_decode_step); a plain decode has append_pos < 0 and
  // out == null.
  int64_t append_pos;    // row the new K/V rows are written to first (< 0: none;
                         // with ctx_lens, batch row b's is ctx_lens[b] - 1)
  AppendParams app_k;    // that append: B = batch, H = n_kv, n_tok = 1
  AppendParams app_v;
  float* out;            // [B][n_q][D] combined output, or null (partials only)
  uint32_t* counters;    // [B][n_kv] split arrival counters, zero between calls
  uint32_t* epochs;      // [B][n_kv] bumped by each group's last arrival (any start value)
  uint32_t* status;      // workspace status word; bits set by a wait that gave up (kvq.h)
  int32_t comb_ctas;     // CTAs per group that combine (the last arrivals), 1 .. G
  int32_t pdl;           // 1: launched to overlap the previous kernel (KVQ_FLAG_OVERLAP_PREVIOUS)
};

struct CombineParams {
  const float* ws_m;
  const float* ws_l;
  const float* ws_acc;
  float* out;          // [B][n_q][D]
  int32_t B, n_q, D, S;
  // Partials of several ranks (context split across GPUs), rank after rank:
  // rank r's m, l and acc start rank_stride floats after rank r-1's; the
  // n_ranks * S partials of a query head are merged as one set of splits.
  int32_t n_ranks;     // 1: one workspace
  int64_t rank_stride;
  int32_t rotated;     // turbo values: apply s * H_un * (.) / D
  TurboConsts tq;
};

// Raises a kernel's dynamic shared memory limit to `bytes` on the current
// device, once per device (the attribute belongs to the device's context; the
// bit set `done` remembers devices 0..63, others are set on every call).
template <typename Kernel>
cudaError_t set_smem_limit_once(Kernel kern, int bytes, std::atomic<uint64_t>& done) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const uint64_t bit = dev >= 0 && dev < 64 ? (1ull << dev) : 0ull;
  if (bit != 0 && (done.load(std::memory_order_relaxed) & bit) != 0) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess && bit != 0) done.fetch_or(bit, std::memory_order_relaxed);
  return e;
}

// Host-side helpers (kvq_api.cu).
int64_t rows_per_plane(int64_t max_ctx);
int32_t code_bytes_of(int32_t type, int32_t d);
int32_t n_scales_of(int32_t type, int32_t d);
void set_last_cuda_error(cudaError_t e);  // text returned by kvq_last_cuda_error()

// Launchers; each returns cudaGetLastError() after its launch.
// Quantize-on-append of K and/or V rows (either may be null) in one launch.
cudaError_t launch_append(const AppendParams* k, int32_t k_type, const AppendParams* v, int32_t v_type,
                          cudaStream_t st);
cudaError_t launch_decode(int32_t k_type, int32_t v_type, const DecodeParams& p, cudaStream_t st);
bool decode_supported(int32_t k_type, int32_t v_type, int32_t G, int32_t D);
// Resident decode CTAs per SM (shared memory decides) that the split heuristic plans for.
int decode_ctas_per_sm(int32_t k_type, int32_t v_type, int32_t D, int32_t G);
cudaError_t launch_combine(const CombineParams& p, cudaStream_t st);

}  // namespace kvq
