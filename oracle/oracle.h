/*
 * oracle.h -- entry points of the CPU oracle for quantized-KV decode attention.
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow restatement of what the
 * quantized-KV decode path computes, written to check the CUDA library and
 * nothing else.  Only tests/, __graft_entry__.smoke() and bench.py's CPU
 * baseline and reference legs load it (through oracle/__init__.py).  It
 * includes nothing from the library's sources or headers, and the library
 * never loads it.
 *
 * Build: g++ -O2 -ffp-contract=off -fno-fast-math (oracle/build.py).  With
 * contraction off and no fast-math, every binary32 and binary64 operation
 * below rounds once, as IEEE 754 states it; nothing is fused or reordered.
 *
 * Formats (the pages name the cache types and print cache sizes, not the
 * arithmetic inside a block; the arithmetic is the format definition):
 *   "llama.cpp für Geschwindigkeit und Speicher optimieren", section
 *   "KV-Cache-Präzision": f16 / q8_0 / q4_0, chosen independently for K and V;
 *   "KVSplit - 2- bis 3-mal längerer Kontext auf Apple Silicon", sections
 *   "Zentrale Benchmark-Ergebnisse" and "Vergleich der Speicherersparnis":
 *   different precisions for K and V (K8V4 and the others), cache sizes;
 *   "Benchmark TurboQuant en Apple Silicon", section "¿Qué es TurboQuant?":
 *   Walsh-Hadamard random rotation, optimal scalar quantizer, QJL residual;
 *   section "Flash Attention" of the llama.cpp guide: tiled attention equal
 *   to standard attention, so the attention oracle is the plain definition.
 *
 * Conventions: arrays are dense and row-major; fp16 values travel as their
 * IEEE binary16 bit patterns (uint16_t); n counts rows, d is the row length
 * (head_dim).  Functions that can fail return 0 on success and -1 on a bad
 * argument, writing nothing.
 */
#ifndef KVQ_ORACLE_H
#define KVQ_ORACLE_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- binary16 conversions (IEEE round to nearest, ties to even) */
void orc_f32_to_f16(const float* x, int64_t n, uint16_t* out);
void orc_f16_to_f64(const uint16_t* x, int64_t n, double* out);

/* ---- byte model: bytes of one cached row of d elements (codes + scales);
 *      type codes: 0 f16, 1 q8_0, 2 q4_0, 3 turbo3, 4 turbo2, 5 turbo4,
 *      6 q5_0, 7 turbo3_qjl; 0 when the pair is not a format */
int64_t orc_row_bytes(int32_t type, int32_t d);

/* ---- 32-element block formats (d a multiple of 32) */
/* q8_0: amax, d = amax/127, q = roundf(x/d) (IEEE divide), fp16 d stored */
int orc_quantize_q8_0(const uint16_t* x, int64_t n, int32_t d, uint16_t* scale, int8_t* qs);
/* q4_0: m = x of largest |x| (lowest index on ties), d = m/-8,
 * q = min(15, trunc(fl(fl(x*fl(1/d)) + 8.5))); codes 0..15 unpacked */
int orc_quantize_q4_0_codes(const uint16_t* x, int64_t n, int32_t d, uint16_t* scale, uint8_t* codes);
/* element j of a block -> low nibble of byte j, element j+16 -> high nibble */
int orc_pack_q4_0(const uint8_t* codes, int64_t n, int32_t d, uint8_t* packed);
int orc_unpack_q4_0(const uint8_t* packed, int64_t n, int32_t d, uint8_t* codes);
/* q5_0: q4_0 widened by one bit: d = m/-16, q = min(31, trunc(fl(fl(x*fl(1/d)) + 16.5))) */
int orc_quantize_q5_0_codes(const uint16_t* x, int64_t n, int32_t d, uint16_t* scale, uint8_t* codes);
/* low four bits as q4_0's nibbles, bit 4 of element j as bit j of the block's qh word */
int orc_pack_q5_0(const uint8_t* codes, int64_t n, int32_t d, uint8_t* qs, uint32_t* qh);
int orc_unpack_q5_0(const uint8_t* qs, const uint32_t* qh, int64_t n, int32_t d, uint8_t* codes);
/* dequantization in binary64: x_hat = d_h * q (q8_0), d_h * (q - 8) (q4_0),
 * d_h * (q - 16) (q5_0), double(x) (f16) */
int orc_dequantize_q8_0(const uint16_t* scale, const int8_t* qs, int64_t n, int32_t d, double* out);
int orc_dequantize_q4_0(const uint16_t* scale, const uint8_t* packed, int64_t n, int32_t d, double* out);
int orc_dequantize_q5_0(const uint16_t* scale, const uint8_t* qs, const uint32_t* qh, int64_t n, int32_t d,
                        double* out);
void orc_dequantize_f16(const uint16_t* x, int64_t n, double* out);

/* ---- turbo rows (d a power of two, 8 .. 4096) */
/* first n outputs of splitmix64 started at state `seed` */
void orc_splitmix64(uint64_t seed, int64_t n, uint64_t* out);
/* the sign vector: s_i = -1 where output i has its top bit set, else +1 */
int orc_signs(uint64_t seed, int32_t d, float* out);
/* unnormalised Sylvester-Hadamard matrix of order d, binary64 [d][d] */
int orc_sylvester(int32_t d, double* out);
/* unnormalised fast Walsh-Hadamard transform of each row, binary32 */
int orc_fwht_f32(const float* v, int64_t n, int32_t d, float* out);
/* strided pairwise sum of each row in binary32 (stride d/2, d/4, ..., 1) */
int orc_tree_sum_f32(const float* a, int64_t n, int32_t d, float* out);
/* n_levels-level Lloyd-Max quantizer of N(0,1) in binary64 (n even, 2..256):
 * ascending levels[n] and thresholds[n-1]; returns the iterations taken, -1 if
 * it did not converge */
int orc_lloyd_max_gaussian(int32_t n_levels, double* levels, double* thresholds);
/* turbo row at `bits` (2, 3, 4): fp16 norm and codes 0 .. 2^bits - 1 */
int orc_turbo_quantize_indices(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, int32_t bits,
                               uint16_t* norm, uint8_t* idx);
/* b-bit little-endian bit stream: code i in bits b*i .. b*i+b-1 (bits 1..8) */
int orc_turbo_pack(const uint8_t* idx, int64_t n, int32_t d, int32_t bits, uint8_t* out);
int orc_turbo_unpack(const uint8_t* codes, int64_t n, int32_t d, int32_t bits, uint8_t* idx);
int orc_turbo_quantize(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, int32_t bits, uint16_t* norm,
                       uint8_t* codes);
/* x_hat = (norm/d) * s * H_un * c[code], binary64 */
int orc_turbo_dequantize(const uint16_t* norm, const uint8_t* codes, int64_t n, int32_t d, uint64_t seed,
                         int32_t bits, double* out);

/* ---- turbo3_qjl key rows: the 2-bit turbo row plus 1-bit QJL signs of its residual
 * (P: binary32 [d][d], row i projects onto sign bit i) */
/* fp32 norm, 2-bit codes and the binary32 residual e = g - c32[code] */
int orc_qjl_residual(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, float* norm, uint8_t* idx,
                     float* e);
/* u[r][i] = sum_j P[i][j] * e[r][j] in binary32, left to right */
int orc_qjl_project(const float* P, const float* e, int64_t n, int32_t d, float* u);
int orc_qjl_quantize_parts(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, const float* P,
                           uint16_t* norm, uint16_t* gamma, uint8_t* idx, uint8_t* z);
/* scales [n][2] = (norm, gamma) fp16; codes [n][3d/8] = 2-bit codes, then the sign bits */
int orc_qjl_quantize(const uint16_t* x, int64_t n, int32_t d, uint64_t seed, const float* P, uint16_t* scales,
                     uint8_t* codes);
int orc_qjl_dequantize(const uint16_t* scales, const uint8_t* codes, int64_t n, int32_t d, uint64_t seed,
                       const float* P, double* out);
/* S = P H_un diag(s) / sqrt(d), binary64 [d][d] */
int orc_qjl_projection_matrix(uint64_t seed, const float* P, int32_t d, double* out);

/* ---- attention in binary64 */
/* out[b][h] = sum_t p_t v[b][g][t] / sum_t p_t, p_t = exp(s_t - max s),
 * s_t = scale * <q[b][h], k[b][g][t]>, g = h / (n_q / n_kv);
 * q [B][n_q][D], k and v [B][n_kv][T][D]; (b, h) pairs spread over n_threads
 * threads (<= 0: all hardware threads) */
int orc_decode_attention(const double* q, const double* k, const double* v, int32_t B, int32_t n_q, int32_t n_kv,
                         int64_t T, int32_t D, double scale, double* out, int32_t n_threads);
/* normalised weights p_t / sum p of one query row over T key rows */
int orc_softmax_weights(const double* q, const double* k, int64_t T, int32_t D, double scale, double* w);
/* split partials of one query row: slice s = rows bounds[s] .. bounds[s+1]-1 gives
 * m_s = max score, l_s = sum exp(s_t - m_s), acc_s = sum exp(s_t - m_s) v_t */
int orc_partials(const double* q, const double* k, const double* v, int32_t D, double scale,
                 const int64_t* bounds, int32_t n_slices, double* m, double* l, double* acc);
/* M = max m_s, w_s = exp(m_s - M), out = sum w_s acc_s / sum w_s l_s */
int orc_combine(const double* m, const double* l, const double* acc, int32_t n_slices, int32_t D, double* out);

/* ---- one decode step over a stored cache (bench baseline and parity at size):
 * dequantize every row (k_codes [B][n_kv][T][code_bytes], k_scales
 * [B][n_kv][T][n_scales] fp16, the same per-row format as orc_row_bytes
 * counts; likewise v), then orc_decode_attention's definition with q fp16
 * [B][n_q][D].  Per batch row: the KV heads' rows are dequantized in
 * parallel, then the query heads attend in parallel, over n_threads threads
 * (<= 0: all hardware threads).  turbo types use `seed`; turbo3_qjl keys use P. */
int orc_decode_cache(int32_t k_type, int32_t v_type, int32_t B, int32_t n_q, int32_t n_kv, int64_t T, int32_t D,
                     const uint8_t* k_codes, const uint16_t* k_scales, const uint8_t* v_codes,
                     const uint16_t* v_scales, uint64_t seed, const float* P, const uint16_t* q, double scale,
                     double* out, int32_t n_threads);

/* threads the hardware runs at once (std::thread::hardware_concurrency) */
int32_t orc_hardware_threads(void);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_ORACLE_H */
