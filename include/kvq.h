/*
 * kvq.h -- C ABI of libkvq: quantized-KV decode attention on NVIDIA B200 (sm_100a).
 *
 * What it computes
 * ----------------
 * Attention decoding over a KV cache whose keys and values are stored at
 * independently chosen precisions.  The pages this library follows:
 *   - "KVSplit - 2- bis 3-mal längerer Kontext auf Apple Silicon", sections
 *     "Zentrale Benchmark-Ergebnisse" and "Anwendungsbeispiele und
 *     Konfigurationsempfehlungen": keys and values quantized at different
 *     precisions (K8V4, K8V8, K4V4, K4V8 demo), chosen per tensor;
 *   - "llama.cpp für Geschwindigkeit und Speicher optimieren", section
 *     "KV-Cache-Präzision": cache types f16 / q8_0 / q4_0, set independently for
 *     K and V; section "Flash Attention": tiled attention that is exactly
 *     standard attention, not an approximation;
 *   - "Benchmark TurboQuant en Apple Silicon", section "¿Qué es TurboQuant?":
 *     a 3-bit value cache ("turbo3") after a random Walsh-Hadamard rotation and
 *     an optimal scalar quantizer; section "Explicación de la configuración":
 *     q8_0 keys with turbo3 values;
 *   - "Eval bug: Metal fails mixed quantized KV on Apple Silicon when Flash
 *     Attention is unavailable, ...", section "Expected behavior": an
 *     unsupported combination must be rejected early and cleanly, without
 *     partial initialization or a crash.
 *
 * Cache types (per 32-element block unless stated):
 *   KVQ_F16    the fp16 input, unchanged (2 bytes / element).
 *   KVQ_Q8_0   fp16 scale d = amax/127 and 32 int8 q_j = round-half-away(x_j/d),
 *              computed in binary32 with an IEEE divide per element; the fp32 d
 *              (not its fp16 image) quantizes; d == 0 gives q_j = 0.  34 bytes.
 *   KVQ_Q4_0   m = signed value of the largest |x_j| (lowest j on ties),
 *              d = m / -8, q_j = min(15, trunc(fl(fl(x_j * fl(1/d)) + 8.5))),
 *              element j in the low nibble of byte j, element j+16 in the high
 *              nibble; d == 0 gives nibble 8.  18 bytes.
 *   KVQ_Q5_0   q4_0 widened by one bit: d = m / -16, q_j = min(31, trunc(fl(fl(
 *              x_j * fl(1/d)) + 16.5))); the low four bits of q_j are packed as
 *              q4_0's nibbles and bit 4 of q_j is bit j of a 32-bit word qh;
 *              d == 0 gives q_j = 16.  22 bytes.  (A comment in the llama.cpp
 *              issue reports q5_0/q5_0 caches as a usable middle ground; no page
 *              prints its arithmetic.)
 *   KVQ_TURBO3 (head_dim a power of two) one row of head_dim
 *              elements: signs s_i = -1 when output i of splitmix64(turbo_seed)
 *              has its top bit set; v = s*x; norm = sqrtf(tree sum of v_i^2,
 *              pairs at stride d/2, d/4, ..., 1); w = unnormalised fast
 *              Walsh-Hadamard transform of v (stages h = 1, 2, ..., d/2);
 *              g_i = w_i * fl(1/norm); code_i = #{k : g_i > tau_k} against the
 *              seven binary32 midpoints of the 8-level Lloyd-Max quantizer of
 *              N(0,1) (so g/sqrt(d) is coded with the N(0,1/d) codebook);
 *              codes packed 3 bits each, little-endian (code i in bits
 *              3i..3i+2); stored norm fp16(min(norm, 65504)).  3d/8 + 2 bytes.
 *              Decoded value: x_hat = (norm/d) * s * H_un * c[code].
 *   KVQ_TURBO2, KVQ_TURBO4 the same row at 2 and 4 bits per value:
 *              the 4- and 16-level Lloyd-Max quantizers of N(0,1) (3 and 15
 *              midpoints), code i in bits b*i .. b*i+b-1.  The TurboQuant page's
 *              FAQ ("¿Qué formato TurboQuant debería usar?") puts values at 2 to 3
 *              bits; 4 bits is the next width.  d/4 + 2 and d/2 + 2 bytes.
 *   KVQ_TURBO3_QJL (keys only; head_dim a power of two) the TurboQuant page's
 *              three parts at 3 bits per value (same section: rotation, optimal
 *              scalar quantizer, QJL to keep inner products), read after the
 *              published QJL / TurboQuant constructions: the turbo2 row (2-bit
 *              codes, norm), then a 1-bit QJL code of its residual.  With g, norm
 *              and code as for turbo2 (binary32, one rounding per operation):
 *              e_i = fl(g_i - c32[code_i]) (c32 the binary32 4-level codebook);
 *              u_i = sum_j P[i][j] * e_j summed left to right for j = 0 .. d-1,
 *              P = desc->qjl_proj; z_i = 1 where u_i < 0;
 *              eps = sqrtf(tree sum of fl(e_i^2));
 *              gamma = fp16(min(fl(fl(norm * eps) * fl(1/sqrt(d))), 65504)),
 *              the residual's norm.  Code row: the 2-bit codes (d/4 bytes),
 *              then z_i in bit i of a d/8-byte field; scale row: (norm, gamma).
 *              3d/8 + 4 bytes.  Decoded key:
 *              x_hat = (norm/d) s H_un c[code]
 *                      + sqrt(pi/2)/d * gamma * s H_un P^T (1 - 2z) / sqrt(d),
 *              i.e. QJL of the residual r with S = P H_un diag(s) / sqrt(d),
 *              whose entries are i.i.d. N(0,1) when P's are, so <q, x_hat> is
 *              an unbiased estimate of <q, x> over the draw of P.  Decodes with
 *              q8_0, q4_0 or turbo3 values; as a value type
 *              KVQ_ERR_UNSUPPORTED.
 *   Turbo keys: a key row x_hat gives the score <q, x_hat> = (norm/d) *
 *   <H_un (s * q), c[code]>, so the decode rotates each query once.  The same
 *   page's FAQ finds keys more sensitive to compression than values.  Turbo keys
 *   decode with q8_0, q4_0 or the same turbo type as values (other pairings are
 *   KVQ_ERR_UNSUPPORTED at decode; append takes any pairing).
 *
 * Memory layout of one cache tensor (K or V) of one layer, in device memory
 * owned by the caller:
 *   rows_per_plane T = max_ctx rounded up to a multiple of 16;
 *   code plane  at byte 0:           [batch][n_kv_heads][T][code_bytes]
 *   scale plane at byte scale_offset: [batch][n_kv_heads][T][n_scales] fp16
 *   with code_bytes = 2d (f16), d (q8_0), d/2 (q4_0, q5_0), b*d/8 (turbo b),
 *   3d/8 (turbo3_qjl);
 *   n_scales = 0 (f16), d/32 (q8_0, q4_0), 3d/32 (q5_0: the d/32 block scales,
 *   then the d/32 qh words, each as two fp16 slots, little-endian), 1 (turbo
 *   types, the norm), 2 (turbo3_qjl: norm, gamma);
 *   scale_offset = code plane bytes rounded up to a multiple of 256.
 *   Within a row, q8_0 codes and q4_0 bytes are in block order, exactly as the
 *   block formats above; scale n of a row belongs to block n.
 *   The base pointer must be 256-byte aligned (cudaMalloc's is).
 *
 * Conventions
 *   Query head h attends with KV head floor(h / G), G = n_q_heads / n_kv_heads.
 *   A decode query attends to cache rows 0 .. ctx_len-1 (no mask).
 *   New K/V rows: fp16 [batch][n_tok][n_kv_heads][head_dim], row-major.
 *   Queries: fp16 [batch][n_q_heads][head_dim].  Output: fp32
 *   [batch][n_q_heads][head_dim].
 *   Split-KV: with S splits, chunk = ceil(ctx_len / S) rounded up to a multiple
 *   of 32 (one tile); split s covers rows [s*chunk, min((s+1)*chunk, ctx_len))
 *   and may be empty.
 *
 * Ownership, threading, errors
 *   The caller owns every buffer.  No entry point allocates device memory,
 *   synchronizes the device or keeps per-call state; kernel launches go to the
 *   given CUDA stream (NULL = legacy default stream) and run asynchronously.
 *   Every argument check happens before any launch; on an error status
 *   nothing has been written and nothing launched.  KVQ_ERR_CUDA means a
 *   launch was refused by the CUDA runtime (see kvq_last_cuda_error()).
 *   Entry points are thread-safe.
 */
#ifndef KVQ_H
#define KVQ_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define KVQ_API __attribute__((visibility("default")))
#else
#define KVQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  KVQ_F16 = 0,
  KVQ_Q8_0 = 1,
  KVQ_Q4_0 = 2,
  KVQ_TURBO3 = 3,
  KVQ_TURBO2 = 4,
  KVQ_TURBO4 = 5,
  KVQ_Q5_0 = 6,
  KVQ_TURBO3_QJL = 7
} kvq_type;

typedef enum {
  KVQ_OK = 0,
  KVQ_ERR_INVALID = 1,      /* null pointer, bad count, range outside the cache */
  KVQ_ERR_UNSUPPORTED = 2,  /* valid arguments this library does not implement */
  KVQ_ERR_WORKSPACE = 3,    /* workspace smaller than kvq_workspace_bytes() */
  KVQ_ERR_CUDA = 4          /* the CUDA runtime refused a launch or a query */
} kvq_status;

/* kvq_cache_desc.flags.
 * KVQ_FLAG_OVERLAP_PREVIOUS: kvq_decode_step (uniform ctx_len, contiguous
 *   cache) is launched so that it may start while the kernel before it on the
 *   stream is still finishing (programmatic dependent launch).  Until that
 *   kernel has completed, the step only reads cache rows 0 .. ctx_len-2 of this
 *   layer (it requests its first tiles); q, k_new, v_new, the workspace and out
 *   are touched only after it.  The caller promises that the kernel right
 *   before the step on the stream does not write those cache rows -- true when
 *   it is another layer's step, a projection producing q, k_new and v_new, or
 *   anything but an append into this same cache.  In a CUDA graph the same
 *   holds for the node before it.  Other entry points ignore the flag. */
#define KVQ_FLAG_OVERLAP_PREVIOUS 1

/* One layer's cache description (K and V of one layer share it). */
typedef struct {
  int32_t n_q_heads;   /* query heads, a multiple of n_kv_heads */
  int32_t n_kv_heads;  /* KV heads */
  int32_t head_dim;    /* multiple of 32, at most 256 */
  int32_t k_type;      /* kvq_type of the key cache: any */
  int32_t v_type;      /* kvq_type of the value cache: any but TURBO3_QJL */
  int32_t flags;       /* KVQ_FLAG_* bits; 0 for none */
  int64_t max_ctx;     /* rows the cache holds per (batch, KV head), >= 1 */
  uint64_t turbo_seed; /* seed of the turbo sign vector (K and V turbo types) */
  /* TURBO3_QJL keys: the QJL projection P, device memory owned by the caller,
   * fp32 [head_dim][head_dim] row-major (row i projects onto code bit i),
   * 16-byte aligned, unchanged while the cache is in use; read by the append
   * and decode calls (NULL there: KVQ_ERR_INVALID).  Ignored otherwise. */
  const float* qjl_proj;
} kvq_cache_desc;

/* Byte layout of one cache tensor, as described above. */
typedef struct {
  int64_t rows_per_plane;  /* T */
  int64_t code_bytes;      /* bytes of codes per row */
  int64_t n_scales;        /* fp16 scales per row */
  int64_t scale_offset;    /* byte offset of the scale plane */
  int64_t total_bytes;     /* bytes to allocate */
} kvq_plane_layout;

/* A paged cache (see "Paged pools" below): the pool's geometry and the block
 * table that maps each sequence's pages into it. */
typedef struct {
  const int32_t* block_table;  /* device int32 [batch][max_pages], 4-byte aligned:
                                  page id of sequence b's logical rows
                                  [j * page_rows, (j + 1) * page_rows) */
  int32_t max_pages;           /* columns of block_table, >= 1 */
  int32_t page_rows;           /* rows per page: a power of two, 32 .. 2^20 */
  int64_t n_pages;             /* pages in the pool, >= 1 (n_pages * n_kv_heads < 2^31) */
} kvq_paged;

/* Human-readable name of a status.  Never NULL. */
KVQ_API const char* kvq_status_string(kvq_status s);

/* Text of the last CUDA error this thread saw (empty if none). */
KVQ_API const char* kvq_last_cuda_error(void);

/* Bytes of one cached row of head_dim elements of `type` (codes + scales),
 * the quantity the pages' cache sizes count; 0 if unsupported. */
KVQ_API size_t kvq_row_bytes(int32_t type, int32_t head_dim);

/* Checks a descriptor: KVQ_OK, KVQ_ERR_INVALID or KVQ_ERR_UNSUPPORTED. */
KVQ_API kvq_status kvq_check_desc(const kvq_cache_desc* desc);

/* Layout of the K (which = 0) or V (which = 1) cache of one layer. */
KVQ_API kvq_status kvq_cache_layout(const kvq_cache_desc* desc, int32_t batch, int32_t which,
                            kvq_plane_layout* out);

/* Bytes to allocate for the K (which = 0) or V (which = 1) cache; 0 on error. */
KVQ_API size_t kvq_cache_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t which);

/* Split count the library picks for this problem on the current device
 * (n_splits = 0 in kvq_decode_attention means this value); >= 1, or 0 on error. */
KVQ_API int32_t kvq_auto_splits(const kvq_cache_desc* desc, int32_t batch, int64_t ctx_len);

/* Workspace bytes kvq_decode_attention / kvq_combine / kvq_decode_step need
 * for n_splits (0 = automatic, resolved as kvq_auto_splits would for ctx_len =
 * max_ctx); 0 on error.  Layout: uint32 arrival counters [batch][n_kv_heads]
 * and uint32 epoch words [batch][n_kv_heads] (used by kvq_decode_step only),
 * then one uint32 status word (see kvq_workspace_status_offset) -- the place
 * of these does not depend on n_splits -- then m and l fp32 [batch][n_q][S]
 * each, then acc fp32 [batch][n_q][S][head_dim], each part 256-byte aligned. */
KVQ_API size_t kvq_workspace_bytes(const kvq_cache_desc* desc, int32_t batch, int32_t n_splits);

/* Byte offset of the workspace's status word for `batch` (the same for every
 * split count).  The decode kernels OR bits into it when something made them
 * write NaN instead of a result, and never clear it:
 *   bit 0  a wait for a cache tile's copy gave up (bounded at about 2 s);
 *   bit 1  kvq_decode_step: a wait in the in-kernel combine gave up (another
 *          CTA's arrival or copy never came, e.g. a workspace whose arrival
 *          counters were not zero);
 *   bit 2  paged decode: a block-table entry outside [0, n_pages).
 * The affected outputs are NaN.  To check a call, zero the word before it and
 * read it back (a 4-byte device-to-host copy on the same stream) after it; the
 * library itself neither reads nor clears it.  Host only. */
KVQ_API kvq_status kvq_workspace_status_offset(const kvq_cache_desc* desc, int32_t batch, size_t* offset);

/* The turbo3 codebook this library uses: 8 binary32 levels (ascending) and
 * the 7 binary32 thresholds between them.  Host only; no device needed. */
KVQ_API kvq_status kvq_turbo3_codebook(float levels[8], float thresholds[7]);

/* The codebook of a turbo type (KVQ_TURBO2, KVQ_TURBO3, KVQ_TURBO4; for
 * KVQ_TURBO3_QJL the 4-level codebook of its 2-bit codes): its 2^b binary32
 * levels (ascending) into levels[] and the 2^b - 1 binary32 thresholds into
 * thresholds[] (room for 16 and 15).  Host only. */
KVQ_API kvq_status kvq_turbo_codebook(int32_t type, float* levels, float* thresholds);

/* The turbo3 sign vector (+1.f / -1.f) for `seed`, head_dim entries (every
 * turbo type uses it).  Host only. */
KVQ_API kvq_status kvq_turbo3_signs(uint64_t seed, int32_t head_dim, float* signs);

/*
 * Quantize-on-append: writes n_tok new rows per (batch, KV head) into both
 * caches at rows pos .. pos+n_tok-1 (the CPY step that precedes attention in
 * the llama.cpp issue's failing path, "Possibly related": unsupported "CPY").
 *   k_cache, v_cache  device, layouts from kvq_cache_layout(desc, batch, 0/1)
 *   k_new, v_new      device fp16 [batch][n_tok][n_kv_heads][head_dim]
 *   pos >= 0, n_tok >= 1, pos + n_tok <= max_ctx.
 * Either cache/row pair may be NULL to skip that tensor (not both).
 * Quantized bytes are deterministic and bit-exact to the formats above.
 */
KVQ_API kvq_status kvq_append_quantize(const kvq_cache_desc* desc, void* k_cache, void* v_cache,
                               const void* k_new, const void* v_new, int32_t batch,
                               int64_t pos, int32_t n_tok, void* cuda_stream);

/*
 * Split-KV decode: for every (batch b, query head h, split s) writes the
 * partial softmax state of rows in split s to the workspace:
 *   m  = max_t s_t * log2(e)       (scores in base-2 units; -inf if empty)
 *   l  = sum_t 2^(s_t*log2(e) - m)
 *   acc= sum_t 2^(s_t*log2(e) - m) * v_hat_t   (turbo3: in the rotated domain,
 *        acc = sum_t p_t * norm_t * c[code_t], before the inverse transform)
 * with s_t = softmax_scale * <q_h, k_hat_t>.
 *   q              device fp16 [batch][n_q_heads][head_dim]
 *   ctx_len        1 <= ctx_len <= max_ctx rows attended
 *   n_splits       0 = kvq_auto_splits, else 1 .. 4096
 *   workspace      device, >= kvq_workspace_bytes(desc, batch, n_splits)
 */
KVQ_API kvq_status kvq_decode_attention(const kvq_cache_desc* desc, const void* k_cache,
                                const void* v_cache, const void* q, int32_t batch,
                                int64_t ctx_len, float softmax_scale, int32_t n_splits,
                                void* workspace, size_t workspace_bytes, void* cuda_stream);

/*
 * Combine: merges the n_splits partials of kvq_decode_attention into
 *   out[b][h] = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,  M = max_s m_s,
 * and for a turbo3 value cache applies the inverse rotation s * H_un * (.) / d.
 *   n_splits must equal the value kvq_decode_attention used (after resolving 0,
 *   pass the same 0 and the same ctx_len).
 *   out            device fp32 [batch][n_q_heads][head_dim]
 */
KVQ_API kvq_status kvq_combine(const kvq_cache_desc* desc, const void* workspace,
                       size_t workspace_bytes, int32_t batch, int64_t ctx_len,
                       int32_t n_splits, float* out, void* cuda_stream);

/*
 * Context split across GPUs.  The sequences' rows are spread over n_ranks GPUs
 * (any partition, a rank may hold none of a sequence's rows).  Each rank runs
 * kvq_decode_attention (or _varlen) over its own rows with the same explicit
 * n_splits.  The ranks' partial regions (m, l, acc; kvq_partials_region) are
 * then gathered rank after rank into one buffer, and kvq_combine_ranks merges
 * all n_ranks * n_splits partials.  Partials merge exactly, so the output is
 * that of one decode over all the rows, up to fp32 rounding order (section
 * "Flash Attention" of "llama.cpp für Geschwindigkeit und Speicher optimieren":
 * the tiled softmax is exact).
 *   kvq_partials_region: byte offset and size of the partials inside a
 *     workspace for (batch, n_splits); host only.
 *   partials: device, n_ranks regions of that size back to back, 16-byte
 *     aligned (an all-gather of each rank's region).
 *   n_ranks * n_splits <= 8192.
 */
KVQ_API kvq_status kvq_partials_region(const kvq_cache_desc* desc, int32_t batch, int32_t n_splits,
                                       size_t* offset, size_t* bytes);
KVQ_API kvq_status kvq_combine_ranks(const kvq_cache_desc* desc, const void* partials, int32_t n_ranks,
                                     int32_t batch, int32_t n_splits, float* out, void* cuda_stream);

/*
 * Allocation-free decode: kvq_decode_attention followed by kvq_combine, with the
 * split partials kept in scratch memory that the library itself owns, so the
 * caller passes only inputs and the output.  The pages have no counterpart; it
 * exists for callers that cannot allocate device memory when they decode (a
 * fixed memory arena handed out up front, a process that must not call the
 * allocator during another stream's graph capture, a foreign-language host that
 * only passes pointers it was given).
 *   Scratch: one 8 MiB array in each GPU's memory (a file-scope __device__
 *   variable), reserved when the CUDA runtime loads the library's module on
 *   that GPU -- at context creation under eager module loading
 *   (CUDA_MODULE_LOADING=EAGER), at the module's first use under lazy loading
 *   -- and held until the process exits.  Problems whose workspace
 *   (kvq_workspace_bytes for the split count used) exceeds 8 MiB return
 *   KVQ_ERR_WORKSPACE without launching anything when n_splits is given; with
 *   n_splits = 0 the automatic count is lowered to the largest count whose
 *   partials fit (KVQ_ERR_WORKSPACE only if even one split does not fit).
 *   Set-up: the first call on a GPU looks up the array's device address there
 *   (cudaGetSymbolAddress, with that GPU current); make that first call before
 *   any stream capture.  The address is kept for the life of the process, so
 *   this entry point must not be used after cudaDeviceReset (or anything else
 *   that destroys the device's primary context) in the same process.
 *   Sharing: every call on a GPU uses the same array, which keeps the previous
 *   call's contents (each call writes every entry before reading it back).
 *   Calls that overlap on the GPU (unordered streams) race and give wrong
 *   results; order them on one stream or use kvq_decode_attention with a
 *   workspace of your own.
 *   Arguments are those of kvq_decode_attention and kvq_combine;
 *   out is device fp32 [batch][n_q_heads][head_dim], 16-byte aligned.
 */
KVQ_API kvq_status kvq_decode_attention_noalloc(const kvq_cache_desc* desc, const void* k_cache,
                                                const void* v_cache, const void* q, int32_t batch,
                                                int64_t ctx_len, float softmax_scale, int32_t n_splits,
                                                float* out, void* cuda_stream);

/*
 * Fused decode step: one launch that does what kvq_append_quantize (one new
 * row per batch entry, at row ctx_len - 1), kvq_decode_attention (rows
 * 0 .. ctx_len-1, the new row included) and kvq_combine do one after the
 * other.  The pages have no such call: it is the decode loop's "append, then
 * attend" (the CPY step before flash attention in the llama.cpp issue,
 * "Possibly related") in one kernel, so a layer step costs one launch.
 *   k_new, v_new   device fp16 [batch][n_kv_heads][head_dim], 16-byte aligned
 *   out            device fp32 [batch][n_q_heads][head_dim], 16-byte aligned
 *   other arguments as in kvq_decode_attention; ctx_len counts the new row.
 * The CTA whose split holds row ctx_len - 1 writes the new rows before it reads
 * any cache row; the last CTAs of each (batch, KV head) to finish combine the
 * group's splits, a share of its query heads each.  The workspace's arrival
 * counters (see kvq_workspace_bytes) must be zero before the first call with a
 * workspace, and every completed call leaves them zero; the epoch words may
 * hold any value.  Calls sharing a workspace must be ordered (one stream).
 * Cached bytes are identical to kvq_append_quantize's; out agrees with
 * kvq_decode_attention + kvq_combine up to fp32 rounding order.
 */
KVQ_API kvq_status kvq_decode_step(const kvq_cache_desc* desc, void* k_cache, void* v_cache,
                                   const void* q, const void* k_new, const void* v_new,
                                   int32_t batch, int64_t ctx_len, float softmax_scale,
                                   int32_t n_splits, void* workspace, size_t workspace_bytes,
                                   float* out, void* cuda_stream);

/*
 * Per-sequence context lengths.  A server's cache holds several sequences (the
 * llama.cpp issue "Eval bug: Metal fails mixed quantized KV on Apple Silicon
 * when Flash Attention is unavailable, ...": the kv-cache line in a comment's
 * "Relevant output" reports 4/1 sequences), and the sequences of one batch need
 * not have equal lengths.  These forms take the lengths from device memory, so a
 * captured CUDA graph can be replayed as the lengths grow, with no host round
 * trip.
 *   ctx_lens      device int32 [batch], 4-byte aligned; read by the kernels when
 *                 they run.
 *   max_ctx_len   host bound on the lengths, 1 <= max_ctx_len <= max_ctx.  It
 *                 takes ctx_len's place in the split choice (n_splits = 0),
 *                 in kvq_workspace_bytes and in kvq_combine.
 * Batch row b attends rows [0, ctx_lens[b]), cut into n_splits chunks of its
 * own (a multiple of 32 rows each; trailing splits may be empty).  A length
 * outside [1, max_ctx_len] attends no row: that row reads no cache byte, every
 * split partial is empty (m = -inf, l = 0), and the combined output is NaN.
 * Nothing is read or written out of bounds, whatever the lengths hold.
 */
KVQ_API kvq_status kvq_decode_attention_varlen(const kvq_cache_desc* desc, const void* k_cache,
                                               const void* v_cache, const void* q, int32_t batch,
                                               const int32_t* ctx_lens, int64_t max_ctx_len,
                                               float softmax_scale, int32_t n_splits, void* workspace,
                                               size_t workspace_bytes, void* cuda_stream);

/*
 * kvq_decode_step with per-sequence lengths: batch row b's new K/V row is
 * written at row ctx_lens[b] - 1, then rows [0, ctx_lens[b]) are attended.  A
 * row whose length lies outside [1, max_ctx_len] writes nothing to the caches,
 * and its output is NaN.
 */
KVQ_API kvq_status kvq_decode_step_varlen(const kvq_cache_desc* desc, void* k_cache, void* v_cache,
                                          const void* q, const void* k_new, const void* v_new,
                                          int32_t batch, const int32_t* ctx_lens, int64_t max_ctx_len,
                                          float softmax_scale, int32_t n_splits, void* workspace,
                                          size_t workspace_bytes, float* out, void* cuda_stream);

/*
 * kvq_append_quantize with per-sequence positions: batch row b's n_tok rows
 * land at rows lens[b] - n_tok .. lens[b] - 1.  lens holds each sequence's
 * length after the append: device int32 [batch], 4-byte aligned, read by the
 * kernel.  A row whose lens[b] lies outside [n_tok, max_ctx] is not written.
 * The stored bytes are those kvq_append_quantize writes at the same positions.
 */
KVQ_API kvq_status kvq_append_quantize_varlen(const kvq_cache_desc* desc, void* k_cache, void* v_cache,
                                              const void* k_new, const void* v_new, int32_t batch,
                                              const int32_t* lens, int32_t n_tok, void* cuda_stream);

/*
 * Paged pools.  Sequences grow and finish at different times, so a server keeps
 * their rows in fixed-size pages drawn from one pool instead of one max_ctx
 * slab per sequence.  A pool tensor (K or V of one layer) has exactly the
 * layout of a contiguous cache of batch = n_pages and max_ctx = page_rows:
 *   code plane  [n_pages][n_kv_heads][page_rows][code_bytes]
 *   scale plane [n_pages][n_kv_heads][page_rows][n_scales] fp16, 256-aligned offset
 * Logical row r of sequence b is row r mod page_rows of page
 * block_table[b * max_pages + r / page_rows].  Rows are those of the formats
 * above, byte for byte.  Sequence lengths are per sequence (as in the _varlen
 * calls) and at most min(max_ctx, max_pages * page_rows).  A block-table entry
 * that is read and is not in [0, n_pages) is never dereferenced: the
 * rows that would go there are not written, and a decode that meets one
 * makes that sequence's output NaN.
 */
KVQ_API kvq_status kvq_paged_layout(const kvq_cache_desc* desc, int32_t page_rows, int64_t n_pages,
                                    int32_t which, kvq_plane_layout* out);

/* Bytes to allocate for a K (which = 0) or V (which = 1) pool; 0 on error. */
KVQ_API size_t kvq_paged_cache_bytes(const kvq_cache_desc* desc, int32_t page_rows, int64_t n_pages,
                                     int32_t which);

/* kvq_append_quantize_varlen into a pool: sequence b's n_tok new rows go to
 * logical rows lens[b] - n_tok .. lens[b] - 1 (lens: its length after the
 * append, device int32 [batch]); a sequence whose length lies outside
 * [n_tok, capacity] is not written. */
KVQ_API kvq_status kvq_append_quantize_paged(const kvq_cache_desc* desc, void* k_pool, void* v_pool,
                                             const void* k_new, const void* v_new, int32_t batch,
                                             const kvq_paged* pages, const int32_t* lens, int32_t n_tok,
                                             void* cuda_stream);

/* kvq_decode_attention_varlen over a pool (max_ctx_len <= the capacity). */
KVQ_API kvq_status kvq_decode_attention_paged(const kvq_cache_desc* desc, const void* k_pool,
                                              const void* v_pool, const void* q, int32_t batch,
                                              const kvq_paged* pages, const int32_t* ctx_lens,
                                              int64_t max_ctx_len, float softmax_scale, int32_t n_splits,
                                              void* workspace, size_t workspace_bytes, void* cuda_stream);

/* kvq_decode_step_varlen over a pool: sequence b's new row goes to logical row
 * ctx_lens[b] - 1, through the block table, before it is read back. */
KVQ_API kvq_status kvq_decode_step_paged(const kvq_cache_desc* desc, void* k_pool, void* v_pool,
                                         const void* q, const void* k_new, const void* v_new,
                                         int32_t batch, const kvq_paged* pages, const int32_t* ctx_lens,
                                         int64_t max_ctx_len, float softmax_scale, int32_t n_splits,
                                         void* workspace, size_t workspace_bytes, float* out,
                                         void* cuda_stream);

#ifdef __cplusplus
}
#endif

#endif /* KVQ_H */
