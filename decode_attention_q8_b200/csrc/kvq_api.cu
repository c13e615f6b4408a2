// libkvq C ABI: argument checks, cache layout, split selection, the turbo3
// constants (sign vector, codebook) and kernel launches.  Declarations and the
// format definitions are in include/kvq.h.
//
// Error convention ("Eval bug: Metal fails mixed quantized KV on Apple Silicon
// when Flash Attention is unavailable, ...", section "Expected behavior"): an
// unsupported combination is rejected early and cleanly -- every check runs on
// the host before any launch, and an error status means nothing was launched.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>
#include <string>

#include "kvq_internal.h"

namespace kvq {

int64_t rows_per_plane(int64_t max_ctx) { return (max_ctx + kRowAlign - 1) / kRowAlign * kRowAlign; }

int32_t code_bytes_of(int32_t type, int32_t d) {
  switch (type) {
    case KVQ_F16: return 2 * d;
    case KVQ_Q8_0: return d;
    case KVQ_Q4_0:
    case KVQ_Q5_0: return d / 2;
    case KVQ_TURBO2:
    case KVQ_TURBO3:
    case KVQ_TURBO4: return turbo_bits(type) * d / 8;
    case KVQ_TURBO3_QJL: return 3 * d / 8;
  }
  return 0;
}

int32_t n_scales_of(int32_t type, int32_t d) {
  switch (type) {
    case KVQ_F16: return 0;
    case KVQ_Q8_0:
    case KVQ_Q4_0: return d / kBlock;
    case KVQ_Q5_0: return 3 * d / kBlock;
    case KVQ_TURBO2:
    case KVQ_TURBO3:
    case KVQ_TURBO4: return 1;
    case KVQ_TURBO3_QJL: return 2;
  }
  return 0;
}

namespace {

thread_local std::string g_last_cuda_error;

constexpr int64_t kMaxCtx = (int64_t)1 << 31;
constexpr int64_t kMinChunk = 256;  // fewest rows per split the heuristic plans

bool known_type(int32_t t) { return t >= KVQ_F16 && t <= KVQ_TURBO3_QJL; }
bool pow2(int32_t v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned(const void* p, uintptr_t a) { return ((uintptr_t)p % a) == 0; }
int64_t round_up(int64_t v, int64_t a) { return (v + a - 1) / a * a; }

kvq_status cuda_fail(cudaError_t e) {
  g_last_cuda_error = cudaGetErrorString(e);
  return KVQ_ERR_CUDA;
}

// ---- turbo3 constants ------------------------------------------------------

// splitmix64 (Steele, Lea & Flood 2014): advance the state by the golden-ratio
// increment, then two xor-shift-multiply rounds and a final xor-shift.
uint64_t splitmix64_next(uint64_t& state) {
  state += 0x9E3779B97F4A7C15ull;
  uint64_t z = state;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

void sign_bits(uint64_t seed, int32_t d, uint32_t out[kMaxHeadDim / 32]) {
  std::memset(out, 0, sizeof(uint32_t) * (kMaxHeadDim / 32));
  uint64_t st = seed;
  for (int i = 0; i < d; ++i)
    if (splitmix64_next(st) >> 63) out[i >> 5] |= 1u << (i & 31);
}

// n-level Lloyd-Max quantizer of N(0,1) (n = 4, 8, 16) by Lloyd's iteration in
// double: thresholds are midpoints of neighbouring levels, each level is the
// mean of N(0,1) on its cell, (phi(a) - phi(b)) / (Q(a) - Q(b)) with Q the
// upper tail.  Symmetric: the positive half is iterated with the middle
// threshold at 0.
struct Codebook {
  int n;
  float levels[16];
  float tau[15];
};

double npdf(double x) { return std::exp(-0.5 * x * x) * 0.39894228040143267794; }
double upper_tail(double x) { return 0.5 * std::erfc(x * 0.70710678118654752440); }

Codebook compute_codebook(int n) {
  const int m = n / 2;
  double c[8];
  for (int k = 0; k < m; ++k) c[k] = 2.5 * (k + 0.5) / m;  // start spread over [0, 2.5]
  for (int it = 0; it < 400000; ++it) {
    double t[9];
    t[0] = 0.0;
    for (int k = 1; k < m; ++k) t[k] = 0.5 * (c[k - 1] + c[k]);
    t[m] = INFINITY;
    double next[8];
    double change = 0.0;
    for (int k = 0; k < m; ++k) {
      const double pa = npdf(t[k]), qa = upper_tail(t[k]);
      const double pb = std::isinf(t[k + 1]) ? 0.0 : npdf(t[k + 1]);
      const double qb = std::isinf(t[k + 1]) ? 0.0 : upper_tail(t[k + 1]);
      next[k] = (pa - pb) / (qa - qb);
      change = std::fmax(change, std::fabs(next[k] - c[k]));
    }
    std::memcpy(c, next, sizeof(double) * m);
    if (change < 1e-15) break;
  }
  double lv[16];
  for (int k = 0; k < m; ++k) {
    lv[m + k] = c[k];
    lv[m - 1 - k] = -c[k];
  }
  Codebook cb{};
  cb.n = n;
  for (int k = 0; k < n; ++k) cb.levels[k] = (float)lv[k];
  for (int k = 0; k + 1 < n; ++k) cb.tau[k] = (float)(0.5 * (lv[k] + lv[k + 1]));
  return cb;
}

// The codebook of turbo type t, computed once per width.
const Codebook& codebook(int32_t t) {
  static std::once_flag once;
  static Codebook cb[3];
  std::call_once(once, [] {
    for (int b = 2; b <= 4; ++b) cb[b - 2] = compute_codebook(1 << b);
  });
  return cb[turbo_bits(t) - 2];
}

TurboConsts turbo_consts(const kvq_cache_desc* d, int32_t type) {
  TurboConsts t{};
  const Codebook& cb = codebook(type);
  std::memcpy(t.levels, cb.levels, sizeof(t.levels));
  std::memcpy(t.tau, cb.tau, sizeof(t.tau));
  sign_bits(d->turbo_seed, d->head_dim, t.sign_bits);
  if (is_qjl(type)) {
    const uint64_t addr = (uint64_t)(uintptr_t)d->qjl_proj;
    const uint32_t lo = (uint32_t)addr, hi = (uint32_t)(addr >> 32);
    std::memcpy(&t.tau[kQjlSlot], &lo, 4);
    std::memcpy(&t.tau[kQjlSlot + 1], &hi, 4);
    t.tau[kQjlSlot + 2] = (float)(1.0 / std::sqrt((double)d->head_dim));
  }
  return t;
}

// turbo3_qjl keys read their projection: present and 16-byte aligned.
bool qjl_ok(const kvq_cache_desc* d) {
  return !is_qjl(d->k_type) || (d->qjl_proj != nullptr && aligned(d->qjl_proj, 16));
}

// ---- splits -----------------------------------------------------------------

int sm_count() {
  int dev = 0, n = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) {
    (void)cudaGetLastError();
    return 148;  // B200
  }
  return n;
}

// Splits for `units` independent (batch, KV head) rows of work over ctx rows:
// as many as the context allows (>= kMinChunk rows each) up to S*, where S*
// maximises the fraction of CTA slots busy over the waves it takes, less 2%
// per extra wave.  Non-decreasing in ctx.
int32_t choose_splits(int64_t units, int64_t ctx, int sms, int per_sm) {
  const int64_t slots = (int64_t)sms * per_sm;
  const int64_t cap = std::max<int64_t>(1, std::min<int64_t>(kMaxSplits, (ctx + kMinChunk - 1) / kMinChunk));
  const int64_t s_min = std::max<int64_t>(1, (slots + units - 1) / units);
  const int64_t s_hi = std::min<int64_t>(kMaxSplits, 4 * s_min);
  int64_t best = 1;
  double best_score = -1e30;
  for (int64_t s = 1; s <= s_hi; ++s) {
    const int64_t ctas = units * s;
    const int64_t waves = (ctas + slots - 1) / slots;
    const double score = (double)ctas / (double)(waves * slots) - 0.02 * (double)(waves - 1);
    if (score > best_score + 1e-12) {
      best_score = score;
      best = s;
    }
  }
  return (int32_t)std::min(best, cap);
}

int64_t chunk_rows(int64_t ctx, int32_t S) { return round_up((ctx + S - 1) / S, kSplitAlign); }

// CTAs per (batch row, KV head) that share the fused step's combine: the last
// arrivals, one per 48 (head, split) partials of the group (at most one per
// head), once a group has more than 200 of them.  Waking a waiting CTA costs
// about a microsecond, which pays only when one CTA would pull the partials
// through its shared memory in several rounds (measured: 8 heads x 37 splits
// 0.6-0.9 us faster; 4 x 37 and 8 x 9 as fast or slower).  All but the last
// arrival wait for it, so the waiting CTAs may hold at most half of the GPU's
// CTA slots; the CTAs they wait for can then always be scheduled.
int32_t combining_ctas(const kvq_cache_desc* d, int32_t batch, int32_t S) {
  const int32_t G = d->n_q_heads / d->n_kv_heads;
  const int64_t groups = (int64_t)batch * d->n_kv_heads;
  const int64_t slots = (int64_t)sm_count() * decode_ctas_per_sm(d->k_type, d->v_type, d->head_dim, G);
  if ((int64_t)G * S <= 200) return 1;
  int32_t k = (int32_t)std::min<int64_t>(G, (int64_t)G * S / 48);
  while (k > 1 && (int64_t)(k - 1) * groups * 2 > slots) --k;
  return std::max(k, 1);
}

// Upper bound of the automatic split count over ctx_len <= ctx (sizes the
// workspace for n_splits = 0).
int32_t auto_splits_bound(const kvq_cache_desc* d, int32_t batch, int64_t ctx) {
  return choose_splits((int64_t)batch * d->n_kv_heads, ctx, sm_count(),
                       decode_ctas_per_sm(d->k_type, d->v_type, d->head_dim, d->n_q_heads / d->n_kv_heads));
}

// Explicit counts are used as given (trailing splits may be empty); the
// automatic count drops the splits that rounding the chunk to 32 rows leaves
// empty, so it never exceeds auto_splits_bound(max_ctx).
int32_t resolve_splits(const kvq_cache_desc* d, int32_t batch, int64_t ctx, int32_t n_splits) {
  if (n_splits > 0) return n_splits;
  const int32_t S = auto_splits_bound(d, batch, ctx);
  return (int32_t)((ctx + chunk_rows(ctx, S) - 1) / chunk_rows(ctx, S));
}

struct WsLayout {
  int64_t m_off, l_off, acc_off, cnt_off, status_off, total;
};

// Counters first (arrival counters, then epoch words, one of each per group,
// then the status word): their place depends on batch and n_kv only, so calls
// with different split counts on one workspace keep them intact.
WsLayout ws_layout(const kvq_cache_desc* d, int32_t batch, int32_t S) {
  WsLayout w;
  const int64_t rows = (int64_t)batch * d->n_q_heads * S;
  w.cnt_off = 0;
  w.status_off = (int64_t)batch * d->n_kv_heads * 8;
  w.m_off = round_up(w.status_off + 4, 256);
  w.l_off = w.m_off + round_up(rows * 4, 256);
  w.acc_off = w.l_off + round_up(rows * 4, 256);
  w.total = w.acc_off + rows * d->head_dim * 4;
  return w;
}

// Byte layout of `planes` planes of T rows of a tensor of `type`.
void fill_layout(int32_t type, int32_t D, int64_t planes, int64_t T, kvq_plane_layout* out) {
  const int64_t cb = code_bytes_of(type, D);
  const int64_t ns = n_scales_of(type, D);
  out->rows_per_plane = T;
  out->code_bytes = cb;
  out->n_scales = ns;
  out->scale_offset = round_up(planes * T * cb, 256);
  out->total_bytes = out->scale_offset + planes * T * ns * 2;
}

// A paged pool's layout: the contiguous layout with the pages as batch rows and
// the page rows as the rows per plane.
kvq_status check_pool(const kvq_cache_desc* d, int32_t page_rows, int64_t n_pages) {
  if (n_pages < 1) return KVQ_ERR_INVALID;
  if (page_rows < 32 || page_rows > (1 << 20) || !pow2(page_rows)) return KVQ_ERR_UNSUPPORTED;
  if (n_pages * d->n_kv_heads >= ((int64_t)1 << 31)) return KVQ_ERR_UNSUPPORTED;  // 32-bit plane coordinates
  const double approx = (double)n_pages * d->n_kv_heads * (double)page_rows * (2.0 * d->head_dim + 16.0);
  if (approx > 9.0e18) return KVQ_ERR_INVALID;
  return KVQ_OK;
}

kvq_status check_paged(const kvq_cache_desc* d, const kvq_paged* pg) {
  if (!pg || !pg->block_table || !aligned(pg->block_table, 4) || pg->max_pages < 1) return KVQ_ERR_INVALID;
  return check_pool(d, pg->page_rows, pg->n_pages);
}

int32_t log2_of(int64_t v) {
  int32_t l = 0;
  while (((int64_t)1 << l) < v) ++l;
  return l;
}

// Longest sequence a paged pool's block table can address, within max_ctx.
int64_t paged_capacity(const kvq_cache_desc* d, const kvq_paged* pg) {
  return std::min<int64_t>(d->max_ctx, (int64_t)pg->max_pages * pg->page_rows);
}

Plane pool_plane_of(const kvq_cache_desc* d, const kvq_paged* pg, int which, void* base) {
  kvq_plane_layout L;
  fill_layout(which ? d->v_type : d->k_type, d->head_dim, pg->n_pages * d->n_kv_heads, pg->page_rows, &L);
  Plane p;
  p.codes = static_cast<uint8_t*>(base);
  p.scales = reinterpret_cast<__half*>(static_cast<uint8_t*>(base) + L.scale_offset);
  p.T = L.rows_per_plane;
  p.code_bytes = (int32_t)L.code_bytes;
  p.n_scales = (int32_t)L.n_scales;
  return p;
}

Plane plane_of(const kvq_cache_desc* d, int32_t batch, int which, void* base) {
  kvq_plane_layout L;
  kvq_cache_layout(d, batch, which, &L);
  Plane p;
  p.codes = static_cast<uint8_t*>(base);
  p.scales = reinterpret_cast<__half*>(static_cast<uint8_t*>(base) + L.scale_offset);
  p.T = L.rows_per_plane;
  p.code_bytes = (int32_t)L.code_bytes;
  p.n_scales = (int32_t)L.n_scales;
  return p;
}


// Checks and fills the parameters of a decode launch (kvq_decode_attention and
// kvq_decode_step, and their per-sequence-length forms, where ctx_len is the
// bound on the lengths); a plain decode appends nothing and writes partials only.
kvq_status fill_decode(const kvq_cache_desc* d, const void* k_cache, const void* v_cache, const void* q,
                       int32_t batch, int64_t ctx_len, const int32_t* ctx_lens, const kvq_paged* pg,
                       float softmax_scale, int32_t n_splits, void* workspace, size_t workspace_bytes,
                       DecodeParams* out) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (pg != nullptr) {
    if ((st = check_paged(d, pg)) != KVQ_OK) return st;
    if (ctx_len > paged_capacity(d, pg)) return KVQ_ERR_INVALID;
  }
  if (!k_cache || !v_cache || !q || !workspace) return KVQ_ERR_INVALID;
  if (batch < 1 || batch > 65535 || ctx_len < 1 || ctx_len > d->max_ctx) return KVQ_ERR_INVALID;
  if (n_splits < 0 || n_splits > kMaxSplits || !std::isfinite(softmax_scale)) return KVQ_ERR_INVALID;
  if (!aligned(k_cache, 256) || !aligned(v_cache, 256) || !aligned(q, 16) || !aligned(workspace, 256))
    return KVQ_ERR_INVALID;
  if (ctx_lens != nullptr && !aligned(ctx_lens, 4)) return KVQ_ERR_INVALID;
  if (!qjl_ok(d)) return KVQ_ERR_INVALID;
  const int32_t G = d->n_q_heads / d->n_kv_heads;
  if (!decode_supported(d->k_type, d->v_type, G, d->head_dim)) return KVQ_ERR_UNSUPPORTED;
  const int32_t S = resolve_splits(d, batch, ctx_len, n_splits);
  const WsLayout w = ws_layout(d, batch, S);
  if (workspace_bytes < (size_t)w.total) return KVQ_ERR_WORKSPACE;

  DecodeParams& p = *out;
  p = DecodeParams{};
  p.k = pg ? pool_plane_of(d, pg, 0, const_cast<void*>(k_cache)) : plane_of(d, batch, 0, const_cast<void*>(k_cache));
  p.v = pg ? pool_plane_of(d, pg, 1, const_cast<void*>(v_cache)) : plane_of(d, batch, 1, const_cast<void*>(v_cache));
  if (pg) {
    p.block_table = pg->block_table;
    p.max_pages = pg->max_pages;
    p.log2_page = log2_of(pg->page_rows);
    p.n_pages = pg->n_pages;
  }
  p.q = static_cast<const __half*>(q);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  p.ws_m = reinterpret_cast<float*>(ws + w.m_off);
  p.ws_l = reinterpret_cast<float*>(ws + w.l_off);
  p.ws_acc = reinterpret_cast<float*>(ws + w.acc_off);
  p.status = reinterpret_cast<uint32_t*>(ws + w.status_off);
  p.B = batch;
  p.n_q = d->n_q_heads;
  p.n_kv = d->n_kv_heads;
  p.G = G;
  p.D = d->head_dim;
  p.S = S;
  p.ctx = ctx_len;
  p.chunk = chunk_rows(ctx_len, S);
  p.ctx_lens = ctx_lens;
  p.qscale = softmax_scale * 1.4426950408889634f;
  if (is_turbo(d->v_type)) p.tq = turbo_consts(d, d->v_type);
  if (is_turbo(d->k_type)) p.tqk = turbo_consts(d, d->k_type);
  p.append_pos = -1;
  p.out = nullptr;
  p.counters = nullptr;
  return KVQ_OK;
}
kvq_status append_impl(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* k_new, const void* v_new,
                       int32_t batch, int64_t pos, const int32_t* lens, const kvq_paged* pg, int32_t n_tok,
                       void* stream) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (pg != nullptr && (st = check_paged(d, pg)) != KVQ_OK) return st;
  if (batch < 1 || batch > 65535 || n_tok < 1 || n_tok > d->max_ctx) return KVQ_ERR_INVALID;
  if (lens == nullptr && (pos < 0 || pos + n_tok > d->max_ctx)) return KVQ_ERR_INVALID;
  if (lens != nullptr && !aligned(lens, 4)) return KVQ_ERR_INVALID;
  const bool do_k = k_cache != nullptr, do_v = v_cache != nullptr;
  if (do_k != (k_new != nullptr) || do_v != (v_new != nullptr) || (!do_k && !do_v)) return KVQ_ERR_INVALID;
  if ((do_k && (!aligned(k_cache, 256) || !aligned(k_new, 16))) ||
      (do_v && (!aligned(v_cache, 256) || !aligned(v_new, 16))))
    return KVQ_ERR_INVALID;
  if (do_k && !qjl_ok(d)) return KVQ_ERR_INVALID;
  const int64_t rows = (int64_t)batch * n_tok * d->n_kv_heads;
  if (rows * (d->head_dim / 4) > ((int64_t)1 << 40)) return KVQ_ERR_UNSUPPORTED;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  AppendParams ap[2];
  for (int which = 0; which < 2; ++which) {
    void* cache = which ? v_cache : k_cache;
    if (!cache) continue;
    AppendParams& p = ap[which];
    p = AppendParams{};
    p.src = static_cast<const __half*>(which ? v_new : k_new);
    p.dst = pg ? pool_plane_of(d, pg, which, cache) : plane_of(d, batch, which, cache);
    p.B = batch;
    p.H = d->n_kv_heads;
    p.D = d->head_dim;
    p.n_tok = n_tok;
    p.pos = lens ? 0 : pos;
    p.lens = lens;
    p.len_max = pg ? paged_capacity(d, pg) : d->max_ctx;
    if (pg) {
      p.block_table = pg->block_table;
      p.max_pages = pg->max_pages;
      p.log2_page = log2_of(pg->page_rows);
      p.n_pages = pg->n_pages;
    }
    p.h_mul = div_multiplier((uint64_t)p.H);
    p.t_mul = div_multiplier((uint64_t)n_tok);
    const int32_t type = which ? d->v_type : d->k_type;
    if (is_turbo(type)) p.tq = turbo_consts(d, type);
  }
  const cudaError_t e = launch_append(do_k ? &ap[0] : nullptr, d->k_type, do_v ? &ap[1] : nullptr, d->v_type, s);
  if (e != cudaSuccess) return cuda_fail(e);
  return KVQ_OK;
}

kvq_status decode_impl(const kvq_cache_desc* d, const void* k_cache, const void* v_cache, const void* q,
                       int32_t batch, int64_t ctx_len, const int32_t* ctx_lens, const kvq_paged* pg,
                       float softmax_scale, int32_t n_splits, void* workspace, size_t workspace_bytes,
                       void* stream) {
  DecodeParams p{};
  const kvq_status st = fill_decode(d, k_cache, v_cache, q, batch, ctx_len, ctx_lens, pg, softmax_scale, n_splits,
                                    workspace, workspace_bytes, &p);
  if (st != KVQ_OK) return st;
  const cudaError_t e = launch_decode(d->k_type, d->v_type, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return KVQ_OK;
}

kvq_status step_impl(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* q, const void* k_new,
                     const void* v_new, int32_t batch, int64_t ctx_len, const int32_t* ctx_lens,
                     const kvq_paged* pg, float softmax_scale, int32_t n_splits, void* workspace,
                     size_t workspace_bytes, float* out, void* stream) {
  if (!k_new || !v_new || !out) return KVQ_ERR_INVALID;
  if (!aligned(k_new, 16) || !aligned(v_new, 16) || !aligned(out, 16)) return KVQ_ERR_INVALID;
  DecodeParams p{};
  const kvq_status st = fill_decode(d, k_cache, v_cache, q, batch, ctx_len, ctx_lens, pg, softmax_scale, n_splits,
                                    workspace, workspace_bytes, &p);
  if (st != KVQ_OK) return st;
  const WsLayout w = ws_layout(d, batch, p.S);
  p.append_pos = ctx_len - 1;  // with ctx_lens the kernel takes ctx_lens[b] - 1
  for (int which = 0; which < 2; ++which) {
    AppendParams& a = which ? p.app_v : p.app_k;
    a.src = static_cast<const __half*>(which ? v_new : k_new);
    a.dst = which ? p.v : p.k;
    a.B = batch;
    a.H = d->n_kv_heads;
    a.D = d->head_dim;
    a.n_tok = 1;
    a.pos = p.append_pos;
    a.lens = ctx_lens;
    a.len_max = ctx_len;
    a.block_table = p.block_table;
    a.max_pages = p.max_pages;
    a.log2_page = p.log2_page;
    a.n_pages = p.n_pages;
    a.h_mul = div_multiplier((uint64_t)a.H);
    a.t_mul = div_multiplier(1);
    const int32_t type = which ? d->v_type : d->k_type;
    if (is_turbo(type)) a.tq = turbo_consts(d, type);
  }
  p.out = out;
  // overlap with the previous kernel only where nothing the step reads before
  // the grid dependency resolves can come from it (no device lengths, no table)
  p.pdl = (d->flags & KVQ_FLAG_OVERLAP_PREVIOUS) && ctx_lens == nullptr && pg == nullptr ? 1 : 0;
  p.counters = reinterpret_cast<uint32_t*>(static_cast<uint8_t*>(workspace) + w.cnt_off);
  p.epochs = p.counters + (int64_t)batch * d->n_kv_heads;
  p.comb_ctas = combining_ctas(d, batch, p.S);
  const cudaError_t e = launch_decode(d->k_type, d->v_type, p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return KVQ_OK;
}

}  // namespace

void set_last_cuda_error(cudaError_t e) { g_last_cuda_error = cudaGetErrorString(e); }

}  // namespace kvq

using namespace kvq;

extern "C" {

const char* kvq_status_string(kvq_status s) {
  switch (s) {
    case KVQ_OK: return "ok";
    case KVQ_ERR_INVALID: return "invalid argument";
    case KVQ_ERR_UNSUPPORTED: return "unsupported configuration";
    case KVQ_ERR_WORKSPACE: return "workspace too small";
    case KVQ_ERR_CUDA: return "CUDA error";
  }
  return "unknown status";
}

const char* kvq_last_cuda_error(void) { return g_last_cuda_error.c_str(); }

size_t kvq_row_bytes(int32_t type, int32_t head_dim) {
  if (!known_type(type) || head_dim <= 0 || head_dim % kBlock || head_dim > kMaxHeadDim) return 0;
  if (is_turbo(type) && !pow2(head_dim)) return 0;
  return (size_t)code_bytes_of(type, head_dim) + 2 * (size_t)n_scales_of(type, head_dim);
}

kvq_status kvq_check_desc(const kvq_cache_desc* d) {
  if (!d) return KVQ_ERR_INVALID;
  if (d->n_q_heads < 1 || d->n_kv_heads < 1 || d->n_q_heads % d->n_kv_heads) return KVQ_ERR_INVALID;
  if (d->head_dim < 1 || (d->flags & ~KVQ_FLAG_OVERLAP_PREVIOUS) != 0) return KVQ_ERR_INVALID;
  if (d->max_ctx < 1 || d->max_ctx > kMaxCtx) return KVQ_ERR_INVALID;
  if (!known_type(d->k_type) || !known_type(d->v_type)) return KVQ_ERR_INVALID;
  if (d->head_dim % kBlock || d->head_dim > kMaxHeadDim) return KVQ_ERR_UNSUPPORTED;
  if ((is_turbo(d->k_type) || is_turbo(d->v_type)) && !pow2(d->head_dim)) return KVQ_ERR_UNSUPPORTED;
  if (is_qjl(d->v_type)) return KVQ_ERR_UNSUPPORTED;  // a key format
  if (d->n_kv_heads > 65535) return KVQ_ERR_UNSUPPORTED;
  return KVQ_OK;
}

kvq_status kvq_cache_layout(const kvq_cache_desc* d, int32_t batch, int32_t which, kvq_plane_layout* out) {
  const kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (!out || batch < 1 || batch > 65535 || (which != 0 && which != 1)) return KVQ_ERR_INVALID;
  const int32_t type = which ? d->v_type : d->k_type;
  const int64_t T = rows_per_plane(d->max_ctx);
  const int64_t planes = (int64_t)batch * d->n_kv_heads;
  const double approx = (double)planes * (double)T * (double)(code_bytes_of(type, d->head_dim) +
                                                             2 * n_scales_of(type, d->head_dim));
  if (approx > 9.0e18) return KVQ_ERR_INVALID;
  fill_layout(type, d->head_dim, planes, T, out);
  return KVQ_OK;
}

kvq_status kvq_paged_layout(const kvq_cache_desc* d, int32_t page_rows, int64_t n_pages, int32_t which,
                            kvq_plane_layout* out) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (!out || (which != 0 && which != 1)) return KVQ_ERR_INVALID;
  if ((st = check_pool(d, page_rows, n_pages)) != KVQ_OK) return st;
  fill_layout(which ? d->v_type : d->k_type, d->head_dim, n_pages * d->n_kv_heads, page_rows, out);
  return KVQ_OK;
}

size_t kvq_paged_cache_bytes(const kvq_cache_desc* d, int32_t page_rows, int64_t n_pages, int32_t which) {
  kvq_plane_layout L;
  if (kvq_paged_layout(d, page_rows, n_pages, which, &L) != KVQ_OK) return 0;
  return (size_t)L.total_bytes;
}

kvq_status kvq_append_quantize_paged(const kvq_cache_desc* d, void* k_pool, void* v_pool, const void* k_new,
                                     const void* v_new, int32_t batch, const kvq_paged* pages, const int32_t* lens,
                                     int32_t n_tok, void* stream) {
  if (!lens || !pages) return KVQ_ERR_INVALID;
  return append_impl(d, k_pool, v_pool, k_new, v_new, batch, 0, lens, pages, n_tok, stream);
}

kvq_status kvq_decode_attention_paged(const kvq_cache_desc* d, const void* k_pool, const void* v_pool, const void* q,
                                      int32_t batch, const kvq_paged* pages, const int32_t* ctx_lens,
                                      int64_t max_ctx_len, float softmax_scale, int32_t n_splits, void* workspace,
                                      size_t workspace_bytes, void* stream) {
  if (!ctx_lens || !pages) return KVQ_ERR_INVALID;
  return decode_impl(d, k_pool, v_pool, q, batch, max_ctx_len, ctx_lens, pages, softmax_scale, n_splits, workspace,
                     workspace_bytes, stream);
}

kvq_status kvq_decode_step_paged(const kvq_cache_desc* d, void* k_pool, void* v_pool, const void* q,
                                 const void* k_new, const void* v_new, int32_t batch, const kvq_paged* pages,
                                 const int32_t* ctx_lens, int64_t max_ctx_len, float softmax_scale,
                                 int32_t n_splits, void* workspace, size_t workspace_bytes, float* out,
                                 void* stream) {
  if (!ctx_lens || !pages) return KVQ_ERR_INVALID;
  return step_impl(d, k_pool, v_pool, q, k_new, v_new, batch, max_ctx_len, ctx_lens, pages, softmax_scale,
                   n_splits, workspace, workspace_bytes, out, stream);
}

size_t kvq_cache_bytes(const kvq_cache_desc* d, int32_t batch, int32_t which) {
  kvq_plane_layout L;
  if (kvq_cache_layout(d, batch, which, &L) != KVQ_OK) return 0;
  return (size_t)L.total_bytes;
}

int32_t kvq_auto_splits(const kvq_cache_desc* d, int32_t batch, int64_t ctx_len) {
  if (kvq_check_desc(d) != KVQ_OK || batch < 1 || ctx_len < 1 || ctx_len > d->max_ctx) return 0;
  return resolve_splits(d, batch, ctx_len, 0);
}

size_t kvq_workspace_bytes(const kvq_cache_desc* d, int32_t batch, int32_t n_splits) {
  if (kvq_check_desc(d) != KVQ_OK || batch < 1 || batch > 65535 || n_splits < 0 || n_splits > kMaxSplits) return 0;
  const int32_t S = n_splits > 0 ? n_splits : auto_splits_bound(d, batch, d->max_ctx);
  return (size_t)ws_layout(d, batch, S).total;
}

kvq_status kvq_workspace_status_offset(const kvq_cache_desc* d, int32_t batch, size_t* offset) {
  const kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (batch < 1 || batch > 65535 || offset == nullptr) return KVQ_ERR_INVALID;
  *offset = (size_t)ws_layout(d, batch, 1).status_off;
  return KVQ_OK;
}

kvq_status kvq_turbo3_codebook(float levels[8], float thresholds[7]) {
  return kvq_turbo_codebook(KVQ_TURBO3, levels, thresholds);
}

kvq_status kvq_turbo_codebook(int32_t type, float* levels, float* thresholds) {
  if (!levels || !thresholds || !is_turbo(type)) return KVQ_ERR_INVALID;
  const Codebook& cb = codebook(type);
  std::memcpy(levels, cb.levels, sizeof(float) * cb.n);
  std::memcpy(thresholds, cb.tau, sizeof(float) * (cb.n - 1));
  return KVQ_OK;
}

kvq_status kvq_turbo3_signs(uint64_t seed, int32_t head_dim, float* signs) {
  if (!signs || head_dim < 1 || head_dim > kMaxHeadDim) return KVQ_ERR_INVALID;
  uint32_t bits[kMaxHeadDim / 32];
  sign_bits(seed, head_dim, bits);
  for (int i = 0; i < head_dim; ++i) signs[i] = ((bits[i >> 5] >> (i & 31)) & 1u) ? -1.f : 1.f;
  return KVQ_OK;
}

kvq_status kvq_append_quantize(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* k_new,
                               const void* v_new, int32_t batch, int64_t pos, int32_t n_tok, void* stream) {
  return append_impl(d, k_cache, v_cache, k_new, v_new, batch, pos, nullptr, nullptr, n_tok, stream);
}

kvq_status kvq_append_quantize_varlen(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* k_new,
                                      const void* v_new, int32_t batch, const int32_t* lens, int32_t n_tok,
                                      void* stream) {
  if (!lens) return KVQ_ERR_INVALID;
  return append_impl(d, k_cache, v_cache, k_new, v_new, batch, 0, lens, nullptr, n_tok, stream);
}

kvq_status kvq_decode_attention(const kvq_cache_desc* d, const void* k_cache, const void* v_cache, const void* q,
                                int32_t batch, int64_t ctx_len, float softmax_scale, int32_t n_splits,
                                void* workspace, size_t workspace_bytes, void* stream) {
  return decode_impl(d, k_cache, v_cache, q, batch, ctx_len, nullptr, nullptr, softmax_scale, n_splits, workspace,
                     workspace_bytes, stream);
}

kvq_status kvq_decode_attention_varlen(const kvq_cache_desc* d, const void* k_cache, const void* v_cache,
                                       const void* q, int32_t batch, const int32_t* ctx_lens, int64_t max_ctx_len,
                                       float softmax_scale, int32_t n_splits, void* workspace,
                                       size_t workspace_bytes, void* stream) {
  if (!ctx_lens) return KVQ_ERR_INVALID;
  return decode_impl(d, k_cache, v_cache, q, batch, max_ctx_len, ctx_lens, nullptr, softmax_scale, n_splits,
                     workspace, workspace_bytes, stream);
}

kvq_status kvq_decode_step(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* q, const void* k_new,
                           const void* v_new, int32_t batch, int64_t ctx_len, float softmax_scale, int32_t n_splits,
                           void* workspace, size_t workspace_bytes, float* out, void* stream) {
  return step_impl(d, k_cache, v_cache, q, k_new, v_new, batch, ctx_len, nullptr, nullptr, softmax_scale, n_splits,
                   workspace, workspace_bytes, out, stream);
}

kvq_status kvq_decode_step_varlen(const kvq_cache_desc* d, void* k_cache, void* v_cache, const void* q,
                                  const void* k_new, const void* v_new, int32_t batch, const int32_t* ctx_lens,
                                  int64_t max_ctx_len, float softmax_scale, int32_t n_splits, void* workspace,
                                  size_t workspace_bytes, float* out, void* stream) {
  if (!ctx_lens) return KVQ_ERR_INVALID;
  return step_impl(d, k_cache, v_cache, q, k_new, v_new, batch, max_ctx_len, ctx_lens, nullptr, softmax_scale,
                   n_splits, workspace, workspace_bytes, out, stream);
}

kvq_status kvq_combine(const kvq_cache_desc* d, const void* workspace, size_t workspace_bytes, int32_t batch,
                       int64_t ctx_len, int32_t n_splits, float* out, void* stream) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (!workspace || !out) return KVQ_ERR_INVALID;
  if (batch < 1 || batch > 65535 || ctx_len < 1 || ctx_len > d->max_ctx) return KVQ_ERR_INVALID;
  if (n_splits < 0 || n_splits > kMaxSplits) return KVQ_ERR_INVALID;
  if (!aligned(workspace, 256) || !aligned(out, 16)) return KVQ_ERR_INVALID;
  const int32_t S = resolve_splits(d, batch, ctx_len, n_splits);
  const WsLayout w = ws_layout(d, batch, S);
  if (workspace_bytes < (size_t)w.total) return KVQ_ERR_WORKSPACE;
  CombineParams p{};
  const uint8_t* ws = static_cast<const uint8_t*>(workspace);
  p.ws_m = reinterpret_cast<const float*>(ws + w.m_off);
  p.ws_l = reinterpret_cast<const float*>(ws + w.l_off);
  p.ws_acc = reinterpret_cast<const float*>(ws + w.acc_off);
  p.out = out;
  p.B = batch;
  p.n_q = d->n_q_heads;
  p.D = d->head_dim;
  p.S = S;
  p.n_ranks = 1;
  p.rank_stride = 0;
  p.rotated = is_turbo(d->v_type);
  if (p.rotated) p.tq = turbo_consts(d, d->v_type);
  const cudaError_t e = launch_combine(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return KVQ_OK;
}

kvq_status kvq_partials_region(const kvq_cache_desc* d, int32_t batch, int32_t n_splits, size_t* offset,
                               size_t* bytes) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (!offset || !bytes || batch < 1 || batch > 65535 || n_splits < 1 || n_splits > kMaxSplits)
    return KVQ_ERR_INVALID;
  const WsLayout w = ws_layout(d, batch, n_splits);
  *offset = (size_t)w.m_off;
  *bytes = (size_t)(w.total - w.m_off);
  return KVQ_OK;
}

kvq_status kvq_combine_ranks(const kvq_cache_desc* d, const void* partials, int32_t n_ranks, int32_t batch,
                             int32_t n_splits, float* out, void* stream) {
  kvq_status st = kvq_check_desc(d);
  if (st != KVQ_OK) return st;
  if (!partials || !out || n_ranks < 1 || n_ranks > 4096) return KVQ_ERR_INVALID;
  if (batch < 1 || batch > 65535 || n_splits < 1 || n_splits > kMaxSplits) return KVQ_ERR_INVALID;
  if ((int64_t)n_ranks * n_splits > 8192) return KVQ_ERR_UNSUPPORTED;  // the combine's weight array
  if (!aligned(partials, 16) || !aligned(out, 16)) return KVQ_ERR_INVALID;
  const WsLayout w = ws_layout(d, batch, n_splits);
  const uint8_t* base = static_cast<const uint8_t*>(partials);
  CombineParams p{};
  p.ws_m = reinterpret_cast<const float*>(base);
  p.ws_l = reinterpret_cast<const float*>(base + (w.l_off - w.m_off));
  p.ws_acc = reinterpret_cast<const float*>(base + (w.acc_off - w.m_off));
  p.out = out;
  p.B = batch;
  p.n_q = d->n_q_heads;
  p.D = d->head_dim;
  p.S = n_splits;
  p.n_ranks = n_ranks;
  p.rank_stride = (w.total - w.m_off) / 4;
  p.rotated = is_turbo(d->v_type);
  if (p.rotated) p.tq = turbo_consts(d, d->v_type);
  const cudaError_t e = launch_combine(p, static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e);
  return KVQ_OK;
}

}  // extern "C"
