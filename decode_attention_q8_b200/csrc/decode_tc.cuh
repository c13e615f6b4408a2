// Split-KV decode attention over a quantized KV cache -- tensor-core version
// for sm_100a.
//
// What it computes is the decode form of flash attention ("llama.cpp für
// Geschwindigkeit und Speicher optimieren", section "Flash Attention": tiled,
// exactly standard attention): each CTA owns one (split, KV head, batch row),
// streams its contiguous slice of cache rows once for the whole GQA group of
// that KV head, keeps an online softmax and writes (m, l, acc) partials that
// kvq_combine merges.  Keys and values are decoded from their own cache types
// ("KV-Cache-Präzision": set independently for K and V; turbo3 values per
// "Benchmark TurboQuant en Apple Silicon", "¿Qué es TurboQuant?").
//
// Why the tensor cores: at the HBM rate a K8V4 row (208 bytes) reaches each SM
// about every 0.1 cycles, and the G query heads of a group need 2*G*d
// multiply-adds per row (2048 at G = 8, d = 128) -- far more than the FMA pipes
// issue in that time.  The QK and PV products of one 16-row tile are
// m16n8k16 tensor-core MMAs (fp16 operands, fp32 accumulation); the kernel stays
// bound by HBM bytes.
//
// Data movement: every warp runs its own ring of kStages shared-memory stages.
// Lane 0 fills a stage with cp.async.bulk.tensor copies (TMA) of one 16-row
// tile -- K codes, K scales, V codes, V scales -- completing on the stage's
// mbarrier; the code planes are copied with the hardware 32/64/128-byte swizzle
// so the fragment loads below are free of bank conflicts.  Rows past ctx_len
// read as zeros (tensor-map bounds).  No warp waits on another warp; every wait
// is bounded by a wall-clock limit (2 s), after which the warp stops, drains its
// own copies (bounded again) and the CTA writes NaN partials, so the affected
// outputs read NaN.
//
// Fragment mapping (lane = 4*g + c; MMA row m is tile row m):
//   QK   S[row][head] = sum_dim K[row][dim] * Q[head][dim]: A = K tile (16
//        rows) read by ldmatrix from the swizzled stage (8 rows x 16 bytes per
//        matrix; the swizzle puts the 8 rows in distinct bank groups), B = Q^T
//        (8 heads), fp32 C.  What ldmatrix hands a lane (4 bytes of a 16-byte
//        segment) fixes the dim order inside each 32-dim block; Q is loaded in
//        the same order.  Integer codes enter the MMA as fp16 subnormals, which
//        are exact: q8_0 k as (k + 128) * 2^-24 (an xor and two byte permutes
//        per four codes), q4_0 n as n * 2^-24 (one AND per two).  The first
//        MMA of a block starts from C = -128 * sum_block(q) * 2^-24 (-8 for
//        q4_0), so the block result is 2^-24 * sum k*q exactly up to fp32
//        rounding; the row's block scale is applied in fp32 and the 2^24 is
//        folded into softmax_scale * log2 e.
//   P    ex2 of the scores in fp32, rounded to fp16; movmatrix.trans turns the
//        (row x head) accumulator layout into the (row x head) B operand of PV.
//   PV   O^T[dim][head] += V^T[dim][row] * P[row][head]: A = V^T (16 dims) by
//        ldmatrix.trans, which hands a lane the same two bytes of rows 2c and
//        2c+1 in one register -- exactly the pair an A fragment holds -- so the
//        codes only need masking into subnormals (q4_0: n * 2^-24 and, for the
//        high nibble, 16 n * 2^-24) or an xor and a permute (q8_0: (k + 128) *
//        2^-24).  Each row's block scale (turbo3: its norm) multiplies P in
//        fp16.  The code offset (8 or 128) times sum_t d[t][blk] p[t] comes from
//        one more MMA per 16 rows whose A operand is the block-scale matrix
//        (m = block, k = row); it and the 2^24 are taken out once at the end.
//        turbo3 codes become codebook levels through a per-lane replicated
//        64-entry table of one row's two consecutive dims, paired across rows
//        by a byte permute.
//   turbo3 values accumulate in the rotated domain; kvq_combine rotates back.
//   Turbo keys score the rotated query H_un (s * q) against level-table A
//   operands (hi/lo fp16 parts, three MMAs per k-step); turbo3_qjl keys add the
//   query projected once more by the QJL matrix against their sign bits as +-1
//   A operands (two more MMAs).  Both are set up once per CTA, below.
#pragma once

#include <cuda.h>

#include "append_rows.cuh"

namespace kvq {
namespace tc {

constexpr int kNWMax = 8;    // warps per CTA (4 for the widest f16 stages)
constexpr int kSub = 32;     // cache rows per warp tile (one TMA box per plane)
constexpr int kHalf = 16;    // rows per MMA row block (two per tile)
constexpr unsigned long long kWaitLimitNs = 2000000000ull;  // 2 s per wait
// Bits of the workspace status word (kvq_workspace_status_offset), set when a
// wait gives up or a block-table entry is outside the pool; the affected
// outputs are NaN.
constexpr uint32_t kStatusTileWait = 1u, kStatusCombineWait = 2u, kStatusBadPage = 4u;

__host__ __device__ constexpr int code_bytes(int t, int d) {
  return t == KVQ_F16 ? 2 * d
         : t == KVQ_Q8_0 ? d
         : (t == KVQ_Q4_0 || t == KVQ_Q5_0) ? d / 2
         : is_qjl(t) ? 3 * d / 8
                     : turbo_bits(t) * d / 8;
}
__host__ __device__ constexpr int n_scales(int t, int d) {
  return t == KVQ_F16 ? 0 : is_qjl(t) ? 2 : is_turbo(t) ? 1 : t == KVQ_Q5_0 ? 3 * d / 32 : d / 32;
}
// swizzle of a code plane: 16-byte chunk index XOR ((offset >> 7) & mask)
__host__ __device__ constexpr int swz_mask(int t, int d) {
  return is_turbo(t) ? 0 : (code_bytes(t, d) >= 128 ? 8 : code_bytes(t, d) / 16) - 1;
}
// Entries of a turbo value type's level table (one copy per lane): the levels
// of two consecutive dims of a row (2^(2b)) at 2 and 3 bits, single levels at 4.
__host__ __device__ constexpr int turbo_table_entries(int t) {
  return !is_turbo(t) ? 0 : turbo_bits(t) <= 3 ? 1 << (2 * turbo_bits(t)) : 1 << turbo_bits(t);
}
__host__ __device__ constexpr int round_up_c(int v, int a) { return (v + a - 1) / a * a; }
__host__ __device__ constexpr int stage_bytes(int kt, int vt, int d) {
  return round_up_c(kSub * code_bytes(kt, d), is_turbo(kt) ? 128 : 1024) +
         round_up_c(kSub * code_bytes(vt, d), is_turbo(vt) ? 128 : 1024) +
         round_up_c(kSub * n_scales(kt, d) * 2, 128) + round_up_c(kSub * n_scales(vt, d) * 2, 128);
}
// Shared memory of one CTA: the 1024-byte alignment pad, one ring of `stages`
// stages per warp (rounded to the 1024-byte swizzle atom), the turbo level
// tables (values, then keys) and, for turbo keys, the rotated queries of up to 16
// heads, the ring barriers and a few bytes of slack.
// Turbo keys: levels as c = c_hi + c_lo to ~2^-22 (the scores enter an
// exponential, so fp16 levels alone are too coarse).  At 2 and 3 bits (turbo2,
// turbo3_qjl, turbo3) one entry per code pair x of two consecutive dims, in two
// tables: half2(c_hi[x mod 2^b], c_hi[x >> b]), then the same of c_lo -- the
// A-operand registers as they are, one lookup each.  At 4 bits (a 2 x 64 KB
// pair table) one entry per level, half2(c_hi, c_lo).
__host__ __device__ constexpr bool key_pair_table(int t) { return is_turbo(t) && turbo_bits(t) <= 3; }
__host__ __device__ constexpr int key_table_entries(int t) {
  return key_pair_table(t) ? 2 << (2 * turbo_bits(t)) : is_turbo(t) ? 1 << turbo_bits(t) : 0;
}
// turbo3_qjl keys: the projected queries P q_rot of up to 16 heads as fp16 hi
// and lo parts, rows padded to d + 8 halves (the MMA B-fragment reads of the 8
// heads of an n-tile then fall in distinct banks).
__host__ __device__ constexpr int qjl_stride(int d) { return d + 8; }
__host__ __device__ constexpr int table_bytes(int kt, int vt, int d) {
  return (turbo_table_entries(vt) + key_table_entries(kt)) * 32 * 4 + (is_turbo(kt) ? 16 * d * 4 : 0) +
         (is_qjl(kt) ? 16 * qjl_stride(d) * 4 : 0);
}
__host__ __device__ constexpr int cta_smem(int kt, int vt, int d, int nw, int stages) {
  return 1024 + nw * round_up_c(stages * stage_bytes(kt, vt, d), 1024) + table_bytes(kt, vt, d) + nw * stages * 8 +
         16;
}
// An SM has 228 KB of shared memory and reserves 1 KB per resident CTA; the
// kernel's static shared variables take a few bytes more.
constexpr int kSmemTwoCtas = 228 * 1024 / 2 - 1024 - 64;  // per CTA, two CTAs per SM
constexpr int kSmemOneCta = 227 * 1024 - 64;               // per CTA, one CTA per SM
// Warps per CTA: 8 while 8 two-stage rings leave room for a second CTA on the
// SM, else 4.  Stages per warp ring: as many (2 to 4) as keep the CTA count
// per SM (two if two fit at 2 stages, else one).
__host__ __device__ constexpr int warps_for(int kt, int vt, int d) {
  return cta_smem(kt, vt, d, kNWMax, 2) <= kSmemTwoCtas ? kNWMax : kNWMax / 2;
}
__host__ __device__ constexpr int ctas_per_sm_for(int kt, int vt, int d) {
  return cta_smem(kt, vt, d, warps_for(kt, vt, d), 2) <= kSmemTwoCtas ? 2 : 1;
}
// Whether an instance is compiled for one resident CTA per SM (launch bounds
// below): then it may use up to 255 registers a thread, and only as many CTAs
// fit as 65536 registers allow -- one of 8 warps.
__host__ __device__ constexpr bool one_cta_bound(int kt, int vt, int d, int nth) {
  return d >= 256 || nth == 2 || ctas_per_sm_for(kt, vt, d) < 2;
}
// Resident CTAs per SM, by shared memory and by registers: the slots the host
// sizes split counts and waiting combines for.
__host__ __device__ constexpr int regs_ctas_for(int kt, int vt, int d) {
  return 65536 / (warps_for(kt, vt, d) * 32 * 256) < 1 ? 1 : 65536 / (warps_for(kt, vt, d) * 32 * 256);
}
__host__ __device__ constexpr int resident_ctas_for(int kt, int vt, int d, int nth) {
  return one_cta_bound(kt, vt, d, nth) && regs_ctas_for(kt, vt, d) < ctas_per_sm_for(kt, vt, d)
             ? regs_ctas_for(kt, vt, d)
             : ctas_per_sm_for(kt, vt, d);
}
__host__ __device__ constexpr int stages_for(int kt, int vt, int d) {
  return cta_smem(kt, vt, d, warps_for(kt, vt, d), 4) <= (ctas_per_sm_for(kt, vt, d) == 2 ? kSmemTwoCtas : kSmemOneCta)
             ? 4
         : cta_smem(kt, vt, d, warps_for(kt, vt, d), 3) <= (ctas_per_sm_for(kt, vt, d) == 2 ? kSmemTwoCtas : kSmemOneCta)
             ? 3
             : 2;
}

template <int KT, int VT, int D>
struct Layout {
  static constexpr int NW = warps_for(KT, VT, D);
  static constexpr int kStages = stages_for(KT, VT, D);
  static constexpr int RBK = code_bytes(KT, D), RBV = code_bytes(VT, D);
  static constexpr int NSK = n_scales(KT, D), NSV = n_scales(VT, D);
  static constexpr int KC = round_up_c(kSub * RBK, is_turbo(KT) ? 128 : 1024);
  static constexpr int VC = round_up_c(kSub * RBV, is_turbo(VT) ? 128 : 1024);
  static constexpr int KS = round_up_c(kSub * NSK * 2, 128);
  static constexpr int VS = round_up_c(kSub * NSV * 2, 128);
  static constexpr int STAGE = KC + VC + KS + VS;
  static constexpr int WARP = round_up_c(kStages * STAGE, 1024);
  // Stage rings of a warp: code tiles, then scale tiles.  A swizzled code tile
  // starts on its swizzle atom (128 bytes per 16-byte chunk the pattern
  // permutes), so with turbo keys and swizzled values the value tiles go first.
  static constexpr bool VFIRST = is_turbo(KT) && !is_turbo(VT);
  static constexpr int KOFF = VFIRST ? kStages * VC : 0;
  static constexpr int VOFF = VFIRST ? 0 : kStages * KC;
  static constexpr int SOFF = kStages * (KC + VC);
  static_assert(KOFF % (128 * (swz_mask(KT, D) + 1)) == 0 && KC % (128 * (swz_mask(KT, D) + 1)) == 0,
                "key code tiles on their swizzle atom");
  static_assert(VOFF % (128 * (swz_mask(VT, D) + 1)) == 0 && VC % (128 * (swz_mask(VT, D) + 1)) == 0,
                "value code tiles on their swizzle atom");
  static constexpr int TABLE = table_bytes(KT, VT, D);
  static constexpr int BARS = NW * kStages * 8;
  static constexpr int TX = kSub * (RBK + 2 * NSK + RBV + 2 * NSV);  // bytes landing per tile
  // CTA-level merge scratch (reuses the stage memory after the main loop)
  static constexpr int MERGE = NW * ((D / 16) * 32 * 4 + 16) * 4;  // fragment chunks + m, l per warp
  static constexpr int TOTAL = 1024 + NW * WARP + TABLE + BARS + 16;
  static_assert(TOTAL == cta_smem(KT, VT, D, NW, kStages), "layout and budget agree");
  // The value level table is a static shared array (its address is then a
  // constant the table loads fold in); the rest is dynamic shared memory.
  static constexpr int VTAB = turbo_table_entries(VT) * 32 * 4;
  static constexpr int DYN = TOTAL - VTAB;
  static_assert(MERGE <= NW * WARP, "merge area must fit in the stage memory");
  static_assert(TOTAL <= 227 * 1024, "shared memory per CTA");
};

// ------------------------------------------------------------------ PTX helpers

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_addr(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits for phase `parity` of `bar`; false after kWaitLimitNs of wall time.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Tensor copies of cache tiles carry an L2 evict-first policy: every cache
// byte is read once per decode, so it should not displace what is read again
// (the split partials the combine reads back, the queries).
__device__ __forceinline__ uint64_t l2_evict_first_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3}], [%4], %5;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z, uint64_t* bar,
                                            uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4}], [%5], %6;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

__device__ __forceinline__ void tma_load_4d(void* dst, const CUtensorMap* map, int x, int y, int z, int w,
                                            uint64_t* bar, uint64_t pol) {
  asm volatile(
      "cp.async.bulk.tensor.4d.shared::cluster.global.tile.mbarrier::complete_tx::bytes.L2::cache_hint "
      "[%0], [%1, {%2, %3, %4, %5}], [%6], %7;" ::"r"(smem_addr(dst)),
      "l"(map), "r"(x), "r"(y), "r"(z), "r"(w), "r"(smem_addr(bar)), "l"(pol)
      : "memory");
}

// Contiguous global -> shared copy by the bulk-copy engine (16-byte aligned
// addresses, size a multiple of 16), completing on `bar`.
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void mma16816(float d[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1, const float c[4]) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%10,%11,%12,%13};"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1), "f"(c[0]), "f"(c[1]), "f"(c[2]), "f"(c[3]));
}

__device__ __forceinline__ uint32_t movmatrix_trans(uint32_t x) {
  uint32_t y;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(y) : "r"(x));
  return y;
}

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t r[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

__device__ __forceinline__ void ldmatrix_x4(uint32_t r[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}

// 2^x by the SFU's ex2 (about 2 ulp; subnormal results flush to 0, which only
// drops weights below 2^-126)
__device__ __forceinline__ float fast_exp2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// byte permute (PRMT) through the intrinsic, so constant operands stay immediates
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) { return __byte_perm(a, b, sel); }

__device__ __forceinline__ uint32_t hmul2_u32(uint32_t a, uint32_t b) {
  __half2 r = __hmul2(*reinterpret_cast<__half2*>(&a), *reinterpret_cast<__half2*>(&b));
  return *reinterpret_cast<uint32_t*>(&r);
}

// Packed binary32 pairs (f32x2): each lane rounded once, exactly as the scalar
// fmaf / __fmul_rn / __fadd_rn / __fsub_rn of the same operands.
__device__ __forceinline__ unsigned long long f2(float lo, float hi) {
  unsigned long long d;
  asm("mov.b64 %0, {%1, %2};" : "=l"(d) : "f"(lo), "f"(hi));
  return d;
}
__device__ __forceinline__ void f2split(unsigned long long v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}
__device__ __forceinline__ unsigned long long f2fma(unsigned long long a, unsigned long long b, unsigned long long c) {
  unsigned long long d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ unsigned long long f2mul(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2add(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ unsigned long long f2sub(unsigned long long a, unsigned long long b) {
  unsigned long long d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

// largest (g * fb) mod 4 over the 8 lane groups g: how far a lane group's
// code bytes can start past a 4-byte boundary
__host__ __device__ constexpr int max_lane_misalign(int fb) {
  int m = 0;
  for (int g = 0; g < 8; ++g) m = (g * fb) % 4 > m ? (g * fb) % 4 : m;
  return m;
}

template <int MASK>
__device__ __forceinline__ int swz(int off) {
  return off ^ (((off >> 7) & MASK) << 4);
}

// Integer codes enter the MMA as fp16 subnormals: a code n in 0..1023 in the
// low bits of an fp16 word is exactly n * 2^-24, the MMA multiplies such values
// exactly and accumulates in fp32, and the factor 2^24 is taken out in fp32.
constexpr float kTwo24 = 16777216.f;
constexpr float kTwo20 = 1048576.f;
constexpr float kTwoM24 = 5.9604644775390625e-08f;
constexpr uint32_t kHalfSixteenth = 0x2C002C00u;  // fp16 1/16 in both halves

// XOR that moves a lane's swizzled ldmatrix offset from block 0 to block blk.
// The swizzle only permutes 16-byte chunks inside a 128-byte span, so within a
// code row the offset of block blk is the block-0 offset with the chunk bits of
// blk flipped; for 256-byte rows the second 128-byte span also flips chunk bit
// 0 (its swizzle row index is odd).
__host__ __device__ constexpr uint32_t blk_xor(int t, int rb, int blk) {
  return t == KVQ_Q8_0 ? (uint32_t)(32 * blk) ^ (rb > 128 && blk >= 4 ? 16u : 0u)
                       : (uint32_t)(16 * (blk & ~1));
}

// ------------------------------------------------------------------ kernel

struct TcArgs {
  DecodeParams p;
};

// PAGED: the cache planes are pages of a pool, reached through the block table
// (a separate instantiation, so the contiguous kernel carries none of it).
template <int KT, int VT, int NB, int NTH, bool PAGED>
__global__ void __launch_bounds__(warps_for(KT, VT, NB * 32) * 32,
                                  one_cta_bound(KT, VT, NB * 32, NTH) ? 1 : 2)
    decode_tc_kernel(const TcArgs args, const __grid_constant__ CUtensorMap tm_kc,
                     const __grid_constant__ CUtensorMap tm_ks, const __grid_constant__ CUtensorMap tm_vc,
                     const __grid_constant__ CUtensorMap tm_vs) {
  constexpr int D = NB * 32;
  using L = Layout<KT, VT, D>;
  constexpr int S = L::kStages;
  constexpr int KMASK = swz_mask(KT, D), VMASK = swz_mask(VT, D);
  constexpr int NMT = D / 16;  // PV m-tiles
  constexpr bool kVQ = VT == KVQ_Q8_0 || VT == KVQ_Q4_0 || VT == KVQ_Q5_0;  // block-scaled integer values
  const DecodeParams& p = args.p;

  extern __shared__ unsigned char smem_raw[];
  // 1024-byte alignment (the swizzle atom) by offsetting inside the shared
  // array, so every derived pointer stays in the shared address space
  unsigned char* smem = smem_raw + ((1024u - (smem_addr(smem_raw) & 1023u)) & 1023u);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, c = lane & 3;
  unsigned char* wbase = smem + warp * L::WARP;
  const uint32_t wbase32 = smem_addr(wbase);
  __shared__ int cta_failed;
  // value level table (static, see Layout), then in dynamic memory the key
  // table and query rows of turbo keys, then the ring barriers
  __shared__ __align__(128) uint32_t s_vtab[L::VTAB > 0 ? L::VTAB / 4 : 1];
  uint32_t* table = reinterpret_cast<uint32_t*>(smem + L::NW * L::WARP);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + L::NW * L::WARP + (L::TABLE - L::VTAB)) + warp * S;

  const int s_idx = blockIdx.x, kvh = blockIdx.y, b = blockIdx.z;
  // rows of this batch row, and its split length (whole 32-row tiles)
  int64_t ctx = p.ctx, chunk = p.chunk, append_pos = p.append_pos;
  if (p.ctx_lens != nullptr) {
    const int64_t len = p.ctx_lens[b];
    ctx = len >= 1 && len <= p.ctx ? len : 0;  // out of range: attends nothing
    chunk = ((ctx + p.S - 1) / p.S + kSplitAlign - 1) / kSplitAlign * kSplitAlign;
    if (append_pos >= 0) append_pos = ctx - 1;
  }
  const int64_t t0l = (int64_t)s_idx * chunk;
  const int64_t t1l = min(ctx, t0l + chunk);
  const int n_sub = t0l < t1l ? (int)((t1l - t0l + kSub - 1) / kSub) : 0;
  // row indices fit in 32 bits (the tensor-map coordinates are 32-bit)
  const int t0 = (int)t0l, t1 = (int)t1l;
  const int plane = b * p.n_kv + kvh;

  // The queries are read before any cache tile is requested: issued after the
  // tiles, these few bytes would wait behind every warp's first stages on the
  // SM's return path (several microseconds when the stages hold most of a
  // split).  Raw words here; their fragment form is built further down.
  //   q8_0 / q4_0: 16-byte segments 2*blk, 2*blk+1, lane c's bytes 4c..4c+3
  //   f16: dims 32*blk + 8*i + 2c, +1 for i = 0..3
  // A launch that overlaps the previous kernel (p.pdl) reads them only after
  // that kernel has completed, which may have written them.
  uint32_t qraw[NTH][NB][4];
  auto load_queries = [&]() {
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      const int head = nt * 8 + g;
      const bool hv = head < p.G;
      const __half* qrow = p.q + ((int64_t)b * p.n_q + (int64_t)kvh * p.G + (hv ? head : 0)) * D;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        uint32_t* w = qraw[nt][blk];
        w[0] = w[1] = w[2] = w[3] = 0u;
        if (hv) {
          if (KT == KVQ_F16) {
#pragma unroll
            for (int i = 0; i < 4; ++i) w[i] = *reinterpret_cast<const uint32_t*>(qrow + blk * 32 + 8 * i + 2 * c);
          } else {
            const uint2 s0 = *reinterpret_cast<const uint2*>(qrow + blk * 32 + 4 * c);
            const uint2 s1 = *reinterpret_cast<const uint2*>(qrow + blk * 32 + 16 + 4 * c);
            w[0] = s0.x;
            w[1] = s0.y;
            w[2] = s1.x;
            w[3] = s1.y;
          }
        }
      }
    }
  };
  if (!p.pdl) load_queries();

  // Paged pool: the page of each of this warp's tiles, a window of 32 tiles
  // per register (lane i: tile j0 + i), read with the queries, before any tile
  // is requested; the next window is read 32 tiles ahead of its first use.
  constexpr bool paged = PAGED;
  const int my_tiles = n_sub > warp ? (n_sub - warp + L::NW - 1) / L::NW : 0;
  auto page_load = [&](int j0) -> int {  // page id of tile j0 + lane (0 past the last tile)
    const int j = j0 + lane;
    if (!paged || j >= my_tiles) return 0;
    const int r0 = t0 + kSub * (warp + L::NW * j);
    return p.block_table[(int64_t)b * p.max_pages + (r0 >> p.log2_page)];
  };
  int pg_win = page_load(0), pg_next = my_tiles > 32 ? page_load(32) : 0;

  if (threadIdx.x == 0) cta_failed = 0;
  if (lane == 0) {
#pragma unroll
    for (int i = 0; i < S; ++i) mbar_init(&bars[i], 1);
    fence_barrier_init();
  }
  if constexpr (is_turbo(VT)) {
    // b <= 3: table[x * 32 + lane] = half2(c[x mod 2^b], c[x >> b]), the levels of
    // a 2b-bit code pair x; b = 4: half2(c[x], c[x]).  One copy per bank.
    constexpr int TB = turbo_bits(VT), NE = turbo_table_entries(VT);
    for (int e = threadIdx.x; e < NE * 32; e += L::NW * 32) {
      const int idx = e >> 5;
      s_vtab[e] = TB <= 3 ? pack_half2(p.tq.levels[idx & ((1 << TB) - 1)], p.tq.levels[idx >> TB])
                         : pack_half2(p.tq.levels[idx], p.tq.levels[idx]);
    }
  }
  // turbo keys: their level table, ktable[x * 32 + lane] (one copy per bank);
  // then the rotated queries as fp16 hi and lo parts
  uint32_t* ktable = table;
  __half* qhi = reinterpret_cast<__half*>(ktable + key_table_entries(KT) * 32);  // [16][D]
  __half* qlo = qhi + 16 * D;                                                        // [16][D]
  constexpr int PST = qjl_stride(D);
  __half* phi = qlo + 16 * D;    // turbo3_qjl: P q_rot, [16][PST]
  __half* plo = phi + 16 * PST;  // [16][PST]
  if constexpr (key_pair_table(KT)) {
    constexpr int TB = turbo_bits(KT), NP = 1 << (2 * TB);
    for (int e = threadIdx.x; e < 2 * NP * 32; e += L::NW * 32) {
      const int x = (e >> 5) & (NP - 1);
      const float c0 = p.tqk.levels[x & ((1 << TB) - 1)], c1 = p.tqk.levels[x >> TB];
      const float h0 = __half2float(__float2half_rn(c0)), h1 = __half2float(__float2half_rn(c1));
      ktable[e] = (e >> 5) < NP ? pack_half2(h0, h1) : pack_half2(c0 - h0, c1 - h1);
    }
  } else if constexpr (is_turbo(KT)) {
    constexpr int NE = key_table_entries(KT);
    for (int e = threadIdx.x; e < NE * 32; e += L::NW * 32) {
      const float cl = p.tqk.levels[e >> 5];
      const float hi = __half2float(__float2half_rn(cl));
      ktable[e] = pack_half2(hi, cl - hi);
    }
  }
  __syncthreads();

  auto kc_of = [&](int st) { return wbase + L::KOFF + st * L::KC; };
  auto vc_of = [&](int st) { return wbase + L::VOFF + st * L::VC; };
  auto ks_of = [&](int st) { return wbase + L::SOFF + st * L::KS; };
  auto vs_of = [&](int st) { return wbase + L::SOFF + S * L::KS + st * L::VS; };

  // tile j of this warp covers rows t0 + 32*(warp + NW*j) ... (logical rows of
  // the sequence; in a paged pool, page pg's rows from r0 mod the page size)
  const uint64_t pol = l2_evict_first_policy();
  // an id that is not a page of the pool: load page 0 instead, partials NaN
  auto page_ok = [&](int pg) -> int {
    if (pg < 0 || pg >= p.n_pages) {
      atomicExch(&cta_failed, 1);
      atomicOr(p.status, kStatusBadPage);
      return 0;
    }
    return pg;
  };
  if (paged) {
    pg_win = page_ok(pg_win);
    pg_next = page_ok(pg_next);
  }
  auto issue = [&](int j, int st, int pg) {
    int r0 = t0 + kSub * (warp + L::NW * j);
    int tplane = plane;
    if (paged) {
      r0 &= (1 << p.log2_page) - 1;
      tplane = pg * p.n_kv + kvh;
    }
    mbar_expect_tx(&bars[st], L::TX);
    if (is_turbo(KT)) {
      if (kSub * L::RBK / 4 <= 256)
        tma_load_2d(kc_of(st), &tm_kc, r0 * L::RBK / 4, tplane, &bars[st], pol);
      else
        tma_load_3d(kc_of(st), &tm_kc, 0, r0, tplane, &bars[st], pol);
    } else if (L::RBK > 128) {
      tma_load_4d(kc_of(st), &tm_kc, 0, 0, r0, tplane, &bars[st], pol);
    } else {
      tma_load_3d(kc_of(st), &tm_kc, 0, r0, tplane, &bars[st], pol);
    }
    if (L::NSK) {  // flat words while a tile is at most 256 of them, else row-wise
      if (kSub * L::NSK / 2 <= 256)
        tma_load_2d(ks_of(st), &tm_ks, r0 * L::NSK / 2, tplane, &bars[st], pol);
      else
        tma_load_3d(ks_of(st), &tm_ks, 0, r0, tplane, &bars[st], pol);
    }
    if (is_turbo(VT)) {
      if (kSub * L::RBV / 4 <= 256)
        tma_load_2d(vc_of(st), &tm_vc, r0 * L::RBV / 4, tplane, &bars[st], pol);
      else
        tma_load_3d(vc_of(st), &tm_vc, 0, r0, tplane, &bars[st], pol);
    } else if (L::RBV > 128) {
      tma_load_4d(vc_of(st), &tm_vc, 0, 0, r0, tplane, &bars[st], pol);
    } else {
      tma_load_3d(vc_of(st), &tm_vc, 0, r0, tplane, &bars[st], pol);
    }
    if (L::NSV) {
      if (kSub * L::NSV / 2 <= 256)
        tma_load_2d(vs_of(st), &tm_vs, r0 * L::NSV / 2, tplane, &bars[st], pol);
      else
        tma_load_3d(vs_of(st), &tm_vs, 0, r0, tplane, &bars[st], pol);
    }
  };
  // Fused decode step: the new row (row append_pos) lies in tile jt of warp wt
  // of the CTA whose split holds it.  That warp issues its other first tiles,
  // then quantizes and writes the row of K and of V itself, makes the writes
  // visible device-wide and to the async proxy, and only then issues the tile
  // that reads the row back; no other warp waits.
  const bool owner = append_pos >= t0l && append_pos < t1l;
  const int t_new = owner ? (int)(append_pos - t0l) / kSub : -1;
  const int wt = owner ? t_new % L::NW : -1, jt = owner ? t_new / L::NW : -1;
  // A launch that overlaps the previous kernel requests only each warp's first
  // tile before the dependency resolves when the values are turbo rows and the
  // keys are not (a smaller burst disturbs the previous step's end less; with
  // turbo keys too it measured slightly slower), the other stages right after
  // it; every stage otherwise.
  constexpr int kEarly = is_turbo(VT) && !is_turbo(KT) ? 1 : S;
#pragma unroll
  for (int j = 0; j < S; ++j) {
    const int pg = paged ? __shfl_sync(0xffffffffu, pg_win, j) : 0;
    if (lane == 0 && j < my_tiles && !(warp == wt && j == jt) && (!p.pdl || j < kEarly)) issue(j, j, pg);
  }
  // The kernel after this one on the stream may be scheduled from here on (a
  // no-op unless it was launched to overlap this one).  A launch that overlaps
  // the previous kernel has requested cache tiles only, which that kernel does
  // not write; everything else waits until that kernel has completed and its
  // writes are visible.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  if (p.pdl) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    load_queries();
    if constexpr (kEarly < S) {
#pragma unroll
      for (int j = kEarly; j < S; ++j) {
        const int pg = paged ? __shfl_sync(0xffffffffu, pg_win, j) : 0;
        if (lane == 0 && j < my_tiles && !(warp == wt && j == jt)) issue(j, j, pg);
      }
    }
  }
  // Fused step with a shared combine: the group's epoch word as it stands
  // before this CTA arrives (the combine below waits for it to change).  Read
  // here, off the critical path at the end; the fence before the arrival
  // orders this read before it.
  __shared__ unsigned int comb_epoch0;
  if (p.out != nullptr && p.comb_ctas > 1 && threadIdx.x == 0)
    comb_epoch0 = *reinterpret_cast<volatile unsigned int*>(p.epochs + plane);
  if (warp == wt) {
    constexpr int rk = rows::row_threads(KT, D), rv = rows::row_threads(VT, D);
#pragma unroll
    for (int t = 0; t < rk; t += 32)
      rows::append_any(KT, p.app_k, (int64_t)plane * rk + t + lane, (int64_t)(plane + 1) * rk);
#pragma unroll
    for (int t = 0; t < rv; t += 32)
      rows::append_any(VT, p.app_v, (int64_t)plane * rv + t + lane, (int64_t)(plane + 1) * rv);
    __threadfence();
    asm volatile("fence.proxy.async.global;" ::: "memory");
    __syncwarp();
    const int pgt = paged ? __shfl_sync(0xffffffffu, pg_win, jt & 31) : 0;
    if (lane == 0 && jt < S && jt < my_tiles) issue(jt, jt, pgt);
  }

  // ---- turbo keys: score = (norm/D) * <H_un (s * q), c[code]>, so each query
  //      is rotated once: one warp per head, D/32 consecutive dims per lane,
  //      unnormalised Walsh-Hadamard butterflies in fp32 (in registers below
  //      stride D/32, shuffles above), stored as fp16 hi + lo parts for every
  //      warp (the heads past G of the last n-tile as zeros).
  if constexpr (is_turbo(KT)) {
    constexpr int E = D / 32;
    for (int h = p.G + warp; h < 8 * NTH; h += L::NW)
#pragma unroll
      for (int e = 0; e < E; ++e) qhi[h * D + lane * E + e] = qlo[h * D + lane * E + e] = __float2half_rn(0.f);
    for (int h = warp; h < p.G; h += L::NW) {
      const __half* qrow = p.q + ((int64_t)b * p.n_q + (int64_t)kvh * p.G + h) * D + lane * E;
      float v[E];
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const int i = lane * E + e;
        const float x = __half2float(qrow[e]);
        v[e] = ((p.tqk.sign_bits[i >> 5] >> (i & 31)) & 1u) ? -x : x;
      }
#pragma unroll
      for (int hs = 1; hs < E; hs <<= 1)
#pragma unroll
        for (int e = 0; e < E; ++e)
          if ((e & hs) == 0) {
            const float a0 = v[e], a1 = v[e + hs];
            v[e] = a0 + a1;
            v[e + hs] = a0 - a1;
          }
#pragma unroll
      for (int hs = E; hs < D; hs <<= 1) {
        const int lm = hs / E;
        const bool upper = (lane & lm) != 0;
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float o = __shfl_xor_sync(0xffffffffu, v[e], lm);
          v[e] = upper ? o - v[e] : v[e] + o;
        }
      }
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const __half hi = __float2half_rn(v[e]);
        qhi[h * D + lane * E + e] = hi;
        qlo[h * D + lane * E + e] = __float2half_rn(v[e] - __half2float(hi));
      }
    }
    __syncthreads();
    // turbo3_qjl: the sign bits z of a key row give <q, x_hat> its second term
    // sqrt(pi/2) / D^1.5 * gamma * <P q_rot, 1 - 2z>, so each rotated query is
    // projected once: p[h][i] = sum_j P[i][j] q_rot[h][j] in fp32 (q_rot =
    // hi + lo), one (row i, 4 heads) item per thread and round, stored as fp16
    // hi + lo parts (the padding heads give zeros).
    if constexpr (is_qjl(KT)) {
      constexpr int NH = 8 * NTH;
      for (int it = threadIdx.x; it < D * (NH / 4); it += L::NW * 32) {
        const int i = it % D, h0 = (it / D) * 4;
        const float4* prow = reinterpret_cast<const float4*>(qjl_proj(p.tqk) + (size_t)i * D);
        float acc4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll 4
        for (int j4 = 0; j4 < D / 4; ++j4) {
          const float4 pv = __ldg(prow + j4);
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) {
            const __half2* qh = reinterpret_cast<const __half2*>(qhi + (h0 + hh) * D + 4 * j4);
            const __half2* ql = reinterpret_cast<const __half2*>(qlo + (h0 + hh) * D + 4 * j4);
            const float2 h01 = __half22float2(qh[0]), h23 = __half22float2(qh[1]);
            const float2 l01 = __half22float2(ql[0]), l23 = __half22float2(ql[1]);
            acc4[hh] += pv.x * (h01.x + l01.x) + pv.y * (h01.y + l01.y) + pv.z * (h23.x + l23.x) +
                        pv.w * (h23.y + l23.y);
          }
        }
#pragma unroll
        for (int hh = 0; hh < 4; ++hh) {
          const __half hi = __float2half_rn(acc4[hh]);
          phi[(h0 + hh) * PST + i] = hi;
          plo[(h0 + hh) * PST + i] = __float2half_rn(acc4[hh] - __half2float(hi));
        }
      }
      __syncthreads();
    }
  }

  // ---- queries: B fragments of Q^T per (block, k-step) and, for quantized
  //      keys, the MMA C input -bias * sum(q) * 2^-24 of heads 2c, 2c+1 of each
  //      n-tile.  The dim order inside a block follows the A-operand loads
  //      below (lane = 4g + c):
  //        q8_0  k-step s = 16-byte segment 2*blk+s; lane c holds bytes 4c..4c+3:
  //              cols 2c,2c+1 <- bytes 4c,4c+1 and cols 2c+8,2c+9 <- 4c+2,4c+3
  //        q4_0  lane c holds bytes 4c..4c+3 of the block; low nibbles (dims
  //              4c..4c+3) feed k-step 0, high nibbles (4c+16..4c+19) k-step 1;
  //              cols 2c,2c+1 <- dims (4c, 4c+2), cols 2c+8,2c+9 <- (4c+1, 4c+3).
  //              The high nibbles enter as 16 n * 2^-24, so k-step 1 takes q / 16.
  //        f16   natural: k-step s covers dims 32*blk + 16*s .. +15
  //      Key codes enter as (k + 128) * 2^-24 (q8_0, sign bit flipped) or
  //      n * 2^-24 (q4_0), so the block dot product needs -128 * sum(q) or
  //      -8 * sum(q), in the same 2^-24 units.
  uint32_t qb[NTH][NB][2][2];
  float cq[NTH][NB][4];
  constexpr float kBiasK = KT == KVQ_Q8_0 ? 128.f : KT == KVQ_Q4_0 ? 8.f : KT == KVQ_Q5_0 ? 16.f : 0.f;
  if constexpr (is_turbo(KT)) {
    // rotated queries (hi parts) in the natural dim order (k-step s of block
    // blk covers dims 32 blk + 16 s .. +15), no code bias
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      const __half* qr = qhi + (nt * 8 + g) * D;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) {
          const int d0 = 32 * blk + 16 * s2 + 2 * c;
          qb[nt][blk][s2][0] = *reinterpret_cast<const uint32_t*>(qr + d0);
          qb[nt][blk][s2][1] = *reinterpret_cast<const uint32_t*>(qr + d0 + 8);
        }
        cq[nt][blk][0] = cq[nt][blk][1] = cq[nt][blk][2] = cq[nt][blk][3] = 0.f;
      }
    }
  } else {
#pragma unroll
  for (int nt = 0; nt < NTH; ++nt) {
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      const uint32_t* r = qraw[nt][blk];
      uint32_t w0 = r[0], w1 = r[1], w2 = r[2], w3 = r[3];
      if (KT == KVQ_Q4_0 || KT == KVQ_Q5_0) {
        w0 = prmt(r[0], r[1], 0x5410);  // (4c, 4c+2)
        w1 = prmt(r[0], r[1], 0x7632);  // (4c+1, 4c+3)
        w2 = prmt(r[2], r[3], 0x5410);
        w3 = prmt(r[2], r[3], 0x7632);
      }
      // partial sum of this lane's 8 dims of head g, then over the 4 lanes of the group
      float part = 0.f;
      const uint32_t ws[4] = {w0, w1, w2, w3};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&ws[i]));
        part += f.x + f.y;
      }
      part += __shfl_xor_sync(0xffffffffu, part, 1);
      part += __shfl_xor_sync(0xffffffffu, part, 2);
      // lane (g', c') needs the sums of heads 2c', 2c'+1 (held by groups 2c', 2c'+1)
      const float s0 = __shfl_sync(0xffffffffu, part, (2 * c) * 4);
      const float s1 = __shfl_sync(0xffffffffu, part, (2 * c + 1) * 4);
      if (KT == KVQ_Q4_0 || KT == KVQ_Q5_0) {
        w2 = hmul2_u32(w2, kHalfSixteenth);
        w3 = hmul2_u32(w3, kHalfSixteenth);
      }
      qb[nt][blk][0][0] = w0;
      qb[nt][blk][0][1] = w1;
      qb[nt][blk][1][0] = w2;
      qb[nt][blk][1][1] = w3;
      const float c0 = -kBiasK * kTwoM24 * s0, c1 = -kBiasK * kTwoM24 * s1;
      cq[nt][blk][0] = c0;
      cq[nt][blk][1] = c1;
      cq[nt][blk][2] = c0;
      cq[nt][blk][3] = c1;
    }
  }
  }
  const float qs = (KT == KVQ_F16 || is_turbo(KT)) ? p.qscale : p.qscale * kTwo24;

  // ---- running state
  float m_run[NTH][2], l_run[NTH][2];
  float acc[NTH][NMT][4];
  float off[NTH][4];  // q8_0 / q4_0 values: sum_t d[t][blk] p[t][head], blk = g, heads 2c, 2c+1
#pragma unroll
  for (int nt = 0; nt < NTH; ++nt) {
    m_run[nt][0] = m_run[nt][1] = -INFINITY;
    l_run[nt][0] = l_run[nt][1] = 0.f;
    off[nt][0] = off[nt][1] = off[nt][2] = off[nt][3] = 0.f;
#pragma unroll
    for (int i = 0; i < NMT; ++i) acc[nt][i][0] = acc[nt][i][1] = acc[nt][i][2] = acc[nt][i][3] = 0.f;
  }

  // ldmatrix addressing: this lane supplies the address of tile row lm_row in
  // matrix lane >> 3; lm_hi selects the second segment / block of an x4 load.
  // koff0 / voff0: the lane's swizzled offset of block 0 inside a 16-row half
  // (the swizzle period divides 16 rows, so both halves use the same offsets).
  const int lm_row = (lane & 7) + 8 * ((lane >> 3) & 1);
  const int lm_hi = lane >> 4;
  const uint32_t koff0 = (uint32_t)swz<KMASK>(lm_row * L::RBK + 16 * lm_hi);
  const uint32_t voff0 = (uint32_t)swz<VMASK>(lm_row * L::RBV + 16 * lm_hi);
  // offset-MMA operand selection: block g of a scale row (lanes g >= NSV give 0)
  const uint32_t osel = (g & 1) ? 0x7632u : 0x5410u;
  const uint32_t omask = g < (L::NSV > 0 ? L::NSV : 1) ? 0xFFFFFFFFu : 0u;
  int failed_at = -1;  // tile whose wait timed out (warp-uniform), -1 if none

  // QK of one 16-row tile: scaled scores S[row][head] of rows g, g+8 (heads 2c, 2c+1)
  auto qk_tile = [&](uint32_t kc, const unsigned char* kcp, const __half* ksc, float (&sc)[NTH][4]) {
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) sc[nt][0] = sc[nt][1] = sc[nt][2] = sc[nt][3] = 0.f;
    if constexpr (is_turbo(KT)) {
      // turbo keys: per 16-dim k-step one 64-bit window of each row's codes
      // (16 b bits); the pair table gives half2(level of dim 2c, of dim 2c+1)
      // of a row, exactly an A-operand register in the natural dim order
      constexpr int TB = turbo_bits(KT);
      const uint32_t* ktl = ktable + lane;
      auto window = [&](int row, int kstep) -> unsigned long long {
        const int byte0 = TB * kstep * 2;  // TB * 16 * kstep / 8
        const unsigned char* rp = kcp + row * L::RBK + (byte0 & ~3);
        unsigned long long v = *reinterpret_cast<const uint32_t*>(rp);
        if (16 * TB + 8 * (byte0 & 3) > 32) v |= (unsigned long long)(*reinterpret_cast<const uint32_t*>(rp + 4)) << 32;
        return v >> (8 * (byte0 & 3));
      };
      // dims j, j+1 of the window: (hi pair, lo pair), from the pair tables
      // at 2 and 3 bits, else from two level lookups
      auto pair = [&](unsigned long long f, int j, uint32_t& hi, uint32_t& lo) {
        if constexpr (key_pair_table(KT)) {
          constexpr uint32_t NP = 1u << (2 * TB);
          const uint32_t x = ((uint32_t)(f >> (TB * j)) & (NP - 1)) << 5;
          hi = ktl[x];
          lo = ktl[x + NP * 32];
        } else {
          constexpr uint32_t M = (1u << TB) - 1;
          const uint32_t e0 = ktl[((uint32_t)(f >> (TB * j)) & M) << 5];
          const uint32_t e1 = ktl[((uint32_t)(f >> (TB * j + TB)) & M) << 5];
          hi = prmt(e0, e1, 0x5410);
          lo = prmt(e0, e1, 0x7632);
        }
      };
      // turbo3_qjl: the 16 sign bits of a row's k-step (bit i of the z field,
      // after the D/4 bytes of level codes); bits j, j+1 of a window as the
      // fp16 pair (1 - 2 z_j, 1 - 2 z_j+1)
      auto zwindow = [&](int row, int kstep) -> uint32_t {
        const int byte0 = D / 4 + 2 * kstep;
        const uint32_t w = *reinterpret_cast<const uint32_t*>(kcp + row * L::RBK + (byte0 & ~3));
        return w >> (8 * (byte0 & 3));
      };
      auto zpair = [](uint32_t f, int j) -> uint32_t {
        return 0x3C003C00u | (((f >> j) & 1u) << 15) | (((f >> (j + 1)) & 1u) << 31);
      };
      float sz[NTH][4];  // turbo3_qjl: <P q_rot, 1 - 2z> of rows g, g+8
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) sz[nt][0] = sz[nt][1] = sz[nt][2] = sz[nt][3] = 0.f;
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) {
          const unsigned long long fa = window(g, 2 * blk + s2), fb = window(g + 8, 2 * blk + s2);
          uint32_t h[4], l[4];  // A operand: rows g, g+8 x dims (2c, 2c+1), (2c+8, 2c+9)
          pair(fa, 2 * c, h[0], l[0]);
          pair(fb, 2 * c, h[1], l[1]);
          pair(fa, 2 * c + 8, h[2], l[2]);
          pair(fb, 2 * c + 8, h[3], l[3]);
          uint32_t zq[4] = {0u, 0u, 0u, 0u};
          if constexpr (is_qjl(KT)) {
            const uint32_t za = zwindow(g, 2 * blk + s2), zb = zwindow(g + 8, 2 * blk + s2);
            zq[0] = zpair(za, 2 * c);
            zq[1] = zpair(zb, 2 * c);
            zq[2] = zpair(za, 2 * c + 8);
            zq[3] = zpair(zb, 2 * c + 8);
          }
          const int d0 = 32 * blk + 16 * s2 + 2 * c;
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt) {
            const __half* ql = qlo + (nt * 8 + g) * D + d0;
            const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(ql);
            const uint32_t bl1 = *reinterpret_cast<const uint32_t*>(ql + 8);
            // k_hi q_hi + k_hi q_lo + k_lo q_hi (k_lo q_lo is below 2^-22 relative)
            mma16816(sc[nt], h[0], h[1], h[2], h[3], qb[nt][blk][s2][0], qb[nt][blk][s2][1], sc[nt]);
            mma16816(sc[nt], h[0], h[1], h[2], h[3], bl0, bl1, sc[nt]);
            mma16816(sc[nt], l[0], l[1], l[2], l[3], qb[nt][blk][s2][0], qb[nt][blk][s2][1], sc[nt]);
            if constexpr (is_qjl(KT)) {  // the +-1 signs are exact: (p_hi + p_lo) . (1 - 2z)
              const __half* ph = phi + (nt * 8 + g) * PST + d0;
              const __half* pl = plo + (nt * 8 + g) * PST + d0;
              mma16816(sz[nt], zq[0], zq[1], zq[2], zq[3], *reinterpret_cast<const uint32_t*>(ph),
                       *reinterpret_cast<const uint32_t*>(ph + 8), sz[nt]);
              mma16816(sz[nt], zq[0], zq[1], zq[2], zq[3], *reinterpret_cast<const uint32_t*>(pl),
                       *reinterpret_cast<const uint32_t*>(pl + 8), sz[nt]);
            }
          }
        }
      }
      // the rows' norms / D (turbo3_qjl: plus the QJL term, gamma * sqrt(pi/2) / D^1.5)
      const float nA = __half2float(ksc[g * L::NSK]) * (1.0f / D);
      const float nB = __half2float(ksc[(g + 8) * L::NSK]) * (1.0f / D);
      if constexpr (is_qjl(KT)) {
        constexpr float kQ = 1.2533141373155003f / D * (D == 64 ? 0.125f : D == 128 ? 0.08838834764831845f : 0.0625f);
        const float gA = __half2float(ksc[g * L::NSK + 1]) * kQ, gB = __half2float(ksc[(g + 8) * L::NSK + 1]) * kQ;
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          sc[nt][0] = qs * (nA * sc[nt][0] + gA * sz[nt][0]);
          sc[nt][1] = qs * (nA * sc[nt][1] + gA * sz[nt][1]);
          sc[nt][2] = qs * (nB * sc[nt][2] + gB * sz[nt][2]);
          sc[nt][3] = qs * (nB * sc[nt][3] + gB * sz[nt][3]);
        }
      } else {
        const unsigned long long fa = f2(qs * nA, qs * nA), fb = f2(qs * nB, qs * nB);
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          f2split(f2mul(f2(sc[nt][0], sc[nt][1]), fa), sc[nt][0], sc[nt][1]);
          f2split(f2mul(f2(sc[nt][2], sc[nt][3]), fb), sc[nt][2], sc[nt][3]);
        }
      }
      return;
    }
    float dA[NB], dB[NB];  // block scales of rows g and g+8
    if constexpr (L::NSK > 0 && !is_turbo(KT)) {
      uint32_t sa[NB / 2], sb[NB / 2];
      if (NB == 2) {
        sa[0] = *reinterpret_cast<const uint32_t*>(ksc + g * L::NSK);
        sb[0] = *reinterpret_cast<const uint32_t*>(ksc + (g + 8) * L::NSK);
      } else {
#pragma unroll
        for (int i = 0; i < NB / 4; ++i) {
          const uint2 xa = *reinterpret_cast<const uint2*>(ksc + g * L::NSK + 4 * i);
          const uint2 xb = *reinterpret_cast<const uint2*>(ksc + (g + 8) * L::NSK + 4 * i);
          sa[2 * i] = xa.x;
          sa[2 * i + 1] = xa.y;
          sb[2 * i] = xb.x;
          sb[2 * i + 1] = xb.y;
        }
      }
#pragma unroll
      for (int i = 0; i < NB / 2; ++i) {
        const float2 fa = __half22float2(*reinterpret_cast<const __half2*>(&sa[i]));
        const float2 fb = __half22float2(*reinterpret_cast<const __half2*>(&sb[i]));
        dA[2 * i] = fa.x;
        dA[2 * i + 1] = fa.y;
        dB[2 * i] = fb.x;
        dB[2 * i + 1] = fb.y;
      }
    }
    const uint32_t kbase = kc + koff0;
    uint32_t kr[4];  // q4_0 keys: one x4 load per two blocks
#pragma unroll
    for (int blk = 0; blk < NB; ++blk) {
      uint32_t a[2][4];  // [k-step][a0..a3]
      if constexpr (KT == KVQ_Q8_0) {
        uint32_t r[4];
        ldmatrix_x4(r, kbase ^ blk_xor(KT, L::RBK, blk));
        const uint32_t u0 = r[0] ^ 0x80808080u, u1 = r[1] ^ 0x80808080u;
        const uint32_t u2 = r[2] ^ 0x80808080u, u3 = r[3] ^ 0x80808080u;
        a[0][0] = prmt(u0, 0u, 0x4140);
        a[0][2] = prmt(u0, 0u, 0x4342);
        a[0][1] = prmt(u1, 0u, 0x4140);
        a[0][3] = prmt(u1, 0u, 0x4342);
        a[1][0] = prmt(u2, 0u, 0x4140);
        a[1][2] = prmt(u2, 0u, 0x4342);
        a[1][1] = prmt(u3, 0u, 0x4140);
        a[1][3] = prmt(u3, 0u, 0x4342);
      } else if constexpr (KT == KVQ_Q4_0 || KT == KVQ_Q5_0) {
        // one x4 load covers blocks blk (regs 0, 1) and blk + 1 (regs 2, 3):
        // reg = bytes 4c..4c+3 of the block in row g (even regs) or g+8 (odd)
        if ((blk & 1) == 0) ldmatrix_x4(kr, kbase ^ blk_xor(KT, L::RBK, blk));
        const uint32_t wa = kr[(blk & 1) * 2], wb = kr[(blk & 1) * 2 + 1];
        const uint32_t was = wa >> 8, wbs = wb >> 8;
        a[0][0] = wa & 0x000F000Fu;   // dims (4c, 4c+2):       n * 2^-24
        a[0][2] = was & 0x000F000Fu;  // dims (4c+1, 4c+3)
        a[1][0] = wa & 0x00F000F0u;   // dims (4c+16, 4c+18):  16 n * 2^-24
        a[1][2] = was & 0x00F000F0u;  // dims (4c+17, 4c+19)
        a[0][1] = wb & 0x000F000Fu;
        a[0][3] = wbs & 0x000F000Fu;
        a[1][1] = wb & 0x00F000F0u;
        a[1][3] = wbs & 0x00F000F0u;
        if constexpr (KT == KVQ_Q5_0) {
          // fifth bits of rows g and g+8 (bit j of the block's qh word: dim j):
          // bit 4 of a low-nibble half, bit 8 of a high-nibble half
          const int hw = NB + 2 * blk;  // the block's qh word, in fp16 slots
          const uint32_t xa = *reinterpret_cast<const uint32_t*>(ksc + g * L::NSK + hw) >> (4 * c);
          const uint32_t xb = *reinterpret_cast<const uint32_t*>(ksc + (g + 8) * L::NSK + hw) >> (4 * c);
          a[0][0] |= ((xa << 4) & 0x10u) | ((xa << 18) & 0x100000u);    // dims 4c, 4c+2
          a[0][2] |= ((xa << 3) & 0x10u) | ((xa << 17) & 0x100000u);    // dims 4c+1, 4c+3
          a[1][0] |= ((xa >> 8) & 0x100u) | ((xa << 6) & 0x1000000u);   // dims 4c+16, 4c+18
          a[1][2] |= ((xa >> 9) & 0x100u) | ((xa << 5) & 0x1000000u);   // dims 4c+17, 4c+19
          a[0][1] |= ((xb << 4) & 0x10u) | ((xb << 18) & 0x100000u);
          a[0][3] |= ((xb << 3) & 0x10u) | ((xb << 17) & 0x100000u);
          a[1][1] |= ((xb >> 8) & 0x100u) | ((xb << 6) & 0x1000000u);
          a[1][3] |= ((xb >> 9) & 0x100u) | ((xb << 5) & 0x1000000u);
        }
      } else {  // f16
#pragma unroll
        for (int s2 = 0; s2 < 2; ++s2) {
          uint32_t r[4];
          ldmatrix_x4(r, kc + (uint32_t)swz<KMASK>(lm_row * L::RBK + 64 * blk + 32 * s2 + 16 * lm_hi));
          a[s2][0] = r[0];
          a[s2][1] = r[1];
          a[s2][2] = r[2];
          a[s2][3] = r[3];
        }
      }
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        if constexpr (L::NSK > 0) {
          // block dot product (k-step 0 starts from the offset correction),
          // then the row's block scale in fp32
          float dblk[4];
          mma16816(dblk, a[0][0], a[0][1], a[0][2], a[0][3], qb[nt][blk][0][0], qb[nt][blk][0][1], cq[nt][blk]);
          mma16816(dblk, a[1][0], a[1][1], a[1][2], a[1][3], qb[nt][blk][1][0], qb[nt][blk][1][1], dblk);
          // sc = fmaf(d, dblk, sc), two scores per packed operation
          f2split(f2fma(f2(dA[blk], dA[blk]), f2(dblk[0], dblk[1]), f2(sc[nt][0], sc[nt][1])), sc[nt][0], sc[nt][1]);
          f2split(f2fma(f2(dB[blk], dB[blk]), f2(dblk[2], dblk[3]), f2(sc[nt][2], sc[nt][3])), sc[nt][2], sc[nt][3]);
        } else {
          // f16 keys: no scale, no correction; accumulate in place
          mma16816(sc[nt], a[0][0], a[0][1], a[0][2], a[0][3], qb[nt][blk][0][0], qb[nt][blk][0][1], sc[nt]);
          mma16816(sc[nt], a[1][0], a[1][1], a[1][2], a[1][3], qb[nt][blk][1][0], qb[nt][blk][1][1], sc[nt]);
        }
      }
    }
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
      const unsigned long long qq = f2(qs, qs);
      f2split(f2mul(f2(sc[nt][0], sc[nt][1]), qq), sc[nt][0], sc[nt][1]);
      f2split(f2mul(f2(sc[nt][2], sc[nt][3]), qq), sc[nt][2], sc[nt][3]);
    }
  };

  // PV of one 16-row tile with its P fragments (rows 2c, 2c+1 | 2c+8, 2c+9);
  // in a tail half, pmask_lo / pmask_hi zero the P rows past the split end
  auto pv_tile = [&](const unsigned char* vc, uint32_t vc32, const __half* vsc, const uint32_t (&pb)[NTH][2],
                     bool tail, uint32_t pmask_lo, uint32_t pmask_hi) {
    if constexpr (VT == KVQ_F16) {
#pragma unroll
      for (int mt = 0; mt < NMT; ++mt) {
        const int jm = lane >> 3;
        const int krow = (lane & 7) + 8 * (jm >> 1);
        uint32_t a[4];
        ldmatrix_x4_trans(a, vc32 + (uint32_t)swz<VMASK>(krow * L::RBV + 2 * (16 * mt + 8 * (jm & 1))));
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          uint32_t b0 = pb[nt][0], b1 = pb[nt][1];
          if (tail) {
            b0 &= pmask_lo;
            b1 &= pmask_hi;
          }
          mma16816(acc[nt][mt], a[0], a[1], a[2], a[3], b0, b1, acc[nt][mt]);
        }
      }
    } else if constexpr (is_turbo(VT)) {
      // lane group g owns dims [g*D/8, (g+1)*D/8): GB = b*D/8 bits of each row's
      // codes, read as one or two 64-bit windows (HB bits, MTH m-tiles each)
      constexpr int TB = turbo_bits(VT);
      constexpr int GB = TB * D / 8;
      constexpr int HALVES = GB > 64 ? 2 : 1;
      constexpr int HB = GB / HALVES;
      constexpr int MTH = NMT / HALVES;
      auto field = [&](int row, int h) -> unsigned long long {  // bits [g*GB + h*HB, +HB) of a row
        const int byte0 = (g * GB + h * HB) >> 3;
        const unsigned char* rp = vc + row * L::RBV + (byte0 & ~3);
        unsigned long long v = *reinterpret_cast<const uint32_t*>(rp);
        if (HB + 8 * (byte0 & 3) > 32) v |= (unsigned long long)(*reinterpret_cast<const uint32_t*>(rp + 4)) << 32;
        return v >> (8 * (byte0 & 3));
      };
      // norms of rows (2c, 2c+1) and (2c+8, 2c+9) are adjacent fp16 pairs
      const uint32_t nAB = *reinterpret_cast<const uint32_t*>(vsc + 2 * c);
      const uint32_t nCD = *reinterpret_cast<const uint32_t*>(vsc + 2 * c + 8);
      uint32_t pbw[NTH][2];
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        pbw[nt][0] = hmul2_u32(pb[nt][0], nAB);
        pbw[nt][1] = hmul2_u32(pb[nt][1], nCD);
        if (tail) {
          pbw[nt][0] &= pmask_lo;
          pbw[nt][1] &= pmask_hi;
        }
      }
      // b <= 3: table[x * 32 + lane] = half2(c[x mod 2^b], c[x >> b]), the levels
      // of one row's two consecutive dims; b = 4: half2(c[x], c[x]), two
      // lookups per dim pair.  A byte permute then pairs rows 2c and 2c+1.
      if constexpr (TB <= 3 && (TB * D) % 64 == 0) {
        // Lane group g's codes of a row start on byte g * FB.  They are read as
        // aligned words and realigned by one byte permute per word (selector
        // from the lane's byte offset), so every pair index below sits at a
        // constant bit position: one shift moves it to bit 7 and one and-or
        // makes the byte offset (x << 7) | (lane << 2) of its table entry in the
        // static table.
        constexpr int FB = TB * D / 64;
        constexpr int NOUT = (FB + 3) / 4;
        constexpr int SMAX = max_lane_misalign(FB);
        constexpr int NLD = (FB + SMAX + 3) / 4;
        constexpr int PW = 2 * TB;                                   // bits of a pair index
        constexpr uint32_t PMASK = ((1u << PW) - 1u) << 7;
        const int off = g * FB;
        const uint32_t sel = 0x3210u + 0x1111u * (uint32_t)(off & 3);
        const uint32_t lane4 = (uint32_t)lane << 2;
        const unsigned char* tab = reinterpret_cast<const unsigned char*>(s_vtab);
        auto load_field = [&](int row, uint32_t (&o)[NOUT]) {
          const uint32_t* wp = reinterpret_cast<const uint32_t*>(vc + row * L::RBV + (off & ~3));
          uint32_t w[NLD + 1];
#pragma unroll
          for (int i = 0; i < NLD; ++i) w[i] = wp[i];
          w[NLD] = 0u;
#pragma unroll
          for (int i = 0; i < NOUT; ++i) o[i] = prmt(w[i], w[i + 1], sel);
        };
        // table entry of the pair at bit position pos of a field (pos is a
        // constant once the loop below is unrolled)
        auto entry = [&](const uint32_t (&o)[NOUT], int pos) -> uint32_t {
          const int i = pos / 32, r = pos % 32;
          uint32_t x;
          if (r + PW > 32) x = __funnelshift_r(o[i], o[i + 1 < NOUT ? i + 1 : i], r - 7);
          else if (r >= 7) x = o[i] >> (r - 7);
          else x = o[i] << (7 - r);
          return *reinterpret_cast<const uint32_t*>(tab + ((x & PMASK) | lane4));
        };
        uint32_t oA[NOUT], oB[NOUT], oC[NOUT], oD[NOUT];
        load_field(2 * c, oA);
        load_field(2 * c + 1, oB);
        load_field(2 * c + 8, oC);
        load_field(2 * c + 9, oD);
#pragma unroll
        for (int mt = 0; mt < NMT; ++mt) {
          const uint32_t tA = entry(oA, PW * mt), tB = entry(oB, PW * mt);
          const uint32_t tC = entry(oC, PW * mt), tD = entry(oD, PW * mt);
          uint32_t a[4];
          a[0] = prmt(tA, tB, 0x5410);  // dim 2mt:   rows 2c, 2c+1
          a[1] = prmt(tA, tB, 0x7632);  // dim 2mt+1
          a[2] = prmt(tC, tD, 0x5410);  // dim 2mt:   rows 2c+8, 2c+9
          a[3] = prmt(tC, tD, 0x7632);
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt)
            mma16816(acc[nt][mt], a[0], a[1], a[2], a[3], pbw[nt][0], pbw[nt][1], acc[nt][mt]);
        }
        return;
      }
      const uint32_t* tl = s_vtab + lane;
#pragma unroll
      for (int h = 0; h < HALVES; ++h) {
        const unsigned long long fA = field(2 * c, h), fB = field(2 * c + 1, h);
        const unsigned long long fC = field(2 * c + 8, h), fD = field(2 * c + 9, h);
#pragma unroll
        for (int k = 0; k < MTH; ++k) {
          const int mt = h * MTH + k;
          uint32_t tA, tB, tC, tD;  // half2(level of dim 2mt, of dim 2mt+1) of each row
          if constexpr (TB <= 3) {
            constexpr uint32_t PM = (1u << (2 * TB)) - 1;
            tA = tl[((uint32_t)(fA >> (2 * TB * k)) & PM) << 5];
            tB = tl[((uint32_t)(fB >> (2 * TB * k)) & PM) << 5];
            tC = tl[((uint32_t)(fC >> (2 * TB * k)) & PM) << 5];
            tD = tl[((uint32_t)(fD >> (2 * TB * k)) & PM) << 5];
          } else {
            auto pair = [&](unsigned long long f) {
              return prmt(tl[((uint32_t)(f >> (8 * k)) & 15u) << 5], tl[((uint32_t)(f >> (8 * k + 4)) & 15u) << 5],
                          0x5410);
            };
            tA = pair(fA);
            tB = pair(fB);
            tC = pair(fC);
            tD = pair(fD);
          }
          uint32_t a[4];
          a[0] = prmt(tA, tB, 0x5410);  // dim 2mt:   rows 2c, 2c+1
          a[1] = prmt(tA, tB, 0x7632);  // dim 2mt+1
          a[2] = prmt(tC, tD, 0x5410);  // dim 2mt:   rows 2c+8, 2c+9
          a[3] = prmt(tC, tD, 0x7632);
#pragma unroll
          for (int nt = 0; nt < NTH; ++nt)
            mma16816(acc[nt][mt], a[0], a[1], a[2], a[3], pbw[nt][0], pbw[nt][1], acc[nt][mt]);
        }
      }
    } else {
      // q8_0 / q4_0 values: per 32-dim block two m-tiles; each row's block scale
      // multiplies P.  The codes enter as subnormals ((k + 128) * 2^-24 for
      // q8_0; n * 2^-24 and 16 n * 2^-24 for the q4_0 nibbles); the code offset
      // (128 or 8) times sum_t d[t][blk] p[t] comes from one more MMA per half
      // tile whose A operand is the block-scale matrix (m = block, k = row).
      // Scales of rows (2c, 2c+1) and (2c+8, 2c+9) are adjacent.
      constexpr int NSD = VT == KVQ_Q5_0 ? NB : L::NSV;  // block scales per row
      uint32_t sAB[NSD], sCD[NSD];  // words: row 2c blocks | row 2c+1 blocks
      if constexpr (VT == KVQ_Q5_0) {
        // a q5_0 row's qh words follow its scales: the two rows are read apart
#pragma unroll
        for (int i = 0; i < NB / 2; ++i) {
          sAB[i] = *reinterpret_cast<const uint32_t*>(vsc + 2 * c * L::NSV + 2 * i);
          sAB[NB / 2 + i] = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 1) * L::NSV + 2 * i);
          sCD[i] = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 8) * L::NSV + 2 * i);
          sCD[NB / 2 + i] = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 9) * L::NSV + 2 * i);
        }
      } else if (L::NSV == 2) {
        const uint2 x = *reinterpret_cast<const uint2*>(vsc + 2 * c * L::NSV);
        const uint2 y = *reinterpret_cast<const uint2*>(vsc + (2 * c + 8) * L::NSV);
        sAB[0] = x.x; sAB[1] = x.y; sCD[0] = y.x; sCD[1] = y.y;
      } else {
#pragma unroll
        for (int i = 0; i < L::NSV / 4; ++i) {
          const uint4 x = *reinterpret_cast<const uint4*>(vsc + 2 * c * L::NSV + 8 * i);
          const uint4 y = *reinterpret_cast<const uint4*>(vsc + (2 * c + 8) * L::NSV + 8 * i);
          sAB[4 * i] = x.x; sAB[4 * i + 1] = x.y; sAB[4 * i + 2] = x.z; sAB[4 * i + 3] = x.w;
          sCD[4 * i] = y.x; sCD[4 * i + 1] = y.y; sCD[4 * i + 2] = y.z; sCD[4 * i + 3] = y.w;
        }
      }
      // row 2c's scales are words 0 .. NSD/2-1, row 2c+1's are NSD/2 ..
      {
        uint32_t xa = sAB[0], xb = sAB[NSD / 2], xc = sCD[0], xd = sCD[NSD / 2];
#pragma unroll
        for (int i = 1; i < NSD / 2; ++i) {
          const bool hit = (g >> 1) == i;
          xa = hit ? sAB[i] : xa;
          xb = hit ? sAB[NSD / 2 + i] : xb;
          xc = hit ? sCD[i] : xc;
          xd = hit ? sCD[NSD / 2 + i] : xd;
        }
        const uint32_t oa0 = prmt(xa, xb, osel) & omask, oa2 = prmt(xc, xd, osel) & omask;
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          uint32_t b0 = pb[nt][0], b1 = pb[nt][1];
          if (tail) {
            b0 &= pmask_lo;
            b1 &= pmask_hi;
          }
          mma16816(off[nt], oa0, 0u, oa2, 0u, b0, b1, off[nt]);
        }
      }
      const uint32_t vbase = vc32 + voff0;
      uint32_t vr[4];  // q4_0: one x4 load per two blocks
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const uint32_t sel = (blk & 1) ? 0x7632u : 0x5410u;
        const uint32_t dAB = prmt(sAB[blk >> 1], sAB[NSD / 2 + (blk >> 1)], sel);
        const uint32_t dCD = prmt(sCD[blk >> 1], sCD[NSD / 2 + (blk >> 1)], sel);
        uint32_t pbw[NTH][2];
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          pbw[nt][0] = hmul2_u32(pb[nt][0], dAB);
          pbw[nt][1] = hmul2_u32(pb[nt][1], dCD);
          if (tail) {
            pbw[nt][0] &= pmask_lo;
            pbw[nt][1] &= pmask_hi;
          }
        }
        uint32_t a0[4], a1[4];  // m-tiles (blk, 0) and (blk, 1)
        if (VT == KVQ_Q4_0 || VT == KVQ_Q5_0) {
          // trans load: reg = [row 2c: bytes 2g, 2g+1 | row 2c+1: bytes 2g, 2g+1]
          // of the block -> dims 2g, 2g+1 (low nibbles), 2g+16, 2g+17 (high)
          if ((blk & 1) == 0) ldmatrix_x4_trans(vr, vbase ^ blk_xor(VT, L::RBV, blk));
          const uint32_t w1 = vr[(blk & 1) * 2], w2 = vr[(blk & 1) * 2 + 1];
          const uint32_t w1s = w1 >> 8, w2s = w2 >> 8;
          a0[0] = w1 & 0x000F000Fu;   // dim 2g, rows 2c, 2c+1:   n * 2^-24
          a0[1] = w1s & 0x000F000Fu;  // dim 2g+1
          a0[2] = w2 & 0x000F000Fu;   // dim 2g, rows 2c+8, 2c+9
          a0[3] = w2s & 0x000F000Fu;
          a1[0] = w1 & 0x00F000F0u;   // dim 2g+16:               16 n * 2^-24
          a1[1] = w1s & 0x00F000F0u;
          a1[2] = w2 & 0x00F000F0u;
          a1[3] = w2s & 0x00F000F0u;
          if constexpr (VT == KVQ_Q5_0) {
            // fifth bits (bit j of a row's qh word: dim j): 16 more in the code,
            // bit 4 of a low-nibble half, bit 8 of a high-nibble half
            const int hw = NB + 2 * blk;  // the block's qh word, in fp16 slots
            const uint32_t xA = *reinterpret_cast<const uint32_t*>(vsc + 2 * c * L::NSV + hw) >> (2 * g);
            const uint32_t xB = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 1) * L::NSV + hw) >> (2 * g);
            const uint32_t xC = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 8) * L::NSV + hw) >> (2 * g);
            const uint32_t xD = *reinterpret_cast<const uint32_t*>(vsc + (2 * c + 9) * L::NSV + hw) >> (2 * g);
            a0[0] |= ((xA << 4) & 0x10u) | ((xB << 20) & 0x100000u);  // dim 2g
            a0[1] |= ((xA << 3) & 0x10u) | ((xB << 19) & 0x100000u);  // dim 2g+1
            a0[2] |= ((xC << 4) & 0x10u) | ((xD << 20) & 0x100000u);
            a0[3] |= ((xC << 3) & 0x10u) | ((xD << 19) & 0x100000u);
            a1[0] |= ((xA >> 8) & 0x100u) | ((xB << 8) & 0x1000000u);  // dim 2g+16
            a1[1] |= ((xA >> 9) & 0x100u) | ((xB << 7) & 0x1000000u);  // dim 2g+17
            a1[2] |= ((xC >> 8) & 0x100u) | ((xD << 8) & 0x1000000u);
            a1[3] |= ((xC >> 9) & 0x100u) | ((xD << 7) & 0x1000000u);
          }
        } else {
          // q8_0 trans load of segments 2blk (regs 0, 1) and 2blk+1 (regs 2, 3):
          // reg = [row 2c: bytes 2g, 2g+1 | row 2c+1: bytes 2g, 2g+1]
          ldmatrix_x4_trans(vr, vbase ^ blk_xor(VT, L::RBV, blk));
          const uint32_t x0 = vr[0] ^ 0x80808080u, x1 = vr[1] ^ 0x80808080u;
          const uint32_t y0 = vr[2] ^ 0x80808080u, y1 = vr[3] ^ 0x80808080u;
          a0[0] = prmt(x0, 0u, 0x4240);  // dim 2g
          a0[1] = prmt(x0, 0u, 0x4341);  // dim 2g+1
          a0[2] = prmt(x1, 0u, 0x4240);
          a0[3] = prmt(x1, 0u, 0x4341);
          a1[0] = prmt(y0, 0u, 0x4240);  // dim 16+2g
          a1[1] = prmt(y0, 0u, 0x4341);  // dim 16+2g+1
          a1[2] = prmt(y1, 0u, 0x4240);
          a1[3] = prmt(y1, 0u, 0x4341);
        }
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) {
          mma16816(acc[nt][2 * blk], a0[0], a0[1], a0[2], a0[3], pbw[nt][0], pbw[nt][1], acc[nt][2 * blk]);
          mma16816(acc[nt][2 * blk + 1], a1[0], a1[1], a1[2], a1[3], pbw[nt][0], pbw[nt][1],
                   acc[nt][2 * blk + 1]);
        }
      }
    }
  };

  int st = 0;
  uint32_t phase = 0;
#pragma unroll 1
  for (int j = 0; j < my_tiles; ++j) {
    // one 32-row tile per iteration, as two 16-row MMA halves (the second may
    // lie past the split end): one wait and one refill per 32 rows
    const bool ok = mbar_wait(&bars[st], phase);
    if (!__all_sync(0xffffffffu, ok)) {
      failed_at = j;
      break;
    }
    const int r0 = t0 + kSub * (warp + L::NW * j);
    const int rem = t1 - r0;  // rows of this tile inside the split (>= 1)
    const int nv0 = rem < kHalf ? rem : kHalf;
    const int nv1 = rem <= kHalf ? 0 : (rem - kHalf < kHalf ? rem - kHalf : kHalf);
    const bool two = nv1 > 0;
    const bool tail0 = nv0 < kHalf, tail1 = two && nv1 < kHalf;
    const uint32_t kc0 = wbase32 + L::KOFF + st * L::KC;
    const uint32_t vc32 = wbase32 + L::VOFF + st * L::VC;
    const __half* ks0 = reinterpret_cast<const __half*>(ks_of(st));
    const unsigned char* vc0 = vc_of(st);
    const __half* vs0 = reinterpret_cast<const __half*>(vs_of(st));

    float sc0[NTH][4], sc1[NTH][4];
    uint32_t pb0[NTH][2], pb1[NTH][2];
    // ---------------- online softmax over the 32 rows (heads 2c, 2c+1).  The
    // running max only moves when a score passes it, which after the first
    // tiles is rare: only then are the row maxima reduced across the warp and
    // the state rescaled.  Every P stays <= 1 either way.
    auto softmax = [&]() {
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        float mx0 = fmaxf(fmaxf(sc0[nt][0], sc0[nt][2]), fmaxf(sc1[nt][0], sc1[nt][2]));
        float mx1 = fmaxf(fmaxf(sc0[nt][1], sc0[nt][3]), fmaxf(sc1[nt][1], sc1[nt][3]));
        if (__any_sync(0xffffffffu, mx0 > m_run[nt][0] || mx1 > m_run[nt][1])) {
#pragma unroll
          for (int o = 4; o <= 16; o <<= 1) {
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, o));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, o));
          }
          const float mn0 = fmaxf(m_run[nt][0], mx0), mn1 = fmaxf(m_run[nt][1], mx1);
          const float al0 = fast_exp2(m_run[nt][0] - mn0), al1 = fast_exp2(m_run[nt][1] - mn1);
          m_run[nt][0] = mn0;
          m_run[nt][1] = mn1;
          const unsigned long long al = f2(al0, al1);
          f2split(f2mul(f2(l_run[nt][0], l_run[nt][1]), al), l_run[nt][0], l_run[nt][1]);
#pragma unroll
          for (int i = 0; i < NMT; ++i) {
            f2split(f2mul(f2(acc[nt][i][0], acc[nt][i][1]), al), acc[nt][i][0], acc[nt][i][1]);
            f2split(f2mul(f2(acc[nt][i][2], acc[nt][i][3]), al), acc[nt][i][2], acc[nt][i][3]);
          }
          if (kVQ) f2split(f2mul(f2(off[nt][0], off[nt][1]), al), off[nt][0], off[nt][1]);
        }
        // exponent arguments and the row sums two heads (2c, 2c+1) at a time
        const unsigned long long mm = f2(m_run[nt][0], m_run[nt][1]);
        float x0, x1, x2, x3, y0, y1, y2, y3;
        f2split(f2sub(f2(sc0[nt][0], sc0[nt][1]), mm), x0, x1);
        f2split(f2sub(f2(sc0[nt][2], sc0[nt][3]), mm), x2, x3);
        f2split(f2sub(f2(sc1[nt][0], sc1[nt][1]), mm), y0, y1);
        f2split(f2sub(f2(sc1[nt][2], sc1[nt][3]), mm), y2, y3);
        const float p0 = fast_exp2(x0), p1 = fast_exp2(x1), p2 = fast_exp2(x2), p3 = fast_exp2(x3);
        const float q0 = fast_exp2(y0), q1 = fast_exp2(y1), q2 = fast_exp2(y2), q3 = fast_exp2(y3);
        const unsigned long long ls = f2add(f2add(f2(p0, p1), f2(p2, p3)), f2add(f2(q0, q1), f2(q2, q3)));
        f2split(f2add(f2(l_run[nt][0], l_run[nt][1]), ls), l_run[nt][0], l_run[nt][1]);
        pb0[nt][0] = movmatrix_trans(pack_half2(p0, p1));
        pb0[nt][1] = movmatrix_trans(pack_half2(p2, p3));
        pb1[nt][0] = movmatrix_trans(pack_half2(q0, q1));
        pb1[nt][1] = movmatrix_trans(pack_half2(q2, q3));
      }
    };
    if (rem >= kSub) {
      // A whole tile: both halves with no masks, in one basic block, so the
      // two halves' dependency chains interleave.
      qk_tile(kc0, kc_of(st), ks0, sc0);
      qk_tile(kc0 + kHalf * L::RBK, kc_of(st) + kHalf * L::RBK, ks0 + kHalf * L::NSK, sc1);
      softmax();
      pv_tile(vc0, vc32, vs0, pb0, false, 0xFFFFFFFFu, 0xFFFFFFFFu);
      pv_tile(vc0 + kHalf * L::RBV, vc32 + kHalf * L::RBV, vs0 + kHalf * L::NSV, pb1, false, 0xFFFFFFFFu,
              0xFFFFFFFFu);
    } else {
      // the split's last tile: rows past its end masked out
      qk_tile(kc0, kc_of(st), ks0, sc0);
      if (two) {
        qk_tile(kc0 + kHalf * L::RBK, kc_of(st) + kHalf * L::RBK, ks0 + kHalf * L::NSK, sc1);
      } else {
#pragma unroll
        for (int nt = 0; nt < NTH; ++nt) sc1[nt][0] = sc1[nt][1] = sc1[nt][2] = sc1[nt][3] = -INFINITY;
      }
#pragma unroll
      for (int nt = 0; nt < NTH; ++nt) {
        if (g >= nv0) sc0[nt][0] = sc0[nt][1] = -INFINITY;
        if (g + 8 >= nv0) sc0[nt][2] = sc0[nt][3] = -INFINITY;
        if (g >= nv1) sc1[nt][0] = sc1[nt][1] = -INFINITY;
        if (g + 8 >= nv1) sc1[nt][2] = sc1[nt][3] = -INFINITY;
      }
      softmax();
      // In a tail half, P rows past the split end contribute exactly 0 whatever
      // the row's scale holds (b operand halves: rows 2c, 2c+1 | 2c+8, 2c+9).
      auto pmask = [&](int nv, uint32_t& lo, uint32_t& hi) {
        lo = (2 * c < nv ? 0x0000FFFFu : 0u) | (2 * c + 1 < nv ? 0xFFFF0000u : 0u);
        hi = (2 * c + 8 < nv ? 0x0000FFFFu : 0u) | (2 * c + 9 < nv ? 0xFFFF0000u : 0u);
      };
      uint32_t mlo = 0xFFFFFFFFu, mhi = 0xFFFFFFFFu;
      if (tail0) pmask(nv0, mlo, mhi);
      pv_tile(vc0, vc32, vs0, pb0, tail0, mlo, mhi);
      if (two) {
        if (tail1) pmask(nv1, mlo, mhi);
        pv_tile(vc0 + kHalf * L::RBV, vc32 + kHalf * L::RBV, vs0 + kHalf * L::NSV, pb1, tail1, mlo, mhi);
      }
    }

    // release the stage and refill it with this warp's tile j + S
    __syncwarp();
    int pg = 0;
    if (paged) {
      const int jn = j + S;
      if ((jn & 31) == 0 && jn < my_tiles) {  // next window: read the one after it
        pg_win = pg_next;
        pg_next = page_ok(page_load(jn + 32));
      }
      pg = __shfl_sync(0xffffffffu, pg_win, jn & 31);
    }
    if (lane == 0 && j + S < my_tiles) {
      fence_proxy_async();
      issue(j + S, st, pg);
    }
    if (++st == S) {
      st = 0;
      phase ^= 1u;
    }
  }

  if (failed_at >= 0) {
    // A copy did not land within the limit.  Wait (bounded again) for every
    // copy this warp still has in flight -- tiles failed_at .. failed_at+S-1 --
    // so none writes into shared memory after the CTA exits, and make this
    // CTA's partials NaN so the outputs show the failure.
    const int last = min(my_tiles, failed_at + S);
    for (int jj = failed_at; jj < last; ++jj) (void)mbar_wait(&bars[jj % S], (uint32_t)((jj / S) & 1));
    if (lane == 0) {
      atomicExch(&cta_failed, 1);
      atomicOr(p.status, kStatusTileWait);
    }
  }
  __syncwarp();

  // ---- reduce l over the 8 row groups; each lane keeps heads 2c, 2c+1
#pragma unroll
  for (int nt = 0; nt < NTH; ++nt)
#pragma unroll
    for (int e = 0; e < 2; ++e)
#pragma unroll
      for (int o = 4; o <= 16; o <<= 1) l_run[nt][e] += __shfl_xor_sync(0xffffffffu, l_run[nt][e], o);

  // ---- q8_0 / q4_0 values: take the 2^24 (2^20) out and subtract the code
  //      offset times sum_t d[t][blk] p[t] (held by lane 4 * blk + c)
  if constexpr (kVQ) {
    constexpr float vb = VT == KVQ_Q8_0 ? 128.f : VT == KVQ_Q5_0 ? 16.f : 8.f;
#pragma unroll
    for (int nt = 0; nt < NTH; ++nt) {
#pragma unroll
      for (int blk = 0; blk < NB; ++blk) {
        const float o0 = -vb * __shfl_sync(0xffffffffu, off[nt][0], blk * 4 + c);
        const float o1 = -vb * __shfl_sync(0xffffffffu, off[nt][1], blk * 4 + c);
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int mt = 2 * blk + h;
          const float f = ((VT == KVQ_Q4_0 || VT == KVQ_Q5_0) && h == 1) ? kTwo20 : kTwo24;
          acc[nt][mt][0] = fmaf(acc[nt][mt][0], f, o0);
          acc[nt][mt][1] = fmaf(acc[nt][mt][1], f, o1);
          acc[nt][mt][2] = fmaf(acc[nt][mt][2], f, o0);
          acc[nt][mt][3] = fmaf(acc[nt][mt][3], f, o1);
        }
      }
    }
  }

  __syncthreads();  // every warp is done with its stages: reuse them for the merge

  // ---- merge of the warps.  Each warp stores its accumulator fragments as
  //      they lie in registers (16-byte chunks, lane-major: no bank conflicts)
  //      and its per-head m and l; thread t then sums chunk t over the warps,
  //      weighted by 2^(m_w - M) of the chunk's two heads (2c, 2c+1).
  constexpr int CH = NMT * 32;          // 16-byte chunks per warp and n-tile
  constexpr int WSTRIDE = CH * 4 + 16;  // floats per warp: chunks, m[8], l[8]
  float* mrg = reinterpret_cast<float*>(smem);
  auto dim_of = [&](int mt, int row) -> int {  // PV m-tile row -> head dim
    if (VT == KVQ_F16) return 16 * mt + row;                       // row in 0..15
    if (is_turbo(VT)) return (row & 7) * (D / 8) + 2 * mt + (row >> 3);
    return 32 * (mt >> 1) + 16 * (mt & 1) + 2 * (row & 7) + (row >> 3);  // q8_0, q4_0
  };
  const bool failed = cta_failed != 0;
#pragma unroll
  for (int nt = 0; nt < NTH; ++nt) {
    float* wf = mrg + warp * WSTRIDE;
#pragma unroll
    for (int mt = 0; mt < NMT; ++mt)
      *reinterpret_cast<float4*>(wf + (mt * 32 + lane) * 4) =
          make_float4(acc[nt][mt][0], acc[nt][mt][1], acc[nt][mt][2], acc[nt][mt][3]);
    if (g == 0) {
      wf[CH * 4 + 2 * c] = m_run[nt][0];
      wf[CH * 4 + 2 * c + 1] = m_run[nt][1];
      wf[CH * 4 + 8 + 2 * c] = l_run[nt][0];
      wf[CH * 4 + 8 + 2 * c + 1] = l_run[nt][1];
    }
    __syncthreads();
    const int heads_here = min(8, p.G - nt * 8);
    const int64_t row0 = ((int64_t)b * p.n_q + (int64_t)kvh * p.G + nt * 8) * p.S + s_idx;  // head 0's row
    for (int i = threadIdx.x; i < CH; i += L::NW * 32) {
      const int mt = i >> 5, gg = (i >> 2) & 7, cc = i & 3;
      const int hA = 2 * cc, hB = 2 * cc + 1;
      float MA = -INFINITY, MB = -INFINITY;
#pragma unroll
      for (int w = 0; w < L::NW; ++w) {
        MA = fmaxf(MA, mrg[w * WSTRIDE + CH * 4 + hA]);
        MB = fmaxf(MB, mrg[w * WSTRIDE + CH * 4 + hB]);
      }
      float fA[L::NW], fB[L::NW];
      float4 sum = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int w = 0; w < L::NW; ++w) {
        // a warp without rows has m = -inf: weight 0 (all weights 0 if no warp has rows)
        fA[w] = MA == -INFINITY ? 0.f : fast_exp2(mrg[w * WSTRIDE + CH * 4 + hA] - MA);
        fB[w] = MB == -INFINITY ? 0.f : fast_exp2(mrg[w * WSTRIDE + CH * 4 + hB] - MB);
        const float4 x = *reinterpret_cast<const float4*>(mrg + w * WSTRIDE + i * 4);
        sum.x = fmaf(fA[w], x.x, sum.x);
        sum.y = fmaf(fB[w], x.y, sum.y);
        sum.z = fmaf(fA[w], x.z, sum.z);
        sum.w = fmaf(fB[w], x.w, sum.w);
      }
      if (failed) sum = make_float4(__int_as_float(0x7fc00000), __int_as_float(0x7fc00000),
                                    __int_as_float(0x7fc00000), __int_as_float(0x7fc00000));
      const int dA = dim_of(mt, gg), dB = dim_of(mt, gg + 8);
      if (hA < heads_here) {
        p.ws_acc[(row0 + (int64_t)hA * p.S) * D + dA] = sum.x;
        p.ws_acc[(row0 + (int64_t)hA * p.S) * D + dB] = sum.z;
      }
      if (hB < heads_here) {
        p.ws_acc[(row0 + (int64_t)hB * p.S) * D + dA] = sum.y;
        p.ws_acc[(row0 + (int64_t)hB * p.S) * D + dB] = sum.w;
      }
      if (mt == 0 && gg == 0) {  // one thread per head pair: m and l
        float lA = 0.f, lB = 0.f;
#pragma unroll
        for (int w = 0; w < L::NW; ++w) {
          lA = fmaf(fA[w], mrg[w * WSTRIDE + CH * 4 + 8 + hA], lA);
          lB = fmaf(fB[w], mrg[w * WSTRIDE + CH * 4 + 8 + hB], lB);
        }
        const float nan = __int_as_float(0x7fc00000);
        if (hA < heads_here) {
          p.ws_m[row0 + (int64_t)hA * p.S] = failed ? nan : MA;
          p.ws_l[row0 + (int64_t)hA * p.S] = failed ? nan : lA;
        }
        if (hB < heads_here) {
          p.ws_m[row0 + (int64_t)hB * p.S] = failed ? nan : MB;
          p.ws_l[row0 + (int64_t)hB * p.S] = failed ? nan : lB;
        }
      }
    }
    __syncthreads();
  }

  // ---- fused decode step: the last CTAs of this (batch row, KV head) to
  //      finish merge the S split partials of the group's G heads into the
  //      output (the arithmetic of kvq_combine, with the inverse rotation of a
  //      turbo3 value cache).  Arrivals are counted modulo S (the counter
  //      returns to 0).  The last arrival (rank 0) may combine at once; the
  //      arrivals of rank 1 .. comb_ctas-1 wait for it through the group's epoch
  //      word, which rank 0 bumps once every partial is visible, so the G heads
  //      are combined by comb_ctas CTAs at a time.  (The host enables that only
  //      when the waiting CTAs leave most of the GPU's CTA slots free, so the
  //      CTAs they wait for can always run; each wait is bounded.)
  if (p.out != nullptr) {
    __shared__ unsigned int comb_rank;
    __shared__ int comb_wait_failed;
    __threadfence();  // this CTA's partials are visible device-wide ...
    __syncthreads();
    if (threadIdx.x == 0) {  // ... before its arrival is counted
      // the epoch was read before this CTA arrives (once the grid dependency
      // resolved, ordered by the fence above): rank 0 bumps it only after the
      // last arrival, so a waiter cannot miss the bump
      const unsigned int e0 = p.comb_ctas > 1 ? comb_epoch0 : 0u;
      const unsigned int ticket = atomicInc(p.counters + plane, (unsigned)(p.S - 1));
      // a counter left outside [0, S) by a caller (it must start at 0) gives a
      // ticket above S - 1: a huge rank, so that CTA only arrives
      const unsigned int rank = (unsigned)(p.S - 1) - ticket;
      int failed = 0;
      if (rank == 0) {
        __threadfence();
        if (p.comb_ctas > 1) atomicAdd(p.epochs + plane, 1u);
      } else if (rank < (unsigned)p.comb_ctas) {
        const unsigned long long w0 = global_ns();
        while (*reinterpret_cast<volatile unsigned int*>(p.epochs + plane) == e0) {
          if (global_ns() - w0 > kWaitLimitNs) {
            failed = 1;
            atomicOr(p.status, kStatusCombineWait);
            break;
          }
          __nanosleep(64);
        }
        __threadfence();
      }
      comb_rank = rank;
      comb_wait_failed = failed;
    }
    __syncthreads();
    if (comb_rank < (unsigned)p.comb_ctas) {
      const int rank = (int)comb_rank;
      __threadfence();
      // the partials were written through the generic proxy by other CTAs and
      // are read here by bulk copies (the async proxy)
      asm volatile("fence.proxy.async.global;" ::: "memory");
      // This CTA's heads [h0, h0 + nh) of the group.  Their partials (nh heads x
      // S splits x D floats) come into the free stage memory by bulk copies,
      // one per head and round of up to 64 splits; m and l are read alongside.
      // One warp per head then folds the round into its running (max, sum,
      // weighted acc), D/32 consecutive dims per lane.
      constexpr int E = D / 32;                        // dims per lane
      constexpr int HPW = (16 + L::NW - 1) / L::NW;    // heads per warp, G <= 16
      constexpr int kAvail = L::NW * L::WARP / 4;      // floats of stage memory
      const int G = p.G, S_ = p.S;
      const int h0 = rank * G / p.comb_ctas, nh = (rank + 1) * G / p.comb_ctas - h0;
      float* buf = reinterpret_cast<float*>(smem);     // [nh][SC][D]
      const int SC = max(1, min(64, min(S_, kAvail / (nh * D))));
      const int64_t grow0 = ((int64_t)b * p.n_q + (int64_t)kvh * G + h0) * S_;  // (head h0, split 0)
      // one mbarrier for the rounds' bulk copies (the pipeline's are idle now)
      __shared__ uint64_t comb_bar[1];
      uint64_t* cbar = comb_bar;
      uint32_t cphase = 0;
      int comb_failed = comb_wait_failed;
      if (threadIdx.x == 0) {
        mbar_init(cbar, 1);
        fence_barrier_init();
      }
      fence_proxy_async();  // the merge's generic writes to the stage memory come before the copies into it
      __syncthreads();
      float Mh[HPW], den[HPW], num[HPW][E];
#pragma unroll
      for (int hi = 0; hi < HPW; ++hi) {
        Mh[hi] = -INFINITY;
        den[hi] = 0.f;
#pragma unroll
        for (int e = 0; e < E; ++e) num[hi][e] = 0.f;
      }
      for (int s0 = 0; !comb_failed && s0 < S_; s0 += SC) {  // comb_failed is uniform
        const int sc = min(SC, S_ - s0);
        if (threadIdx.x == 0) {
          mbar_expect_tx(cbar, (uint32_t)(nh * sc * D * 4));
          for (int hl = 0; hl < nh; ++hl)
            bulk_load(buf + hl * SC * D, p.ws_acc + (grow0 + (int64_t)hl * S_ + s0) * D, (uint32_t)(sc * D * 4),
                      cbar);
        }
        // this round's m, l of splits s0 + lane and s0 + 32 + lane
        float mj[HPW][2], lj[HPW][2];
#pragma unroll
        for (int hi = 0; hi < HPW; ++hi) {
          const int hl = warp + hi * L::NW;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            const int j = lane + 32 * u;
            mj[hi][u] = -INFINITY;
            lj[hi][u] = 0.f;
            if (hl < nh && j < sc) {
              mj[hi][u] = __ldcg(p.ws_m + grow0 + (int64_t)hl * S_ + s0 + j);
              lj[hi][u] = __ldcg(p.ws_l + grow0 + (int64_t)hl * S_ + s0 + j);
            }
          }
        }
        const bool landed = mbar_wait(cbar, cphase);
        if (!__syncthreads_and(landed)) {
          // a copy did not land within the limit: let it drain (bounded
          // again) so nothing writes shared memory after the CTA exits; the
          // heads' outputs read NaN
          if (threadIdx.x == 0) {
            (void)mbar_wait(cbar, cphase);
            atomicOr(p.status, kStatusCombineWait);
          }
          __syncthreads();
          comb_failed = 1;
          break;
        }
        cphase ^= 1u;
#pragma unroll
        for (int hi = 0; hi < HPW; ++hi) {
          const int hl = warp + hi * L::NW;
          if (hl >= nh) break;
          float mc = fmaxf(mj[hi][0], mj[hi][1]);
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
          const float mn = fmaxf(Mh[hi], mc);
          // an empty split (m = -inf) weighs 0; so does the old state while no split had rows
          const float alpha = Mh[hi] == -INFINITY ? 0.f : exp2f(Mh[hi] - mn);
          float wl[2], dl = 0.f;
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            wl[u] = mj[hi][u] == -INFINITY ? 0.f : exp2f(mj[hi][u] - mn);
            dl += wl[u] * lj[hi][u];
          }
#pragma unroll
          for (int o = 16; o >= 1; o >>= 1) dl += __shfl_xor_sync(0xffffffffu, dl, o);
          den[hi] = fmaf(den[hi], alpha, dl);
#pragma unroll
          for (int e = 0; e < E; ++e) num[hi][e] *= alpha;
          const float* hb = buf + hl * SC * D + lane * E;
          for (int j = 0; j < sc; ++j) {
            const float wj = __shfl_sync(0xffffffffu, j < 32 ? wl[0] : wl[1], j & 31);
#pragma unroll
            for (int e4 = 0; e4 < E; e4 += 2) {
              const float2 x2 = *reinterpret_cast<const float2*>(hb + j * D + e4);
              num[hi][e4] = fmaf(wj, x2.x, num[hi][e4]);
              num[hi][e4 + 1] = fmaf(wj, x2.y, num[hi][e4 + 1]);
            }
          }
          Mh[hi] = mn;
        }
        fence_proxy_async();  // this round's reads of the buffer come before the next round's copies
        __syncthreads();
      }
#pragma unroll
      for (int hi = 0; hi < HPW; ++hi) {
        const int hl = warp + hi * L::NW;
        if (hl >= nh) break;
        const int h = h0 + hl;
        float o_v[E];
#pragma unroll
        for (int e = 0; e < E; ++e) o_v[e] = comb_failed ? __int_as_float(0x7fc00000) : num[hi][e] / den[hi];
        if (is_turbo(VT)) {
          // o <- s * H_un * o / D: butterflies of strides 1 .. E/2 in registers,
          // E .. D/2 across lanes
#pragma unroll
          for (int hs = 1; hs < E; hs <<= 1)
#pragma unroll
            for (int e = 0; e < E; ++e)
              if ((e & hs) == 0) {
                const float a0 = o_v[e], a1 = o_v[e + hs];
                o_v[e] = a0 + a1;
                o_v[e + hs] = a0 - a1;
              }
#pragma unroll
          for (int hs = E; hs < D; hs <<= 1) {
            const int lm = hs / E;
            const bool upper = (lane & lm) != 0;
#pragma unroll
            for (int e = 0; e < E; ++e) {
              const float other = __shfl_xor_sync(0xffffffffu, o_v[e], lm);
              o_v[e] = upper ? other - o_v[e] : o_v[e] + other;
            }
          }
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const int d = lane * E + e;
            const float sgn = ((p.tq.sign_bits[d >> 5] >> (d & 31)) & 1u) ? -1.f : 1.f;
            o_v[e] = o_v[e] * sgn / (float)D;
          }
        }
        float* dst = p.out + ((int64_t)b * p.n_q + (int64_t)kvh * G + h) * D + lane * E;
        if constexpr (E == 2) {
          *reinterpret_cast<float2*>(dst) = make_float2(o_v[0], o_v[1]);
        } else {
#pragma unroll
          for (int e4 = 0; e4 < E; e4 += 4)
            *reinterpret_cast<float4*>(dst + e4) = make_float4(o_v[e4], o_v[e4 + 1], o_v[e4 + 2], o_v[e4 + 3]);
        }
      }
    }
  }
}

// ------------------------------------------------------------------ host side

struct TcMaps {
  CUtensorMap kc, ks, vc, vs;
};

template <int KT, int VT, int NB, int NTH, bool PAGED>
cudaError_t launch_one(const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  using L = Layout<KT, VT, NB * 32>;
  auto kern = decode_tc_kernel<KT, VT, NB, NTH, PAGED>;
  static std::atomic<uint64_t> attr_done{0};
  const cudaError_t e = set_smem_limit_once(kern, L::DYN, attr_done);
  if (e != cudaSuccess) return e;
  const dim3 grid(a.p.S, a.p.n_kv, a.p.B);
  if (!a.p.pdl) {
    kern<<<grid, L::NW * 32, L::DYN, st>>>(a, m.kc, m.ks, m.vc, m.vs);
    return cudaGetLastError();
  }
  // programmatic dependent launch: may start once the previous kernel on the
  // stream has triggered (griddepcontrol.launch_dependents) or finished
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(L::NW * 32);
  cfg.dynamicSmemBytes = L::DYN;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, a, m.kc, m.ks, m.vc, m.vs);
}

template <int KT, int VT, int NB, bool PAGED>
cudaError_t launch_nb(int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  return nth == 1 ? launch_one<KT, VT, NB, 1, PAGED>(a, m, st) : launch_one<KT, VT, NB, 2, PAGED>(a, m, st);
}

template <int KT, int VT, bool PAGED>
cudaError_t launch_v(int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  switch (nb) {
    case 2: return launch_nb<KT, VT, 2, PAGED>(nth, a, m, st);
    case 4: return launch_nb<KT, VT, 4, PAGED>(nth, a, m, st);
    case 8:
      if constexpr (KT == KVQ_F16 && VT == KVQ_F16) return cudaErrorInvalidValue;
      else return launch_nb<KT, VT, 8, PAGED>(nth, a, m, st);
  }
  return cudaErrorInvalidValue;
}

template <int KT, bool PAGED>
cudaError_t launch_k(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  if constexpr (is_qjl(KT)) {  // turbo3_qjl keys: q8_0, q4_0 or turbo3 values
    if (vt == KVQ_Q8_0) return launch_v<KT, KVQ_Q8_0, PAGED>(nb, nth, a, m, st);
    if (vt == KVQ_Q4_0) return launch_v<KT, KVQ_Q4_0, PAGED>(nb, nth, a, m, st);
    if (vt == KVQ_TURBO3) return launch_v<KT, KVQ_TURBO3, PAGED>(nb, nth, a, m, st);
    return cudaErrorInvalidValue;
  } else if constexpr (is_turbo(KT)) {  // turbo keys: q8_0, q4_0 or the same turbo type as values
    if (vt == KVQ_Q8_0) return launch_v<KT, KVQ_Q8_0, PAGED>(nb, nth, a, m, st);
    if (vt == KVQ_Q4_0) return launch_v<KT, KVQ_Q4_0, PAGED>(nb, nth, a, m, st);
    if (vt == KT) return launch_v<KT, KT, PAGED>(nb, nth, a, m, st);
    return cudaErrorInvalidValue;
  } else {
    switch (vt) {
      case KVQ_F16: return launch_v<KT, KVQ_F16, PAGED>(nb, nth, a, m, st);
      case KVQ_Q8_0: return launch_v<KT, KVQ_Q8_0, PAGED>(nb, nth, a, m, st);
      case KVQ_Q4_0: return launch_v<KT, KVQ_Q4_0, PAGED>(nb, nth, a, m, st);
      case KVQ_Q5_0: return launch_v<KT, KVQ_Q5_0, PAGED>(nb, nth, a, m, st);
      case KVQ_TURBO2: return launch_v<KT, KVQ_TURBO2, PAGED>(nb, nth, a, m, st);
      case KVQ_TURBO3: return launch_v<KT, KVQ_TURBO3, PAGED>(nb, nth, a, m, st);
      case KVQ_TURBO4: return launch_v<KT, KVQ_TURBO4, PAGED>(nb, nth, a, m, st);
    }
    return cudaErrorInvalidValue;
  }
}

// one per key type and cache kind (contiguous, paged pool), each in its own
// translation unit so they compile in parallel
cudaError_t launch_kf16(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq8(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq4(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq5(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt2(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt3(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt4(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kqjl(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kf16_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq8_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq4_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kq5_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt2_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt3_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kt4_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);
cudaError_t launch_kqjl_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st);

}  // namespace tc
}  // namespace kvq
