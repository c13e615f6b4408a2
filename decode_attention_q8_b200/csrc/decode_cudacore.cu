// Split-KV decode attention over a quantized KV cache -- CUDA-core version.
//
// Flash attention computes attention tile by tile and is exactly standard
// attention ("llama.cpp für Geschwindigkeit und Speicher optimieren", section
// "Flash Attention").  In decode form each CTA owns one (split, KV head,
// batch row) and streams its contiguous slice of cache rows once, for the whole
// GQA group of that KV head, keeping an online softmax (running max and sum)
// and an fp32 PV accumulator; the partials go to the workspace and
// kvq_combine merges them.
//
// Mapping (4 warps, each an independent online-softmax stream over every 4th
// 32-row chunk of the slice):
//   QK  lane = cache row: the lane dequantizes its row block by block and dots
//       it with the group's queries, which sit pre-scaled (scale*log2 e) in
//       shared memory as q_s[dim][head] and are read as broadcasts;
//       quantized blocks accumulate sum q*code and multiply by the block scale
//       once;
//   PV  lane = DPL contiguous output dims: for each row of the chunk the lane
//       dequantizes its dims and accumulates p[row][head] (broadcast from
//       shared memory) times value.
// turbo3 values accumulate norm_t * c[code] in the rotated domain; the combine
// applies the inverse rotation once per output.
#include <cfloat>

#include "kvq_internal.h"

namespace kvq {
namespace {

constexpr int kGP = 8;   // heads per KV group handled by this kernel (G <= 8)
constexpr int kNW = 4;   // warps per CTA

template <int KT>
__device__ __forceinline__ void qk_block(const uint8_t* row, const __half* scales, int blk,
                                         const float (*q_s)[kGP], float sc[kGP]) {
  float part[kGP];
#pragma unroll
  for (int h = 0; h < kGP; ++h) part[h] = 0.f;
  if (KT == KVQ_F16) {
    const uint4* src = reinterpret_cast<const uint4*>(row + blk * 64);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint4 raw = src[c];
      const __half* hv = reinterpret_cast<const __half*>(&raw);
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float kv = __half2float(hv[e]);
        const float4 qa = *reinterpret_cast<const float4*>(&q_s[blk * 32 + c * 8 + e][0]);
        const float4 qb = *reinterpret_cast<const float4*>(&q_s[blk * 32 + c * 8 + e][4]);
        part[0] += qa.x * kv; part[1] += qa.y * kv; part[2] += qa.z * kv; part[3] += qa.w * kv;
        part[4] += qb.x * kv; part[5] += qb.y * kv; part[6] += qb.z * kv; part[7] += qb.w * kv;
      }
    }
#pragma unroll
    for (int h = 0; h < kGP; ++h) sc[h] += part[h];
  } else {
    uint8_t bytes[32];
    if (KT == KVQ_Q8_0) {
      const uint4* src = reinterpret_cast<const uint4*>(row + blk * 32);
      *reinterpret_cast<uint4*>(bytes) = src[0];
      *reinterpret_cast<uint4*>(bytes + 16) = src[1];
    } else {
      *reinterpret_cast<uint4*>(bytes) = *reinterpret_cast<const uint4*>(row + blk * 16);
    }
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      float kv;
      if (KT == KVQ_Q8_0) kv = (float)(int8_t)bytes[e];
      else kv = (float)((e < 16 ? (bytes[e] & 0xF) : (bytes[e - 16] >> 4)) - 8);
      const float4 qa = *reinterpret_cast<const float4*>(&q_s[blk * 32 + e][0]);
      const float4 qb = *reinterpret_cast<const float4*>(&q_s[blk * 32 + e][4]);
      part[0] += qa.x * kv; part[1] += qa.y * kv; part[2] += qa.z * kv; part[3] += qa.w * kv;
      part[4] += qb.x * kv; part[5] += qb.y * kv; part[6] += qb.z * kv; part[7] += qb.w * kv;
    }
    const float d = __half2float(scales[blk]);
#pragma unroll
    for (int h = 0; h < kGP; ++h) sc[h] += d * part[h];
  }
}

// DPL contiguous dims starting at lane*DPL of one value row, dequantized.
template <int VT, int DPL>
__device__ __forceinline__ void load_v(const uint8_t* row, const __half* scales, int lane,
                                       const Turbo3Consts& t3, float out[DPL]) {
  const int j0 = lane * DPL;
  if (VT == KVQ_F16) {
    const __half* hv = reinterpret_cast<const __half*>(row) + j0;
#pragma unroll
    for (int e = 0; e < DPL; ++e) out[e] = __half2float(hv[e]);
  } else if (VT == KVQ_Q8_0) {
    const float d = __half2float(scales[j0 / 32]);
#pragma unroll
    for (int e = 0; e < DPL; ++e) out[e] = d * (float)(int8_t)row[j0 + e];
  } else if (VT == KVQ_Q4_0) {
    const int blk = j0 / 32, pos = j0 % 32;
    const float d = __half2float(scales[blk]);
    const uint8_t* bb = row + blk * 16 + (pos % 16);
#pragma unroll
    for (int e = 0; e < DPL; ++e) {
      const int code = pos < 16 ? (bb[e] & 0xF) : (bb[e] >> 4);
      out[e] = d * (float)(code - 8);
    }
  } else {  // turbo3: norm * c[code], rotated domain
    const float nrm = __half2float(scales[0]);
    const int bit0 = 3 * j0;
    uint32_t w = 0;
    const int nbytes = (3 * DPL + (bit0 & 7) + 7) / 8;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      if (i < nbytes) w |= (uint32_t)row[bit0 / 8 + i] << (8 * i);
    w >>= (bit0 & 7);
#pragma unroll
    for (int e = 0; e < DPL; ++e) out[e] = nrm * t3.levels[(w >> (3 * e)) & 7];
  }
}

template <int KT, int VT, int DPL>
__global__ void __launch_bounds__(kNW * 32) decode_cudacore_kernel(DecodeParams p) {
  constexpr int D = DPL * 32;
  __shared__ __align__(16) float q_s[D][kGP];
  __shared__ __align__(16) float p_s[kNW][32][kGP];
  __shared__ float m_w[kNW][kGP], l_w[kNW][kGP];
  __shared__ float acc_w[kNW][kGP][D];

  const int s = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const int tid = threadIdx.x, w = tid >> 5, lane = tid & 31;
  const int64_t t0 = (int64_t)s * p.chunk;
  const int64_t t1 = min(p.ctx, t0 + p.chunk);

  for (int i = tid; i < D * kGP; i += kNW * 32) {
    const int j = i / kGP, h = i % kGP;
    q_s[j][h] = h < p.G ? __half2float(p.q[((int64_t)b * p.n_q + (int64_t)g * p.G + h) * D + j]) * p.qscale
                        : 0.f;
  }
  __syncthreads();

  const int64_t plane = (int64_t)b * p.n_kv + g;
  const uint8_t* kc = p.k.codes + plane * p.k.T * p.k.code_bytes;
  const __half* ks = p.k.scales + plane * p.k.T * p.k.n_scales;
  const uint8_t* vc = p.v.codes + plane * p.v.T * p.v.code_bytes;
  const __half* vs = p.v.scales + plane * p.v.T * p.v.n_scales;

  float m[kGP], lsum[kGP], acc[kGP][DPL];
#pragma unroll
  for (int h = 0; h < kGP; ++h) {
    m[h] = -INFINITY;
    lsum[h] = 0.f;
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc[h][e] = 0.f;
  }

  for (int64_t base = t0 + (int64_t)w * 32; base < t1; base += kNW * 32) {
    const int64_t t = base + lane;
    const bool valid = t < t1;
    float sc[kGP];
#pragma unroll
    for (int h = 0; h < kGP; ++h) sc[h] = 0.f;
    if (valid) {
      const uint8_t* row = kc + t * p.k.code_bytes;
      const __half* srow = ks + t * p.k.n_scales;
#pragma unroll 1
      for (int blk = 0; blk < D / 32; ++blk) qk_block<KT>(row, srow, blk, q_s, sc);
    }
#pragma unroll
    for (int h = 0; h < kGP; ++h) {
      float mc = valid ? sc[h] : -INFINITY;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
      const float mn = fmaxf(m[h], mc);  // finite: lane 0 of a chunk is always valid
      const float alpha = exp2f(m[h] - mn);
      const float pv = valid ? exp2f(sc[h] - mn) : 0.f;
      lsum[h] = lsum[h] * alpha + pv;
#pragma unroll
      for (int e = 0; e < DPL; ++e) acc[h][e] *= alpha;
      m[h] = mn;
      p_s[w][lane][h] = pv;
    }
    __syncwarp();
    const int nvalid = (int)(t1 - base < 32 ? t1 - base : 32);
#pragma unroll 1
    for (int tt = 0; tt < nvalid; ++tt) {
      float vv[DPL];
      load_v<VT, DPL>(vc + (base + tt) * p.v.code_bytes, vs + (base + tt) * p.v.n_scales, lane, p.t3, vv);
      const float4 pa = *reinterpret_cast<const float4*>(&p_s[w][tt][0]);
      const float4 pb = *reinterpret_cast<const float4*>(&p_s[w][tt][4]);
      const float pp[kGP] = {pa.x, pa.y, pa.z, pa.w, pb.x, pb.y, pb.z, pb.w};
#pragma unroll
      for (int h = 0; h < kGP; ++h)
#pragma unroll
        for (int e = 0; e < DPL; ++e) acc[h][e] += pp[h] * vv[e];
    }
    __syncwarp();
  }

#pragma unroll
  for (int h = 0; h < kGP; ++h) {
    float l = lsum[h];
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) l += __shfl_xor_sync(0xffffffffu, l, o);
    if (lane == 0) {
      m_w[w][h] = m[h];
      l_w[w][h] = l;
    }
#pragma unroll
    for (int e = 0; e < DPL; ++e) acc_w[w][h][lane * DPL + e] = acc[h][e];
  }
  __syncthreads();

  for (int i = tid; i < p.G * D; i += kNW * 32) {
    const int h = i / D, j = i % D;
    float M = -INFINITY;
#pragma unroll
    for (int ww = 0; ww < kNW; ++ww) M = fmaxf(M, m_w[ww][h]);
    float a = 0.f, l = 0.f;
    if (M != -INFINITY) {
#pragma unroll
      for (int ww = 0; ww < kNW; ++ww) {
        const float f = exp2f(m_w[ww][h] - M);
        a += f * acc_w[ww][h][j];
        l += f * l_w[ww][h];
      }
    }
    const int64_t row = ((int64_t)b * p.n_q + (int64_t)g * p.G + h) * p.S + s;
    p.ws_acc[row * D + j] = a;
    if (j == 0) {
      p.ws_m[row] = M;
      p.ws_l[row] = l;
    }
  }
}

template <int KT, int VT>
cudaError_t launch_kv(const DecodeParams& p, cudaStream_t st) {
  const dim3 grid(p.S, p.n_kv, p.B);
  switch (p.D) {
    case 64: decode_cudacore_kernel<KT, VT, 2><<<grid, kNW * 32, 0, st>>>(p); break;
    case 128: decode_cudacore_kernel<KT, VT, 4><<<grid, kNW * 32, 0, st>>>(p); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

template <int KT>
cudaError_t launch_k(int32_t v_type, const DecodeParams& p, cudaStream_t st) {
  switch (v_type) {
    case KVQ_F16: return launch_kv<KT, KVQ_F16>(p, st);
    case KVQ_Q8_0: return launch_kv<KT, KVQ_Q8_0>(p, st);
    case KVQ_Q4_0: return launch_kv<KT, KVQ_Q4_0>(p, st);
    case KVQ_TURBO3: return launch_kv<KT, KVQ_TURBO3>(p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace

bool decode_supported(int32_t k_type, int32_t v_type, int32_t G, int32_t D) {
  (void)v_type;
  return k_type != KVQ_TURBO3 && G >= 1 && G <= kGP && (D == 64 || D == 128);
}

int decode_ctas_per_sm() { return 8; }

cudaError_t launch_decode(int32_t k_type, int32_t v_type, const DecodeParams& p, cudaStream_t st) {
  switch (k_type) {
    case KVQ_F16: return launch_k<KVQ_F16>(v_type, p, st);
    case KVQ_Q8_0: return launch_k<KVQ_Q8_0>(v_type, p, st);
    case KVQ_Q4_0: return launch_k<KVQ_Q4_0>(v_type, p, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
