// Split combine: merges the per-split softmax partials (m, l, acc) of the
// decode kernel into the attention output,
//   o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,   M = max_s m_s,
// which equals plain softmax attention over the whole context ("llama.cpp für
// Geschwindigkeit und Speicher optimieren", section "Flash Attention": the
// tiled form is exact).  For a turbo value cache the accumulators live in the
// rotated domain (sum_t p_t norm_t c[code_t]); the output is rotated back once:
// o <- s * H_un * o / d, with H_un the unnormalised Walsh-Hadamard matrix and
// s the seeded sign vector ("Benchmark TurboQuant en Apple Silicon", section
// "¿Qué es TurboQuant?").
//
// One CTA per (query head, batch row), one thread per output dim.  The
// workspace is a few MB at most and stays in L2 behind the decode kernel.
#include "kvq_internal.h"

namespace kvq {
namespace {

__device__ __forceinline__ float block_reduce(float v, bool is_max, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const float x = __shfl_xor_sync(0xffffffffu, v, o);
    v = is_max ? fmaxf(v, x) : v + x;
  }
  __syncthreads();  // red[] may still be read from a previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = red[0];
  for (int w = 1; w < nw; ++w) v = is_max ? fmaxf(v, red[w]) : v + red[w];
  return v;
}

// One CTA per (query head, batch row), one thread per output dim.  The split
// partials are read in parallel: the maxima and sums with one load per thread,
// then every thread's accumulator column with independent loads (the workspace
// is L2-resident behind the decode kernel).
__global__ void __launch_bounds__(256) combine_kernel(CombineParams p) {
  extern __shared__ float sm[];
  const int SS = p.S * p.n_ranks;  // splits of all ranks
  float* red = sm;              // 8 floats
  float* wts = sm + 8;          // SS weights
  float* xs = wts + SS;         // D values (turbo inverse transform)
  const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
  const int64_t base = ((int64_t)b * p.n_q + h) * p.S;
  // split k = r * S + s: rank r's split s
  auto at = [&](int k) -> int64_t { return (int64_t)(k / p.S) * p.rank_stride + base + k % p.S; };
  float M = -INFINITY;
  for (int s = j; s < SS; s += blockDim.x) M = fmaxf(M, p.ws_m[at(s)]);
  M = block_reduce(M, true, red);
  float den = 0.f;
  for (int s = j; s < SS; s += blockDim.x) {
    const float ms = p.ws_m[at(s)];
    const float w = ms == -INFINITY ? 0.f : exp2f(ms - M);  // empty split: weight 0
    wts[s] = w;
    den += w * p.ws_l[at(s)];
  }
  den = block_reduce(den, false, red);  // its barriers also publish wts[]
  float num = 0.f;
  int s = 0;
  constexpr int kU = 16;  // independent loads per round: the partials may come from HBM
  if (p.n_ranks == 1) {
    const float* acc = p.ws_acc + base * p.D + j;
    for (; s + kU <= SS; s += kU) {
      float a[kU];
#pragma unroll
      for (int u = 0; u < kU; ++u) a[u] = acc[(int64_t)(s + u) * p.D];
#pragma unroll
      for (int u = 0; u < kU; ++u) num = fmaf(wts[s + u], a[u], num);
    }
  }
  for (; s < SS; ++s) {
    const int64_t k = (int64_t)(s / p.S) * p.rank_stride + (base + s % p.S) * p.D + j;
    num = fmaf(wts[s], p.ws_acc[k], num);
  }
  float o = num / den;
  if (p.rotated) {
    xs[j] = o;
    for (int hs = 1; hs < p.D; hs <<= 1) {
      __syncthreads();
      if ((j & hs) == 0) {
        const float a = xs[j], c = xs[j + hs];
        xs[j] = a + c;
        xs[j + hs] = a - c;
      }
    }
    __syncthreads();
    const float sgn = ((p.tq.sign_bits[j >> 5] >> (j & 31)) & 1u) ? -1.f : 1.f;
    o = xs[j] * sgn / (float)p.D;
  }
  p.out[((int64_t)b * p.n_q + h) * p.D + j] = o;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t st) {
  const dim3 grid(p.n_q, p.B);
  const size_t smem = (8 + (size_t)p.S * p.n_ranks + (size_t)p.D) * sizeof(float);
  if (smem > 48 * 1024) return cudaErrorInvalidValue;
  combine_kernel<<<grid, p.D, smem, st>>>(p);
  return cudaGetLastError();
}

}  // namespace kvq
