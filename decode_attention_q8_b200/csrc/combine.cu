// Split combine: merges the per-split softmax partials (m, l, acc) of the
// decode kernel into the attention output,
//   o = sum_s 2^(m_s - M) acc_s / sum_s 2^(m_s - M) l_s,   M = max_s m_s,
// which equals plain softmax attention over the whole context ("llama.cpp für
// Geschwindigkeit und Speicher optimieren", section "Flash Attention": the
// tiled form is exact).  For a turbo3 value cache the accumulators live in the
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

__global__ void combine_kernel(CombineParams p) {
  extern __shared__ float x_s[];
  const int h = blockIdx.x, b = blockIdx.y, j = threadIdx.x;
  const int64_t base = ((int64_t)b * p.n_q + h) * p.S;
  float M = -INFINITY;
  for (int s = 0; s < p.S; ++s) M = fmaxf(M, p.ws_m[base + s]);
  float num = 0.f, den = 0.f;
  for (int s = 0; s < p.S; ++s) {
    const float ms = p.ws_m[base + s];
    if (ms == -INFINITY) continue;  // empty split
    const float w = exp2f(ms - M);
    num += w * p.ws_acc[(base + s) * p.D + j];
    den += w * p.ws_l[base + s];
  }
  float o = num / den;
  if (p.turbo3) {
    x_s[j] = o;
    for (int hs = 1; hs < p.D; hs <<= 1) {
      __syncthreads();
      if ((j & hs) == 0) {
        const float a = x_s[j], c = x_s[j + hs];
        x_s[j] = a + c;
        x_s[j + hs] = a - c;
      }
    }
    __syncthreads();
    const float sgn = ((p.t3.sign_bits[j >> 5] >> (j & 31)) & 1u) ? -1.f : 1.f;
    o = x_s[j] * sgn / (float)p.D;
  }
  p.out[((int64_t)b * p.n_q + h) * p.D + j] = o;
}

}  // namespace

cudaError_t launch_combine(const CombineParams& p, cudaStream_t st) {
  const dim3 grid(p.n_q, p.B);
  combine_kernel<<<grid, p.D, p.turbo3 ? p.D * sizeof(float) : 0, st>>>(p);
  return cudaGetLastError();
}

}  // namespace kvq
