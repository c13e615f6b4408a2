// Quantize-on-append kernel: fp16 K/V rows -> f16 / q8_0 / q4_0 / turbo3 cache
// rows, K and V of one call in one launch.  The row bodies (formats, rounding,
// work mapping) are in append_rows.cuh.
#include "append_rows.cuh"

namespace kvq {
namespace {

constexpr int kAppendThreads = 256;

// CTAs a tensor of `type` needs (each CTA: 256 threads).
int64_t append_ctas(int32_t type, const AppendParams& p) {
  const int64_t rows = (int64_t)p.B * p.n_tok * p.H;
  const int64_t threads = rows * rows::row_threads(type, p.D);
  return (threads + kAppendThreads - 1) / kAppendThreads;
}

// K and V rows of one append call in one launch: CTAs [0, ctas0) quantize the
// first tensor, the rest the second; the branch on the type is uniform per CTA.
struct AppendPair {
  AppendParams p[2];
  int32_t type[2];
  int64_t ctas0;
};

__global__ void __launch_bounds__(kAppendThreads) append_pair_kernel(const AppendPair pp) {
  const int which = (int64_t)blockIdx.x < pp.ctas0 ? 0 : 1;
  const int64_t cta = which ? (int64_t)blockIdx.x - pp.ctas0 : (int64_t)blockIdx.x;
  const AppendParams& p = pp.p[which];
  const int64_t gend = (int64_t)p.B * p.n_tok * p.H * rows::row_threads(pp.type[which], p.D);
  rows::append_any(pp.type[which], p, cta * blockDim.x + threadIdx.x, gend);
}

}  // namespace

cudaError_t launch_append(const AppendParams* k, int32_t k_type, const AppendParams* v, int32_t v_type,
                          cudaStream_t st) {
  AppendPair pp{};
  int n = 0;
  int64_t ctas[2] = {0, 0};
  if (k) {
    pp.p[n] = *k;
    pp.type[n] = k_type;
    ctas[n++] = append_ctas(k_type, *k);
  }
  if (v) {
    pp.p[n] = *v;
    pp.type[n] = v_type;
    ctas[n++] = append_ctas(v_type, *v);
  }
  if (n == 0) return cudaSuccess;
  if (n == 1) ctas[1] = 0;
  pp.ctas0 = ctas[0];
  const int64_t total = ctas[0] + ctas[1];
  if (total <= 0 || total > 0x7fffffff) return cudaErrorInvalidValue;
  append_pair_kernel<<<(unsigned)total, kAppendThreads, 0, st>>>(pp);
  return cudaGetLastError();
}

}  // namespace kvq
