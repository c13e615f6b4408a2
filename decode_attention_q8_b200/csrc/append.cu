// Quantize-on-append kernel: fp16 K/V rows -> f16 / q8_0 / q4_0 / q5_0 / turbo
// cache rows, K and V of one call in one launch.  The row bodies (formats, rounding,
// work mapping) are in append_rows.cuh.
#include <algorithm>

#include "append_rows.cuh"

namespace kvq {
namespace {

constexpr int kAppendThreads = 256;
constexpr int kAppendRound = 4;  // work items per thread and round: loads in flight
constexpr int kBlockRound = 1;   // q8_0 / q4_0 blocks per thread and round (a block is 4 loads)

// Work items of one row in this kernel: a 32-element block for q8_0 / q4_0,
// otherwise the row bodies' threads.
__host__ __device__ constexpr int bulk_items(int32_t type, int d) {
  return type == KVQ_Q8_0 || type == KVQ_Q4_0 || type == KVQ_Q5_0 ? d / kBlock : rows::bulk_row_threads(type, d);
}

// K and V rows of one append call in one launch.  Every CTA takes its share of
// the first tensor's rows, then of the second's (the branch on the type is
// uniform per CTA), so the two parts stay balanced whatever their cost.  Each
// part runs grid-stride over its flat work: a thread loads several items
// (stride apart) before it quantizes and stores them, so a grid of one
// resident wave keeps enough reads in flight to stream at HBM rates.  Strides
// are multiples of 32, so each lane keeps its place in the 8-lane block groups
// and the warps of the shuffles stay whole.
struct AppendPair {
  AppendParams p[2];
  int32_t type[2];
  int32_t n;           // tensors in the call (1 or 2)
  int32_t stage_proj;  // turbo3_qjl keys: copy P to shared memory first
};

template <int TYPE, int E>
__device__ __forceinline__ void append_stream(const AppendParams& p, int64_t first, int64_t stride, int64_t gend,
                                              const float* pt = nullptr) {
  for (int64_t base = first; (base & ~(int64_t)31) < gend; base += kAppendRound * stride) {
    uint4 raw[kAppendRound];
#pragma unroll
    for (int u = 0; u < kAppendRound; ++u) raw[u] = rows::load_raw<TYPE, E>(p, base + u * stride, gend);
#pragma unroll
    for (int u = 0; u < kAppendRound; ++u) {
      const int64_t g = base + u * stride;
      if ((g & ~(int64_t)31) < gend) rows::finish<TYPE, E>(p, g, gend, raw[u], pt);  // warp-uniform
    }
  }
}

// q8_0 / q4_0: one thread per 32-element block; kBlockRound blocks (four
// 16-byte loads each) in flight per thread.  One block per round measured
// fastest: the smaller body keeps the instruction cache warm and the
// registers at 64 (four CTAs per SM).
template <int TYPE>
__device__ __forceinline__ void append_blocks(const AppendParams& p, int64_t first, int64_t stride, int64_t nblk) {
  for (int64_t base = first; base < nblk; base += kBlockRound * stride) {
    rows::BlockRaw raw[kBlockRound];
#pragma unroll
    for (int u = 0; u < kBlockRound; ++u) raw[u] = rows::load_block(p, base + u * stride, nblk);
#pragma unroll
    for (int u = 0; u < kBlockRound; ++u) {
      const int64_t g = base + u * stride;
      if (g < nblk) {
        if constexpr (TYPE == KVQ_Q8_0) rows::q8_0_block(p, g, raw[u]);
        else if constexpr (TYPE == KVQ_Q4_0) rows::q4_0_block(p, g, raw[u]);
        else rows::q5_0_block(p, g, raw[u]);
      }
    }
  }
}

// Turbo rows other than turbo3_qjl: D/16 lanes per row (rows::append_turbo_wide),
// kWideRound items (32 bytes of fp16 each) in flight per thread.
constexpr int kWideRound = 2;
template <int TYPE, int D>
__device__ __forceinline__ void append_stream_wide(const AppendParams& p, int64_t first, int64_t stride, int64_t gend) {
  for (int64_t base = first; (base & ~(int64_t)31) < gend; base += kWideRound * stride) {
    rows::Raw32 raw[kWideRound];
#pragma unroll
    for (int u = 0; u < kWideRound; ++u) raw[u] = rows::load_wide(p, base + u * stride, gend);
#pragma unroll
    for (int u = 0; u < kWideRound; ++u) {
      const int64_t g = base + u * stride;
      if ((g & ~(int64_t)31) < gend) rows::append_turbo_wide<turbo_bits(TYPE), D>(p, g, gend, raw[u]);  // warp-uniform
    }
  }
}

template <int TYPE>
__device__ __forceinline__ void append_turbo_part(const AppendParams& p, int64_t first, int64_t stride, int64_t gend,
                                                  const float* pt = nullptr) {
  if constexpr (!is_qjl(TYPE)) {
    switch (p.D) {
      case 32: append_stream_wide<TYPE, 32>(p, first, stride, gend); break;
      case 64: append_stream_wide<TYPE, 64>(p, first, stride, gend); break;
      case 128: append_stream_wide<TYPE, 128>(p, first, stride, gend); break;
      case 256: append_stream_wide<TYPE, 256>(p, first, stride, gend); break;
    }
  } else {
    switch (p.D) {
      case 32: append_stream<TYPE, 1>(p, first, stride, gend, pt); break;
      case 64: append_stream<TYPE, 2>(p, first, stride, gend, pt); break;
      case 128: append_stream<TYPE, 4>(p, first, stride, gend, pt); break;
      case 256: append_stream<TYPE, 8>(p, first, stride, gend, pt); break;
    }
  }
}

// QJL: the instance that also takes turbo3_qjl rows (their projection loop
// needs far more registers; the other types keep the lean instance).
template <bool QJL>
__device__ __forceinline__ void append_part(const AppendParams& p, int32_t type, int64_t first, int64_t stride,
                                            const float* pt) {
  const int64_t gend = (int64_t)p.B * p.n_tok * p.H * bulk_items(type, p.D);
  switch (type) {
    case KVQ_F16: append_stream<KVQ_F16, 0>(p, first, stride, gend); break;
    case KVQ_Q8_0: append_blocks<KVQ_Q8_0>(p, first, stride, gend); break;
    case KVQ_Q4_0: append_blocks<KVQ_Q4_0>(p, first, stride, gend); break;
    case KVQ_Q5_0: append_blocks<KVQ_Q5_0>(p, first, stride, gend); break;
    case KVQ_TURBO2: append_turbo_part<KVQ_TURBO2>(p, first, stride, gend); break;
    case KVQ_TURBO3: append_turbo_part<KVQ_TURBO3>(p, first, stride, gend); break;
    case KVQ_TURBO4: append_turbo_part<KVQ_TURBO4>(p, first, stride, gend); break;
    case KVQ_TURBO3_QJL:
      if constexpr (QJL) append_turbo_part<KVQ_TURBO3_QJL>(p, first, stride, gend, pt);
      break;
  }
}

// The QJL instance first copies the keys' projection P transposed into shared
// memory when it fits (D <= kQjlSmemDim) and a CTA has enough rows to repay
// the copy (at least kQjlStageRows), so each step of a row's projection reads
// one contiguous line; every output still sums its D terms in order.
constexpr int kQjlSmemDim = 128;
constexpr int kQjlStageRows = 32;

template <bool QJL>
__global__ void __launch_bounds__(kAppendThreads) append_pair_kernel(const AppendPair pp) {
  const int64_t first = (int64_t)blockIdx.x * kAppendThreads + threadIdx.x;
  const int64_t stride = (int64_t)gridDim.x * kAppendThreads;
  const float* pt = nullptr;
  if constexpr (QJL) {
    extern __shared__ float pt_smem[];
    const AppendParams& pk = pp.p[0];  // turbo3_qjl is a key type: the first tensor
    if (pp.stage_proj) {
      const int D = pk.D;
      for (int t = threadIdx.x; t < D * D; t += kAppendThreads) {
        const int i = t / D, j = t - i * D;  // coalesced read of P[i][j]
        pt_smem[j * D + i] = __ldg(qjl_proj(pk.tq) + t);
      }
      __syncthreads();
      pt = pt_smem;
    }
  }
  append_part<QJL>(pp.p[0], pp.type[0], first, stride, pt);
  if (pp.n == 2) append_part<QJL>(pp.p[1], pp.type[1], first, stride, pt);
}

// Resident 256-thread CTAs of the append kernel on the whole current device
// (one wave); 148 SMs x 4 if the device cannot be asked.
template <bool QJL>
int64_t resident_ctas(size_t smem) {
  int dev = 0, sms = 0, per_sm = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
      cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, append_pair_kernel<QJL>, kAppendThreads, smem) !=
          cudaSuccess ||
      sms <= 0 || per_sm <= 0) {
    (void)cudaGetLastError();
    return 148 * 4;
  }
  return (int64_t)sms * per_sm;
}

// CTAs the work of a tensor needs (one item per thread).
int64_t append_ctas(int32_t type, const AppendParams& p) {
  const int64_t threads = (int64_t)p.B * p.n_tok * p.H * bulk_items(type, p.D);
  return (threads + kAppendThreads - 1) / kAppendThreads;
}

}  // namespace

cudaError_t launch_append(const AppendParams* k, int32_t k_type, const AppendParams* v, int32_t v_type,
                          cudaStream_t st) {
  AppendPair pp{};
  int n = 0;
  const AppendParams* ps[2] = {k, v};
  const int32_t ts[2] = {k_type, v_type};
  for (int i = 0; i < 2; ++i) {
    if (!ps[i]) continue;
    pp.p[n] = *ps[i];
    pp.type[n] = ts[i];
    ++n;
  }
  if (n == 0) return cudaSuccess;
  pp.n = n;
  int64_t need = append_ctas(pp.type[0], pp.p[0]);
  if (n == 2) need = std::max(need, append_ctas(pp.type[1], pp.p[1]));
  const bool qjl = is_qjl(pp.type[0]) || (n == 2 && is_qjl(pp.type[1]));
  if (!qjl) {
    const int64_t ctas = std::min(need, resident_ctas<false>(0));
    if (ctas <= 0) return cudaSuccess;  // no rows
    append_pair_kernel<false><<<(unsigned)ctas, kAppendThreads, 0, st>>>(pp);
    return cudaGetLastError();
  }
  // turbo3_qjl keys come first (a key type); P transposed in shared memory
  const int D = pp.p[0].D;
  const bool can_stage = is_qjl(pp.type[0]) && D <= kQjlSmemDim;
  static std::atomic<uint64_t> attr_done{0};
  const cudaError_t e =
      set_smem_limit_once(append_pair_kernel<true>, (int)(sizeof(float) * kQjlSmemDim * kQjlSmemDim), attr_done);
  if (e != cudaSuccess) return e;
  const int64_t ctas = std::min(need, resident_ctas<true>(can_stage ? sizeof(float) * D * D : 0));
  if (ctas <= 0) return cudaSuccess;
  const int64_t key_rows = (int64_t)pp.p[0].B * pp.p[0].n_tok * pp.p[0].H;
  pp.stage_proj = can_stage && key_rows >= kQjlStageRows * ctas ? 1 : 0;
  const size_t smem = pp.stage_proj ? sizeof(float) * D * D : 0;
  append_pair_kernel<true><<<(unsigned)ctas, kAppendThreads, smem, st>>>(pp);
  return cudaGetLastError();
}

}  // namespace kvq
