// Host side of the tensor-core decode kernel: TMA tensor maps over the cache
// planes and the launch.
//
// Code planes of f16 / q8_0 / q4_0 caches are described row by row
// ([planes][rows][row bytes], bytes as uint8) with the hardware swizzle whose
// span equals the row (32, 64 or 128 bytes; wider rows split into 128-byte
// segments).  turbo code planes and all scale planes are described as flat
// uint32 arrays per plane.  The row extent is ctx_len, so a 16-row tile that
// runs past the context reads zeros there.
#include <cudaTypedefs.h>

#include <mutex>

#include "decode_tc.cuh"

namespace kvq {
namespace {

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    (void)cudaGetLastError();
  });
  return fn;
}

// Swizzled row-wise map of a code plane.
bool code_map(CUtensorMap* m, const void* base, int rb, int64_t T, int64_t planes, int64_t ctx) {
  auto enc = encode_fn();
  if (!enc) return false;
  const CUtensorMapSwizzle swz = rb >= 128 ? CU_TENSOR_MAP_SWIZZLE_128B
                                 : rb == 64 ? CU_TENSOR_MAP_SWIZZLE_64B
                                            : CU_TENSOR_MAP_SWIZZLE_32B;
  CUresult r;
  if (rb <= 128) {
    const cuuint64_t dims[3] = {(cuuint64_t)rb, (cuuint64_t)ctx, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {(cuuint64_t)rb, (cuuint64_t)(T * rb)};
    const cuuint32_t box[3] = {(cuuint32_t)rb, (cuuint32_t)tc::kSub, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[4] = {128, (cuuint64_t)(rb / 128), (cuuint64_t)ctx, (cuuint64_t)planes};
    const cuuint64_t strides[3] = {128, (cuuint64_t)rb, (cuuint64_t)(T * rb)};
    const cuuint32_t box[4] = {128, (cuuint32_t)(rb / 128), (cuuint32_t)tc::kSub, 1};
    const cuuint32_t es[4] = {1, 1, 1, 1};
    r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 4, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

// Unswizzled map of a plane whose rows are rb bytes (rb a multiple of 2):
// flat uint32 per plane when a 16-row tile is at most 256 words, else row-wise.
bool flat_map(CUtensorMap* m, const void* base, int rb, int64_t T, int64_t planes, int64_t ctx) {
  auto enc = encode_fn();
  if (!enc) return false;
  const int tile_words = tc::kSub * rb / 4;
  CUresult r;
  if (tile_words <= 256) {
    const cuuint64_t dims[2] = {(cuuint64_t)((ctx * rb + 3) / 4), (cuuint64_t)planes};
    const cuuint64_t strides[1] = {(cuuint64_t)(T * rb)};
    const cuuint32_t box[2] = {(cuuint32_t)tile_words, 1};
    const cuuint32_t es[2] = {1, 1};
    r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  } else {
    const cuuint64_t dims[3] = {(cuuint64_t)(rb / 4), (cuuint64_t)ctx, (cuuint64_t)planes};
    const cuuint64_t strides[2] = {(cuuint64_t)rb, (cuuint64_t)(T * rb)};
    const cuuint32_t box[3] = {(cuuint32_t)(rb / 4), (cuuint32_t)tc::kSub, 1};
    const cuuint32_t es[3] = {1, 1, 1};
    r = enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, es,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  }
  return r == CUDA_SUCCESS;
}

bool plane_maps(const Plane& pl, int type, int64_t planes, int64_t ctx, CUtensorMap* codes, CUtensorMap* scales) {
  const bool ok = is_turbo(type) ? flat_map(codes, pl.codes, pl.code_bytes, pl.T, planes, ctx)
                                     : code_map(codes, pl.codes, pl.code_bytes, pl.T, planes, ctx);
  if (!ok) return false;
  if (pl.n_scales == 0) {
    *scales = *codes;  // unused by the kernel
    return true;
  }
  return flat_map(scales, pl.scales, 2 * pl.n_scales, pl.T, planes, ctx);
}

}  // namespace

bool decode_supported(int32_t k_type, int32_t v_type, int32_t G, int32_t D) {
  if (G < 1 || G > 16) return false;
  // turbo3_qjl keys: with q8_0, q4_0 or turbo3 values; other turbo keys: with
  // q8_0, q4_0 or the same turbo type as values
  if (is_qjl(k_type) && v_type != KVQ_Q8_0 && v_type != KVQ_Q4_0 && v_type != KVQ_TURBO3) return false;
  if (is_turbo(k_type) && !is_qjl(k_type) && v_type != KVQ_Q8_0 && v_type != KVQ_Q4_0 && v_type != k_type)
    return false;
  if (D != 64 && D != 128 && D != 256) return false;
  if (D == 256 && k_type == KVQ_F16 && v_type == KVQ_F16) return false;  // stage would not fit
  return true;
}

namespace {
template <int KT>
int ctas_k(int32_t v_type, int32_t D, int nth) {
  switch (v_type) {
    case KVQ_F16: return tc::resident_ctas_for(KT, KVQ_F16, D, nth);
    case KVQ_Q8_0: return tc::resident_ctas_for(KT, KVQ_Q8_0, D, nth);
    case KVQ_Q4_0: return tc::resident_ctas_for(KT, KVQ_Q4_0, D, nth);
    case KVQ_Q5_0: return tc::resident_ctas_for(KT, KVQ_Q5_0, D, nth);
    case KVQ_TURBO2: return tc::resident_ctas_for(KT, KVQ_TURBO2, D, nth);
    case KVQ_TURBO3: return tc::resident_ctas_for(KT, KVQ_TURBO3, D, nth);
    case KVQ_TURBO4: return tc::resident_ctas_for(KT, KVQ_TURBO4, D, nth);
  }
  return 1;
}
}  // namespace

int decode_ctas_per_sm(int32_t k_type, int32_t v_type, int32_t D, int32_t G) {
  const int nth = G > 8 ? 2 : 1;  // query-head n-tiles of the instance
  switch (k_type) {
    case KVQ_F16: return ctas_k<KVQ_F16>(v_type, D, nth);
    case KVQ_Q8_0: return ctas_k<KVQ_Q8_0>(v_type, D, nth);
    case KVQ_Q4_0: return ctas_k<KVQ_Q4_0>(v_type, D, nth);
    case KVQ_Q5_0: return ctas_k<KVQ_Q5_0>(v_type, D, nth);
    case KVQ_TURBO2: return ctas_k<KVQ_TURBO2>(v_type, D, nth);
    case KVQ_TURBO3: return ctas_k<KVQ_TURBO3>(v_type, D, nth);
    case KVQ_TURBO4: return ctas_k<KVQ_TURBO4>(v_type, D, nth);
    case KVQ_TURBO3_QJL: return ctas_k<KVQ_TURBO3_QJL>(v_type, D, nth);
  }
  return 1;
}


cudaError_t launch_decode(int32_t k_type, int32_t v_type, const DecodeParams& p, cudaStream_t st) {
  tc::TcMaps maps;
  // a paged pool is a cache of n_pages "batch rows" of one page each
  const bool paged = p.block_table != nullptr;
  const int64_t planes = (paged ? p.n_pages : (int64_t)p.B) * p.n_kv;
  const int64_t rows = paged ? ((int64_t)1 << p.log2_page) : p.ctx;
  if (!plane_maps(p.k, k_type, planes, rows, &maps.kc, &maps.ks) ||
      !plane_maps(p.v, v_type, planes, rows, &maps.vc, &maps.vs))
    return cudaErrorInvalidValue;
  tc::TcArgs a;
  a.p = p;
  const int nb = p.D / 32, nth = p.G <= 8 ? 1 : 2;
  if (paged) {
    switch (k_type) {
      case KVQ_F16: return tc::launch_kf16_paged(v_type, nb, nth, a, maps, st);
      case KVQ_Q8_0: return tc::launch_kq8_paged(v_type, nb, nth, a, maps, st);
      case KVQ_Q4_0: return tc::launch_kq4_paged(v_type, nb, nth, a, maps, st);
      case KVQ_Q5_0: return tc::launch_kq5_paged(v_type, nb, nth, a, maps, st);
      case KVQ_TURBO2: return tc::launch_kt2_paged(v_type, nb, nth, a, maps, st);
      case KVQ_TURBO3: return tc::launch_kt3_paged(v_type, nb, nth, a, maps, st);
      case KVQ_TURBO4: return tc::launch_kt4_paged(v_type, nb, nth, a, maps, st);
      case KVQ_TURBO3_QJL: return tc::launch_kqjl_paged(v_type, nb, nth, a, maps, st);
    }
    return cudaErrorInvalidValue;
  }
  switch (k_type) {
    case KVQ_F16: return tc::launch_kf16(v_type, nb, nth, a, maps, st);
    case KVQ_Q8_0: return tc::launch_kq8(v_type, nb, nth, a, maps, st);
    case KVQ_Q4_0: return tc::launch_kq4(v_type, nb, nth, a, maps, st);
    case KVQ_Q5_0: return tc::launch_kq5(v_type, nb, nth, a, maps, st);
    case KVQ_TURBO2: return tc::launch_kt2(v_type, nb, nth, a, maps, st);
    case KVQ_TURBO3: return tc::launch_kt3(v_type, nb, nth, a, maps, st);
    case KVQ_TURBO4: return tc::launch_kt4(v_type, nb, nth, a, maps, st);
    case KVQ_TURBO3_QJL: return tc::launch_kqjl(v_type, nb, nth, a, maps, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace kvq
