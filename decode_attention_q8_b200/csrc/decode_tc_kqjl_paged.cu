// Instantiations of the tensor-core decode kernel for turbo3_qjl key caches over
// a paged pool (split across translation units so they compile in parallel).
#include "decode_tc.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_kqjl_paged(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  return launch_k<KVQ_TURBO3_QJL, true>(vt, nb, nth, a, m, st);
}

}  // namespace tc
}  // namespace kvq
