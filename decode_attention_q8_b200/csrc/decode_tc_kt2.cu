// Instantiations of the tensor-core decode kernel for turbo2 key caches
// (split across translation units so they compile in parallel).
#include "decode_tc.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_kt2(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  return launch_k<KVQ_TURBO2, false>(vt, nb, nth, a, m, st);
}

}  // namespace tc
}  // namespace kvq
