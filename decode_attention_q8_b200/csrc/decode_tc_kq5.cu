// Instantiations of the tensor-core decode kernel for one key cache type
// (split across translation units so they compile in parallel).
#include "decode_tc.cuh"

namespace kvq {
namespace tc {

cudaError_t launch_kq5(int vt, int nb, int nth, const TcArgs& a, const TcMaps& m, cudaStream_t st) {
  return launch_k<KVQ_Q5_0, false>(vt, nb, nth, a, m, st);
}

}  // namespace tc
}  // namespace kvq
