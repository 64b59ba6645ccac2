// k1_mode0.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 0 (fp32 transform output), with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<0, false>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<0, true>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
