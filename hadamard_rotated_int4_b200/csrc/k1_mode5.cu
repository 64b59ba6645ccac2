// k1_mode5.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 5 (INT4 codes one per byte, interleaved layout), with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<5, false>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<5, true>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
