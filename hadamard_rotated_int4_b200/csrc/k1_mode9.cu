// k1_mode9.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 9 (INT8 codes, interleaved layout), with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<9, false>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<9, true>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
