// k1_mode9.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 9: RMSNorm + Hadamard, with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<9, 0>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<9, kFlGain>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
