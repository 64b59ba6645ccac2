// k1_mode5.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 5: RMSNorm + Hadamard, with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<5, 0>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<5, kFlGain>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
