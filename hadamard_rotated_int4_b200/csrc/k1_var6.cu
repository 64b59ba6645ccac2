// k1_var6.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 6, variants: no Hadamard transform and/or LayerNorm, each
// with and without a gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<6, kFlNoHadamard>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<6, kFlNoHadamard | kFlGain>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<6, kFlLayerNorm>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<6, kFlLayerNorm | kFlGain>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<6, kFlLayerNorm | kFlNoHadamard>(int, const Params&, cudaStream_t,
                                                               int);
template hbl_status dispatch<6, kFlLayerNorm | kFlNoHadamard | kFlGain>(int, const Params&,
                                                                         cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
