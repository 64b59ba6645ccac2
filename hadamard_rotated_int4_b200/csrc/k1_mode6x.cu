// k1_mode6x.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 6 (INT4 codes one per byte) with the packed ternary weights
// widened beside the rows: the large-batch forward's K1, with and without a
// gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<6, kFlExpand>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<6, kFlExpand | kFlGain>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
