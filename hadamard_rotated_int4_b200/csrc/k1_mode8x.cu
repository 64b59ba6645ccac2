// k1_mode8x.cu -- instantiations of the fused norm + transform + quantisation
// kernel for mode 8 (INT8 codes) with the packed ternary weights
// widened beside the rows: the large-batch forward's K1, with and without a
// gain vector.
#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
template hbl_status dispatch<8, kFlExpand>(int, const Params&, cudaStream_t, int);
template hbl_status dispatch<8, kFlExpand | kFlGain>(int, const Params&, cudaStream_t, int);
}  // namespace k1
}  // namespace hbl
