// k6_decode_l12.cu -- instantiations of the one-kernel decode forward for K = 2^12.
#include "k6_decode_fused.cuh"

namespace hbl {
namespace k6 {
hbl_status launch_l12(const DecodeArgs& d, cudaStream_t s, int sms) { return launch_l<12>(d, s, sms); }
int smem_l12(int N, int MT, int sms) { return smem_bytes<12>(N, MT, sms); }
}  // namespace k6
}  // namespace hbl
