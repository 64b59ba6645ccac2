// k6_decode_l13.cu -- instantiations of the one-kernel decode forward for K = 2^13.
#include "k6_decode_fused.cuh"

namespace hbl {
namespace k6 {
hbl_status launch_l13(const DecodeArgs& d, cudaStream_t s, int sms) { return launch_l<13>(d, s, sms); }
int smem_l13(int N, int MT, int sms) { return smem_bytes<13>(N, MT, sms); }
}  // namespace k6
}  // namespace hbl
