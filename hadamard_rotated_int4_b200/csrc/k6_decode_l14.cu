// k6_decode_l14.cu -- instantiations of the decode kernels (one-kernel forward and
// GEMV half) for K = 2^14.
#include "k6_decode_fused.cuh"

namespace hbl {
namespace k6 {
hbl_status launch_l14(const DecodeArgs& d, cudaStream_t s, int sms) { return launch_l<14>(d, s, sms); }
int smem_l14(int N, int MT, int sms) { return smem_bytes<14>(N, MT, sms); }
hbl_status launch_gemv_l14(const GemvArgs& g, cudaStream_t s, int sms) {
    return launch_gemv_l<14>(g, s, sms);
}
int gemv_smem_l14(int N, int MT, int sms) { return gemv_smem_bytes<14>(N, MT, sms); }
}  // namespace k6
}  // namespace hbl
