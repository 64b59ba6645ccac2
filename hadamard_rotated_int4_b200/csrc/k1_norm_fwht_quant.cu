// k1_norm_fwht_quant.cu -- host launcher of the fused RMSNorm + Walsh-Hadamard
// + per-token quantisation kernel (the kernel itself is in k1_impl.cuh).
#include <cuda_runtime.h>
#include <math.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k1 {
struct Params;
template <int MODE, bool GAIN>
hbl_status dispatch(int L, const Params& prm, cudaStream_t s, int sms);
}  // namespace k1
}  // namespace hbl

#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
extern template hbl_status dispatch<0, false>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<0, true>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<4, false>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<4, true>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<5, false>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<5, true>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<9, false>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<9, true>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<8, false>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<8, true>(int, const Params&, cudaStream_t, int);
}  // namespace k1

hbl_status launch_norm_fwht_quant(const uint16_t* X, const float* gain, int64_t M, int K,
                                  float norm_eps, float quant_eps, int mode, void* codes,
                                  float* scales, int32_t* rowsum, float* V, cudaStream_t stream,
                                  int num_sms) {
    if (M == 0) return HBL_OK;
    k1::Params prm;
    prm.X = X;
    prm.gain = gain;
    prm.M = M;
    prm.norm_eps = norm_eps;
    prm.quant_eps = quant_eps;
    prm.cK = (float)(1.0 / sqrt((double)K));
    prm.s7 = (float)sqrt(7.0);
    prm.codes = static_cast<uint8_t*>(codes);
    prm.scales = scales;
    prm.rowsum = rowsum;
    prm.V = V;
    const int L = ilog2((unsigned)K);
    const bool g = gain != nullptr;
    switch (mode) {
        case 0: return g ? k1::dispatch<0, true>(L, prm, stream, num_sms)
                         : k1::dispatch<0, false>(L, prm, stream, num_sms);
        case 4: return g ? k1::dispatch<4, true>(L, prm, stream, num_sms)
                         : k1::dispatch<4, false>(L, prm, stream, num_sms);
        case 5: return g ? k1::dispatch<5, true>(L, prm, stream, num_sms)
                         : k1::dispatch<5, false>(L, prm, stream, num_sms);
        case 9: return g ? k1::dispatch<9, true>(L, prm, stream, num_sms)
                         : k1::dispatch<9, false>(L, prm, stream, num_sms);
        case 8: return g ? k1::dispatch<8, true>(L, prm, stream, num_sms)
                         : k1::dispatch<8, false>(L, prm, stream, num_sms);
        default: return HBL_ERR_INVALID_ARG;
    }
}

}  // namespace hbl
