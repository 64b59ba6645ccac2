// k1_norm_fwht_quant.cu -- host launcher of the fused RMSNorm + Walsh-Hadamard
// + per-token quantisation kernel (the kernel itself is in k1_impl.cuh).
#include <cuda_runtime.h>
#include <math.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k1 {
struct Params;
template <int MODE, int FL>
hbl_status dispatch(int L, const Params& prm, cudaStream_t s, int sms);
}  // namespace k1
}  // namespace hbl

#include "k1_impl.cuh"

namespace hbl {
namespace k1 {
#define HBL_K1_EXTERN(MODE)                                                                      \
    extern template hbl_status dispatch<MODE, 0>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 1>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 2>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 3>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 4>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 5>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 6>(int, const Params&, cudaStream_t, int);        \
    extern template hbl_status dispatch<MODE, 7>(int, const Params&, cudaStream_t, int);
HBL_K1_EXTERN(0)
HBL_K1_EXTERN(4)
HBL_K1_EXTERN(5)
HBL_K1_EXTERN(6)
HBL_K1_EXTERN(8)
HBL_K1_EXTERN(9)
#undef HBL_K1_EXTERN
extern template hbl_status dispatch<6, kFlExpand>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<6, kFlExpand | kFlGain>(int, const Params&, cudaStream_t,
                                                            int);
extern template hbl_status dispatch<8, kFlExpand>(int, const Params&, cudaStream_t, int);
extern template hbl_status dispatch<8, kFlExpand | kFlGain>(int, const Params&, cudaStream_t,
                                                            int);

template <int MODE>
static hbl_status by_flags(int fl, int L, const Params& prm, cudaStream_t s, int sms) {
    switch (fl) {
        case 0: return dispatch<MODE, 0>(L, prm, s, sms);
        case 1: return dispatch<MODE, 1>(L, prm, s, sms);
        case 2: return dispatch<MODE, 2>(L, prm, s, sms);
        case 3: return dispatch<MODE, 3>(L, prm, s, sms);
        case 4: return dispatch<MODE, 4>(L, prm, s, sms);
        case 5: return dispatch<MODE, 5>(L, prm, s, sms);
        case 6: return dispatch<MODE, 6>(L, prm, s, sms);
        case 7: return dispatch<MODE, 7>(L, prm, s, sms);
        default: break;
    }
    if constexpr (MODE == 6 || MODE == 8) {
        if (fl == kFlExpand) return dispatch<MODE, kFlExpand>(L, prm, s, sms);
        if (fl == (kFlExpand | kFlGain)) return dispatch<MODE, kFlExpand | kFlGain>(L, prm, s, sms);
    }
    return HBL_ERR_INVALID_ARG;
}
}  // namespace k1

bool norm_quant_expand_rides_along(int64_t M, int K, int N, int num_sms) {
    if (M <= 0 || N <= 0 || N % 16 != 0 || K < 128 || (K & (K - 1)) != 0) return false;
    switch (ilog2((unsigned)K)) {
        case 7: return k1::expand_rides_along_l<7>(M, N, num_sms);
        case 8: return k1::expand_rides_along_l<8>(M, N, num_sms);
        case 9: return k1::expand_rides_along_l<9>(M, N, num_sms);
        case 10: return k1::expand_rides_along_l<10>(M, N, num_sms);
        case 11: return k1::expand_rides_along_l<11>(M, N, num_sms);
        case 12: return k1::expand_rides_along_l<12>(M, N, num_sms);
        case 13: return k1::expand_rides_along_l<13>(M, N, num_sms);
        case 14: return k1::expand_rides_along_l<14>(M, N, num_sms);
        case 15: return k1::expand_rides_along_l<15>(M, N, num_sms);
        default: return false;
    }
}

hbl_status launch_norm_fwht_quant(const uint16_t* X, const float* gain, int64_t M, int K,
                                  float norm_eps, float quant_eps, int mode, void* codes,
                                  float* scales, int32_t* rowsum, float* V, cudaStream_t stream,
                                  int num_sms, unsigned variant, const uint32_t* W_packed, int N,
                                  int8_t* W_s8) {
    const bool expand = W_packed != nullptr && N > 0;
    if (expand && ((mode != 6 && mode != 8) || W_s8 == nullptr || K % 128 != 0 || N % 16 != 0 ||
                   (variant & (HBL_NORM_NO_HADAMARD | HBL_NORM_LAYERNORM)) != 0))
        return HBL_ERR_INVALID_ARG;
    if (M == 0) return HBL_OK;
    k1::Params prm = {};
    if (expand) {
        prm.W = W_packed;
        prm.N = N;
        prm.wdst = reinterpret_cast<uint4*>(W_s8);
    }
    prm.X = X;
    prm.gain = gain;
    prm.M = M;
    prm.norm_eps = norm_eps;
    prm.quant_eps = quant_eps;
    prm.cK = (float)(1.0 / sqrt((double)K));
    prm.s7 = (float)sqrt(7.0);
    prm.thr16 = k1::thr16_for(K);
    prm.codes = static_cast<uint8_t*>(codes);
    prm.scales = scales;
    prm.rowsum = rowsum;
    prm.V = V;
    const int L = ilog2((unsigned)K);
    const int fl = (gain != nullptr ? k1::kFlGain : 0) |
                   ((variant & HBL_NORM_NO_HADAMARD) ? k1::kFlNoHadamard : 0) |
                   ((variant & HBL_NORM_LAYERNORM) ? k1::kFlLayerNorm : 0) |
                   (expand ? k1::kFlExpand : 0);
    switch (mode) {
        case 0: return k1::by_flags<0>(fl, L, prm, stream, num_sms);
        case 4: return k1::by_flags<4>(fl, L, prm, stream, num_sms);
        case 5: return k1::by_flags<5>(fl, L, prm, stream, num_sms);
        case 6: return k1::by_flags<6>(fl, L, prm, stream, num_sms);
        case 8: return k1::by_flags<8>(fl, L, prm, stream, num_sms);
        case 9: return k1::by_flags<9>(fl, L, prm, stream, num_sms);
        default: return HBL_ERR_INVALID_ARG;
    }
}

}  // namespace hbl
