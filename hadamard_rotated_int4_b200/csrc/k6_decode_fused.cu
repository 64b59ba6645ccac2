// k6_decode_fused.cu -- host entries of the decode kernels: the one-kernel
// forward and its GEMV half (the kernels are in k6_decode_fused.cuh,
// instantiated per K in k6_decode_l*.cu).
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k6 {
hbl_status launch_l12(const DecodeArgs& d, cudaStream_t s, int sms);
hbl_status launch_l13(const DecodeArgs& d, cudaStream_t s, int sms);
hbl_status launch_l14(const DecodeArgs& d, cudaStream_t s, int sms);
int smem_l12(int N, int MT, int sms);
int smem_l13(int N, int MT, int sms);
int smem_l14(int N, int MT, int sms);
hbl_status launch_gemv_l14(const GemvArgs& g, cudaStream_t s, int sms);
int gemv_smem_l14(int N, int MT, int sms);
}  // namespace k6

int decode_fused_rows(int N, int num_sms) {
    const int ctas = N < num_sms ? N : num_sms;
    return (N + ctas - 1) / ctas;
}

static int token_capacity(int M) { return M <= 1 ? 1 : (M <= 2 ? 2 : 4); }

bool decode_fused_supported(int M, int K, int N, int act_bits, unsigned variant, int num_sms) {
    // one K1 row group (K / 64 threads) per token within the CTA's 256 threads:
    // past that the rows would be quantised one after another and the
    // two-kernel forward is faster
    if (M < 1 || K < 4096 || M > 16384 / K || N < 1 || variant != 0 ||
        (act_bits != 4 && act_bits != 8))
        return false;
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
        return false;
    const int mt = token_capacity(M);
    int bytes = 0;
    switch (K) {
        case 4096: bytes = k6::smem_l12(N, mt, num_sms); break;
        case 8192: bytes = k6::smem_l13(N, mt, num_sms); break;
        case 16384: bytes = k6::smem_l14(N, mt, num_sms); break;
        default: return false;
    }
    return bytes <= optin;
}

static int optin_smem() {
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
            cudaSuccess)
        return 0;
    return optin;
}

// Used at K = 16384 only: at smaller K a lane's slice of a row is short, the
// shuffle reductions outweigh the dp4a work, and K1 + the row GEMV is faster
// (K = 8192, 4 tokens: 12.8 vs 10.4 us).
bool decode_gemv_supported(int M, int K, int N, int num_sms) {
    if (M < 1 || M > 8 || N < 1 || K != 16384) return false;
    return k6::gemv_smem_l14(N, M <= 4 ? token_capacity(M) : 8, num_sms) <= optin_smem();
}

hbl_status launch_decode_gemv(const GemvArgs& g, cudaStream_t stream, int num_sms) {
    if (g.M == 0) return HBL_OK;
    if (g.K != 16384) return HBL_ERR_SHAPE;
    return k6::launch_gemv_l14(g, stream, num_sms);
}

hbl_status launch_decode_fused(const DecodeArgs& d, cudaStream_t stream, int num_sms) {
    if (d.M == 0) return HBL_OK;
    switch (d.K) {
        case 4096: return k6::launch_l12(d, stream, num_sms);
        case 8192: return k6::launch_l13(d, stream, num_sms);
        case 16384: return k6::launch_l14(d, stream, num_sms);
        default: return HBL_ERR_SHAPE;
    }
}

}  // namespace hbl
