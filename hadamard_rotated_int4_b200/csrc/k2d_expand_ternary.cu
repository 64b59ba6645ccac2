// k2d_expand_ternary.cu -- packed 2-bit ternary weights expanded to one signed
// byte per weight, the operand layout of the TMA-fed tensor-core GEMM
// (tcgen05 has no integer MMA narrower than 8 bits).  Memory-bound: N*K/4
// bytes read, N*K written.  The per-tensor absmean ternary weights and their
// packing several to an integer follow the BitNet v2 write-up (0755model.com,
// section "H-BitLinear") and the "[论文品鉴] 1-bit LLM" post (section "掩码存储").
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k2d {

// Packed 2-bit codes (16 per word, expand_ternary_word) -> one signed byte t
// per weight, row-major [N x K].  Consecutive threads take consecutive words,
// so every warp load is 128 contiguous bytes and every warp store 512; each
// thread has four words in flight per step.  (Where its token rows carry it,
// the large-batch forward widens the weights inside K1 instead.)
__global__ void expand_kernel(const uint32_t* __restrict__ Wp, int64_t words,
                              uint4* __restrict__ out) {
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t base = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; base < words;
         base += 4 * stride) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = base + j * stride;
            w[j] = i < words ? Wp[i] : 0u;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int64_t i = base + j * stride;
            if (i < words) out[i] = expand_ternary_word(w[j]);
        }
    }
}

}  // namespace k2d

hbl_status launch_expand_ternary(const uint32_t* W_packed, int N, int K, int8_t* W_s8,
                                 cudaStream_t stream, int num_sms) {
    const int64_t words = (int64_t)N * (K / 16);
    if (words == 0) return HBL_OK;
    int64_t blocks = (words + 255) / 256;
    if (blocks > (int64_t)num_sms * 8) blocks = (int64_t)num_sms * 8;
    if (blocks < 1) blocks = 1;
    k2d::expand_kernel<<<(unsigned)blocks, 256, 0, stream>>>(W_packed, words,
                                                             reinterpret_cast<uint4*>(W_s8));
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace hbl
