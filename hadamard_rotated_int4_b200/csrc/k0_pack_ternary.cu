// k0_pack_ternary.cu -- per-tensor absmean ternarisation of latent weights and
// 2-bit packing, for sm_100a (offline, once per weight).
//
// BitNet v2 write-up (0755model.com), section "H-BitLinear": weights are
// ternarised to {-1, 0, 1} with a per-tensor absmean scale.  Formula used (the
// page shows it as an image):
//   alpha = S / (float)(N*K),   S = left-complete pairwise tree of |W| over the
//           row-major flat index (for K a power of two: the perfect tree of
//           each row, then the left-complete tree over the N row sums);
//   t = clip(round_half_even(W / (alpha + eps)), -1, 1).
// Packing ("[论文品鉴] 1-bit LLM", section "掩码存储": several ternary values
// packed into one integer): 16 weights per uint32, local weight j at bits
// [8*(j%4) + 2*(j/4), +2) as t + 1.  With that placement a shift by 2m and a
// mask 0x03030303 yields the codes of weights 4m..4m+3 as four bytes.
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k0 {

// One warp per row: perfect pairwise tree of |W| over the row (K = 2^L).
// Lane l owns the contiguous chunk [l*E, (l+1)*E) (E = K/32, or 1 element per
// lane for K < 32); chunks are reduced in index order with a binary-counter
// stack, then lanes combine by xor shuffles (lane bit b = chunk bit b).
__global__ void row_abs_sum_kernel(const float* __restrict__ W, int N, int K,
                                   float* __restrict__ rowsums) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    const int lanes = K < 32 ? K : 32;
    const int E = K / lanes;
    for (int n = warp; n < N; n += nwarps) {
        float total = 0.f;
        if (lane < lanes) {
            const float* src = W + (int64_t)n * K + (int64_t)lane * E;
            float stk[16];
            int cnt = 0;  // elements consumed; stack level l holds a 2^l partial
            for (int e = 0; e < E; ++e) {
                float x = fabsf(src[e]);
                int c = cnt;
                int l = 0;
                while (c & 1) {
                    x = __fadd_rn(stk[l], x);
                    c >>= 1;
                    ++l;
                }
                stk[l] = x;
                ++cnt;
            }
            total = stk[ilog2((unsigned)E)];
        }
        for (int b = 1; b < lanes; b <<= 1) {
            float o = __shfl_xor_sync(0xffffffffu, total, b);
            total = __fadd_rn(total, o);
        }
        if (lane == 0) rowsums[n] = total;
    }
}

// Single thread: left-complete tree over the N row sums, then alpha.
// The left-complete tree equals perfect trees over the blocks given by the
// binary digits of N (largest first), combined right to left.
__global__ void alpha_kernel(const float* __restrict__ rowsums, int N, int64_t nk,
                             float* __restrict__ alpha) {
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    float stk[32];
    int64_t cnt = 0;
    for (int n = 0; n < N; ++n) {
        float x = rowsums[n];
        int64_t c = cnt;
        int l = 0;
        while (c & 1) {
            x = __fadd_rn(stk[l], x);
            c >>= 1;
            ++l;
        }
        stk[l] = x;
        ++cnt;
    }
    float acc = 0.f;
    bool have = false;
    for (int l = 0; l < 32; ++l)
        if ((cnt >> l) & 1) {
            acc = have ? __fadd_rn(stk[l], acc) : stk[l];
            have = true;
        }
    *alpha = __fdiv_rn(acc, __ll2float_rn((long long)nk));
}

// One thread per packed word (16 weights).
__global__ void pack_kernel(const float* __restrict__ W, int64_t nwords, float eps,
                            const float* __restrict__ alpha, uint32_t* __restrict__ out) {
    const float d = __fadd_rn(*alpha, eps);
    for (int64_t wi = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; wi < nwords;
         wi += (int64_t)gridDim.x * blockDim.x) {
        const float4* src = reinterpret_cast<const float4*>(W + wi * 16);
        float v[16];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            float4 f = src[q];
            v[4 * q] = f.x;
            v[4 * q + 1] = f.y;
            v[4 * q + 2] = f.z;
            v[4 * q + 3] = f.w;
        }
        uint32_t word = 0;
#pragma unroll
        for (int jj = 0; jj < 16; ++jj) {
            float tq = rintf(__fdiv_rn(v[jj], d));
            tq = fminf(fmaxf(tq, -1.0f), 1.0f);
            uint32_t code = (uint32_t)((int)tq + 1);
            word |= code << (8 * (jj & 3) + 2 * (jj >> 2));
        }
        out[wi] = word;
    }
}

}  // namespace k0

size_t pack_ternary_workspace(int N, int /*K*/) {
    return ((size_t)N * sizeof(float) + 255) & ~(size_t)255;
}

hbl_status launch_pack_ternary(const float* W, int N, int K, float eps, uint32_t* W_packed,
                               float* alpha, void* ws, cudaStream_t stream, int num_sms) {
    float* rowsums = static_cast<float*>(ws);
    int warps_needed = N;
    int blocks = (warps_needed + 7) / 8;
    if (blocks > num_sms * 8) blocks = num_sms * 8;
    k0::row_abs_sum_kernel<<<blocks, 256, 0, stream>>>(W, N, K, rowsums);
    k0::alpha_kernel<<<1, 32, 0, stream>>>(rowsums, N, (int64_t)N * K, alpha);
    const int64_t nwords = (int64_t)N * (K / 16);
    int64_t pb = (nwords + 255) / 256;
    if (pb > (int64_t)num_sms * 16) pb = (int64_t)num_sms * 16;
    k0::pack_kernel<<<(unsigned)pb, 256, 0, stream>>>(W, nwords, eps, alpha, W_packed);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace hbl
