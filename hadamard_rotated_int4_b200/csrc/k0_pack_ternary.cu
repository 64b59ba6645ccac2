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

// Pushes x, the perfect-tree sum of the 2^lvl elements that follow the cnt
// elements already pushed (cnt a multiple of 2^lvl), onto a binary-counter
// stack of partial sums: level l holds the sum of a 2^l-element block.
__device__ __forceinline__ void push_block(float (&stk)[40], int64_t& cnt, float x, int lvl) {
    int64_t c = cnt >> lvl;
    int l = lvl;
    while (c & 1) {
        x = __fadd_rn(stk[l], x);
        c >>= 1;
        ++l;
    }
    stk[l] = x;
    cnt += (int64_t)1 << lvl;
}

// Perfect pairwise tree of |W| over the 128 consecutive floats that lane l
// holds four of (l*4 .. l*4+3): in-lane pairs, then xor shuffles (lane bit b =
// block bit b).  Every lane ends with the sum.
__device__ __forceinline__ float warp_tree128(float4 q) {
    float s = __fadd_rn(__fadd_rn(fabsf(q.x), fabsf(q.y)), __fadd_rn(fabsf(q.z), fabsf(q.w)));
#pragma unroll
    for (int b = 1; b < 32; b <<= 1) s = __fadd_rn(s, __shfl_xor_sync(0xffffffffu, s, b));
    return s;
}

// One warp per row: perfect pairwise tree of |W| over the row (K = 2^L).
// K >= 1024: the warp reads the row in coalesced 1024-float blocks (eight
// 16-byte loads per lane in flight), reduces each 128-float sub-block as a
// perfect tree across the warp, the eight sub-blocks as a perfect tree, and
// pushes the block on a (warp-uniform) binary-counter stack.  K < 1024: lane
// l reduces [l*E, (l+1)*E) (E = K/32, or one element per lane for K < 32) in
// index order and lanes combine by xor shuffles.
__global__ void row_abs_sum_kernel(const float* __restrict__ W, int N, int K,
                                   float* __restrict__ rowsums) {
    const int lane = threadIdx.x & 31;
    const int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int nwarps = (gridDim.x * blockDim.x) >> 5;
    for (int n = warp; n < N; n += nwarps) {
        const float* row = W + (int64_t)n * K;
        float total = 0.f;
        if (K >= 1024) {
            float stk[40];
            int64_t cnt = 0;
            for (int e0 = 0; e0 < K; e0 += 1024) {
                const float4* s4 = reinterpret_cast<const float4*>(row + e0) + lane;
                float4 q[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) q[i] = __ldg(s4 + 32 * i);
                float t[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) t[i] = warp_tree128(q[i]);
#pragma unroll
                for (int w = 1; w < 8; w <<= 1)
#pragma unroll
                    for (int i = 0; i < 8; i += 2 * w) t[i] = __fadd_rn(t[i], t[i + w]);
                push_block(stk, cnt, t[0], 10);
            }
            total = stk[ilog2((unsigned)K)];
        } else {
            const int lanes = K < 32 ? K : 32;
            const int E = K / lanes;
            if (lane < lanes) {
                const float* src = row + (int64_t)lane * E;
                float stk[40];
                int64_t cnt = 0;
                for (int e = 0; e < E; ++e) push_block(stk, cnt, fabsf(src[e]), 0);
                total = stk[ilog2((unsigned)E)];
            }
            for (int b = 1; b < lanes; b <<= 1)
                total = __fadd_rn(total, __shfl_xor_sync(0xffffffffu, total, b));
        }
        if (lane == 0) rowsums[n] = total;
    }
}

// One block of kAlphaThreads: left-complete tree over the N row sums, then
// alpha.  The left-complete tree equals perfect trees over the blocks given by
// the binary digits of N (largest first), combined right to left.  Each block
// of 2^b sums is reduced by min(2^b, kAlphaThreads) threads, each summing a
// contiguous power-of-two run in index order, then by adjacent pairs in
// shared memory.
constexpr int kAlphaThreads = 1024;

__global__ void __launch_bounds__(kAlphaThreads) alpha_kernel(const float* __restrict__ rowsums,
                                                              int N, int64_t nk,
                                                              float* __restrict__ alpha) {
    __shared__ float part[kAlphaThreads];
    __shared__ float blk[32];
    const int t = threadIdx.x;
    int64_t off = 0;
    int nb = 0;
    for (int b = 30; b >= 0; --b) {
        if (!((N >> b) & 1)) continue;
        const int P = 1 << b;
        const int T = P < kAlphaThreads ? P : kAlphaThreads;
        const int E = P / T;
        if (t < T) {
            const float* src = rowsums + off + (int64_t)t * E;
            float stk[40];
            int64_t cnt = 0;
            for (int e = 0; e < E; ++e) push_block(stk, cnt, src[e], 0);
            part[t] = stk[ilog2((unsigned)E)];
        }
        __syncthreads();
        for (int w = 1; w < T; w <<= 1) {
            if (t < T && (t & (2 * w - 1)) == 0) part[t] = __fadd_rn(part[t], part[t + w]);
            __syncthreads();
        }
        if (t == 0) blk[nb] = part[0];
        ++nb;
        off += P;
        __syncthreads();
    }
    if (t == 0) {
        float acc = nb > 0 ? blk[nb - 1] : 0.f;
        for (int i = nb - 2; i >= 0; --i) acc = __fadd_rn(blk[i], acc);
        *alpha = __fdiv_rn(acc, __ll2float_rn((long long)nk));
    }
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
    k0::alpha_kernel<<<1, k0::kAlphaThreads, 0, stream>>>(rowsums, N, (int64_t)N * K, alpha);
    const int64_t nwords = (int64_t)N * (K / 16);
    int64_t pb = (nwords + 255) / 256;
    if (pb > (int64_t)num_sms * 16) pb = (int64_t)num_sms * 16;
    k0::pack_kernel<<<(unsigned)pb, 256, 0, stream>>>(W, nwords, eps, alpha, W_packed);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace hbl
