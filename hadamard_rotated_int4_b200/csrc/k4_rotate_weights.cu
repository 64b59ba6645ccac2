// k4_rotate_weights.cu -- offline rotation of latent weights into the
// Hadamard basis:  W_rot[n] = ((W[n] * s) . H_K) * c_K  for every row n.
//
// The BitNet v2 write-up (0755model.com) ablates the rotation applied to
// weights and activations against activations only (table 5), and describes
// QuaRot's randomised Hadamard transform H . diag(s); the sign vector s (+-1,
// or all ones) is an input.  Rotated weights pair with activations whose
// per-channel gain carries the same signs: (x D H c) . (w D H c) = x . w.
//
// The butterflies run in the order of the activation transform (stages
// h = 1, 2, ..., K/2, (a, b) -> (a + b, a - b)), then one multiply by
// c_K = fp32(1/sqrt(K)), so the result is bit-identical to a scalar evaluation
// in that order.  Weights are processed once, offline; the kernel is HBM-bound
// (one read and one write of 4*K bytes per row).
//
// One CTA per row at a time (grid-stride over rows).  The row is loaded with
// coalesced 16-byte loads into shared memory padded by one word per 32 (the
// element at index i lives at i + i/32), then transformed in passes of up to
// five stages: a thread gathers the 2^c elements of one butterfly group (index
// bits [s, s + c) varying), runs the c stages in registers and scatters them
// back.  For s = 0 the group is 32 contiguous elements, which the padding
// spreads over all 32 banks; for s >= 5 consecutive threads touch consecutive
// words.  The last pass multiplies by c_K and stores to global memory, where
// consecutive threads again write consecutive words.
#include <cuda_runtime.h>
#include <math.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k4 {

constexpr int kThreads = 256;

__device__ __forceinline__ int pad(int i) { return i + (i >> 5); }

template <int L>
__global__ void __launch_bounds__(kThreads) rotate_kernel(const float* W, const float* signs,
                                                          int64_t N, float* out, float cK) {
    constexpr int K = 1 << L;
    extern __shared__ __align__(16) float row[];  // K + K/32 floats (padded)
    const int tid = threadIdx.x;
    for (int64_t n = blockIdx.x; n < N; n += gridDim.x) {
        const float* src = W + n * K;
        float* dst = out + n * K;
        // coalesced load (times the signs) into the padded row; with signs,
        // kLoadBatch 16-byte loads per thread are issued before any is used
        // (the signs' loads otherwise serialise the row's; without signs the
        // one-at-a-time loop measured faster: 126 against 131 us on W_down)
        constexpr int kChunks = K / 4;
        constexpr int kLoadBatch = 8;
        if (signs == nullptr) {
            for (int c = tid; c < kChunks; c += kThreads) {
                const float4 v = *reinterpret_cast<const float4*>(src + 4 * c);
                const int i = 4 * c;  // four consecutive words never straddle a pad
                row[pad(i)] = v.x;
                row[pad(i) + 1] = v.y;
                row[pad(i) + 2] = v.z;
                row[pad(i) + 3] = v.w;
            }
        } else {
            for (int c0 = 0; c0 < kChunks; c0 += kThreads * kLoadBatch) {
                float4 v[kLoadBatch];
#pragma unroll
                for (int b = 0; b < kLoadBatch; ++b) {
                    const int c = c0 + b * kThreads + tid;
                    if (c < kChunks) v[b] = *reinterpret_cast<const float4*>(src + 4 * c);
                }
#pragma unroll
                for (int b = 0; b < kLoadBatch; ++b) {
                    const int c = c0 + b * kThreads + tid;
                    if (c < kChunks) {
                        float4 x = v[b];
                        const float4 sg = *reinterpret_cast<const float4*>(signs + 4 * c);
                        x.x = __fmul_rn(x.x, sg.x);
                        x.y = __fmul_rn(x.y, sg.y);
                        x.z = __fmul_rn(x.z, sg.z);
                        x.w = __fmul_rn(x.w, sg.w);
                        const int i = 4 * c;  // four consecutive words never straddle a pad
                        row[pad(i)] = x.x;
                        row[pad(i) + 1] = x.y;
                        row[pad(i) + 2] = x.z;
                        row[pad(i) + 3] = x.w;
                    }
                }
            }
        }
        __syncthreads();
        static_for<0, (L + 4) / 5>([&](auto pp) {
            constexpr int P = decltype(pp)::value;
            constexpr int s = 5 * P;                     // first stage of this pass
            constexpr int c = (L - s) < 5 ? (L - s) : 5;  // stages in this pass
            constexpr int G = 1 << c;
            constexpr bool kLast = (s + c == L);
            for (int g = tid; g < K / G; g += kThreads) {
                const int low = g & ((1 << s) - 1), high = g >> s;
                const int base = low | (high << (s + c));
                float v[G];
#pragma unroll
                for (int j = 0; j < G; ++j) v[j] = row[pad(base | (j << s))];
#pragma unroll
                for (int t = 0; t < c; ++t) {
                    const int h = 1 << t;
#pragma unroll
                    for (int j = 0; j < G; ++j)
                        if ((j & h) == 0) {
                            const float a = v[j], b = v[j | h];
                            v[j] = __fadd_rn(a, b);
                            v[j | h] = __fsub_rn(a, b);
                        }
                }
#pragma unroll
                for (int j = 0; j < G; ++j) {
                    if constexpr (kLast)
                        dst[base | (j << s)] = __fmul_rn(v[j], cK);
                    else
                        row[pad(base | (j << s))] = v[j];
                }
            }
            __syncthreads();
        });
    }
}

template <int L>
static hbl_status launch_one(const float* W, const float* signs, int64_t N, float* out,
                             cudaStream_t stream, int sms) {
    constexpr int K = 1 << L;
    const int smem = (K + K / 32) * 4;
    auto kern = rotate_kernel<L>;
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), smem)) return HBL_ERR_CUDA;
    int per_sm = 227 * 1024 / (smem + 1024);
    if (per_sm > 8) per_sm = 8;
    if (per_sm < 1) per_sm = 1;
    int64_t grid = (int64_t)sms * per_sm;
    if (grid > N) grid = N;
    kern<<<(unsigned)grid, kThreads, smem, stream>>>(W, signs, N, out,
                                                      (float)(1.0 / sqrt((double)K)));
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace k4

hbl_status launch_rotate_weights(const float* W, const float* signs, int N, int K, float* W_rot,
                                 cudaStream_t stream, int num_sms) {
    if (N == 0) return HBL_OK;
    switch (ilog2((unsigned)K)) {
        case 4: return k4::launch_one<4>(W, signs, N, W_rot, stream, num_sms);
        case 5: return k4::launch_one<5>(W, signs, N, W_rot, stream, num_sms);
        case 6: return k4::launch_one<6>(W, signs, N, W_rot, stream, num_sms);
        case 7: return k4::launch_one<7>(W, signs, N, W_rot, stream, num_sms);
        case 8: return k4::launch_one<8>(W, signs, N, W_rot, stream, num_sms);
        case 9: return k4::launch_one<9>(W, signs, N, W_rot, stream, num_sms);
        case 10: return k4::launch_one<10>(W, signs, N, W_rot, stream, num_sms);
        case 11: return k4::launch_one<11>(W, signs, N, W_rot, stream, num_sms);
        case 12: return k4::launch_one<12>(W, signs, N, W_rot, stream, num_sms);
        case 13: return k4::launch_one<13>(W, signs, N, W_rot, stream, num_sms);
        case 14: return k4::launch_one<14>(W, signs, N, W_rot, stream, num_sms);
        case 15: return k4::launch_one<15>(W, signs, N, W_rot, stream, num_sms);
        default: return HBL_ERR_SHAPE;
    }
}

}  // namespace hbl
