// k5_kv_quant.cu -- per-head absmax quantiser of Q, K, V states (after RoPE)
// to unsigned `bits`-bit integers, for low-bit attention and the KV cache.
//
// BitNet v2 write-up (0755model.com), section "实验结果" (tables 2 and 3): the
// QKV states are quantised after RoPE, per head, with absmax, directly to
// unsigned integers and without calibration data; a 3-bit KV cache is
// reported.  The quantiser is the INT8 absmax quantiser of the activations
// taken to b bits and offset into the unsigned range:
//   Qp = 2^(b-1) - 1;  gamma = max|x|;  inv = Qp / (gamma + eps)  (one division)
//   q = clip(rhe(x * inv), -Qp-1, Qp);  u = q + 2^(b-1);  scale = gamma / Qp
// (inv = 0 when gamma + eps == 0, so a zero row gives u = 2^(b-1), scale 0).
// Each code rounds the exact product x * inv once (an fma with 1.5 * 2^23).
//
// Layout: a row of D codes is D*b/8 bytes; each group of 32 codes is 4*b bytes
// and code j of a group sits at bits [b*j, b*j + b) of the group read as a
// little-endian integer.
//
// Mapping: D/8 lanes per row, 8 values (one 16-byte load) per lane, so a warp
// covers 32*8/D rows per step and a lane's 8 codes are 8*b contiguous bits;
// lanes combine them with one shuffle where a 32-bit word spans two lanes.
// Memory-bound: 2*D bytes in, D*b/8 + 4 out per row; each warp keeps U steps of
// loads in flight.
#include <cuda_runtime.h>

#include <type_traits>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k5 {

constexpr int kThreads = 256;
constexpr int U = 4;  // row steps per warp with their loads in flight together

template <int D, int B>
__global__ void __launch_bounds__(kThreads) kv_quant_kernel(const uint16_t* __restrict__ X,
                                                            int64_t rows, float eps,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
    constexpr int LPR = D / 8;       // lanes per row
    constexpr int RPW = 32 / LPR;    // rows per warp step
    constexpr int ROW_BYTES = D * B / 8;
    constexpr int QP = (1 << (B - 1)) - 1;
    constexpr int32_t kMagicBits = 0x4B400000;  // 1.5 * 2^23
    const int lane = threadIdx.x & 31;
    const int sub = lane / LPR, li = lane % LPR;
    const int64_t warp0 = ((int64_t)blockIdx.x * kThreads + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * kThreads) >> 5;
    const float qp = (float)QP;

    for (int64_t base = warp0 * (RPW * U); base < rows; base += nwarps * (RPW * U)) {
        uint4 raw[U];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * RPW + sub;
            raw[u] = row < rows ? *reinterpret_cast<const uint4*>(X + row * D + li * 8)
                                : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * RPW + sub;
            float x[8];
            {
                const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const float2 f = bf16x2_to_f2(w[i]);
                    x[2 * i] = f.x;
                    x[2 * i + 1] = f.y;
                }
            }
            float g = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) g = fmaxf(g, fabsf(x[i]));
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
            const float den = __fadd_rn(g, eps);
            const float inv = den > 0.f ? __fdiv_rn(qp, den) : 0.f;
            // 8 codes of this lane, code i at bits [B*i, B*i + B).  No clamp is
            // needed: |x| <= gamma, so |x * inv| <= Qp * gamma / (gamma + eps)
            // up to the rounding of inv (well under half a unit), and rounding
            // to the nearest integer stays within [-Qp, Qp].
            using Word = typename std::conditional<(8 * B <= 32), uint32_t, uint64_t>::type;
            Word bits = 0;
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const int32_t b = __float_as_int(__fmaf_rn(x[i], inv, 12582912.0f));
                const uint32_t code = (uint32_t)(b - kMagicBits + (QP + 1));
                bits |= (Word)code << (B * i);
            }
            const bool ok = row < rows;
            uint8_t* dst = codes + row * ROW_BYTES;
            if constexpr (B == 8) {
                if (ok)
                    *reinterpret_cast<uint2*>(dst + li * 8) =
                        make_uint2((uint32_t)bits, (uint32_t)((uint64_t)bits >> 32));
            } else if constexpr (B == 4) {
                if (ok) *reinterpret_cast<uint32_t*>(dst + li * 4) = (uint32_t)bits;
            } else if constexpr (B == 2) {  // 16 bits per lane: even lanes write pairs
                const uint32_t mine = (uint32_t)bits;
                const uint32_t next = __shfl_down_sync(0xffffffffu, mine, 1);
                if (ok && (li & 1) == 0)
                    *reinterpret_cast<uint32_t*>(dst + (li >> 1) * 4) = mine | (next << 16);
            } else {  // B == 3: 24 bits per lane; four lanes make one 12-byte group
                const uint32_t mine = (uint32_t)bits;
                const uint32_t next = __shfl_down_sync(0xffffffffu, mine, 1);
                const int k = li & 3;
                const uint32_t word = k == 0 ? (mine | (next << 24))
                                    : k == 1 ? ((mine >> 8) | (next << 16))
                                             : ((mine >> 16) | (next << 8));
                if (ok && k < 3)
                    *reinterpret_cast<uint32_t*>(dst + (li >> 2) * 12 + 4 * k) = word;
            }
            if (ok && li == 0) scales[row] = __fdiv_rn(g, qp);
        }
    }
}

template <int D, int B>
static hbl_status launch_one(const uint16_t* X, int64_t rows, float eps, uint8_t* codes,
                             float* scales, cudaStream_t stream, int sms) {
    constexpr int RPW = 32 / (D / 8);
    const int64_t per_cta = (int64_t)(kThreads / 32) * RPW * U;
    int64_t grid = (rows + per_cta - 1) / per_cta;
    const int64_t cap = (int64_t)sms * 8;
    if (grid > cap) grid = cap;
    kv_quant_kernel<D, B><<<(unsigned)grid, kThreads, 0, stream>>>(X, rows, eps, codes, scales);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

template <int D>
static hbl_status by_bits(int bits, const uint16_t* X, int64_t rows, float eps, uint8_t* codes,
                          float* scales, cudaStream_t s, int sms) {
    switch (bits) {
        case 2: return launch_one<D, 2>(X, rows, eps, codes, scales, s, sms);
        case 3: return launch_one<D, 3>(X, rows, eps, codes, scales, s, sms);
        case 4: return launch_one<D, 4>(X, rows, eps, codes, scales, s, sms);
        case 8: return launch_one<D, 8>(X, rows, eps, codes, scales, s, sms);
        default: return HBL_ERR_INVALID_ARG;
    }
}

}  // namespace k5

hbl_status launch_kv_quant(const uint16_t* X, int64_t rows, int D, int bits, float eps,
                           uint8_t* codes, float* scales, cudaStream_t stream, int num_sms) {
    if (rows == 0) return HBL_OK;
    switch (D) {
        case 32: return k5::by_bits<32>(bits, X, rows, eps, codes, scales, stream, num_sms);
        case 64: return k5::by_bits<64>(bits, X, rows, eps, codes, scales, stream, num_sms);
        case 128: return k5::by_bits<128>(bits, X, rows, eps, codes, scales, stream, num_sms);
        case 256: return k5::by_bits<256>(bits, X, rows, eps, codes, scales, stream, num_sms);
        default: return HBL_ERR_SHAPE;
    }
}

}  // namespace hbl
