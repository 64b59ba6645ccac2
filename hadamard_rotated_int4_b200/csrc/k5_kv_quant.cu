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
// Mapping: D/16 lanes per row, 16 values (two 16-byte loads) per lane, so a
// warp covers 32*16/D rows per step and a lane's 16 codes are 16*b contiguous
// bits; the per-step costs (the max over the row's lanes, the division, the
// scale) are shared by 16 values per lane.  For b = 3 lane pairs make one
// 12-byte group (one shuffle).  Memory-bound: 2*D bytes in, D*b/8 + 4 out per
// row; each warp keeps U steps of loads in flight.
#include <cuda_runtime.h>

#include <type_traits>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k5 {

constexpr int kThreads = 256;
constexpr int U = 2;     // row steps per warp with their loads in flight together
constexpr int VPL = 16;  // values per lane

template <int D, int B>
__global__ void __launch_bounds__(kThreads) kv_quant_kernel(const uint16_t* __restrict__ X,
                                                            int64_t rows, float eps,
                                                            uint8_t* __restrict__ codes,
                                                            float* __restrict__ scales) {
    constexpr int LPR = D / VPL;     // lanes per row
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
        uint4 raw[U][2];
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * RPW + sub;
            const uint4* src = reinterpret_cast<const uint4*>(X + row * D + li * VPL);
            raw[u][0] = row < rows ? src[0] : make_uint4(0, 0, 0, 0);
            raw[u][1] = row < rows ? src[1] : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < U; ++u) {
            const int64_t row = base + u * RPW + sub;
            float x[VPL];
            {
                const uint32_t w[8] = {raw[u][0].x, raw[u][0].y, raw[u][0].z, raw[u][0].w,
                                       raw[u][1].x, raw[u][1].y, raw[u][1].z, raw[u][1].w};
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float2 f = bf16x2_to_f2(w[i]);
                    x[2 * i] = f.x;
                    x[2 * i + 1] = f.y;
                }
            }
            float g = 0.f;
#pragma unroll
            for (int i = 0; i < VPL; ++i) g = fmaxf(g, fabsf(x[i]));
#pragma unroll
            for (int o = 1; o < LPR; o <<= 1) g = fmaxf(g, __shfl_xor_sync(0xffffffffu, g, o));
            const float den = __fadd_rn(g, eps);
            const float inv = den > 0.f ? __fdiv_rn(qp, den) : 0.f;
            // 16 codes of this lane, code i at bits [B*i, B*i + B) of a 16*B-bit
            // field (two 32-bit halves of 8 codes each).  No clamp is needed:
            // |x| <= gamma, so |x * inv| <= Qp * gamma / (gamma + eps) up to the
            // rounding of inv (well under half a unit), and rounding to the
            // nearest integer stays within [-Qp, Qp].
            using Half = typename std::conditional<(8 * B <= 32), uint32_t, uint64_t>::type;
            Half h[2] = {0, 0};
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int32_t b = __float_as_int(__fmaf_rn(x[i], inv, 12582912.0f));
                const uint32_t code = (uint32_t)(b - kMagicBits + (QP + 1));
                h[i / 8] |= (Half)code << (B * (i % 8));
            }
            const bool ok = row < rows;
            uint8_t* dst = codes + row * ROW_BYTES;
            if constexpr (B == 8) {  // 16 bytes per lane
                if (ok)
                    *reinterpret_cast<uint4*>(dst + li * 16) =
                        make_uint4((uint32_t)h[0], (uint32_t)((uint64_t)h[0] >> 32), (uint32_t)h[1],
                                   (uint32_t)((uint64_t)h[1] >> 32));
            } else if constexpr (B == 4) {  // 8 bytes per lane
                if (ok) *reinterpret_cast<uint2*>(dst + li * 8) = make_uint2(h[0], h[1]);
            } else if constexpr (B == 2) {  // 4 bytes per lane
                if (ok) *reinterpret_cast<uint32_t*>(dst + li * 4) = h[0] | (h[1] << 16);
            } else {  // B == 3: 48 bits per lane; a lane pair makes one 12-byte group
                const uint64_t mine = (uint64_t)h[0] | ((uint64_t)h[1] << 24);
                const uint64_t next = __shfl_down_sync(0xffffffffu, mine, 1);
                if (ok && (li & 1) == 0) {
                    uint32_t* d32 = reinterpret_cast<uint32_t*>(dst + (li >> 1) * 12);
                    d32[0] = (uint32_t)mine;
                    d32[1] = (uint32_t)(mine >> 32) | ((uint32_t)next << 16);
                    d32[2] = (uint32_t)(next >> 16);
                }
            }
            if (ok && li == 0) scales[row] = __fdiv_rn(g, qp);
        }
    }
}

template <int D, int B>
static hbl_status launch_one(const uint16_t* X, int64_t rows, float eps, uint8_t* codes,
                             float* scales, cudaStream_t stream, int sms) {
    constexpr int RPW = 32 / (D / VPL);
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
