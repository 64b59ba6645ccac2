// k3b_gemv_rows.cu -- ternary x int8/int4 GEMV for decode batches (M <= 8
// tokens, K >= 2048) on CUDA cores, one weight row per warp over the whole K,
// with the dequantisation epilogue in the same kernel.
//
// acc[m][n] = sum_k q[m][k] * t[n][k] = sum_k q*c - rowsum[m], c = t + 1 the
// stored 2-bit code (BitNet v2 write-up, 0755model.com, section "H-BitLinear":
// the ternary matmul of the quantised activations, then the rescale by the
// weight and activation scales).  Y = bf16_rne((float)acc * (alpha * s[m])).
//
// Decode is bound by reading the packed weights once (N*K/4 bytes).  Each warp
// owns one weight row and loads all of it into registers at once (lane l takes
// the 16-byte chunks l, l + 32, ...: K/2048 chunks, every load a coalesced
// 512-byte warp access), so a warp has its whole row in flight and no load
// waits on another.  Launched as a programmatic dependent of the activation
// kernel (PRE), the weight loads are issued before the dependency wait and
// overlap that kernel; the activations are then staged in shared memory as
// int8 in a chunk-transposed layout (16-byte piece p of chunk c of token m at
// ((m * 4 + p) * (K / 64) + c) * 16), so the lanes of a warp read consecutive
// 16-byte words.  The int32 sums are exact; lanes reduce them by shuffles and
// the warp writes its row's outputs directly (no split-K partials, no second
// kernel, no workspace).
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k3b {

constexpr int kWarps = 8;

__device__ __forceinline__ int dp4a_su(int a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

// 8 signed nibbles (element 2i low) -> 8 int8 in two words (natural order).
__device__ __forceinline__ uint2 widen_nibbles(uint32_t w) {
    uint32_t lo = ((w & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    uint32_t hi = (((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    lo ^= 0x80808080u;
    hi ^= 0x80808080u;
    return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

// L = log2 K (>= 11), MT = token capacity (1, 2, 4, 8), PRE = weights loaded
// before the programmatic-dependency wait.  Each warp owns RPW consecutive
// weight rows (RPW = 2 for two or more tokens: every activation word read from
// shared memory then feeds two rows, halving that traffic).
template <int L, int MT, bool PRE>
__global__ void __launch_bounds__(kWarps * 32)
    gemv_rows_kernel(const uint8_t* __restrict__ codes, int act_bits, int M,
                     const uint32_t* __restrict__ Wp, int N, const int32_t* __restrict__ rowsum,
                     const float* __restrict__ scales, const float* __restrict__ alpha,
                     uint16_t* __restrict__ Y, int32_t* __restrict__ acc_out) {
    constexpr int K = 1 << L;
    constexpr int CH = K / 2048;  // 16-byte weight chunks per lane per row
    constexpr int NC = K / 64;    // 16-byte chunks per weight row
    constexpr int RPW = MT >= 2 ? 2 : 1;
    extern __shared__ __align__(16) uint8_t sact[];  // [MT][4][NC] x 16 B
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int nb = (blockIdx.x * kWarps + warp) * RPW;  // first row of this warp

    uint4 w[RPW][CH];
    auto load_w = [&]() {
#pragma unroll
        for (int r = 0; r < RPW; ++r) {
            const int n = min(nb + r, N - 1);  // rows past N read a valid row, never stored
            const uint4* wrow = reinterpret_cast<const uint4*>(Wp + (int64_t)n * (K / 16));
#pragma unroll
            for (int i = 0; i < CH; ++i) w[r][i] = __ldg(wrow + lane + 32 * i);
        }
    };
    if constexpr (PRE) load_w();
    pdl_wait();
    if constexpr (!PRE) load_w();

    // stage activations: item = (m, piece p, chunk c) with c fastest, so the
    // shared-memory stores of a warp are consecutive 16-byte words; the
    // 16-weight piece g = 4c + p of token m comes from the codes in L2.
    for (int it = tid; it < MT * 4 * NC; it += kWarps * 32) {
        const int c = it % NC, p = (it / NC) & 3, m = it / (4 * NC);
        const int g = 4 * c + p;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M) {
            if (act_bits == 8) {
                v = *reinterpret_cast<const uint4*>(codes + (int64_t)m * K + g * 16);
            } else {
                const uint2 pk =
                    *reinterpret_cast<const uint2*>(codes + (int64_t)m * (K / 2) + g * 8);
                const uint2 a = widen_nibbles(pk.x), b = widen_nibbles(pk.y);
                v = make_uint4(a.x, a.y, b.x, b.y);
            }
        }
        *reinterpret_cast<uint4*>(sact + ((size_t)(m * 4 + p) * NC + c) * 16) = v;
    }
    __syncthreads();

    int acc[RPW][MT];
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;
#pragma unroll
    for (int i = 0; i < CH; ++i) {
        const int c = lane + 32 * i;
#pragma unroll
        for (int m = 0; m < MT; ++m) {
#pragma unroll
            for (int p = 0; p < 4; ++p) {
                const uint4 a = *reinterpret_cast<const uint4*>(
                    sact + ((size_t)(m * 4 + p) * NC + c) * 16);
#pragma unroll
                for (int r = 0; r < RPW; ++r) {
                    const uint32_t wp = p == 0 ? w[r][i].x
                                      : p == 1 ? w[r][i].y
                                      : p == 2 ? w[r][i].z
                                               : w[r][i].w;
                    int s = acc[r][m];
                    s = dp4a_su((int)a.x, wp & 0x03030303u, s);
                    s = dp4a_su((int)a.y, (wp >> 2) & 0x03030303u, s);
                    s = dp4a_su((int)a.z, (wp >> 4) & 0x03030303u, s);
                    s = dp4a_su((int)a.w, (wp >> 6) & 0x03030303u, s);
                    acc[r][m] = s;
                }
            }
        }
    }
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m)
#pragma unroll
            for (int b = 16; b >= 1; b >>= 1)
                acc[r][m] += __shfl_xor_sync(0xffffffffu, acc[r][m], b);

    const float a = *alpha;
#pragma unroll
    for (int r = 0; r < RPW; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const int n = nb + r;
            if (lane == r * MT + m && m < M && n < N) {
                const int s = acc[r][m] - rowsum[m];
                if (acc_out != nullptr) acc_out[(int64_t)m * N + n] = s;
                const float y = __fmul_rn((float)s, __fmul_rn(a, scales[m]));
                Y[(int64_t)m * N + n] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
            }
        }
}

template <int L, int MT>
static hbl_status launch_mt(const GemmArgs& a, bool pre, cudaStream_t stream) {
    constexpr int K = 1 << L;
    constexpr int RPW = MT >= 2 ? 2 : 1;
    const size_t smem = (size_t)MT * K;
    const dim3 grid((unsigned)((a.N + kWarps * RPW - 1) / (kWarps * RPW))), block(kWarps * 32);
    const uint8_t* codes = static_cast<const uint8_t*>(a.codes);
    const int M = (int)a.M;
    if (pre) {
        auto kern = gemv_rows_kernel<L, MT, true>;
        if (smem > 48 * 1024 && !smem_attr_once(reinterpret_cast<const void*>(kern), (int)smem))
            return HBL_ERR_CUDA;
        return launch_pdl(kern, grid, block, smem, stream, codes, a.act_bits, M, a.W_packed, a.N,
                          a.rowsum, a.scales, a.alpha, a.Y, a.acc_out);
    }
    auto kern = gemv_rows_kernel<L, MT, false>;
    if (smem > 48 * 1024 && !smem_attr_once(reinterpret_cast<const void*>(kern), (int)smem))
        return HBL_ERR_CUDA;
    kern<<<grid, block, smem, stream>>>(codes, a.act_bits, M, a.W_packed, a.N, a.rowsum, a.scales,
                                        a.alpha, a.Y, a.acc_out);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

template <int L>
static hbl_status launch_l(const GemmArgs& a, bool pre, cudaStream_t stream) {
    const int M = (int)a.M;
    if (M <= 1) return launch_mt<L, 1>(a, pre, stream);
    if (M <= 2) return launch_mt<L, 2>(a, pre, stream);
    if (M <= 4) return launch_mt<L, 4>(a, pre, stream);
    if constexpr (L <= 14) return launch_mt<L, 8>(a, pre, stream);  // 8 x K bytes of smem
    return HBL_ERR_SHAPE;
}

}  // namespace k3b

// Tokens one launch of the row GEMV takes at this K: the CTA stages M x K int8
// activations in shared memory; up to 64 KB keeps three or more CTAs (24 warps
// of weight loads in flight) per SM.  Larger token counts go to the split-K GEMV.
int gemv_rows_max_m(int K) { return K >= 16384 ? (K >= 32768 ? 2 : 4) : 8; }

bool gemv_rows_supported(int K) { return K >= 2048 && K <= 32768; }

hbl_status launch_gemv_rows(const GemmArgs& a, bool pdl_after_producer, cudaStream_t stream) {
    if (a.M == 0) return HBL_OK;
    if (a.M > gemv_rows_max_m(a.K)) return HBL_ERR_SHAPE;
    switch (ilog2((unsigned)a.K)) {
        case 11: return k3b::launch_l<11>(a, pdl_after_producer, stream);
        case 12: return k3b::launch_l<12>(a, pdl_after_producer, stream);
        case 13: return k3b::launch_l<13>(a, pdl_after_producer, stream);
        case 14: return k3b::launch_l<14>(a, pdl_after_producer, stream);
        case 15: return k3b::launch_l<15>(a, pdl_after_producer, stream);
        default: return HBL_ERR_SHAPE;
    }
}

}  // namespace hbl
