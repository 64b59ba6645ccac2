// k6_decode_fused.cuh -- the whole H-BitLinear forward of a decode batch
// (M <= 16384 / K tokens: 4 at K = 4096, 2 at 8192, 1 at 16384) in one
// kernel, for sm_100a.
//
// What it computes (BitNet v2 write-up, 0755model.com, sections
// "BitNet v2：原生4位激活" and "H-BitLinear"): the codes q[m][k] and scales
// s[m] of RMSNorm + Walsh-Hadamard transform + per-token INT4 / INT8
// quantisation (K1's row loop, the same fp32 operations in the same order),
// then Y[m][n] = bf16((sum_k q[m][k] * t[n][k]) * (alpha * s[m])) over the
// 2-bit ternary weights: the two-kernel forward's values, bit for bit.
//
// One CTA of 256 threads per SM; CTA b owns weight rows [b R, b R + R):
//  1. one thread hints the M token rows into L2 and, once the first row has
//     arrived, starts bulk copies of the CTA's packed weight rows (R K / 4
//     bytes) into shared memory, completing on an mbarrier, so the weights
//     stream from HBM while
//  2. the CTA quantises the M token rows itself with K1's kernel (the same
//     template, extended; every CTA
//     repeats this small amount of work instead of waiting for another
//     kernel), writing one code byte per element into shared memory.  Latency
//     sets the shape: 64 values per thread (K / 64 threads per row, two
//     shared-memory exchanges), one row group per token;
//  3. a warp covers KSEG = 512 * WPL elements of a weight row, WPL = the
//     larger of 8 / M' (M' = token capacity) and K / 4096 packed words per
//     lane: each lane keeps the codes of its WPL words per token in registers
//     and, for each row of the warp's row group, reads those words once from
//     shared memory.  The four 2-bit fields g of a packed byte
//     are masked in place (value c * 4^g, c = t + 1 in {0, 1, 2}) and summed by
//     dp4a into four accumulators that exact shifts bring back to one sum of
//     q * c, reduced over the lanes by xor shuffles;
//  4. the K / KSEG warps sharing a row add their partial sums through shared
//     memory and the epilogue writes bf16((sum - rowsum) * (alpha * s)), as
//     sum_k q * t = sum_k q * c - sum_k q.
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"
#include "k1_impl.cuh"

namespace hbl {
namespace k6 {

constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint32_t kCopyChunk = 32768;  // bytes per bulk copy

__host__ __device__ constexpr int up128(int x) { return (x + 127) & ~127; }

// Launch shape for K = 2^L and token capacity MT.  Q: the quantiser runs in
// the kernel (GPC K1 row groups of T threads, 64 values each); otherwise the
// codes come from global memory.  The GEMV phase's warps cover KSEG elements
// of a row, KSPLIT warps per row, RG row groups.
template <int L, int MT, bool Q = true>
struct Shape {
    static constexpr int NT = 256;
    static constexpr int NW = NT / 32;
    static constexpr int RLOG = 6;
    static constexpr int T = 1 << (L - RLOG);
    static constexpr int GPC = MT < NT / T ? MT : NT / T;
    using C = k1::Cfg<L, RLOG>;
    // packed words per lane per row: 8 / MT (32 code registers), at least
    // enough for NW warps to cover a row (then MT * 4 * WPL code registers)
    static constexpr int WPL = (8 / MT) > ((1 << L) / (512 * NW)) ? (8 / MT)
                                                                  : ((1 << L) / (512 * NW));
    static_assert(MT * 4 * WPL <= 128, "code registers");
    static constexpr int KSEG = 512 * WPL;
    static constexpr int KSPLIT = (1 << L) / KSEG;
    static constexpr int RG = NW / KSPLIT;
    // shared memory: [K1 row buffers, codes [MT][K]] (Q only), scales [4] +
    // rowsum [4], mbarrier + flag, partial sums [rows][KSPLIT][MT], packed
    // weight rows
    static constexpr int kCodes = Q ? up128(GPC * (C::kBufBytes + k1::kRedFloats * 4)) : 0;
    static constexpr int kScales = kCodes + (Q ? MT * (1 << L) : 0);
    static constexpr int kRowsum = kScales + 16;
    static constexpr int kBar = kScales + 32;
    static constexpr int kPart = kBar + 16;
    __host__ __device__ static constexpr int weights(int rows) {
        return up128(kPart + rows * KSPLIT * MT * 4);
    }
    __host__ __device__ static constexpr int total(int rows) {
        return weights(rows) + rows * ((1 << L) / 4);
    }
    static_assert(!Q || (C::T == T && C::kRowsPerGroup == 1 && GPC * T <= NT), "K1 grouping");
    static_assert(KSPLIT >= 1 && KSPLIT <= NW && NW % KSPLIT == 0, "GEMV split");
    static_assert(WPL == 2 || WPL == 4 || WPL == 8, "lane words");
};

__device__ __forceinline__ int dp4a_su(uint32_t a, uint32_t b, int c) {
    int d;
    asm("dp4a.s32.u32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes)
                 : "memory");
}
// 1-D bulk copy global -> shared (16-byte aligned, size a multiple of 16),
// completing `bytes` of transaction count on mbar.
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes,
                                          uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
            dst),
        "l"(__cvta_generic_to_global(src)), "r"(bytes), "r"(mbar)
        : "memory");
}

__device__ __forceinline__ uint8_t* dyn_smem() {
    extern __shared__ __align__(128) uint8_t dyn[];
    return dyn;
}

// CTA blockIdx.x's weight rows [n0, n0 + rows): at most p.rows, fewer in the last CTA.
__device__ __forceinline__ int cta_rows(const k1::Params& p) {
    return min(p.rows, p.N - (int)blockIdx.x * p.rows);  // >= 1 by the grid size
}

// Thread 0: the mbarrier the weights complete on.
template <class S>
__device__ __forceinline__ void init_weight_barrier(uint8_t* sm) {
    mbar_init_count(smem_addr(sm + S::kBar), 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// Thread 0: bulk copies of the CTA's packed weight rows into shared memory.
template <class S, int L>
__device__ __forceinline__ void issue_weights(const k1::Params& p, uint8_t* sm) {
    constexpr int K = 1 << L;
    const uint32_t bar = smem_addr(sm + S::kBar);
    const uint32_t bytes = (uint32_t)cta_rows(p) * (K / 4);
    mbar_expect_tx(bar, bytes);
    const uint8_t* src =
        reinterpret_cast<const uint8_t*>(p.W + (int64_t)blockIdx.x * p.rows * (K / 16));
    const uint32_t dst = smem_addr(sm + S::weights(p.rows));
    for (uint32_t off = 0; off < bytes; off += kCopyChunk)
        bulk_load(dst + off, src + off, min(kCopyChunk, bytes - off), bar);
}

// The GEMV over the CTA's weight rows (in shared memory once the mbarrier
// completes) and the dequantising epilogue.  codes: one byte per code,
// row-major [M][K] (shared or global memory); sc / rs: scales and row sums.
template <class S, int L, int MT>
__device__ __forceinline__ void gemv_phase(const k1::Params& p, uint8_t* sm,
                                           const uint8_t* codes, const float* sc,
                                           const int32_t* rs) {
    constexpr int K = 1 << L;
    constexpr int NT = S::NT, WPL = S::WPL, KSEG = S::KSEG, KSPLIT = S::KSPLIT, RG = S::RG;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int n0 = blockIdx.x * p.rows;
    const int rows = cta_rows(p);
    const int M = (int)p.M;
    volatile int* flag = reinterpret_cast<volatile int*>(sm + S::kBar + 8);

    // warp = (row group, K segment); lane word j covers elements e(j) .. +15
    // of the segment: 16-byte chunks lane + 32 i (WPL >= 4) or the 8-byte
    // piece `lane` (WPL = 2), so the shared-memory reads of a warp are
    // consecutive
    const int seg = warp % KSPLIT, rgp = warp / KSPLIT;
    auto elem = [&](int j) -> int {
        return WPL >= 4 ? seg * KSEG + 64 * (lane + 32 * (j / 4)) + 16 * (j % 4)
                        : seg * KSEG + 32 * lane + 16 * j;
    };
    uint32_t a[MT][4 * WPL];
#pragma unroll
    for (int m = 0; m < MT; ++m)
#pragma unroll
        for (int j = 0; j < WPL; ++j) {
            const uint4 v = *reinterpret_cast<const uint4*>(codes + m * K + elem(j));
            a[m][4 * j] = v.x;
            a[m][4 * j + 1] = v.y;
            a[m][4 * j + 2] = v.z;
            a[m][4 * j + 3] = v.w;
        }
    if (tid == 0)
        *flag = mbar_wait_bounded<false>(smem_addr(sm + S::kBar), 0, kTimeoutNs) ? 1 : 0;
    __syncthreads();
    if (*flag == 0) {
        if (tid == 0) report_status(p.status, HBL_ERR_TIMEOUT);
        return;
    }
    const uint8_t* wsm = sm + S::weights(p.rows);
    int32_t* part = reinterpret_cast<int32_t*>(sm + S::kPart);
    // two rows of the row group per step (independent chains overlap)
    for (int r0 = rgp; r0 < rows; r0 += 2 * RG) {
        uint32_t wd[2][WPL];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = r0 + u * RG;
            const uint8_t* wr = wsm + (r < rows ? r : r0) * (K / 4);
#pragma unroll
            for (int j = 0; j < WPL; j += (WPL >= 4 ? 4 : 2)) {
                if constexpr (WPL >= 4) {
                    const uint4 t = *reinterpret_cast<const uint4*>(wr + elem(j) / 4);
                    wd[u][j] = t.x, wd[u][j + 1] = t.y, wd[u][j + 2] = t.z, wd[u][j + 3] = t.w;
                } else {
                    const uint2 t = *reinterpret_cast<const uint2*>(wr + elem(j) / 4);
                    wd[u][j] = t.x, wd[u][j + 1] = t.y;
                }
            }
        }
        int v[2][MT];
#pragma unroll
        for (int u = 0; u < 2; ++u)
#pragma unroll
            for (int m = 0; m < MT; ++m) {
                int s0 = 0, s1 = 0, s2 = 0, s3 = 0;
#pragma unroll
                for (int j = 0; j < WPL; ++j) {
                    s0 = dp4a_su(a[m][4 * j + 0], wd[u][j] & 0x03030303u, s0);
                    s1 = dp4a_su(a[m][4 * j + 1], wd[u][j] & 0x0C0C0C0Cu, s1);
                    s2 = dp4a_su(a[m][4 * j + 2], wd[u][j] & 0x30303030u, s2);
                    s3 = dp4a_su(a[m][4 * j + 3], wd[u][j] & 0xC0C0C0C0u, s3);
                }
                v[u][m] = s0 + (s1 >> 2) + (s2 >> 4) + (s3 >> 6);
            }
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1)
#pragma unroll
            for (int u = 0; u < 2; ++u)
#pragma unroll
                for (int m = 0; m < MT; ++m) v[u][m] += __shfl_xor_sync(0xffffffffu, v[u][m], o);
#pragma unroll
        for (int u = 0; u < 2; ++u) {
            const int r = r0 + u * RG;
            if (lane < MT && r < rows) {
                int x = v[u][0];
#pragma unroll
                for (int m = 1; m < MT; ++m) x = lane == m ? v[u][m] : x;
                part[(r * KSPLIT + seg) * MT + lane] = x;
            }
        }
    }
    __syncthreads();

    // sum over the K segments, dequantise, store
    const float al = *p.alpha;
    for (int vi = tid; vi < rows * MT; vi += NT) {
        const int m = vi % MT, r = vi / MT;
        if (m >= M) continue;
        int s = -rs[m];
#pragma unroll
        for (int g = 0; g < KSPLIT; ++g) s += part[(r * KSPLIT + g) * MT + m];
        const float y = __fmul_rn((float)s, __fmul_rn(al, sc[m]));
        p.Y[(int64_t)m * p.N + n0 + r] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
}

// The one-kernel decode forward as an extension of K1's kernel template.
template <int L, int MT>
struct DecodeExt {
    using S = Shape<L, MT>;
    static constexpr bool kOn = true;
    template <int>
    __host__ __device__ static constexpr int threads() { return S::NT; }
    template <int>
    __host__ __device__ static constexpr int min_blocks() { return 1; }
    template <int>
    __host__ __device__ static constexpr int rlog() { return S::RLOG; }
    template <int>
    __host__ __device__ static constexpr int groups() { return S::GPC; }

    static __device__ uint8_t* codes() { return dyn_smem() + S::kCodes; }
    static __device__ float* scales() { return reinterpret_cast<float*>(dyn_smem() + S::kScales); }
    static __device__ int32_t* rowsum() {
        return reinterpret_cast<int32_t*>(dyn_smem() + S::kRowsum);
    }
    // 1a. token rows into L2 ahead of the weight traffic; the weights' mbarrier
    static __device__ void prologue(const k1::Params& p) {
        if (threadIdx.x == 0) {
            prefetch_l2_bulk(p.X, (uint32_t)(p.M * (1 << L) * 2));
            init_weight_barrier<S>(dyn_smem());
        }
    }
    // 1b. (thread 0, first row staged) the CTA's packed weight rows -> shared memory
    static __device__ void staged(const k1::Params& p) { issue_weights<S, L>(p, dyn_smem()); }
    // 3-4. after the rows: the GEMV over this CTA's weight rows and the epilogue
    static __device__ void finish(const k1::Params& p) {
        __syncthreads();  // codes, scales, row sums complete
        gemv_phase<S, L, MT>(p, dyn_smem(), codes(), scales(), rowsum());
    }
};

// The GEMV half alone, for decode batches K6 does not take (M <= 8): launched
// as a programmatic dependent of K1, it starts its weight rows' bulk copies
// before the dependency wait (the weights are not K1's output), then reads
// K1's codes (one byte each, row-major), scales and row sums from global
// memory.
template <int L, int MT>
__global__ void __launch_bounds__(256, 1) decode_gemv_kernel(const __grid_constant__ k1::Params p) {
    using S = Shape<L, MT, false>;
    uint8_t* sm = dyn_smem();
    if (threadIdx.x == 0) {
        init_weight_barrier<S>(sm);
        issue_weights<S, L>(p, sm);
    }
    pdl_wait();
    gemv_phase<S, L, MT>(p, sm, p.codes, p.scales, p.rowsum);
}

template <int L, int MT, int MODE, int FL>
hbl_status launch(const DecodeArgs& d, cudaStream_t stream, int num_sms) {
    k1::Params p = {};
    p.X = d.X;
    p.gain = d.gain;
    p.M = d.M;
    p.norm_eps = d.norm_eps;
    p.quant_eps = d.quant_eps;
    p.cK = (float)(1.0 / sqrt((double)(1 << L)));
    p.s7 = (float)sqrt(7.0);
    p.thr16 = k1::thr16_for(1 << L);
    p.W = d.W_packed;
    p.alpha = d.alpha;
    p.Y = d.Y;
    p.status = d.status;
    p.N = d.N;
    p.rows = decode_fused_rows(d.N, num_sms);
    const int smem = Shape<L, MT>::total(p.rows);
    auto kern = k1::norm_fwht_quant_kernel<L, MODE, FL, DecodeExt<L, MT>>;
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), smem)) return HBL_ERR_CUDA;
    const unsigned grid = (unsigned)((d.N + p.rows - 1) / p.rows);
    kern<<<grid, Shape<L, MT>::NT, smem, stream>>>(p);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

// Token capacities: up to 2^(14 - L) (one K1 row group per token): 1, 2, 4
// at K = 4096, 1, 2 at K = 8192, 1 at K = 16384.
template <int L, int MT>
hbl_status launch_gemv(const GemvArgs& g, cudaStream_t stream, int num_sms) {
    k1::Params p = {};
    p.M = g.M;
    p.codes = const_cast<uint8_t*>(g.codes);
    p.scales = const_cast<float*>(g.scales);
    p.rowsum = const_cast<int32_t*>(g.rowsum);
    p.W = g.W_packed;
    p.alpha = g.alpha;
    p.Y = g.Y;
    p.status = g.status;
    p.N = g.N;
    p.rows = decode_fused_rows(g.N, num_sms);
    const int smem = Shape<L, MT, false>::total(p.rows);
    auto kern = decode_gemv_kernel<L, MT>;
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), smem)) return HBL_ERR_CUDA;
    const unsigned grid = (unsigned)((g.N + p.rows - 1) / p.rows);
    return launch_pdl(kern, dim3(grid), dim3(256), (size_t)smem, stream, p);
}

template <int L>
int gemv_smem_bytes(int N, int MT, int num_sms) {
    const int rows = decode_fused_rows(N, num_sms);
    if (MT == 1) return Shape<L, 1, false>::total(rows);
    if (MT == 2) return Shape<L, 2, false>::total(rows);
    if (MT == 4) return Shape<L, 4, false>::total(rows);
    return Shape<L, 8, false>::total(rows);
}

// Token capacities 1, 2, 4, 8 (8: the codes take 128 registers per lane).
template <int L>
hbl_status launch_gemv_l(const GemvArgs& g, cudaStream_t s, int sms) {
    if (g.M <= 1) return launch_gemv<L, 1>(g, s, sms);
    if (g.M <= 2) return launch_gemv<L, 2>(g, s, sms);
    if (g.M <= 4) return launch_gemv<L, 4>(g, s, sms);
    return launch_gemv<L, 8>(g, s, sms);
}

template <int L>
int smem_bytes(int N, int MT, int num_sms) {
    const int rows = decode_fused_rows(N, num_sms);
    if (MT == 1) return Shape<L, 1>::total(rows);
    if constexpr (L <= 13)
        if (MT == 2) return Shape<L, 2>::total(rows);
    if constexpr (L <= 12)
        if (MT == 4) return Shape<L, 4>::total(rows);
    return 1 << 30;
}

template <int L, int MODE, int FL>
hbl_status by_m(const DecodeArgs& d, cudaStream_t s, int sms) {
    if (d.M <= 1) return launch<L, 1, MODE, FL>(d, s, sms);
    if constexpr (L <= 13)
        if (d.M <= 2) return launch<L, 2, MODE, FL>(d, s, sms);
    if constexpr (L <= 12)
        if (d.M <= 4) return launch<L, 4, MODE, FL>(d, s, sms);
    return HBL_ERR_SHAPE;
}

// All launches of one K: INT4 / INT8, with or without the per-channel gain.
template <int L>
hbl_status launch_l(const DecodeArgs& d, cudaStream_t s, int sms) {
    const bool gain = d.gain != nullptr;
    if (d.act_bits == 4)
        return gain ? by_m<L, 6, k1::kFlGain>(d, s, sms) : by_m<L, 6, 0>(d, s, sms);
    return gain ? by_m<L, 8, k1::kFlGain>(d, s, sms) : by_m<L, 8, 0>(d, s, sms);
}

}  // namespace k6
}  // namespace hbl
