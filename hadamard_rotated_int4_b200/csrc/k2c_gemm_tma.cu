// k2c_gemm_tma.cu -- ternary-weight GEMM for large token batches on the
// sm_100a tensor cores: TMA loads of both operands, tcgen05.mma kind::i8 from
// shared memory, int32 accumulators in TMEM, fused dequantisation epilogue.
//
// Computes (BitNet v2 write-up, 0755model.com, section "H-BitLinear": the
// ternary matmul of the per-token quantised activations, rescaled by the
// weight and activation scales)
//   acc[m][n] = sum_k q[m][k] * t[n][k]   (exact, int32)
//   Y[m][n]   = bf16_rne((float)acc * (alpha * s[m]))
// with q one byte per code (INT8 values, or INT4 values in [-8, 7]) row-major,
// and t in {-1, 0, +1} one signed byte per weight, row-major [N x K].  The
// library's packed 2-bit weights are expanded to that form in workspace by
// the expansion kernel (k2d_expand_ternary.cu: N*K bytes written, N*K/4 read)
// before the GEMM.
//
// There is no narrower integer MMA than 8 bits in tcgen05, so the weights must
// reach shared memory as bytes; expanding them once per call in HBM (67 MB for
// 4096 x 16384, about 1% of the GEMM's time) lets the TMA engine stream both
// operands, leaving every SM's threads free: one thread issues TMA loads, one
// issues MMAs, four warps run the epilogue.
//
// Tile 128 tokens x 256 weight rows, K in stages of 128 bytes (one 128-byte
// swizzled row per token / weight row: the TMA SWIZZLE_128B pattern is the
// K-major layout the MMA descriptors name), 4 stages (48 KB each).  Persistent
// CTAs walk the tiles in groups of 8 weight blocks, token blocks in order within
// a group, so a group's weights stay in L2 while the activations stream past.  TMEM holds two 128 x 256 int32 accumulators: the
// epilogue drains one while the MMAs fill the other.  Every wait is bounded by
// the global timer; on expiry the kernel records HBL_ERR_TIMEOUT and stops,
// letting its own TMA loads and MMAs land before it frees TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k2c {

constexpr int BM = 128;  // tokens per tile (TMEM lanes)
constexpr int BN = 256;  // weight rows per tile (MMA N)
constexpr int BK = 128;  // K bytes per stage
constexpr int S = 4;     // pipeline stages
constexpr int kAStage = BM * BK;
constexpr int kBStage = BN * BK;
constexpr int kStage = kAStage + kBStage;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kBarBytes = 256;
constexpr int kSmemBytes = S * kStage + kBarBytes + 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// kind::i8: D s32 (bits 4-5 = 2), A s8 (bits 7-9 = 1), B s8 (bits 10-12 = 1),
// both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

// mbarrier helpers over the library's bounded wait (kTimeoutNs of global time)
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) { mbar_init_count(a, count); }
__device__ __forceinline__ void mbar_arrive(uint32_t a) { mbar_arrive_one(a); }
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes)
                 : "memory");
}
template <bool SLEEP>
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<SLEEP>(a, parity, kTimeoutNs);
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// K-major, 128-byte-swizzled shared-memory matrix descriptor (8-row atoms of
// 1024 bytes, SBO = 1024), version 1.
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accum) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
        : "memory");
}
// 2-D tiled TMA load of box (x, y) into shared memory, completing on mbar.
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, int x, int y,
                                         uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}

struct Params {
    int64_t M;
    int N, K;
    int tiles_m;    // token tiles
    const float* scales;
    const float* alpha;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* status;
    int tiles_n;    // weight-row tiles
    int64_t tiles;  // total tiles
};

// Tile t -> (token block, weight block).  Weight blocks go in groups of kGroup
// (kGroup x 4 MB of expanded weights at K = 16384); within a group the token
// blocks run in order, so the group's weights stay in L2 while the
// activations stream past, and a wave of 148 tiles spans ~18 token blocks.
constexpr int kGroup = 8;
__device__ __forceinline__ void tile_coords(const Params& p, int64_t t, int& mb, int& nb) {
    const int64_t per_group = (int64_t)p.tiles_m * kGroup;
    const int g = (int)(t / per_group);
    const int gw = min(kGroup, p.tiles_n - g * kGroup);
    const int64_t idx = t - (int64_t)g * per_group;
    mb = (int)(idx / gw);
    nb = g * kGroup + (int)(idx % gw);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_tma_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                    Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t bar_s = base_s + S * kStage;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + S * kStage + 8 * (2 * S + 5));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto full_bar = [&](int s) { return bar_s + 8u * s; };
    auto empty_bar = [&](int s) { return bar_s + 8u * (S + s); };
    auto accf_bar = [&](int b) { return bar_s + 8u * (2 * S + b); };
    auto acce_bar = [&](int b) { return bar_s + 8u * (2 * S + 2 + b); };
    const uint32_t drain_bar = bar_s + 8u * (2 * S + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int num_kb = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 1);
            mbar_init(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(accf_bar(b), 1);
            mbar_init(acce_bar(b), kEpiWarps);
        }
        mbar_init(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA))
                     : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB))
                     : "memory");
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // the codes come from the previous kernel (programmatic dependent launch)
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (one thread)
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
                int mb, nb;
                tile_coords(p, t, mb, nb);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = (int)(it % S);
                    if (it >= (uint32_t)S &&
                        !mbar_wait<true>(empty_bar(s), ((it / S) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    const uint32_t sa = base_s + s * kStage;
                    mbar_expect_tx(full_bar(s), (uint32_t)kStage);
                    tma_load(sa, &tmA, kb * BK, mb * BM, full_bar(s));
                    tma_load(sa + kAStage, &tmB, kb * BK, nb * BN, full_bar(s));
                }
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // let every load this thread issued land before the CTA may exit
            const uint32_t first = it > (uint32_t)S ? it - S : 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait<true>(full_bar((int)(j % S)), (j / S) & 1)) break;
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
                const int b = (int)(tc & 1);
                if (tc >= 2 && !mbar_wait<true>(acce_bar(b), ((tc >> 1) - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint32_t d = tmem + (uint32_t)(BN * b);
                for (int kb = 0; kb < num_kb; ++kb, ++it) {
                    const int s = (int)(it % S);
                    if (!mbar_wait<false>(full_bar(s), (it / S) & 1) || *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint32_t sa = base_s + s * kStage, sb = sa + kAStage;
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        mma_ss(d, sdesc(sa + 32 * k), sdesc(sb + 32 * k), (kb | k) != 0 ? 1u : 0u);
                    mma_commit(empty_bar(s));
                }
                if (ok) mma_commit(accf_bar(b));
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // every MMA issued has completed once this commit arrives
            mma_commit(drain_bar);
            if (!mbar_wait<true>(drain_bar, 0)) report_status(p.status, HBL_ERR_TIMEOUT);
        }
    } else {
        // ---------------- epilogue: warps 2..5, one TMEM lane (token row) per thread
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float alpha = *p.alpha;
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tc) {
            const int b = (int)(tc & 1);
            bool ok = true;
            if (lane == 0) ok = mbar_wait<true>(accf_bar(b), (tc >> 1) & 1) && !*abort_flag;
            if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) {
                if (lane == 0) {
                    *abort_flag = 1;
                    report_status(p.status, HBL_ERR_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            int mb, nb;
            tile_coords(p, t, mb, nb);
            const int64_t m = (int64_t)mb * BM + 32 * q + lane;
            const bool mok = m < p.M;
            const float sc = mok ? __fmul_rn(alpha, p.scales[m]) : 0.f;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                const uint32_t taddr = tmem + lane_base + (uint32_t)(BN * b + 32 * cc);
                asm volatile(
                    "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
                    "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
                    "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
                    "%31}, [%32];"
                    : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]),
                      "=r"(v[6]), "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]),
                      "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]),
                      "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]),
                      "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]), "=r"(v[26]),
                      "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
                    : "r"(taddr));
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                const int nc = nb * BN + 32 * cc;
                if (mok && nc < p.N) {
                    uint32_t out[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float y0 = __fmul_rn((float)(int)v[2 * e], sc);
                        const float y1 = __fmul_rn((float)(int)v[2 * e + 1], sc);
                        out[e] = (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y0)) |
                                 ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(y1)) << 16);
                    }
                    uint4* dst = reinterpret_cast<uint4*>(p.Y + m * (int64_t)p.N + nc);
                    const int halves = (p.N - nc) >= 32 ? 2 : 1;
#pragma unroll
                    for (int hh = 0; hh < 2; ++hh)
                        if (hh < halves) {
                            dst[2 * hh] = make_uint4(out[8 * hh], out[8 * hh + 1], out[8 * hh + 2],
                                                     out[8 * hh + 3]);
                            dst[2 * hh + 1] = make_uint4(out[8 * hh + 4], out[8 * hh + 5],
                                                         out[8 * hh + 6], out[8 * hh + 7]);
                        }
                    if (p.acc_out != nullptr) {
                        int4* ad = reinterpret_cast<int4*>(p.acc_out + m * (int64_t)p.N + nc);
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (e < halves * 4)
                                ad[e] = make_int4((int)v[4 * e], (int)v[4 * e + 1],
                                                  (int)v[4 * e + 2], (int)v[4 * e + 3]);
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(acce_bar(b));
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point (the library
// links the CUDA runtime statically and not libcuda directly).
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
    static std::once_flag once;
    static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
    std::call_once(once, [] {
        void* f = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
    });
    return fn;
}

// Row-major int8 matrix [rows x K] with a (box_rows x 128-byte) box, 128B swizzle.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int K, int box_rows) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)BK, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace k2c

size_t gemm_tma_workspace(int K, int N) { return ((size_t)N * (size_t)K + 255) & ~(size_t)255; }

hbl_status launch_gemm_tma_s8w(const GemmArgs& a, const int8_t* W_s8, cudaStream_t stream,
                               int num_sms) {
    if (a.M == 0) return HBL_OK;
    CUtensorMap mA, mB;
    if (!k2c::make_map(&mA, a.codes, a.M, a.K, k2c::BM) ||
        !k2c::make_map(&mB, W_s8, a.N, a.K, k2c::BN))
        return HBL_ERR_CUDA;
    k2c::Params prm;
    prm.M = a.M;
    prm.N = a.N;
    prm.K = a.K;
    prm.scales = a.scales;
    prm.alpha = a.alpha;
    prm.Y = a.Y;
    prm.acc_out = a.acc_out;
    prm.status = a.dev_status;
    prm.tiles_n = (a.N + k2c::BN - 1) / k2c::BN;
    prm.tiles_m = (int)((a.M + k2c::BM - 1) / k2c::BM);
    prm.tiles = (int64_t)prm.tiles_m * prm.tiles_n;
    if (!smem_attr_once(reinterpret_cast<const void*>(k2c::gemm_tma_kernel), k2c::kSmemBytes))
        return HBL_ERR_CUDA;
    const int64_t grid = prm.tiles < num_sms ? prm.tiles : num_sms;
    k2c::gemm_tma_kernel<<<(unsigned)grid, k2c::kThreads, k2c::kSmemBytes, stream>>>(mA, mB, prm);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

hbl_status launch_gemm_tma(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                           int num_sms) {
    if (a.M == 0) return HBL_OK;
    if (ws == nullptr || ws_bytes < gemm_tma_workspace(a.K, a.N)) return HBL_ERR_WORKSPACE;
    int8_t* wexp = static_cast<int8_t*>(ws);
    hbl_status st = launch_expand_ternary(a.W_packed, a.N, a.K, wexp, stream, num_sms);
    if (st != HBL_OK) return st;
    return launch_gemm_tma_s8w(a, wexp, stream, num_sms);
}

}  // namespace hbl
