// k8_gemm_wt.cu -- ternary-weight GEMM for large token batches on the sm_100a
// tensor cores, reading the 2-bit packed weights directly (no expanded copy).
//
// Computes (BitNet v2 write-up, 0755model.com, section "H-BitLinear": the
// ternary matmul of the per-token quantised activations, rescaled by the
// weight and activation scales)
//   acc[m][n] = sum_k q[m][k] * t[n][k]     (exact, int32)
//   Y[m][n]   = bf16_rne((float)acc * (alpha * s[m]))
// for codes q one byte each, row-major [M x K] (INT8, or INT4 values in
// [-8, 7]) and the library's packed weights (16 per uint32, code t + 1).
//
// The weights are the MMA's A operand, in tensor memory: 128 weight rows per
// tile (TMEM lanes), and the tokens its B operand from shared memory: 256
// tokens per tile (MMA N).  Shared memory then carries only the tokens' codes
// (TMA, 128-byte swizzle) and the packed weights (TMA, 32 bytes per row and
// stage, 32-byte swizzle): per 128 x 256 x 32 MMA it reads 8 KB and is written
// 9 KB, against 12 + 12 KB when both byte operands sit in shared memory; the
// weights are widened to bytes in registers by eight converter warps
// ((w >> 2m) & 0x03030303 is the codes of weights 4m..4m+3 in natural order)
// and stored with tcgen05.st.  The weights enter as c = t + 1 (unsigned), so
// the accumulator holds acc + rowsum[m]; the epilogue subtracts rowsum.
//
// Persistent CTAs, one per SM, walk the tiles token block by token block (the
// weight block varies fastest): the packed weights (16.8 MB for 4096 x 16384)
// and the token blocks in flight stay in L2, so HBM sees each code once.
// Warp 0 allocates TMEM (512 columns: the 128 x 256 int32 accumulator in
// [0, 256), a 3-stage ring of A tiles in [256, 448)) and one lane issues the
// MMAs, eight per 256-byte K stage (a stage's barrier waits and commits cost
// about as much issue time as four MMAs, so stages are long); warp 1 issues
// the TMA loads (3-stage ring of 72 KB: 64 KB of codes in two 128-byte-wide
// boxes and 8 KB of packed weights in two 32-byte-wide boxes); warps 2-13 convert, in three groups of four warps
// that take the stages round-robin (one stage's conversion is a chain of
// waits, loads and a TMEM store round trip; three in flight keep up with the
// MMAs); warps 14-21 drain the
// accumulator (tcgen05.ld), subtract rowsum, scale and store bf16 Y.  Every
// mbarrier wait is bounded by the global timer; on expiry the kernel records
// HBL_ERR_TIMEOUT, stops issuing, lets its copies and MMAs land (bounded) and
// frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k8 {

constexpr int kRows = 128;  // weight rows per tile (MMA M, TMEM lanes)
constexpr int NT = 256;     // tokens per tile (MMA N)
constexpr int BK = 256;     // K bytes per stage: 8 MMAs of K = 32
constexpr int kSub = BK / 128;  // 128-byte K sub-tiles per stage (one TMA box of codes each)
constexpr int S = 3;        // stages of the shared-memory ring (codes + packed weights)
// stages of the TMEM A ring (32 columns each).  SA <= S keeps every mbarrier
// wait within one phase of the barrier's state: a converter group waits for
// stage j's codes and weights only after the MMAs of stage j - SA (hence the
// loads of stage j - S) are done, and groups run at most one A round apart.
constexpr int SA = S;
constexpr int kConvGroups = 3;  // converter groups of four warps, stages round-robin
constexpr int kConvWarps = 4 * kConvGroups;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (2 + kConvWarps + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol = 256;
constexpr int kBBytes = NT * BK;         // 64 KB of codes per stage (two 32 KB boxes)
constexpr int kWBytes = kRows * BK / 4;  // 8 KB of packed weights per stage (two 4 KB boxes)
constexpr int kStage = kBBytes + kWBytes;
constexpr int kBarOff = S * kStage;
constexpr int kEpiOff = kBarOff + 256;  // per-tile token scales and row sums, double-buffered
constexpr int kSmemBytes = kEpiOff + 2 * NT * 8 + 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// kind::i8: D s32, A u8 (weights from TMEM), B s8 (codes), K-major, N = 256, M = 128.
constexpr uint32_t kIdesc = (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
                            ((uint32_t)(kRows >> 4) << 24);

struct Params {
    int64_t M;
    int N, K;
    int tiles_n;  // weight blocks
    int64_t tiles;
    const float* scales;
    const int32_t* rowsum;
    const float* alpha;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* status;
};

__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<false>(a, parity, kTimeoutNs);
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<true>(a, parity, kTimeoutNs);
}
__device__ __forceinline__ bool warp_wait(uint32_t a, uint32_t parity) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait_sleep(a, parity);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes)
                 : "memory");
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
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t accum) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %3, 0;\n"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %4, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(accum), "r"(kIdesc)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
        : "memory");
}
// 2-D tiled TMA load (no multicast) of box (x, y) into this CTA's shared memory.
__device__ __forceinline__ void tma_load(uint32_t dst, const CUtensorMap* map, int x, int y,
                                         uint32_t mbar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar)
        : "memory");
}
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}
__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16, "
        "%17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31, %32};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
        "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
        "r"(r[29]), "r"(r[30]), "r"(r[31])
        : "memory");
}
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, "
        "%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]),
          "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]),
          "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]),
          "=r"(v[31])
        : "r"(taddr));
}

// tile t -> token block mb, weight block nb (weight blocks fastest)
__device__ __forceinline__ void tile_coords(const Params& p, int64_t t, int64_t& mb, int& nb) {
    mb = t / p.tiles_n;
    nb = (int)(t - mb * p.tiles_n);
}

__global__ void __launch_bounds__(kThreads, 1)
    gemm_wt_kernel(const __grid_constant__ CUtensorMap tmB, const __grid_constant__ CUtensorMap tmW,
                   Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t bar_s = base_s + kBarOff;
    auto full = [&](int s) { return bar_s + 8u * s; };
    auto empty = [&](int s) { return bar_s + 8u * (S + s); };
    auto full_a = [&](int s) { return bar_s + 8u * (2 * S + s); };
    auto empty_a = [&](int s) { return bar_s + 8u * (2 * S + SA + s); };
    const uint32_t acc_full = bar_s + 8u * (2 * S + 2 * SA);
    const uint32_t acc_empty = bar_s + 8u * (2 * S + 2 * SA + 1);
    const uint32_t drain = bar_s + 8u * (2 * S + 2 * SA + 2);
    uint32_t* tmem_slot =
        reinterpret_cast<uint32_t*>(base + kBarOff + 8 * (2 * S + 2 * SA + 3));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int nkb = p.K / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init_count(full(s), 1);
            mbar_init_count(empty(s), 1);
        }
        for (int s = 0; s < SA; ++s) {
            mbar_init_count(full_a(s), 4);  // the four warps of one converter group
            mbar_init_count(empty_a(s), 1);
        }
        mbar_init_count(acc_full, 1);
        mbar_init_count(acc_empty, kEpiWarps);
        mbar_init_count(drain, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    pdl_wait();  // the codes come from the previous kernel
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x, ++tc) {
                if (tc >= 1 && !mbar_wait_sleep(acc_empty, (tc - 1) & 1)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = (int)(it % S), a = (int)(it % SA);
                    if (!mbar_wait(full_a(a), (it / SA) & 1) || !mbar_wait(full(s), (it / S) & 1) ||
                        *abort_flag) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    // descriptors of the stage: the MMAs step through them by
                    // constant offsets of the start-address field
                    const uint64_t bd0 = sdesc(base_s + (uint32_t)(s * kStage));
                    const uint32_t ad0 = tmem + kACol + (uint32_t)(BK / 4) * a;
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        mma_ts(tmem, ad0 + 8u * k,
                               bd0 + (uint64_t)(((k >> 2) * NT * 128 + 32 * (k & 3)) >> 4),
                               (kb | k) != 0 ? 1u : 0u);
                    mma_commit(empty(s));
                    mma_commit(empty_a(a));
                }
                if (ok) mma_commit(acc_full);
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // every MMA issued has completed once this commit arrives
            mma_commit(drain);
            if (!mbar_wait_sleep(drain, 0)) report_status(p.status, HBL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- TMA producer (one thread): codes and packed weights
        if (lane == 0) {
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = blockIdx.x; t < p.tiles && ok; t += gridDim.x) {
                int64_t mb;
                int nb;
                tile_coords(p, t, mb, nb);
                for (int kb = 0; kb < nkb; ++kb, ++it) {
                    const int s = (int)(it % S);
                    if (it >= (uint32_t)S && !mbar_wait_sleep(empty(s), ((it / S) - 1) & 1)) {
                        ok = false;
                        break;
                    }
                    if (*abort_flag) {
                        ok = false;
                        break;
                    }
                    const uint32_t sb = base_s + (uint32_t)(s * kStage);
                    mbar_expect_tx(full(s), (uint32_t)kStage);
#pragma unroll
                    for (int j = 0; j < kSub; ++j) {
                        tma_load(sb + j * NT * 128, &tmB, kb * BK + 128 * j, (int)(mb * NT), full(s));
                        tma_load(sb + kBBytes + j * kRows * 32, &tmW, kb * (BK / 4) + 32 * j,
                                 nb * kRows, full(s));
                    }
                }
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // let every load issued land before the CTA may exit
            const uint32_t first = it > (uint32_t)S ? it - S : 0;
            for (uint32_t j = first; j < it; ++j)
                if (!mbar_wait_sleep(full((int)(j % S)), (j / S) & 1)) break;
        }
        __syncwarp();
    } else if (warp < 2 + kConvWarps) {
        // ---------------- converters: group g takes the stages it = g (mod
        // kConvGroups) of the CTA's stage sequence; a thread converts its weight
        // row (TMEM lane) of the stage: 32 bytes read (the 32-byte swizzle puts
        // 16-byte chunk c of row r at chunk c ^ ((r >> 2) & 1)), 32 words, one store
        const int cw = warp - 2;
        const int q = warp & 3;
        const int grp = cw >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const uint32_t sw = (uint32_t)((r >> 2) & 1);
        const uint32_t w0off = (uint32_t)kBBytes + (uint32_t)(r * 32) + (sw << 4);
        const uint32_t w1off = (uint32_t)kBBytes + (uint32_t)(r * 32) + ((sw ^ 1u) << 4);
        static_assert(kSub * kRows * 32 == kWBytes, "weight boxes fill the stage's weight part");
        const uint32_t total = (uint32_t)(((p.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x) * nkb);
        bool ok = true;
        for (uint32_t it = (uint32_t)grp; it < total; it += kConvGroups) {
            const int s = (int)(it % S), a = (int)(it % SA);
            if (!warp_wait(full(s), (it / S) & 1) ||
                (it >= (uint32_t)SA && !warp_wait(empty_a(a), ((it / SA) - 1) & 1)) ||
                __shfl_sync(0xffffffffu, *abort_flag, 0) != 0) {
                ok = false;
                break;
            }
            tc_fence_after();
            const uint32_t st_s = base_s + (uint32_t)(s * kStage);
#pragma unroll
            for (int j = 0; j < kSub; ++j) {  // each 4 KB weight box: 128 weights of row r
                const uint32_t bx = st_s + (uint32_t)(j * kRows * 32);
                const uint4 w0 = lds128(bx + w0off), w1 = lds128(bx + w1off);
                const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                uint32_t v[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v[4 * e + 0] = wv[e] & 0x03030303u;
                    v[4 * e + 1] = (wv[e] >> 2) & 0x03030303u;
                    v[4 * e + 2] = (wv[e] >> 4) & 0x03030303u;
                    v[4 * e + 3] = (wv[e] >> 6) & 0x03030303u;
                }
                tmem_st32(tmem + lane_base + kACol + (uint32_t)(BK / 4) * a + 32u * j, v);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_one(full_a(a));
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_status(p.status, HBL_ERR_TIMEOUT);
        }
    } else {
        // ---------------- epilogue: weight row r (TMEM lane), 128 of the 256 token columns
        const int ew = warp - 2 - kConvWarps;
        const int q = warp & 3;
        const int half = ew >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float alpha = *p.alpha;
        uint32_t tc = 0;
        for (int64_t t = blockIdx.x; t < p.tiles; t += gridDim.x, ++tc) {
            int64_t mb;
            int nb;
            tile_coords(p, t, mb, nb);
            const bool ready = warp_wait(acc_full, tc & 1);
            if (!ready || __shfl_sync(0xffffffffu, *abort_flag, 0) != 0) {
                if (lane == 0) {
                    *abort_flag = 1;
                    report_status(p.status, HBL_ERR_TIMEOUT);
                }
                break;
            }
            tc_fence_after();
            // the tile's 256 token scales (alpha * s) and row sums, one per thread
            float* tsc = reinterpret_cast<float*>(base + kEpiOff) + (tc & 1) * 2 * NT;
            int* trs = reinterpret_cast<int*>(tsc + NT);
            {
                const int j = 32 * ew + lane;
                const int64_t m = mb * NT + j;
                tsc[j] = m < p.M ? __fmul_rn(alpha, p.scales[m]) : 0.f;
                trs[j] = m < p.M ? p.rowsum[m] : 0;
            }
            named_barrier(1, 32 * kEpiWarps);
            const int n = nb * kRows + r;
            const bool nok = n < p.N;
#pragma unroll 1
            for (int cc = 0; cc < NT / 2 / 32; ++cc) {
                const int c0 = 128 * half + 32 * cc;
                uint32_t v[32];
                tmem_ld32(tmem + lane_base + (uint32_t)c0, v);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
                if (cc == NT / 2 / 32 - 1) {  // the accumulator is free for the next tile
                    tc_fence_before();
                    __syncwarp();
                    if (lane == 0) mbar_arrive_one(acc_empty);
                }
                const int64_t m0 = mb * NT + c0;
#pragma unroll
                for (int e = 0; e < 32; ++e) {
                    const int64_t m = m0 + e;
                    if (nok && m < p.M) {
                        const int a = (int)v[e] - trs[c0 + e];
                        const float sc = tsc[c0 + e];
                        p.Y[m * p.N + n] =
                            __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a, sc)));
                        if (p.acc_out != nullptr) p.acc_out[m * p.N + n] = a;
                    }
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

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

// 2-D uint8 map [rows x cols] (row stride = cols bytes) with the given box and swizzle.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int64_t cols, int box_x,
                     int box_y, CUtensorMapSwizzle sw) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)cols};
    const cuuint32_t box[2] = {(cuuint32_t)box_x, (cuuint32_t)box_y};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace k8

hbl_status launch_gemm_wt(const GemmArgs& a, cudaStream_t stream, int num_sms) {
    if (a.M == 0) return HBL_OK;
    if (a.K < k8::BK || a.K % k8::BK != 0) return HBL_ERR_SHAPE;
    CUtensorMap mB, mW;
    if (!k8::make_map(&mB, a.codes, a.M, a.K, 128, k8::NT, CU_TENSOR_MAP_SWIZZLE_128B) ||
        !k8::make_map(&mW, a.W_packed, a.N, a.K / 4, 32, k8::kRows,
                      CU_TENSOR_MAP_SWIZZLE_32B))
        return HBL_ERR_CUDA;
    k8::Params prm;
    prm.M = a.M;
    prm.N = a.N;
    prm.K = a.K;
    prm.tiles_n = (a.N + k8::kRows - 1) / k8::kRows;
    prm.tiles = (int64_t)prm.tiles_n * ((a.M + k8::NT - 1) / k8::NT);
    prm.scales = a.scales;
    prm.rowsum = a.rowsum;
    prm.alpha = a.alpha;
    prm.Y = a.Y;
    prm.acc_out = a.acc_out;
    prm.status = a.dev_status;
    if (!smem_attr_once(reinterpret_cast<const void*>(k8::gemm_wt_kernel), k8::kSmemBytes))
        return HBL_ERR_CUDA;
    const int64_t grid = prm.tiles < num_sms ? prm.tiles : num_sms;
    return launch_pdl(k8::gemm_wt_kernel, dim3((unsigned)grid), dim3(k8::kThreads),
                      (size_t)k8::kSmemBytes, stream, mB, mW, prm);
}

}  // namespace hbl
