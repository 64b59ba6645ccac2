// k10_gemm_pair.cu -- ternary-weight GEMM for large token batches on pairs of
// sm_100a SMs: tcgen05.mma.cta_group::2 over a 256-token x 256-weight-row tile
// shared by the two CTAs of a cluster, both operands TMA-fed.
//
// Computes (BitNet v2 write-up, 0755model.com, section "H-BitLinear": the
// ternary matmul of the per-token quantised activations, rescaled by the
// weight and activation scales)
//   acc[m][n] = sum_k q[m][k] * t[n][k]   (exact, int32)
//   Y[m][n]   = bf16_rne((float)acc * (alpha * s[m]))
// with q one byte per code, row-major [M x K], and t in {-1, 0, +1} one signed
// byte per weight, row-major [N x K] (the expansion kernel's output).
//
// Why pairs: with both operands in shared memory a one-SM 128 x 256 x 32 MMA
// reads 12 KB of shared memory and the TMA writes 12 KB per 128 tensor cycles,
// more than the SM's shared memory moves, so the one-SM kernel tops out near
// three quarters of the tensor peak.  In the paired form the MMA is issued by
// the even CTA of the cluster for both SMs: each SM holds its 128 token rows of
// A and one half (128 weight rows) of B, and each SM's tensor core reads its
// own A and both halves of B.  Per SM and 128 tensor cycles that is 4 KB of A,
// 4 KB of B and 8 KB of TMA writes: two thirds of the one-SM traffic, and half
// the L2 -> SM bytes per output.
//
// Per CTA: one thread issues the TMA loads of its A half and B half for each
// 128-byte K stage (6 stages of 32 KB), signalling the even CTA's "full"
// barrier (the .cta_group::2 form of the load names a barrier in either CTA
// of the pair; no multicast); the even CTA's MMA thread waits there, issues four
// tcgen05.mma.cta_group::2.kind::i8 (M = 256, N = 256, K = 32) and commits to
// both CTAs' "empty" barriers; four warps per CTA drain that CTA's 128 x 256
// int32 accumulator (double-buffered in TMEM, 512 columns allocated by the
// pair) and report to the even CTA's "accumulator empty" barrier.  Every wait
// is bounded by the global timer; on expiry the kernel records HBL_ERR_TIMEOUT,
// stops issuing, lets its own loads and MMAs land, and both CTAs meet at a
// cluster barrier before the pair frees its TMEM and exits.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k10 {

constexpr int BM = 256;       // tokens per pair tile (128 per CTA: TMEM lanes)
constexpr int BMC = BM / 2;   // tokens per CTA
constexpr int BN = 256;       // weight rows per pair tile (MMA N)
constexpr int BNC = BN / 2;   // weight rows held by one CTA
constexpr int BK = 128;       // K bytes per stage
constexpr int S = 6;          // pipeline stages
constexpr int kAStage = BMC * BK;
constexpr int kBStage = BNC * BK;
constexpr int kStage = kAStage + kBStage;
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kBarBytes = 256;
constexpr int kSmemBytes = S * kStage + kBarBytes + 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;
constexpr uint16_t kPairMask = 0x3;

// kind::i8: D s32 (bits 4-5 = 2), A s8 (bits 7-9 = 1), B s8 (bits 10-12 = 1),
// both K-major, N >> 3 at bit 17, M >> 4 at bit 24 (M = 256: the pair's rows).
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

template <bool SLEEP>
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<SLEEP>(a, parity, kTimeoutNs);
}
// Bounded wait with cluster-scope acquire, for a barrier other CTAs arrive on.
__device__ __forceinline__ bool mbar_wait_cluster(uint32_t a, uint32_t parity) {
    auto test = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n.reg .pred p;\n"
            "mbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2;\n"
            "selp.u32 %0, 1, 0, p;\n}\n"
            : "=r"(ok)
            : "r"(a), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (test()) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        __nanosleep(64);
        if (test()) return true;
        if (global_ns() - t0 > kTimeoutNs) return false;
    }
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t a, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(a), "r"(bytes)
                 : "memory");
}
// arrive on a barrier of any CTA of the cluster (shared::cluster address)
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(
                     cluster_addr)
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
// One paired MMA: the descriptors name the same shared-memory offsets in both
// CTAs (A: each CTA's 128 token rows; B: each CTA's 128 weight rows).
__device__ __forceinline__ void mma_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accum) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::2.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accum)
        : "memory");
}
// Arrive (once the pair's prior MMAs complete) on the barrier at this
// shared-memory offset in both CTAs of the pair.
__device__ __forceinline__ void commit_pair_both(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 "
        "[%0], %1;" ::"r"(mbar),
        "h"(kPairMask)
        : "memory");
}
// Arrive on this CTA's own barrier once the pair's prior MMAs complete.
__device__ __forceinline__ void commit_pair_own(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
        : "memory");
}
// 2-D tiled TMA load (no multicast) into this CTA's shared memory, completing
// on a barrier of either CTA of the pair (shared::cluster address), with an
// L2 eviction-priority policy.
__device__ __forceinline__ void tma_load_pair(uint32_t dst, const CUtensorMap* map, int x, int y,
                                              uint32_t mbar_cluster, uint64_t policy) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
        ".L2::cache_hint [%0], [%1, {%2, %3}], [%4], %5;" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(mbar_cluster), "l"(policy)
        : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
// Every thread of both CTAs; prior shared-memory writes visible to the pair.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}

struct Params {
    int64_t M;
    int N, K;
    int tiles_m;    // token tiles of 256
    int tiles_n;    // weight-row tiles of 256
    int64_t tiles;  // total pair tiles
    const float* scales;
    const float* alpha;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* status;
};

// Pair tile t -> (token block, weight block): weight blocks in groups of
// kGroup (8 x 4 MB of expanded weights at K = 16384), token blocks in order
// within a group, so a group's weights stay in L2 (loaded with evict_last)
// while the activations stream past (evict_first).  A wave of 74 pairs covers
// about 9 token blocks x 8 weight blocks, all reading the same K slice at about
// the same time.  (W_down, 8192 tokens, a stand-alone copy of the kernel:
// DRAM reads 533 MB without the eviction hints, 414 MB with them; groups of 4
// or 16 read more.)
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
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA,
                     const __grid_constant__ CUtensorMap tmB, Params p) {
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
    const uint32_t rank = cluster_rank();
    const bool leader = rank == 0;
    const int64_t cid = blockIdx.x >> 1, nclusters = gridDim.x >> 1;
    const int num_kb = (p.K + BK - 1) / BK;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init_count(full_bar(s), 1);
            mbar_init_count(empty_bar(s), 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init_count(accf_bar(b), 1);
            mbar_init_count(acce_bar(b), 2 * kEpiWarps);
        }
        mbar_init_count(drain_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA))
                     : "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB))
                     : "memory");
    }
    if (warp == 1) {
        // the same warp of both CTAs allocates the pair's columns
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    // the codes and the expanded weights come from previous kernels
    pdl_wait();
    tc_fence_before();
    // barriers initialised and TMEM allocated in both CTAs before any remote use
    cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- TMA producer (one thread per CTA)
        if (lane == 0) {
            // a group's weight blocks are re-read by every token block of the
            // group (over several waves of tiles): keep them in L2 ahead of the
            // codes, which all the tiles that read them read at about the same time
            uint64_t pol_a, pol_b;
            asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol_a));
            asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol_b));
            uint32_t it = 0;
            bool ok = true;
            for (int64_t t = cid; t < p.tiles && ok; t += nclusters) {
                int mb, nb;
                tile_coords(p, t, mb, nb);
                // a half tile wholly past the end of A or B loads a valid
                // (partly out-of-range, zero-filled) box instead; its rows or
                // columns are never stored
                int64_t arow = (int64_t)mb * BM + (int64_t)rank * BMC;
                if (arow >= p.M) arow = p.M - 1;
                int brow = nb * BN + (int)rank * BNC;
                if (brow >= p.N) brow = p.N - 1;
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
                    if (leader) mbar_expect_tx(full_bar(s), 2u * (uint32_t)kStage);
                    const uint32_t fb = mapa(full_bar(s), 0);
                    tma_load_pair(sa, &tmA, kb * BK, (int)arow, fb, pol_a);
                    tma_load_pair(sa + kAStage, &tmB, kb * BK, brow, fb, pol_b);
                }
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // let every load of the pair land before either CTA may exit: the
            // even CTA's "full" phases count both CTAs' bytes; the odd CTA's
            // loads are also behind its "empty" phases (the MMAs read them)
            const uint32_t first = it > (uint32_t)S ? it - S : 0;
            for (uint32_t j = first; j < it; ++j) {
                const uint32_t bar = leader ? full_bar((int)(j % S)) : empty_bar((int)(j % S));
                if (!mbar_wait<true>(bar, (j / S) & 1)) break;
            }
        }
    } else if (warp == 1) {
        // ---------------- MMA issuer (one thread of the even CTA)
        if (leader && lane == 0) {
            uint32_t it = 0, tc = 0;
            bool ok = true;
            for (int64_t t = cid; t < p.tiles && ok; t += nclusters, ++tc) {
                const int b = (int)(tc & 1);
                if (tc >= 2 && !mbar_wait_cluster(acce_bar(b), ((tc >> 1) - 1) & 1)) {
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
                    const uint32_t sa = base_s + s * kStage;
                    const uint64_t ad = sdesc(sa), bd = sdesc(sa + kAStage);
#pragma unroll
                    for (int k = 0; k < BK / 32; ++k)
                        mma_pair(d, ad + (uint64_t)(2 * k), bd + (uint64_t)(2 * k),
                                 (kb | k) != 0 ? 1u : 0u);
                    commit_pair_both(empty_bar(s));
                }
                if (ok) commit_pair_both(accf_bar(b));
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // every MMA issued has completed once this commit arrives
            commit_pair_own(drain_bar);
            if (!mbar_wait<true>(drain_bar, 0)) report_status(p.status, HBL_ERR_TIMEOUT);
        }
    } else {
        // ---------------- epilogue: warps 2..5, one TMEM lane (token row) per thread
        const int q = warp & 3;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        const float alpha = *p.alpha;
        uint32_t tc = 0;
        for (int64_t t = cid; t < p.tiles; t += nclusters, ++tc) {
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
            const int64_t m = (int64_t)mb * BM + (int64_t)rank * BMC + 32 * q + lane;
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
            // the even CTA's MMA thread reuses this accumulator once all eight
            // epilogue warps of the pair have drained it
            if (lane == 0) mbar_arrive_cluster(mapa(acce_bar(b), 0));
        }
    }
    tc_fence_before();
    __syncthreads();
    // neither CTA frees the pair's TMEM or its shared memory while the other
    // may still use them
    cluster_sync_all();
    if (warp == 1) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols)
                     : "memory");
    }
}

// cuTensorMapEncodeTiled through the runtime's driver entry point.
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

// Row-major int8 matrix [rows x K] with a (128 rows x 128 bytes) box, 128B swizzle.
static bool make_map(CUtensorMap* map, const void* ptr, int64_t rows, int K) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {(cuuint32_t)BK, 128u};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(ptr), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Pairs of CTAs that can be resident at once (cached; 0 if the query fails).
static int max_pairs() {
    static std::once_flag once;
    static int n = 0;
    std::call_once(once, [] {
        if (!smem_attr_once(reinterpret_cast<const void*>(gemm_pair_kernel), kSmemBytes)) return;
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(2, 1, 1);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = 2;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int c = 0;
        if (cudaOccupancyMaxActiveClusters(&c, gemm_pair_kernel, &cfg) != cudaSuccess) {
            cudaGetLastError();
            c = 0;
        }
        n = c;
    });
    return n;
}

}  // namespace k10

bool gemm_pair_supported(int K) { return K >= k10::BK && K % k10::BK == 0 && k10::max_pairs() > 0; }

bool gemm_pair_preferred(int64_t M, int N, int num_sms) {
    const int64_t pairs = k10::max_pairs();
    if (pairs <= 0 || num_sms <= 0) return false;
    const int64_t tn = (N + 255) / 256;
    const int64_t pair_tiles = (M + 255) / 256 * tn, one_tiles = (M + 127) / 128 * tn;
    return (pair_tiles + pairs - 1) / pairs <= (one_tiles + num_sms - 1) / num_sms;
}

hbl_status launch_gemm_pair_s8w(const GemmArgs& a, const int8_t* W_s8, cudaStream_t stream) {
    if (a.M == 0) return HBL_OK;
    const int pairs = k10::max_pairs();
    if (pairs <= 0) return HBL_ERR_CUDA;
    CUtensorMap mA, mB;
    if (!k10::make_map(&mA, a.codes, a.M, a.K) || !k10::make_map(&mB, W_s8, a.N, a.K))
        return HBL_ERR_CUDA;
    k10::Params prm;
    prm.M = a.M;
    prm.N = a.N;
    prm.K = a.K;
    prm.tiles_m = (int)((a.M + k10::BM - 1) / k10::BM);
    prm.tiles_n = (a.N + k10::BN - 1) / k10::BN;
    prm.tiles = (int64_t)prm.tiles_m * prm.tiles_n;
    prm.scales = a.scales;
    prm.alpha = a.alpha;
    prm.Y = a.Y;
    prm.acc_out = a.acc_out;
    prm.status = a.dev_status;
    const int64_t nclusters = prm.tiles < pairs ? prm.tiles : pairs;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(2 * nclusters), 1, 1);
    cfg.blockDim = dim3(k10::kThreads);
    cfg.dynamicSmemBytes = k10::kSmemBytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, k10::gemm_pair_kernel, mA, mB, prm) == cudaSuccess
               ? HBL_OK
               : HBL_ERR_CUDA;
}

hbl_status launch_gemm_pair(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                            int num_sms) {
    if (a.M == 0) return HBL_OK;
    if (ws == nullptr || ws_bytes < gemm_tma_workspace(a.K, a.N)) return HBL_ERR_WORKSPACE;
    int8_t* wexp = static_cast<int8_t*>(ws);
    hbl_status st = launch_expand_ternary(a.W_packed, a.N, a.K, wexp, stream, num_sms);
    if (st != HBL_OK) return st;
    return launch_gemm_pair_s8w(a, wexp, stream);
}

}  // namespace hbl
