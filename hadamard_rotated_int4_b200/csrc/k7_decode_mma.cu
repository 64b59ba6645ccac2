// k7_decode_mma.cu -- ternary-weight GEMM for decode batches (9 to 128
// tokens) on the sm_100a tensor cores, bound by the stream of packed weights.
//
// Computes (BitNet v2 write-up, 0755model.com, section "H-BitLinear": the
// ternary matmul of the per-token quantised activations, rescaled by the
// weight and activation scales)
//   acc[m][n] = sum_k q[m][k] * t[n][k]     (exact, int32)
//   Y[m][n]   = bf16_rne((float)acc * (alpha * s[m]))
// for codes q one byte each, row-major [M x K] (INT8, or INT4 values in
// [-8, 7]), and the library's 2-bit packed weights.
//
// The roles of the operands are swapped against the large-batch GEMM: the
// weights are the MMA's A operand (M = 128 weight rows per CTA, read from
// tensor memory) and the tokens its B operand (N = NT = the batch rounded up to
// 16, 32, 64 or 128, from shared memory), so a decode batch of 32 tokens wastes
// no tensor-core rows.  Per CTA:
//   - before the dependency wait (the weights are not the previous kernel's
//     output), one thread starts TMA loads of the CTA's 128 weight rows, its
//     K slice only, into shared memory: G boxes of 128 rows x 128 bytes with
//     the 128-byte swizzle (so the converters' 16-byte reads are free of bank
//     conflicts), each on its own mbarrier: the whole weight stream runs under
//     the quantiser kernel, in a few large requests;
//   - one thread TMA-loads the tokens' codes for each 512-byte K stage (four
//     128-byte-wide boxes) into a ring that takes the rest of shared memory
//     (all of the CTA's codes when they fit: the loads are L2 round trips, so
//     many must be in flight; SWIZZLE_128B, the K-major layout the MMA
//     descriptor names; rows past M are zero-filled);
//   - three groups of four converter warps take the stages round-robin (a
//     stage's conversion is a chain of waits, loads and TMEM store round
//     trips; three in flight keep up with the MMAs); a thread unpacks its
//     weight row's 512 weights of the stage in registers ((w >> 2m) &
//     0x03030303 is the codes of weights 4m..4m+3 as bytes, in natural order)
//     and stores them with four tcgen05.st into a 3-stage ring of A tiles in
//     TMEM (128 columns = 512 bytes per row and stage);
//   - one thread issues tcgen05.mma.cta_group::1.kind::i8 (A u8 from TMEM,
//     B s8 from shared memory, D s32 in TMEM), sixteen per stage (a stage's
//     barrier waits and commits cost about as much issue time as four MMAs),
//     and commits each stage back.
// The weights enter as the unsigned code c = t + 1, so the result carries
// sum_k q*c = acc + rowsum[m]; rowsum is subtracted once in the epilogue.
//
// K is split over the CS CTAs of a thread-block cluster (CS = 1, 2, 4 or 8,
// chosen so that ceil(N/128) * CS CTAs fill the SMs in one wave).  Each CTA
// leaves its int32 partials [NT x 128] in its own shared memory; after a
// cluster barrier CTA c sums rows [c * 128/CS, (c + 1) * 128/CS) over the CS
// CTAs through distributed shared memory (integer sums: exact in any order),
// subtracts rowsum and writes bf16 Y.  No workspace, no second kernel.
//
// TMEM: all 512 columns (D in [0, NT), the A ring in [128, 512)); the dynamic
// shared memory is at least 116 KB, so no two CTAs of this kernel share an SM.
// Every mbarrier
// wait is bounded by the global timer; on expiry the kernel records
// HBL_ERR_TIMEOUT, stops issuing, lets its own copies and MMAs land (bounded
// waits again), still takes part in both cluster barriers (every thread of
// every CTA reaches them after bounded work) and frees its TMEM.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <mutex>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k7 {

constexpr int kRows = 128;  // weight rows per CTA (MMA M, TMEM lanes)
constexpr int BK = 512;     // K bytes per stage: 16 MMAs of K = 32 (a stage's barrier
                            // waits and commits cost about as much issue time as
                            // four MMAs, so stages are long)
constexpr int kSub = BK / 128;  // 128-byte K sub-tiles per stage (one TMA box of codes each)
constexpr int kMaxSA = 3;   // stages of the A ring in TMEM (128 columns each)
constexpr int kMaxSB = 32;  // stages of the B ring in shared memory
// converter warp groups (stages round-robin); no more groups than A stages, so
// every empty-slot wait is within one phase of the barrier's state
constexpr int kConvGroups = kMaxSA;
constexpr int kConvWarps = 4 * kConvGroups;
constexpr int kThreads = 32 * (2 + kConvWarps);
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kACol = 128;  // first TMEM column of the A ring
constexpr int kMaxGroups = 16;
constexpr int kBoxBytes = 128 * 128;  // one swizzled weight box: 128 rows x 128 bytes
constexpr int kMinSmem = 116 * 1024;  // one CTA per SM: it may take all 512 TMEM columns
constexpr uint64_t kTimeoutNs = 2000000000ull;

// kind::i8: D s32 (bits 4-5 = 2), A u8 (bits 7-9 = 0), B s8 (bits 10-12 = 1),
// both K-major, N >> 3 at bit 17, M >> 4 at bit 24.
template <int NT>
__host__ __device__ constexpr uint32_t idesc() {
    return (2u << 4) | (0u << 7) | (1u << 10) | ((uint32_t)(NT >> 3) << 17) |
           ((uint32_t)(kRows >> 4) << 24);
}

struct Params {
    int M, K, N;
    int Kc;        // K per CTA (K / cluster size), a multiple of BK
    int G;         // weight boxes: Kc / 512 swizzled 128-byte boxes, one per stage
    int sw;        // the weight boxes are 128-byte swizzled (always, Kc >= 512)
    uint32_t b_off;  // offset of the B ring from the 1024-aligned base
    uint32_t bar_off;
    int SA, SB;      // ring depths (A in TMEM, B in shared memory)
    const uint32_t* W;
    const float* scales;
    const int32_t* rowsum;
    const float* alpha;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* status;
    int early_weights;  // launched after the kernel that writes the codes: the
                        // weight copies start before the dependency wait
};

__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<false>(a, parity, kTimeoutNs);
}
__device__ __forceinline__ bool mbar_wait_sleep(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<true>(a, parity, kTimeoutNs);
}
// Warp-uniform bounded wait: lane 0 waits, every lane gets its verdict.
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
template <int NT>
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                       uint32_t accum) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %3, 0;\n"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %4, p;\n}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(bdesc), "r"(accum), "r"(idesc<NT>())
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
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
__device__ __forceinline__ uint32_t cluster_size() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
    return r;
}
// Every thread of every CTA of the cluster: prior shared-memory writes are
// visible to the cluster after it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release;" ::: "memory");
    asm volatile("barrier.cluster.wait.acquire;" ::: "memory");
}
__device__ __forceinline__ uint32_t mapa(uint32_t saddr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
    return r;
}
__device__ __forceinline__ uint4 ld_cluster_v4(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared::cluster.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
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
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0, %1, %2, %3, %4, %5, %6, %7}, [%8];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t* v) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, "
        "%11, %12, %13, %14, %15}, [%16];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),
          "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]),
          "=r"(v[13]), "=r"(v[14]), "=r"(v[15])
        : "r"(taddr));
}

template <int NT>
__global__ void __launch_bounds__(kThreads, 1)
    decode_mma_kernel(const __grid_constant__ CUtensorMap tmB,
                      const __grid_constant__ CUtensorMap tmW, Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t w_s = base_s;              // weights, later the partial sums
    const uint32_t b_s = base_s + p.b_off;    // B ring: SB x NT x 128 bytes
    const uint32_t bar_s = base_s + p.bar_off;
    const int SA = p.SA, SB = p.SB;
    auto full_b = [&](int s) { return bar_s + 8u * s; };
    auto empty_b = [&](int s) { return bar_s + 8u * (kMaxSB + s); };
    auto full_a = [&](int s) { return bar_s + 8u * (2 * kMaxSB + s); };
    auto empty_a = [&](int s) { return bar_s + 8u * (2 * kMaxSB + kMaxSA + s); };
    auto wbar = [&](int g) { return bar_s + 8u * (2 * kMaxSB + 2 * kMaxSA + g); };
    const uint32_t acc_bar = bar_s + 8u * (2 * kMaxSB + 2 * kMaxSA + kMaxGroups);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(
        base + p.bar_off + 8 * (2 * kMaxSB + 2 * kMaxSA + kMaxGroups + 1));
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const uint32_t crank = cluster_rank(), csize = cluster_size();
    const int n0 = (int)blockIdx.y * kRows;
    const int k0 = (int)blockIdx.x * p.Kc;  // blockIdx.x == cluster rank (cluster along x)
    const int nkb = p.Kc / BK;
    const int rows = min(kRows, p.N - n0);

    // ---- the CTA's weight rows (its K slice) into shared memory: the weights
    // are not the previous kernel's output, so this runs before the dependency
    // wait, under that kernel, and first of all: warp 1 initialises the weight
    // barriers itself and starts the copies while the other barriers are set up
    // box g (= stage g): bytes [k0/4 + 128 g, + 128) of rows [n0, n0 + 128)
    // (rows past N read as zeros; the full box counts toward the transaction
    // bytes)
    constexpr int inner = 128;
    auto load_weights = [&] {
        if (lane == 0)
            for (int g = 0; g < p.G; ++g) {
                mbar_expect_tx(wbar(g), (uint32_t)(kRows * inner));
                tma_load(w_s + (uint32_t)(g * kRows * inner), &tmW, k0 / 4 + g * inner, n0,
                         wbar(g));
            }
        __syncwarp();
    };
    if (warp == 1) {
        if (lane == 0) {
            for (int g = 0; g < kMaxGroups; ++g) mbar_init_count(wbar(g), 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW))
                         : "memory");
        }
        __syncwarp();
        if (p.early_weights) load_weights();
    }
    // the other barriers, one per thread of warps 2 and up
    {
        const int i = (int)threadIdx.x - 64;
        const int nb = 2 * SB + 2 * SA + 1;
        if (i >= 0 && i < nb) {
            uint32_t a;
            uint32_t count = 1;
            if (i < SB) a = full_b(i);
            else if (i < 2 * SB) a = empty_b(i - SB);
            else if (i < 2 * SB + SA) { a = full_a(i - 2 * SB); count = 4; }  // a converter group
            else if (i < 2 * SB + 2 * SA) a = empty_a(i - 2 * SB - SA);
            else a = acc_bar;
            mbar_init_count(a, count);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        if (threadIdx.x == 64) {
            *abort_flag = 0;
            asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB))
                         : "memory");
        }
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();  // every barrier initialised, TMEM allocated
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- MMA issuer (one thread)
        if (lane == 0) {
            bool ok = true;
            int sa = 0, sb = 0;
            uint32_t pa = 0, pb = 0;  // phases of the current A and B slots
            for (int kb = 0; kb < nkb; ++kb) {
                if (!mbar_wait(full_a(sa), pa) || !mbar_wait(full_b(sb), pb) || *abort_flag) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                // descriptors of the stage: the 16 MMAs step through them by
                // constant offsets of the start-address field
                const uint64_t bd0 = sdesc(b_s + (uint32_t)(sb * NT * BK));
                const uint32_t ad0 = tmem + kACol + (uint32_t)(BK / 4) * sa;
#pragma unroll
                for (int k = 0; k < BK / 32; ++k)
                    mma_ts<NT>(tmem, ad0 + 8u * k,
                               bd0 + (uint64_t)(((k >> 2) * NT * 128 + 32 * (k & 3)) >> 4),
                               (kb | k) != 0 ? 1u : 0u);
                mma_commit(empty_a(sa));
                mma_commit(empty_b(sb));
                if (++sa == SA) { sa = 0; pa ^= 1u; }
                if (++sb == SB) { sb = 0; pb ^= 1u; }
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // arrives once every MMA issued above has completed; this thread
            // also waits for it, so no MMA is in flight when TMEM is freed
            mma_commit(acc_bar);
            if (!mbar_wait_sleep(acc_bar, 0)) report_status(p.status, HBL_ERR_TIMEOUT);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ---------------- TMA producer of the token stages (one thread).  Only
        // this warp waits for the previous kernel, whose output the codes are:
        // the converters unpack the first stages' weights meanwhile, and all
        // that reads the codes, scales or row sums is ordered after these
        // loads (MMAs after "full", the epilogue after the accumulator).
        pdl_wait();
        if (!p.early_weights) load_weights();
        if (lane == 0) {
            bool ok = true;
            int issued = 0;
            for (int kb = 0; kb < nkb; ++kb) {
                const int s = kb % SB;
                if (kb >= SB && !mbar_wait_sleep(empty_b(s), (uint32_t)(((kb / SB) - 1) & 1))) {
                    ok = false;
                    break;
                }
                if (*abort_flag) {
                    ok = false;
                    break;
                }
                mbar_expect_tx(full_b(s), (uint32_t)(NT * BK));
#pragma unroll
                for (int j = 0; j < kSub; ++j)
                    tma_load(b_s + (uint32_t)(s * NT * BK + j * NT * 128), &tmB,
                             k0 + kb * BK + 128 * j, 0, full_b(s));
                ++issued;
            }
            if (!ok) {
                *abort_flag = 1;
                report_status(p.status, HBL_ERR_TIMEOUT);
            }
            // every load issued lands before the CTA may move on
            for (int j = issued > SB ? issued - SB : 0; j < issued; ++j)
                if (!mbar_wait_sleep(full_b(j % SB), (uint32_t)((j / SB) & 1))) break;
        }
        __syncwarp();
    } else {
        // ---------------- converters: kConvGroups groups of four warps; group g
        // takes the stages kb = g (mod kConvGroups), each thread one weight row
        // (its TMEM lane) of the stage: two 16-byte reads, 32 words, one store
        const int cw = warp - 2;
        const int q = warp & 3;  // the TMEM lane quarter this warp may access
        const int grp = cw >> 2;
        const int r = 32 * q + lane;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        bool ok = true;
        for (int kb = grp; kb < nkb; kb += kConvGroups) {
            if (!warp_wait(wbar(kb), 0) ||
                (kb >= SA && !warp_wait(empty_a(kb % SA), (uint32_t)(((kb / SA) - 1) & 1))) ||
                __shfl_sync(0xffffffffu, *abort_flag, 0) != 0) {
                ok = false;
                break;
            }
            tc_fence_after();
            // row r's 128 bytes (512 weights) of stage kb: the row's line in box
            // kb, 16-byte chunk c at c ^ (r % 8); sub-tile j = chunks 2j, 2j + 1
            const uint32_t line = w_s + (uint32_t)(kb * kBoxBytes + r * 128);
#pragma unroll
            for (int j = 0; j < kSub; ++j) {
                const uint4 w0 = lds128(line + (((uint32_t)(2 * j) ^ (uint32_t)(r & 7)) << 4));
                const uint4 w1 = lds128(line + (((uint32_t)(2 * j + 1) ^ (uint32_t)(r & 7)) << 4));
                const uint32_t wv[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
                uint32_t v[32];
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    v[4 * e + 0] = wv[e] & 0x03030303u;
                    v[4 * e + 1] = (wv[e] >> 2) & 0x03030303u;
                    v[4 * e + 2] = (wv[e] >> 4) & 0x03030303u;
                    v[4 * e + 3] = (wv[e] >> 6) & 0x03030303u;
                }
                tmem_st32(tmem + lane_base + kACol + (uint32_t)(BK / 4) * (uint32_t)(kb % SA) +
                              32u * j,
                          v);
            }
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive_one(full_a(kb % SA));
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_status(p.status, HBL_ERR_TIMEOUT);
        }
        // every weight copy has landed before its bytes are reused (bounded)
        for (int g = 0; g < p.G; ++g)
            if (!warp_wait(wbar(g), 0)) break;
        const bool ready = warp_wait(acc_bar, 0);
        if (!ready && lane == 0) report_status(p.status, HBL_ERR_TIMEOUT);
        tc_fence_after();
        const bool aborted = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
        if (ready && !aborted && cw < 8) {  // the first two groups drain D
            const int h = cw >> 2;
            // partials [NT][128] int32 over the (consumed) weight rows
            int32_t* part = reinterpret_cast<int32_t*>(base);
            constexpr int HC = NT / 2;  // columns (tokens) of this warp
            const uint32_t taddr = tmem + lane_base + (uint32_t)(HC * h);
#pragma unroll
            for (int c0 = 0; c0 < HC; c0 += 8) {
                uint32_t d[8];
                tmem_ld8(taddr + (uint32_t)c0, d);
                asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
                for (int e = 0; e < 8; ++e) part[(HC * h + c0 + e) * kRows + r] = (int32_t)d[e];
            }
        }
    }
    // ---- reduction over the cluster: CTA c sums rows [c RC, (c + 1) RC)
    tc_fence_before();
    __syncwarp();
    cluster_sync_all();
    {
        const int RC = kRows / (int)csize;
        const int quads = RC / 4;
        const float alpha = *p.alpha;
        const uint32_t part_s = w_s;
        for (int it = threadIdx.x; it < p.M * quads; it += kThreads) {
            const int j = it / quads;
            const int r = (int)crank * RC + 4 * (it % quads);
            const int n = n0 + r;
            if (n >= p.N) continue;
            const uint32_t off = part_s + (uint32_t)((j * kRows + r) * 4);
            // the cluster's partials: all remote loads in flight, then the sums
            constexpr int kMaxCS = 8;
            uint4 v[kMaxCS];
#pragma unroll
            for (int c = 0; c < kMaxCS; ++c)
                if (c < (int)csize) v[c] = ld_cluster_v4(mapa(off, (uint32_t)c));
            int a0 = 0, a1 = 0, a2 = 0, a3 = 0;
#pragma unroll
            for (int c = 0; c < kMaxCS; ++c)
                if (c < (int)csize) {
                    a0 += (int)v[c].x;
                    a1 += (int)v[c].y;
                    a2 += (int)v[c].z;
                    a3 += (int)v[c].w;
                }
            const int rs = p.rowsum[j];
            a0 -= rs;
            a1 -= rs;
            a2 -= rs;
            a3 -= rs;
            const float sc = __fmul_rn(alpha, p.scales[j]);
            const uint32_t y01 =
                (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a0, sc))) |
                ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a1, sc)))
                 << 16);
            const uint32_t y23 =
                (uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a2, sc))) |
                ((uint32_t)__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn((float)a3, sc)))
                 << 16);
            *reinterpret_cast<uint2*>(p.Y + (int64_t)j * p.N + n) = make_uint2(y01, y23);
            if (p.acc_out != nullptr)
                *reinterpret_cast<int4*>(p.acc_out + (int64_t)j * p.N + n) = make_int4(a0, a1, a2, a3);
        }
    }
    // peers have finished reading this CTA's partials
    __syncwarp();
    cluster_sync_all();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
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

// Codes [M x K] bytes, box (128 bytes x NT rows), 128-byte swizzle; rows past M
// read as zeros.
static bool make_codes_map(CUtensorMap* map, const void* codes, int M, int K, int NT) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K};
    const cuuint32_t box[2] = {128u, (cuuint32_t)NT};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(codes), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Packed weights as bytes [N x K/4], box (inner bytes x 128 rows): the
// 128-byte swizzle when inner is 128, else no swizzle; rows past N read as zeros.
static bool make_weight_map(CUtensorMap* map, const uint32_t* W, int N, int K, int inner, bool sw) {
    auto fn = encode_fn();
    if (fn == nullptr) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)(K / 4), (cuuint64_t)N};
    const cuuint64_t strides[1] = {(cuuint64_t)(K / 4)};
    const cuuint32_t box[2] = {(cuuint32_t)inner, (cuuint32_t)kRows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint32_t*>(W), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
              sw ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_NONE,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

struct Plan {
    int NT, CS, Kc, G, sw, smem, SA, SB;
    uint32_t b_off, bar_off;
};

static int nt_for(int M) { return M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128; }

constexpr int kBarBytes = 8 * (2 * kMaxSB + 2 * kMaxSA + kMaxGroups + 1) + 16;

// Shared memory of a plan: the weights (or the partial sums, whichever is
// larger), then as deep a B ring as fits `budget` bytes (all of the CTA's B
// when it fits), then the barriers.  0 if not even two B stages fit.
static int smem_for(int NT, int Kc, int budget, int* SB, uint32_t* b_off, uint32_t* bar_off) {
    const int wbytes = kRows * Kc / 4;
    const int pbytes = NT * kRows * 4;
    const int region0 = ((wbytes > pbytes ? wbytes : pbytes) + 1023) & ~1023;
    const int stage = NT * BK;
    const int nkb = Kc / BK;
    int sb = (budget - region0 - kBarBytes - 1024) / stage;
    if (sb > nkb) sb = nkb;
    if (sb > kMaxSB) sb = kMaxSB;
    if (sb < 2 && sb < nkb) return 0;
    *SB = sb;
    *b_off = (uint32_t)region0;
    *bar_off = (uint32_t)(region0 + sb * stage);
    const int total = region0 + sb * stage + kBarBytes + 1024;
    return total < kMinSmem ? kMinSmem : total;
}

template <int NT>
static int max_active_clusters(int CS, int smem) {
    // cached per (cluster size, shared memory) for this instantiation
    static std::mutex mu;
    static int cache[4][8] = {};  // [log2 CS][smem bucket] -> clusters + 1
    int lcs = CS == 1 ? 0 : CS == 2 ? 1 : CS == 4 ? 2 : 3;
    int bucket = smem / (32 * 1024);
    if (bucket > 7) bucket = 7;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[lcs][bucket] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(CS, 1, 1);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = smem;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = CS;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, decode_mma_kernel<NT>, &cfg) != cudaSuccess) {
            cudaGetLastError();
            n = 0;
        }
        cache[lcs][bucket] = n + 1;
    }
    return cache[lcs][bucket] - 1;
}

template <int NT>
static bool plan_for(int M, int K, int N, int sms, int optin, Plan* pl) {
    const int RB = (N + kRows - 1) / kRows;
    for (int CS = 8; CS >= 1; CS /= 2) {
        if (CS > 1 && RB * CS > sms) continue;
        const int Kc = K / CS;
        if (Kc < BK || K % CS != 0) continue;
        const int sw = Kc >= 512 ? 1 : 0;
        const int G = sw ? Kc / 512 : 1;
        if (G > kMaxGroups) continue;
        uint32_t b_off, bar_off;
        int SB = 0;
        const int smem = smem_for(NT, Kc, optin, &SB, &b_off, &bar_off);
        if (smem == 0 || smem > optin) continue;
        if (!smem_attr_once(reinterpret_cast<const void*>(decode_mma_kernel<NT>), smem)) return false;
        if (CS > 1 && max_active_clusters<NT>(CS, smem) < RB) continue;
        const int SA = kMaxSA < Kc / BK ? kMaxSA : Kc / BK;
        *pl = Plan{NT, CS, Kc, G, sw, smem, SA, SB, b_off, bar_off};
        return true;
    }
    return false;
}

template <int NT>
static hbl_status launch_nt(const GemmArgs& a, cudaStream_t stream, int sms, int optin) {
    Plan pl;
    if (!plan_for<NT>((int)a.M, a.K, a.N, sms, optin, &pl)) return HBL_ERR_SHAPE;
    CUtensorMap map, wmap;
    if (!make_codes_map(&map, a.codes, (int)a.M, a.K, NT) ||
        !make_weight_map(&wmap, a.W_packed, a.N, a.K, pl.sw ? 128 : pl.Kc / 4, pl.sw != 0))
        return HBL_ERR_CUDA;
    Params p;
    p.M = (int)a.M;
    p.K = a.K;
    p.N = a.N;
    p.Kc = pl.Kc;
    p.G = pl.G;
    p.sw = pl.sw;
    p.SA = pl.SA;
    p.SB = pl.SB;
    p.b_off = pl.b_off;
    p.bar_off = pl.bar_off;
    p.W = a.W_packed;
    p.scales = a.scales;
    p.rowsum = a.rowsum;
    p.alpha = a.alpha;
    p.Y = a.Y;
    p.acc_out = a.acc_out;
    p.status = a.dev_status;
    p.early_weights = a.pdl ? 1 : 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pl.CS, (a.N + kRows - 1) / kRows, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.dynamicSmemBytes = pl.smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = pl.CS;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, decode_mma_kernel<NT>, map, wmap, p) == cudaSuccess
               ? HBL_OK
               : HBL_ERR_CUDA;
}

static int optin_smem() {
    int dev = 0, optin = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess)
        return 0;
    return optin;
}

}  // namespace k7

int decode_mma_max_m() { return 128; }

bool decode_mma_supported(int64_t M, int K, int N, int num_sms) {
    if (M < 1 || M > decode_mma_max_m() || K < k7::BK || N < 16) return false;
    const int optin = k7::optin_smem();
    if (optin <= 0) return false;
    k7::Plan pl;
    switch (k7::nt_for((int)M)) {
        case 16: return k7::plan_for<16>((int)M, K, N, num_sms, optin, &pl);
        case 32: return k7::plan_for<32>((int)M, K, N, num_sms, optin, &pl);
        case 64: return k7::plan_for<64>((int)M, K, N, num_sms, optin, &pl);
        default: return k7::plan_for<128>((int)M, K, N, num_sms, optin, &pl);
    }
}

hbl_status launch_decode_mma(const GemmArgs& a, cudaStream_t stream, int num_sms) {
    if (a.M == 0) return HBL_OK;
    if (a.M > decode_mma_max_m()) return HBL_ERR_SHAPE;
    const int optin = k7::optin_smem();
    switch (k7::nt_for((int)a.M)) {
        case 16: return k7::launch_nt<16>(a, stream, num_sms, optin);
        case 32: return k7::launch_nt<32>(a, stream, num_sms, optin);
        case 64: return k7::launch_nt<64>(a, stream, num_sms, optin);
        default: return k7::launch_nt<128>(a, stream, num_sms, optin);
    }
}

}  // namespace hbl
