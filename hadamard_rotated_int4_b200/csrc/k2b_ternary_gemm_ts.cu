// k2b_ternary_gemm_ts.cu -- ternary-weight GEMM on the sm_100a tensor cores
// with the activation operand in tensor memory (tcgen05.mma kind::i8, A from
// TMEM, B from shared memory, int32 accumulators in TMEM).
//
// Computes, as the BitNet v2 write-up (0755model.com, section "H-BitLinear")
// describes the layer after quantisation,
//   acc[m][n] = sum_k q[m][k] * t[n][k],   Y = bf16_rne((float)acc * (alpha * s[m])).
// Weights enter as the unsigned stored code c = t + 1 in {0, 1, 2}; the
// epilogue subtracts rowsum[m] = sum_k q[m][k] (exact integer arithmetic).
//
// CTA tile: 256 tokens x 128 weight rows, K in stages of 128 bytes, 4 stages.
// The 256 tokens are two accumulators of 128 rows (TMEM lanes) that share each
// weight tile, so a weight tile written once to shared memory feeds two MMAs:
// per stage the tensor core reads 2 x 16 KB of weights from shared memory and
// nothing else (activations come from TMEM).
//   TMEM (512 columns): D_a = [128 a, 128 a + 128) for a = 0, 1;
//                       A(s, a) = 256 + 32 (2 s + a), 32 columns (128 int8 per lane).
// Warp 0 allocates TMEM and one lane issues the MMAs and tcgen05.commit.
// Warps 1..8 convert: each thread owns one token row (its TMEM lane) and one
// 16-byte chunk of packed weights per stage; it loads its row's codes (int8, or
// int4 widened to int8) into registers and writes them to TMEM with
// tcgen05.st, unpacks its weight chunk ((w >> 2m) & 0x03030303 gives the codes
// of weights 4m..4m+3 as bytes) into the 128-byte-swizzled K-major tile, then
// signals the stage.  The same warps run the epilogue.  All waits are bounded
// by the global timer and warp-uniform; on expiry the kernel records
// HBL_ERR_TIMEOUT, stops, waits (bounded) for its own MMAs and frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k2b {

constexpr int BM = 256;  // tokens per CTA (2 accumulators x 128 TMEM lanes)
constexpr int BN = 128;  // weight rows per CTA (MMA N)
constexpr int BK = 128;  // K bytes per stage
constexpr int S = 4;     // pipeline stages
constexpr int kConvWarps = 8;
constexpr int kThreads = 32 * (1 + kConvWarps);
constexpr uint32_t kTmemCols = 512;
constexpr int kBStageBytes = BN * BK;  // 16 KB
constexpr int kSmemBytes = S * kBStageBytes + 256 + 1024;
constexpr uint64_t kTimeoutNs = 2000000000ull;

// mbarrier helpers over the library's bounded wait (kTimeoutNs of global time)
__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) { mbar_init_count(a, count); }
__device__ __forceinline__ void mbar_arrive(uint32_t a) { mbar_arrive_one(a); }
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<false>(a, parity, kTimeoutNs);
}
// Backs off with a short sleep between polls, so a waiting lane does not take
// issue slots from the warps that share its scheduler.
__device__ __forceinline__ bool mbar_wait_backoff(uint32_t a, uint32_t parity) {
    return mbar_wait_bounded<true>(a, parity, kTimeoutNs);
}
// Warp-uniform bounded wait: lane 0 waits, every lane gets its verdict.
template <bool BACKOFF = false>
__device__ __forceinline__ bool warp_wait(uint32_t a, uint32_t parity) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = BACKOFF ? mbar_wait_backoff(a, parity) : mbar_wait(a, parity);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
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
// kind::i8, D s32, A s8 (from TMEM, K-major), B u8 (K-major), M = 128, N = BN.
constexpr uint32_t kIdesc =
    (2u << 4) | (1u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);

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

__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

// 8 signed nibbles (element 2i low) -> 8 int8 in two words, natural order.
__device__ __forceinline__ uint2 widen_nibbles(uint32_t w) {
    uint32_t lo = ((w & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    uint32_t hi = (((w >> 4) & 0x0F0F0F0Fu) ^ 0x08080808u) + 0x78787878u;
    lo ^= 0x80808080u;
    hi ^= 0x80808080u;
    return make_uint2(__byte_perm(lo, hi, 0x5140), __byte_perm(lo, hi, 0x7362));
}

struct Params {
    const uint8_t* codes;
    const float* scales;
    const int32_t* rowsum;
    int64_t M;
    int K;
    const uint32_t* W;
    const float* alpha;
    int N;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* status;
    int32_t* part;  // split-K: raw int32 partials [gridDim.z][M][N] (null: full epilogue)
    int kps;        // K-blocks per split
};

template <int ABITS>
struct Packed {
    static constexpr int kA = ABITS == 8 ? 8 : 4;  // 16-byte chunks of this row per stage
    uint4 a[kA];
    uint4 b;
    uint4 b2;  // second 16-byte weight chunk (HALF: each thread owns a whole 128-weight row piece)
};

// Per-thread constants of the converter loop.
struct ConvPtrs {
    const uint8_t* a;      // this row's codes at K offset 0 (null: row absent)
    const uint32_t* b;     // this thread's weight row at word 0 (null: row absent)
    int bh;                // which 64-weight half of the stage's 128 weights
};

// IL: codes one per byte in the 32-row interleaved layout (16-code chunk c of
// row m at (((m/32)*(K/16) + c)*32 + m%32)*16): a warp's 32 rows read 512
// contiguous bytes per chunk.  Otherwise row-major codes (int8 or packed int4).
template <int ABITS, bool IL>
__device__ __forceinline__ void load_stage(const ConvPtrs& cp, int K, int kb, Packed<ABITS>& P) {
    const int kbase = kb * BK;
    const int kleft = K - kbase;  // > 0; < BK only when K < 128
    if constexpr (ABITS == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (cp.a != nullptr && 16 * i < kleft) {
                const uint8_t* src = IL ? cp.a + ((int64_t)(kb * 8 + i) << 9) : cp.a + kbase + 16 * i;
                v = *reinterpret_cast<const uint4*>(src);
            }
            P.a[i] = v;
        }
    } else {
        const uint8_t* src = cp.a + kbase / 2;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            uint4 v = make_uint4(0, 0, 0, 0);
            if (cp.a != nullptr && 32 * i < kleft) {
                if (32 * i + 32 <= kleft) {
                    v = *reinterpret_cast<const uint4*>(src + 16 * i);
                } else {  // 16 elements left (K == 16)
                    const uint2 hv = *reinterpret_cast<const uint2*>(src + 16 * i);
                    v = make_uint4(hv.x, hv.y, 0u, 0u);
                }
            }
            P.a[i] = v;
        }
    }
    uint4 b = make_uint4(0, 0, 0, 0);
    const int kk = 64 * cp.bh;
    if (cp.b != nullptr && kk < kleft) {
        const uint32_t* src = cp.b + (kbase + kk) / 16;
        if (kk + 64 <= kleft) {
            b = *reinterpret_cast<const uint4*>(src);
        } else {  // fewer than 4 words left in this row (K < 128)
            const int nw = (kleft - kk) / 16;
            b.x = src[0];
            if (nw > 1) b.y = src[1];
            if (nw > 2) b.z = src[2];
        }
    }
    P.b = b;
}

// Loader for K % 128 == 0: no guards (rows past M or N read a valid row whose
// results are never stored), running pointers, immediate offsets.
// a_on = false (warp-uniform): this warp's token rows are all past M, so its
// activation loads are skipped (the MMA rows they would feed are never stored).
template <int ABITS, bool IL, bool TWO = false>
struct FastLoader {
    const uint8_t* a;
    const uint32_t* b;
    bool a_on;
    __device__ __forceinline__ void load(Packed<ABITS>& P) {
        if (a_on) {
            if constexpr (ABITS == 8) {
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    P.a[i] = *reinterpret_cast<const uint4*>(a + (IL ? 512 * i : 16 * i));
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) P.a[i] = *reinterpret_cast<const uint4*>(a + 16 * i);
            }
        }
        a += ABITS == 8 ? (IL ? 8 * 512 : BK) : BK / 2;
        P.b = *reinterpret_cast<const uint4*>(b);
        if constexpr (TWO) P.b2 = *reinterpret_cast<const uint4*>(b + 4);
        b += BK / 16;
    }
};

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

template <int ABITS, bool TWO = false>
__device__ __forceinline__ void store_stage(uint32_t a_taddr, uint32_t sB, const uint32_t (&boff)[4],
                                            const uint32_t (&boff2)[4], const Packed<ABITS>& P,
                                            bool a_on) {
    uint32_t av[32];
    if constexpr (ABITS == 8) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            av[4 * i] = P.a[i].x;
            av[4 * i + 1] = P.a[i].y;
            av[4 * i + 2] = P.a[i].z;
            av[4 * i + 3] = P.a[i].w;
        }
    } else {
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const uint32_t w4[4] = {P.a[i].x, P.a[i].y, P.a[i].z, P.a[i].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const uint2 x = widen_nibbles(w4[j]);
                av[8 * i + 2 * j] = x.x;
                av[8 * i + 2 * j + 1] = x.y;
            }
        }
    }
    if (a_on) tmem_st32(a_taddr, av);  // warp-uniform
    const uint32_t wv[4] = {P.b.x, P.b.y, P.b.z, P.b.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const uint32_t w = wv[j];
        sts128(sB + boff[j],
               make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                          (w >> 6) & 0x03030303u));
    }
    if constexpr (TWO) {
        const uint32_t wv2[4] = {P.b2.x, P.b2.y, P.b2.z, P.b2.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const uint32_t w = wv2[j];
            sts128(sB + boff2[j],
                   make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                              (w >> 6) & 0x03030303u));
        }
    }
}

// SMALL: a single tile of tokens (M <= 256, decode batches): split-K over
// grid.z, one accumulator when M <= 128, and the weights prefetched into L2
// before the dependency wait.  The large-M instantiation keeps none of these.
// HALF (SMALL, M <= 128, K % 128 == 0): only the four converter warps of the
// one accumulator run; each thread converts a whole 32-byte piece of its
// weight row per stage, so the per-stage synchronisation is paid by half as
// many warps.
template <int ABITS, bool IL, bool FULLK, bool SMALL, bool HALF = false>
__global__ void __launch_bounds__(kThreads, 1) gemm_ts_kernel(Params p) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t bar_s = base_s + S * kBStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * kBStageBytes);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto full_bar = [&](int s) { return bar_s + 8u * s; };
    auto empty_bar = [&](int s) { return bar_s + 8u * (S + s); };
    const uint32_t acc_bar = bar_s + 8u * (2 * S);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * BN;
    const int64_t m0 = (int64_t)blockIdx.y * BM;
    // this CTA's K-blocks: [kb0, kb0 + num_kb) of the whole K (split-K over grid.z)
    const int num_kb_total = (p.K + BK - 1) / BK;
    const int kb0 = SMALL ? (int)blockIdx.z * p.kps : 0;
    const int num_kb = SMALL ? min(p.kps, num_kb_total - kb0) : num_kb_total;
    // rows of this tile that exist: one accumulator suffices when M - m0 <= 128
    const int nacc = HALF ? 1 : ((!SMALL || p.M - m0 > 128) ? 2 : 1);

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), HALF ? kConvWarps / 2 : kConvWarps);  // one per converter warp
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    // Packed weights of this CTA into L2 while the previous kernel finishes
    // (a hint: it reads nothing into registers), then wait for its outputs.
    // (K >= 64 keeps every row start and length a multiple of 16 bytes.)
    if (SMALL && tid >= 32 && tid < 32 + BN && p.K >= 64 && num_kb > 0) {
        const int n = n0 + tid - 32;
        if (n < p.N) {
            const int k_lo = kb0 * BK, k_hi = min((kb0 + num_kb) * BK, p.K);
            prefetch_l2_bulk(p.W + (int64_t)n * (p.K / 16) + k_lo / 16, (uint32_t)(k_hi - k_lo) / 4);
        }
    }
    pdl_wait();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- MMA issuer
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % S;
            if (!warp_wait<true>(full_bar(s), (uint32_t)((kb / S) & 1))) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sB = base_s + s * kBStageBytes;
#pragma unroll
                for (int k = 0; k < BK / 32; ++k) {
                    const uint64_t bd = sdesc(sB + 32 * k);
#pragma unroll
                    for (int a = 0; a < 2; ++a)
                        if (a < nacc)
                            mma_ts(tmem + 128u * a, tmem + 256u + 32u * (2 * s + a) + 8u * k, bd,
                               (kb > 0 || k > 0) ? 1u : 0u);
                }
                mma_commit(empty_bar(s));
            }
            __syncwarp();
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_status(p.status, HBL_ERR_TIMEOUT);
        }
        if (lane == 0) mma_commit(acc_bar);
        __syncwarp();
        if (!warp_wait(acc_bar, 0) && lane == 0) report_status(p.status, HBL_ERR_TIMEOUT);
    } else if (HALF && warp > kConvWarps / 2) {
        // ---------------- HALF: the second accumulator's warps have nothing to do
    } else {
        // ---------------- converters, then epilogue
        const int ct = tid - 32;                 // 0..255
        const int q = warp & 3;                  // TMEM lane quarter of this warp
        const int acc = (warp - 1) >> 2;         // accumulator 0 or 1
        const int trow = 128 * acc + 32 * q + lane;  // token row within the tile
        const int64_t m = m0 + trow;
        // one-tile batches: warps whose 32 rows all lie past M skip their
        // activation loads and TMEM stores (warp-uniform)
        const bool a_on = !SMALL || (m0 + 128 * acc + 32 * q < p.M);
        // weight row / half of this thread's 16-byte chunk (HALF: both halves)
        const int br = HALF ? ct : (ct >> 1), bh = HALF ? 0 : (ct & 1);
        const int n = n0 + br;
        const uint32_t lane_base = (uint32_t)(32 * q) << 16;
        ConvPtrs cp;
        if constexpr (IL) {
            const int64_t mpad = (p.M + 31) & ~(int64_t)31;
            cp.a = (m < mpad) ? p.codes + (((m >> 5) * (int64_t)(p.K >> 4)) << 9) + ((m & 31) << 4)
                              : nullptr;
        } else {
            cp.a = (m < p.M) ? p.codes + m * (int64_t)(ABITS == 8 ? p.K : p.K / 2) : nullptr;
        }
        cp.b = (n < p.N) ? p.W + (int64_t)n * (p.K / 16) : nullptr;
        cp.bh = bh;
        uint32_t boff[4], boff2[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            boff[j] = sw128(br, 4 * bh + j);
            boff2[j] = sw128(br, 4 + j);
        }
        const uint32_t a_col0 = tmem + lane_base + 256u + 32u * acc;

        // one stage: wait for the slot, write A to TMEM and B to shared memory, signal
        auto stage = [&](int kb, const Packed<ABITS>& P) -> bool {
            const int s = kb % S;
            bool go = true;
            if (kb >= S) go = warp_wait<true>(empty_bar(s), (uint32_t)(((kb / S) - 1) & 1));
            go = go && (__shfl_sync(0xffffffffu, *abort_flag, 0) == 0);
            if (!go) return false;  // warp-uniform
            tc_fence_after();
            store_stage<ABITS, HALF>(a_col0 + 64u * s, base_s + s * kBStageBytes, boff, boff2, P,
                                     a_on);
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
            tc_fence_before();
            __syncwarp();  // the warp's shared and TMEM writes are ordered before lane 0's arrive
            if (lane == 0) mbar_arrive(full_bar(s));
            return true;
        };
        Packed<ABITS> P0, P1;
        bool ok = true;
        if constexpr (FULLK) {
            FastLoader<ABITS, IL, HALF> ld;
            ld.a_on = a_on;
            {
                int64_t mm = m;
                if constexpr (IL) {
                    const int64_t mpad = (p.M + 31) & ~(int64_t)31;
                    if (mm >= mpad) mm = mpad - 1;
                    ld.a = p.codes + (((mm >> 5) * (int64_t)(p.K >> 4)) << 9) + ((mm & 31) << 4);
                } else {
                    if (mm >= p.M) mm = p.M - 1;
                    ld.a = p.codes + mm * (int64_t)(ABITS == 8 ? p.K : p.K / 2);
                }
                const int nn = n < p.N ? n : p.N - 1;
                ld.b = p.W + (int64_t)nn * (p.K / 16) + 4 * bh;
                if constexpr (SMALL) {
                    ld.a += (int64_t)kb0 * (IL ? 8 * 512 : (ABITS == 8 ? BK : BK / 2));
                    ld.b += kb0 * (BK / 16);
                }
            }
            // three stages of operands in flight in registers
            Packed<ABITS> P2;
            ld.load(P0);
            if (num_kb > 1) ld.load(P1);
            if (num_kb > 2) ld.load(P2);
            for (int kb = 0; kb < num_kb; kb += 3) {
                if (!stage(kb, P0)) {
                    ok = false;
                    break;
                }
                if (kb + 3 < num_kb) ld.load(P0);
                if (kb + 1 >= num_kb) break;
                if (!stage(kb + 1, P1)) {
                    ok = false;
                    break;
                }
                if (kb + 4 < num_kb) ld.load(P1);
                if (kb + 2 >= num_kb) break;
                if (!stage(kb + 2, P2)) {
                    ok = false;
                    break;
                }
                if (kb + 5 < num_kb) ld.load(P2);
            }
        } else {
            load_stage<ABITS, IL>(cp, p.K, kb0, P0);
            for (int kb = 0; kb < num_kb; kb += 2) {
                if (kb + 1 < num_kb) load_stage<ABITS, IL>(cp, p.K, kb0 + kb + 1, P1);
                if (!stage(kb, P0)) {
                    ok = false;
                    break;
                }
                if (kb + 1 >= num_kb) break;
                if (kb + 2 < num_kb) load_stage<ABITS, IL>(cp, p.K, kb0 + kb + 2, P0);
                if (!stage(kb + 1, P1)) {
                    ok = false;
                    break;
                }
            }
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_status(p.status, HBL_ERR_TIMEOUT);
        }
        const bool ready = warp_wait(acc_bar, 0);
        if (!ready && lane == 0) report_status(p.status, HBL_ERR_TIMEOUT);
        tc_fence_after();
        const bool aborted = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
        if (ready && !aborted) {
            const bool mok = m < p.M;
            const float sc = mok ? __fmul_rn(*p.alpha, p.scales[m]) : 0.f;
            const int rs = mok ? p.rowsum[m] : 0;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                const uint32_t taddr = tmem + lane_base + 128u * acc + (uint32_t)(32 * cc);
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
                const int nc = n0 + 32 * cc;
                if (SMALL && p.part != nullptr) {  // split-K: raw partial sums, reduced by a second kernel
                    if (mok && nc < p.N) {
                        int4* pd = reinterpret_cast<int4*>(
                            p.part + ((int64_t)blockIdx.z * p.M + m) * p.N + nc);
                        const int nq = (p.N - nc) >= 32 ? 8 : 4;
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (e < nq)
                                pd[e] = make_int4((int)v[4 * e], (int)v[4 * e + 1], (int)v[4 * e + 2],
                                                  (int)v[4 * e + 3]);
                    }
                    continue;
                }
                if (mok && nc < p.N) {
                    uint32_t out[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const int a0 = (int)v[2 * e] - rs, a1 = (int)v[2 * e + 1] - rs;
                        const float y0 = __fmul_rn((float)a0, sc), y1 = __fmul_rn((float)a1, sc);
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
                        const int nq = halves * 4;
#pragma unroll
                        for (int e = 0; e < 8; ++e)
                            if (e < nq)
                                ad[e] = make_int4((int)v[4 * e] - rs, (int)v[4 * e + 1] - rs,
                                                  (int)v[4 * e + 2] - rs, (int)v[4 * e + 3] - rs);
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

template <int ABITS, bool IL>
static hbl_status launch(const Params& prm, cudaStream_t stream) {
    const bool full = prm.K % BK == 0, small = prm.M <= BM, half = small && prm.M <= 128;
    auto kern = full ? (small ? (half ? gemm_ts_kernel<ABITS, IL, true, true, true>
                                      : gemm_ts_kernel<ABITS, IL, true, true>)
                              : gemm_ts_kernel<ABITS, IL, true, false>)
                     : (small ? gemm_ts_kernel<ABITS, IL, false, true>
                              : gemm_ts_kernel<ABITS, IL, false, false>);
    const int smem = kSmemBytes;
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), smem)) return HBL_ERR_CUDA;
    const int num_kb = (prm.K + BK - 1) / BK;
    dim3 grid((prm.N + BN - 1) / BN, (unsigned)((prm.M + BM - 1) / BM),
              (unsigned)((num_kb + prm.kps - 1) / prm.kps));
    return launch_pdl(kern, grid, dim3(kThreads), smem, stream, prm);
}

}  // namespace k2b

// Split factor over K for one-tile-high problems (M <= 256), so that a decode
// batch still fills the GPU in one wave (one CTA per SM: the kernel holds all
// of TMEM), at least 8 K-blocks per CTA.
int gemm_ts_ksplit(int64_t M, int K, int N) {
    if (M > k2b::BM) return 1;
    const int tiles = (N + k2b::BN - 1) / k2b::BN;
    const int num_kb = (K + k2b::BK - 1) / k2b::BK;
    int ks = 1;
    while (tiles * ks * 2 <= 148 && num_kb / (ks * 2) >= 8) ks *= 2;
    return ks;
}

size_t gemm_ts_workspace(int64_t M, int K, int N) {
    const int ks = gemm_ts_ksplit(M, K, N);
    return ks > 1 ? (((size_t)ks * (size_t)M * (size_t)N * 4 + 255) & ~(size_t)255) : 0;
}

hbl_status launch_gemm_ts(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                          int /*num_sms*/) {
    if (a.M == 0) return HBL_OK;
    const int ks = gemm_ts_ksplit(a.M, a.K, a.N);
    const int num_kb = (a.K + k2b::BK - 1) / k2b::BK;
    if (ks > 1 && (ws == nullptr || ws_bytes < gemm_ts_workspace(a.M, a.K, a.N)))
        return HBL_ERR_WORKSPACE;
    k2b::Params prm;
    prm.part = ks > 1 ? static_cast<int32_t*>(ws) : nullptr;
    prm.kps = (num_kb + ks - 1) / ks;
    prm.codes = static_cast<const uint8_t*>(a.codes);
    prm.scales = a.scales;
    prm.rowsum = a.rowsum;
    prm.M = a.M;
    prm.K = a.K;
    prm.W = a.W_packed;
    prm.alpha = a.alpha;
    prm.N = a.N;
    prm.Y = a.Y;
    prm.acc_out = a.acc_out;
    prm.status = a.dev_status;
    hbl_status st;
    if (a.interleaved)
        st = k2b::launch<8, true>(prm, stream);
    else if (a.act_bits == 4)
        st = k2b::launch<4, false>(prm, stream);
    else
        st = k2b::launch<8, false>(prm, stream);
    if (st != HBL_OK || ks == 1) return st;
    const int nsplit = (num_kb + prm.kps - 1) / prm.kps;  // grid.z: every split has K-blocks
    return launch_splitk_epilogue(prm.part, nsplit, a.M, a.N, a.rowsum, a.scales, a.alpha, a.Y,
                                  a.acc_out, stream);
}

}  // namespace hbl
