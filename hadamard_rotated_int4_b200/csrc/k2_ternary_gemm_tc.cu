// k2_ternary_gemm_tc.cu -- ternary-weight x int8/int4-activation GEMM on the
// sm_100a tensor cores (tcgen05.mma kind::i8, int32 accumulator in TMEM).
//
// BitNet v2 write-up (0755model.com), section "H-BitLinear": the quantised
// activations are multiplied by the ternary weights with an integer
// accumulator and the result is dequantised by alpha * s_x:
//   acc[m][n] = sum_k q[m][k] * t[n][k],   Y = bf16_rne((float)acc * (alpha * s[m])).
// The weights are fed to the MMA as unsigned bytes c = t + 1 in {0, 1, 2}
// (the stored 2-bit code), so the MMA computes sum q*c and the epilogue
// subtracts rowsum[m] = sum_k q[m][k]: exact integer arithmetic.
//
// CTA tile BM x BN (128 x 256 by default), K in stages of 128 bytes.  Warp 0
// allocates TMEM and one lane issues the MMAs (4 x K=32 per stage) and
// tcgen05.commit; warps 1..4 are converters: they read the packed operands
// from global memory (one stage of prefetch in registers), widen int4 codes to
// int8 and 2-bit weights to bytes, and store both into 128-byte-swizzled
// K-major shared-memory tiles (the UMMA SWIZZLE_128B layout).  The same warps
// run the epilogue (tcgen05.ld 32x32b, one TMEM lane quarter each).  Every
// mbarrier wait is bounded by the global timer; on expiry the kernel records
// HBL_ERR_TIMEOUT, stops issuing work, waits (bounded) for its own MMAs and
// frees its TMEM.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k2 {

constexpr int BM = 128;
constexpr int BK = 128;  // int8 elements (bytes) of K per stage
constexpr int kConvWarps = 4;
constexpr int kThreads = 32 * (1 + kConvWarps);
constexpr uint64_t kTimeoutNs = 2000000000ull;  // 2 s per wait

template <int BN>
struct Cfg {
    static constexpr int kStageBytes = (BM + BN) * BK;
    static constexpr int kStages = BN >= 256 ? 4 : (BN >= 128 ? 5 : 6);
    static constexpr int kTmemCols = BN < 32 ? 32 : BN;
    static constexpr int kBarBytes = 256;
    static constexpr int kSmemBytes = kStages * kStageBytes + kBarBytes + 1024;
};

__device__ __forceinline__ uint64_t gtime() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t a) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t a, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred p;\n"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        "selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity)
        : "memory");
    return ok != 0;
}
// Bounded wait; false on timeout.
__device__ __forceinline__ bool mbar_wait(uint32_t a, uint32_t parity) {
    if (mbar_try(a, parity)) return true;
    const uint64_t t0 = gtime();
    while (true) {
        if (mbar_try(a, parity)) return true;
        if (gtime() - t0 > kTimeoutNs) return false;
    }
}

// Warp-uniform bounded wait: lane 0 waits, every lane gets its verdict.
__device__ __forceinline__ bool warp_wait(uint32_t a, uint32_t parity) {
    bool ok = true;
    if ((threadIdx.x & 31) == 0) ok = mbar_wait(a, parity);
    return __shfl_sync(0xffffffffu, ok ? 1 : 0, 0) != 0;
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row atoms of
// 1024 bytes (SBO = 1024), descriptor version 1 (sm_100).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;             // leading byte offset (unused with 128B swizzle)
    d |= (uint64_t)(1024 >> 4) << 32;   // stride byte offset
    d |= (uint64_t)1 << 46;             // version
    d |= (uint64_t)2 << 61;             // SWIZZLE_128B
    return d;
}

// Instruction descriptor, kind::i8: D s32, A s8 (K-major), B u8 (K-major).
template <int BN>
__host__ __device__ constexpr uint32_t idesc_i8() {
    return (2u << 4) | (1u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) |
           ((uint32_t)(BM >> 4) << 24);
}

__device__ __forceinline__ void mma_i8(uint32_t tmem_d, uint64_t da, uint64_t db, uint32_t idesc,
                                       uint32_t accum) {
    asm volatile(
        "{\n.reg .pred p;\n"
        "setp.ne.b32 p, %4, 0;\n"
        "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem_d),
        "l"(da), "l"(db), "r"(idesc), "r"(accum)
        : "memory");
}
__device__ __forceinline__ void mma_commit(uint32_t mbar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar)
        : "memory");
}

// byte offset of 16-byte chunk c (0..7) of row r in a SWIZZLE_128B K-major tile
__device__ __forceinline__ uint32_t sw128(int r, int c) {
    return (uint32_t)((r >> 3) * 1024 + (r & 7) * 128 + ((c ^ (r & 7)) << 4));
}

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
};

// Packed operand data of one stage held by one converter thread.
template <int ABITS, int BN>
struct Packed {
    static constexpr int kAChunks = ABITS == 4 ? (BM * BK / 2) / 16 / 128 : (BM * BK) / 16 / 128;
    static constexpr int kBChunks = (BN * BK / 4) / 16 / 128;
    uint4 a[kAChunks];
    uint4 b[kBChunks];
};

template <int ABITS, int BN>
__device__ __forceinline__ void load_stage(const Params& p, int64_t m0, int n0, int kb, int ct,
                                           Packed<ABITS, BN>& P) {
    using PK = Packed<ABITS, BN>;
    const int kbase = kb * BK;
    const int kleft = p.K - kbase;  // > 0
#pragma unroll
    for (int i = 0; i < PK::kAChunks; ++i) {
        const int g = ct + 128 * i;
        uint4 v = make_uint4(0, 0, 0, 0);
        if constexpr (ABITS == 4) {
            const int r = g >> 2, cp = g & 3;  // 4 chunks of 32 nibbles per row
            const int64_t m = m0 + r;
            const int kk = cp * 32;            // first element of this chunk
            if (m < p.M && kk < kleft) {
                const uint8_t* src = p.codes + m * (int64_t)(p.K / 2) + (kbase + kk) / 2;
                if (kk + 32 <= kleft) {
                    v = *reinterpret_cast<const uint4*>(src);
                } else {  // 16 elements left (K == 16)
                    const uint2 h = *reinterpret_cast<const uint2*>(src);
                    v = make_uint4(h.x, h.y, 0u, 0u);  // missing elements: code 0
                }
            }
        } else {
            const int r = g >> 3, c = g & 7;
            const int64_t m = m0 + r;
            const int kk = c * 16;
            if (m < p.M && kk < kleft)
                v = *reinterpret_cast<const uint4*>(p.codes + m * (int64_t)p.K + kbase + kk);
        }
        P.a[i] = v;
    }
#pragma unroll
    for (int i = 0; i < PK::kBChunks; ++i) {
        const int g = ct + 128 * i;
        const int r = g >> 1, h = g & 1;  // 2 chunks (4 words each) per row
        const int n = n0 + r;
        const int kk = h * 64;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (n < p.N && kk < kleft) {
            const uint32_t* src = p.W + (int64_t)n * (p.K / 16) + (kbase + kk) / 16;
            if (kk + 64 <= kleft) {
                v = *reinterpret_cast<const uint4*>(src);
            } else {  // fewer than 4 words left in this row (K < 128)
                const int nw = (kleft - kk) / 16;
                v.x = src[0];
                if (nw > 1) v.y = src[1];
                if (nw > 2) v.z = src[2];
            }
        }
        P.b[i] = v;
    }
}

template <int ABITS, int BN>
__device__ __forceinline__ void store_stage(uint32_t sA, uint32_t sB, int ct,
                                            const Packed<ABITS, BN>& P) {
    using PK = Packed<ABITS, BN>;
#pragma unroll
    for (int i = 0; i < PK::kAChunks; ++i) {
        const int g = ct + 128 * i;
        if constexpr (ABITS == 4) {
            const int r = g >> 2, cp = g & 3;
            uint2 x0 = widen_nibbles(P.a[i].x), x1 = widen_nibbles(P.a[i].y);
            uint2 x2 = widen_nibbles(P.a[i].z), x3 = widen_nibbles(P.a[i].w);
            sts128(sA + sw128(r, 2 * cp), make_uint4(x0.x, x0.y, x1.x, x1.y));
            sts128(sA + sw128(r, 2 * cp + 1), make_uint4(x2.x, x2.y, x3.x, x3.y));
        } else {
            const int r = g >> 3, c = g & 7;
            sts128(sA + sw128(r, c), P.a[i]);
        }
    }
#pragma unroll
    for (int i = 0; i < PK::kBChunks; ++i) {
        const int g = ct + 128 * i;
        const int r = g >> 1, h = g & 1;
        const uint32_t wv[4] = {P.b[i].x, P.b[i].y, P.b[i].z, P.b[i].w};
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) {
            const uint32_t w = wv[jj];
            sts128(sB + sw128(r, 4 * h + jj),
                   make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u, (w >> 4) & 0x03030303u,
                              (w >> 6) & 0x03030303u));
        }
    }
}

template <int ABITS, int BN>
__global__ void __launch_bounds__(kThreads, 1) gemm_tc_kernel(Params p) {
    using C = Cfg<BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t bar_s = base_s + S * C::kStageBytes;
    uint64_t* bars = reinterpret_cast<uint64_t*>(base + S * C::kStageBytes);
    // bars[0..S) full, [S..2S) empty, [2S] accumulator ready; then tmem addr, abort flag
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
    auto full_bar = [&](int s) { return bar_s + 8u * s; };
    auto empty_bar = [&](int s) { return bar_s + 8u * (S + s); };
    const uint32_t acc_bar = bar_s + 8u * (2 * S);

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int n0 = blockIdx.x * BN;
    const int64_t m0 = (int64_t)blockIdx.y * BM;
    const int num_kb = (p.K + BK - 1) / BK;

    if (tid == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(full_bar(s), 32 * kConvWarps);
            mbar_init(empty_bar(s), 1);
        }
        mbar_init(acc_bar, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"((uint32_t)C::kTmemCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------- MMA issuer
        constexpr uint32_t idesc = idesc_i8<BN>();
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % S;
            const uint32_t par = (uint32_t)((kb / S) & 1);
            if (!warp_wait(full_bar(s), par)) {
                ok = false;
                break;
            }
            tc_fence_after();
            if (lane == 0) {
                const uint32_t sA = base_s + s * C::kStageBytes;
                const uint32_t sB = sA + BM * BK;
#pragma unroll
                for (int k = 0; k < BK / 32; ++k) {
                    mma_i8(tmem, sdesc(sA + 32 * k), sdesc(sB + 32 * k), idesc,
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
        if (lane == 0) mma_commit(acc_bar);  // fires once every issued MMA has completed
        __syncwarp();
        // wait for our own MMAs before the CTA may free TMEM
        if (!warp_wait(acc_bar, 0) && lane == 0) report_status(p.status, HBL_ERR_TIMEOUT);
    } else {
        // ---------------- converters, then epilogue
        const int ct = tid - 32;
        Packed<ABITS, BN> cur, nxt;
        load_stage<ABITS, BN>(p, m0, n0, 0, ct, cur);
        bool ok = true;
        for (int kb = 0; kb < num_kb; ++kb) {
            const int s = kb % S;
            if (kb + 1 < num_kb) load_stage<ABITS, BN>(p, m0, n0, kb + 1, ct, nxt);
            bool go = true;
            if (kb >= S) go = warp_wait(empty_bar(s), (uint32_t)(((kb / S) - 1) & 1));
            go = go && (__shfl_sync(0xffffffffu, *abort_flag, 0) == 0);
            if (!go) {  // warp-uniform
                ok = false;
                break;
            }
            const uint32_t sA = base_s + s * C::kStageBytes;
            store_stage<ABITS, BN>(sA, sA + BM * BK, ct, cur);
            fence_async_smem();
            mbar_arrive(full_bar(s));
            cur = nxt;
        }
        if (!ok && lane == 0) {
            *abort_flag = 1;
            report_status(p.status, HBL_ERR_TIMEOUT);
        }
        // epilogue: one TMEM lane quarter per warp
        const bool ready = warp_wait(acc_bar, 0);
        if (!ready && lane == 0) report_status(p.status, HBL_ERR_TIMEOUT);
        tc_fence_after();
        const bool aborted = __shfl_sync(0xffffffffu, *abort_flag, 0) != 0;
        if (ready && !aborted) {
            const int q = warp & 3;
            const int64_t m = m0 + 32 * q + lane;
            const bool mok = m < p.M;
            const float sc = mok ? __fmul_rn(*p.alpha, p.scales[m]) : 0.f;
            const int rs = mok ? p.rowsum[m] : 0;
#pragma unroll 1
            for (int cc = 0; cc < BN / 32; ++cc) {
                uint32_t v[32];
                const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + (uint32_t)(32 * cc);
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
                     "r"((uint32_t)C::kTmemCols)
                     : "memory");
    }
}

template <int ABITS, int BN>
static hbl_status launch(const Params& prm, cudaStream_t stream) {
    using C = Cfg<BN>;
    auto kern = gemm_tc_kernel<ABITS, BN>;
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), C::kSmemBytes)) return HBL_ERR_CUDA;
    dim3 grid((prm.N + BN - 1) / BN, (unsigned)((prm.M + BM - 1) / BM));
    kern<<<grid, kThreads, C::kSmemBytes, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace k2

hbl_status launch_gemm_tc(const GemmArgs& a, cudaStream_t stream, int /*num_sms*/) {
    if (a.M == 0) return HBL_OK;
    k2::Params prm;
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
    if (a.act_bits == 4) return k2::launch<4, 256>(prm, stream);
    return k2::launch<8, 256>(prm, stream);
}

}  // namespace hbl
