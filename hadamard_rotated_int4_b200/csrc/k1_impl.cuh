// k1_impl.cuh -- fused RMSNorm + online Walsh-Hadamard transform +
// per-token INT8 (absmax) / INT4 (absmean) quantisation, one token row per
// group of T threads, for sm_100a.
//
// What it computes (BitNet v2 write-up, 0755model.com, sections
// "BitNet v2：原生4位激活" and "H-BitLinear"; shengxinai.com section 2.2):
//   r = 1/sqrt(tree_sum(x*x) * (1/K) + norm_eps),  u = (x * r) * gain
//   v = (u . H_K) * c_K                        (butterflies h = 1, 2, ..., K/2)
//   INT8: q = clip(rhe(v * (127/(max|v| + eps))), -128, 127), scale = max|v|/127
//   INT4: beta = tree_sum(|v|) * (1/K), q = clip(rhe(v * (sqrt7/(beta+eps))), -8, 7),
//         scale = beta/sqrt7
// Every fp32 operation is a single IEEE round-to-nearest operation (no FMA
// contraction, explicit _rn intrinsics), the butterfly stages run in ascending
// order and every sum is the perfect pairwise tree over index order, so the
// codes are bit-identical to a scalar evaluation in that order.
//
// Thread mapping.  Each thread holds R = 128 fp32 values of its row (R = K for
// K < 128).  Index bits of the row are assigned to register bits and thread
// bits by a sequence of layouts:
//   N  (natural): register bits <-> index bits 0..6, thread bits <-> 7..L-1.
//      Stages 0..6 run in registers.
//   P_b (pass b): register bits <-> {0, 1} + stage bits [b, b+5) (+ the lowest
//      free bits when fewer than 5 stages remain), thread bits <-> the rest.
//      Index bits 0 and 1 stay in registers so every shared-memory access is a
//      16-byte vector.  Stages [b, b+5) run in registers.
// Between layouts the row is written to shared memory and read back; an XOR
// swizzle of the 16-byte chunk index keeps every access of every layout free
// of bank conflicts.  K = 4096 needs one exchange, K = 16384 two.
// The row is staged bf16 -> shared memory with coalesced 16-byte cp.async
// (swizzled so the per-thread reads are conflict-free too), and the next
// group's rows are prefetched into L2 with one bulk prefetch.
#pragma once
#include <cuda_runtime.h>
#include <math.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k1 {

constexpr int kRegLog = 7;
constexpr int kRedFloats = 128;  // per-group cross-warp reduction scratch

// Kernel variant bits (template parameter FL).
constexpr int kFlGain = 1;
constexpr int kFlNoHadamard = 2;
constexpr int kFlLayerNorm = 4;
constexpr int kFlExpand = 8;  // modes 6 and 8: also widen the packed weights (Params::W)

// log2 of the fp32 values each thread holds: 128 in general (K = 16384: four
// warps per row, three rows per SM, 149 us on 8192 rows against 169 us with
// 64 values and eight warps per row); 64 for K = 8192, where it keeps two
// exchanges while doubling the resident warps.
__host__ __device__ constexpr int reg_log(int L) {
    return (L == 13) ? 6 : (L < kRegLog ? L : kRegLog);
}

template <int L, int RLOG = reg_log(L)>
struct Cfg {
    static constexpr int K = 1 << L;
    static constexpr int r = RLOG;
    static constexpr int R = 1 << r;           // values per thread
    static constexpr int t = L - r;            // thread bits of a row
    static constexpr int T = 1 << t;           // threads per row
    static constexpr int W = T > 32 ? T : 32;  // threads sharing one staging buffer
    static constexpr int kRowsPerGroup = W / T;
    static constexpr int kGroupsPerCta = T >= 128 ? 1 : 128 / W;
    static constexpr int kCtaThreads = kGroupsPerCta * W;
    static constexpr int kLaneBits = t < 5 ? t : 5;
    static constexpr int kWarpBits = t > 5 ? t - 5 : 0;
    static constexpr int kStagesPerPass = r - 2;  // index bits 0 and 1 stay in registers
    static constexpr int kPasses = L <= r ? 0 : (L - r + kStagesPerPass - 1) / kStagesPerPass;
    static constexpr int kBufBytes = kRowsPerGroup * K * 4;  // fp32 row(s) of the group
    static constexpr int kStageShift = ilog2(R / 8);         // chunks per thread = R/8
    static constexpr int kSmemBytes = kGroupsPerCta * (kBufBytes + kRedFloats * 4);
    // 3 CTAs (12 warps) per SM where the register budget (170) suffices
    static constexpr int kMinBlocks =
        r == 6 ? (kCtaThreads >= 256 ? 2 : 4)
               : (kCtaThreads >= 256 ? 1 : ((L >= 8 && L != 12 && L != 14) ? 2 : 3));
};

// Layout p: 0 = natural, p >= 1 = pass p (stage base r + (r - 2)(p - 1)).
template <int L, int RLOG = reg_log(L)>
struct Lay {
    using C = Cfg<L, RLOG>;
    __host__ __device__ static constexpr int pass_base(int p) {
        return C::r + C::kStagesPerPass * (p - 1);
    }
    __host__ __device__ static constexpr int pass_count(int p) {
        return (L - pass_base(p)) < C::kStagesPerPass ? (L - pass_base(p)) : C::kStagesPerPass;
    }
    __host__ __device__ static constexpr uint32_t reg_mask(int p) {
        if (p == 0) return (1u << C::r) - 1u;
        int b = pass_base(p);
        int n = pass_count(p);
        uint32_t m = 3u;
        for (int s = b; s < b + n; ++s) m |= 1u << s;
        int cnt = 2 + n;
        for (int f = 2; cnt < C::r; ++f)
            if (!((m >> f) & 1u)) {
                m |= 1u << f;
                ++cnt;
            }
        return m;
    }
    __host__ __device__ static constexpr int reg_idx(int p, int rb) {
        uint32_t m = reg_mask(p);
        int c = 0;
        for (int i = 0; i < 32; ++i)
            if ((m >> i) & 1u) {
                if (c == rb) return i;
                ++c;
            }
        return -1;
    }
    __host__ __device__ static constexpr int thr_idx(int p, int tb) {
        uint32_t m = reg_mask(p);
        int c = 0;
        for (int i = 0; i < L; ++i)
            if (!((m >> i) & 1u)) {
                if (c == tb) return i;
                ++c;
            }
        return -1;
    }
    __host__ __device__ static constexpr int reg_off(int p, int i) {
        int e = 0;
        for (int rb = 0; rb < C::r; ++rb)
            if ((i >> rb) & 1) e |= 1 << reg_idx(p, rb);
        return e;
    }
    __host__ __device__ static constexpr int reg_bit_of(int p, int idx) {
        for (int rb = 0; rb < C::r; ++rb)
            if (reg_idx(p, rb) == idx) return rb;
        return -1;
    }
    // number of lowest index bits held in registers (the contiguous run)
    __host__ __device__ static constexpr int run_bits(int p) {
        uint32_t m = reg_mask(p);
        int c = 0;
        while (c < L && ((m >> c) & 1u)) ++c;
        return c;
    }
};

// XOR swizzle of a 16-byte chunk index for the fp32 row exchanges; linear over
// GF(2), so swz(a ^ b) = swz(a) ^ swz(b).
__host__ __device__ constexpr uint32_t swz(uint32_t ch) {
    uint32_t b3 = (ch >> 3) & 1u, b4 = (ch >> 4) & 1u, b5 = (ch >> 5) & 1u;
    uint32_t b6 = (ch >> 6) & 1u, b7 = (ch >> 7) & 1u;
    return ch ^ ((b3 ^ b4 ^ b5) | ((b3 ^ b6) << 1) | ((b4 ^ b7) << 2));
}
// Swizzle of the bf16 staging chunks (8 elements each); linear too.
template <int S>
__host__ __device__ constexpr uint32_t stage_swz(uint32_t g) {
    return g ^ ((g >> S) & 7u);
}

struct Params {
    const uint16_t* X;
    const float* gain;
    int64_t M;
    float norm_eps, quant_eps, cK, s7;
    uint8_t* codes;
    float* scales;
    int32_t* rowsum;
    float* V;
    // INT4 at K >= 16384: rows with norm_eps-free energy (sum x^2 >= 2^-100)
    // and den > thr16 have every |q| < 2^15 (see the quantisation below)
    float thr16;
    // used only by an extension (Ext below) that consumes the codes in-kernel,
    // and (W, N, wdst) by the weight expansion run beside the rows (FL &
    // kFlExpand, modes 6 and 8 of the plain kernel, for the large-batch
    // forward): the N x K packed ternary weights W widened to one signed byte
    // per weight in wdst (16 bytes per packed word).  The struct keeps its
    // size: a larger parameter block changed the plain kernels' register
    // allocation.
    const uint32_t* W;
    const float* alpha;
    union {
        uint16_t* Y;
        uint4* wdst;
    };
    int32_t* status;
    int N, rows;
};

// den above this keeps every INT4 |q| below 2^15 at K >= 16384 without a gain
// (Params::thr16): sqrt(7 K) (1 + 2^-8) / 32767, rounded up.
inline float thr16_for(int K) {
    return nextafterf((float)(sqrt(7.0 * K) * (1.0 + 1.0 / 256) / 32767.0), INFINITY);
}

// Kernel extension points.  The plain kernel (NoExt) quantises rows spread
// over the grid into global memory.  An extension (the one-kernel decode
// forward) sets its own block shape and values per thread, keeps codes (one
// byte each, row-major), scales and row sums in its shared memory, runs
// `prologue` before the rows,
// `staged` (thread 0) once the first row is in shared memory, and `finish`
// after the rows, with the whole block.
struct NoExt {
    static constexpr bool kOn = false;
    template <int L>
    __host__ __device__ static constexpr int threads() { return Cfg<L>::kCtaThreads; }
    template <int L>
    __host__ __device__ static constexpr int min_blocks() { return Cfg<L>::kMinBlocks; }
    template <int L>
    __host__ __device__ static constexpr int rlog() { return reg_log(L); }
    template <int L>
    __host__ __device__ static constexpr int groups() { return Cfg<L>::kGroupsPerCta; }
    static __device__ uint8_t* codes() { return nullptr; }
    static __device__ float* scales() { return nullptr; }
    static __device__ int32_t* rowsum() { return nullptr; }
    static __device__ void prologue(const Params&) {}
    static __device__ void staged(const Params&) {}
    static __device__ void finish(const Params&) {}
};
// The plain kernel with 2^RL values per thread instead of reg_log(L).
template <int RL>
struct NoExtR : NoExt {
    template <int L>
    __host__ __device__ static constexpr int threads() { return Cfg<L, RL>::kCtaThreads; }
    template <int L>
    __host__ __device__ static constexpr int min_blocks() { return Cfg<L, RL>::kMinBlocks; }
    template <int L>
    __host__ __device__ static constexpr int rlog() { return RL; }
    template <int L>
    __host__ __device__ static constexpr int groups() { return Cfg<L, RL>::kGroupsPerCta; }
};

template <int T>
__device__ __forceinline__ void group_sync(int grp) {
    if constexpr (T <= 32)
        __syncwarp();
    else
        named_barrier(1 + grp, T);
}

// ---- register-level pieces ------------------------------------------------

// Butterfly stage on register bit RB of the float2 array (R/2 entries).
template <int R, int RB>
__device__ __forceinline__ void stage_regs(float2 (&d)[R / 2]) {
    if constexpr (RB == 0) {
        static_for<0, R / 2>([&](auto kk) {
            constexpr int k = decltype(kk)::value;
            float a = d[k].x, b = d[k].y;
            d[k].x = __fadd_rn(a, b);
            d[k].y = __fsub_rn(a, b);
        });
    } else {
        constexpr int h = 1 << (RB - 1);
        static_for<0, R / 2>([&](auto kk) {
            constexpr int k = decltype(kk)::value;
            if constexpr ((k & h) == 0) {
                float2 a = d[k], b = d[k | h];
                d[k] = add2(a, b);
                d[k | h] = sub2(a, b);
            }
        });
    }
}

// Perfect pairwise tree (index order) of f(k) for k in [0, N), streaming with a
// stack of partial sums so only log2(N) partials stay live.
template <int N, class F>
__device__ __forceinline__ float stream_tree(F&& f) {
    constexpr int D = ilog2(N) + 1;
    float stk[D] = {};
    float out = 0.f;
    static_for<0, N>([&](auto kk) {
        constexpr int k = decltype(kk)::value;
        float x = f(kk);
        constexpr int ones = [] {
            int c = 0;
            while ((k >> c) & 1) ++c;
            return c;
        }();
        static_for<0, ones>([&](auto ll) {
            constexpr int l = decltype(ll)::value;
            x = __fadd_rn(stk[l], x);
        });
        if constexpr (k == N - 1)
            out = x;
        else
            stk[ones] = x;
    });
    return out;
}

// ---- the kernel -------------------------------------------------------------

// MODE: 0 = write fp32 V (norm + transform only), 4 = INT4 codes (packed nibbles),
// 6 = INT4 codes one per byte (row-major), 8 = INT8 codes (row-major);
// 5 / 9 = INT4 / INT8 codes one per byte in the
// 32-row interleaved layout the fused forward's GEMM loads (16-code chunk c of
// row m at byte (((m / 32) * (K / 16) + c) * 32 + m % 32) * 16).
// FL: kFlGain = multiply by the per-channel gain (else a gain of one, exact
// skip); kFlNoHadamard = no transform (the plain BitLinear of the layers
// without H: the codes are those of the normalised row itself); kFlLayerNorm =
// subtract the row mean first (LayerNorm without bias) instead of RMSNorm;
// kFlExpand = widen the packed ternary weights beside the rows (below).
template <int L, int MODE, int FL, class Ext = NoExt>
__global__ void __launch_bounds__(Ext::template threads<L>(), Ext::template min_blocks<L>())
    norm_fwht_quant_kernel(Params p) {
    constexpr bool kAbsmax = (MODE == 8 || MODE == 9);       // INT8 absmax statistic
    constexpr bool kInterleaved = (MODE == 5 || MODE == 9);  // fused-forward code layout
    constexpr bool GAIN = (FL & kFlGain) != 0;
    constexpr bool kHadamard = (FL & kFlNoHadamard) == 0;
    constexpr bool kLayerNorm = (FL & kFlLayerNorm) != 0;
    constexpr int RLOG = Ext::template rlog<L>();
    constexpr int GPC = Ext::template groups<L>();  // row groups per block
    using C = Cfg<L, RLOG>;
    using Y = Lay<L, RLOG>;
    constexpr int R = C::R, T = C::T, W = C::W, K = C::K;
    constexpr int P_LAST = kHadamard ? C::kPasses : 0;  // final layout (natural without H)
    extern __shared__ __align__(128) uint8_t smem[];
    if constexpr (Ext::kOn) Ext::prologue(p);

    const int tid = threadIdx.x;
    const int grp = tid / W;
    const int w = tid % W;
    const int lane = tid & 31;
    const int j = (T >= 32) ? w : (lane % T);    // thread index within its row
    const int rig = (T >= 32) ? 0 : (lane / T);  // row within the group
    const int wig = w >> 5;                      // warp within the row (T > 32)
    uint8_t* buf = smem + grp * C::kBufBytes;
    const uint32_t buf_s = smem_addr(buf);
    float* red = reinterpret_cast<float*>(smem + GPC * C::kBufBytes) + grp * kRedFloats;

    // thread part of the element index in layout P (plus the row offset)
    auto thr_off = [&](auto pp) -> uint32_t {
        constexpr int P = decltype(pp)::value;
        uint32_t e = 0;
        static_for<0, C::t>([&](auto tt) {
            constexpr int tb = decltype(tt)::value;
            constexpr int sh = Y::thr_idx(P, tb);
            e |= ((uint32_t)(j >> tb) & 1u) << sh;
        });
        return e + (uint32_t)rig * K;
    };

    // sum over the threads of a row, ascending thread bits (lanes by xor
    // shuffle, warps through shared memory in warp order)
    auto row_sum = [&](float x) -> float {
        static_for<0, C::kLaneBits>([&](auto tt) {
            constexpr int tb = decltype(tt)::value;
            x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 1 << tb));
        });
        if constexpr (C::kWarpBits > 0) {
            constexpr int NW = 1 << C::kWarpBits;
            if (lane == 0) red[wig] = x;
            group_sync<T>(grp);
            x = stream_tree<NW>([&](auto kk) { return red[decltype(kk)::value]; });
            group_sync<T>(grp);
        }
        return x;
    };
    auto row_max = [&](float x) -> float {
        static_for<0, C::kLaneBits>([&](auto tt) {
            constexpr int tb = decltype(tt)::value;
            x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1 << tb));
        });
        if constexpr (C::kWarpBits > 0) {
            constexpr int NW = 1 << C::kWarpBits;
            if (lane == 0) red[wig] = x;
            group_sync<T>(grp);
            x = red[0];
            static_for<1, NW>([&](auto kk) { x = fmaxf(x, red[decltype(kk)::value]); });
            group_sync<T>(grp);
        }
        return x;
    };
    auto row_isum = [&](int x) -> int {
        static_for<0, C::kLaneBits>([&](auto tt) {
            constexpr int tb = decltype(tt)::value;
            x += __shfl_xor_sync(0xffffffffu, x, 1 << tb);
        });
        if constexpr (C::kWarpBits > 0) {
            constexpr int NW = 1 << C::kWarpBits;
            int* ired = reinterpret_cast<int*>(red);
            if (lane == 0) ired[wig] = x;
            group_sync<T>(grp);
            x = 0;
            static_for<0, NW>([&](auto kk) { x += ired[decltype(kk)::value]; });
            group_sync<T>(grp);
        }
        return x;
    };

    // an extension's block does all rows itself, with threads [0, GPC W)
    const int64_t stride_groups = (int64_t)(Ext::kOn ? 1u : gridDim.x) * GPC;
    const int64_t rg_first = (!Ext::kOn || tid < GPC * W)
                                 ? (int64_t)(Ext::kOn ? 0u : blockIdx.x) * GPC + grp
                                 : p.M;
    // Stage a group's bf16 rows in shared memory with coalesced 16-byte
    // cp.async (zero-filled past M); also hint the group after it into L2.
    auto issue_load = [&](int64_t g_rg) {
        const int64_t g_row0 = g_rg * C::kRowsPerGroup;
        if (g_row0 >= p.M) return;
        const uint16_t* src0 = p.X + g_row0 * K;
        const uint32_t wsw = stage_swz<C::kStageShift>((uint32_t)w);
        static_for<0, R / 8>([&](auto ii) {
            constexpr int i = decltype(ii)::value;
            const int g = i * W + w;
            const bool ok = g_row0 + ((g * 8) >> L) < p.M;
            const uint32_t phys = stage_swz<C::kStageShift>((uint32_t)(i * W)) ^ wsw;
            cp_async16(buf_s + phys * 16u, ok ? (const void*)(src0 + g * 8) : (const void*)p.X,
                       ok ? 16 : 0);
        });
        cp_async_commit();
        if (w == 0) {
            const int64_t nrow0 = g_row0 + stride_groups * C::kRowsPerGroup;
            if (nrow0 < p.M) {
                int64_t nrows = p.M - nrow0;
                if (nrows > C::kRowsPerGroup) nrows = C::kRowsPerGroup;
                prefetch_l2_bulk(p.X + nrow0 * K, (uint32_t)(nrows * K * 2));
            }
        }
    };

    // Weight expansion beside the rows (the large-batch forward): the packed
    // words go in chunks of W x 4 words, and a group widens the chunks whose
    // index is one of its row groups' (rg_first, rg_first + stride_groups, ...,
    // continuing past the rows).  At a row's start (after the wait and group
    // barrier that the staged row needs anyway, before the row's values are
    // live) each thread copies 16 bytes of the next chunk with cp.async into
    // one of the group's two slots (it lands while the row is worked on), and
    // the group widens the chunk in the other, thread w taking words w, w + W,
    // w + 2W, w + 3W, so every warp store is 512 contiguous bytes.
    // Chunks left when the rows run out are widened after the loop straight
    // from global memory.  Chunks are whole: the launcher takes N % 16 == 0
    // and K % 128 == 0, so the W x 4 = max(K / 32, 128) words of a chunk
    // divide the N K / 16 words.
    constexpr bool kExpand = !Ext::kOn && (FL & kFlExpand) != 0;
    static_assert(!kExpand || MODE == 6 || MODE == 8, "expansion beside modes 6 and 8 only");
    constexpr int kWChunkLog = ilog2(W) + 2;  // W x 4 words per chunk
    auto w_chunks = [&]() -> int64_t { return ((int64_t)p.N << (L - 4)) >> kWChunkLog; };
    // two slots per group, taken in turn
    [[maybe_unused]] uint32_t w_buf = 0;  // byte offset of the slot the next chunk lands in
    auto w_slot = [&]() -> uint32_t {
        return smem_addr(smem + C::kSmemBytes) + (uint32_t)grp * (uint32_t)(W * 32);
    };
    auto w_issue = [&](int64_t c) {
        if (c >= w_chunks()) return;  // uniform over the group
        cp_async16(w_slot() + w_buf + (uint32_t)w * 16u, p.W + (c << kWChunkLog) + w * 4, 16);
        cp_async_commit();
    };
    auto w_widen = [&](int64_t c, uint32_t buf) {  // the group's copies of chunk c have landed
        if (c >= w_chunks()) return;
        uint4* dst = p.wdst + (c << kWChunkLog) + w;
        static_for<0, 4>([&](auto jj) {
            constexpr int jw = decltype(jj)::value;
            dst[jw * W] = expand_ternary_word(lds32(w_slot() + buf + (uint32_t)(jw * W + w) * 4u));
        });
    };

    // One row group per thread (small M, e.g. decode): let the next kernel
    // start its prologue (weight prefetch) while this one works.
    if (!Ext::kOn && stride_groups * C::kRowsPerGroup >= p.M) pdl_launch_dependents();
    issue_load(rg_first);
    if constexpr (kExpand) w_issue(rg_first);
    int64_t rg = rg_first;
    for (;; rg += stride_groups) {
        const int64_t row0 = rg * C::kRowsPerGroup;
        if (row0 >= p.M) break;
        const int64_t row = row0 + rig;
        cp_async_wait_all();
        group_sync<T>(grp);
        if constexpr (Ext::kOn) {
            if (rg == rg_first && tid == 0) Ext::staged(p);
        }
        if constexpr (kExpand) {
            // the other slot was last read a row ago, before this row's barrier
            const uint32_t cur = w_buf;
            w_buf ^= (uint32_t)(W * 16);
            w_issue(rg + stride_groups);
            w_widen(rg, cur);
        }

        float2 d[R / 2];
        {
            const uint32_t base = stage_swz<C::kStageShift>((uint32_t)w << C::kStageShift);
            static_for<0, R / 8>([&](auto ii) {
                constexpr int i = decltype(ii)::value;
                uint4 q = lds128(buf_s + (base ^ (uint32_t)i) * 16u);
                d[4 * i + 0] = bf16x2_to_f2(q.x);
                d[4 * i + 1] = bf16x2_to_f2(q.y);
                d[4 * i + 2] = bf16x2_to_f2(q.z);
                d[4 * i + 3] = bf16x2_to_f2(q.w);
            });
        }
        group_sync<T>(grp);  // staging buffer free again
        if constexpr (P_LAST == 0) issue_load(rg + stride_groups);  // overlaps this row's work

        // ---- LayerNorm: mean by the same tree (leaves x0 + x1), subtracted first
        if constexpr (kLayerNorm) {
            float sx = stream_tree<R / 2>([&](auto kk) {
                constexpr int k = decltype(kk)::value;
                return __fadd_rn(d[k].x, d[k].y);
            });
            sx = row_sum(sx);
            const float mu = __fmul_rn(sx, 1.0f / (float)K);
            const float2 mu2 = make_float2(mu, mu);
            static_for<0, R / 2>([&](auto kk) {
                constexpr int k = decltype(kk)::value;
                d[k] = sub2(d[k], mu2);
            });
        }
        // ---- RMS of the row (of x - mean for LayerNorm): tree over the row in
        // ascending index order of the squares, each square rounded to fp32
        // (one packed multiply per pair), the first tree level adding the pair
        float ss = stream_tree<R / 2>([&](auto kk) {
            constexpr int k = decltype(kk)::value;
            const float2 sq = mul2(d[k], d[k]);
            return __fadd_rn(sq.x, sq.y);
        });
        ss = row_sum(ss);
        [[maybe_unused]] const bool ss_ok = ss >= 0x1p-100f;
        const float ms = __fmul_rn(ss, 1.0f / (float)K);
        const float rn = __fdiv_rn(1.0f, __fsqrt_rn(__fadd_rn(ms, p.norm_eps)));
        {
            const float2 r2 = make_float2(rn, rn);
            static_for<0, R / 2>([&](auto kk) {
                constexpr int k = decltype(kk)::value;
                d[k] = mul2(d[k], r2);
            });
            if constexpr (GAIN) {
                const float* g = p.gain + (thr_off(ic<0>{}) - (uint32_t)rig * K);
                static_for<0, R / 4>([&](auto cc) {
                    constexpr int c = decltype(cc)::value;
                    float4 gv = *reinterpret_cast<const float4*>(g + 4 * c);
                    d[2 * c] = mul2(d[2 * c], make_float2(gv.x, gv.y));
                    d[2 * c + 1] = mul2(d[2 * c + 1], make_float2(gv.z, gv.w));
                });
            }
        }

        // ---- Walsh-Hadamard butterflies: natural layout, stages 0..r-1
        if constexpr (kHadamard)
            static_for<0, C::r>([&](auto rr) { stage_regs<R, decltype(rr)::value>(d); });

        // ---- exchanges through shared memory, one per pass
        static_for<1, P_LAST + 1>([&](auto pp) {
            constexpr int P = decltype(pp)::value;
            {  // write in layout P-1
                const uint32_t tb = swz(thr_off(ic<P - 1>{}) >> 2);
                static_for<0, R / 4>([&](auto cc) {
                    constexpr int c = decltype(cc)::value;
                    constexpr uint32_t rc = swz((uint32_t)Y::reg_off(P - 1, 4 * c) >> 2);
                    uint4 v;
                    v.x = __float_as_uint(d[2 * c].x);
                    v.y = __float_as_uint(d[2 * c].y);
                    v.z = __float_as_uint(d[2 * c + 1].x);
                    v.w = __float_as_uint(d[2 * c + 1].y);
                    sts128(buf_s + ((tb ^ rc) << 4), v);
                });
            }
            group_sync<T>(grp);
            {  // read in layout P
                const uint32_t tb = swz(thr_off(ic<P>{}) >> 2);
                static_for<0, R / 4>([&](auto cc) {
                    constexpr int c = decltype(cc)::value;
                    constexpr uint32_t rc = swz((uint32_t)Y::reg_off(P, 4 * c) >> 2);
                    uint4 v = lds128(buf_s + ((tb ^ rc) << 4));
                    d[2 * c] = make_float2(__uint_as_float(v.x), __uint_as_float(v.y));
                    d[2 * c + 1] = make_float2(__uint_as_float(v.z), __uint_as_float(v.w));
                });
            }
            group_sync<T>(grp);
            constexpr int b = Y::pass_base(P);
            constexpr int n = Y::pass_count(P);
            static_for<0, n>([&](auto ss_) {
                constexpr int s = b + decltype(ss_)::value;
                stage_regs<R, Y::reg_bit_of(P, s)>(d);
            });
        });

        // the row buffer is free from here on: start the next group's load so it
        // overlaps the rest of this row's work
        if constexpr (P_LAST > 0) issue_load(rg + stride_groups);

        // ---- normalise by 1/sqrt(K)
        if constexpr (kHadamard) {
            const float2 c2 = make_float2(p.cK, p.cK);
            static_for<0, R / 2>([&](auto kk) {
                constexpr int k = decltype(kk)::value;
                d[k] = mul2(d[k], c2);
            });
        }

        const uint32_t toff = thr_off(ic<P_LAST>{});  // includes rig * K
        constexpr int RUN = Y::run_bits(P_LAST);       // contiguous run length 2^RUN

        if constexpr (MODE == 0) {
            if (row < p.M) {
                float* vrow = p.V + row0 * K;
                static_for<0, R / 4>([&](auto cc) {
                    constexpr int c = decltype(cc)::value;
                    constexpr uint32_t e = (uint32_t)Y::reg_off(P_LAST, 4 * c);
                    *reinterpret_cast<float4*>(vrow + (toff | e)) =
                        make_float4(d[2 * c].x, d[2 * c].y, d[2 * c + 1].x, d[2 * c + 1].y);
                });
            }
        } else {
            // ---- per-token statistic
            float stat;
            if constexpr (kAbsmax) {
                float m = 0.f;
                static_for<0, R / 2>([&](auto kk) {
                    constexpr int k = decltype(kk)::value;
                    m = fmaxf(m, fmaxf(fabsf(d[k].x), fabsf(d[k].y)));
                });
                stat = row_max(m);
            } else {
                // tree_sum(|v|): runs in registers, then lanes: the first NSC
                // lane levels scatter the remaining register partials (each
                // lane keeps the half its lane bit selects), the rest add.
                constexpr int NRUN = R >> RUN;  // partials per thread after the runs
                constexpr int NSC = ilog2(NRUN);
                static_assert(NSC <= C::kLaneBits, "partials exceed lane bits");
                const float total_thread = [&] {
                    float stk[NSC + 1] = {};
                    float fin = 0.f;
                    static_for<0, NRUN>([&](auto mm) {
                        constexpr int m = decltype(mm)::value;
                        constexpr int RL = 1 << RUN;  // elements per run
                        float x = stream_tree<RL / 2>([&](auto kk) {
                            constexpr int k = (m * RL) / 2 + decltype(kk)::value;
                            return __fadd_rn(fabsf(d[k].x), fabsf(d[k].y));
                        });
                        constexpr int ones = [] {
                            int c = 0;
                            while (c < NSC && ((m >> c) & 1)) ++c;
                            return c;
                        }();
                        static_for<0, ones>([&](auto ll) {
                            constexpr int l = decltype(ll)::value;
                            const bool hi = (j >> l) & 1;
                            const float a = stk[l];  // partial bit = 0
                            const float keep = hi ? x : a;
                            const float send = hi ? a : x;
                            x = __fadd_rn(keep, __shfl_xor_sync(0xffffffffu, send, 1 << l));
                        });
                        if constexpr (m == NRUN - 1)
                            fin = x;
                        else
                            stk[ones] = x;
                    });
                    return fin;
                }();
                float x = total_thread;
                static_for<NSC, C::kLaneBits>([&](auto tt) {
                    constexpr int tb = decltype(tt)::value;
                    x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 1 << tb));
                });
                if constexpr (C::kWarpBits == 0) {
                    static_for<0, NSC>([&](auto ll) {
                        constexpr int l = decltype(ll)::value;
                        x = __fadd_rn(x, __shfl_xor_sync(0xffffffffu, x, 1 << l));
                    });
                } else {
                    constexpr int WB = C::kWarpBits;
                    constexpr int NV = 1 << (WB + NSC);
                    static_assert(NV <= kRedFloats, "reduction scratch too small");
                    if ((lane >> NSC) == 0) red[wig | (lane << WB)] = x;
                    group_sync<T>(grp);
                    x = stream_tree<NV>([&](auto kk) { return red[decltype(kk)::value]; });
                    group_sync<T>(grp);
                }
                stat = __fmul_rn(x, 1.0f / (float)K);
            }

            const float cq = kAbsmax ? 127.0f : p.s7;
            // (a zero row with quant_eps = 0: inv = 0, so every code is 0)
            const float den = __fadd_rn(stat, p.quant_eps);
            const bool pos = den > 0.f;
            const float inv = __fdiv_rn(pos ? cq : 0.f, pos ? den : 1.f);
            const float2 inv2 = make_float2(inv, inv);
            // One rounding of the exact product v*inv to an integer: fma with
            // 1.5*2^23 (+8 for packed INT4, making the stored nibble q + 8).
            // |v*inv| <= 127 (INT8) or <= sqrt7*K (INT4), far below 2^22.
            constexpr float kMagic = (MODE == 4) ? 12582920.0f : 12582912.0f;
            constexpr int32_t kMagicBits = (MODE == 4) ? 0x4B400008 : 0x4B400000;
            const float2 magic2 = make_float2(kMagic, kMagic);
            // INT4 clamp on the integer bit pattern: q in [-8, 7]
            constexpr int32_t kLoBits = kMagicBits - 8, kHiBits = kMagicBits + 7;
            constexpr bool kPackNibbles = (MODE == 4);
            // ... or on int16 halves where |q| < 2^15 is guaranteed: always for
            // K <= 8192 (|q| <= sqrt7 K); for larger K without a gain, on rows
            // where max|v| <= ||v|| <= sqrt(K) (1 + 2^-8) bounds |q| by
            // sqrt(7 K) (1 + 2^-8) / den < 2^15 - 1, i.e. den > thr16 (||u||^2 =
            // r^2 sum x^2 <= K up to rounding, the transform is orthonormal; the
            // sum x^2 >= 2^-100 test keeps squares out of the subnormal range)
            constexpr bool kClamp16Static = !kAbsmax && L <= 13;
            constexpr bool kClamp16Dyn = !kAbsmax && L >= 14 && !GAIN;
            constexpr uint32_t kLo2 = kPackNibbles ? 0x00000000u : 0xFFF8FFF8u;
            constexpr uint32_t kHi2 = kPackNibbles ? 0x000F000Fu : 0x00070007u;
            constexpr int RL = 1 << RUN;                                 // elements per run
            constexpr int BYTES = kPackNibbles ? RL / 2 : RL;            // code bytes per run
            constexpr int EPW = kPackNibbles ? (RL >= 8 ? 8 : 4) : 4;    // elements per word
            constexpr int NWORD = RL / EPW;
            const bool row_ok = row < p.M;
            uint8_t* crow = (Ext::kOn ? Ext::codes() : p.codes) +
                            row0 * (int64_t)(kPackNibbles ? K / 2 : K);
            // codes of the thread's runs, stored; returns the sum of its codes
            auto quant_runs = [&](auto c16) -> int {
            constexpr bool kClamp16 = decltype(c16)::value;
            uint32_t qsum = 0;
            static_for<0, R / RL>([&](auto mm) {
                constexpr int m = decltype(mm)::value;
                uint32_t wv[NWORD];
                static_for<0, NWORD>([&](auto ww) {
                    constexpr int wi = decltype(ww)::value;
                    if constexpr (kClamp16) {
                        // INT4 at K <= 8192: |q| <= sqrt7 * K < 2^15, so the low 16
                        // bits of each rounded pattern hold q (+8 for nibbles)
                        // exactly; pairs of codes are clamped as int16 halves
                        uint32_t pr[EPW / 2];
                        static_for<0, EPW / 2>([&](auto kk) {
                            constexpr int k = (m * RL + wi * EPW) / 2 + decltype(kk)::value;
                            const float2 y = __ffma2_rn(d[k], inv2, magic2);
                            uint32_t h = __byte_perm(__float_as_uint(y.x),
                                                     __float_as_uint(y.y), 0x5410);
                            asm("min.s16x2 %0, %0, %1;" : "+r"(h) : "r"(kHi2));
                            asm("max.s16x2 %0, %0, %1;" : "+r"(h) : "r"(kLo2));
                            pr[decltype(kk)::value] = h;
                        });
                        if constexpr (!kPackNibbles) {  // bytes q0..q3
                            wv[wi] = __byte_perm(pr[0], pr[1], 0x6420);
                            qsum = (uint32_t)__dp4a((int)wv[wi], 0x01010101, (int)qsum);
                        } else {  // byte = (q_odd + 8) << 4 | (q_even + 8), then q's nibbles
                            uint32_t by[EPW / 2];
                            static_for<0, EPW / 2>([&](auto kk) {
                                constexpr int i = decltype(kk)::value;
                                qsum = (uint32_t)__dp2a_lo((int)pr[i], 0x0101, (int)qsum);
                                by[i] = pr[i] | (pr[i] >> 12);
                            });
                            const uint32_t lo2 = __byte_perm(by[0], by[1], 0x0040);
                            if constexpr (EPW == 8) {
                                const uint32_t hi2 = __byte_perm(by[2], by[3], 0x0040);
                                wv[wi] = __byte_perm(lo2, hi2, 0x5410) ^ 0x88888888u;
                            } else {
                                wv[wi] = lo2 ^ 0x8888u;
                            }
                        }
                    } else {
                        uint32_t qv[EPW];
                        static_for<0, EPW / 2>([&](auto kk) {
                            constexpr int k = (m * RL + wi * EPW) / 2 + decltype(kk)::value;
                            const float2 y = __ffma2_rn(d[k], inv2, magic2);
                            int32_t b0 = __float_as_int(y.x), b1 = __float_as_int(y.y);
                            if constexpr (!kAbsmax) {  // INT8 codes never leave [-127, 127]
                                b0 = min(max(b0, kLoBits), kHiBits);
                                b1 = min(max(b1, kLoBits), kHiBits);
                            }
                            qv[2 * decltype(kk)::value] = (uint32_t)b0;
                            qv[2 * decltype(kk)::value + 1] = (uint32_t)b1;
                        });
                        if constexpr (!kPackNibbles) {  // one byte per code: low byte = q
                            const uint32_t lo2 = __byte_perm(qv[0], qv[1], 0x0040);
                            const uint32_t hi2 = __byte_perm(qv[2], qv[3], 0x0040);
                            wv[wi] = __byte_perm(lo2, hi2, 0x5410);
                            // rowsum: the four signed bytes summed by one dp4a
                            qsum = (uint32_t)__dp4a((int)wv[wi], 0x01010101, (int)qsum);
                        } else {
                            // low nibble = q + 8; pairs by shift-add, bytes by permute
                            static_for<0, EPW>([&](auto ee) { qsum += qv[decltype(ee)::value]; });
                            const uint32_t p01 = (qv[1] << 4) + qv[0];
                            const uint32_t p23 = (qv[3] << 4) + qv[2];
                            const uint32_t lo2 = __byte_perm(p01, p23, 0x0040);
                            if constexpr (EPW == 8) {
                                const uint32_t p45 = (qv[5] << 4) + qv[4];
                                const uint32_t p67 = (qv[7] << 4) + qv[6];
                                const uint32_t hi2 = __byte_perm(p45, p67, 0x0040);
                                wv[wi] = __byte_perm(lo2, hi2, 0x5410) ^ 0x88888888u;
                            } else {
                                wv[wi] = lo2 ^ 0x8888u;
                            }
                        }
                    }
                });
                if (row_ok) {
                    constexpr uint32_t e0 = (uint32_t)Y::reg_off(P_LAST, m * RL);
                    uint8_t* dst = crow + (kPackNibbles ? ((toff | e0) >> 1) : (toff | e0));
                    if constexpr (kInterleaved) {
                        // 32-row interleaved layout: 16-code chunk c of row m at
                        // (((m / 32) * (K / 16) + c) * 32 + m % 32) * 16
                        const uint32_t ein = (toff | e0) & (uint32_t)(K - 1);
                        dst = p.codes + (((row >> 5) * (int64_t)(K >> 4) + (ein >> 4)) << 9) +
                              ((row & 31) << 4) + (ein & 15u);
                    }
                    if constexpr (BYTES == 2) {
                        *reinterpret_cast<uint16_t*>(dst) = (uint16_t)wv[0];
                    } else if constexpr (BYTES == 4) {
                        *reinterpret_cast<uint32_t*>(dst) = wv[0];
                    } else if constexpr (BYTES == 8) {
                        *reinterpret_cast<uint2*>(dst) = make_uint2(wv[0], wv[1]);
                    } else {
                        static_for<0, BYTES / 16>([&](auto vv) {
                            constexpr int v = decltype(vv)::value;
                            constexpr int step = kInterleaved ? 512 : 16;  // next 16-code chunk
                            *reinterpret_cast<uint4*>(dst + step * v) =
                                make_uint4(wv[4 * v], wv[4 * v + 1], wv[4 * v + 2], wv[4 * v + 3]);
                        });
                    }
                }
            });
            // sum of codes: packed nibbles added kMagicBits + q per code (mod 2^32),
            // or q + 8 per code on the int16 path; one-byte codes were summed directly
            return !kPackNibbles ? (int)qsum
                   : kClamp16    ? (int)qsum - 8 * R
                                 : (int)(qsum - (uint32_t)R * (uint32_t)kMagicBits);
            };
            int qs;
            if constexpr (kClamp16Dyn) {
                if (ss_ok && den > p.thr16)  // uniform over the row
                    qs = quant_runs(ic_bool<true>{});
                else
                    qs = quant_runs(ic_bool<false>{});
            } else {
                qs = quant_runs(ic_bool<kClamp16Static>{});
            }
            qs = row_isum(qs);

            if (row_ok) {
                if (j == 0) {
                    (Ext::kOn ? Ext::scales() : p.scales)[row] = __fdiv_rn(stat, cq);
                    if constexpr (Ext::kOn)
                        Ext::rowsum()[row] = qs;
                    else if (p.rowsum != nullptr)
                        p.rowsum[row] = qs;
                }
            }
        }
    }
    if constexpr (kExpand) {
        // chunk rg is in flight (or past the end): finish it, then the rest
        // from global memory with four chunks' loads in flight per thread
        cp_async_wait_all();
        group_sync<T>(grp);
        w_widen(rg, w_buf);  // the last copy went to slot w_buf
        for (int64_t c0 = rg + stride_groups; c0 < w_chunks(); c0 += 4 * stride_groups) {
            uint32_t v[4][4];
            static_for<0, 4>([&](auto ee) {
                constexpr int e = decltype(ee)::value;
                const int64_t c = c0 + e * stride_groups;
                static_for<0, 4>([&](auto jj) {
                    constexpr int jw = decltype(jj)::value;
                    v[e][jw] = c < w_chunks() ? __ldg(p.W + (c << kWChunkLog) + jw * W + w) : 0u;
                });
            });
            static_for<0, 4>([&](auto ee) {
                constexpr int e = decltype(ee)::value;
                const int64_t c = c0 + e * stride_groups;
                static_for<0, 4>([&](auto jj) {
                    constexpr int jw = decltype(jj)::value;
                    if (c < w_chunks())
                        p.wdst[(c << kWChunkLog) + jw * W + w] = expand_ternary_word(v[e][jw]);
                });
            });
        }
    }
    if constexpr (Ext::kOn) Ext::finish(p);
}

template <int L, int MODE, int FL, class Ext>
static hbl_status launch_cfg(const Params& prm, cudaStream_t stream, int num_sms) {
    using C = Cfg<L, Ext::template rlog<L>()>;
    auto kern = norm_fwht_quant_kernel<L, MODE, FL, Ext>;
    // the weight expansion's two slots: 32 bytes per thread after the rows' buffers
    constexpr bool expand = !Ext::kOn && (FL & kFlExpand) != 0;
    const int smem = C::kSmemBytes + (expand ? C::kCtaThreads * 32 : 0);
    if (!smem_attr_once(reinterpret_cast<const void*>(kern), smem)) return HBL_ERR_CUDA;
    const int64_t groups = (prm.M + C::kRowsPerGroup - 1) / C::kRowsPerGroup;
    const int64_t ctas_needed = (groups + C::kGroupsPerCta - 1) / C::kGroupsPerCta;
    int64_t grid = (int64_t)num_sms * C::kMinBlocks;
    if (ctas_needed < grid) grid = ctas_needed;
    if (grid < 1) grid = 1;
    kern<<<(unsigned)grid, C::kCtaThreads, smem, stream>>>(prm);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

// Whether K1's rows carry the weight expansion well: every group widens at
// most one chunk more than it has row groups, so hardly any of it is left for
// after the rows (measured: 8192 tokens at K = 16384 gained 6 us over the
// separate expansion kernel; 2048 tokens, most chunks after the rows, lost 12).
template <int L, int RL>
static bool expand_rides_along_cfg(int64_t M, int N, int num_sms) {
    using C = Cfg<L, RL>;
    const int64_t groups = (M + C::kRowsPerGroup - 1) / C::kRowsPerGroup;
    int64_t ctas = (groups + C::kGroupsPerCta - 1) / C::kGroupsPerCta;
    if (ctas > (int64_t)num_sms * C::kMinBlocks) ctas = (int64_t)num_sms * C::kMinBlocks;
    const int64_t ng = (ctas < 1 ? 1 : ctas) * C::kGroupsPerCta;
    const int64_t chunks = ((int64_t)N << (L - 4)) >> (ilog2(C::W) + 2);
    return (chunks + ng - 1) / ng <= (groups + ng - 1) / ng + 1;
}
template <int L>
static bool expand_rides_along_l(int64_t M, int N, int num_sms) {
    if constexpr (L == 14)  // the launch choice of launch_one below
        if (M <= (int64_t)num_sms * Cfg<L>::kMinBlocks)
            return expand_rides_along_cfg<L, 6>(M, N, num_sms);
    return expand_rides_along_cfg<L, reg_log(L)>(M, N, num_sms);
}

template <int L, int MODE, int FL>
static hbl_status launch_one(const Params& prm, cudaStream_t stream, int num_sms) {
    // K = 16384 with at most one row per CTA: latency per row decides, and 64
    // values per thread (eight warps per row) finish a row sooner
    if constexpr (L == 14)
        if (prm.M <= (int64_t)num_sms * Cfg<L>::kMinBlocks)
            return launch_cfg<L, MODE, FL, NoExtR<6>>(prm, stream, num_sms);
    return launch_cfg<L, MODE, FL, NoExt>(prm, stream, num_sms);
}

template <int MODE, int FL>
hbl_status dispatch(int L, const Params& prm, cudaStream_t s, int sms) {
    switch (L) {
        case 4: return launch_one<4, MODE, FL>(prm, s, sms);
        case 5: return launch_one<5, MODE, FL>(prm, s, sms);
        case 6: return launch_one<6, MODE, FL>(prm, s, sms);
        case 7: return launch_one<7, MODE, FL>(prm, s, sms);
        case 8: return launch_one<8, MODE, FL>(prm, s, sms);
        case 9: return launch_one<9, MODE, FL>(prm, s, sms);
        case 10: return launch_one<10, MODE, FL>(prm, s, sms);
        case 11: return launch_one<11, MODE, FL>(prm, s, sms);
        case 12: return launch_one<12, MODE, FL>(prm, s, sms);
        case 13: return launch_one<13, MODE, FL>(prm, s, sms);
        case 14: return launch_one<14, MODE, FL>(prm, s, sms);
        case 15: return launch_one<15, MODE, FL>(prm, s, sms);
        default: return HBL_ERR_SHAPE;
    }
}

}  // namespace k1
}  // namespace hbl
