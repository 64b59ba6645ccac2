// k3_ternary_gemv.cu -- split-K ternary x int8/int4 GEMV on CUDA cores for small
// token counts (decode), sm_100a.
//
// acc[m][n] = sum_k q[m][k] * t[n][k] is computed as sum_k q*c - rowsum[m]
// with c = t + 1 in {0, 1, 2} the stored 2-bit code, using dp4a (signed
// activation bytes x unsigned weight bytes).  The weight word layout makes
// (w >> 2i) & 0x03030303 the codes of weights 4i..4i+3, one byte each.
// Each CTA owns 64 output features and one K slice; the slice's activations
// (all M tokens, widened to int8) sit in shared memory; each warp owns 8
// output features, each lane a strided set of 16-weight words.  Integer
// partials go to workspace [KSPLIT][M][N] and a second kernel sums them (exact
// in any order), subtracts rowsum and applies (alpha * scale[m]) -> bf16.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

#include <atomic>

namespace hbl {
namespace k3 {

constexpr int kMaxM = 8;        // tokens per launch handled in registers
constexpr int kRowsPerWarp = 8;
constexpr int kWarps = 8;
constexpr int kRowsPerCta = kRowsPerWarp * kWarps;  // 64
constexpr int kSmemBytes = 64 * 1024;               // activation slice budget

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

template <int MT>
__global__ void __launch_bounds__(kWarps * 32)
    gemv_kernel(const uint8_t* __restrict__ codes, int act_bits, int M, int K,
                const uint32_t* __restrict__ Wp, int N, int kslice, int32_t* __restrict__ part) {
    extern __shared__ __align__(16) uint8_t sact[];  // [MT][kslice] int8
    const int ks = blockIdx.y;
    const int k0 = ks * kslice;
    const int klen = min(kslice, K - k0);
    const int n0 = blockIdx.x * kRowsPerCta;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;

    // this CTA's weight slice into L2 while the previous kernel finishes, then wait
    if (tid < kRowsPerCta && n0 + tid < N && klen >= 64)
        prefetch_l2_bulk(Wp + (int64_t)(n0 + tid) * (K / 16) + k0 / 16, (uint32_t)(klen / 4));
    pdl_wait();

    // stage activations [MT][klen] as int8 (rows >= M zero)
    const int chunks = klen / 16;  // 16 int8 per chunk
    for (int c = tid; c < MT * chunks; c += blockDim.x) {
        const int m = c / chunks, kc = c % chunks;
        uint4 v = make_uint4(0, 0, 0, 0);
        if (m < M) {
            if (act_bits == 8) {
                v = *reinterpret_cast<const uint4*>(codes + (int64_t)m * K + k0 + kc * 16);
            } else {
                uint2 p = *reinterpret_cast<const uint2*>(codes + (int64_t)m * (K / 2) +
                                                          (k0 + kc * 16) / 2);
                uint2 a = widen_nibbles(p.x), b = widen_nibbles(p.y);
                v = make_uint4(a.x, a.y, b.x, b.y);
            }
        }
        *reinterpret_cast<uint4*>(sact + m * kslice + kc * 16) = v;
    }
    __syncthreads();

    int acc[kRowsPerWarp][MT];
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) acc[r][m] = 0;

    const int nbase = n0 + warp * kRowsPerWarp;
    const int wpr = K / 16;  // words per weight row
    const int nw = klen / 16;
    for (int wi = lane; wi < nw; wi += 32) {
        uint32_t wv[kRowsPerWarp];
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int n = nbase + r;
            wv[r] = (n < N) ? __ldg(Wp + (int64_t)n * wpr + k0 / 16 + wi) : 0x55555555u;
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const uint4 a = *reinterpret_cast<const uint4*>(sact + m * kslice + wi * 16);
#pragma unroll
            for (int r = 0; r < kRowsPerWarp; ++r) {
                int s = acc[r][m];
                s = dp4a_su((int)a.x, wv[r] & 0x03030303u, s);
                s = dp4a_su((int)a.y, (wv[r] >> 2) & 0x03030303u, s);
                s = dp4a_su((int)a.z, (wv[r] >> 4) & 0x03030303u, s);
                s = dp4a_su((int)a.w, (wv[r] >> 6) & 0x03030303u, s);
                acc[r][m] = s;
            }
        }
    }
    // reduce over lanes (integer: exact in any order)
#pragma unroll
    for (int r = 0; r < kRowsPerWarp; ++r)
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            int s = acc[r][m];
#pragma unroll
            for (int b = 16; b >= 1; b >>= 1) s += __shfl_xor_sync(0xffffffffu, s, b);
            acc[r][m] = s;
        }
    if (lane < kRowsPerWarp) {
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r)
            if (r == lane) {
                const int n = nbase + r;
                if (n < N)
#pragma unroll
                    for (int m = 0; m < MT; ++m)
                        if (m < M) part[((int64_t)ks * M + m) * N + n] = acc[r][m];
            }
    }
}

__global__ void gemv_epilogue_kernel(const int32_t* __restrict__ part, int ksplit, int M, int N,
                                     const int32_t* __restrict__ rowsum,
                                     const float* __restrict__ scales,
                                     const float* __restrict__ alpha, uint16_t* __restrict__ Y,
                                     int32_t* __restrict__ acc_out) {
    pdl_wait();
    const float a = *alpha;
    const int64_t total = (int64_t)M * N;
    for (int64_t i = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; i < total;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int m = (int)(i / N);
        int s = 0;
        for (int k = 0; k < ksplit; ++k) s += part[(int64_t)k * total + i];
        s -= rowsum[m];
        if (acc_out) acc_out[i] = s;
        const float sc = __fmul_rn(a, scales[m]);
        const float y = __fmul_rn((float)s, sc);
        Y[i] = __bfloat16_as_ushort(__float2bfloat16_rn(y));
    }
}

static int choose_ksplit(int K, int N, int num_sms) {
    const int ctas_n = (N + kRowsPerCta - 1) / kRowsPerCta;
    int ks = 1;
    // aim for >= 2 CTAs per SM, slices of at least 512 weights (one word per lane)
    while (ctas_n * ks < 2 * num_sms && K / (ks * 2) >= 512) ks *= 2;
    // slice must fit shared memory for kMaxM tokens
    while ((int64_t)(K / ks) * kMaxM > kSmemBytes) ks *= 2;
    return ks;
}

}  // namespace k3

int gemv_max_m() { return k3::kMaxM; }

hbl_status launch_splitk_epilogue(const int32_t* part, int ksplit, int64_t M, int N,
                                  const int32_t* rowsum, const float* scales, const float* alpha,
                                  uint16_t* Y, int32_t* acc_out, cudaStream_t stream) {
    const int64_t total = M * N;
    int64_t eb = (total + 255) / 256;
    if (eb > 148 * 8) eb = 148 * 8;
    return launch_pdl(k3::gemv_epilogue_kernel, dim3((unsigned)eb), dim3(256), 0, stream, part,
                      ksplit, (int)M, N, rowsum, scales, alpha, Y, acc_out);
}

size_t gemv_workspace(int64_t M, int K, int N, int num_sms) {
    const int ks = k3::choose_ksplit(K, N, num_sms);
    return ((size_t)ks * (size_t)M * (size_t)N * 4 + 255) & ~(size_t)255;
}

hbl_status launch_gemv(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                       int num_sms) {
    if (a.M == 0) return HBL_OK;
    if (a.M > k3::kMaxM) return HBL_ERR_SHAPE;
    num_sms = num_sms < 148 ? num_sms : 148;  // workspace queries size for 148 SMs
    const int ks = k3::choose_ksplit(a.K, a.N, num_sms);
    const int kslice = a.K / ks;
    if (gemv_workspace(a.M, a.K, a.N, num_sms) > ws_bytes || ws == nullptr)
        return HBL_ERR_WORKSPACE;
    int32_t* part = static_cast<int32_t*>(ws);
    const int M = (int)a.M;
    const int mt = M <= 1 ? 1 : (M <= 2 ? 2 : (M <= 4 ? 4 : 8));
    const size_t smem = (size_t)mt * kslice;
    dim3 grid((a.N + k3::kRowsPerCta - 1) / k3::kRowsPerCta, ks);
    const uint8_t* codes = static_cast<const uint8_t*>(a.codes);
#define HBL_GEMV_CASE(MT)                                                                       \
    case MT:                                                                                    \
        if (smem > 48 * 1024 &&                                                                 \
            !smem_attr_once(reinterpret_cast<const void*>(k3::gemv_kernel<MT>), (int)smem))     \
            return HBL_ERR_CUDA;                                                                \
        if (launch_pdl(k3::gemv_kernel<MT>, grid, dim3(k3::kWarps * 32), smem, stream, codes,    \
                       a.act_bits, M, a.K, a.W_packed, a.N, kslice, part) != HBL_OK)             \
            return HBL_ERR_CUDA;                                                                \
        break;
    switch (mt) {
        HBL_GEMV_CASE(1)
        HBL_GEMV_CASE(2)
        HBL_GEMV_CASE(4)
        HBL_GEMV_CASE(8)
        default: return HBL_ERR_SHAPE;
    }
#undef HBL_GEMV_CASE
    const int64_t total = a.M * a.N;
    int64_t eb = (total + 255) / 256;
    if (eb > (int64_t)num_sms * 8) eb = (int64_t)num_sms * 8;
    return launch_pdl(k3::gemv_epilogue_kernel, dim3((unsigned)eb), dim3(256), 0, stream,
                      (const int32_t*)part, ks, M, a.N, a.rowsum, a.scales, a.alpha, a.Y,
                      a.acc_out);
}


// ---------------------------------------------------------------------------
// Allocation-free variant: the split-K partials live in a fixed device array
// owned by this file instead of caller-provided workspace.  Some callers cannot
// hand the library scratch memory or let it allocate: an engine's custom-op or
// plugin hook that receives only its inputs and outputs, or a per-token decode
// loop that must not take the allocator's lock, stall on an implicit device
// synchronisation, or fail with out-of-memory halfway through a step.
// The array below is reserved on every GPU that loads the library and stays
// reserved until the process exits.  Its host-side name is only a stand-in,
// never a device address, so the address is looked up once per device with
// cudaGetSymbolAddress while that device is current.
constexpr size_t kNoAllocScratchBytes = (size_t)2 << 20;  // 2 MiB
static __device__ __align__(256) int32_t g_noalloc_scratch[kNoAllocScratchBytes / 4];

namespace {
constexpr int kNoAllocMaxDevices = 64;
std::atomic<void*> g_noalloc_ptr[kNoAllocMaxDevices];
}  // namespace

size_t gemv_noalloc_scratch_bytes() { return kNoAllocScratchBytes; }

// Device address of the fixed scratch array on the current device, or null.
void* gemv_noalloc_scratch(int dev) {
    if (dev < 0 || dev >= kNoAllocMaxDevices) return nullptr;
    void* p = g_noalloc_ptr[dev].load(std::memory_order_acquire);
    if (p != nullptr) return p;
    void* q = nullptr;
    if (cudaGetSymbolAddress(&q, g_noalloc_scratch) != cudaSuccess || q == nullptr)
        return nullptr;
    g_noalloc_ptr[dev].store(q, std::memory_order_release);
    return q;
}

}  // namespace hbl
