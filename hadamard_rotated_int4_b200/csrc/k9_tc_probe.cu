// k9_tc_probe.cu -- measures the dense INT8 tensor-core rate of this GPU, the
// denominator of the ternary GEMM's roofline.  Every CTA (one per SM: its
// shared-memory request leaves room for no second CTA) zeroes one 128 x 128-byte
// A tile and one 256 x 128-byte B tile in shared memory, allocates a
// 128 x 256 int32 accumulator in TMEM, and one thread issues `n_mma`
// back-to-back tcgen05.mma.cta_group::1.kind::i8 of shape 128 x 256 x 32 (the
// GEMM's own instruction shape and operand layout) into it.  No global memory
// is read or written except the status word, so the time the caller measures
// around the launch is tensor-pipe time plus one launch.  The final wait for
// the MMAs is bounded by global time (HBL_ERR_TIMEOUT in dev_status).
#include <cuda_runtime.h>

#include "hbl_internal.cuh"
#include "hbl_launch.h"

namespace hbl {
namespace k9 {

constexpr int kThreads = 128;
constexpr int kATile = 128 * 128;
constexpr int kBTile = 256 * 128;
// above half of the SM's shared memory: one CTA per SM
constexpr int kSmemBytes = 120 * 1024;
constexpr uint32_t kCols = 256;
// kind::i8, D s32, A s8, B s8, both K-major, N = 256, M = 128
constexpr uint32_t kIdesc = (2u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) |
                            ((uint32_t)(128 >> 4) << 24);

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)1 << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)2 << 61;
    return d;
}

__global__ void __launch_bounds__(kThreads, 1) tc_int8_probe_kernel(int n_mma, int32_t* status) {
    extern __shared__ uint8_t smem_raw[];
    const uint32_t raw_s = smem_addr(smem_raw);
    const uint32_t base_s = (raw_s + 1023u) & ~1023u;
    uint8_t* base = smem_raw + (base_s - raw_s);
    const uint32_t a_s = base_s, b_s = base_s + kATile;
    const uint32_t bar_s = b_s + kBTile;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(base + kATile + kBTile + 64);
    const int warp = threadIdx.x >> 5;

    uint4* z = reinterpret_cast<uint4*>(base);
    for (int i = threadIdx.x; i < (kATile + kBTile) / 16; i += kThreads) z[i] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x == 0) {
        mbar_init_count(bar_s, 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    // the tiles were written by ordinary stores; the tensor core reads them
    // through the async proxy
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_addr(tmem_slot)),
                     "r"(kCols)
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
    const uint32_t tmem = *tmem_slot;

    if (threadIdx.x == 0) {
        for (int i = 0; i < n_mma; ++i) {
            const uint32_t k = (uint32_t)(i & 3) * 32u;
            const uint64_t ad = sw128_desc(a_s + k), bd = sw128_desc(b_s + k);
            asm volatile(
                "{\n.reg .pred p;\n"
                "setp.ne.b32 p, %4, 0;\n"
                "tcgen05.mma.cta_group::1.kind::i8 [%0], %1, %2, %3, p;\n}\n" ::"r"(tmem),
                "l"(ad), "l"(bd), "r"(kIdesc), "r"(i)
                : "memory");
        }
        asm volatile(
            "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                bar_s)
            : "memory");
        if (!mbar_wait_bounded<true>(bar_s, 0, 2000000000ull)) report_status(status, HBL_ERR_TIMEOUT);
    }
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
    __syncthreads();
    if (warp == 0) {
        asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kCols)
                     : "memory");
    }
}

}  // namespace k9

hbl_status launch_tc_int8_probe(int ctas, int mmas_per_cta, int32_t* status, cudaStream_t stream) {
    if (!smem_attr_once(reinterpret_cast<const void*>(k9::tc_int8_probe_kernel), k9::kSmemBytes))
        return HBL_ERR_CUDA;
    k9::tc_int8_probe_kernel<<<ctas, k9::kThreads, k9::kSmemBytes, stream>>>(mmas_per_cta, status);
    return cudaGetLastError() == cudaSuccess ? HBL_OK : HBL_ERR_CUDA;
}

}  // namespace hbl
