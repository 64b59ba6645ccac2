// hbl_internal.cuh -- device helpers shared by the sm_100a kernels of libhbl.
// Inline PTX wrappers (cp.async, bulk prefetch, named barriers, packed fp32x2
// arithmetic, mbarriers, TMA, tcgen05) and a compile-time loop helper.
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <type_traits>
#include <utility>

#include "hbl.h"

namespace hbl {

// ------------------------------------------------------------ compile time

template <int I>
using ic = std::integral_constant<int, I>;
template <bool B>
using ic_bool = std::integral_constant<bool, B>;

template <int Begin, int End, class F>
__device__ __forceinline__ void static_for(F&& f) {
    if constexpr (Begin < End) {
        f(ic<Begin>{});
        static_for<Begin + 1, End>(f);
    }
}

__host__ __device__ constexpr int ilog2(unsigned v) {
    int r = 0;
    while ((1u << r) < v) ++r;
    return r;
}

// ------------------------------------------------------------ status

// First non-zero status wins; the host reads it after synchronising.
__device__ __forceinline__ void report_status(int32_t* st, int code) {
    if (st != nullptr) atomicCAS(reinterpret_cast<int*>(st), 0, code);
}

// Upper bound on spins of any device-side wait (each spin also sleeps), so a
// wait that can never be satisfied returns an error instead of hanging.
constexpr uint32_t kSpinLimit = 1u << 22;

// ------------------------------------------------------------ bounded waits

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}
__device__ __forceinline__ void mbar_init_count(uint32_t a, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(a), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_one(uint32_t a) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(a) : "memory");
}
// true once the phase of the given parity has completed
__device__ __forceinline__ bool mbar_test_parity(uint32_t a, uint32_t parity) {
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
// Waits for an mbarrier phase for at most limit_ns of global time; SLEEP backs
// off between polls.  Returns false on expiry (the caller reports
// HBL_ERR_TIMEOUT and unwinds instead of hanging).
template <bool SLEEP>
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t a, uint32_t parity, uint64_t limit_ns) {
    if (mbar_test_parity(a, parity)) return true;
    const uint64_t t0 = global_ns();
    while (true) {
        if constexpr (SLEEP) __nanosleep(64);
        if (mbar_test_parity(a, parity)) return true;
        if (global_ns() - t0 > limit_ns) return false;
    }
}

// ------------------------------------------------------------ memory

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// 16-byte async copy global -> shared; src_bytes 0 zero-fills without reading.
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;\n" ::"r"(dst), "l"(src),
                 "r"(src_bytes)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
    asm volatile("cp.async.commit_group;\n" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
    asm volatile("cp.async.wait_group 0;\n" ::: "memory");
}

// Hint: bring [src, src + bytes) into L2 (bytes a multiple of 16, src 16B aligned).
__device__ __forceinline__ void prefetch_l2_bulk(const void* src, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(src), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ void named_barrier(int id, int nthreads) {
    asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t addr) {
    uint4 v;
    asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];\n"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "r"(addr)
                 : "memory");
    return v;
}
__device__ __forceinline__ uint32_t lds32(uint32_t addr) {
    uint32_t v;
    asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void sts128(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};\n" ::"r"(addr), "r"(v.x), "r"(v.y),
                 "r"(v.z), "r"(v.w)
                 : "memory");
}

// ------------------------------------------------------------ dependent launch

// Programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while the previous kernel on the stream is still
// running; it must call pdl_wait() before reading anything that kernel (or any
// earlier work) produced.  pdl_wait() is a no-op for a normal launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
// Lets the next kernel on the stream (if launched as a dependent) start early.
// No memory clobber: the dependent's pdl_wait() still waits for this whole grid
// to finish and its writes to be visible, so no ordering is needed here.
__device__ __forceinline__ void pdl_launch_dependents() {
    asm volatile("griddepcontrol.launch_dependents;");
}

// ------------------------------------------------------------ fp32x2 (sm_100)

__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
// a - b as one packed fma: b * (-1) + a rounds the exact a - b once, so it is
// bit-identical to an IEEE subtraction.
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
    return __ffma2_rn(b, make_float2(-1.0f, -1.0f), a);
}

// One packed ternary word (16 two-bit codes t + 1; weight j at bits 8(j%4) +
// 2(j/4)) -> its 16 weights t as signed bytes in index order: bytes 4i..4i+3
// are ((w >> 2i) & 0x03030303) - 1 per byte.  The per-byte subtraction sets
// each byte's top bit first, so no borrow crosses a byte, and clears it after:
// a byte b <= 3 becomes (0x80 + b - 1) ^ 0x80 = b - 1 (mod 256).
__host__ __device__ __forceinline__ uint32_t ternary_bytes(uint32_t m) {
    return ((m | 0x80808080u) - 0x01010101u) ^ 0x80808080u;
}
__host__ __device__ __forceinline__ uint4 expand_ternary_word(uint32_t w) {
    return make_uint4(ternary_bytes(w & 0x03030303u), ternary_bytes((w >> 2) & 0x03030303u),
                      ternary_bytes((w >> 4) & 0x03030303u),
                      ternary_bytes((w >> 6) & 0x03030303u));
}

// bf16 pair (low half = first element) -> two fp32 (exact widening).
__device__ __forceinline__ float2 bf16x2_to_f2(uint32_t w) {
    return make_float2(__uint_as_float(w << 16), __uint_as_float(w & 0xffff0000u));
}

}  // namespace hbl
