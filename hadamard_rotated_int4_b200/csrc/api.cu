// api.cu -- the C ABI of libhbl: argument validation (before any CUDA call),
// device checks, workspace carving and dispatch to the sm_100a kernels.
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <unordered_map>

#include "hbl.h"
#include "hbl_launch.h"

namespace hbl {

namespace {

constexpr int kMaxDevices = 64;
struct DevInfo {
    std::atomic<int> state{0};  // 0 unknown, 1 ok, 2 unsupported
    int sms = 0;
};
DevInfo g_dev[kMaxDevices];

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool finite_nonneg(float e) { return isfinite(e) && e >= 0.0f; }
size_t up256(size_t v) { return (v + 255) & ~(size_t)255; }

hbl_status check_k(int K) {
    return (K >= 16 && K <= 32768 && is_pow2(K)) ? HBL_OK : HBL_ERR_SHAPE;
}
hbl_status check_n(int N) { return (N >= 16 && N % 16 == 0) ? HBL_OK : HBL_ERR_SHAPE; }

// Current device must be sm_100; caches the SM count.
hbl_status device(int* sms) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HBL_ERR_CUDA;
    if (dev < 0 || dev >= kMaxDevices) return HBL_ERR_CUDA;
    DevInfo& d = g_dev[dev];
    int st = d.state.load(std::memory_order_acquire);
    if (st == 0) {
        int major = 0, minor = 0, n = 0;
        if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return HBL_ERR_CUDA;
        d.sms = n;
        st = (major == 10 && minor == 0) ? 1 : 2;
        d.state.store(st, std::memory_order_release);
    }
    if (st != 1) return HBL_ERR_UNSUPPORTED_ARCH;
    *sms = d.sms;
    return HBL_OK;
}

// act_bits: 4 / 8 (row-major), HBL_ACT_INT4_BYTES (INT4 values one byte each,
// row-major) or HBL_ACT_INT{4,8}_I32 (interleaved bytes)
bool act_valid(int a) {
    return a == 4 || a == 8 || a == HBL_ACT_INT4_BYTES || a == HBL_ACT_INT4_I32 ||
           a == HBL_ACT_INT8_I32;
}
bool act_il(int a) { return a == HBL_ACT_INT4_I32 || a == HBL_ACT_INT8_I32; }
int act_base(int a) { return a & 0xFF; }
// bits each code occupies in memory (row-major layouts): 4 for packed nibbles, else 8
int act_width(int a) { return a == 4 ? 4 : 8; }
int codes_row_bytes(int K, int act_bits) { return act_width(act_bits) == 4 ? K / 2 : K; }

// Ternary-GEMM back ends.
// TMA: the one-SM TMA-fed kernel; PAIR: the paired-SM kernel; BIG (automatic
// choice for large batches): whichever of the two fills the device in fewer
// waves of tiles, the pair on a tie.
enum class Back { GEMV, SS, TS, TMA, DEC, WT, PAIR, BIG };

// The GEMV back end uses the row GEMV when K allows it and the tokens fit one
// launch; otherwise the split-K GEMV (8-token chunks).
bool rows_gemv(int64_t M, int K) { return gemv_rows_supported(K) && M <= gemv_rows_max_m(K); }

// Batches above this many tokens take the TMA-fed kernel (automatic choice).
constexpr int64_t kTmaMinM = 257;

bool path_valid(int path) { return path >= HBL_PATH_AUTO && path <= HBL_PATH_TC_PAIR; }

// Shapes the decode-batch tensor-core kernel takes (one-byte codes); whether a
// launch plan fits the device is checked again at launch, which falls back to
// the TMEM-activation kernel (its workspace is reserved for that).
bool dec_shape(int64_t M, int K) { return M >= 1 && M <= decode_mma_max_m() && K >= 512; }
// Automatic choice: batches of kDecMinM..kDecMaxM tokens take it (when its
// launch plan fits the device; otherwise the TMEM-activation kernel).
constexpr int64_t kDecMinM = 5, kDecMaxM = 128;

// The back end for M tokens under `path` (HBL_PATH_*); `bytes`: the codes are
// (or can be made) one byte each.
Back pick(int64_t M, int K, bool bytes, int path) {
    if (path == 1) return Back::SS;
    if (path == 2) return Back::GEMV;
    if (path == 3) return Back::TS;
    if (path == 4) return (bytes && K >= 128) ? Back::TMA : Back::TS;
    if (path == 5) return (bytes && dec_shape(M, K)) ? Back::DEC : Back::TS;
    if (path == 6) return (bytes && K >= 256) ? Back::WT : Back::TS;
    if (path == 7) return (bytes && K >= 128) ? Back::PAIR : Back::TS;
    // CUDA cores for a few tokens: the row GEMV where it takes the batch in one
    // launch; past that at K >= 16384 the tensor-core kernel is faster than the
    // split-K GEMV
    if (bytes && dec_shape(M, K) && M >= kDecMinM && M <= kDecMaxM) return Back::DEC;
    if (M <= gemv_max_m() && (rows_gemv(M, K) || K < 16384)) return Back::GEMV;
    if (bytes && K >= 128 && M >= kTmaMinM) return Back::BIG;
    return Back::TS;
}

// Large-batch back ends on expanded weights: whether the paired-SM kernel runs.
bool use_pair(Back b, int64_t M, int K, int N, int sms) {
    if (b == Back::PAIR) return gemm_pair_supported(K);
    if (b == Back::BIG) return gemm_pair_supported(K) && gemm_pair_preferred(M, N, sms);
    return false;
}
bool big_back(Back b) { return b == Back::TMA || b == Back::PAIR || b == Back::BIG; }

size_t backend_ws(Back b, int64_t M, int K, int N) {
    switch (b) {
        case Back::SS: return 0;
        case Back::TS: return gemm_ts_workspace(M, K, N);
        case Back::DEC: return gemm_ts_workspace(M, K, N);  // its fallback's
        case Back::WT: return 0;
        case Back::TMA:
        case Back::PAIR:
        case Back::BIG: return gemm_tma_workspace(K, N);
        case Back::GEMV:
        default: {
            if (rows_gemv(M, K)) return 0;  // the row GEMV needs no scratch
            const int64_t mchunk = M < gemv_max_m() ? M : gemv_max_m();
            return gemv_workspace(mchunk, K, N, 148);
        }
    }
}

// SM count for sizing when no device is queried yet (workspace queries must
// not need a GPU): the split factor only grows with SM count, so size for 148.
constexpr int kSizingSms = 148;

hbl_status run_gemm(Back b, const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t s,
                    int sms) {
    if (b == Back::SS) return launch_gemm_tc(a, s, sms);
    if (b == Back::TS) return launch_gemm_ts(a, ws, ws_bytes, s, sms);
    if (b == Back::TMA) return launch_gemm_tma(a, ws, ws_bytes, s, sms);
    if (b == Back::PAIR || b == Back::BIG)
        return use_pair(b, a.M, a.K, a.N, sms) ? launch_gemm_pair(a, ws, ws_bytes, s, sms)
                                               : launch_gemm_tma(a, ws, ws_bytes, s, sms);
    if (b == Back::WT) return launch_gemm_wt(a, s, sms);
    if (b == Back::DEC) {
        if (!a.interleaved && a.act_bits == 8 && decode_mma_supported(a.M, a.K, a.N, sms))
            return launch_decode_mma(a, s, sms);
        return launch_gemm_ts(a, ws, ws_bytes, s, sms);
    }
    if (rows_gemv(a.M, a.K)) {  // row GEMV in chunks of up to gemv_rows_max_m(K) tokens
        const int64_t step = gemv_rows_max_m(a.K);
        for (int64_t r0 = 0; r0 < a.M; r0 += step) {
            GemmArgs c = a;
            c.M = (a.M - r0) < step ? (a.M - r0) : step;
            c.codes = static_cast<const uint8_t*>(a.codes) + r0 * codes_row_bytes(a.K, a.act_bits);
            c.scales = a.scales + r0;
            c.rowsum = a.rowsum + r0;
            c.Y = a.Y + r0 * a.N;
            c.acc_out = a.acc_out ? a.acc_out + r0 * a.N : nullptr;
            hbl_status st = launch_gemv_rows(c, a.pdl, s);
            if (st != HBL_OK) return st;
        }
        return HBL_OK;
    }
    // split-K CUDA-core path in chunks of up to gemv_max_m() tokens (workspace reused in order)
    const int64_t step = gemv_max_m();
    for (int64_t r0 = 0; r0 < a.M; r0 += step) {
        GemmArgs c = a;
        c.M = (a.M - r0) < step ? (a.M - r0) : step;
        c.codes = static_cast<const uint8_t*>(a.codes) + r0 * codes_row_bytes(a.K, a.act_bits);
        c.scales = a.scales + r0;
        c.rowsum = a.rowsum + r0;
        c.Y = a.Y + r0 * a.N;
        c.acc_out = a.acc_out ? a.acc_out + r0 * a.N : nullptr;
        hbl_status st = launch_gemv(c, ws, ws_bytes, s, sms);
        if (st != HBL_OK) return st;
    }
    return HBL_OK;
}

// The fused forward's choice: back end, K1 mode and the codes layout it feeds.
struct FwdPlan {
    Back back;
    int k1_mode;
    int gemm_act_bits;  // value width the GEMM reads (4 or 8)
    bool interleaved;
};
FwdPlan forward_plan(int64_t M, int K, int act_bits, int path) {
    FwdPlan f;
    f.back = pick(M, K, true, path);
    f.interleaved = f.back == Back::TS;
    if (big_back(f.back) || f.back == Back::DEC || f.back == Back::WT) {
        f.k1_mode = act_bits == 4 ? 6 : 8;
        f.gemm_act_bits = 8;
    } else if (f.back == Back::TS) {
        f.k1_mode = act_bits == 4 ? 5 : 9;
        f.gemm_act_bits = 8;
    } else {
        f.k1_mode = act_bits;
        f.gemm_act_bits = act_bits;
    }
    return f;
}

}  // namespace

bool smem_attr_once(const void* func, int bytes) {
    static std::mutex mu;
    static std::unordered_map<uint64_t, int> done;  // (device, func) -> bytes set
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return false;
    const uint64_t key = (reinterpret_cast<uintptr_t>(func) << 6) ^ (uint64_t)dev;
    std::lock_guard<std::mutex> lock(mu);
    auto it = done.find(key);
    if (it != done.end() && it->second >= bytes) return true;
    if (cudaFuncSetAttribute(func, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
        cudaSuccess)
        return false;
    done[key] = bytes;
    return true;
}

}  // namespace hbl

using namespace hbl;

extern "C" {

const char* hbl_status_string(int status) {
    switch (status) {
        case HBL_OK: return "ok";
        case HBL_ERR_INVALID_ARG: return "invalid argument";
        case HBL_ERR_SHAPE: return "unsupported shape";
        case HBL_ERR_ALIGNMENT: return "pointer not 16-byte aligned";
        case HBL_ERR_UNSUPPORTED_ARCH: return "device is not sm_100";
        case HBL_ERR_WORKSPACE: return "workspace missing or too small";
        case HBL_ERR_CUDA: return "CUDA runtime error";
        case HBL_ERR_TIMEOUT: return "device-side wait timed out";
        default: return "unknown status";
    }
}

int hbl_version(void) { return 100; }

hbl_status hbl_workspace_size(int op, int M, int K, int N, int act_bits, size_t* bytes) {
    return hbl_workspace_size_path(op, M, K, N, act_bits, HBL_PATH_AUTO, bytes);
}

hbl_status hbl_workspace_size_path(int op, int M, int K, int N, int act_bits, int path,
                                   size_t* bytes) {
    if (bytes == nullptr || !path_valid(path)) return HBL_ERR_INVALID_ARG;
    *bytes = 0;
    switch (op) {
        case HBL_OP_PACK_TERNARY:
            if (N < 1) return HBL_ERR_SHAPE;
            if (check_k(K) != HBL_OK) return HBL_ERR_SHAPE;
            *bytes = pack_ternary_workspace(N, K);
            return HBL_OK;
        case HBL_OP_TERNARY_GEMM:
        case HBL_OP_HBITLINEAR_FORWARD:
        case HBL_OP_HBITLINEAR_FORWARD_HOSTIO: {
            if (M < 0 || check_k(K) != HBL_OK || check_n(N) != HBL_OK) return HBL_ERR_SHAPE;
            if (!act_valid(act_bits)) return HBL_ERR_INVALID_ARG;
            if (op != HBL_OP_TERNARY_GEMM && act_bits != 4 && act_bits != 8)
                return HBL_ERR_INVALID_ARG;
            size_t b;
            if (op == HBL_OP_TERNARY_GEMM)
                b = act_il(act_bits)
                        ? up256(gemm_ts_workspace(M, K, N))
                        : up256(backend_ws(pick(M, K, act_width(act_bits) == 8, path), M, K, N));
            else
                b = up256(backend_ws(forward_plan(M, K, act_bits, path).back, M, K, N));
            if (op != HBL_OP_TERNARY_GEMM) {
                b += up256((size_t)((M + 31) & ~31) * K);  // codes, one byte each, rows padded to 32
                b += up256((size_t)M * 4) * 2;                         // scales, rowsum
            }
            if (op == HBL_OP_HBITLINEAR_FORWARD_HOSTIO) {
                b += up256((size_t)M * K * 2);  // device copy of X
                b += up256((size_t)M * N * 2);  // device copy of Y
            }
            *bytes = b;
            return HBL_OK;
        }
        default: return HBL_ERR_INVALID_ARG;
    }
}

hbl_status hbl_pack_ternary(const float* W, int N, int K, float eps, uint32_t* W_packed,
                            float* alpha, void* ws, size_t ws_bytes, void* stream) {
    if (!W || !W_packed || !alpha) return HBL_ERR_INVALID_ARG;
    if (!finite_nonneg(eps)) return HBL_ERR_INVALID_ARG;
    if (N < 1 || check_k(K) != HBL_OK) return HBL_ERR_SHAPE;
    if (!aligned16(W) || !aligned16(W_packed) || !aligned16(alpha)) return HBL_ERR_ALIGNMENT;
    if (ws == nullptr || ws_bytes < pack_ternary_workspace(N, K)) return HBL_ERR_WORKSPACE;
    if (!aligned16(ws)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_pack_ternary(W, N, K, eps, W_packed, alpha, ws,
                               static_cast<cudaStream_t>(stream), sms);
}

// K1 mode writing the codes layout `act_bits` names.
static int k1_mode_of(int act_bits) {
    if (act_il(act_bits)) return act_base(act_bits) == 4 ? 5 : 9;
    if (act_bits == HBL_ACT_INT4_BYTES) return 6;
    return act_bits;
}

// Scalars and shapes first; pointers only matter when there is work (M > 0).
static hbl_status check_act_args(const uint16_t* X, const float* gain, int M, int K,
                                 float norm_eps) {
    if (!finite_nonneg(norm_eps)) return HBL_ERR_INVALID_ARG;
    if (M < 0 || check_k(K) != HBL_OK) return HBL_ERR_SHAPE;
    if (M == 0) return HBL_OK;
    if (!X) return HBL_ERR_INVALID_ARG;
    if (!aligned16(X) || (gain && !aligned16(gain))) return HBL_ERR_ALIGNMENT;
    return HBL_OK;
}

hbl_status hbl_norm_fwht(const uint16_t* X, const float* gain, int M, int K, float norm_eps,
                         float* V, int32_t* dev_status, void* stream) {
    (void)dev_status;
    hbl_status st = check_act_args(X, gain, M, K, norm_eps);
    if (st != HBL_OK) return st;
    if (M == 0) return HBL_OK;
    if (!V) return HBL_ERR_INVALID_ARG;
    if (!aligned16(V)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return launch_norm_fwht_quant(X, gain, M, K, norm_eps, 0.f, 0, nullptr, nullptr, nullptr, V,
                                  static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_norm_fwht_quant(const uint16_t* X, const float* gain, int M, int K,
                               float norm_eps, float quant_eps, int act_bits, void* codes,
                               float* scales, int32_t* rowsum, int32_t* dev_status,
                               void* stream) {
    (void)dev_status;
    hbl_status st = check_act_args(X, gain, M, K, norm_eps);
    if (st != HBL_OK) return st;
    if (!act_valid(act_bits)) return HBL_ERR_INVALID_ARG;
    if (!finite_nonneg(quant_eps)) return HBL_ERR_INVALID_ARG;
    if (M == 0) return HBL_OK;
    if (!codes || !scales) return HBL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || (rowsum && !aligned16(rowsum)))
        return HBL_ERR_ALIGNMENT;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return launch_norm_fwht_quant(X, gain, M, K, norm_eps, quant_eps, k1_mode_of(act_bits),
                                  codes, scales, rowsum, nullptr,
                                  static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_ternary_gemm(const void* codes, const float* scales, const int32_t* rowsum,
                            int act_bits, int M, int K, const uint32_t* W_packed,
                            const float* alpha, int N, uint16_t* Y, int32_t* acc_out,
                            void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
    return hbl_ternary_gemm_path(codes, scales, rowsum, act_bits, M, K, W_packed, alpha, N, Y,
                                 acc_out, ws, ws_bytes, dev_status, HBL_PATH_AUTO, stream);
}

hbl_status hbl_ternary_gemm_path(const void* codes, const float* scales, const int32_t* rowsum,
                                 int act_bits, int M, int K, const uint32_t* W_packed,
                                 const float* alpha, int N, uint16_t* Y, int32_t* acc_out,
                                 void* ws, size_t ws_bytes, int32_t* dev_status, int path,
                                 void* stream) {
    if (!act_valid(act_bits) || !path_valid(path)) return HBL_ERR_INVALID_ARG;
    if (M < 0 || check_k(K) != HBL_OK || check_n(N) != HBL_OK) return HBL_ERR_SHAPE;
    if (M == 0) return HBL_OK;
    if (!codes || !scales || !rowsum || !W_packed || !alpha || !Y) return HBL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(rowsum) || !aligned16(W_packed) ||
        !aligned16(alpha) || !aligned16(Y) || (acc_out && !aligned16(acc_out)) ||
        (dev_status && !aligned16(dev_status)))
        return HBL_ERR_ALIGNMENT;
    const Back bk = act_il(act_bits) ? Back::TS : pick(M, K, act_width(act_bits) == 8, path);
    const size_t need = backend_ws(bk, M, K, N);
    if (need > 0 && (ws == nullptr || ws_bytes < need)) return HBL_ERR_WORKSPACE;
    if (ws && !aligned16(ws)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    GemmArgs a{codes, scales, rowsum, act_width(act_bits), M, K, W_packed, alpha, N, Y, acc_out,
               dev_status};
    a.interleaved = act_il(act_bits);  // interleaved one-byte codes: the TMEM-activation kernel
    return run_gemm(bk, a, ws, ws_bytes, static_cast<cudaStream_t>(stream), sms);
}

static hbl_status forward_impl(const uint16_t* X, const float* gain, int M, int K, int N,
                               const uint32_t* W_packed, const float* alpha, int act_bits,
                               float norm_eps, float quant_eps, uint16_t* Y, uint8_t* ws,
                               size_t ws_bytes, int32_t* dev_status, cudaStream_t s, int sms,
                               unsigned variant, int path) {
    // Decode batches: one kernel quantises and multiplies (no workspace used);
    // a forced GEMM path keeps the two-kernel forward.
    if (path == HBL_PATH_AUTO && decode_fused_supported(M, K, N, act_bits, variant, sms)) {
        DecodeArgs d{X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps, quant_eps, Y,
                     dev_status};
        return launch_decode_fused(d, s, sms);
    }
    // For the default tensor-core kernel the codes stay in workspace one per
    // byte (INT4 values too) in the 32-row interleaved layout, so the GEMM
    // loads them coalesced and without widening; other back ends take the
    // public row-major layouts.
    const size_t cb = up256((size_t)((M + 31) & ~31) * K);
    const size_t sb = up256((size_t)M * 4);
    uint8_t* codes = ws;
    float* scales = reinterpret_cast<float*>(ws + cb);
    int32_t* rowsum = reinterpret_cast<int32_t*>(ws + cb + sb);
    uint8_t* gws = ws + cb + 2 * sb;
    const size_t gws_bytes = ws_bytes - (cb + 2 * sb);
    // Other decode batches of up to 8 tokens at K = 16384: K1 (one byte per
    // code, row-major), then the one-kernel forward's GEMV half, its weight
    // rows streaming into shared memory under K1.
    if (path == HBL_PATH_AUTO && M < kDecMinM && decode_gemv_supported(M, K, N, sms)) {
        hbl_status st = launch_norm_fwht_quant(X, gain, M, K, norm_eps, quant_eps,
                                               act_bits == 4 ? 6 : 8, codes, scales, rowsum,
                                               nullptr, s, sms, variant);
        if (st != HBL_OK) return st;
        GemvArgs g{codes, scales, rowsum, M, K, N, W_packed, alpha, Y, dev_status};
        return launch_decode_gemv(g, s, sms);
    }
    FwdPlan f = forward_plan(M, K, act_bits, path);
    if (f.back == Back::DEC && path == HBL_PATH_AUTO && !decode_mma_supported(M, K, N, sms)) {
        // no decode plan fits (e.g. too many tokens for the shared memory left
        // next to the weights): the TMEM-activation kernel with its codes layout
        f.back = Back::TS;
        f.k1_mode = act_bits == 4 ? 5 : 9;
        f.interleaved = true;
    }
    // The GEMMs on expanded weights get them from K1, which widens the packed
    // words beside its rows (its FP32 work leaves HBM bandwidth to spare), so
    // the GEMM follows K1 directly -- where the rows are enough to carry the
    // expansion; other shapes and the norm variants keep the separate
    // expansion kernel.
    const bool expand = big_back(f.back) &&
                        (variant & (HBL_NORM_NO_HADAMARD | HBL_NORM_LAYERNORM)) == 0 &&
                        norm_quant_expand_rides_along(M, K, N, sms);
    if (expand && gws_bytes < gemm_tma_workspace(K, N)) return HBL_ERR_WORKSPACE;
    int8_t* wexp = reinterpret_cast<int8_t*>(gws);
    hbl_status st = launch_norm_fwht_quant(X, gain, M, K, norm_eps, quant_eps, f.k1_mode, codes,
                                           scales, rowsum, nullptr, s, sms, variant,
                                           expand ? W_packed : nullptr, expand ? N : 0,
                                           expand ? wexp : nullptr);
    if (st != HBL_OK) return st;
    GemmArgs a{codes, scales, rowsum, f.gemm_act_bits, M, K, W_packed, alpha, N, Y, nullptr,
               dev_status};
    a.interleaved = f.interleaved;
    a.pdl = true;  // right after K1 on the same stream
    if (expand)
        return use_pair(f.back, M, K, N, sms) ? launch_gemm_pair_s8w(a, wexp, s)
                                              : launch_gemm_tma_s8w(a, wexp, s, sms);
    return run_gemm(f.back, a, gws, gws_bytes, s, sms);
}

static hbl_status check_forward(const uint16_t* X, const float* gain, int M, int K, int N,
                                const uint32_t* W_packed, const float* alpha, int act_bits,
                                float norm_eps, float quant_eps, const uint16_t* Y, void* ws,
                                size_t ws_bytes, int32_t* dev_status, int op, bool host_xy,
                                int path) {
    if (act_bits != 4 && act_bits != 8) return HBL_ERR_INVALID_ARG;
    if (!path_valid(path)) return HBL_ERR_INVALID_ARG;
    if (!finite_nonneg(norm_eps) || !finite_nonneg(quant_eps)) return HBL_ERR_INVALID_ARG;
    if (M < 0 || check_k(K) != HBL_OK || check_n(N) != HBL_OK) return HBL_ERR_SHAPE;
    if (M == 0) return HBL_OK;
    if (!X || !W_packed || !alpha || !Y) return HBL_ERR_INVALID_ARG;
    if ((!host_xy && (!aligned16(X) || !aligned16(Y))) || (gain && !aligned16(gain)) ||
        !aligned16(W_packed) || !aligned16(alpha) || (dev_status && !aligned16(dev_status)))
        return HBL_ERR_ALIGNMENT;
    size_t need = 0;
    hbl_workspace_size_path(op, M, K, N, act_bits, path, &need);
    if (ws == nullptr || ws_bytes < need) return HBL_ERR_WORKSPACE;
    if (!aligned16(ws)) return HBL_ERR_ALIGNMENT;
    return HBL_OK;
}

hbl_status hbl_hbitlinear_forward(const uint16_t* X, const float* gain, int M, int K, int N,
                                  const uint32_t* W_packed, const float* alpha, int act_bits,
                                  float norm_eps, float quant_eps, uint16_t* Y, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream) {
    return hbl_hbitlinear_forward_path(X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps,
                                       quant_eps, Y, ws, ws_bytes, dev_status, HBL_PATH_AUTO,
                                       stream);
}

hbl_status hbl_hbitlinear_forward_path(const uint16_t* X, const float* gain, int M, int K, int N,
                                       const uint32_t* W_packed, const float* alpha,
                                       int act_bits, float norm_eps, float quant_eps,
                                       uint16_t* Y, void* ws, size_t ws_bytes,
                                       int32_t* dev_status, int path, void* stream) {
    hbl_status st = check_forward(X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps,
                                  quant_eps, Y, ws, ws_bytes, dev_status,
                                  HBL_OP_HBITLINEAR_FORWARD, false, path);
    if (st != HBL_OK) return st;
    if (M == 0) return HBL_OK;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return forward_impl(X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps, quant_eps, Y,
                        static_cast<uint8_t*>(ws), ws_bytes, dev_status,
                        static_cast<cudaStream_t>(stream), sms, 0, path);
}

namespace {
// Per-device copy streams and events of the host-buffer forward: the input
// copies, the layer and the output copies of consecutive row chunks overlap.
constexpr int kMaxChunks = 8;
struct CopyLanes {
    cudaStream_t in = nullptr, out = nullptr;
    cudaEvent_t start = nullptr, done = nullptr;
    cudaEvent_t in_ev[kMaxChunks] = {}, fwd_ev[kMaxChunks] = {};
    bool ready = false;
};
CopyLanes g_lanes[kMaxDevices];
std::mutex g_lanes_mu;

hbl_status copy_lanes(CopyLanes** out) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return HBL_ERR_CUDA;
    CopyLanes& c = g_lanes[dev];
    if (!c.ready) {
        const unsigned ef = cudaEventDisableTiming;
        if (cudaStreamCreateWithFlags(&c.in, cudaStreamNonBlocking) != cudaSuccess ||
            cudaStreamCreateWithFlags(&c.out, cudaStreamNonBlocking) != cudaSuccess ||
            cudaEventCreateWithFlags(&c.start, ef) != cudaSuccess ||
            cudaEventCreateWithFlags(&c.done, ef) != cudaSuccess)
            return HBL_ERR_CUDA;
        for (int i = 0; i < kMaxChunks; ++i)
            if (cudaEventCreateWithFlags(&c.in_ev[i], ef) != cudaSuccess ||
                cudaEventCreateWithFlags(&c.fwd_ev[i], ef) != cudaSuccess)
                return HBL_ERR_CUDA;
        c.ready = true;
    }
    *out = &c;
    return HBL_OK;
}
}  // namespace

hbl_status hbl_hbitlinear_forward_hostio(const uint16_t* X_host, const float* gain, int M,
                                         int K, int N, const uint32_t* W_packed,
                                         const float* alpha, int act_bits, float norm_eps,
                                         float quant_eps, uint16_t* Y_host, void* ws,
                                         size_t ws_bytes, int32_t* dev_status, void* stream) {
    hbl_status st = check_forward(X_host, gain, M, K, N, W_packed, alpha, act_bits, norm_eps,
                                  quant_eps, Y_host, ws, ws_bytes, dev_status,
                                  HBL_OP_HBITLINEAR_FORWARD_HOSTIO, true, HBL_PATH_AUTO);
    if (st != HBL_OK) return st;
    if (M == 0) return HBL_OK;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const size_t xb = up256((size_t)M * K * 2), yb = up256((size_t)M * N * 2);
    uint8_t* w8 = static_cast<uint8_t*>(ws);
    uint16_t* Xd = reinterpret_cast<uint16_t*>(w8);
    uint16_t* Yd = reinterpret_cast<uint16_t*>(w8 + xb);
    uint8_t* fws = w8 + xb + yb;
    const size_t fws_bytes = ws_bytes - xb - yb;
    const FwdPlan plan = forward_plan(M, K, act_bits, HBL_PATH_AUTO);
    // Batches on the TMA-fed GEMM run in row chunks of at least kTmaMinM rows
    // (so every chunk keeps that plan and fits its workspace): chunk c's input
    // copy, its layer and chunk c-1's output copy overlap on three streams.
    const bool big = big_back(plan.back) || plan.back == Back::WT;
    const int nch = big ? (int)((int64_t)M / kTmaMinM < kMaxChunks ? (int64_t)M / kTmaMinM
                                                                   : kMaxChunks)
                        : 1;
    if (nch <= 1) {
        if (cudaMemcpyAsync(Xd, X_host, (size_t)M * K * 2, cudaMemcpyHostToDevice, s) !=
            cudaSuccess)
            return HBL_ERR_CUDA;
        st = forward_impl(Xd, gain, M, K, N, W_packed, alpha, act_bits, norm_eps, quant_eps, Yd,
                          fws, fws_bytes, dev_status, s, sms, 0, HBL_PATH_AUTO);
        if (st != HBL_OK) return st;
        if (cudaMemcpyAsync(Y_host, Yd, (size_t)M * N * 2, cudaMemcpyDeviceToHost, s) !=
            cudaSuccess)
            return HBL_ERR_CUDA;
        return HBL_OK;
    }
    std::lock_guard<std::mutex> lock(g_lanes_mu);  // the lanes' events are shared
    CopyLanes* c = nullptr;
    if ((st = copy_lanes(&c)) != HBL_OK) return st;
    // workspace of one chunk: codes (rows padded to 32), scales, rowsum, then the
    // expanded weights (written once, shared by the chunks)
    const int64_t rows = ((int64_t)M + nch - 1) / nch;
    const size_t cb = up256((size_t)((rows + 31) & ~31) * K), sb = up256((size_t)rows * 4);
    uint8_t* codes = fws;
    float* scales = reinterpret_cast<float*>(fws + cb);
    int32_t* rowsum = reinterpret_cast<int32_t*>(fws + cb + sb);
    int8_t* wexp = reinterpret_cast<int8_t*>(fws + cb + 2 * sb);
    const bool expand = big_back(plan.back);
    if (cb + 2 * sb + (expand ? gemm_tma_workspace(K, N) : 0) > fws_bytes)
        return HBL_ERR_WORKSPACE;
#define HBL_CK(x) \
    if ((x) != cudaSuccess) return HBL_ERR_CUDA
    HBL_CK(cudaEventRecord(c->start, s));
    HBL_CK(cudaStreamWaitEvent(c->in, c->start, 0));
    HBL_CK(cudaStreamWaitEvent(c->out, c->start, 0));
    if (expand && (st = launch_expand_ternary(W_packed, N, K, wexp, s, sms)) != HBL_OK)
        return st;
    for (int i = 0; i < nch; ++i) {
        const int64_t r0 = (int64_t)i * rows;
        const int64_t mc = ((int64_t)M - r0) < rows ? ((int64_t)M - r0) : rows;
        if (mc <= 0) break;
        HBL_CK(cudaMemcpyAsync(Xd + r0 * K, X_host + r0 * K, (size_t)mc * K * 2,
                               cudaMemcpyHostToDevice, c->in));
        HBL_CK(cudaEventRecord(c->in_ev[i], c->in));
        HBL_CK(cudaStreamWaitEvent(s, c->in_ev[i], 0));
        if ((st = launch_norm_fwht_quant(Xd + r0 * K, gain, mc, K, norm_eps, quant_eps,
                                         plan.k1_mode, codes, scales, rowsum, nullptr, s, sms)) !=
            HBL_OK)
            return st;
        GemmArgs a{codes, scales, rowsum, plan.gemm_act_bits, mc, K, W_packed, alpha, N,
                   Yd + r0 * N, nullptr, dev_status};
        a.pdl = true;  // right after K1 on the same stream
        if ((st = use_pair(plan.back, mc, K, N, sms) ? launch_gemm_pair_s8w(a, wexp, s)
                   : expand ? launch_gemm_tma_s8w(a, wexp, s, sms)
                            : launch_gemm_wt(a, s, sms)) != HBL_OK)
            return st;
        HBL_CK(cudaEventRecord(c->fwd_ev[i], s));
        HBL_CK(cudaStreamWaitEvent(c->out, c->fwd_ev[i], 0));
        HBL_CK(cudaMemcpyAsync(Y_host + r0 * N, Yd + r0 * N, (size_t)mc * N * 2,
                               cudaMemcpyDeviceToHost, c->out));
    }
    HBL_CK(cudaEventRecord(c->done, c->out));
    HBL_CK(cudaStreamWaitEvent(s, c->done, 0));  // later work on `stream` follows the copies
#undef HBL_CK
    return HBL_OK;
}

static bool flags_valid(unsigned f) {
    return (f & ~(unsigned)(HBL_NORM_LAYERNORM | HBL_NORM_NO_HADAMARD)) == 0;
}

hbl_status hbl_norm_transform(const uint16_t* X, const float* gain, int M, int K, float norm_eps,
                              unsigned flags, float* V, int32_t* dev_status, void* stream) {
    (void)dev_status;
    if (!flags_valid(flags)) return HBL_ERR_INVALID_ARG;
    hbl_status st = check_act_args(X, gain, M, K, norm_eps);
    if (st != HBL_OK) return st;
    if (M == 0) return HBL_OK;
    if (!V) return HBL_ERR_INVALID_ARG;
    if (!aligned16(V)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return launch_norm_fwht_quant(X, gain, M, K, norm_eps, 0.f, 0, nullptr, nullptr, nullptr, V,
                                  static_cast<cudaStream_t>(stream), sms, flags);
}

hbl_status hbl_norm_quant(const uint16_t* X, const float* gain, int M, int K, float norm_eps,
                          float quant_eps, int act_bits, unsigned flags, void* codes,
                          float* scales, int32_t* rowsum, int32_t* dev_status, void* stream) {
    (void)dev_status;
    if (!flags_valid(flags)) return HBL_ERR_INVALID_ARG;
    hbl_status st = check_act_args(X, gain, M, K, norm_eps);
    if (st != HBL_OK) return st;
    if (!act_valid(act_bits)) return HBL_ERR_INVALID_ARG;
    if (!finite_nonneg(quant_eps)) return HBL_ERR_INVALID_ARG;
    if (M == 0) return HBL_OK;
    if (!codes || !scales) return HBL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || (rowsum && !aligned16(rowsum)))
        return HBL_ERR_ALIGNMENT;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return launch_norm_fwht_quant(X, gain, M, K, norm_eps, quant_eps, k1_mode_of(act_bits),
                                  codes, scales, rowsum, nullptr,
                                  static_cast<cudaStream_t>(stream), sms, flags);
}

hbl_status hbl_bitlinear_forward(const uint16_t* X, const float* gain, int M, int K, int N,
                                 const uint32_t* W_packed, const float* alpha, int act_bits,
                                 unsigned flags, float norm_eps, float quant_eps, uint16_t* Y,
                                 void* ws, size_t ws_bytes, int32_t* dev_status, void* stream) {
    if (!flags_valid(flags)) return HBL_ERR_INVALID_ARG;
    hbl_status st = check_forward(X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps,
                                  quant_eps, Y, ws, ws_bytes, dev_status,
                                  HBL_OP_HBITLINEAR_FORWARD, false, HBL_PATH_AUTO);
    if (st != HBL_OK) return st;
    if (M == 0) return HBL_OK;
    int sms = 0;
    if ((st = device(&sms)) != HBL_OK) return st;
    return forward_impl(X, gain, M, K, N, W_packed, alpha, act_bits, norm_eps, quant_eps, Y,
                        static_cast<uint8_t*>(ws), ws_bytes, dev_status,
                        static_cast<cudaStream_t>(stream), sms, flags, HBL_PATH_AUTO);
}

hbl_status hbl_rotate_weights(const float* W, const float* signs, int N, int K, float* W_rot,
                              int32_t* dev_status, void* stream) {
    (void)dev_status;
    if (N < 0 || check_k(K) != HBL_OK) return HBL_ERR_SHAPE;
    if (N == 0) return HBL_OK;
    if (!W || !W_rot) return HBL_ERR_INVALID_ARG;
    if (!aligned16(W) || !aligned16(W_rot) || (signs && !aligned16(signs)))
        return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_rotate_weights(W, signs, N, K, W_rot, static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_kv_quant(const uint16_t* X, int64_t rows, int D, int bits, float eps,
                        uint8_t* codes, float* scales, int32_t* dev_status, void* stream) {
    (void)dev_status;
    if (!finite_nonneg(eps)) return HBL_ERR_INVALID_ARG;
    if (bits != 2 && bits != 3 && bits != 4 && bits != 8) return HBL_ERR_INVALID_ARG;
    if (rows < 0 || (D != 32 && D != 64 && D != 128 && D != 256)) return HBL_ERR_SHAPE;
    if (rows == 0) return HBL_OK;
    if (!X || !codes || !scales) return HBL_ERR_INVALID_ARG;
    if (!aligned16(X) || !aligned16(codes) || !aligned16(scales)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_kv_quant(X, rows, D, bits, eps, codes, scales,
                           static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_expand_ternary(const uint32_t* W_packed, int N, int K, int8_t* W_s8,
                              int32_t* dev_status, void* stream) {
    (void)dev_status;
    if (N < 0 || check_k(K) != HBL_OK) return HBL_ERR_SHAPE;
    if (N == 0) return HBL_OK;
    if (!W_packed || !W_s8) return HBL_ERR_INVALID_ARG;
    if (!aligned16(W_packed) || !aligned16(W_s8)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_expand_ternary(W_packed, N, K, W_s8, static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_ternary_gemm_s8w(const void* codes, const float* scales, int act_bits, int M,
                                int K, const int8_t* W_s8, const float* alpha, int N, uint16_t* Y,
                                int32_t* acc_out, int32_t* dev_status, void* stream) {
    if (act_bits != 8 && act_bits != HBL_ACT_INT4_BYTES) return HBL_ERR_INVALID_ARG;
    if (M < 0 || check_k(K) != HBL_OK || K < 128 || check_n(N) != HBL_OK) return HBL_ERR_SHAPE;
    if (M == 0) return HBL_OK;
    if (!codes || !scales || !W_s8 || !alpha || !Y) return HBL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(W_s8) || !aligned16(alpha) ||
        !aligned16(Y) || (acc_out && !aligned16(acc_out)) ||
        (dev_status && !aligned16(dev_status)))
        return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    GemmArgs a{codes, scales, nullptr, 8, M, K, nullptr, alpha, N, Y, acc_out, dev_status};
    if (use_pair(Back::BIG, M, K, N, sms))
        return launch_gemm_pair_s8w(a, W_s8, static_cast<cudaStream_t>(stream));
    return launch_gemm_tma_s8w(a, W_s8, static_cast<cudaStream_t>(stream), sms);
}

hbl_status hbl_selftest_bounded_wait(int arrive, int timeout_us, int32_t* dev_status,
                                     void* stream) {
    if (dev_status == nullptr) return HBL_ERR_INVALID_ARG;
    if (timeout_us < 1 || timeout_us > 1000000) return HBL_ERR_INVALID_ARG;
    if (!aligned16(dev_status)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_bounded_wait_probe(arrive, timeout_us, dev_status,
                                     static_cast<cudaStream_t>(stream));
}

hbl_status hbl_probe_tc_int8(int ctas, int mmas_per_cta, int32_t* dev_status, void* stream) {
    if (dev_status == nullptr) return HBL_ERR_INVALID_ARG;
    if (ctas < 1 || ctas > 4096 || mmas_per_cta < 1 || mmas_per_cta > (1 << 22))
        return HBL_ERR_INVALID_ARG;
    if (!aligned16(dev_status)) return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    return launch_tc_int8_probe(ctas, mmas_per_cta, dev_status, static_cast<cudaStream_t>(stream));
}

// Allocation-free ternary GEMV: the CUDA-core split-K path with its partial
// sums in the library's fixed 2 MiB device array instead of caller workspace.
hbl_status hbl_ternary_gemv_noalloc(const void* codes, const float* scales,
                                    const int32_t* rowsum, int act_bits, int M, int K,
                                    const uint32_t* W_packed, const float* alpha, int N,
                                    uint16_t* Y, int32_t* acc_out, int32_t* dev_status,
                                    void* stream) {
    if (act_bits != 4 && act_bits != 8) return HBL_ERR_INVALID_ARG;
    if (M < 0 || check_k(K) != HBL_OK || check_n(N) != HBL_OK) return HBL_ERR_SHAPE;
    const int64_t mchunk = M < gemv_max_m() ? M : gemv_max_m();
    if (gemv_workspace(mchunk, K, N, kSizingSms) > gemv_noalloc_scratch_bytes())
        return HBL_ERR_WORKSPACE;  // shape needs more than the fixed scratch holds
    if (M == 0) return HBL_OK;
    if (!codes || !scales || !rowsum || !W_packed || !alpha || !Y) return HBL_ERR_INVALID_ARG;
    if (!aligned16(codes) || !aligned16(scales) || !aligned16(rowsum) || !aligned16(W_packed) ||
        !aligned16(alpha) || !aligned16(Y) || (acc_out && !aligned16(acc_out)) ||
        (dev_status && !aligned16(dev_status)))
        return HBL_ERR_ALIGNMENT;
    int sms = 0;
    hbl_status st = device(&sms);
    if (st != HBL_OK) return st;
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return HBL_ERR_CUDA;
    void* scratch = gemv_noalloc_scratch(dev);
    if (scratch == nullptr) return HBL_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int64_t step = gemv_max_m();
    for (int64_t r0 = 0; r0 < M; r0 += step) {
        GemmArgs c{codes, scales, rowsum, act_bits, M, K, W_packed, alpha, N, Y, acc_out,
                   dev_status};
        c.M = (M - r0) < step ? (M - r0) : step;
        c.codes = static_cast<const uint8_t*>(codes) + r0 * codes_row_bytes(K, act_bits);
        c.scales = scales + r0;
        c.rowsum = rowsum + r0;
        c.Y = Y + r0 * N;
        c.acc_out = acc_out ? acc_out + r0 * N : nullptr;
        st = launch_gemv(c, scratch, gemv_noalloc_scratch_bytes(), s, sms);
        if (st != HBL_OK) return st;
    }
    return HBL_OK;
}

}  // extern "C"
