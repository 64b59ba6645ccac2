// hbl_launch.h -- host-side launchers of the sm_100a kernels (internal to libhbl).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "hbl.h"

namespace hbl {

// Sets the dynamic shared-memory limit of `func` once per device (idempotent).
bool smem_attr_once(const void* func, int bytes);

// Launch with programmatic stream serialisation (the kernel must pdl_wait()
// before reading inputs).  Returns HBL_ERR_CUDA on failure.
template <class... KArgs, class... Args>
hbl_status launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                      cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, static_cast<KArgs>(args)...) == cudaSuccess ? HBL_OK
                                                                                         : HBL_ERR_CUDA;
}

// K1: mode 0 writes fp32 V; modes 4 / 8 write INT4 (packed nibbles) / INT8 codes +
// scales (+ rowsum); mode 6 writes INT4 codes one per byte, row-major;
// modes 5 / 9 write INT4 / INT8 codes one per byte in the
// 32-row interleaved layout of the fused forward.  variant: HBL_NORM_* bits
// (LayerNorm instead of RMSNorm, no Hadamard transform).  Modes 6 and 8 with
// W_packed set also widen the N x K packed ternary weights to one signed byte
// each into W_s8 (N*K bytes, 16-byte aligned; K a multiple of 128, N of 16), beside the
// rows -- the large-batch forward's operand, without a kernel of its own.
hbl_status launch_norm_fwht_quant(const uint16_t* X, const float* gain, int64_t M, int K,
                                  float norm_eps, float quant_eps, int mode, void* codes,
                                  float* scales, int32_t* rowsum, float* V, cudaStream_t stream,
                                  int num_sms, unsigned variant = 0,
                                  const uint32_t* W_packed = nullptr, int N = 0,
                                  int8_t* W_s8 = nullptr);
// Whether that expansion rides along K1's rows for this shape (nearly all of it
// inside the row loop); otherwise the separate expansion kernel is faster.
bool norm_quant_expand_rides_along(int64_t M, int K, int N, int num_sms);

// K6: the whole forward of a decode batch in one kernel (quantiser and ternary
// GEMV fused; see k6_decode_fused.cuh).  Supported for M <= 16384 / K tokens
// (K = 4096 / 8192 / 16384), RMSNorm + transform (no variant bits), when the
// CTA's shared memory fits (decode_fused_supported).
struct DecodeArgs {
    const uint16_t* X;
    const float* gain;
    int M, K, N;
    const uint32_t* W_packed;
    const float* alpha;
    int act_bits;
    float norm_eps, quant_eps;
    uint16_t* Y;
    int32_t* status;
};
// Weight rows per CTA for N rows: spread evenly over at most num_sms CTAs.
int decode_fused_rows(int N, int num_sms);

// K6's GEMV half alone, after K1 (programmatic dependent launch; the weight
// rows stream into shared memory under K1): codes one byte each, row-major
// [M][K]; M <= 8 at K = 16384, when the CTA's weight rows fit its shared
// memory (decode_gemv_supported).
struct GemvArgs {
    const uint8_t* codes;
    const float* scales;
    const int32_t* rowsum;
    int M, K, N;
    const uint32_t* W_packed;
    const float* alpha;
    uint16_t* Y;
    int32_t* status;
};
bool decode_gemv_supported(int M, int K, int N, int num_sms);
hbl_status launch_decode_gemv(const GemvArgs& g, cudaStream_t stream, int num_sms);
bool decode_fused_supported(int M, int K, int N, int act_bits, unsigned variant, int num_sms);
hbl_status launch_decode_fused(const DecodeArgs& d, cudaStream_t stream, int num_sms);

// K4: offline weight rotation W_rot[n] = FWHT(W[n] * signs) * c_K (in place allowed).
hbl_status launch_rotate_weights(const float* W, const float* signs, int N, int K, float* W_rot,
                                 cudaStream_t stream, int num_sms);

// K5: per-head absmax quantiser of Q/K/V states to unsigned `bits`-bit codes.
hbl_status launch_kv_quant(const uint16_t* X, int64_t rows, int D, int bits, float eps,
                           uint8_t* codes, float* scales, cudaStream_t stream, int num_sms);

// Self-test of the bounded-wait failure path (see k9_selftest.cu).
hbl_status launch_bounded_wait_probe(int arrive, int timeout_us, int32_t* status,
                                     cudaStream_t stream);

// Dense INT8 tensor-core rate probe (see k9_tc_probe.cu).
hbl_status launch_tc_int8_probe(int ctas, int mmas_per_cta, int32_t* status, cudaStream_t stream);

// K0: absmean ternarisation + 2-bit packing (K a power of two).
size_t pack_ternary_workspace(int N, int K);
hbl_status launch_pack_ternary(const float* W, int N, int K, float eps, uint32_t* W_packed,
                               float* alpha, void* ws, cudaStream_t stream, int num_sms);

// Ternary GEMM back ends.  All compute acc = sum_k q*t exactly, Y = bf16(acc*alpha*s).
struct GemmArgs {
    const void* codes;
    const float* scales;
    const int32_t* rowsum;
    int act_bits;
    int64_t M;
    int K;
    const uint32_t* W_packed;
    const float* alpha;
    int N;
    uint16_t* Y;
    int32_t* acc_out;
    int32_t* dev_status;
    bool interleaved = false;  // codes one per byte in the 32-row interleaved layout
    // launched right after the activation kernel of the fused forward: the
    // weights (not produced by that kernel) may be read before the dependency wait
    bool pdl = false;
};

// K2: tcgen05 tensor-core GEMM, both operands in shared memory, any M.
hbl_status launch_gemm_tc(const GemmArgs& a, cudaStream_t stream, int num_sms);
// K2b: tcgen05 tensor-core GEMM with the activations in TMEM, any M.  For
// M <= 256 it splits K over CTAs and needs gemm_ts_workspace() bytes of ws.
int gemm_ts_ksplit(int64_t M, int K, int N);
size_t gemm_ts_workspace(int64_t M, int K, int N);
hbl_status launch_gemm_ts(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                          int num_sms);
// Sum int32 split-K partials [ksplit][M][N], subtract rowsum, dequantise to bf16.
hbl_status launch_splitk_epilogue(const int32_t* part, int ksplit, int64_t M, int N,
                                  const int32_t* rowsum, const float* scales, const float* alpha,
                                  uint16_t* Y, int32_t* acc_out, cudaStream_t stream);

// K3: CUDA-core split-K GEMV for small M (M <= gemv_max_m()).
// TMA-fed tcgen05 GEMM for large batches: codes one byte each, row-major;
// the packed weights are expanded to signed bytes in workspace (N*K bytes).
size_t gemm_tma_workspace(int K, int N);
hbl_status launch_gemm_tma(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                           int num_sms);
// The two halves of launch_gemm_tma: packed 2-bit weights -> signed bytes
// [N x K], and the GEMM on already expanded weights (a.W_packed unused).
hbl_status launch_expand_ternary(const uint32_t* W_packed, int N, int K, int8_t* W_s8,
                                 cudaStream_t stream, int num_sms);
hbl_status launch_gemm_tma_s8w(const GemmArgs& a, const int8_t* W_s8, cudaStream_t stream,
                               int num_sms);
// K10: the large-batch GEMM on pairs of SMs (tcgen05 cta_group::2, a
// 256-token x 256-weight-row tile per cluster of two CTAs, both operands
// TMA-fed; same expanded weights and workspace as K2c).  Supported when K is a
// multiple of 128 and the device can hold a pair of its CTAs.
bool gemm_pair_supported(int K);
// Whether M x N fills the device in no more waves of paired tiles (256 x 256
// per pair) than of one-SM tiles (128 x 256 per SM of `num_sms`).
bool gemm_pair_preferred(int64_t M, int N, int num_sms);
hbl_status launch_gemm_pair(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                            int num_sms);
hbl_status launch_gemm_pair_s8w(const GemmArgs& a, const int8_t* W_s8, cudaStream_t stream);

// Row GEMV (one weight row per warp over the whole K, epilogue fused, no
// workspace) for M <= gemv_rows_max_m(K) tokens and 2048 <= K <= 32768.
// pdl_after_producer: launched as a programmatic dependent of the kernel that
// wrote the codes; the weights are then loaded before the dependency wait.
bool gemv_rows_supported(int K);
int gemv_rows_max_m(int K);
hbl_status launch_gemv_rows(const GemmArgs& a, bool pdl_after_producer, cudaStream_t stream);

int gemv_max_m();
size_t gemv_workspace(int64_t M, int K, int N, int num_sms);
hbl_status launch_gemv(const GemmArgs& a, void* ws, size_t ws_bytes, cudaStream_t stream,
                       int num_sms);

// K7: tensor-core GEMM for decode batches (1..decode_mma_max_m() tokens): the
// weights as the MMA's A operand in TMEM (128 weight rows per CTA), the
// tokens as B (TMA from one-byte row-major codes), K split over a thread-block
// cluster and reduced through distributed shared memory.  Codes one byte per
// code (a.act_bits 8), row-major; launched as a programmatic dependent (the
// weight rows stream into shared memory before the dependency wait).  No
// workspace.  decode_mma_supported: the shape has a plan that fits.
int decode_mma_max_m();
bool decode_mma_supported(int64_t M, int K, int N, int num_sms);
hbl_status launch_decode_mma(const GemmArgs& a, cudaStream_t stream, int num_sms);

// K8: tensor-core GEMM for large batches on the packed weights: weights widened
// in registers into TMEM as the MMA's A operand (128 rows per tile), codes one
// byte each (a.act_bits 8, row-major) as B by TMA (256 tokens per tile).  No
// workspace.  K a multiple of 256.
hbl_status launch_gemm_wt(const GemmArgs& a, cudaStream_t stream, int num_sms);

// Fixed scratch of the allocation-free GEMV entry point (file-scope device array).
size_t gemv_noalloc_scratch_bytes();
void* gemv_noalloc_scratch(int dev);

}  // namespace hbl
