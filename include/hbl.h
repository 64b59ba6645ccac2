/*
 * hbl.h -- C ABI of the B200 (sm_100a) H-BitLinear library (libhbl.so).
 *
 * H-BitLinear is the linear layer of BitNet v2 that replaces the attention
 * output projection (Wo) and the FFN down projection (W_down).  Per token row
 * x it computes
 *
 *     y = (alpha * s_x) * ( Quant_act( H_K/sqrt(K) . RMSNorm(x) ) . W_t^T )
 *
 * Sources: the BitNet v2 write-up on 0755model.com, sections
 * "BitNet v2：原生4位激活" (RMS normalisation, no bias; H-BitLinear at Wo and
 * W_down) and "H-BitLinear" (per-tensor absmean ternary weights; online
 * Hadamard transform before activation quantisation, computed with the fast
 * Hadamard transform in O(n log n); INT8 / INT4 activation quantisers; the
 * layer's overall expression LN -> Hadamard -> quantise -> matmul); the
 * shengxinai.com explainer, section 2.2 (4-bit activations take 16 values);
 * the "[论文品鉴] 1-bit LLM" post, section "掩码存储" (ternary weights packed
 * several to an integer).  The pages show their formulas as images only; the
 * formulas used are written out at each call below.
 *
 * Conventions for every call:
 *   - Pointers are device pointers owned by the caller, unless a call says
 *     "host".  The library allocates no memory; scratch space comes from the
 *     caller's workspace `ws` of at least hbl_workspace_size() bytes.
 *   - Every device pointer must be 16-byte aligned (HBL_ERR_ALIGNMENT).
 *   - bf16 tensors are passed as uint16_t bit patterns.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls are
 *     asynchronous: HBL_OK means the arguments were valid and the kernels were
 *     launched.  Errors are returned before any launch; nothing is written then.
 *   - `dev_status` (nullable) is a device int32 the kernels set to a non-zero
 *     hbl_status if a bounded device-side wait gives up (HBL_ERR_TIMEOUT); the
 *     caller reads it after synchronising.  Kernels never trap.
 *   - Shapes: K is a power of two with 16 <= K <= 32768 (the fast transform
 *     needs a power of two); M >= 0 (M == 0 launches nothing); N >= 16 and
 *     N % 16 == 0.  Violations return HBL_ERR_SHAPE.
 *   - act_bits is 4 or 8.  Codes layout: act_bits 8 -> int8 [M x K] row-major;
 *     act_bits 4 -> two's-complement nibbles [M x K/2], element 2j in the low
 *     nibble of byte j.
 *   - Packed ternary weights: uint32 [N x K/16] row-major; word (n, k/16) holds
 *     16 weights; local weight j = k % 16 sits at bits [8*(j%4) + 2*(j/4), +2)
 *     as the code t + 1 (0 -> -1, 1 -> 0, 2 -> +1; 3 is never written).
 *   - Only sm_100 devices are supported (HBL_ERR_UNSUPPORTED_ARCH otherwise).
 *   - Non-finite inputs give unspecified (but memory-safe) results.
 */
#ifndef HBL_H
#define HBL_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__) || defined(__clang__)
#define HBL_API __attribute__((visibility("default")))
#else
#define HBL_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    HBL_OK = 0,
    HBL_ERR_INVALID_ARG = 1,      /* null pointer, bad act_bits, negative/non-finite eps, bad op */
    HBL_ERR_SHAPE = 2,            /* K not a power of two in [16, 32768], N % 16, M < 0 */
    HBL_ERR_ALIGNMENT = 3,        /* a pointer is not 16-byte aligned */
    HBL_ERR_UNSUPPORTED_ARCH = 4, /* current device is not sm_100 */
    HBL_ERR_WORKSPACE = 5,        /* ws is NULL or smaller than hbl_workspace_size() */
    HBL_ERR_CUDA = 6,             /* a CUDA runtime call failed (launch, copy, query) */
    HBL_ERR_TIMEOUT = 7           /* a bounded device-side wait gave up (dev_status only) */
} hbl_status;

/* Static string for a status code ("unknown status" for other values). */
HBL_API const char* hbl_status_string(int status);

/* Library ABI version (major * 10000 + minor * 100 + patch). */
HBL_API int hbl_version(void);

/* Ternary-GEMM back ends, chosen per call through the *_path variants below
 * (a test and tuning aid; the library keeps no process-wide choice):
 *   HBL_PATH_AUTO (0) = what hbl_ternary_gemm / hbl_hbitlinear_forward do: the
 *       one-kernel decode forward where it applies; CUDA-core GEMV for M <= 8
 *       tokens (one weight row per warp for K >= 2048, split-K below); the
 *       tcgen05 kernel with activations in tensor memory (split over K for
 *       M <= 256) up to 256 tokens; above that the TMA-fed tcgen05 kernel when
 *       the codes are one byte each (the packed weights are widened to
 *       signed bytes in workspace first: by hbl_hbitlinear_forward's quantiser
 *       beside its token rows where the batch is large enough to carry it,
 *       else by a separate kernel),
 *   HBL_PATH_TC_SS (1)  = tcgen05 with both operands staged in shared memory by threads,
 *   HBL_PATH_GEMV (2)   = always the GEMV path (large M runs in chunks of 8 tokens),
 *   HBL_PATH_TC_TS (3)  = always the tcgen05 kernel with activations in tensor memory,
 *   HBL_PATH_TC_TMA (4) = the TMA-fed tcgen05 kernel whenever the codes are one
 *       byte each and K >= 128 (else as 3),
 *   HBL_PATH_TC_DECODE (5) = the decode-batch tcgen05 kernel (weights as the
 *       MMA's A operand in tensor memory, tokens as B, K split over a cluster
 *       of CTAs and reduced in distributed shared memory) whenever the codes
 *       are one byte each, M <= 128 and K >= 512 (else as 3),
 *   HBL_PATH_TC_PACKED (6) = the large-batch tcgen05 kernel on the packed
 *       weights (widened in registers into tensor memory as the MMA's A
 *       operand, codes as B by TMA; no expanded copy) whenever the codes are
 *       one byte each and K >= 256 (else as 3),
 *   HBL_PATH_TC_PAIR (7) = the TMA-fed large-batch kernel on pairs of SMs
 *       (tcgen05.mma.cta_group::2: a 256-token x 256-weight-row tile per
 *       cluster of two CTAs, each holding half of each operand) whenever the
 *       codes are one byte each and K >= 128 (else as 3; as 4 on a device
 *       that cannot hold a pair of its CTAs).
 * Every path computes the same values.  No counterpart on the BitNet v2 pages. */
enum {
    HBL_PATH_AUTO = 0,
    HBL_PATH_TC_SS = 1,
    HBL_PATH_GEMV = 2,
    HBL_PATH_TC_TS = 3,
    HBL_PATH_TC_TMA = 4,
    HBL_PATH_TC_DECODE = 5,
    HBL_PATH_TC_PACKED = 6,
    HBL_PATH_TC_PAIR = 7
};

/* act_bits also accepts these two values: the same INT4 / INT8 codes stored
 * one byte per code (two's complement) in a 32-row interleaved layout.  Rows
 * are padded to a multiple of 32 (the buffer holds ceil(M/32)*32*K bytes; the
 * padding rows are neither written nor used), and the 16-code chunk c of row m
 * starts at byte (((m / 32) * (K / 16) + c) * 32 + m % 32) * 16.  A warp that
 * owns 32 consecutive rows reads each chunk as 512 contiguous bytes; the
 * tensor-core GEMM takes this layout without widening, and
 * hbl_hbitlinear_forward uses it internally.  hbl_ternary_gemm always runs its
 * tcgen05 kernel with activations in tensor memory for these layouts, whatever
 * path is asked for. */
enum { HBL_ACT_INT4_I32 = 0x104, HBL_ACT_INT8_I32 = 0x108 };

/* act_bits may also be HBL_ACT_INT4_BYTES: INT4 codes stored one byte each
 * (two's complement), row-major [M x K], like the INT8 layout.  The TMA-fed
 * tensor-core GEMM (large batches) reads one-byte codes; hbl_hbitlinear_forward
 * uses this layout internally for INT4 batches above 256 tokens. */
enum { HBL_ACT_INT4_BYTES = 0x204 };

/* Operation identifiers for hbl_workspace_size(). */
enum {
    HBL_OP_PACK_TERNARY = 0,
    HBL_OP_TERNARY_GEMM = 1,
    HBL_OP_HBITLINEAR_FORWARD = 2,
    HBL_OP_HBITLINEAR_FORWARD_HOSTIO = 3
};

/* Bytes of device workspace that `op` needs for the given shape (0 is a valid
 * answer).  Unused shape arguments may be 0.  Writes *bytes; HBL_ERR_SHAPE or
 * HBL_ERR_INVALID_ARG on bad input. */
HBL_API hbl_status hbl_workspace_size(int op, int M, int K, int N, int act_bits, size_t* bytes);

/* hbl_workspace_size for the calls' *_path variants: the bytes `op` needs when
 * run on back end `path` (HBL_PATH_*; HBL_ERR_INVALID_ARG for other values). */
HBL_API hbl_status hbl_workspace_size_path(int op, int M, int K, int N, int act_bits, int path,
                                           size_t* bytes);

/* Ternary weight quantisation and packing (offline, once per weight).
 * Formula (per-tensor absmean; the page's formula is an image):
 *   alpha = S / (float)(N*K),  S = fp32 left-complete pairwise tree sum of |W|
 *           over the row-major flat index (row sums, then a tree over rows);
 *   t     = clip(round_half_even(W / (alpha + eps)), -1, 1)   (IEEE division);
 * W:        fp32 [N x K] row-major, device.
 * W_packed: uint32 [N x K/16] out, layout above.   alpha: device float, out.
 * ws:       >= hbl_workspace_size(HBL_OP_PACK_TERNARY, 0, K, N, 0) bytes.
 * K follows the layer's rule (a power of two in [16, 32768]); N >= 1. */
HBL_API hbl_status hbl_pack_ternary(const float* W, int N, int K, float eps, uint32_t* W_packed,
                            float* alpha, void* ws, size_t ws_bytes, void* stream);

/* RMSNorm followed by the normalised online Hadamard transform, fp32 out:
 *   r = 1 / sqrt(tree_sum(x*x) * (1/K) + norm_eps),   u = (x * r) * gain
 *   (every square x*x rounded to fp32, then summed by the perfect pairwise
 *   tree over index order)
 *   V = (u . H_K) * c_K,   c_K = fp32(1/sqrt(K)),
 * H_K the Sylvester Hadamard matrix in natural order, evaluated as butterfly
 * stages h = 1, 2, ..., K/2 in that order, (a, b) -> (a + b, a - b).
 * X: bf16 [M x K]; gain: fp32 [K] or NULL (all ones); V: fp32 [M x K] out.
 * This exposes the first two steps of the layer on their own. */
HBL_API hbl_status hbl_norm_fwht(const uint16_t* X, const float* gain, int M, int K, float norm_eps,
                         float* V, int32_t* dev_status, void* stream);

/* Fused RMSNorm + online Hadamard transform + per-token activation quantisation
 * (one kernel; V above is never written to memory).
 *   act_bits 8 (absmax):  gamma = max|v|;  q = clip(rhe(v * (127/(gamma+eps))), -128, 127);
 *                         scale = gamma / 127
 *   act_bits 4 (absmean): beta = tree_sum(|v|) * (1/K);
 *                         q = clip(rhe(v * (sqrt7/(beta+eps))), -8, 7);  scale = beta / sqrt7
 * rhe = round half to even; 127/(gamma+eps) and sqrt7/(beta+eps) are one IEEE
 * division per row; sqrt7 = fp32(sqrt(7)).
 * codes: out, layout above.  scales: fp32 [M] out.  rowsum: int32 [M] out = sum
 * of the row's codes, or NULL. */
HBL_API hbl_status hbl_norm_fwht_quant(const uint16_t* X, const float* gain, int M, int K,
                               float norm_eps, float quant_eps, int act_bits, void* codes,
                               float* scales, int32_t* rowsum, int32_t* dev_status,
                               void* stream);

/* Ternary x integer matmul with int32 accumulation and bf16 dequantisation:
 *   acc[m][n] = sum_k q[m][k] * t[n][k]            (exact)
 *   Y[m][n]   = bf16_rne( (float)acc * (alpha * scales[m]) )
 * codes/scales/rowsum as written by hbl_norm_fwht_quant (rowsum is REQUIRED:
 * the kernels multiply by the stored code t+1 and subtract rowsum[m]).
 * W_packed/alpha as written by hbl_pack_ternary.  Y: bf16 [M x N] out.
 * acc_out: int32 [M x N] out, or NULL (debug/parity aid).
 * ws: >= hbl_workspace_size(HBL_OP_TERNARY_GEMM, M, K, N, act_bits) bytes
 * (may be NULL when that size is 0). */
HBL_API hbl_status hbl_ternary_gemm(const void* codes, const float* scales, const int32_t* rowsum,
                            int act_bits, int M, int K, const uint32_t* W_packed,
                            const float* alpha, int N, uint16_t* Y, int32_t* acc_out,
                            void* ws, size_t ws_bytes, int32_t* dev_status, void* stream);

/* hbl_ternary_gemm on the back end `path` (HBL_PATH_*; HBL_PATH_AUTO is
 * hbl_ternary_gemm itself).  Same results on every path; ws sized by
 * hbl_workspace_size_path(HBL_OP_TERNARY_GEMM, ..., path, ...). */
HBL_API hbl_status hbl_ternary_gemm_path(const void* codes, const float* scales,
                                         const int32_t* rowsum, int act_bits, int M, int K,
                                         const uint32_t* W_packed, const float* alpha, int N,
                                         uint16_t* Y, int32_t* acc_out, void* ws, size_t ws_bytes,
                                         int32_t* dev_status, int path, void* stream);

/* The whole layer: hbl_norm_fwht_quant into workspace, then hbl_ternary_gemm.
 * Decode batches (M <= 16384 / K tokens at K = 4096 / 8192 / 16384, while the
 * packed weight rows of one SM's share fit its shared memory, GEMM path 0) run
 * both steps in one kernel instead: every CTA quantises the M rows itself
 * while its weight rows stream in; up to 8 tokens at K = 16384 run
 * hbl_norm_fwht_quant followed by that kernel's GEMV half, whose weight rows
 * stream into shared memory during the quantiser.  The results are the same
 * values on every path.
 * X: bf16 [M x K]; Y: bf16 [M x N] out; other arguments as above.
 * ws: >= hbl_workspace_size(HBL_OP_HBITLINEAR_FORWARD, M, K, N, act_bits). */
HBL_API hbl_status hbl_hbitlinear_forward(const uint16_t* X, const float* gain, int M, int K, int N,
                                  const uint32_t* W_packed, const float* alpha, int act_bits,
                                  float norm_eps, float quant_eps, uint16_t* Y, void* ws,
                                  size_t ws_bytes, int32_t* dev_status, void* stream);

/* hbl_hbitlinear_forward with the GEMM on back end `path` (HBL_PATH_*); any
 * path other than HBL_PATH_AUTO runs the two-kernel forward (quantiser, then
 * that GEMM).  ws sized by hbl_workspace_size_path(HBL_OP_HBITLINEAR_FORWARD,
 * ..., path, ...). */
HBL_API hbl_status hbl_hbitlinear_forward_path(const uint16_t* X, const float* gain, int M, int K,
                                               int N, const uint32_t* W_packed,
                                               const float* alpha, int act_bits, float norm_eps,
                                               float quant_eps, uint16_t* Y, void* ws,
                                               size_t ws_bytes, int32_t* dev_status, int path,
                                               void* stream);

/* The whole layer with HOST activations in and HOST outputs out: copies X_host
 * to the device, runs hbl_hbitlinear_forward, copies Y back to Y_host
 * (asynchronous; pinned host memory makes the copies asynchronous).  Ordered
 * as if everything ran on `stream`: it starts after the work already queued on
 * `stream`, and work queued on `stream` afterwards starts after Y_host is
 * written.  Batches above 513 tokens run in up to 8 row chunks whose input
 * copies, layer and output copies overlap; for that the library keeps two
 * copy streams and a few events per device, created on the first such call
 * and kept until exit (they are not memory).  Concurrent calls of this
 * function on one device are serialised while they enqueue.
 * X_host: bf16 [M x K] host; Y_host: bf16 [M x N] host, out.
 * ws: >= hbl_workspace_size(HBL_OP_HBITLINEAR_FORWARD_HOSTIO, M, K, N, act_bits)
 * bytes of device memory (it holds the device copies of X and Y as well). */
HBL_API hbl_status hbl_hbitlinear_forward_hostio(const uint16_t* X_host, const float* gain, int M,
                                         int K, int N, const uint32_t* W_packed,
                                         const float* alpha, int act_bits, float norm_eps,
                                         float quant_eps, uint16_t* Y_host, void* ws,
                                         size_t ws_bytes, int32_t* dev_status, void* stream);

/* ---------------------------------------------------------------- variants
 * BitNet v2 uses H-BitLinear only at Wo and W_down; its other linear layers are
 * the plain BitLinear: the same normalise -> quantise -> ternary matmul without
 * the Hadamard transform (write-up on 0755model.com, section "BitNet v2：原生4位
 * 激活": all linears except the embeddings are fine-tuned to 4-bit activations).
 * The layer expression there writes the normalisation as LN and glosses it as
 * layer normalisation, while the architecture uses RMS normalisation; both are
 * offered.  Flags (bitwise or):
 *   HBL_NORM_LAYERNORM:   LayerNorm without bias instead of RMSNorm:
 *       mu = tree_sum(x) * (1/K);  d = x - mu;
 *       r = 1 / sqrt(tree_sum(d*d) * (1/K) + norm_eps);  u = (d * r) * gain
 *       (tree sums as for RMSNorm; every square d*d is rounded to fp32
 *        before the tree adds it).
 *   HBL_NORM_NO_HADAMARD: no transform: the codes quantise u itself.
 * flags = 0 is exactly the H-BitLinear path of the calls above.  Other bits
 * return HBL_ERR_INVALID_ARG.  Shapes and layouts as above (K a power of two). */
enum { HBL_NORM_LAYERNORM = 1, HBL_NORM_NO_HADAMARD = 2 };

/* hbl_norm_fwht with variant flags: V = T(N(x)) fp32 [M x K]. */
HBL_API hbl_status hbl_norm_transform(const uint16_t* X, const float* gain, int M, int K,
                                      float norm_eps, unsigned flags, float* V,
                                      int32_t* dev_status, void* stream);

/* hbl_norm_fwht_quant with variant flags (act_bits 4, 8, or the interleaved
 * HBL_ACT_INT*_I32 layouts). */
HBL_API hbl_status hbl_norm_quant(const uint16_t* X, const float* gain, int M, int K,
                                  float norm_eps, float quant_eps, int act_bits, unsigned flags,
                                  void* codes, float* scales, int32_t* rowsum,
                                  int32_t* dev_status, void* stream);

/* The whole BitLinear / H-BitLinear layer with variant flags; workspace as for
 * HBL_OP_HBITLINEAR_FORWARD. */
HBL_API hbl_status hbl_bitlinear_forward(const uint16_t* X, const float* gain, int M, int K,
                                         int N, const uint32_t* W_packed, const float* alpha,
                                         int act_bits, unsigned flags, float norm_eps,
                                         float quant_eps, uint16_t* Y, void* ws, size_t ws_bytes,
                                         int32_t* dev_status, void* stream);

/* Offline weight rotation (BitNet v2 write-up, table 5: the Hadamard rotation
 * applied to weights and activations; the QuaRot baseline there uses a
 * randomised Hadamard transform H . diag(s)):
 *   W_rot[n] = ((W[n] * s) . H_K) * c_K      for every row n,
 * with the butterfly order and c_K of hbl_norm_fwht.  Then
 * (x D H c_K) . (w D H c_K) = x . w for D = diag(s), so rotated weights pair with
 * activations normalised with gain' = gain * s (hbl_norm_* with that gain: the
 * product with +-1 is exact) and transformed as usual.  Ternarise W_rot with
 * hbl_pack_ternary.
 * W: fp32 [N x K] device; signs: fp32 [K] of +-1 or NULL (all ones; the plain
 * transform); W_rot: fp32 [N x K] out, may be W itself (in place).
 * K: power of two in [16, 32768]; N >= 0. */
HBL_API hbl_status hbl_rotate_weights(const float* W, const float* signs, int N, int K,
                                      float* W_rot, int32_t* dev_status, void* stream);

/* Per-head absmax quantiser of Q, K, V states after RoPE, to unsigned integers
 * (BitNet v2 write-up, section "实验结果", tables 2 and 3: QKV heads quantised
 * with absmax directly to unsigned integers, no calibration; 3-bit KV cache).
 * One row = one head of one token, D values:
 *   Qp = 2^(bits-1) - 1;  gamma = max|x|;  inv = Qp / (gamma + eps)  (one division)
 *   q = clip(rhe(x * inv), -Qp-1, Qp);  u = q + 2^(bits-1);  scales[row] = gamma / Qp
 * (the INT8 activation quantiser taken to `bits` bits and offset into the
 * unsigned range; dequantise as (u - 2^(bits-1)) * scale).
 * X: bf16 [rows x D] (e.g. [tokens x heads x D]); bits in {2, 3, 4, 8};
 * D in {32, 64, 128, 256}; eps >= 0 finite.
 * codes: [rows x D*bits/8] bytes out: each group of 32 consecutive codes of a
 * row is 4*bits bytes, code j of the group at bits [bits*j, bits*j + bits) of
 * the group read as a little-endian integer.  scales: fp32 [rows] out. */
HBL_API hbl_status hbl_kv_quant(const uint16_t* X, int64_t rows, int D, int bits, float eps,
                                uint8_t* codes, float* scales, int32_t* dev_status, void* stream);

/* --------------------------------------------------- expanded-weight GEMM
 * For large token batches the tensor-core GEMM reads the ternary weights as
 * one signed byte each (tcgen05 has no integer MMA narrower than 8 bits);
 * hbl_ternary_gemm and hbl_hbitlinear_forward expand the packed weights into
 * workspace on every call (the forward inside its quantiser kernel where the
 * token rows carry it).  A caller that keeps the expanded copy (N*K bytes,
 * 4x the packed size) can skip that step with these two calls.  No
 * counterpart on the BitNet v2 pages: a deployment aid.
 *
 * hbl_expand_ternary: W_s8[n][k] = t[n][k] in {-1, 0, +1} (int8, row-major
 * [N x K]) from W_packed (layout above).  K as for the layer; N >= 0. */
HBL_API hbl_status hbl_expand_ternary(const uint32_t* W_packed, int N, int K, int8_t* W_s8,
                                      int32_t* dev_status, void* stream);

/* The TMA-fed tensor-core GEMM on expanded weights (the paired-SM kernel, or
 * the one-SM kernel where that fills the device in fewer waves of tiles):
 *   Y[m][n] = bf16_rne((float)(sum_k q[m][k] * W_s8[n][k]) * (alpha * scales[m]))
 * codes: one byte per code, row-major [M x K]: act_bits 8 (INT8) or
 * HBL_ACT_INT4_BYTES.  K >= 128 (a power of two as above).  acc_out: int32
 * [M x N] or NULL.  No workspace; no rowsum needed (the weights are signed). */
HBL_API hbl_status hbl_ternary_gemm_s8w(const void* codes, const float* scales, int act_bits,
                                        int M, int K, const int8_t* W_s8, const float* alpha,
                                        int N, uint16_t* Y, int32_t* acc_out,
                                        int32_t* dev_status, void* stream);

/* Self-test of the failure path (no counterpart on the pages).  Every
 * pipelined kernel here waits on mbarriers with a bound on global time and, if
 * the bound runs out, records HBL_ERR_TIMEOUT in dev_status and returns
 * instead of hanging.  This launches one probe kernel running the same bounded
 * wait on a barrier that receives its arrival first (arrive != 0: dev_status
 * stays 0) or never (arrive == 0: after timeout_us microseconds dev_status
 * becomes HBL_ERR_TIMEOUT).  dev_status: device int32 (required); timeout_us
 * in [1, 1000000]. */
HBL_API hbl_status hbl_selftest_bounded_wait(int arrive, int timeout_us, int32_t* dev_status,
                                             void* stream);

/* Dense INT8 tensor-core rate probe (no counterpart on the pages; it measures
 * the denominator of the ternary GEMM's roofline on the GPU at hand).  Launches
 * `ctas` CTAs (at most one per SM); each zeroes a 128 x 128-byte and a
 * 256 x 128-byte operand tile in its shared memory and one thread issues
 * `mmas_per_cta` back-to-back tcgen05.mma.cta_group::1.kind::i8 instructions of
 * shape M = 128, N = 256, K = 32 (2 * 128 * 256 * 32 integer operations each)
 * into one TMEM accumulator, then waits (bounded) for them.  No global memory
 * is touched except dev_status.  Time the launch with events on `stream`: the
 * rate is ctas * mmas_per_cta * 2097152 operations over that time.
 * ctas in [1, 4096]; mmas_per_cta in [1, 2^22]; dev_status: device int32
 * (required; HBL_ERR_TIMEOUT if the MMAs did not finish within 2 s). */
HBL_API hbl_status hbl_probe_tc_int8(int ctas, int mmas_per_cta, int32_t* dev_status,
                                     void* stream);

/* Allocation-free ternary GEMV (no counterpart on the BitNet v2 pages; it is a
 * deployment aid).  Same arguments, layouts and results as hbl_ternary_gemm
 * run on its CUDA-core split-K path, but without a workspace argument: the
 * split-K partial sums live in one fixed 2 MiB array that the library reserves
 * on every GPU that loads it, until the process exits.
 * For callers that cannot supply scratch memory or let a library allocate:
 * e.g. an engine's custom-op hook that is handed only inputs and outputs, or a
 * token-by-token decode loop that must not block on the allocator, trigger an
 * implicit device synchronisation, or risk an out-of-memory failure mid-step.
 * This call never allocates device or host memory.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture.
 *   - All calls on a device share the array and leave their partial sums in
 *     it; nothing in it needs to start at zero (every partial read is written
 *     first by the same call).  Calls that overlap on the GPU (two streams or
 *     two host threads at once) race on the array: serialise them.
 *   - Shapes whose partials exceed the array (ksplit * min(M, 8) * N * 4 bytes,
 *     ksplit chosen as for hbl_ternary_gemm) return HBL_ERR_WORKSPACE before
 *     any launch; e.g. N = 4096 with K = 16384 needs 1 MiB at M >= 8.
 *   - M > 8 runs in consecutive 8-token chunks on `stream`. */
HBL_API hbl_status hbl_ternary_gemv_noalloc(const void* codes, const float* scales,
                                            const int32_t* rowsum, int act_bits, int M, int K,
                                            const uint32_t* W_packed, const float* alpha, int N,
                                            uint16_t* Y, int32_t* acc_out, int32_t* dev_status,
                                            void* stream);

#ifdef __cplusplus
}
#endif

#endif /* HBL_H */
