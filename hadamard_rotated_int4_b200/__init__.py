"""Python binding of libhbl.so, the sm_100a H-BitLinear library (BitNet v2).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  torch supplies device memory and the current CUDA stream.  There is
no CPU fallback: calls raise if the library is not built or the device is not
an sm_100 GPU.

Names follow include/hbl.h:
  pack_ternary(W)                         -> (W_packed int32 view [N, K/16], alpha [1])
  norm_fwht(X)                            -> V fp32 [M, K]
  norm_fwht_quant(X, act_bits)            -> (codes uint8, scales fp32 [M], rowsum int32 [M])
  ternary_gemm(codes, scales, rowsum, act_bits, K, W_packed, alpha)  -> Y bf16 [M, N] (, acc)
  hbitlinear_forward(X, W_packed, alpha, act_bits)                   -> Y bf16 [M, N]
  hbitlinear_forward_hostio(X_host, W_packed, alpha, act_bits, Y_host, ws)
  ternary_gemv_noalloc(codes, scales, rowsum, act_bits, K, W_packed, alpha)  -> Y (, acc)
  norm_transform(X, flags)                -> V fp32 [M, K]       (variants: NORM_* flags)
  norm_quant(X, act_bits, flags)          -> (codes, scales, rowsum)
  bitlinear_forward(X, W_packed, alpha, act_bits, flags)            -> Y bf16 [M, N]
  rotate_weights(W, signs)                -> W_rot fp32 [N, K]
  kv_quant(X, bits)                       -> (codes uint8 [rows, D*bits/8], scales fp32 [rows])
"""
import ctypes
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libhbl.so")

HBL_OK = 0
STATUS_NAMES = {0: "HBL_OK", 1: "HBL_ERR_INVALID_ARG", 2: "HBL_ERR_SHAPE", 3: "HBL_ERR_ALIGNMENT",
                4: "HBL_ERR_UNSUPPORTED_ARCH", 5: "HBL_ERR_WORKSPACE", 6: "HBL_ERR_CUDA",
                7: "HBL_ERR_TIMEOUT"}
OP_PACK_TERNARY, OP_TERNARY_GEMM, OP_HBITLINEAR_FORWARD, OP_HBITLINEAR_FORWARD_HOSTIO = 0, 1, 2, 3
ACT_INT4_I32, ACT_INT8_I32 = 0x104, 0x108  # one byte per code, 32-row interleaved layout
ACT_INT4_BYTES = 0x204                      # INT4 codes one byte each, row-major
NORM_LAYERNORM, NORM_NO_HADAMARD = 1, 2     # variant flags of norm_transform / norm_quant / bitlinear_forward
PATH_AUTO, PATH_TC_SS, PATH_GEMV, PATH_TC_TS, PATH_TC_TMA, PATH_TC_DECODE = 0, 1, 2, 3, 4, 5
PATH_TC_PACKED, PATH_TC_PAIR = 6, 7
EXPORTS = ("hbl_status_string", "hbl_version", "hbl_workspace_size", "hbl_workspace_size_path",
           "hbl_pack_ternary", "hbl_norm_fwht", "hbl_norm_fwht_quant", "hbl_ternary_gemm",
           "hbl_ternary_gemm_path", "hbl_hbitlinear_forward", "hbl_hbitlinear_forward_path",
           "hbl_hbitlinear_forward_hostio",
           "hbl_ternary_gemv_noalloc", "hbl_norm_transform", "hbl_norm_quant",
           "hbl_bitlinear_forward", "hbl_rotate_weights", "hbl_kv_quant",
           "hbl_expand_ternary", "hbl_ternary_gemm_s8w", "hbl_selftest_bounded_wait",
           "hbl_probe_tc_int8")

_lib = None


class HblError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__("%s failed: %s (%s)" % (what, STATUS_NAMES.get(status, status),
                                                  lib().hbl_status_string(status).decode()))


def lib():
    """Load libhbl.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libhbl.so is not built (run __graft_entry__.build() or "
                               "python hadamard_rotated_int4_b200/build.py)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, F, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        L.hbl_status_string.restype = ctypes.c_char_p
        L.hbl_status_string.argtypes = [I]
        L.hbl_version.restype = I
        L.hbl_version.argtypes = []
        L.hbl_workspace_size.restype = I
        L.hbl_workspace_size.argtypes = [I, I, I, I, I, ctypes.POINTER(SZ)]
        L.hbl_workspace_size_path.restype = I
        L.hbl_workspace_size_path.argtypes = [I, I, I, I, I, I, ctypes.POINTER(SZ)]
        L.hbl_pack_ternary.restype = I
        L.hbl_pack_ternary.argtypes = [P, I, I, F, P, P, P, SZ, P]
        L.hbl_norm_fwht.restype = I
        L.hbl_norm_fwht.argtypes = [P, P, I, I, F, P, P, P]
        L.hbl_norm_fwht_quant.restype = I
        L.hbl_norm_fwht_quant.argtypes = [P, P, I, I, F, F, I, P, P, P, P, P]
        L.hbl_ternary_gemm.restype = I
        L.hbl_ternary_gemm.argtypes = [P, P, P, I, I, I, P, P, I, P, P, P, SZ, P, P]
        L.hbl_ternary_gemm_path.restype = I
        L.hbl_ternary_gemm_path.argtypes = [P, P, P, I, I, I, P, P, I, P, P, P, SZ, P, I, P]
        L.hbl_hbitlinear_forward.restype = I
        L.hbl_hbitlinear_forward.argtypes = [P, P, I, I, I, P, P, I, F, F, P, P, SZ, P, P]
        L.hbl_hbitlinear_forward_path.restype = I
        L.hbl_hbitlinear_forward_path.argtypes = [P, P, I, I, I, P, P, I, F, F, P, P, SZ, P, I, P]
        L.hbl_hbitlinear_forward_hostio.restype = I
        L.hbl_hbitlinear_forward_hostio.argtypes = [P, P, I, I, I, P, P, I, F, F, P, P, SZ, P, P]
        L.hbl_ternary_gemv_noalloc.restype = I
        L.hbl_ternary_gemv_noalloc.argtypes = [P, P, P, I, I, I, P, P, I, P, P, P, P]
        U, I64 = ctypes.c_uint, ctypes.c_int64
        L.hbl_norm_transform.restype = I
        L.hbl_norm_transform.argtypes = [P, P, I, I, F, U, P, P, P]
        L.hbl_norm_quant.restype = I
        L.hbl_norm_quant.argtypes = [P, P, I, I, F, F, I, U, P, P, P, P, P]
        L.hbl_bitlinear_forward.restype = I
        L.hbl_bitlinear_forward.argtypes = [P, P, I, I, I, P, P, I, U, F, F, P, P, SZ, P, P]
        L.hbl_rotate_weights.restype = I
        L.hbl_rotate_weights.argtypes = [P, P, I, I, P, P, P]
        L.hbl_kv_quant.restype = I
        L.hbl_kv_quant.argtypes = [P, I64, I, I, F, P, P, P, P]
        L.hbl_expand_ternary.restype = I
        L.hbl_expand_ternary.argtypes = [P, I, I, P, P, P]
        L.hbl_ternary_gemm_s8w.restype = I
        L.hbl_ternary_gemm_s8w.argtypes = [P, P, I, I, I, P, P, I, P, P, P, P]
        L.hbl_selftest_bounded_wait.restype = I
        L.hbl_selftest_bounded_wait.argtypes = [I, I, P, P]
        L.hbl_probe_tc_int8.restype = I
        L.hbl_probe_tc_int8.argtypes = [I, I, P, P]
        _lib = L
    return _lib


def _check(status, what):
    if status != HBL_OK:
        raise HblError(status, what)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream():
    import torch

    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _dev(t, dtype, name):
    import torch

    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError("%s must be a CUDA tensor" % name)
    if t.dtype != dtype:
        raise TypeError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    return t


def workspace_size(op, M, K, N, act_bits, path=PATH_AUTO):
    """Workspace bytes of `op` on GEMM back end `path` (PATH_*)."""
    out = ctypes.c_size_t(0)
    _check(lib().hbl_workspace_size_path(op, M, K, N, act_bits, int(path), ctypes.byref(out)),
           "workspace_size")
    return out.value


def _workspace(nbytes, device):
    import torch

    return torch.empty(max(int(nbytes), 16), dtype=torch.uint8, device=device)


def new_status(device):
    import torch

    return torch.zeros(4, dtype=torch.int32, device=device)


def pack_ternary(W, eps=1e-5, ws=None):
    import torch

    _dev(W, torch.float32, "W")
    N, K = W.shape
    packed = torch.empty((N, K // 16), dtype=torch.int32, device=W.device)
    alpha = torch.empty(4, dtype=torch.float32, device=W.device)
    need = workspace_size(OP_PACK_TERNARY, 0, K, N, 0)
    if ws is None:
        ws = _workspace(need, W.device)
    _check(lib().hbl_pack_ternary(_ptr(W), N, K, float(eps), _ptr(packed), _ptr(alpha), _ptr(ws),
                                  ws.numel(), _stream()), "hbl_pack_ternary")
    return packed, alpha[:1]


def norm_fwht(X, gain=None, norm_eps=1e-6, status=None):
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    V = torch.empty((M, K), dtype=torch.float32, device=X.device)
    _check(lib().hbl_norm_fwht(_ptr(X), _ptr(gain), M, K, float(norm_eps), _ptr(V), _ptr(status),
                               _stream()), "hbl_norm_fwht")
    return V


def codes_shape(M, K, act_bits):
    if act_bits in (ACT_INT4_I32, ACT_INT8_I32):
        return ((M + 31) // 32 * 32, K)
    return (M, K // 2 if act_bits == 4 else K)


def norm_fwht_quant(X, act_bits, gain=None, norm_eps=1e-6, quant_eps=1e-5, out=None,
                    status=None):
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    if out is None:
        codes = torch.empty(codes_shape(M, K, act_bits), dtype=torch.uint8, device=X.device)
        scales = torch.empty(max(M, 4), dtype=torch.float32, device=X.device)
        rowsum = torch.empty(max(M, 4), dtype=torch.int32, device=X.device)
    else:
        codes, scales, rowsum = out
    _check(lib().hbl_norm_fwht_quant(_ptr(X), _ptr(gain), M, K, float(norm_eps),
                                     float(quant_eps), int(act_bits), _ptr(codes), _ptr(scales),
                                     _ptr(rowsum), _ptr(status), _stream()),
           "hbl_norm_fwht_quant")
    return codes, scales[:M], rowsum[:M]


def ternary_gemm(codes, scales, rowsum, act_bits, K, W_packed, alpha, want_acc=False, ws=None,
                 out=None, status=None, path=PATH_AUTO):
    """hbl_ternary_gemm (hbl_ternary_gemm_path for a back end other than PATH_AUTO:
    PATH_TC_SS tensor cores with both operands staged by threads, PATH_GEMV
    CUDA-core GEMV, PATH_TC_TS tensor cores with activations in TMEM,
    PATH_TC_TMA TMA-fed tensor cores for one-byte codes, PATH_TC_DECODE the
    decode-batch tensor-core kernel for one-byte codes and M <= 128,
    PATH_TC_PACKED the large-batch tensor-core kernel on the packed weights,
    PATH_TC_PAIR the TMA-fed large-batch kernel on pairs of SMs)."""
    import torch

    M = scales.shape[0]  # the interleaved layouts pad the codes buffer to 32 rows
    N = W_packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16,
                                                device=codes.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=codes.device) if want_acc else None
    need = workspace_size(OP_TERNARY_GEMM, M, K, N, act_bits, path)
    if ws is None:
        ws = _workspace(need, codes.device)
    _check(lib().hbl_ternary_gemm_path(_ptr(codes), _ptr(scales), _ptr(rowsum), int(act_bits), M,
                                       K, _ptr(W_packed), _ptr(alpha), N, _ptr(Y), _ptr(acc),
                                       _ptr(ws), ws.numel(), _ptr(status), int(path), _stream()),
           "hbl_ternary_gemm")
    return (Y, acc) if want_acc else Y


def ternary_gemv_noalloc(codes, scales, rowsum, act_bits, K, W_packed, alpha, want_acc=False,
                         out=None, status=None):
    """hbl_ternary_gemv_noalloc: the split-K GEMV with the library's fixed scratch
    array (no workspace argument; the library allocates nothing)."""
    import torch

    M = scales.shape[0]
    N = W_packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16,
                                                device=codes.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=codes.device) if want_acc else None
    _check(lib().hbl_ternary_gemv_noalloc(_ptr(codes), _ptr(scales), _ptr(rowsum),
                                          int(act_bits), M, K, _ptr(W_packed), _ptr(alpha), N,
                                          _ptr(Y), _ptr(acc), _ptr(status), _stream()),
           "hbl_ternary_gemv_noalloc")
    return (Y, acc) if want_acc else Y


def hbitlinear_forward(X, W_packed, alpha, act_bits, gain=None, norm_eps=1e-6, quant_eps=1e-5,
                       ws=None, out=None, status=None, path=PATH_AUTO):
    """hbl_hbitlinear_forward (hbl_hbitlinear_forward_path for another GEMM back end)."""
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    N = W_packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(workspace_size(OP_HBITLINEAR_FORWARD, M, K, N, act_bits, path), X.device)
    _check(lib().hbl_hbitlinear_forward_path(_ptr(X), _ptr(gain), M, K, N, _ptr(W_packed),
                                             _ptr(alpha), int(act_bits), float(norm_eps),
                                             float(quant_eps), _ptr(Y), _ptr(ws), ws.numel(),
                                             _ptr(status), int(path), _stream()),
           "hbl_hbitlinear_forward")
    return Y


def hbitlinear_forward_hostio(X_host, W_packed, alpha, act_bits, Y_host, ws, gain=None,
                              norm_eps=1e-6, quant_eps=1e-5, status=None):
    """Host bf16 X in, host bf16 Y out (pinned memory makes the copies asynchronous)."""
    M, K = X_host.shape
    N = W_packed.shape[0]
    _check(lib().hbl_hbitlinear_forward_hostio(_ptr(X_host), _ptr(gain), M, K, N, _ptr(W_packed),
                                               _ptr(alpha), int(act_bits), float(norm_eps),
                                               float(quant_eps), _ptr(Y_host), _ptr(ws),
                                               ws.numel(), _ptr(status), _stream()),
           "hbl_hbitlinear_forward_hostio")
    return Y_host


# ------------------------------------------------------------------ variants

def norm_transform(X, flags=0, gain=None, norm_eps=1e-6, status=None):
    """hbl_norm_transform: V = T(N(X)) with NORM_LAYERNORM / NORM_NO_HADAMARD flags."""
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    V = torch.empty((M, K), dtype=torch.float32, device=X.device)
    _check(lib().hbl_norm_transform(_ptr(X), _ptr(gain), M, K, float(norm_eps), int(flags),
                                    _ptr(V), _ptr(status), _stream()), "hbl_norm_transform")
    return V


def norm_quant(X, act_bits, flags=0, gain=None, norm_eps=1e-6, quant_eps=1e-5, out=None,
               status=None):
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    if out is None:
        codes = torch.empty(codes_shape(M, K, act_bits), dtype=torch.uint8, device=X.device)
        scales = torch.empty(max(M, 4), dtype=torch.float32, device=X.device)
        rowsum = torch.empty(max(M, 4), dtype=torch.int32, device=X.device)
    else:
        codes, scales, rowsum = out
    _check(lib().hbl_norm_quant(_ptr(X), _ptr(gain), M, K, float(norm_eps), float(quant_eps),
                                int(act_bits), int(flags), _ptr(codes), _ptr(scales),
                                _ptr(rowsum), _ptr(status), _stream()), "hbl_norm_quant")
    return codes, scales[:M], rowsum[:M]


def bitlinear_forward(X, W_packed, alpha, act_bits, flags=0, gain=None, norm_eps=1e-6,
                      quant_eps=1e-5, ws=None, out=None, status=None):
    import torch

    _dev(X, torch.bfloat16, "X")
    M, K = X.shape
    N = W_packed.shape[0]
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16, device=X.device)
    if ws is None:
        ws = _workspace(workspace_size(OP_HBITLINEAR_FORWARD, M, K, N, act_bits), X.device)
    _check(lib().hbl_bitlinear_forward(_ptr(X), _ptr(gain), M, K, N, _ptr(W_packed),
                                       _ptr(alpha), int(act_bits), int(flags), float(norm_eps),
                                       float(quant_eps), _ptr(Y), _ptr(ws), ws.numel(),
                                       _ptr(status), _stream()), "hbl_bitlinear_forward")
    return Y


def rotate_weights(W, signs=None, out=None, status=None):
    """hbl_rotate_weights: W_rot = FWHT(W * signs) / sqrt(K) per row (out may be W)."""
    import torch

    _dev(W, torch.float32, "W")
    N, K = W.shape
    if signs is not None:
        _dev(signs, torch.float32, "signs")
    Wr = out if out is not None else torch.empty_like(W)
    _check(lib().hbl_rotate_weights(_ptr(W), _ptr(signs), N, K, _ptr(Wr), _ptr(status),
                                    _stream()), "hbl_rotate_weights")
    return Wr


def kv_code_bytes(D, bits):
    return D * bits // 8


def kv_quant(X, bits, eps=1e-5, out=None, status=None):
    """hbl_kv_quant over the last dimension (one head of one token per row)."""
    import torch

    _dev(X, torch.bfloat16, "X")
    D = X.shape[-1]
    rows = X.numel() // D if D else 0
    if out is None:
        codes = torch.empty((rows, kv_code_bytes(D, bits)), dtype=torch.uint8, device=X.device)
        scales = torch.empty(max(rows, 4), dtype=torch.float32, device=X.device)
    else:
        codes, scales = out
    _check(lib().hbl_kv_quant(_ptr(X), rows, D, int(bits), float(eps), _ptr(codes),
                              _ptr(scales), _ptr(status), _stream()), "hbl_kv_quant")
    return codes, scales[:rows]


# ------------------------------------------------------- expanded weights

def expand_ternary(W_packed, K, out=None, status=None):
    """hbl_expand_ternary: packed 2-bit weights -> int8 t in {-1, 0, 1} [N, K]."""
    import torch

    N = W_packed.shape[0]
    Ws = out if out is not None else torch.empty((N, K), dtype=torch.int8,
                                                 device=W_packed.device)
    _check(lib().hbl_expand_ternary(_ptr(W_packed), N, K, _ptr(Ws), _ptr(status), _stream()),
           "hbl_expand_ternary")
    return Ws


def ternary_gemm_s8w(codes, scales, act_bits, W_s8, alpha, want_acc=False, out=None,
                     status=None):
    """hbl_ternary_gemm_s8w: the TMA-fed tensor-core GEMM on expanded weights."""
    import torch

    M = scales.shape[0]
    N, K = W_s8.shape
    Y = out if out is not None else torch.empty((M, N), dtype=torch.bfloat16,
                                                device=codes.device)
    acc = torch.empty((M, N), dtype=torch.int32, device=codes.device) if want_acc else None
    _check(lib().hbl_ternary_gemm_s8w(_ptr(codes), _ptr(scales), int(act_bits), M, K, _ptr(W_s8),
                                      _ptr(alpha), N, _ptr(Y), _ptr(acc), _ptr(status),
                                      _stream()), "hbl_ternary_gemm_s8w")
    return (Y, acc) if want_acc else Y


def selftest_bounded_wait(arrive, timeout_us, status):
    """hbl_selftest_bounded_wait: the bounded-wait failure path on one probe kernel."""
    _check(lib().hbl_selftest_bounded_wait(int(bool(arrive)), int(timeout_us), _ptr(status),
                                           _stream()), "hbl_selftest_bounded_wait")


def probe_tc_int8(ctas, mmas_per_cta, status):
    """hbl_probe_tc_int8: back-to-back 128 x 256 x 32 kind::i8 MMAs from shared
    memory on `ctas` SMs (time it with events on the current stream)."""
    _check(lib().hbl_probe_tc_int8(int(ctas), int(mmas_per_cta), _ptr(status), _stream()),
           "hbl_probe_tc_int8")


OPS_PER_PROBE_MMA = 2 * 128 * 256 * 32


def measure_int8_tensor_peak(ctas, mmas_per_cta=1 << 15, reps=5):
    """Best-of-reps dense INT8 rate (TOPS) from the probe, with its launch timed
    by CUDA events on the current stream; returns (tops, status word)."""
    import torch

    status = new_status(torch.device("cuda", torch.cuda.current_device()))
    probe_tc_int8(ctas, 64, status)  # warm-up (shared-memory attribute, clocks)
    torch.cuda.synchronize()
    best = None
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        probe_tc_int8(ctas, mmas_per_cta, status)
        b.record()
        torch.cuda.synchronize()
        t = a.elapsed_time(b) * 1e-3
        best = t if best is None else min(best, t)
    tops = ctas * mmas_per_cta * OPS_PER_PROBE_MMA / best / 1e12
    return tops, int(status[0].item())
