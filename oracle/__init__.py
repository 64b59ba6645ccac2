"""CPU oracle for the H-BitLinear forward pass (BitNet v2).

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this package.  The product path (the
CUDA library and its Python binding) never imports, links or calls it, and it
shares no code with them.

Each function wraps the scalar C implementation in ``hbl_oracle.c`` (built with
``-ffp-contract=off``), whose header states the sources and the fixed fp32
evaluation order.  Inputs and outputs are numpy arrays; bf16 tensors travel as
their uint16 bit patterns.

Pins (what fixes each function other than itself; see tests/test_oracle_pins.py):
  sylvester          closed form (-1)^popcount(i&j); H H^T = n I; scipy.linalg.hadamard
  fwht_f32/_f64      dense product with scipy's Hadamard matrix (bit-exact on
                     integer inputs); involution; Parseval; delta / all-ones cases
  rmsnorm            constant-row closed form; torch.nn.functional.rms_norm in fp64;
                     a hand-derived row whose squares underflow (each square rounded
                     to binary32 before the tree: the plain reading of sum x^2)
  norm_fwht          within 1e-6 relative (fp32 vs fp64 composition of the pinned steps)
  quantize_rows      hand-made rows with exact .5 ties; absmax element -> +-127;
                     INT4 range [-8, 7] with -8 reachable; zero row; brute-force
                     per-element rounding against Python's round-half-even
  ternarize/pack     codes in {-1,0,1}; threshold form sign(W)[|W| > (alpha+eps)/2];
                     pack/unpack round trip; code 3 never written; W = I case
  ternary_gemm       integer brute force (numpy int64 matmul) on small shapes;
                     identity weights give acc = q; all-ones weights give acc = rowsum
  bf16 conversion    torch's float32 -> bfloat16 rounding
  outlier invariant  INT4 reconstruction error lower after the transform
  norm_transform     LayerNorm: balanced-row closed form, shift invariance on exact
                     integer rows, torch.nn.functional.layer_norm in fp64; the
                     (RMS, Hadamard) case equals norm_fwht's pins; no-Hadamard case:
                     torch rms_norm / layer_norm in fp64
  norm_quant         the quantiser pins above, applied to the pinned transforms;
                     codes vs a torch fp64 evaluation away from rounding ties
  rotate_weights     dense product with scipy's Hadamard matrix and the signs (fp64,
                     1e-6); (x D H)(w D H)^T = x w^T; involution with the signs
  kv_quant           brute force against Python's round-half-even per element;
                     exact ties; max element -> 2^b - 1 or 1; zero row; packing
                     against Python big-integer bit strings; round trip
No function is left with parity unpinned.
"""
import ctypes
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

from . import build as _build

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        I64 = ctypes.c_int64
        F = ctypes.c_float
        D = ctypes.c_double
        sig = {
            "oracle_tree_sum": (F, [P, I64]),
            "oracle_bf16_to_f32": (F, [ctypes.c_uint16]),
            "oracle_f32_to_bf16": (ctypes.c_uint16, [F]),
            "oracle_sylvester": (I, [I, P]),
            "oracle_fwht_f32": (I, [P, I]),
            "oracle_fwht_f64": (I, [P, I]),
            "oracle_inv_sqrt_n": (F, [I]),
            "oracle_sqrt7": (F, []),
            "oracle_rmsnorm": (I, [P, P, I, I, F, P]),
            "oracle_norm_fwht": (I, [P, P, I, I, F, P]),
            "oracle_norm_fwht_f64": (I, [P, P, I, I, D, P]),
            "oracle_quantize_rows": (I, [P, I, I, F, I, P, P, P]),
            "oracle_decode_codes": (I, [P, I, I, I, P]),
            "oracle_norm_fwht_quant": (I, [P, P, I, I, F, F, I, P, P, P]),
            "oracle_ternarize": (I, [P, I, I, F, P, P]),
            "oracle_pack_codes": (I, [P, I, I, P]),
            "oracle_unpack_codes": (I, [P, I, I, P]),
            "oracle_pack_ternary": (I, [P, I, I, F, P, P]),
            "oracle_ternary_gemm_rows": (I, [P, P, I, I, I, P, F, I, I, I, P, P]),
            "oracle_ternary_gemm_rows_t": (I, [P, P, I, I, I, P, F, I, I, I, P, P]),
            "oracle_hbitlinear_forward_rows": (I, [P, P, I, I, I, P, F, I, F, F, I, I, P]),
            "oracle_hbitlinear_forward_rows_t": (I, [P, P, I, I, I, P, F, I, F, F, I, I, P]),
            "oracle_norm_transform": (I, [P, P, I, I, F, I, I, P]),
            "oracle_norm_quant": (I, [P, P, I, I, F, F, I, I, I, P, P, P]),
            "oracle_bitlinear_forward_rows": (I, [P, P, I, I, I, P, F, I, F, F, I, I, I, I, P]),
            "oracle_rotate_weights": (I, [P, P, I, I, P]),
            "oracle_kv_quant": (I, [P, I64, I, I, F, P, P]),
            "oracle_kv_unpack": (I, [P, I64, I, I, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _check(rc, what):
    if rc != 0:
        raise RuntimeError("oracle %s failed with code %d" % (what, rc))


def _threads(n_rows, threads):
    if threads is None:
        threads = os.cpu_count() or 1
    return max(1, min(int(threads), n_rows))


def _split(n, parts):
    step = (n + parts - 1) // parts
    return [(i, min(n, i + step)) for i in range(0, n, step)]


# ----------------------------------------------------------------- primitives

def tree_sum(v):
    v = _c(v, np.float32)
    return float(_load().oracle_tree_sum(_p(v), v.size))


def bf16_to_f32(bits):
    bits = _c(bits, np.uint16)
    return (bits.astype(np.uint32) << 16).view(np.float32)


def f32_to_bf16(x):
    x = _c(x, np.float32).ravel()
    lib = _load()
    out = np.empty(x.size, dtype=np.uint16)
    for i, v in enumerate(x):
        out[i] = lib.oracle_f32_to_bf16(float(v))
    return out


def sylvester(n):
    H = np.empty((n, n), dtype=np.int8)
    _check(_load().oracle_sylvester(n, _p(H)), "sylvester")
    return H


def fwht_f32(u):
    u = np.array(u, dtype=np.float32, copy=True)
    n = u.shape[-1]
    flat = u.reshape(-1, n)
    for row in flat:
        r = np.ascontiguousarray(row)
        _check(_load().oracle_fwht_f32(_p(r), n), "fwht_f32")
        row[:] = r
    return flat.reshape(u.shape)


def fwht_f64(u):
    u = np.array(u, dtype=np.float64, copy=True)
    n = u.shape[-1]
    flat = u.reshape(-1, n)
    for row in flat:
        r = np.ascontiguousarray(row)
        _check(_load().oracle_fwht_f64(_p(r), n), "fwht_f64")
        row[:] = r
    return flat.reshape(u.shape)


def inv_sqrt_n(n):
    return np.float32(_load().oracle_inv_sqrt_n(n))


def sqrt7():
    return np.float32(_load().oracle_sqrt7())


# ---------------------------------------------------------- layer components

def rmsnorm(X_bits, gain=None, norm_eps=1e-6):
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    U = np.empty((M, K), dtype=np.float32)
    _check(_load().oracle_rmsnorm(_p(X_bits), _p(g), M, K, norm_eps, _p(U)), "rmsnorm")
    return U


def norm_fwht(X_bits, gain=None, norm_eps=1e-6, threads=None):
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    V = np.empty((M, K), dtype=np.float32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_norm_fwht(_p(X_bits[a:b]), _p(g), b - a, K, norm_eps, _p(V[a:b])),
               "norm_fwht")

    with ThreadPoolExecutor(_threads(M, threads)) as ex:
        list(ex.map(run, _split(M, _threads(M, threads))))
    return V


def norm_fwht_f64(X_bits, gain=None, norm_eps=1e-6):
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    V = np.empty((M, K), dtype=np.float64)
    _check(_load().oracle_norm_fwht_f64(_p(X_bits), _p(g), M, K, norm_eps, _p(V)), "norm_fwht_f64")
    return V


def code_bytes_per_row(K, act_bits):
    return K if act_bits == 8 else K // 2


def quantize_rows(V, act_bits, quant_eps=1e-5):
    V = _c(V, np.float32)
    M, K = V.shape
    codes = np.empty((M, code_bytes_per_row(K, act_bits)), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    rowsum = np.empty(M, dtype=np.int32)
    _check(_load().oracle_quantize_rows(_p(V), M, K, quant_eps, act_bits, _p(codes), _p(scales),
                                        _p(rowsum)), "quantize_rows")
    return codes, scales, rowsum


def decode_codes(codes, K, act_bits):
    codes = _c(codes, np.uint8)
    M = codes.shape[0]
    q = np.empty((M, K), dtype=np.int8)
    _check(_load().oracle_decode_codes(_p(codes), M, K, act_bits, _p(q)), "decode_codes")
    return q


def norm_fwht_quant(X_bits, act_bits, gain=None, norm_eps=1e-6, quant_eps=1e-5, threads=None):
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    codes = np.empty((M, code_bytes_per_row(K, act_bits)), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    rowsum = np.empty(M, dtype=np.int32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_norm_fwht_quant(_p(X_bits[a:b]), _p(g), b - a, K, norm_eps, quant_eps,
                                          act_bits, _p(codes[a:b]), _p(scales[a:b]),
                                          _p(rowsum[a:b])), "norm_fwht_quant")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return codes, scales, rowsum


def ternarize(W, eps=1e-5):
    W = _c(W, np.float32)
    N, K = W.shape
    t = np.empty((N, K), dtype=np.int8)
    alpha = ctypes.c_float()
    _check(_load().oracle_ternarize(_p(W), N, K, eps, _p(t), ctypes.byref(alpha)), "ternarize")
    return t, np.float32(alpha.value)


def pack_codes(t):
    t = _c(t, np.int8)
    N, K = t.shape
    packed = np.empty((N, K // 16), dtype=np.uint32)
    _check(_load().oracle_pack_codes(_p(t), N, K, _p(packed)), "pack_codes")
    return packed


def unpack_codes(packed, K):
    packed = _c(packed, np.uint32)
    N = packed.shape[0]
    t = np.empty((N, K), dtype=np.int8)
    _check(_load().oracle_unpack_codes(_p(packed), N, K, _p(t)), "unpack_codes")
    return t


def pack_ternary(W, eps=1e-5):
    W = _c(W, np.float32)
    N, K = W.shape
    packed = np.empty((N, K // 16), dtype=np.uint32)
    alpha = ctypes.c_float()
    _check(_load().oracle_pack_ternary(_p(W), N, K, eps, _p(packed), ctypes.byref(alpha)),
           "pack_ternary")
    return packed, np.float32(alpha.value)


def ternary_gemm(codes, scales, act_bits, K, packed, alpha, rows=None, threads=None,
                 want_acc=True):
    """Y (bf16 bits) and acc (int32) for the given rows (default: all)."""
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.float32)
    packed = _c(packed, np.uint32)
    M = codes.shape[0]
    N = packed.shape[0]
    lib = _load()
    if rows is not None:
        rows = np.asarray(rows, dtype=np.int64)
        sub_c = np.ascontiguousarray(codes[rows])
        sub_s = np.ascontiguousarray(scales[rows])
        return ternary_gemm(sub_c, sub_s, act_bits, K, packed, alpha, None, threads, want_acc)
    Y = np.empty((M, N), dtype=np.uint16)
    acc = np.empty((M, N), dtype=np.int32) if want_acc else None
    t = unpack_codes(packed, K) if M else None  # once, shared by the threads

    def run(r):
        a, b = r
        _check(lib.oracle_ternary_gemm_rows_t(_p(codes), _p(scales), act_bits, M, K, _p(t),
                                              float(alpha), N, a, b, _p(Y), _p(acc)),
               "ternary_gemm")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return Y, acc


def hbitlinear_forward(X_bits, packed, alpha, act_bits, gain=None, norm_eps=1e-6,
                       quant_eps=1e-5, rows=None, threads=None):
    """Y (bf16 bits) [M x N] for all rows, or [len(rows) x N] for the given rows."""
    X_bits = _c(X_bits, np.uint16)
    if rows is not None:
        X_bits = np.ascontiguousarray(X_bits[np.asarray(rows, dtype=np.int64)])
    packed = _c(packed, np.uint32)
    M, K = X_bits.shape
    N = packed.shape[0]
    g = None if gain is None else _c(gain, np.float32)
    Y = np.empty((M, N), dtype=np.uint16)
    lib = _load()
    t = unpack_codes(packed, K) if M else None  # once, shared by the threads

    def run(r):
        a, b = r
        _check(lib.oracle_hbitlinear_forward_rows_t(_p(X_bits), _p(g), M, K, N, _p(t),
                                                    float(alpha), act_bits, norm_eps, quant_eps,
                                                    a, b, _p(Y)), "hbitlinear_forward")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return Y


# ------------------------------------------------------------------ variants

def norm_transform(X_bits, gain=None, norm_eps=1e-6, layernorm=False, hadamard=True,
                   threads=None):
    """fp32 V = T(N(X)): RMSNorm or LayerNorm, then the normalised FWHT or nothing."""
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    V = np.empty((M, K), dtype=np.float32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_norm_transform(_p(X_bits[a:b]), _p(g), b - a, K, norm_eps,
                                         int(layernorm), int(hadamard), _p(V[a:b])),
               "norm_transform")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return V


def norm_quant(X_bits, act_bits, gain=None, norm_eps=1e-6, quant_eps=1e-5, layernorm=False,
               hadamard=True, threads=None):
    X_bits = _c(X_bits, np.uint16)
    M, K = X_bits.shape
    g = None if gain is None else _c(gain, np.float32)
    codes = np.empty((M, code_bytes_per_row(K, act_bits)), dtype=np.uint8)
    scales = np.empty(M, dtype=np.float32)
    rowsum = np.empty(M, dtype=np.int32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_norm_quant(_p(X_bits[a:b]), _p(g), b - a, K, norm_eps, quant_eps,
                                     act_bits, int(layernorm), int(hadamard), _p(codes[a:b]),
                                     _p(scales[a:b]), _p(rowsum[a:b])), "norm_quant")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return codes, scales, rowsum


def bitlinear_forward(X_bits, packed, alpha, act_bits, gain=None, norm_eps=1e-6,
                      quant_eps=1e-5, layernorm=False, hadamard=True, rows=None, threads=None):
    """Y (bf16 bits) of the layer with the variant choices of norm_transform."""
    X_bits = _c(X_bits, np.uint16)
    if rows is not None:
        X_bits = np.ascontiguousarray(X_bits[np.asarray(rows, dtype=np.int64)])
    packed = _c(packed, np.uint32)
    M, K = X_bits.shape
    N = packed.shape[0]
    g = None if gain is None else _c(gain, np.float32)
    Y = np.empty((M, N), dtype=np.uint16)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_bitlinear_forward_rows(_p(X_bits), _p(g), M, K, N, _p(packed),
                                                 float(alpha), act_bits, norm_eps, quant_eps,
                                                 int(layernorm), int(hadamard), a, b, _p(Y)),
               "bitlinear_forward")

    if M:
        nt = _threads(M, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(M, nt)))
    return Y


def rotate_weights(W, signs=None, threads=None):
    """W_rot = FWHT(W * signs) / sqrt(K) row by row (fp32)."""
    W = _c(W, np.float32)
    N, K = W.shape
    s = None if signs is None else _c(signs, np.float32)
    out = np.empty((N, K), dtype=np.float32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_rotate_weights(_p(W[a:b]), _p(s), b - a, K, _p(out[a:b])),
               "rotate_weights")

    if N:
        nt = _threads(N, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(N, nt)))
    return out


def kv_code_bytes(D, bits):
    return D // 32 * 4 * bits


def kv_quant(X_bits, bits, eps=1e-5, threads=None):
    """Packed unsigned codes [rows x D*bits/8] and fp32 scales [rows] per head row."""
    X_bits = _c(X_bits, np.uint16)
    D = X_bits.shape[-1]
    flat = X_bits.reshape(-1, D)
    rows = flat.shape[0]
    codes = np.empty((rows, kv_code_bytes(D, bits)), dtype=np.uint8)
    scales = np.empty(rows, dtype=np.float32)
    lib = _load()

    def run(r):
        a, b = r
        _check(lib.oracle_kv_quant(_p(flat[a:b]), b - a, D, int(bits), float(eps),
                                   _p(codes[a:b]), _p(scales[a:b])), "kv_quant")

    if rows:
        nt = _threads(rows, threads)
        with ThreadPoolExecutor(nt) as ex:
            list(ex.map(run, _split(rows, nt)))
    return codes, scales


def kv_unpack(codes, D, bits):
    codes = _c(codes, np.uint8)
    rows = codes.shape[0]
    u = np.empty((rows, D), dtype=np.uint8)
    _check(_load().oracle_kv_unpack(_p(codes), rows, D, int(bits), _p(u)), "kv_unpack")
    return u
