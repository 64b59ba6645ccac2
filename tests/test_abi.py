"""The C ABI: the library loads, exports every call include/hbl.h declares, and
rejects bad arguments on the host before touching the GPU.  CPU only: every
call here fails validation before any CUDA call, so no device is needed --
except one, which runs in a child process with no device visible and checks
that a well-formed call then fails with HBL_ERR_CUDA instead of running on the
host."""
import ctypes
import os
import re

import pytest

import hadamard_rotated_int4_b200 as hbl

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "hbl.h")

# fake but 16-byte-aligned device addresses: validation never dereferences them
A = ctypes.c_void_p(0x10000)
B = ctypes.c_void_p(0x20000)
C = ctypes.c_void_p(0x30000)
D = ctypes.c_void_p(0x40000)
E = ctypes.c_void_p(0x50000)
MIS = ctypes.c_void_p(0x10004)  # misaligned
NUL = None


def declared():
    src = open(HEADER).read()
    return sorted(set(re.findall(r"HBL_API\s+[\w\s\*]*?\b(hbl_\w+)\s*\(", src)))


def test_header_declares_the_expected_calls():
    names = declared()
    for n in ("hbl_pack_ternary", "hbl_norm_fwht_quant", "hbl_ternary_gemm",
              "hbl_hbitlinear_forward", "hbl_workspace_size", "hbl_status_string"):
        assert n in names
    assert set(names) == set(hbl.EXPORTS)


def test_library_exports_every_declared_symbol():
    lib = hbl.lib()
    for n in declared():
        assert hasattr(lib, n), n
    out = os.popen("nm -D --defined-only %s" % hbl.LIB_PATH).read()
    exported = set(re.findall(r"\bT (hbl_\w+)", out))
    assert set(declared()) <= exported


def test_status_strings_and_version():
    lib = hbl.lib()
    for code in range(8):
        assert lib.hbl_status_string(code).decode() not in ("", "unknown status")
    assert lib.hbl_status_string(99).decode() == "unknown status"
    assert lib.hbl_version() >= 100


def test_workspace_sizes():
    # pack: one float per weight row (rounded to 256 B)
    assert hbl.workspace_size(hbl.OP_PACK_TERNARY, 0, 4096, 100, 0) == 512
    # forward: codes + scales + rowsum, each 256-aligned (tensor-core path: no GEMM scratch)
    M, K, N = 8192, 16384, 4096
    ss = hbl.PATH_TC_SS
    got = hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, M, K, N, 4, ss)
    assert got == M * K + 2 * M * 4  # codes one byte each inside the layer (M % 32 == 0)
    got8 = hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, M, K, N, 8, ss)
    assert got8 == M * K + 2 * M * 4
    hio = hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD_HOSTIO, M, K, N, 4, ss)
    assert hio == got + M * K * 2 + M * N * 2
    assert hbl.workspace_size(hbl.OP_TERNARY_GEMM, M, K, N, 4, ss) == 0
    # automatic choice at this batch: the TMA-fed GEMM, plus N*K bytes of expanded weights
    auto = hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, M, K, N, 4)
    assert auto == M * K + 2 * M * 4 + N * K
    assert hbl.workspace_size(hbl.OP_TERNARY_GEMM, M, K, N, hbl.ACT_INT4_BYTES) == N * K
    assert hbl.workspace_size(hbl.OP_TERNARY_GEMM, M, K, N, 8) == N * K
    # small M: the row GEMV (K >= 2048) needs no scratch; below that the split-K
    # GEMV needs integer partials
    assert hbl.workspace_size(hbl.OP_TERNARY_GEMM, 1, 16384, 4096, 4) == 0
    assert hbl.workspace_size(hbl.OP_TERNARY_GEMM, 8, 1024, 4096, 4) > 0


@pytest.mark.parametrize("K", [0, 8, 24, 100, 65536])
def test_bad_K_is_a_shape_error(K):
    lib = hbl.lib()
    s = lib.hbl_norm_fwht_quant(A, NUL, 4, K, 1e-6, 1e-5, 4, B, C, D, NUL, NUL)
    assert s == 2
    sz = ctypes.c_size_t()
    assert lib.hbl_workspace_size(hbl.OP_HBITLINEAR_FORWARD, 4, K, 64, 4, ctypes.byref(sz)) == 2


def test_validation_errors():
    lib = hbl.lib()
    # null pointer, bad act_bits, bad eps
    assert lib.hbl_norm_fwht_quant(NUL, NUL, 4, 256, 1e-6, 1e-5, 4, B, C, D, NUL, NUL) == 1
    assert lib.hbl_norm_fwht_quant(A, NUL, 4, 256, 1e-6, 1e-5, 3, B, C, D, NUL, NUL) == 1
    assert lib.hbl_norm_fwht_quant(A, NUL, 4, 256, -1.0, 1e-5, 4, B, C, D, NUL, NUL) == 1
    assert lib.hbl_norm_fwht_quant(A, NUL, 4, 256, float("nan"), 1e-5, 4, B, C, D, NUL, NUL) == 1
    # negative M
    assert lib.hbl_norm_fwht_quant(A, NUL, -1, 256, 1e-6, 1e-5, 4, B, C, D, NUL, NUL) == 2
    # misaligned pointers
    assert lib.hbl_norm_fwht_quant(MIS, NUL, 4, 256, 1e-6, 1e-5, 4, B, C, D, NUL, NUL) == 3
    assert lib.hbl_norm_fwht_quant(A, MIS, 4, 256, 1e-6, 1e-5, 4, B, C, D, NUL, NUL) == 3
    assert lib.hbl_norm_fwht(A, NUL, 4, 256, 1e-6, MIS, NUL, NUL) == 3
    # M == 0 is a no-op that succeeds without a device
    assert lib.hbl_norm_fwht_quant(A, NUL, 0, 256, 1e-6, 1e-5, 4, B, C, D, NUL, NUL) == 0
    # GEMM: N not a multiple of 16, rowsum required, workspace required for small M
    gemm = lib.hbl_ternary_gemm
    assert gemm(A, B, C, 4, 64, 256, D, E, 40, A, NUL, NUL, 0, NUL, NUL) == 2
    assert gemm(A, B, NUL, 4, 64, 256, D, E, 64, A, NUL, NUL, 0, NUL, NUL) == 1
    assert gemm(A, B, C, 4, 1, 256, D, E, 64, A, NUL, NUL, 0, NUL, NUL) == 5
    # forward: workspace too small
    fwd = lib.hbl_hbitlinear_forward
    assert fwd(A, NUL, 64, 256, 64, B, C, 4, 1e-6, 1e-5, D, E, 16, NUL, NUL) == 5
    assert fwd(A, NUL, 64, 256, 64, B, C, 5, 1e-6, 1e-5, D, E, 1 << 20, NUL, NUL) == 1
    # pack
    pack = lib.hbl_pack_ternary
    assert pack(A, 16, 100, 1e-5, B, C, D, 1024, NUL) == 2
    assert pack(A, 16, 256, 1e-5, B, C, NUL, 0, NUL) == 5
    assert pack(A, 0, 256, 1e-5, B, C, D, 1024, NUL) == 2
    # per-call back-end choice: out-of-range paths are refused
    sz = ctypes.c_size_t()
    assert lib.hbl_workspace_size_path(hbl.OP_TERNARY_GEMM, 4, 256, 64, 4, 8, ctypes.byref(sz)) == 1
    assert lib.hbl_workspace_size_path(hbl.OP_TERNARY_GEMM, 4, 256, 64, 4, -1,
                                       ctypes.byref(sz)) == 1
    assert lib.hbl_ternary_gemm_path(A, B, C, 4, 64, 256, D, E, 64, A, NUL, E, 1 << 20, NUL, 9,
                                     NUL) == 1
    assert lib.hbl_hbitlinear_forward_path(A, NUL, 64, 256, 64, B, C, 4, 1e-6, 1e-5, D, E,
                                           1 << 20, NUL, 8, NUL) == 1


def test_binding_rejects_non_cuda_tensors():
    import torch

    with pytest.raises(TypeError):
        hbl.norm_fwht_quant(torch.zeros(4, 256, dtype=torch.bfloat16), 4)


def test_variant_rotation_and_kv_validation():
    lib = hbl.lib()
    # variant flags: only HBL_NORM_LAYERNORM | HBL_NORM_NO_HADAMARD
    assert lib.hbl_norm_transform(A, NUL, 4, 256, 1e-6, 4, B, NUL, NUL) == 1
    assert lib.hbl_norm_quant(A, NUL, 4, 256, 1e-6, 1e-5, 4, 8, B, C, D, NUL, NUL) == 1
    assert lib.hbl_norm_quant(A, NUL, 4, 100, 1e-6, 1e-5, 4, 2, B, C, D, NUL, NUL) == 2
    assert lib.hbl_norm_quant(A, NUL, 0, 256, 1e-6, 1e-5, 4, 3, B, C, D, NUL, NUL) == 0
    fwd = lib.hbl_bitlinear_forward
    assert fwd(A, NUL, 64, 256, 64, B, C, 4, 16, 1e-6, 1e-5, D, E, 1 << 20, NUL, NUL) == 1
    assert fwd(A, NUL, 64, 256, 64, B, C, 4, 2, 1e-6, 1e-5, D, E, 16, NUL, NUL) == 5
    # rotation: K rule, alignment, N == 0 is a no-op
    assert lib.hbl_rotate_weights(A, NUL, 8, 100, B, NUL, NUL) == 2
    assert lib.hbl_rotate_weights(A, NUL, -1, 256, B, NUL, NUL) == 2
    assert lib.hbl_rotate_weights(MIS, NUL, 8, 256, B, NUL, NUL) == 3
    assert lib.hbl_rotate_weights(A, MIS, 8, 256, B, NUL, NUL) == 3
    assert lib.hbl_rotate_weights(A, NUL, 0, 256, B, NUL, NUL) == 0
    # KV quantiser: bits, head size, eps, alignment, empty
    kv = lib.hbl_kv_quant
    assert kv(A, 10, 128, 5, 1e-5, B, C, NUL, NUL) == 1
    assert kv(A, 10, 128, 3, -1.0, B, C, NUL, NUL) == 1
    assert kv(A, 10, 96, 3, 1e-5, B, C, NUL, NUL) == 2
    assert kv(A, -1, 128, 3, 1e-5, B, C, NUL, NUL) == 2
    assert kv(MIS, 10, 128, 3, 1e-5, B, C, NUL, NUL) == 3
    assert kv(A, 10, 128, 3, 1e-5, NUL, C, NUL, NUL) == 1
    assert kv(A, 0, 128, 3, 1e-5, B, C, NUL, NUL) == 0


def test_expanded_weight_calls_validation():
    lib = hbl.lib()
    assert lib.hbl_expand_ternary(A, 8, 100, B, NUL, NUL) == 2
    assert lib.hbl_expand_ternary(A, 0, 256, B, NUL, NUL) == 0
    assert lib.hbl_expand_ternary(MIS, 8, 256, B, NUL, NUL) == 3
    s8w = lib.hbl_ternary_gemm_s8w
    assert s8w(A, B, 4, 16, 256, C, D, 64, E, NUL, NUL, NUL) == 1    # packed nibbles refused
    assert s8w(A, B, 8, 16, 64, C, D, 64, E, NUL, NUL, NUL) == 2     # K < 128
    assert s8w(A, B, 0x204, 16, 256, C, D, 40, E, NUL, NUL, NUL) == 2
    assert s8w(A, B, 8, 0, 256, C, D, 64, E, NUL, NUL, NUL) == 0


def test_selftest_validation():
    lib = hbl.lib()
    assert lib.hbl_probe_tc_int8(148, 100, NUL, NUL) == 1
    assert lib.hbl_probe_tc_int8(0, 100, A, NUL) == 1
    assert lib.hbl_probe_tc_int8(148, 0, A, NUL) == 1
    assert lib.hbl_probe_tc_int8(148, (1 << 22) + 1, A, NUL) == 1
    assert lib.hbl_probe_tc_int8(148, 100, MIS, NUL) == 3
    assert lib.hbl_selftest_bounded_wait(0, 100, NUL, NUL) == 1
    assert lib.hbl_selftest_bounded_wait(0, 0, A, NUL) == 1
    assert lib.hbl_selftest_bounded_wait(0, 100, MIS, NUL) == 3


def test_no_device_is_an_error_not_a_fallback():
    # With no GPU visible, a well-formed call reaches the device query and
    # returns HBL_ERR_CUDA (nothing runs on the host instead), and the binding
    # raises when the library is missing.  Run in a child process with no
    # device visible, so the fake pointers can never reach a GPU.
    import subprocess
    import sys

    code = r'''
import ctypes, sys
sys.path.insert(0, %r)
import hadamard_rotated_int4_b200 as hbl
lib = hbl.lib()
A, B, C, D, E = (ctypes.c_void_p(a) for a in (0x10000, 0x20000, 0x30000, 0x40000, 0x50000))
need = ctypes.c_size_t(0)
assert lib.hbl_workspace_size(hbl.OP_HBITLINEAR_FORWARD, 512, 4096, 256, 4, ctypes.byref(need)) == 0
st = lib.hbl_hbitlinear_forward(A, None, 512, 4096, 256, B, C, 4, ctypes.c_float(1e-6),
                                ctypes.c_float(1e-5), D, E, ctypes.c_size_t(need.value), None, None)
print("forward", st)
st = lib.hbl_norm_fwht_quant(A, None, 512, 4096, ctypes.c_float(1e-6), ctypes.c_float(1e-5), 4,
                             B, C, D, None, None)
print("quant", st)
hbl.LIB_PATH = "/nonexistent/libhbl.so"
hbl._lib = None
try:
    hbl.lib()
    print("missing none")
except RuntimeError:
    print("missing raises")
''' % ROOT
    env = dict(os.environ, CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code], env=env, capture_output=True, text=True,
                       timeout=300)
    assert r.returncode == 0, r.stderr[-2000:]
    out = r.stdout.split()
    assert out == ["forward", "6", "quant", "6", "missing", "raises"], r.stdout
