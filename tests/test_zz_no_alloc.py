"""The allocation-free GEMV entry point (hbl_ternary_gemv_noalloc).

Some callers cannot give a library scratch memory or let it allocate: an
engine's custom-op hook that is handed only its inputs and outputs, or a
token-by-token decode loop that must not block on the allocator or risk an
out-of-memory failure mid-step.  For them the library keeps the split-K
partial sums of its CUDA-core GEMV in one fixed device array.

This file calls that entry point through the C ABI twice in a row (different
shapes, so the second call runs over the first call's leftovers in the shared
array) and checks each result against the CPU oracle element by element:
int32 accumulators exactly, bf16 outputs within 1 ulp (the stated tolerance;
both sides evaluate the same IEEE operations, so they are expected equal).  It
also checks the Python wrapper (with the accumulators, and with more than 8
tokens, which run in consecutive 8-token chunks) and the regular workspace
entry point on the same inputs.

Kept in a file of its own that pytest collects last.
"""
import ctypes

import numpy as np
import pytest
import torch

import hadamard_rotated_int4_b200 as hbl
import oracle
from hadamard_rotated_int4_b200 import inputs

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _case(M, K, N, bits, seed):
    X = inputs.swiglu_acts(M, K, seed=seed)
    codes, scales, rowsum = oracle.norm_fwht_quant(X, bits)
    packed, alpha = oracle.pack_ternary(inputs.latent_weights(N, K, seed=seed))
    want_Y, want_acc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to(DEV)
    dev = (t(codes), t(scales), t(rowsum), t(packed.view(np.int32)),
           t(np.array([alpha, 0, 0, 0], dtype=np.float32)))
    return dev, want_Y, want_acc


def _ulp(a_bits, b_bits):
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    a = np.where(a & 0x8000, 0x8000 - a, a)
    b = np.where(b & 0x8000, 0x8000 - b, b)
    return int(np.abs(a - b).max()) if a.size else 0


def _bits(Y):
    return Y.view(torch.int16).cpu().numpy().view(np.uint16)


def test_noalloc_gemv_matches_oracle_twice():
    lib = hbl.lib()
    cases = [(8, 16384, 4096, 4, 11), (5, 4096, 1040, 8, 12)]
    for (M, K, N, bits, seed) in cases:
        (codes, scales, rowsum, packed, alpha), want_Y, want_acc = _case(M, K, N, bits, seed)
        Y = torch.empty((M, N), dtype=torch.bfloat16, device=DEV)
        acc = torch.empty((M, N), dtype=torch.int32, device=DEV)
        status = torch.zeros(4, dtype=torch.int32, device=DEV)
        p = lambda t: ctypes.c_void_p(t.data_ptr())
        st = lib.hbl_ternary_gemv_noalloc(p(codes), p(scales), p(rowsum), bits, M, K, p(packed),
                                          p(alpha), N, p(Y), p(acc), p(status),
                                          ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert st == 0, hbl.STATUS_NAMES.get(st, st)
        torch.cuda.synchronize()
        assert int(status[0].item()) == 0
        assert np.array_equal(acc.cpu().numpy(), want_acc)
        assert _ulp(_bits(Y), want_Y) <= 1
        # the regular entry point with a workspace gives the same results
        Yw, accw = hbl.ternary_gemm(codes, scales, rowsum, bits, K, packed, alpha, want_acc=True)
        torch.cuda.synchronize()
        assert np.array_equal(accw.cpu().numpy(), want_acc)
        assert _ulp(_bits(Yw), want_Y) <= 1


def test_noalloc_python_wrapper_with_accumulators_and_chunks():
    # 19 tokens: three consecutive chunks (8, 8, 3) through the fixed array
    (codes, scales, rowsum, packed, alpha), want_Y, want_acc = _case(19, 4096, 4096, 4, 13)
    for _ in range(2):
        Y, acc = hbl.ternary_gemv_noalloc(codes, scales, rowsum, 4, 4096, packed, alpha,
                                          want_acc=True)
        torch.cuda.synchronize()
        assert np.array_equal(acc.cpu().numpy(), want_acc)
        assert _ulp(_bits(Y), want_Y) <= 1
    Y = hbl.ternary_gemv_noalloc(codes, scales, rowsum, 4, 4096, packed, alpha)
    torch.cuda.synchronize()
    assert _ulp(_bits(Y), want_Y) <= 1


def test_noalloc_rejects_shapes_beyond_the_fixed_scratch():
    # 8 tokens x 131072 outputs at K = 16384 (ksplit 1) need 4 MiB of partials,
    # more than the fixed 2 MiB: refused before any pointer is touched.
    lib = hbl.lib()
    a = ctypes.c_void_p(0x10000)
    st = lib.hbl_ternary_gemv_noalloc(a, a, a, 4, 8, 16384, a, a, 131072, a, None, None, None)
    assert st == 5
