"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.  Integer outputs (codes, rowsum, packed weights, int32
accumulators) and the fp32 per-token scales and alpha must be bit-identical;
fp32 transform values are bit-identical to the oracle's fp32 evaluation and
within 1e-6 (relative to the row's largest |v|) of the fp64 evaluation; bf16
outputs must be within 1 bf16 ulp (they are expected bit-identical, since both
sides evaluate the same IEEE operations in the same order).
"""
import numpy as np
import pytest
import torch

import hadamard_rotated_int4_b200 as hbl
import oracle
from hadamard_rotated_int4_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def to_dev_bf16(bits):
    return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).to(DEV)


def bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def bf16_ulp_diff(a_bits, b_bits):
    a = a_bits.astype(np.int32)
    b = b_bits.astype(np.int32)
    # order-preserving map of bf16 bit patterns to integers
    a = np.where(a & 0x8000, 0x8000 - a, a)
    b = np.where(b & 0x8000, 0x8000 - b, b)
    return np.abs(a - b)


def acts(M, K, seed=0, kind="gauss"):
    if kind == "gauss":
        return inputs.gaussian_acts(M, K, seed=seed, frac=0.01, mult=30.0)
    if kind == "t":
        return inputs.student_t_acts(M, K, seed=seed)
    if kind == "swiglu":
        return inputs.swiglu_acts(M, K, seed=seed)
    raise KeyError(kind)


# ------------------------------------------------------------ norm + FWHT

@pytest.mark.parametrize("K", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768])
@pytest.mark.parametrize("M", [1, 37])
def test_norm_fwht_values(K, M):
    X = acts(M, K, seed=K + M)
    V = hbl.norm_fwht(to_dev_bf16(X)).cpu().numpy()
    want32 = oracle.norm_fwht(X)
    assert np.array_equal(V.view(np.uint32), want32.view(np.uint32))
    want64 = oracle.norm_fwht_f64(X)
    rel = np.abs(V - want64).max(axis=1) / np.abs(want64).max(axis=1)
    assert rel.max() < 1e-6


@pytest.mark.parametrize("K", [256, 4096])
def test_norm_fwht_with_gain(K):
    X = acts(5, K, seed=3)
    g = np.random.default_rng(1).uniform(0.5, 1.5, K).astype(np.float32)
    V = hbl.norm_fwht(to_dev_bf16(X), gain=torch.from_numpy(g).to(DEV)).cpu().numpy()
    assert np.array_equal(V.view(np.uint32), oracle.norm_fwht(X, gain=g).view(np.uint32))


def underflow_rows(K, seed):
    """Rows whose squares fall below the fp32 normal range, so the rounding of
    each square decides the RMS statistic: the hand-pinned (2^-75, 1.5*2^-75)
    pattern, the same with its second half negated, and N(0,1) rows scaled to
    ~1e-20 and ~1e-22 (squares ~1e-40 / 1e-44, subnormal)."""
    rng = np.random.default_rng(seed)
    X = np.empty((4, K), dtype=np.uint16)
    X[0] = np.tile(np.array([0x1A00, 0x1A40], np.uint16), K // 2)
    X[1] = X[0]
    X[1, K // 2:] |= 0x8000
    for r, sc in ((2, 1e-20), (3, 1e-22)):
        v = torch.from_numpy((rng.standard_normal(K) * sc).astype(np.float32))
        X[r] = v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    return X


@pytest.mark.parametrize("K", [16, 256, 4096, 16384])
def test_norm_with_underflowing_squares(K):
    # every square rounded to fp32 before the tree: the pinned rows with
    # norm_eps = 2^-149, the scaled rows also with norm_eps = 0
    X = underflow_rows(K, seed=K)
    for eps, rows in ((float(2.0 ** -149), slice(0, 4)), (0.0, slice(2, 4))):
        Xr = np.ascontiguousarray(X[rows])
        V = hbl.norm_fwht(to_dev_bf16(Xr), norm_eps=eps).cpu().numpy()
        want = oracle.norm_fwht(Xr, norm_eps=eps)
        assert np.all(np.isfinite(want))
        assert np.array_equal(V.view(np.uint32), want.view(np.uint32))
        for bits in (4, 8):
            codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(Xr), bits, norm_eps=eps)
            wc, ws, wr = oracle.norm_fwht_quant(Xr, bits, norm_eps=eps)
            assert np.array_equal(codes.cpu().numpy(), wc)
            assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
            assert np.array_equal(rowsum.cpu().numpy(), wr)


# ------------------------------------------------- fused norm+FWHT+quant

def check_quant(X, bits, gain=None):
    g_dev = None if gain is None else torch.from_numpy(gain).to(DEV)
    codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(X), bits, gain=g_dev)
    torch.cuda.synchronize()
    wc, ws, wr = oracle.norm_fwht_quant(X, bits, gain=gain)
    c = codes.cpu().numpy()
    if not np.array_equal(c, wc):
        bad = np.argwhere(c != wc)
        raise AssertionError("codes differ at %d bytes, first %s" % (len(bad), bad[:5].tolist()))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [16, 32, 64, 128, 256, 512, 1024, 2048, 4096, 8192, 16384, 32768])
def test_quant_all_K(bits, K):
    M = 45  # ragged against every rows-per-group size
    check_quant(acts(M, K, seed=K, kind="t"), bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [256, 2048, 16384])
def test_quant_with_gain(bits, K):
    g = np.random.default_rng(K).uniform(0.25, 2.0, K).astype(np.float32)
    check_quant(acts(9, K, seed=5), bits, gain=g)


@pytest.mark.parametrize("bits", [4, 8])
def test_quant_edge_rows(bits):
    K = 4096
    X = acts(6, K, seed=2)
    X[0] = 0                                      # zero row
    X[1] = np.uint16(0x3F80)                      # constant 1.0
    X[2, :] = 0
    X[2, 17] = np.uint16(0x4120)                  # single spike (10.0)
    X[3] = np.uint16(0x0001)                      # smallest bf16 subnormal
    X[4, ::2] = np.uint16(0x7F00)                 # large values (~1.7e38)
    check_quant(X, bits)


def hadamard_row_bits(K, k, scale=1.0):
    # bf16 bits of scale * (row k of the Sylvester Hadamard matrix): its
    # transform is a single spike of height scale * sqrt(K)
    i = np.arange(K)
    par = np.array([bin(int(k) & int(t)).count("1") & 1 for t in i])
    v = np.where(par == 1, -scale, scale).astype(np.float32)
    return (v.view(np.uint32) >> 16).astype(np.uint16)


@pytest.mark.parametrize("K", [16384, 32768])
def test_quant_int4_large_k_spiky_rows(K):
    # INT4 codes at K >= 16384 are clamped as int16 pairs on rows whose
    # statistic bounds |q| below 2^15, else on 32-bit patterns: spike rows
    # (|q| would reach sqrt7 K), near-spikes on both sides of the bound,
    # normal rows; packed nibbles, one byte per code, interleaved bytes
    rng = np.random.default_rng(K)
    X = acts(8, K, seed=3)
    X[0] = hadamard_row_bits(K, 5)
    X[1] = hadamard_row_bits(K, 77, scale=-3.0)
    h = (hadamard_row_bits(K, 9).astype(np.uint32) << 16).view(np.float32)
    for r, eps in ((2, 0.02), (3, 0.1), (4, 0.5)):
        v = (h + eps * rng.standard_normal(K)).astype(np.float32)
        X[r] = (v.view(np.uint32) >> 16).astype(np.uint16)
    X[5] = 0
    wc, ws, wr = oracle.norm_fwht_quant(X, 4)
    want_q = oracle.decode_codes(wc, K, 4)
    for bits in (4, hbl.ACT_INT4_BYTES, hbl.ACT_INT4_I32):
        codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(X), bits)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
        assert np.array_equal(rowsum.cpu().numpy()[:8], wr)
        got = codes.cpu().numpy()
        if bits == 4:
            assert np.array_equal(got, wc)
        elif bits == hbl.ACT_INT4_BYTES:
            assert np.array_equal(got.view(np.int8).astype(np.int32), want_q)
        else:
            assert np.array_equal(il_decode(got, 8, K).astype(np.int32), want_q)
    # the same rows through the one-kernel decode forward (one token)
    if K == 16384:
        W = inputs.latent_weights(512, K, seed=1)
        packed, alpha = oracle.pack_ternary(W)
        for r in range(6):
            assert np.array_equal(forward(X[r:r + 1], packed, alpha, 4),
                                  oracle.hbitlinear_forward(X[r:r + 1], packed, alpha, 4))


@pytest.mark.parametrize("K", [8192, 16384])
def test_quant_many_rows_large_k(K):
    # more rows than three per SM: at K = 16384 the 128-values-per-thread
    # launch (fewer rows take the 64-values one, covered above)
    X = acts(1000, K, seed=K, kind="t")
    for bits in (4, 8):
        check_quant(X, bits)
    codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(X), hbl.ACT_INT4_BYTES)
    wc, ws, wr = oracle.norm_fwht_quant(X, 4)
    assert np.array_equal(codes.cpu().numpy().view(np.int8).astype(np.int32),
                          oracle.decode_codes(wc, K, 4))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))


def test_quant_workloads_full_size():
    # quant workload (8192 x 4096, Student-t, 1% channels x 20), both widths
    X = inputs.activations("quant")
    for bits in (4, 8):
        check_quant(X, bits)


def test_quant_empty_M():
    codes, scales, rowsum = hbl.norm_fwht_quant(
        torch.zeros((0, 256), dtype=torch.bfloat16, device=DEV), 4)
    assert codes.numel() == 0


def test_quant_deterministic():
    X = to_dev_bf16(acts(300, 4096, seed=9))
    c0, s0, r0 = hbl.norm_fwht_quant(X, 4)
    for _ in range(5):
        c, s, r = hbl.norm_fwht_quant(X, 4)
        assert torch.equal(c, c0) and torch.equal(s, s0) and torch.equal(r, r0)


# ------------------------------------------- interleaved one-byte code layout

def il_decode(buf, M, K):
    """[ceil32(M), K] bytes in the 32-row interleaved layout -> int8 [M, K]."""
    Mp = (M + 31) // 32 * 32
    b = np.asarray(buf, dtype=np.uint8).reshape(Mp // 32, K // 16, 32, 16)
    return b.transpose(0, 2, 1, 3).reshape(Mp, K)[:M].view(np.int8)


def il_encode(q, K):
    M = q.shape[0]
    Mp = (M + 31) // 32 * 32
    full = np.zeros((Mp, K), dtype=np.int8)
    full[:M] = q
    return np.ascontiguousarray(
        full.view(np.uint8).reshape(Mp // 32, 32, K // 16, 16).transpose(0, 2, 1, 3)).reshape(Mp, K)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K", [16, 128, 256, 2048, 4096, 16384])
def test_quant_interleaved_layout(bits, K):
    M = 45
    X = acts(M, K, seed=K + 1, kind="t")
    flag = hbl.ACT_INT4_I32 if bits == 4 else hbl.ACT_INT8_I32
    codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(X), flag)
    torch.cuda.synchronize()
    wc, ws, wr = oracle.norm_fwht_quant(X, bits)
    assert codes.shape == ((M + 31) // 32 * 32, K)
    assert np.array_equal(il_decode(codes.cpu().numpy(), M, K), oracle.decode_codes(wc, K, bits))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 16, 16), (45, 128, 272), (300, 4096, 256), (520, 2048, 400)])
def test_gemm_interleaved_layout(bits, M, K, N):
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M)
    q = oracle.decode_codes(codes, K, bits)
    flag = hbl.ACT_INT4_I32 if bits == 4 else hbl.ACT_INT8_I32
    Y, acc = hbl.ternary_gemm(
        torch.from_numpy(il_encode(q, K)).to(DEV), torch.from_numpy(scales).to(DEV),
        torch.from_numpy(rowsum).to(DEV), flag, K,
        torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV), want_acc=True)
    torch.cuda.synchronize()
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc.cpu().numpy(), wacc)
    assert np.array_equal(bf16_bits(Y), wY)


# ------------------------------------------------------------ ternary pack

@pytest.mark.parametrize("N,K", [(16, 16), (1, 16), (7, 32), (48, 256), (128, 256), (100, 2048),
                                 (1500, 512), (3001, 1024), (4096, 4096), (4096, 16384)])
def test_pack_ternary(N, K):
    # N = 3001 = 2048 + 512 + 256 + 128 + 32 + 16 + 8 + 1 exercises every
    # block size of the left-complete tree over the row sums (two row sums
    # per thread in the 2048 block); K < 1024 takes the lane-chunk row sums
    W = inputs.latent_weights(N, K, seed=N + K)
    packed, alpha = hbl.pack_ternary(torch.from_numpy(W).to(DEV))
    wp, wa = oracle.pack_ternary(W)
    assert alpha.cpu().numpy()[0].view(np.uint32) == np.float32(wa).view(np.uint32)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), wp)


# ------------------------------------------------------------ GEMM

def make_gemm_case(M, K, N, bits, seed=0):
    X = acts(M, K, seed=seed, kind="swiglu")
    codes, scales, rowsum = oracle.norm_fwht_quant(X, bits)
    W = inputs.latent_weights(N, K, seed=seed)
    packed, alpha = oracle.pack_ternary(W)
    return codes, scales, rowsum, packed, alpha


def run_gemm(codes, scales, rowsum, bits, K, packed, alpha, path):
    Y, acc = hbl.ternary_gemm(
        torch.from_numpy(codes).to(DEV), torch.from_numpy(scales).to(DEV),
        torch.from_numpy(rowsum).to(DEV), bits, K,
        torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV),
        want_acc=True, path=path)
    torch.cuda.synchronize()
    return bf16_bits(Y), acc.cpu().numpy()


@pytest.mark.parametrize("path", [1, 2, 3])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 256, 128), (3, 16, 16), (8, 64, 48), (9, 128, 272),
                                   (127, 256, 256), (128, 512, 256), (129, 2048, 512),
                                   (300, 4096, 272)])
def test_gemm_paths(path, bits, M, K, N):
    if path == 2 and M > 129:
        M = 40  # the CUDA-core path is exercised in 8-token chunks; keep it quick
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M + N)
    Y, acc = run_gemm(codes, scales, rowsum, bits, K, packed, alpha, path)
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc, wacc)
    assert bf16_ulp_diff(Y, wY).max() <= 1
    assert np.array_equal(Y, wY)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 128, 16), (45, 256, 272), (128, 512, 256),
                                   (300, 4096, 400), (1000, 2048, 512), (257, 16384, 4096)])
def test_gemm_tma_one_byte_codes(bits, M, K, N):
    # the TMA-fed kernel reads one byte per code: INT8 row-major, or INT4 values
    # one byte each (HBL_ACT_INT4_BYTES)
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M + K)
    q = oracle.decode_codes(codes, K, bits)
    act = 8 if bits == 8 else hbl.ACT_INT4_BYTES
    Y, acc = hbl.ternary_gemm(
        torch.from_numpy(q.view(np.uint8).copy()).to(DEV), torch.from_numpy(scales).to(DEV),
        torch.from_numpy(rowsum).to(DEV), act, K,
        torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV),
        want_acc=True, path=hbl.PATH_TC_TMA)
    torch.cuda.synchronize()
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc.cpu().numpy(), wacc)
    assert np.array_equal(bf16_bits(Y), wY)


# decode-batch tensor-core kernel: weights as the MMA's A operand in TMEM,
# tokens as B (NT = 16 / 32 / 64 / 128), K split over clusters of 1-8 CTAs and
# reduced through distributed shared memory; ragged N (last 128-row block
# partly filled) and shapes whose plan does not fit (largest K: the fallback)
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 128, 16), (9, 256, 48), (16, 4096, 4096), (17, 4096, 1040),
                                   (32, 16384, 4096), (33, 2048, 272), (64, 16384, 4096),
                                   (65, 8192, 2048), (100, 4096, 11008), (128, 16384, 4096),
                                   (5, 16384, 4096), (128, 32768, 4096)])
def test_gemm_decode_mma(bits, M, K, N):
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M + K + N)
    q = oracle.decode_codes(codes, K, bits)
    act = 8 if bits == 8 else hbl.ACT_INT4_BYTES
    Y, acc = hbl.ternary_gemm(
        torch.from_numpy(q.view(np.uint8).copy()).to(DEV), torch.from_numpy(scales).to(DEV),
        torch.from_numpy(rowsum).to(DEV), act, K,
        torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV),
        want_acc=True, path=hbl.PATH_TC_DECODE)
    torch.cuda.synchronize()
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc.cpu().numpy(), wacc)
    assert np.array_equal(bf16_bits(Y), wY)


# large-batch tensor-core kernel on the packed weights (weights widened into
# TMEM as A, codes as B by TMA): ragged token blocks (M % 256), ragged weight
# blocks (N % 128), several tiles per CTA (more than 148 tiles)
# PATH_TC_PAIR: a 256 x 256 tile per pair of CTAs; M = 300 and N = 272 leave the
# odd CTA's half of the last tile wholly past the end of A / B
@pytest.mark.parametrize("path", ["packed", "pair"])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 128, 16), (45, 256, 272), (256, 512, 128),
                                   (300, 4096, 400), (1000, 2048, 512), (257, 16384, 4096),
                                   (600, 4096, 11008), (1300, 1024, 4096), (300, 128, 272)])
def test_gemm_packed_weights(path, bits, M, K, N):
    if path == "packed" and K < 256:
        pytest.skip("the packed-weight kernel takes K >= 256 (smaller K runs as path 3)")
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M + K + 2 * N)
    q = oracle.decode_codes(codes, K, bits)
    act = 8 if bits == 8 else hbl.ACT_INT4_BYTES
    Y, acc = hbl.ternary_gemm(
        torch.from_numpy(q.view(np.uint8).copy()).to(DEV), torch.from_numpy(scales).to(DEV),
        torch.from_numpy(rowsum).to(DEV), act, K,
        torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV),
        want_acc=True, path=hbl.PATH_TC_PACKED if path == "packed" else hbl.PATH_TC_PAIR)
    torch.cuda.synchronize()
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc.cpu().numpy(), wacc)
    assert np.array_equal(bf16_bits(Y), wY)


@pytest.mark.parametrize("path", [6, 7])
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(520, 4096, 256), (1000, 2048, 528), (300, 16384, 1024)])
def test_forward_packed_weights_path(path, bits, M, K, N):
    # path 6: packed-weight kernel; path 7: the paired-SM kernel
    X = acts(M, K, seed=M + 5 * K, kind="swiglu")
    packed, alpha = oracle.pack_ternary(inputs.latent_weights(N, K, seed=M + N))
    want = oracle.hbitlinear_forward(X, packed, alpha, bits)
    assert np.array_equal(forward(X, packed, alpha, bits, path=path), want)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N,with_gain", [(257, 128, 16, False), (1777, 4096, 2048, True),
                                             (445, 16384, 656, True), (600, 8192, 1200, False)])
def test_forward_widens_weights_beside_the_rows(bits, M, K, N, with_gain):
    # Where the token rows are enough to carry it, the large-batch forward's
    # quantiser (K1) also widens the packed weights for the GEMM: one chunk
    # per row group while the rows are worked on, the rest after them.  These
    # shapes give some groups one row and up to three chunks (so the loop
    # after the rows runs), groups without a row (257 tokens: 9 row groups
    # over 12), a single chunk (N = 16), and the gain variant; every column
    # of Y checks one widened weight row.
    X = acts(M, K, seed=M + K)
    g = (np.random.default_rng(N).uniform(0.25, 2.0, K).astype(np.float32)
         if with_gain else None)
    W = inputs.latent_weights(N, K, seed=N)
    packed, alpha = oracle.pack_ternary(W)
    Y = forward(X, packed, alpha, bits, gain=g)
    rows = np.array([0, 1, M // 2, M - 2, M - 1])
    want = oracle.hbitlinear_forward(X, packed, alpha, bits, gain=g, rows=rows)
    assert np.array_equal(Y[rows], want)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (3, 16384, 4096), (12, 4096, 4096),
                                   (40, 16384, 4096), (128, 4096, 2048)])
def test_forward_decode_mma_path(bits, M, K, N):
    # the whole layer with its GEMM on the decode tensor-core kernel (K1 writes
    # one-byte codes, the kernel follows it as a programmatic dependent)
    X = acts(M, K, seed=M + 3 * K, kind="swiglu")
    packed, alpha = oracle.pack_ternary(inputs.latent_weights(N, K, seed=M + N))
    want = oracle.hbitlinear_forward(X, packed, alpha, bits)
    assert np.array_equal(forward(X, packed, alpha, bits, path=hbl.PATH_TC_DECODE), want)


@pytest.mark.parametrize("K", [16, 256, 4096, 16384])
def test_quant_int4_one_byte_layout(K):
    X = acts(45, K, seed=K + 7, kind="t")
    codes, scales, rowsum = hbl.norm_fwht_quant(to_dev_bf16(X), hbl.ACT_INT4_BYTES)
    torch.cuda.synchronize()
    wc, ws, wr = oracle.norm_fwht_quant(X, 4)
    assert codes.shape == (45, K)
    assert np.array_equal(codes.cpu().numpy().view(np.int8), oracle.decode_codes(wc, K, 4))
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("bits", [4, 8])
def test_gemm_identity_weights(bits):
    K = 256
    codes, scales, rowsum, _, _ = make_gemm_case(130, K, 16, bits)
    pI = oracle.pack_codes(np.eye(K, dtype=np.int8))
    for path in (1, 3):
        Y, acc = run_gemm(codes, scales, rowsum, bits, K, pI, np.float32(1.0), path)
        assert np.array_equal(acc, oracle.decode_codes(codes, K, bits).astype(np.int32))


# ------------------------------------------------------------ whole layer

def forward(X, packed, alpha, bits, path=0, gain=None):
    Y = hbl.hbitlinear_forward(
        to_dev_bf16(X), torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV), bits,
        gain=None if gain is None else torch.from_numpy(gain).to(DEV), path=path)
    torch.cuda.synchronize()
    return bf16_bits(Y)


@pytest.mark.parametrize("bits", [4, 8])
def test_forward_tiny_workload(bits):
    X = inputs.activations("tiny")
    packed, alpha = oracle.pack_ternary(inputs.weights("tiny"))
    for path in (0, 1, 2, 3, 4):
        Y = forward(X, packed, alpha, bits, path)
        assert np.array_equal(Y, oracle.hbitlinear_forward(X, packed, alpha, bits))


@pytest.mark.parametrize("bits", [4, 8])
def test_forward_attn_wo_workload_every_row(bits):
    # 4096 x 2048 -> 2048: weights packed on the GPU against the oracle, then
    # every output element of the forward against the threaded oracle
    X = inputs.activations("attn_wo")
    W = inputs.weights("attn_wo")
    Wd = torch.from_numpy(W).to(DEV)
    p_dev, a_dev = hbl.pack_ternary(Wd)
    packed, alpha = oracle.pack_ternary(W)
    assert np.array_equal(p_dev.cpu().numpy().view(np.uint32), packed)
    assert a_dev.cpu().numpy()[0].view(np.uint32) == np.float32(alpha).view(np.uint32)
    Y = forward(X, packed, alpha, bits)
    want = oracle.hbitlinear_forward(X, packed, alpha, bits)
    assert np.array_equal(Y, want)


@pytest.mark.slow
@pytest.mark.parametrize("bits", [4, 8])
def test_ffn_wdown_workload_every_row(bits):
    # 8192 x 16384 -> 4096 in the launch configuration the benchmark times:
    # codes/scales/rowsum and every output element against the threaded oracle
    # (the TMA-fed GEMM runs 2 tiles per CTA here, alternating its two TMEM
    # accumulators)
    X = inputs.activations("ffn_wdown")
    W = inputs.weights("ffn_wdown")
    packed, alpha = oracle.pack_ternary(W)
    Xd = to_dev_bf16(X)
    codes, scales, rowsum = hbl.norm_fwht_quant(Xd, bits)
    wc, ws, wr = oracle.norm_fwht_quant(X, bits)
    assert np.array_equal(codes.cpu().numpy(), wc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(rowsum.cpu().numpy(), wr)
    del codes, scales, rowsum
    wY, _ = oracle.ternary_gemm(wc, ws, bits, 16384, packed, alpha, want_acc=False)
    Wd = torch.from_numpy(packed.view(np.int32)).to(DEV)
    ad = torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV)
    # the automatic path, and both large-batch tensor-core kernels forced (one
    # SM per tile; pairs of SMs per 256 x 256 tile)
    for path in (hbl.PATH_AUTO, hbl.PATH_TC_TMA, hbl.PATH_TC_PAIR):
        Y = bf16_bits(hbl.hbitlinear_forward(Xd, Wd, ad, bits, path=path))
        bad = np.argwhere(Y != wY)
        assert bad.size == 0, "path %d: outputs differ at %d elements, first %s" % (
            path, len(bad), bad[:5].tolist())


@pytest.mark.parametrize("T", sorted(set(inputs.DECODE_TOKENS) | {5, 9, 16, 64, 100}))
@pytest.mark.parametrize("shape", ["wo", "wdown"])
def test_decode_sweep(T, shape):
    # every row of the decode batches the benchmark times, on the automatic path
    K = 4096 if shape == "wo" else 16384
    N = 4096
    X = inputs.activations("decode_" + shape, M=T, K=K, seed=T)
    W = inputs.latent_weights(N, K, seed=7)
    packed, alpha = oracle.pack_ternary(W)
    Y = forward(X, packed, alpha, 4)
    want = oracle.hbitlinear_forward(X, packed, alpha, 4)
    assert np.array_equal(Y, want)


# one-kernel decode forward (M <= 16384 / K tokens at K = 4096 / 8192 / 16384
# where the CTA's weight rows fit shared memory) against the oracle and
# against the two-kernel forward (GEMM path 2: K1, then the row GEMV).  N (a
# multiple of 16) spans fewer rows than SMs, ragged splits over the SMs and the
# largest split that fits; the other (M, K) pairs take K1 and then the same
# kernel's GEMV half (K = 16384, up to 8 tokens) or the row GEMV.
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("K,N", [(4096, 4096), (4096, 1008), (4096, 16384), (8192, 304),
                                 (8192, 4096), (16384, 112), (16384, 4096)])
@pytest.mark.parametrize("M", [1, 2, 3, 4, 6, 8])
def test_decode_one_kernel_forward(bits, K, N, M):
    X = acts(M, K, seed=M + K, kind="t" if M % 2 else "gauss")
    W = inputs.latent_weights(N, K, seed=N + M)
    packed, alpha = oracle.pack_ternary(W)
    want = oracle.hbitlinear_forward(X, packed, alpha, bits)
    assert np.array_equal(forward(X, packed, alpha, bits), want)
    assert np.array_equal(forward(X, packed, alpha, bits, path=2), want)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K", [(1, 4096), (2, 8192), (4, 4096), (1, 16384)])
def test_decode_one_kernel_forward_with_gain(bits, M, K):
    X = acts(M, K, seed=5)
    g = np.random.default_rng(K).uniform(0.25, 2.0, K).astype(np.float32)
    W = inputs.latent_weights(512, K, seed=9)
    packed, alpha = oracle.pack_ternary(W)
    want = oracle.hbitlinear_forward(X, packed, alpha, bits, gain=g)
    assert np.array_equal(forward(X, packed, alpha, bits, gain=g), want)


def test_decode_one_kernel_edge_rows():
    # zero, constant and single-spike rows (the transform of a spike is flat;
    # of a Hadamard row, a spike) next to a normal row, M = 4
    K, N = 4096, 704
    X = np.zeros((4, K), dtype=np.uint16)
    X[1] = np.float32(0.75).view(np.uint32) >> 16
    X[2, 77] = np.float32(-3.0).view(np.uint32) >> 16
    X[3] = acts(1, K, seed=11)[0]
    W = inputs.latent_weights(N, K, seed=3)
    packed, alpha = oracle.pack_ternary(W)
    for bits in (4, 8):
        assert np.array_equal(forward(X, packed, alpha, bits),
                              oracle.hbitlinear_forward(X, packed, alpha, bits))


@pytest.mark.parametrize("K,N", [(4096, 4096), (8192, 1008), (16384, 4096)])
def test_decode_one_token_edge_rows(K, N):
    # one token through the one-kernel forward: zero, constant, single-spike
    # and a Hadamard-row input (whose transform is a spike), and a normal row,
    # each as its own one-token forward
    W = inputs.latent_weights(N, K, seed=K + 1)
    packed, alpha = oracle.pack_ternary(W)
    rows = np.zeros((5, K), dtype=np.uint16)
    rows[1] = np.float32(0.75).view(np.uint32) >> 16
    rows[2, K // 3] = np.float32(-3.0).view(np.uint32) >> 16
    h = np.array([1.0 - 2.0 * (bin(5 & j).count("1") & 1) for j in range(K)], np.float32)  # row 5 of H_K
    rows[3] = h.view(np.uint32) >> 16
    rows[4] = acts(1, K, seed=K)[0]
    for r in range(5):
        X = rows[r:r + 1].copy()
        for bits in (4, 8):
            assert np.array_equal(forward(X, packed, alpha, bits),
                                  oracle.hbitlinear_forward(X, packed, alpha, bits)), (r, bits)


@pytest.mark.parametrize("T,K", [(1, 4096), (32, 16384), (300, 2048)])
def test_forward_replays_from_cuda_graph(T, K):
    # the forward launches only on the caller's stream, so it can be captured
    X = inputs.activations("decode_wdown", M=T, K=K, seed=3)
    packed, alpha = oracle.pack_ternary(inputs.latent_weights(512, K, seed=2))
    Xd = to_dev_bf16(X)
    Pd = torch.from_numpy(packed.view(np.int32)).to(DEV)
    Ad = torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV)
    ws = torch.empty(max(16, hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD, T, K, 512, 4)),
                     dtype=torch.uint8, device=DEV)
    Y = torch.empty((T, 512), dtype=torch.bfloat16, device=DEV)
    hbl.hbitlinear_forward(Xd, Pd, Ad, 4, ws=ws, out=Y)  # warm-up outside capture
    torch.cuda.synchronize()
    Y.zero_()
    g = torch.cuda.CUDAGraph()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            hbl.hbitlinear_forward(Xd, Pd, Ad, 4, ws=ws, out=Y)
    torch.cuda.current_stream().wait_stream(s)
    g.replay()
    torch.cuda.synchronize()
    rows = np.arange(min(T, 6))
    assert np.array_equal(bf16_bits(Y)[rows],
                          oracle.hbitlinear_forward(X, packed, alpha, 4, rows=rows))


def test_hostio_matches_device_forward():
    X = inputs.activations("tiny")
    packed, alpha = oracle.pack_ternary(inputs.weights("tiny"))
    M, K = X.shape
    N = packed.shape[0]
    ws = torch.empty(hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD_HOSTIO, M, K, N, 4),
                     dtype=torch.uint8, device=DEV)
    Xh = torch.from_numpy(X.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    hbl.hbitlinear_forward_hostio(
        Xh, torch.from_numpy(packed.view(np.int32)).to(DEV),
        torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV), 4, Yh, ws)
    torch.cuda.synchronize()
    assert np.array_equal(Yh.view(torch.int16).numpy().view(np.uint16),
                          oracle.hbitlinear_forward(X, packed, alpha, 4))


@pytest.mark.parametrize("M,bits", [(1000, 4), (2600, 8), (8192, 4)])
def test_hostio_chunked_pipeline(M, bits):
    # batches above 513 tokens run in overlapped row chunks (ragged last chunk);
    # the result must equal the device-buffer forward bit for bit, and work
    # queued on the stream afterwards must see Y on the host
    K, N = 2048, 512
    X = inputs.activations("attn_wo", M=M, K=K, seed=M)
    W = torch.from_numpy(inputs.latent_weights(N, K, seed=M)).to(DEV)
    packed, alpha = hbl.pack_ternary(W)
    ws = torch.empty(hbl.workspace_size(hbl.OP_HBITLINEAR_FORWARD_HOSTIO, M, K, N, bits),
                     dtype=torch.uint8, device=DEV)
    Xh = torch.from_numpy(X.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    Yh = torch.empty((M, N), dtype=torch.bfloat16).pin_memory()
    Yh.fill_(0)
    hbl.hbitlinear_forward_hostio(Xh, packed, alpha, bits, Yh, ws)
    Yd = hbl.hbitlinear_forward(Xh.to(DEV), packed, alpha, bits)
    torch.cuda.synchronize()
    assert torch.equal(Yh.view(torch.int16), Yd.cpu().view(torch.int16))
    rows = np.array([0, 1, M // 2, M - 1])
    want = oracle.hbitlinear_forward(X, packed.cpu().numpy().view(np.uint32),
                                     alpha.cpu().numpy()[0], bits, rows=rows)
    assert np.array_equal(Yh.view(torch.int16).numpy().view(np.uint16)[rows], want)


def test_int8_tensor_probe_runs_and_is_plausible():
    # the dense INT8 tensor-core probe (the GEMM roofline's denominator):
    # finishes within its bounded wait and measures a rate between the GEMM's
    # own measured rate (about 3 POPS) and well above the datasheet figure
    n = torch.cuda.get_device_properties(0).multi_processor_count
    tops, st = hbl.measure_int8_tensor_peak(n, mmas_per_cta=1 << 13, reps=3)
    assert st == 0
    assert 1000.0 < tops < 6000.0


def test_status_word_stays_clear():
    st = hbl.new_status(DEV)
    X = to_dev_bf16(acts(200, 2048, seed=1))
    packed, alpha = hbl.pack_ternary(torch.from_numpy(inputs.latent_weights(256, 2048)).to(DEV))
    hbl.hbitlinear_forward(X, packed, alpha, 4, status=st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == 0


@pytest.mark.parametrize("arrive", [True, False])
def test_bounded_wait_reports_timeout_and_context_survives(arrive):
    # a wait that nothing satisfies runs out and reports HBL_ERR_TIMEOUT (7);
    # the context stays usable for the next launch
    st = hbl.new_status(DEV)
    hbl.selftest_bounded_wait(arrive, 2000, st)
    torch.cuda.synchronize()
    assert int(st[0].item()) == (0 if arrive else 7)
    X = to_dev_bf16(acts(3, 256, seed=1))
    codes, scales, rowsum = hbl.norm_fwht_quant(X, 4)
    torch.cuda.synchronize()
    wc, _, _ = oracle.norm_fwht_quant(acts(3, 256, seed=1), 4)
    assert np.array_equal(codes.cpu().numpy(), wc)


@pytest.mark.parametrize("N,K", [(16, 256), (272, 2048), (4096, 16384)])
def test_expand_ternary_matches_unpacked_codes(N, K):
    W = inputs.latent_weights(N, K, seed=N)
    packed, _ = oracle.pack_ternary(W)
    Ws = hbl.expand_ternary(torch.from_numpy(packed.view(np.int32)).to(DEV), K)
    torch.cuda.synchronize()
    assert np.array_equal(Ws.cpu().numpy(), oracle.unpack_codes(packed, K))


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 128, 16), (300, 4096, 400), (1030, 2048, 512)])
def test_gemm_on_kept_expanded_weights(bits, M, K, N):
    codes, scales, rowsum, packed, alpha = make_gemm_case(M, K, N, bits, seed=M + 3)
    q = oracle.decode_codes(codes, K, bits)
    Ws = hbl.expand_ternary(torch.from_numpy(packed.view(np.int32)).to(DEV), K)
    act = 8 if bits == 8 else hbl.ACT_INT4_BYTES
    Y, acc = hbl.ternary_gemm_s8w(
        torch.from_numpy(q.view(np.uint8).copy()).to(DEV), torch.from_numpy(scales).to(DEV), act,
        Ws, torch.from_numpy(np.array([alpha, 0, 0, 0], dtype=np.float32)).to(DEV),
        want_acc=True)
    torch.cuda.synchronize()
    wY, wacc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc.cpu().numpy(), wacc)
    assert np.array_equal(bf16_bits(Y), wY)


@pytest.mark.parametrize("M", [1, 3, 300])
def test_forward_at_the_largest_K(M):
    # K = 32768 (the largest transform): row GEMV (1 token), tensor-core kernel
    # with activations in TMEM (3), TMA-fed GEMM (300); sampled rows vs the oracle
    K, N = 32768, 256
    X = inputs.student_t_acts(M, K, seed=M)
    W = inputs.latent_weights(N, K, seed=M)
    packed, alpha = oracle.pack_ternary(W)
    Y = forward(X, packed, alpha, 4)
    rows = np.arange(M) if M <= 3 else np.array([0, 1, 150, M - 1])
    assert np.array_equal(Y[rows], oracle.hbitlinear_forward(X, packed, alpha, 4, rows=rows))
