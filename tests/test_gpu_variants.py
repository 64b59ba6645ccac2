"""GPU parity for the layer variants and the neighbouring kernels, through the
C ABI, against the CPU oracle on the same seeded inputs:

  - BitLinear without the Hadamard transform and the LayerNorm normalisation
    (hbl_norm_transform / hbl_norm_quant / hbl_bitlinear_forward with flags):
    fp32 values, codes, scales and rowsum bit-identical; Y within 1 bf16 ulp;
  - offline weight rotation (hbl_rotate_weights), plain and with random signs,
    in place and out of place: fp32 bit-identical;
  - the per-head unsigned absmax QKV / KV-cache quantiser (hbl_kv_quant):
    packed codes and scales bit-identical.

Sources: BitNet v2 write-up (0755model.com), sections "H-BitLinear" (the layer
as LN, transform, quantise, matmul), "实验结果" (QKV states after RoPE quantised
per head by absmax to unsigned integers) and the Hadamard ablation (table 5).
"""
import numpy as np
import pytest
import torch

import hadamard_rotated_int4_b200 as hbl
import oracle
from hadamard_rotated_int4_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
FLAGS = [0, hbl.NORM_NO_HADAMARD, hbl.NORM_LAYERNORM, hbl.NORM_LAYERNORM | hbl.NORM_NO_HADAMARD]


def to_dev_bf16(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16).copy()).view(
        torch.bfloat16).to(DEV)


def bf16_bits(t):
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def okw(flags):
    return dict(layernorm=bool(flags & hbl.NORM_LAYERNORM),
                hadamard=not (flags & hbl.NORM_NO_HADAMARD))


def il_decode(buf, M, K):
    Mp = (M + 31) // 32 * 32
    b = np.asarray(buf, dtype=np.uint8).reshape(Mp // 32, K // 16, 32, 16)
    return b.transpose(0, 2, 1, 3).reshape(Mp, K)[:M].view(np.int8)


# ------------------------------------------------------- BitLinear variants

@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("K", [16, 128, 256, 2048, 4096, 8192, 16384, 32768])
def test_variant_values(flags, K):
    M = 37
    X = inputs.student_t_acts(M, K, seed=K + flags)
    V = hbl.norm_transform(to_dev_bf16(X), flags).cpu().numpy()
    want = oracle.norm_transform(X, **okw(flags))
    assert np.array_equal(V.view(np.uint32), want.view(np.uint32))


@pytest.mark.parametrize("flags", FLAGS[1:])
@pytest.mark.parametrize("bits", [4, 8, hbl.ACT_INT4_I32, hbl.ACT_INT8_I32])
@pytest.mark.parametrize("K", [16, 64, 256, 1024, 4096, 16384])
def test_variant_codes(flags, bits, K):
    M = 45  # ragged against every rows-per-group size
    X = inputs.swiglu_acts(M, K, seed=K + 3 * flags)
    g = np.random.default_rng(K).uniform(0.5, 1.5, K).astype(np.float32) if K == 1024 else None
    codes, scales, rowsum = hbl.norm_quant(to_dev_bf16(X), bits, flags,
                                           gain=None if g is None else torch.from_numpy(g).to(DEV))
    torch.cuda.synchronize()
    base = bits & 0xFF
    wc, ws, wr = oracle.norm_quant(X, base, gain=g, **okw(flags))
    if bits in (hbl.ACT_INT4_I32, hbl.ACT_INT8_I32):
        assert np.array_equal(il_decode(codes.cpu().numpy(), M, K),
                              oracle.decode_codes(wc, K, base))
    else:
        assert np.array_equal(codes.cpu().numpy(), wc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
    assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("flags", FLAGS[1:])
@pytest.mark.parametrize("bits", [4, 8])
def test_variant_edge_rows_and_zero_eps(flags, bits):
    K = 4096
    X = inputs.gaussian_acts(6, K, seed=2)
    X[0] = 0                          # zero row (with quant_eps = 0 below too)
    X[1] = np.uint16(0x3F80)          # constant row: LayerNorm gives d = 0
    X[2, :] = 0
    X[2, 17] = np.uint16(0x4120)      # single spike
    for qe in (1e-5, 0.0):
        codes, scales, rowsum = hbl.norm_quant(to_dev_bf16(X), bits, flags, quant_eps=qe)
        torch.cuda.synchronize()
        wc, ws, wr = oracle.norm_quant(X, bits, quant_eps=qe, **okw(flags))
        assert np.array_equal(codes.cpu().numpy(), wc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
        assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("K", [16, 4096, 16384])
def test_variant_values_with_underflowing_squares(flags, K):
    # the squares of d = x (- mean) are rounded to fp32 before the tree sum:
    # rows whose squares are subnormal decide that reading
    rng = np.random.default_rng(K + flags)
    X = np.empty((4, K), dtype=np.uint16)
    X[0] = np.tile(np.array([0x1A00, 0x1A40], np.uint16), K // 2)
    X[1] = X[0]
    X[1, K // 2:] |= 0x8000
    for r, sc in ((2, 1e-20), (3, 1e-22)):
        v = torch.from_numpy((rng.standard_normal(K) * sc).astype(np.float32))
        X[r] = v.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    eps = float(2.0 ** -149)
    V = hbl.norm_transform(to_dev_bf16(X), flags, norm_eps=eps).cpu().numpy()
    want = oracle.norm_transform(X, norm_eps=eps, **okw(flags))
    assert np.array_equal(V.view(np.uint32), want.view(np.uint32))
    for bits in (4, 8):
        codes, scales, rowsum = hbl.norm_quant(to_dev_bf16(X), bits, flags, norm_eps=eps)
        wc, ws, wr = oracle.norm_quant(X, bits, norm_eps=eps, **okw(flags))
        assert np.array_equal(codes.cpu().numpy(), wc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))
        assert np.array_equal(rowsum.cpu().numpy(), wr)


@pytest.mark.parametrize("flags", FLAGS)
@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 4096, 4096), (8, 256, 128), (45, 2048, 272),
                                   (300, 4096, 256)])
def test_bitlinear_forward_variants(flags, bits, M, K, N):
    X = inputs.gaussian_acts(M, K, seed=M + K)
    W = inputs.latent_weights(N, K, seed=N)
    packed, alpha = oracle.pack_ternary(W)
    Y = hbl.bitlinear_forward(to_dev_bf16(X), torch.from_numpy(packed.view(np.int32)).to(DEV),
                              torch.from_numpy(np.array([alpha, 0, 0, 0], np.float32)).to(DEV),
                              bits, flags)
    torch.cuda.synchronize()
    want = oracle.bitlinear_forward(X, packed, alpha, bits, **okw(flags))
    assert np.array_equal(bf16_bits(Y), want)


def test_bitlinear_forward_flag_zero_is_h_bitlinear():
    X = to_dev_bf16(inputs.gaussian_acts(64, 2048, seed=4))
    W = torch.from_numpy(inputs.latent_weights(256, 2048, seed=4)).to(DEV)
    packed, alpha = hbl.pack_ternary(W)
    for bits in (4, 8):
        a = hbl.bitlinear_forward(X, packed, alpha, bits, 0)
        b = hbl.hbitlinear_forward(X, packed, alpha, bits)
        assert torch.equal(a, b)


def test_bad_flags_rejected():
    X = torch.zeros((4, 256), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(hbl.HblError) as e:
        hbl.norm_transform(X, 4)
    assert e.value.status == 1


# ------------------------------------------------------------ weight rotation

@pytest.mark.parametrize("K", [16, 32, 128, 1024, 2048, 4096, 16384, 32768])
@pytest.mark.parametrize("signed", [False, True])
def test_rotate_weights(K, signed):
    N = 70
    W = inputs.latent_weights(N, K, seed=K)
    s = inputs.random_signs(K, seed=K) if signed else None
    Wr = hbl.rotate_weights(torch.from_numpy(W).to(DEV),
                            None if s is None else torch.from_numpy(s).to(DEV))
    torch.cuda.synchronize()
    want = oracle.rotate_weights(W, s)
    assert np.array_equal(Wr.cpu().numpy().view(np.uint32), want.view(np.uint32))


def test_rotate_weights_in_place_then_pack():
    N, K = 512, 4096
    W = inputs.latent_weights(N, K, seed=1)
    s = inputs.random_signs(K, seed=1)
    Wd = torch.from_numpy(W).to(DEV)
    hbl.rotate_weights(Wd, torch.from_numpy(s).to(DEV), out=Wd)
    packed, alpha = hbl.pack_ternary(Wd)
    torch.cuda.synchronize()
    Wr = oracle.rotate_weights(W, s)
    assert np.array_equal(Wd.cpu().numpy().view(np.uint32), Wr.view(np.uint32))
    wp, wa = oracle.pack_ternary(Wr)
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), wp)
    assert alpha.cpu().numpy()[0].view(np.uint32) == np.float32(wa).view(np.uint32)


def test_randomised_hadamard_layer_end_to_end():
    # rotated weights (signs s) with activations whose gain carries the same s
    M, K, N = 33, 2048, 256
    X = inputs.gaussian_acts(M, K, seed=6)
    W = inputs.latent_weights(N, K, seed=6)
    s = inputs.random_signs(K, seed=6)
    sd = torch.from_numpy(s).to(DEV)
    Wr = hbl.rotate_weights(torch.from_numpy(W).to(DEV), sd)
    packed, alpha = hbl.pack_ternary(Wr)
    Y = hbl.hbitlinear_forward(to_dev_bf16(X), packed, alpha, 4, gain=sd)
    torch.cuda.synchronize()
    wp, wa = oracle.pack_ternary(oracle.rotate_weights(W, s))
    want = oracle.hbitlinear_forward(X, wp, wa, 4, gain=s)
    assert np.array_equal(bf16_bits(Y), want)


# ------------------------------------------------------- QKV / KV quantiser

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("D", [32, 64, 128, 256])
def test_kv_quant(bits, D):
    X = inputs.qkv_states(T=37, H=5, D=D, seed=bits + D)  # 185 rows: ragged warp steps
    codes, scales = hbl.kv_quant(to_dev_bf16(X), bits)
    torch.cuda.synchronize()
    wc, ws = oracle.kv_quant(X, bits)
    assert np.array_equal(codes.cpu().numpy(), wc)
    assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))


@pytest.mark.parametrize("bits", [3, 4])
def test_kv_quant_edge_rows_and_zero_eps(bits):
    X = inputs.qkv_states(T=4, H=4, D=128, seed=3).reshape(16, 128)
    X[0] = 0                          # zero head
    X[1] = np.uint16(0x3F80)          # constant
    X[2, :] = 0
    X[2, 5] = np.uint16(0xC120)       # single negative spike
    X[3, ::2] = np.uint16(0x7F00)     # very large values
    for eps in (1e-5, 0.0):
        codes, scales = hbl.kv_quant(to_dev_bf16(X), bits, eps=eps)
        torch.cuda.synchronize()
        wc, ws = oracle.kv_quant(X, bits, eps=eps)
        assert np.array_equal(codes.cpu().numpy(), wc)
        assert np.array_equal(scales.cpu().numpy().view(np.uint32), ws.view(np.uint32))


def test_kv_quant_full_workload_sampled():
    X = inputs.qkv_states(seed=0)  # 8192 x 96 x 128
    Xd = to_dev_bf16(X)
    rows = np.random.default_rng(0).choice(X.shape[0] * X.shape[1], 4096, replace=False)
    flat = X.reshape(-1, X.shape[-1])
    for bits in (3, 4):
        codes, scales = hbl.kv_quant(Xd, bits)
        torch.cuda.synchronize()
        wc, ws = oracle.kv_quant(flat[rows], bits)
        assert np.array_equal(codes.cpu().numpy()[rows], wc)
        assert np.array_equal(scales.cpu().numpy()[rows].view(np.uint32), ws.view(np.uint32))


def test_kv_quant_empty():
    codes, scales = hbl.kv_quant(torch.zeros((0, 128), dtype=torch.bfloat16, device=DEV), 3)
    assert codes.numel() == 0 and scales.numel() == 0
