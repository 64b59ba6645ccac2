"""Pins for the oracle's variant functions: LayerNorm and no-Hadamard BitLinear,
offline weight rotation (plain and randomised Hadamard), and the per-head
QKV / KV-cache quantiser.  Each check fixes the oracle against something other
than itself: closed forms, exact-arithmetic cases, library routines in fp64,
brute force with exact rationals, or Python big-integer bit strings.  CPU only.

Sources: BitNet v2 write-up (0755model.com), sections "H-BitLinear" (the layer
written as LN, transform, quantise, matmul), "实验结果" (Q, K, V states after
RoPE quantised per head by absmax to unsigned integers; 3-bit KV cache) and the
Hadamard ablation of table 5 (weights and activations, or activations only);
QuaRot's randomised Hadamard transform as described in the same write-up.
"""
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle


def _bf16_bits(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(
        torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def _rows(M, K, seed, scale=1.0):
    rng = np.random.default_rng(seed)
    return _bf16_bits(rng.standard_normal((M, K)) * scale)


# ------------------------------------------------------------------ LayerNorm

@pytest.mark.parametrize("K", [16, 256, 4096])
@pytest.mark.parametrize("a,b", [(3.0, 2.0), (-5.0, 1.0), (0.0, 7.0)])
def test_layernorm_balanced_row_closed_form(K, a, b):
    # x = a + b*s with s a balanced +-1 pattern: every partial sum is an exact
    # integer, so mu = a, d = b*s and var = b^2 exactly, and u = s*b/sqrt(b^2+eps).
    s = np.where(np.random.default_rng(K).permutation(K) < K // 2, 1.0, -1.0)
    x = _bf16_bits((a + b * s)[None, :])
    eps = 1e-6
    u = oracle.norm_transform(x, norm_eps=eps, layernorm=True, hadamard=False)[0]
    want = s * (b / np.sqrt(b * b + eps))
    assert np.allclose(u, want, rtol=3e-7, atol=0)


@pytest.mark.parametrize("K", [64, 256])
def test_layernorm_shift_invariance_on_exact_rows(K):
    # small integer rows: the mean is a dyadic rational and x - mu is exact, so
    # LN(x + c) is bit-identical to LN(x) (RMSNorm is not shift invariant)
    rng = np.random.default_rng(1)
    x = rng.integers(-100, 100, size=(4, K)).astype(np.float32)
    for c in (1.0, -37.0, 100.0):
        u0 = oracle.norm_transform(_bf16_bits(x), layernorm=True, hadamard=False)
        u1 = oracle.norm_transform(_bf16_bits(x + c), layernorm=True, hadamard=False)
        assert np.array_equal(u0, u1)
        r0 = oracle.norm_transform(_bf16_bits(x), layernorm=False, hadamard=False)
        r1 = oracle.norm_transform(_bf16_bits(x + c), layernorm=False, hadamard=False)
        assert not np.array_equal(r0, r1)


@pytest.mark.parametrize("K", [16, 512, 4096])
@pytest.mark.parametrize("with_gain", [False, True])
def test_layernorm_matches_torch_fp64(K, with_gain):
    X = _rows(6, K, seed=K, scale=3.0)
    g = (np.random.default_rng(7).uniform(0.5, 1.5, K).astype(np.float32)
         if with_gain else None)
    u = oracle.norm_transform(X, gain=g, norm_eps=1e-6, layernorm=True, hadamard=False)
    xf = torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64))
    w = None if g is None else torch.from_numpy(g.astype(np.float64))
    ref = torch.nn.functional.layer_norm(xf, (K,), weight=w, eps=1e-6).numpy()
    assert np.max(np.abs(u - ref)) <= 2e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("K", [16, 1024])
def test_rmsnorm_without_transform_matches_torch_fp64(K):
    X = _rows(5, K, seed=3, scale=2.0)
    u = oracle.norm_transform(X, layernorm=False, hadamard=False)
    xf = torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64))
    ref = torch.nn.functional.rms_norm(xf, (K,), eps=1e-6).numpy()
    assert np.max(np.abs(u - ref)) <= 1e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("K", [64, 2048])
def test_layernorm_then_hadamard_matches_fp64_dense(K):
    X = _rows(3, K, seed=11, scale=4.0)
    v = oracle.norm_transform(X, layernorm=True, hadamard=True)
    xf = torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64))
    ln = torch.nn.functional.layer_norm(xf, (K,), eps=1e-6).numpy()
    ref = ln @ scipy.linalg.hadamard(K).astype(np.float64) / np.sqrt(K)
    assert np.max(np.abs(v - ref)) <= 2e-6 * np.max(np.abs(ref))


def test_default_variant_is_the_h_bitlinear_path():
    X = _rows(4, 256, seed=5)
    assert np.array_equal(oracle.norm_transform(X), oracle.norm_fwht(X))
    for bits in (4, 8):
        a = oracle.norm_quant(X, bits)
        b = oracle.norm_fwht_quant(X, bits)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


@pytest.mark.parametrize("layernorm", [False, True])
@pytest.mark.parametrize("hadamard", [False, True])
@pytest.mark.parametrize("bits", [4, 8])
def test_variant_codes_match_fp64_evaluation_away_from_ties(layernorm, hadamard, bits):
    K = 512
    X = _rows(8, K, seed=21, scale=2.0)
    codes, scales, rowsum = oracle.norm_quant(X, bits, layernorm=layernorm, hadamard=hadamard)
    q = oracle.decode_codes(codes, K, bits).astype(np.int64)
    xf = torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64))
    if layernorm:
        u = torch.nn.functional.layer_norm(xf, (K,), eps=1e-6).numpy()
    else:
        u = torch.nn.functional.rms_norm(xf, (K,), eps=1e-6).numpy()
    v = u @ scipy.linalg.hadamard(K).astype(np.float64) / np.sqrt(K) if hadamard else u
    if bits == 8:
        stat = np.max(np.abs(v), axis=1, keepdims=True)
        y = v * (127.0 / (stat + 1e-5))
        lo, hi = -128, 127
        sc = stat[:, 0] / 127.0
    else:
        stat = np.mean(np.abs(v), axis=1, keepdims=True)
        y = v * (np.sqrt(7.0) / (stat + 1e-5))
        lo, hi = -8, 7
        sc = stat[:, 0] / np.sqrt(7.0)
    frac = np.abs(y - np.floor(y) - 0.5)
    clear = frac > 1e-3  # not within reach of a rounding tie
    assert clear.mean() > 0.99
    want = np.clip(np.rint(y), lo, hi).astype(np.int64)
    assert np.array_equal(q[clear], want[clear])
    assert np.allclose(scales, sc, rtol=1e-5)
    assert np.array_equal(rowsum, q.sum(axis=1))


# ------------------------------------------------------------ weight rotation

@pytest.mark.parametrize("K", [16, 256, 2048])
@pytest.mark.parametrize("signed", [False, True])
def test_rotate_weights_matches_dense_fp64(K, signed):
    rng = np.random.default_rng(K)
    W = (rng.standard_normal((8, K)) * 0.02).astype(np.float32)
    s = rng.choice([-1.0, 1.0], K).astype(np.float32) if signed else None
    Wr = oracle.rotate_weights(W, s)
    D = np.ones(K) if s is None else s.astype(np.float64)
    ref = (W.astype(np.float64) * D) @ scipy.linalg.hadamard(K).astype(np.float64) / np.sqrt(K)
    assert np.max(np.abs(Wr - ref)) <= 1e-6 * np.max(np.abs(ref))


@pytest.mark.parametrize("K", [64, 1024])
def test_rotation_preserves_inner_products_with_rotated_activations(K):
    # (x D H/sqrt K) . (w D H/sqrt K) = x . w: the activation side takes the signs
    # as its per-channel gain, the weight side through rotate_weights
    rng = np.random.default_rng(2)
    X = _rows(6, K, seed=4)
    W = (rng.standard_normal((10, K)) * 0.02).astype(np.float32)
    s = rng.choice([-1.0, 1.0], K).astype(np.float32)
    v = oracle.norm_transform(X, gain=s).astype(np.float64)
    wr = oracle.rotate_weights(W, s).astype(np.float64)
    u = oracle.norm_transform(X, hadamard=False).astype(np.float64)
    lhs, rhs = v @ wr.T, u @ W.astype(np.float64).T
    assert np.max(np.abs(lhs - rhs)) <= 1e-5 * np.max(np.abs(rhs))


def test_rotation_is_an_involution_up_to_the_signs():
    K = 512
    rng = np.random.default_rng(8)
    W = rng.standard_normal((4, K)).astype(np.float32)
    s = rng.choice([-1.0, 1.0], K).astype(np.float32)
    back = oracle.rotate_weights(oracle.rotate_weights(W, s))  # W D H H / K = W D
    assert np.max(np.abs(back * s - W)) <= 1e-5 * np.max(np.abs(W))


# --------------------------------------------------------- QKV / KV quantiser

def _kv_brute(xrow, bits, eps):
    """Exact-rational evaluation: gamma, inv as fp32 (one IEEE division), then
    the exact product rounded half to even, clipped, offset by 2^(b-1)."""
    qp = 2 ** (bits - 1) - 1
    xs = oracle.bf16_to_f32(xrow).astype(np.float32)
    g = np.float32(np.max(np.abs(xs)))
    inv = np.float32(np.float32(qp) / np.float32(g + np.float32(eps)))
    out = []
    for x in xs:
        y = Fraction(float(x)) * Fraction(float(inv))
        fl = y.numerator // y.denominator
        rem = y - fl
        if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
            fl += 1
        q = max(-qp - 1, min(qp, fl))
        out.append(q + 2 ** (bits - 1))
    return np.array(out, dtype=np.int64), np.float32(g / np.float32(qp))


def _pack_bigint(u, bits):
    out = bytearray()
    for g0 in range(0, len(u), 32):
        val = 0
        for j, c in enumerate(u[g0:g0 + 32]):
            val |= int(c) << (bits * j)
        out += val.to_bytes(4 * bits, "little")
    return np.frombuffer(bytes(out), dtype=np.uint8)


@pytest.mark.parametrize("bits", [2, 3, 4, 8])
@pytest.mark.parametrize("D", [32, 128])
def test_kv_quant_brute_force_and_packing(bits, D):
    X = _rows(12, D, seed=bits * 100 + D, scale=1.5)
    codes, scales = oracle.kv_quant(X, bits)
    assert codes.shape == (12, D * bits // 8)
    for r in range(X.shape[0]):
        u, sc = _kv_brute(X[r], bits, 1e-5)
        assert np.array_equal(oracle.kv_unpack(codes[r:r + 1], D, bits)[0].astype(np.int64), u)
        assert np.array_equal(codes[r], _pack_bigint(u, bits))
        assert scales[r] == sc


def test_kv_quant_hand_ties_3bit():
    # gamma = 3 and eps = 0 make inv = 3/3 = 1 exactly, so x * inv = x:
    # 2.5 -> 2, 1.5 -> 2, 0.5 -> 0, -0.5 -> -0, -2.5 -> -2 (ties to even),
    # 3 -> 3, -3 -> -3; stored with the offset 4.
    vals = [2.5, 1.5, 0.5, -0.5, -2.5, 3.0, -3.0, 0.0]
    x = np.array(vals * 4, dtype=np.float32)[None, :]
    codes, scales = oracle.kv_quant(_bf16_bits(x), 3, eps=0.0)
    u = oracle.kv_unpack(codes, 32, 3)[0]
    assert list(u[:8]) == [6, 6, 4, 4, 2, 7, 1, 4]
    assert scales[0] == np.float32(1.0)


@pytest.mark.parametrize("bits", [3, 4, 8])
def test_kv_quant_extremes_zero_row_and_error_bound(bits):
    D = 128
    X = _rows(16, D, seed=bits, scale=2.0)
    X[3] = 0
    codes, scales = oracle.kv_quant(X, bits)
    u = oracle.kv_unpack(codes, D, bits).astype(np.int64)
    off = 2 ** (bits - 1)
    xf = oracle.bf16_to_f32(X).astype(np.float64)
    assert np.all(u[3] == off) and scales[3] == 0
    for r in range(16):
        if r == 3:
            continue
        k = int(np.argmax(np.abs(xf[r])))
        assert u[r, k] == (2 * off - 1 if xf[r, k] > 0 else 1)
        assert u[r].min() >= 1 and u[r].max() <= 2 * off - 1
        # x - q*s = ((y - q)*gamma + y*eps)/Qp with |y - q| <= 1/2, |y| <= Qp
        err = np.abs(xf[r] - (u[r] - off) * np.float64(scales[r]))
        assert np.all(err <= 0.5 * np.float64(scales[r]) + 1e-5 + 1e-6 * np.abs(xf[r]))
