"""Pins for the CPU oracle: each check fixes the oracle against something other
than itself (closed forms, library routines, hand-derived cases, brute force,
invariants).  CPU only.

Sources: BitNet v2 write-up (0755model.com), sections "BitNet v2：原生4位激活"
and "H-BitLinear"; BitNet v2 explainer (shengxinai.com) section 2.2; the
"[论文品鉴] 1-bit LLM" post, sections "掩码存储" and "量化函数".
"""
import json
import os
from fractions import Fraction

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from hadamard_rotated_int4_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_cases.json")


def _golden():
    with open(GOLDEN) as f:
        return json.load(f)


def _pow2expr(s):
    """Parse the small expressions used in the golden file into binary32."""
    s = s.replace(" ", "")
    table = {
        "1": 1.0, "-1": -1.0, "2": 2.0, "2^-24": 2.0 ** -24, "-2^-24": -(2.0 ** -24),
        "1+2^-23": 1.0 + 2.0 ** -23, "1+2^-22": 1.0 + 2.0 ** -22,
    }
    return np.float32(table[s])


# ------------------------------------------------------------------ Hadamard

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_sylvester_closed_form_and_orthogonality(n):
    H = oracle.sylvester(n).astype(np.int64)
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    popc = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    assert np.array_equal(H, np.where(popc % 2 == 0, 1, -1))
    assert np.array_equal(H @ H.T, n * np.eye(n, dtype=np.int64))
    assert np.array_equal(H, scipy.linalg.hadamard(n))


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_fwht_equals_dense_product_on_integers(n):
    rng = np.random.default_rng(n)
    u = rng.integers(-1000, 1000, size=(5, n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    want = u.astype(np.float64) @ H  # integer sums, exact in fp32 and fp64
    assert np.array_equal(oracle.fwht_f32(u), want.astype(np.float32))
    assert np.array_equal(oracle.fwht_f64(u), want)


@pytest.mark.parametrize("n", [16, 64])
def test_fwht_random_close_to_dense(n):
    rng = np.random.default_rng(7)
    u = rng.standard_normal((4, n)).astype(np.float32)
    H = scipy.linalg.hadamard(n).astype(np.float64)
    want = u.astype(np.float64) @ H
    got = oracle.fwht_f32(u).astype(np.float64)
    assert np.max(np.abs(got - want) / np.abs(want).max(axis=1, keepdims=True)) < 1e-6
    assert np.allclose(oracle.fwht_f64(u), want, rtol=0, atol=1e-12)


@pytest.mark.parametrize("n", [8, 256, 4096])
def test_fwht_involution_parseval_special_cases(n):
    rng = np.random.default_rng(3)
    u = rng.standard_normal(n)
    v = oracle.fwht_f64(u)
    assert np.allclose(oracle.fwht_f64(v) / n, u, atol=1e-12)
    assert np.isclose(np.sum(v * v) / n, np.sum(u * u), rtol=1e-12)
    for j in (0, 1, n // 2 + 1, n - 1):
        d = np.zeros(n)
        d[j] = 1.0
        row = oracle.fwht_f64(d)
        i = np.arange(n)
        sign = np.array([1 if bin(int(x & j)).count("1") % 2 == 0 else -1 for x in i])
        assert np.array_equal(row, sign.astype(np.float64))
    ones = oracle.fwht_f64(np.ones(n))
    e0 = np.zeros(n)
    e0[0] = n
    assert np.array_equal(ones, e0)


def test_fwht_stage_order_hand_case():
    g = _golden()["fwht_stage_order"]
    u = np.array([_pow2expr(s) for s in g["input"]], dtype=np.float32)
    want = np.array([_pow2expr(s) for s in g["expected_unnormalised"]], dtype=np.float32)
    assert np.array_equal(oracle.fwht_f32(u), want)


def test_inv_sqrt_n_and_sqrt7_are_correctly_rounded():
    # Compare against exact rational arithmetic: the binary32 value nearest
    # to the real constant has the smallest |c^2 * n - 1| among its neighbours.
    def nearest(val_sq_target, c):
        c = np.float32(c)
        cands = [np.nextafter(c, np.float32(-np.inf)), c, np.nextafter(c, np.float32(np.inf))]
        errs = [abs(Fraction(float(x)) ** 2 - val_sq_target) for x in cands]
        return cands[int(np.argmin(errs))] == c

    for n in [16, 32, 256, 2048, 4096, 8192, 16384, 32768]:
        c = oracle.inv_sqrt_n(n)
        assert nearest(Fraction(1, n), c)
        if (n.bit_length() - 1) % 2 == 0:
            assert float(c) == 2.0 ** (-(n.bit_length() - 1) / 2)
    assert nearest(Fraction(7), oracle.sqrt7())
    assert oracle.sqrt7() == np.sqrt(np.float32(7.0))


# ------------------------------------------------------------------ tree sum

def test_tree_sum_hand_cases():
    for case in _golden()["tree_sum"]["cases"]:
        v = np.array([_pow2expr(s) for s in case["input"]], dtype=np.float32)
        assert oracle.tree_sum(v) == _pow2expr(case["expected"])


def test_tree_sum_exact_on_integers():
    rng = np.random.default_rng(11)
    for m in [1, 2, 3, 5, 7, 100, 1000, 4096]:
        v = rng.integers(-1000, 1000, size=m).astype(np.float32)
        assert oracle.tree_sum(v) == float(v.astype(np.int64).sum())


# ------------------------------------------------------------------ bf16

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(5)
    bits = rng.integers(0, 2 ** 32, size=20000, dtype=np.uint64).astype(np.uint32)
    special = np.array([0x00000000, 0x80000000, 0x3f808000, 0x3f818000, 0x3f80ffff, 0x7f7fffff,
                        0x7f800000, 0xff800000, 0x00000001, 0x007fffff, 0x3f7fffff],
                       dtype=np.uint32)
    x = np.concatenate([bits, special]).view(np.float32)
    x = x[~np.isnan(x)]
    want = torch.from_numpy(x.copy()).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(oracle.f32_to_bf16(x), want)
    back = oracle.bf16_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(want.view(np.int16).copy()).view(
        torch.bfloat16).float().numpy())


# ------------------------------------------------------------------ RMSNorm

@pytest.mark.parametrize("c", [1e-3, 0.5, 3.0, -7.25])
def test_rmsnorm_constant_row_closed_form(c):
    K = 256
    cb = np.float32(torch.tensor(c, dtype=torch.float32).to(torch.bfloat16).float().item())
    bits = np.full((1, K), torch.tensor(c).to(torch.bfloat16).view(torch.int16).item(),
                   dtype=np.int16).view(np.uint16)
    u = oracle.rmsnorm(bits, norm_eps=1e-6)
    want = float(cb) / np.sqrt(float(cb) ** 2 + 1e-6)
    assert np.allclose(u, want, rtol=3e-7, atol=0)
    g = np.linspace(0.5, 2.0, K).astype(np.float32)
    ug = oracle.rmsnorm(bits, gain=g, norm_eps=1e-6)
    assert np.allclose(ug, want * g.astype(np.float64), rtol=5e-7, atol=0)


def test_rmsnorm_matches_torch_fp64():
    X = inputs.activations("tiny")
    x64 = torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64))
    want = torch.nn.functional.rms_norm(x64, (x64.shape[1],), eps=1e-6).numpy()
    got = oracle.rmsnorm(X, norm_eps=1e-6)
    assert np.max(np.abs(got - want) / np.abs(want).max(axis=1, keepdims=True)) < 1e-6


def _f32_nearest(q):
    """The binary32 value nearest to the positive rational q (ties to even) for a
    q in the normal range, derived exactly (no floating-point arithmetic)."""
    q = Fraction(q)
    assert q > 0
    e = 0
    while q >= 2:
        q /= 2
        e += 1
    while q < 1:
        q *= 2
        e -= 1
    assert -126 <= e <= 127
    m = q * 2 ** 23
    n = m.numerator // m.denominator
    rem = m - n
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and n % 2 == 1):
        n += 1
    return Fraction(n, 2 ** 23) * Fraction(2) ** e


def _f32_sqrt_nearest(q):
    """Nearest binary32 to sqrt(q) for a positive rational q with a normal root."""
    q = Fraction(q)
    e = 0
    while q >= 4:
        q /= 4
        e += 1
    while q < 1:
        q *= 4
        e -= 1
    # sqrt(q) in [1, 2): candidates n / 2^23; pick by comparing squares exactly
    target = q * 2 ** 46
    n = int(target.numerator // target.denominator)
    lo = int(np.floor(np.sqrt(float(n))))
    while (lo + 1) ** 2 <= target:
        lo += 1
    while lo ** 2 > target:
        lo -= 1
    mid = Fraction(2 * lo + 1, 2)
    if mid * mid < target or (mid * mid == target and lo % 2 == 1):
        lo += 1
    return Fraction(lo, 2 ** 23) * Fraction(2) ** e


def test_sum_of_squares_rounds_every_square_hand_case():
    # The RMS statistic is tree_sum(x*x): each square is one binary32 multiply
    # (rounded), then the pairwise tree adds them.  Hand-derived row of K = 16
    # pairs (a, b) = (2^-75, 1.5 * 2^-75), norm_eps = 2^-149:
    #   a*a = 2^-150 rounds to 0 (a tie, to even); b*b = 1.125 * 2^-149 rounds to
    #   2^-149; every pair adds to 2^-149 and the tree to 8 * 2^-149 = 2^-146;
    #   mean 2^-146 / 16 = 2^-150 rounds to 0; + eps = 2^-149;
    #   r = fl(1 / fl(sqrt(2^-149))) = 2^75 * fl(1 / fl(sqrt 2));
    #   u = (fl(1/fl(sqrt 2)), fl(1.5 * fl(1/fl(sqrt 2)))) per pair.
    # (Summing each pair with one rounding, a*a + fl(b*b) = 1.5 * 2^-149 -> 2^-148,
    # would give r = 2^74 and u = (0.5, 0.75) instead.)
    K = 16
    a_bits, b_bits = 0x1A00, 0x1A40  # bf16 of 2^-75 and 1.5 * 2^-75
    assert oracle.bf16_to_f32(np.array([a_bits], np.uint16))[0] == np.float32(2.0 ** -75)
    assert oracle.bf16_to_f32(np.array([b_bits], np.uint16))[0] == np.float32(1.5 * 2.0 ** -75)
    row = np.tile(np.array([a_bits, b_bits], np.uint16), K // 2)[None, :]
    h = _f32_nearest(1 / _f32_sqrt_nearest(2))
    want = np.tile(np.array([float(h), float(_f32_nearest(Fraction(3, 2) * h))],
                            np.float32), K // 2)
    eps = float(2.0 ** -149)
    got = oracle.rmsnorm(row, norm_eps=eps)
    assert np.array_equal(got[0].view(np.uint32), want.view(np.uint32))
    # the same row through norm_transform without the transform
    got_t = oracle.norm_transform(row, norm_eps=eps, hadamard=False)
    assert np.array_equal(got_t[0].view(np.uint32), want.view(np.uint32))
    # LayerNorm of the row with its second half negated: the tree sum of x is 0
    # exactly (each half sums to +-10 * 2^-75), so d = x and the statistic is the
    # same sum of rounded squares
    neg = row.copy()
    neg[0, K // 2:] |= 0x8000
    want_ln = want.copy()
    want_ln[K // 2:] = -want_ln[K // 2:]
    got_ln = oracle.norm_transform(neg, norm_eps=eps, layernorm=True, hadamard=False)
    assert np.array_equal(got_ln[0].view(np.uint32), want_ln.view(np.uint32))


# ------------------------------------------------------- norm + transform

@pytest.mark.parametrize("name,M,K", [("tiny", 16, 256), ("attn_wo", 8, 2048),
                                      ("quant", 8, 4096), ("ffn_wdown", 4, 16384)])
def test_norm_fwht_fp32_within_1e6_of_fp64(name, M, K):
    X = inputs.activations(name, M=M, K=K) if name != "tiny" else inputs.activations("tiny")
    v32 = oracle.norm_fwht(X).astype(np.float64)
    v64 = oracle.norm_fwht_f64(X)
    rel = np.abs(v32 - v64).max(axis=1) / np.abs(v64).max(axis=1)
    assert rel.max() < 1e-6
    # the fp64 composition is an orthonormal map of the normalised row (Parseval)
    u64 = torch.nn.functional.rms_norm(
        torch.from_numpy(oracle.bf16_to_f32(X).astype(np.float64)), (K,), eps=1e-6).numpy()
    assert np.allclose((v64 ** 2).sum(1), (u64 ** 2).sum(1), rtol=1e-10)


def test_rotation_identity_for_linear_layers():
    # (x H/sqrt(n)) (W H/sqrt(n))^T = x W^T: the transform is orthonormal
    rng = np.random.default_rng(2)
    n = 64
    x = rng.standard_normal((3, n))
    W = rng.standard_normal((5, n))
    xh = oracle.fwht_f64(x) / np.sqrt(n)
    wh = oracle.fwht_f64(W) / np.sqrt(n)
    assert np.allclose(xh @ wh.T, x @ W.T, atol=1e-10)


# ------------------------------------------------------------ quantisers

def test_int8_ties_hand_case():
    g = _golden()["int8_ties"]
    v = np.array([g["input"]], dtype=np.float32)
    codes, scales, rowsum = oracle.quantize_rows(v, 8, quant_eps=g["quant_eps"])
    assert codes.view(np.int8).tolist()[0] == g["expected_codes"]
    assert scales[0] == np.float32(g["expected_scale"])
    assert rowsum[0] == g["expected_rowsum"]


def test_int4_ties_hand_case():
    g = _golden()["int4_ties"]
    s7 = oracle.sqrt7()
    y = np.float32(np.float32(4) * s7 - np.float32(6.5))
    v = np.array([[2.5, -0.5, 3.5, y]], dtype=np.float32)
    # precondition of the derivation: the pairwise tree of |v| is exactly 4*s7
    assert (np.float32(2.5) + np.float32(0.5)) + (np.float32(3.5) + y) == np.float32(4) * s7
    codes, scales, rowsum = oracle.quantize_rows(v, 4, quant_eps=g["quant_eps"])
    assert codes.tolist()[0] == g["expected_packed"]
    assert oracle.decode_codes(codes, 4, 4).tolist()[0] == g["expected_codes"]
    assert scales[0] == np.float32(g["expected_scale"])
    assert rowsum[0] == g["expected_rowsum"]


def _tie_case():
    """Find binary32 gamma, v with inv = fl(127/gamma) such that fl(v*inv) is a
    .5 tie while the exact product is not: one rounding of the exact product
    and rounding the binary32 product then the tie give different integers."""
    rng = np.random.default_rng(123)
    for _ in range(200000):
        gamma = np.float32(rng.uniform(100.0, 127.0))
        inv = np.float32(127.0) / gamma
        k = int(rng.integers(1, 60))
        v = np.float32((k + 0.5) / float(inv))
        for cand in (v, np.nextafter(v, np.float32(0)), np.nextafter(v, np.float32(1e9))):
            if abs(float(cand)) > float(gamma):
                continue
            p32 = np.float32(cand * inv)
            ex = Fraction(float(cand)) * Fraction(float(inv))
            if float(p32) == k + 0.5 and ex != Fraction(2 * k + 1, 2):
                if round(ex) != round(Fraction(float(p32))):
                    return gamma, cand, inv, ex, p32
    raise AssertionError("no tie case found")


def test_quantiser_rounds_the_exact_product_once():
    # Reading: each code rounds the exact product v * (127/(gamma+eps)) once.
    gamma, v, inv, exact, p32 = _tie_case()
    row = np.array([[v, gamma]], dtype=np.float32)
    codes, _, _ = oracle.quantize_rows(row, 8, quant_eps=0.0)
    got = int(codes.view(np.int8)[0, 0])
    assert got == round(exact)
    assert got != round(Fraction(float(p32)))


def test_int4_clip_hand_case():
    g = _golden()["int4_clip"]
    v = np.array([g["input"]], dtype=np.float32)
    codes, _, _ = oracle.quantize_rows(v, 4, quant_eps=g["quant_eps"])
    assert oracle.decode_codes(codes, 8, 4).tolist()[0] == g["expected_codes"]


@pytest.mark.parametrize("bits", [4, 8])
def test_zero_row(bits):
    v = np.zeros((2, 16), dtype=np.float32)
    codes, scales, rowsum = oracle.quantize_rows(v, bits)
    assert not codes.any() and not scales.any() and not rowsum.any()
    X = np.zeros((2, 64), dtype=np.uint16)
    c2, s2, r2 = oracle.norm_fwht_quant(X, bits)
    assert not c2.any() and not s2.any() and not r2.any()


@pytest.mark.parametrize("bits", [4, 8])
def test_quantiser_brute_force_rounding(bits):
    # Per-element rounding checked against Python's round-half-even on the
    # binary32 product, for rows that straddle many .5 boundaries.
    rng = np.random.default_rng(bits)
    K = 64
    v = (rng.integers(-40, 40, size=(6, K)) / 4.0).astype(np.float32)
    v[0, :4] = [0.5, 1.5, 2.5, -3.5]
    codes, scales, rowsum = oracle.quantize_rows(v, bits, quant_eps=1e-5)
    q = oracle.decode_codes(codes, K, bits).astype(np.int64)
    lo, hi = (-8, 7) if bits == 4 else (-128, 127)
    for m in range(v.shape[0]):
        row = v[m]
        if bits == 8:
            inv = np.float32(127.0) / (np.abs(row).max() + np.float32(1e-5))
            scale = np.abs(row).max() / np.float32(127.0)
        else:
            beta = np.float32(oracle.tree_sum(np.abs(row))) * np.float32(1.0 / K)
            inv = oracle.sqrt7() / (beta + np.float32(1e-5))
            scale = beta / oracle.sqrt7()
        for k in range(K):
            # the exact product of the two binary32 values, rounded once
            y = Fraction(float(row[k])) * Fraction(float(inv))
            assert q[m, k] == min(hi, max(lo, round(y)))
        assert scales[m] == np.float32(scale)
        assert rowsum[m] == q[m].sum()
    assert q.min() >= lo and q.max() <= hi


def test_code_ranges_and_reachability():
    X = inputs.activations("tiny")
    c4, _, _ = oracle.norm_fwht_quant(X, 4)
    q4 = oracle.decode_codes(c4, 256, 4)
    assert q4.min() == -8 and q4.max() == 7
    c8, s8, _ = oracle.norm_fwht_quant(X, 8)
    q8 = oracle.decode_codes(c8, 256, 8).astype(np.int64)
    assert q8.min() >= -128 and q8.max() <= 127
    # the absmax element of every row maps to +-127 (gamma >> eps)
    assert np.all(np.abs(q8).max(axis=1) == 127)


def test_outlier_invariant_int4_error_lower_after_transform():
    # BitNet v2 write-up, section "H-BitLinear": the transform turns the sharp,
    # outlier-heavy distribution into a Gaussian-like one that suits INT4.
    X = inputs.activations("tiny")
    K = X.shape[1]
    u = oracle.rmsnorm(X)
    v = oracle.norm_fwht(X)

    def err(rows):
        codes, scales, _ = oracle.quantize_rows(rows, 4)
        deq = oracle.decode_codes(codes, K, 4).astype(np.float64) * scales[:, None]
        return np.linalg.norm(rows.astype(np.float64) - deq, axis=1)

    eu, ev = err(u), err(v)
    assert np.all(ev < eu)
    assert ev.sum() < 0.5 * eu.sum()


# ------------------------------------------------------------ ternary

def test_ternary_codes_and_threshold_form():
    # "[论文品鉴] 1-bit LLM", section "量化函数": t = +1 above a threshold,
    # -1 below minus it, 0 in between; with round-half-even the threshold is
    # (alpha + eps) / 2.
    W = inputs.latent_weights(128, 256, seed=0)
    t, alpha = oracle.ternarize(W, eps=1e-5)
    assert set(np.unique(t)).issubset({-1, 0, 1})
    assert np.isclose(alpha, np.abs(W.astype(np.float64)).mean(), rtol=1e-6)
    d = np.float64(alpha) + 1e-5
    thr = d / 2
    ref = np.sign(W) * (np.abs(W) > thr)
    away = np.abs(np.abs(W.astype(np.float64)) - thr) > 4 * np.spacing(np.float32(thr))
    assert np.array_equal(t[away], ref[away].astype(np.int8))


def test_ternarize_constant_magnitude_and_identity():
    N, K = 48, 16  # N*K = 768, not a power of two
    sgn = np.where(np.random.default_rng(1).random((N, K)) < 0.5, -1.0, 1.0)
    t, alpha = oracle.ternarize((0.25 * sgn).astype(np.float32))
    assert alpha == np.float32(0.25)
    assert np.array_equal(t, sgn.astype(np.int8))
    I = np.eye(64, dtype=np.float32)
    tI, aI = oracle.ternarize(I)
    assert aI == np.float32(1.0 / 64)
    assert np.array_equal(tI, np.eye(64, dtype=np.int8))


def test_pack_word_hand_case_and_round_trip():
    g = _golden()["pack_word"]
    t = np.array([g["t"]], dtype=np.int8)
    w = oracle.pack_codes(t)
    assert w[0, 0] == int(g["expected_word_hex"], 16)
    W = inputs.latent_weights(32, 512, seed=4)
    packed, _ = oracle.pack_ternary(W)
    tt, _ = oracle.ternarize(W)
    assert np.array_equal(oracle.unpack_codes(packed, 512), tt)
    # code 3 is never written
    for shift in range(0, 32, 2):
        assert not np.any(((packed >> shift) & 3) == 3)


# ------------------------------------------------------------ GEMM + dequant

def _rand_codes(rng, M, K, bits):
    V = rng.standard_normal((M, K)).astype(np.float32)
    V[:, 3] *= 30
    return oracle.quantize_rows(V, bits)


@pytest.mark.parametrize("bits", [4, 8])
@pytest.mark.parametrize("M,K,N", [(1, 16, 16), (5, 64, 32), (7, 256, 48)])
def test_gemm_integer_brute_force_and_dequant(bits, M, K, N):
    rng = np.random.default_rng(M * 100 + K + N + bits)
    codes, scales, rowsum = _rand_codes(rng, M, K, bits)
    W = rng.standard_normal((N, K)).astype(np.float32) * 0.02
    packed, alpha = oracle.pack_ternary(W)
    t = oracle.unpack_codes(packed, K).astype(np.int64)
    q = oracle.decode_codes(codes, K, bits).astype(np.int64)
    Y, acc = oracle.ternary_gemm(codes, scales, bits, K, packed, alpha)
    assert np.array_equal(acc, q @ t.T)
    sc = torch.from_numpy((np.float32(alpha) * scales).astype(np.float32))
    want = (torch.from_numpy(acc.astype(np.float32)) * sc[:, None]).to(torch.bfloat16)
    assert np.array_equal(Y, want.view(torch.int16).numpy().view(np.uint16))


@pytest.mark.parametrize("bits", [4, 8])
def test_gemm_identity_and_all_ones_weights(bits):
    rng = np.random.default_rng(9)
    K = 64
    codes, scales, rowsum = _rand_codes(rng, 6, K, bits)
    q = oracle.decode_codes(codes, K, bits).astype(np.int32)
    pI = oracle.pack_codes(np.eye(K, dtype=np.int8))
    _, acc = oracle.ternary_gemm(codes, scales, bits, K, pI, np.float32(1.0))
    assert np.array_equal(acc, q)
    p1 = oracle.pack_codes(np.ones((16, K), dtype=np.int8))
    _, acc1 = oracle.ternary_gemm(codes, scales, bits, K, p1, np.float32(1.0))
    assert np.array_equal(acc1, np.repeat(rowsum[:, None], 16, axis=1))


def test_forward_composition():
    X = inputs.activations("tiny")
    W = inputs.weights("tiny")
    packed, alpha = oracle.pack_ternary(W)
    for bits in (4, 8):
        Y = oracle.hbitlinear_forward(X, packed, alpha, bits)
        codes, scales, _ = oracle.norm_fwht_quant(X, bits)
        Y2, _ = oracle.ternary_gemm(codes, scales, bits, 256, packed, alpha)
        assert np.array_equal(Y, Y2)
        # dequantised output approximates the float layer x_hat W_t^T alpha
        v = oracle.norm_fwht(X).astype(np.float64)
        t = oracle.unpack_codes(packed, 256).astype(np.float64)
        ref = (v @ t.T) * np.float64(alpha)
        y = oracle.bf16_to_f32(Y).astype(np.float64)
        rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
        assert rel < (0.25 if bits == 4 else 0.02)
