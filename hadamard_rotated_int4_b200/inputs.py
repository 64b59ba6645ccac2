"""Seeded synthetic inputs for the H-BitLinear workloads.

This module holds only random-number recipes (no normalisation, transform,
quantisation or matmul): the same arrays feed both the CUDA path and the CPU
oracle in tests and in the benchmark.

All draws use numpy's PCG64 (``numpy.random.default_rng(seed)``).  Activations
are built in float64/float32, then rounded once to bfloat16 (round to nearest
even, via torch) and returned as uint16 bit patterns.  Outlier channels are
chosen with ``rng.choice(K, count, replace=False)`` and multiplied before the
bf16 rounding, standing in for the outlier-heavy inputs of the attention output
projection (Wo) and the FFN down projection (W_down) that the BitNet v2 pages
describe.  Latent weights are N(0, 0.02^2) in float32.

Workloads (tokens x in-features -> out-features):
  tiny       16 x 256 -> 128, N(0,1), channels {3, 77, 140, 201} x 50
  quant      8192 x 4096 (activations only), Student-t nu=3, 1% channels x 20
  attn_wo    4096 x 2048 -> 2048, N(0,1), 0.5% channels x 30
  ffn_wdown  8192 x 16384 -> 4096, silu(a)*b with a, b ~ N(0,1), 1% channels x 40
  decode     T x 4096 -> 4096 (attn_wo recipe) and T x 16384 -> 4096 (ffn_wdown
             recipe), T in {1, 8, 32, 128, 256}
  qkv        Q, K, V states after RoPE for the KV-cache quantiser: 8192 tokens x
             (3 x 32) heads x 128, N(0,1) times a per-(token, head) log-normal
             magnitude (sigma 0.5), with 2% of the head dimensions (the same for
             every token) x 8, standing in for the outlier dimensions of keys
  signs      +-1 fp32 vector (fair coin) for the randomised Hadamard transform
"""
import numpy as np


def _to_bf16_bits(x):
    import torch

    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16).copy()


def outlier_channels(rng, K, frac=None, count=None):
    if count is None:
        count = int(round(frac * K))
    return np.sort(rng.choice(K, size=count, replace=False))


def gaussian_acts(M, K, seed=0, frac=0.005, mult=30.0, channels=None):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((M, K), dtype=np.float32)
    ch = outlier_channels(rng, K, frac=frac) if channels is None else np.asarray(channels)
    x[:, ch] *= np.float32(mult)
    return _to_bf16_bits(x)


def student_t_acts(M, K, seed=0, nu=3.0, frac=0.01, mult=20.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_t(nu, size=(M, K)).astype(np.float32)
    ch = outlier_channels(rng, K, frac=frac)
    x[:, ch] *= np.float32(mult)
    return _to_bf16_bits(x)


def swiglu_acts(M, K, seed=0, frac=0.01, mult=40.0):
    rng = np.random.default_rng(seed)
    a = rng.standard_normal((M, K), dtype=np.float32)
    b = rng.standard_normal((M, K), dtype=np.float32)
    x = (a / (np.float32(1.0) + np.exp(-a))) * b
    del a, b
    ch = outlier_channels(rng, K, frac=frac)
    x[:, ch] *= np.float32(mult)
    return _to_bf16_bits(x)


def latent_weights(N, K, seed=0, std=0.02):
    rng = np.random.default_rng(seed + 1000003)
    return (rng.standard_normal((N, K), dtype=np.float32) * np.float32(std)).astype(np.float32)


WORKLOADS = {
    "tiny": dict(M=16, K=256, N=128),
    "quant": dict(M=8192, K=4096, N=None),
    "attn_wo": dict(M=4096, K=2048, N=2048),
    "ffn_wdown": dict(M=8192, K=16384, N=4096),
}

DECODE_TOKENS = (1, 2, 4, 8, 32, 128, 256)


def activations(name, seed=0, M=None, K=None):
    """bf16 bit patterns [M x K] for a named workload (M/K overridable for sub-cases)."""
    w = WORKLOADS.get(name, {})
    M = w.get("M") if M is None else M
    K = w.get("K") if K is None else K
    if name == "tiny":
        return gaussian_acts(M, K, seed, mult=50.0, channels=[3, 77, 140, 201])
    if name == "quant":
        return student_t_acts(M, K, seed)
    if name in ("attn_wo", "decode_wo"):
        return gaussian_acts(M, K, seed, frac=0.005, mult=30.0)
    if name in ("ffn_wdown", "decode_wdown"):
        return swiglu_acts(M, K, seed)
    raise KeyError(name)


def weights(name, seed=0, N=None, K=None):
    w = WORKLOADS.get(name, {})
    N = w.get("N") if N is None else N
    K = w.get("K") if K is None else K
    return latent_weights(N, K, seed)


QKV = dict(T=8192, H=96, D=128)  # 7B-like: 32 query + 32 key + 32 value heads of 128


def qkv_states(T=None, H=None, D=None, seed=0, frac=0.02, mult=8.0):
    """bf16 bit patterns [T x H x D] of attention states after RoPE."""
    T = QKV["T"] if T is None else T
    H = QKV["H"] if H is None else H
    D = QKV["D"] if D is None else D
    rng = np.random.default_rng(seed + 7919)
    x = rng.standard_normal((T, H, D), dtype=np.float32)
    mag = np.exp(rng.standard_normal((T, H, 1)) * 0.5).astype(np.float32)
    x *= mag
    dims = outlier_channels(rng, D, count=max(1, int(round(frac * D))))
    x[:, :, dims] *= np.float32(mult)
    return _to_bf16_bits(x)


def random_signs(K, seed=0):
    rng = np.random.default_rng(seed + 104729)
    return np.where(rng.random(K) < 0.5, -1.0, 1.0).astype(np.float32)
