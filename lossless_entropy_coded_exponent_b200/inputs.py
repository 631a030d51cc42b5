"""Seeded synthetic BF16 weight tensors.

This module holds only input generation: random draws and the fp32 -> BF16
round-to-nearest-even conversion that produces the test and benchmark
tensors.  It contains none of the codec's arithmetic, so both the CPU oracle
and the CUDA library can be fed from it.

The workloads stand in for trained LLM weights, which are not available
here.  The pages measure on Llama 2 7B ("From a Lossless (~1.5:1)
Compression Algorithm for Llama2 7B Weights ...", abstract) and on large
BF16 LLMs in general ("DFloat11: lossless LLM compression for GPU",
aikraft.ru blog, sections 01-02); trained weights are close to zero-mean
Gaussians with a few large outliers, which is what is drawn here:

* ``gaussian``: numpy ``default_rng(seed)`` (PCG64), ``standard_normal`` in
  float32 times sigma (one fp32 multiply), then fp32 -> BF16 with
  round-to-nearest-even done in integer arithmetic;
* ``with_outliers``: ``floor(frac * n)`` positions drawn without
  replacement from the same generator are replaced by N(0, sigma_out^2)
  draws, rounded the same way.

Every tensor is returned as a flat ``np.uint16`` array of BF16 bit patterns.
"""
from __future__ import annotations

import math

import numpy as np


def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    """fp32 -> BF16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((u >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((u + bias) >> np.uint32(16)).astype(np.uint16)


def gaussian(n: int, sigma: float, seed: int, rng: np.random.Generator | None = None) -> np.ndarray:
    rng = np.random.default_rng(seed) if rng is None else rng
    x = rng.standard_normal(n, dtype=np.float32)
    x *= np.float32(sigma)
    return bf16_from_f32(x)


def with_outliers(w: np.ndarray, frac: float, sigma_out: float, rng: np.random.Generator) -> np.ndarray:
    n = w.size
    k = int(math.floor(frac * n))
    if k == 0:
        return w
    pos = rng.choice(n, size=k, replace=False)
    vals = rng.standard_normal(k, dtype=np.float32) * np.float32(sigma_out)
    w = w.copy()
    w[pos] = bf16_from_f32(vals)
    return w


# --------------------------------------------------------------------------
# The five workload families.

def small_gaussian() -> np.ndarray:
    """One 1024x1024 tensor, N(0, 0.02^2), seed 1."""
    return gaussian(1024 * 1024, 0.02, seed=1)


def projection_with_outliers() -> np.ndarray:
    """4096x4096, N(0, 0.02^2) with 0.1 % of entries replaced by N(0, 1), seed 3."""
    rng = np.random.default_rng(3)
    w = gaussian(4096 * 4096, 0.02, seed=3, rng=rng)
    return with_outliers(w, 0.001, 1.0, rng)


# Llama-3-8B decoder layer: (name, rows = out features, cols = in features).
LLAMA3_8B_LAYER = [
    ("q_proj", 4096, 4096),
    ("k_proj", 1024, 4096),
    ("v_proj", 1024, 4096),
    ("o_proj", 4096, 4096),
    ("gate_proj", 14336, 4096),
    ("up_proj", 14336, 4096),
    ("down_proj", 4096, 14336),
]


def llama3_8b_layer_tensor(i: int) -> np.ndarray:
    """Tensor i of the Llama-3-8B-shaped layer: N(0, 1/fan_in), seed 40 + i."""
    _, rows, cols = LLAMA3_8B_LAYER[i]
    return gaussian(rows * cols, 1.0 / math.sqrt(cols), seed=40 + i)


LAYER70B_SHAPE = (8192, 28672)
LAYER70B_COUNT = 24


def layer70b_tensor(i: int, seed_base: int = 500) -> np.ndarray:
    """Tensor i of the 70B-shaped layer stream: 8192x28672, N(0, 1/8192) plus
    0.05 % outliers drawn N(0, 0.5^2); seed seed_base + i."""
    rows, cols = LAYER70B_SHAPE
    rng = np.random.default_rng(seed_base + i)
    w = gaussian(rows * cols, 1.0 / math.sqrt(8192), seed=seed_base + i, rng=rng)
    return with_outliers(w, 0.0005, 0.5, rng)


def layer70b_sample(n: int, seed: int) -> np.ndarray:
    """A smaller tensor with the 70B-layer value distribution (for CPU timing)."""
    rng = np.random.default_rng(seed)
    w = gaussian(n, 1.0 / math.sqrt(8192), seed=seed, rng=rng)
    return with_outliers(w, 0.0005, 0.5, rng)


# --------------------------------------------------------------------------
# Edge cases.

def special_mix(n: int, seed: int) -> np.ndarray:
    """Quarters of +-0, subnormals (exponent 0, mantissa != 0), +-Inf and NaNs
    with random non-zero payloads and signs, shuffled."""
    rng = np.random.default_rng(seed)
    q = n // 4
    sign = (rng.integers(0, 2, size=n, dtype=np.uint16) << np.uint16(15)).astype(np.uint16)
    zeros = np.zeros(q, dtype=np.uint16)
    subn = rng.integers(1, 128, size=q, dtype=np.uint16)
    infs = np.full(q, 0x7F80, dtype=np.uint16)
    nans = (np.uint16(0x7F80) | rng.integers(1, 128, size=n - 3 * q, dtype=np.uint16)).astype(np.uint16)
    w = np.concatenate([zeros, subn, infs, nans]) | sign
    rng.shuffle(w)
    return w.astype(np.uint16)


def uniform_patterns(n: int, seed: int) -> np.ndarray:
    """Uniformly random 16-bit patterns: all 256 exponents about equally likely."""
    return np.random.default_rng(seed).integers(0, 1 << 16, size=n, dtype=np.uint16)


def all_patterns_shuffled(seed: int) -> np.ndarray:
    w = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    np.random.default_rng(seed).shuffle(w)
    return w


def fibonacci_counts(n_symbols: int = 28) -> list[int]:
    f = [1, 1]
    while len(f) < n_symbols:
        f.append(f[-1] + f[-2])
    return f[:n_symbols]


def fibonacci_clamp_tensor(seed: int, n_symbols: int = 28, first_exponent: int = 100) -> np.ndarray:
    """Exponent counts F1..F28 (sum 832 039): the unlimited Huffman tree is
    27 deep, so a 24-bit length limit must bind.  Sign and mantissa random."""
    rng = np.random.default_rng(seed)
    counts = fibonacci_counts(n_symbols)
    e = np.concatenate([np.full(c, first_exponent + i, dtype=np.uint16) for i, c in enumerate(counts)])
    rng.shuffle(e)
    sign = rng.integers(0, 2, size=e.size, dtype=np.uint16)
    mant = rng.integers(0, 128, size=e.size, dtype=np.uint16)
    # the BF16 encoding of (-1)^sign * 1.mant * 2^(e - 127)
    return ((sign << np.uint16(15)) | (e << np.uint16(7)) | mant).astype(np.uint16)


def exponent_spread(n: int, n_values: int, seed: int, first_exponent: int = 40, decay: float = 0.95) -> np.ndarray:
    """Exactly n_values distinct exponents, first_exponent .. first_exponent + n_values - 1:
    each once, the other n - n_values drawn with probability proportional to decay^i, so the
    code lengths spread out.  Sign and mantissa are random.  It sets the number of leaves
    of the code book's package-merge."""
    assert n_values <= n and first_exponent + n_values <= 255
    rng = np.random.default_rng(seed)
    p = decay ** np.arange(n_values, dtype=np.float64)
    p /= p.sum()
    e = np.concatenate([np.arange(n_values), rng.choice(n_values, size=n - n_values, p=p)]).astype(np.uint16)
    e += np.uint16(first_exponent)
    rng.shuffle(e)
    sign = rng.integers(0, 2, size=n, dtype=np.uint16)
    mant = rng.integers(0, 128, size=n, dtype=np.uint16)
    return ((sign << np.uint16(15)) | (e << np.uint16(7)) | mant).astype(np.uint16)


def edge_cases() -> dict[str, np.ndarray]:
    """The edge-case set: ragged lengths, one-symbol, incompressible, specials."""
    cases = {}
    for i, n in enumerate((1, 7, 4097, 1_000_003)):
        cases[f"len{n}"] = gaussian(n, 0.02, seed=20 + i)
    cases["empty"] = np.zeros(0, dtype=np.uint16)
    cases["all_zero"] = np.zeros(65536, dtype=np.uint16)
    cases["uniform_exponents"] = uniform_patterns(1 << 20, seed=24)
    cases["special_mix"] = special_mix(1 << 20, seed=25)
    cases["all_patterns"] = all_patterns_shuffled(seed=26)
    cases["fibonacci_clamp"] = fibonacci_clamp_tensor(seed=27)
    return cases


# --------------------------------------------------------------------------
# Device-side generation for the large benchmark stream.  Same recipe as
# ``layer70b_tensor`` (fp32 normal draws times sigma, round-to-nearest-even to
# BF16, 0.05 % of positions replaced by N(0, 0.5^2) outliers) but drawn with
# torch's seeded CUDA generator (Philox), because drawing 5.6 B normals on the
# host takes minutes.  The values differ from the numpy draws; the distribution
# is the same.  Anything checked against the oracle is copied back to the host
# first, so both sides always see identical bytes.

def bf16_from_f32_torch(x):
    """fp32 -> BF16 bit patterns (int16 tensor), round to nearest, ties to even."""
    import torch

    u = x.contiguous().view(torch.int32)
    bias = ((u >> 16) & 1) + 0x7FFF
    return ((u + bias) >> 16).to(torch.int16)


def llama3_8b_layer_tensor_cuda(i: int, device="cuda"):
    """Tensor i of the Llama-3-8B-shaped layer drawn on the device: the same recipe as
    llama3_8b_layer_tensor (N(0, 1/fan_in), seed 40 + i) with torch's seeded generator."""
    import torch

    _, rows, cols = LLAMA3_8B_LAYER[i]
    g = torch.Generator(device=device)
    g.manual_seed(40 + i)
    x = torch.randn(rows * cols, device=device, dtype=torch.float32, generator=g)
    x.mul_(1.0 / math.sqrt(cols))
    return bf16_from_f32_torch(x)


def layer70b_tensor_cuda(i: int, seed_base: int = 500, device="cuda"):
    import torch

    rows, cols = LAYER70B_SHAPE
    n = rows * cols
    g = torch.Generator(device=device)
    g.manual_seed(seed_base + i)
    x = torch.randn(n, device=device, dtype=torch.float32, generator=g)
    x.mul_(1.0 / math.sqrt(8192))
    w = bf16_from_f32_torch(x)
    del x
    k = int(math.floor(0.0005 * n))
    pos = torch.randperm(n, device=device, generator=g)[:k]
    vals = torch.randn(k, device=device, dtype=torch.float32, generator=g) * 0.5
    w[pos] = bf16_from_f32_torch(vals)
    return w
