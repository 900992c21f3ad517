"""Seeded synthetic inputs shared by the oracle tests, the CUDA parity tests,
``__graft_entry__.smoke()`` and ``bench.py``.

This module draws random numbers and nothing else: it holds none of the
layer's arithmetic (no rotation, no scale computation, no codebook fit, no
quantisation).  The real checkpoints are not available, so every input is
synthetic, with the distributions the workloads are described with:

* weights: fp32 N(0, 0.02^2), 0.5 % of the entries replaced by N(0, 0.2^2)
  outliers;
* activations: bf16 N(0, 1), a chosen set of input channels scaled by 20;
* stored-format tensors (for throughput runs and full-size parity): packed
  indices uniform over all 256 byte values, e4m3 group-scale codes uniform
  over the codes of [1/8, 1], positive fp32 row scales and an ascending
  16-entry fp32 codebook in [-1, 1].

Seeds: numpy PCG64 from ``SeedSequence([config, layer, kind])``.
"""

from __future__ import annotations

import numpy as np

KINDS = {"weight": 0, "act": 1, "qfmt": 2, "sample": 3}


def rng_for(config: int, layer: int = 0, kind: str = "weight") -> np.random.Generator:
    """numpy PCG64 generator for (config, layer, tensor kind)."""
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([config, layer, KINDS[kind]])))


def weights(n: int, k: int, rng: np.random.Generator, sigma: float = 0.02,
            outlier_frac: float = 0.005, outlier_sigma: float = 0.2) -> np.ndarray:
    """fp32 W[n, k] ~ N(0, sigma^2) with a fraction of entries replaced by
    N(0, outlier_sigma^2) draws at positions chosen by the generator."""
    w = rng.normal(0.0, sigma, size=(n, k)).astype(np.float32)
    count = int(round(outlier_frac * n * k))
    if count:
        pos = rng.choice(n * k, size=count, replace=False)
        w.reshape(-1)[pos] = rng.normal(0.0, outlier_sigma, size=count).astype(np.float32)
    return w


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Nearest bf16 (round half to even) of finite fp32 values, as uint16 bits."""
    bits = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bits = bits + 0x7FFF + ((bits >> 16) & 1)
    return (bits >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bits -> the fp32 values they denote (exact)."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def activations(m: int, k: int, rng: np.random.Generator, outlier_channels: int,
                scale: float = 20.0):
    """bf16 x[m, k] ~ N(0, 1) with ``outlier_channels`` input channels scaled.

    Returns (bf16 bits uint16 [m, k], fp32 values [m, k], chosen channels).
    """
    x = rng.normal(0.0, 1.0, size=(m, k)).astype(np.float32)
    ch = np.sort(rng.choice(k, size=outlier_channels, replace=False)) if outlier_channels else np.zeros(0, np.int64)
    x[:, ch] *= np.float32(scale)
    bits = f32_to_bf16_bits(x)
    return bits, bf16_bits_to_f32(bits), ch


def codebook(rng: np.random.Generator) -> np.ndarray:
    """16 distinct ascending fp32 levels in [-1, 1] (sorted normal draws
    divided by their largest magnitude)."""
    while True:
        c = np.sort(rng.normal(0.0, 1.0, size=16))
        c = (c / np.abs(c).max()).astype(np.float32)
        if np.all(np.diff(c.astype(np.float64)) > 0):
            return c


def quantized_format(n: int, k: int, rng: np.random.Generator) -> dict:
    """Stored-format tensors drawn directly: packed [n, k/2] uint8, s_rel
    e4m3 codes [n, k/16] uint8 (codes 32..56, the values 1/8 .. 1), s_ch fp32
    [n] in [0.05, 0.15], cb fp32 [16]."""
    return {
        "packed": rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8),
        "s_rel": rng.integers(32, 57, size=(n, k // 16), dtype=np.uint8),
        "s_ch": rng.uniform(0.05, 0.15, size=n).astype(np.float32),
        "cb": codebook(rng),
    }


def nvfp4_operands(rows: int, k: int, rng: np.random.Generator) -> dict:
    """NVFP4-format operands drawn directly: packed codes [rows, k/2] uint8
    (every byte value), e4m3 scale codes [rows, k/16] uint8 in 0x20..0x58
    (the values 1/8 .. 16), fp32 scalars [rows] in [1e-3, 1e-2]."""
    return {
        "codes": rng.integers(0, 256, size=(rows, k // 2), dtype=np.uint8),
        "scales": rng.integers(0x20, 0x59, size=(rows, k // 16), dtype=np.uint8),
        "g": rng.uniform(1e-3, 1e-2, size=rows).astype(np.float32),
    }


def quantized_format_device(n: int, k: int, seed: int, device):
    """Same distributions as :func:`quantized_format`, drawn by torch's
    generator directly on ``device`` (for multi-GB throughput inputs)."""
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    packed = torch.randint(0, 256, (n, k // 2), generator=g, device=device, dtype=torch.uint8)
    s_rel = torch.randint(32, 57, (n, k // 16), generator=g, device=device, dtype=torch.uint8)
    s_ch = torch.rand(n, generator=g, device=device, dtype=torch.float32) * 0.1 + 0.05
    cb = torch.from_numpy(codebook(np.random.Generator(np.random.PCG64(seed)))).to(device)
    return {"packed": packed, "s_rel": s_rel, "s_ch": s_ch, "cb": cb}


EXTREME_CODEBOOK = np.array([-8.0, -4.5, -2.5, -1.5, -0.9, -0.5, -0.2, -3e-5, 2e-5, 0.15, 0.4, 0.8, 1.3,
                             2.2, 4.0, 7.5], dtype=np.float32)


def quantized_format_edges(n: int, k: int, rng: np.random.Generator) -> dict:
    """Stored-format tensors at the edges of the format: group-scale codes
    mixed with e4m3 subnormals (codes 1..7) and zeros inside live rows, a row
    with every group scale zero, a row whose only live group is its first,
    a row with a zero row scale, and a codebook with two levels within 1e-4
    of zero and levels out to -8 and 7.5.  Indices uniform over all bytes."""
    if n < 4:
        raise ValueError("needs at least 4 rows")
    s_rel = rng.integers(32, 57, size=(n, k // 16), dtype=np.uint8)
    u = rng.random(size=s_rel.shape)
    s_rel[u < 0.15] = rng.integers(1, 8, size=int((u < 0.15).sum()), dtype=np.uint8)   # subnormal codes
    s_rel[(u >= 0.15) & (u < 0.22)] = 0                                                # zero groups
    s_rel[0] = 0                                  # a dead row
    s_rel[1, 1:] = 0                              # one live group
    s_ch = rng.uniform(0.05, 0.15, size=n).astype(np.float32)
    s_ch[2] = 0.0                                 # a zero row scale
    return {"packed": rng.integers(0, 256, size=(n, k // 2), dtype=np.uint8), "s_rel": s_rel,
            "s_ch": s_ch, "cb": EXTREME_CODEBOOK.copy()}


def weights_with_edges(n: int, k: int, rng: np.random.Generator) -> np.ndarray:
    """:func:`weights` with edge rows for the converter: an all-zero row, a
    row with one large entry (300, about 10^4 times the rest: its other
    groups' ratios to the row maximum fall to e4m3 subnormals or zero), a
    row whose first half is zero, and a row with one zero block of 256 (16
    zero groups, after rotation too) between live ones."""
    if n < 5 or k < 768:
        raise ValueError("needs at least 5 rows and 768 columns")
    w = weights(n, k, rng)
    w[1] = 0.0
    w[2, 5] = 300.0
    w[3, : k // 2] = 0.0
    w[4, 256:512] = 0.0
    return w
