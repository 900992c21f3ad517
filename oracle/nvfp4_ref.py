"""Plain CPU statement of an NVFP4 linear layer (4-bit weights AND 4-bit
activations), the speed and accuracy foil for the codebook path.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this file and this file imports nothing from the library.

Source: "Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på
Blackwell-GPU:er" (the *NVFP4 runbook* below), section "Vad NVFP4 är, och hur
det skiljer sig från FP8 och från INT8/AWQ".  What it fixes:

* a value is E2M1: one sign bit, two exponent bits, one mantissa bit;
* every 16 consecutive values share one E4M3 (fp8) scale;
* the whole tensor carries one fp32 scalar on top of the block scales, which
  restores the dynamic range a bare 4-bit float would lose;
* for contrast, MXFP4 uses 32-value blocks with power-of-two (E8M0) scales;
* Blackwell tensor cores run the FP4 matmul natively.

Readings taken where the page is silent (each also listed in the design
notes of the repository):

N1  E2M1 has exponent bias 1 and a subnormal step of 0.5, so the eight
    magnitudes are 0, 0.5, 1, 1.5, 2, 3, 4, 6.  Code = sign << 3 | e << 1 | m;
    two codes per byte, even k in the low nibble (as the codebook path packs
    its indices).
N2  Encoding rounds to the nearest magnitude, a tie going to the even code
    (mantissa bit 0), and saturates at 6.  The sign bit is kept when the
    magnitude rounds to 0.
N3  The fp32 scalar is g = amax / (6 * 448): the largest block of the tensor
    then gets the largest finite e4m3 scale.  Weights take one g per tensor,
    as the page states.  Activations take one g per token: a token's row is
    the tensor it forms in the product, and a per-token scalar needs no pass
    over the whole batch before quantising.  amax = 0 gives g = 0, and then
    every scale and code of that tensor (row) is 0.
N4  All decisions are taken in fp32, in this order: d = fp32(g * 6),
    t = fp32(bmax / d), s = e4m3(t) (round half to even, saturating at 448),
    S = fp32(decode(s) * g), code = e2m1(fp32(x / S)) where S > 0, else 0.
    bmax is the largest magnitude of the 16 values.
N5  Both operands live in the codebook path's rotated basis: each 256-block of
    K multiplied by the Sylvester Hadamard matrix over 16, the rotated value
    rounded to fp32 before any decision.  (Rotation is optional: the GPU
    quantiser can take rows that are already rotated.)
N6  y[m, n] = g_x[m] * g_w[n] * sum_k (e2m1(cx) e4m3(sx))[m, k] *
    (e2m1(cw) e4m3(sw))[n, k], unrounded in fp64: the comparison target of
    the tensor-core product.  g_w[n] is the tensor's g repeated per row (a
    per-row fp32 scale is the same formula).
"""

from __future__ import annotations

import numpy as np

from .w4a8_ref import e4m3_decode, e4m3_encode, rotate_blocks

BLOCK = 16                   # NVFP4 runbook: 16 values share one E4M3 scale
E2M1_MAX = 6.0               # largest E2M1 magnitude (reading N1)
E4M3_MAX = 448.0             # largest finite e4m3fn value
G_DIV = E2M1_MAX * E4M3_MAX  # reading N3: g = amax / 2688

# reading N1: magnitude of the 3-bit code e << 1 | m
E2M1_MAGNITUDES = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])

__all__ = [
    "BLOCK", "E2M1_MAX", "E2M1_MAGNITUDES", "G_DIV",
    "e2m1_decode", "e2m1_encode", "pack_codes", "unpack_codes",
    "quantize_rows", "dequant_rows", "gemm", "linear",
]


def e2m1_decode(codes: np.ndarray) -> np.ndarray:
    """4-bit E2M1 codes -> fp64 values (reading N1), built from the bit
    fields: e = 0 is subnormal (m * 0.5), else (1 + m/2) * 2**(e-1)."""
    c = np.asarray(codes).astype(np.int64) & 0xF
    e = (c >> 1) & 3
    m = (c & 1).astype(np.float64)
    mag = np.where(e == 0, m * 0.5, (1.0 + m / 2.0) * np.exp2(e - 1.0))
    return np.where(c & 8, -mag, mag)


def e2m1_encode(values: np.ndarray) -> np.ndarray:
    """fp64 values -> 4-bit E2M1 codes (reading N2): nearest magnitude, ties
    to the code with mantissa bit 0, saturating at 6, sign kept."""
    v = np.asarray(values, dtype=np.float64)
    a = np.minimum(np.abs(v), E2M1_MAX)
    # distance to every magnitude; on a tie the even code wins
    dist = np.abs(a[..., None] - E2M1_MAGNITUDES)
    best = dist.min(axis=-1, keepdims=True)
    cand = dist == best
    odd = (np.arange(8) & 1) == 1
    even_hit = cand & ~odd
    pick = np.where(even_hit.any(axis=-1), np.argmax(even_hit, axis=-1), np.argmax(cand, axis=-1))
    return (pick | np.where(np.signbit(v), 8, 0)).astype(np.uint8)


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """[R, K] 4-bit codes -> [R, K/2] bytes, even k in the low nibble."""
    c = np.asarray(codes, dtype=np.uint8)
    return (c[..., 0::2] & 0xF) | ((c[..., 1::2] & 0xF) << 4)


def unpack_codes(packed: np.ndarray) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0xF
    out[..., 1::2] = p >> 4
    return out


def quantize_rows(x: np.ndarray, rotate: bool = True, per_row: bool = True):
    """NVFP4-quantise the rows of x[R, K] (readings N3-N5).

    per_row=True: one g per row (activations); False: one g for the whole
    tensor (weights).  Returns (codes uint8 [R, K] (unpacked), scale codes
    uint8 e4m3 [R, K/16], g fp32 [R]).
    """
    x = np.asarray(x, dtype=np.float64)
    r, k = x.shape
    if k % BLOCK:
        raise ValueError(f"K={k} is not a multiple of {BLOCK}")
    xr = (rotate_blocks(x) if rotate else x).astype(np.float32)
    a = np.abs(xr)
    amax = a.max(axis=1) if per_row else np.full(r, a.max(), dtype=np.float32)
    g = (amax.astype(np.float32) / np.float32(G_DIV)).astype(np.float32)
    d = (g * np.float32(E2M1_MAX)).astype(np.float32)
    bmax = a.reshape(r, k // BLOCK, BLOCK).max(axis=2)
    safe_d = np.where(d > 0, d, np.float32(1.0)).astype(np.float32)
    t = (bmax / safe_d[:, None]).astype(np.float32)
    s = np.where(d[:, None] > 0, e4m3_encode(t.astype(np.float64)), 0).astype(np.uint8)
    big_s = (e4m3_decode(s).astype(np.float32) * g[:, None]).astype(np.float32)
    safe_s = np.where(big_s > 0, big_s, np.float32(1.0)).astype(np.float32)
    quot = (xr.reshape(r, k // BLOCK, BLOCK) / safe_s[:, :, None]).astype(np.float32)
    codes = np.where(big_s[:, :, None] > 0, e2m1_encode(quot.astype(np.float64)), 0)
    return codes.reshape(r, k).astype(np.uint8), s, g


def dequant_rows(codes, scales, g=None) -> np.ndarray:
    """e2m1(codes) * e4m3(scales) [* g per row] in fp64, shape [R, K]."""
    c = np.asarray(codes)
    r, k = c.shape
    v = e2m1_decode(c).reshape(r, k // BLOCK, BLOCK) * e4m3_decode(scales)[:, :, None]
    v = v.reshape(r, k)
    if g is not None:
        v = v * np.asarray(g, dtype=np.float64)[:, None]
    return v


def gemm(cx, sx, gx, cw, sw, gw) -> np.ndarray:
    """Reading N6: unrounded fp64 y[M, N] from quantised operands (unpacked
    codes, e4m3 scale codes, fp32 scalars per row)."""
    return dequant_rows(cx, sx, gx) @ dequant_rows(cw, sw, gw).T


def linear(x, w, rotate: bool = True) -> np.ndarray:
    """The whole NVFP4 layer from bf16-valued x[M, K] and fp32 W[N, K]:
    activations per token, weights per tensor (reading N3)."""
    cx, sx, gx = quantize_rows(x, rotate=rotate, per_row=True)
    cw, sw, gw = quantize_rows(w, rotate=rotate, per_row=False)
    return gemm(cx, sx, gx, cw, sw, gw)
