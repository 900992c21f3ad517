"""Plain fp64 CPU statement of the asym_w4a8_int8 ConvRot linear layer.

TEST INFRASTRUCTURE ONLY (see the package docstring): the CUDA library never
imports this file and this file imports nothing from the library.

What the pages fix, and where:

* ConvRot card, "Format": each quantised layer stores four tensors -- packed
  int4 indices (two per byte), an fp8 e4m3 scale per group of 16 values, an
  fp32 scale per output row and a 16-entry fp32 codebook.  The weight is
  rebuilt from three tiers: codebook shape x group magnitude x row magnitude.
  The codebook is a Lloyd-Max quantiser fitted to the tensor's own values.
  A group-wise Hadamard rotation ("ConvRot", group 256) is applied before
  quantisation.
* W4A8 card, "Model Overview": weight group size 16, rotation group size 256,
  int8 activations, fp8 group scales, fp32 channel scales.
* ConvRot card, "Reproducing": the codebook fit samples, and a seed (42)
  pins it.

Readings taken where the pages are silent or disagree (each also listed in
the design notes of the repository):

R1  One codebook per tensor.  The W4A8 card says "per-group" codebook; the
    ConvRot card says "per-tensor" and lists a single fp32 tensor of "the 16
    quantization levels" per layer.  The per-tensor reading is used.
R2  The rotation is the Sylvester-ordered Hadamard matrix scaled by 1/16
    (orthonormal for n = 256), no random signs or permutation: no sign or
    permutation tensor is among the four stored tensors.
R3  s_channel[n] = max_k |R[n,k]| of the rotated row, stored as fp32.
R4  s_rel[n,g] = e4m3(max over the group of |R[n,k]| / s_channel[n]),
    round-to-nearest-even, saturating.  Values are <= 1 so saturation never
    triggers in practice.
R5  The normalised value v = R / (s_rel * s_channel) uses the STORED scales.
    Positions whose scale product is 0 get v = 0 and are left out of the fit.
R6  Lloyd-Max with 16 levels on all normalised values of the tensor: start at
    the empirical quantiles (i + 0.5) / 16, alternate "boundaries are
    midpoints" and "levels are cell means", stop when no level moves by more
    than 1e-12 or after 500 rounds.  An empty cell keeps its level.  More
    than 2**22 values: fit on a uniform sample of 2**22 drawn without
    replacement by numpy PCG64 seeded with 42.  Levels are stored ascending
    as fp32.
R7  Index = nearest stored (fp32) level; a value exactly on a midpoint takes
    the lower index.  Packing: two indices per byte, even k in the low nibble.
R8  Activations: per token, symmetric, s_x = absmax / 127, q = round half to
    even of x_rot / s_x, clamped to [-127, 127].  The pages fix no precision
    for this integer decision, so it is taken in the kernel's precision,
    fp32: x_rot rounded to fp32, s_x = fp32(amax / 127), q from the fp32
    quotient.  An all-zero token gives s_x = 0 and q = 0.
R9  "asym" has no zero point among the stored tensors; the asymmetry lives
    in the freely fitted codebook.
R10 The layer output is y = s_x[m] * sum_k q[m,k] * W_hat[n,k] with
    W_hat = fp32(fp32(cb[idx] * s_rel) * s_channel) in the rotated basis.
    This unrounded fp64 value is the comparison target.
"""

from __future__ import annotations

import numpy as np

ROT_BLOCK = 256   # ConvRot card "Format": rotation group size 256
GROUP = 16        # ConvRot card "Format" / W4A8 card "Model Overview": group 16
LEVELS = 16       # 4-bit indices into a 16-level codebook
E4M3_MAX = 448.0  # largest finite e4m3fn value (1.75 * 2**8)

FIT_SEED = 42          # ConvRot card "Reproducing": --seed 42 pins the fit
FIT_SAMPLE_CAP = 2 ** 22
FIT_MAX_ITER = 500
FIT_TOL = 1e-12

__all__ = [
    "ROT_BLOCK", "GROUP", "LEVELS", "E4M3_MAX",
    "sylvester_hadamard", "rotate_blocks",
    "e4m3_encode", "e4m3_decode",
    "lloyd_max", "lloyd_residuals", "nearest_level",
    "pack_nibbles", "unpack_nibbles",
    "convert_weight", "dequant", "dequant_packed",
    "quantize_activations", "linear", "linear_packed", "round_to_bf16",
]


# --------------------------------------------------------------------------
# Rotation (ConvRot card "Format"; W4A8 card "Model Overview")
# --------------------------------------------------------------------------

def sylvester_hadamard(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (a power of two), int64 entries.

    H_1 = [1];  H_2m = [[H_m, H_m], [H_m, -H_m]].  Reading R2.
    """
    if n < 1 or n & (n - 1):
        raise ValueError("order must be a power of two")
    h = np.ones((1, 1), dtype=np.int64)
    while h.shape[0] < n:
        h = np.block([[h, h], [h, -h]])
    return h


def rotate_blocks(a: np.ndarray, block: int = ROT_BLOCK) -> np.ndarray:
    """a[..., K] @ blockdiag(H_block / sqrt(block)) in fp64.

    ConvRot card "Format": a group-wise Hadamard rotation with group size 256
    along the input dimension.  For block = 256 the scale is exactly 1/16, so
    the rotation is orthonormal (and symmetric: x @ H = H @ x per block).
    """
    a = np.asarray(a, dtype=np.float64)
    k = a.shape[-1]
    if k % block:
        raise ValueError(f"K={k} is not a multiple of the rotation block {block}")
    h = sylvester_hadamard(block).astype(np.float64) / np.sqrt(block)
    blocks = a.reshape(a.shape[:-1] + (k // block, block))
    return (blocks @ h).reshape(a.shape)


# --------------------------------------------------------------------------
# fp8 e4m3 (e4m3fn: bias 7, 3 mantissa bits, no infinities, 0x7F/0xFF = NaN)
# ConvRot card "Format": weight_s_rel is fp8_e4m3
# --------------------------------------------------------------------------

def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """uint8 e4m3fn codes -> fp64 values (exact)."""
    c = np.asarray(codes).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    mag = np.where((e == 15) & ((c & 0x7) == 7), np.nan, mag)
    return sign * mag


def e4m3_encode(values: np.ndarray) -> np.ndarray:
    """fp64 values -> uint8 e4m3fn codes, round half to even, saturating.

    Magnitudes >= 2**-6 are normal: a = t * 2**(E-3) with t in [8, 16] after
    rounding, code = (E + 7) * 8 + (t - 8) (t = 16 rolls into the next
    binade, which the code arithmetic handles).  Smaller magnitudes are
    subnormal multiples of 2**-9.  Magnitudes past 448 saturate to 448 (code
    0x7E); NaN maps to 0x7F; the sign bit is kept, so -0.0 maps to 0x80.
    """
    v = np.asarray(values, dtype=np.float64)
    neg = np.signbit(v)
    a = np.abs(v)
    nan = np.isnan(a)
    a = np.where(nan, 0.0, np.minimum(a, 2.0 * E4M3_MAX))  # inf -> large finite
    mant, ex = np.frexp(a)                  # a = mant * 2**ex, mant in [0.5, 1)
    e_unb = ex.astype(np.int64) - 1         # a in [2**e_unb, 2**(e_unb+1))
    normal = a >= 2.0 ** -6
    e_cl = np.where(normal, e_unb, -6)
    step = np.exp2(e_cl - 3.0)              # spacing of the grid in that binade
    t = np.rint(a / step).astype(np.int64)  # exact division by a power of two
    code = np.where(normal, (e_cl + 7) * 8 + (t - 8), t)
    code = np.minimum(code, 0x7E)           # saturate to 448
    code = np.where(neg, code | 0x80, code)   # the sign survives rounding to zero
    code = np.where(nan, 0x7F, code)
    return code.astype(np.uint8)


# --------------------------------------------------------------------------
# Lloyd-Max codebook (ConvRot card "Format"; W4A8 card "Model Overview")
# --------------------------------------------------------------------------

def _cells(sorted_s: np.ndarray, levels: np.ndarray) -> list[slice]:
    """Cells of a sorted sample: boundaries are level midpoints, and a value
    equal to a midpoint belongs to the lower cell (reading R7)."""
    mids = 0.5 * (levels[:-1] + levels[1:])
    ends = np.searchsorted(sorted_s, mids, side="right")
    starts = np.concatenate([[0], ends])
    stops = np.concatenate([ends, [sorted_s.size]])
    return [slice(int(a), int(b)) for a, b in zip(starts, stops)]


def lloyd_max(samples: np.ndarray, levels: int = LEVELS,
              max_iter: int = FIT_MAX_ITER, tol: float = FIT_TOL):
    """Lloyd-Max scalar quantiser fitted to a sample (reading R6).

    Returns (levels ascending in fp64, rounds taken).
    """
    s = np.sort(np.asarray(samples, dtype=np.float64).ravel())
    if s.size == 0:
        raise ValueError("empty sample")
    c = np.quantile(s, (np.arange(levels) + 0.5) / levels)
    rounds = 0
    for rounds in range(1, max_iter + 1):
        new = c.copy()
        for i, cell in enumerate(_cells(s, c)):
            if cell.stop > cell.start:
                new[i] = s[cell].mean()
        moved = np.max(np.abs(new - c))
        c = new
        if moved < tol:
            break
    return c, rounds


def lloyd_residuals(samples: np.ndarray, levels: np.ndarray):
    """Fixed-point residuals of a Lloyd-Max quantiser on a sample.

    Returns (max |level - mean of its cell| over non-empty cells,
    number of empty cells).  Boundaries are midpoints by construction.
    """
    s = np.sort(np.asarray(samples, dtype=np.float64).ravel())
    lv = np.asarray(levels, dtype=np.float64)
    worst, empty = 0.0, 0
    for i, cell in enumerate(_cells(s, lv)):
        if cell.stop > cell.start:
            worst = max(worst, abs(lv[i] - s[cell].mean()))
        else:
            empty += 1
    return worst, empty


def nearest_level(v: np.ndarray, cb32: np.ndarray) -> np.ndarray:
    """Index of the nearest stored level; midpoint ties take the lower index.

    ConvRot card "Format": the packed values are indices into the learned
    table.  Reading R7 for ties.
    """
    lv = np.asarray(cb32, dtype=np.float32).astype(np.float64)
    if np.any(np.diff(lv) <= 0):
        raise ValueError("codebook levels must be strictly ascending")
    mids = 0.5 * (lv[:-1] + lv[1:])      # exact: fp32 inputs, fp64 arithmetic
    return np.searchsorted(mids, np.asarray(v, dtype=np.float64), side="left").astype(np.uint8)


# --------------------------------------------------------------------------
# int4 packing (ConvRot card "Format": "packed int4 indices, two per byte")
# --------------------------------------------------------------------------

def pack_nibbles(idx: np.ndarray) -> np.ndarray:
    """[N, K] indices in 0..15 -> [N, K/2] bytes, even k in the low nibble (R7)."""
    idx = np.asarray(idx)
    if idx.shape[-1] % 2:
        raise ValueError("K must be even")
    if np.any((idx < 0) | (idx > 15)):
        raise ValueError("indices must be in 0..15")
    lo = idx[..., 0::2].astype(np.uint8)
    hi = idx[..., 1::2].astype(np.uint8)
    return (lo | (hi << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray) -> np.ndarray:
    """[N, K/2] bytes -> [N, K] indices (inverse of :func:`pack_nibbles`)."""
    p = np.asarray(packed, dtype=np.uint8)
    out = np.empty(p.shape[:-1] + (2 * p.shape[-1],), dtype=np.uint8)
    out[..., 0::2] = p & 0x0F
    out[..., 1::2] = p >> 4
    return out


# --------------------------------------------------------------------------
# Weight converter (ConvRot card "Format", "Reproducing"; W4A8 card
# "Model Overview")
# --------------------------------------------------------------------------

def convert_weight(w: np.ndarray, seed: int = FIT_SEED,
                   sample_cap: int = FIT_SAMPLE_CAP,
                   max_iter: int = FIT_MAX_ITER, tol: float = FIT_TOL,
                   codebook: np.ndarray | None = None) -> dict:
    """Quantise a weight W[N, K] (K % 256 == 0) to the asym_w4a8 format.

    Steps, in the pages' order: rotate (R2), row scale (R3), group scale (R4),
    normalise (R5), fit the codebook (R6), assign indices (R7).  Passing
    ``codebook`` skips the fit and assigns against the given fp32 levels.

    Returns a dict with ``idx`` uint8 [N, K] (0..15), ``packed`` uint8
    [N, K/2], ``s_rel`` uint8 e4m3 codes [N, K/16], ``s_ch`` fp32 [N],
    ``cb`` fp32 [16], ``fit_rounds`` and ``v`` (the normalised values).
    """
    w = np.asarray(w, dtype=np.float64)
    n, k = w.shape
    if k % ROT_BLOCK:
        raise ValueError(f"K={k} is not a multiple of {ROT_BLOCK}")
    r = rotate_blocks(w)                                        # R2
    s_ch = np.abs(r).max(axis=1).astype(np.float32)             # R3
    s_ch64 = s_ch.astype(np.float64)
    rg = r.reshape(n, k // GROUP, GROUP)
    gmax = np.abs(rg).max(axis=2)
    safe_ch = np.where(s_ch64 > 0, s_ch64, 1.0)[:, None]
    ratio = np.where(s_ch64[:, None] > 0, gmax / safe_ch, 0.0)
    s_rel = e4m3_encode(ratio)                                  # R4
    denom = e4m3_decode(s_rel) * s_ch64[:, None]                # exact product
    live = np.broadcast_to((denom > 0)[:, :, None], rg.shape)
    v = np.where(live, rg / np.where(denom > 0, denom, 1.0)[:, :, None], 0.0)   # R5
    if codebook is None:
        pool = v[live]
        if pool.size == 0:
            pool = np.zeros(1)
        if pool.size > sample_cap:
            rng = np.random.Generator(np.random.PCG64(seed))
            pool = rng.choice(pool, size=sample_cap, replace=False)
        levels, rounds = lloyd_max(pool, LEVELS, max_iter, tol)   # R6
        cb = levels.astype(np.float32)
    else:
        cb, rounds = np.asarray(codebook, dtype=np.float32), 0
    v = v.reshape(n, k)
    idx = nearest_level(v, cb)                                  # R7
    return {"idx": idx, "packed": pack_nibbles(idx), "s_rel": s_rel,
            "s_ch": s_ch, "cb": cb, "fit_rounds": rounds, "v": v}


# --------------------------------------------------------------------------
# Dequantisation (ConvRot card "Format": three tiers of scaling)
# --------------------------------------------------------------------------

def dequant(idx: np.ndarray, s_rel: np.ndarray, s_ch: np.ndarray, cb: np.ndarray,
            rows: np.ndarray | None = None) -> np.ndarray:
    """W_hat[n,k] = fp32(fp32(cb[idx] * s_rel) * s_channel), rotated basis.

    Each product of an fp32 value and an e4m3 / fp32 value is exact in fp64,
    so rounding it once to fp32 gives the correctly rounded fp32 product.
    ``rows`` restricts the result to those output rows.
    """
    idx = np.asarray(idx)
    s_rel = np.asarray(s_rel)
    s_ch = np.asarray(s_ch, dtype=np.float32)
    if rows is not None:
        idx, s_rel, s_ch = idx[rows], s_rel[rows], s_ch[rows]
    cbv = np.asarray(cb, dtype=np.float32).astype(np.float64)[idx.astype(np.int64)]
    sr = np.repeat(e4m3_decode(s_rel), GROUP, axis=-1)
    t = (cbv * sr).astype(np.float32)
    return (t.astype(np.float64) * s_ch.astype(np.float64)[:, None]).astype(np.float32)


def dequant_packed(packed, s_rel, s_ch, cb, rows=None) -> np.ndarray:
    """:func:`dequant` on packed [N, K/2] indices."""
    packed = np.asarray(packed)
    if rows is not None:
        packed, s_rel, s_ch = packed[rows], np.asarray(s_rel)[rows], np.asarray(s_ch)[rows]
    return dequant(unpack_nibbles(packed), s_rel, s_ch, cb)


# --------------------------------------------------------------------------
# Activations (W4A8 card "Model Overview": int8 activations; reading R8)
# --------------------------------------------------------------------------

def quantize_activations(x: np.ndarray):
    """Rotate bf16-valued activations x[M, K] and quantise them per token.

    Returns (q int8 [M, K], s_x fp32 [M], x_rot fp64 [M, K]).
    """
    x_rot = rotate_blocks(np.asarray(x, dtype=np.float64))
    xr32 = x_rot.astype(np.float32)
    amax = np.abs(xr32).max(axis=-1)
    s_x = (amax / np.float32(127.0)).astype(np.float32)
    safe = np.where(s_x > 0, s_x, np.float32(1.0)).astype(np.float32)
    quot = (xr32 / safe[:, None]).astype(np.float32)
    q = np.where(s_x[:, None] > 0, np.clip(np.rint(quot), -127, 127), 0).astype(np.int8)
    return q, s_x, x_rot


# --------------------------------------------------------------------------
# The linear layer (reading R10)
# --------------------------------------------------------------------------

def linear(x, idx, s_rel, s_ch, cb, rows=None) -> np.ndarray:
    """Unrounded fp64 y[M, N] = s_x[m] * sum_k q[m,k] * W_hat[n,k].

    ``rows`` (output columns n) restricts the result to those columns.
    """
    q, s_x, _ = quantize_activations(x)
    w_hat = dequant(idx, s_rel, s_ch, cb, rows=rows).astype(np.float64)
    acc = q.astype(np.float64) @ w_hat.T
    return s_x.astype(np.float64)[:, None] * acc


def linear_packed(x, packed, s_rel, s_ch, cb, rows=None) -> np.ndarray:
    """:func:`linear` on packed [N, K/2] indices."""
    packed = np.asarray(packed)
    if rows is not None:
        return linear(x, unpack_nibbles(packed[rows]), np.asarray(s_rel)[rows],
                      np.asarray(s_ch)[rows], cb)
    return linear(x, unpack_nibbles(packed), s_rel, s_ch, cb)


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Nearest bfloat16 value (8 significant bits, round half to even), as fp64.

    Used only to report the bf16-rounded oracle output; subnormal bf16 values
    are not needed at these magnitudes and are not handled specially.
    """
    a = np.asarray(a, dtype=np.float64)
    mant, ex = np.frexp(a)
    step = np.exp2(ex.astype(np.float64) - 8.0)
    out = np.rint(a / step) * step
    return np.where(a == 0, 0.0, out)
