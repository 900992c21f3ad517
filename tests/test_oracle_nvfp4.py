"""Pins of the NVFP4 oracle (oracle/nvfp4_ref.py) against what the NVFP4
runbook ("Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på
Blackwell-GPU:er", section "Vad NVFP4 är, och hur det skiljer sig från FP8
och från INT8/AWQ") and arithmetic fix: E2M1 values, 16-value blocks with an
e4m3 scale, one fp32 scalar per tensor.  Hand-computed cases, closed forms
and brute force -- never the oracle's own formulas retyped."""

import itertools

import numpy as np
import pytest

from oracle import nvfp4_ref as N
from oracle import w4a8_ref as O

# E2M1 = 1 sign, 2 exponent, 1 mantissa bit (the runbook); with bias 1 the
# positive codes 0..7 are these values (OCP microscaling E2M1), typed by hand.
E2M1_TABLE = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def test_e2m1_decode_table():
    got = N.e2m1_decode(np.arange(16))
    assert list(got[:8]) == E2M1_TABLE
    assert list(-got[8:]) == E2M1_TABLE
    assert np.all(np.signbit(got[8:]))            # code 8 is -0


def test_e2m1_encode_round_trips_every_value():
    for c, v in enumerate(E2M1_TABLE):
        assert N.e2m1_encode(np.array([v]))[0] == c
        assert N.e2m1_encode(np.array([-v]))[0] == c | 8


@pytest.mark.parametrize("v,code", [
    (0.25, 0), (0.75, 2), (1.25, 2), (1.75, 4), (2.5, 4), (3.5, 6), (5.0, 6),   # ties: even code
    (0.2499, 0), (0.2501, 1), (5.0001, 7), (4.9999, 6),                          # either side of a tie
    (6.0, 7), (7.0, 7), (1e30, 7),                                               # saturation
    (-0.1, 8), (-2.6, 13),
])
def test_e2m1_encode_hand_cases(v, code):
    assert N.e2m1_encode(np.array([v]))[0] == code


def test_e2m1_encode_is_nearest_brute_force():
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.uniform(-7, 7, 20000), rng.normal(0, 0.3, 5000)])
    got = np.abs(v - N.e2m1_decode(N.e2m1_encode(v)))
    grid = np.array(E2M1_TABLE + [-x for x in E2M1_TABLE])
    best = np.abs(np.clip(v, -6, 6)[:, None] - grid[None, :]).min(axis=1) + np.maximum(np.abs(v) - 6, 0)
    assert np.allclose(got, best, rtol=0, atol=1e-12)


def test_pack_nibble_order():
    codes = np.array([[1, 2, 3, 4, 15, 0]], dtype=np.uint8)
    assert list(N.pack_codes(codes)[0]) == [0x21, 0x43, 0x0F]
    assert np.array_equal(N.unpack_codes(N.pack_codes(codes)), codes)


def test_quantize_worked_example_on_the_grid():
    """A row that is the E2M1 grid divided by 8: amax = 0.75, so the block
    scale is t = 0.75 / (6 g) with g = 0.75 / 2688, i.e. 448 (e4m3 code
    0x7E), the effective scale 448 g = 1/8, and every value sits exactly on
    a grid point: the codes are the grid's own codes."""
    vals = [0, 0.5, 1, 1.5, 2, 3, 4, 6, -6, -4, -3, -2, -1.5, -1, -0.5, 0]
    x = np.array([vals], dtype=np.float64) / 8.0
    codes, s, g = N.quantize_rows(x, rotate=False)
    assert list(codes[0]) == [0, 1, 2, 3, 4, 5, 6, 7, 15, 14, 13, 12, 11, 10, 9, 0]
    assert s[0, 0] == 0x7E
    assert g[0] == np.float32(np.float32(0.75) / np.float32(2688.0))


def test_quantize_blocks_are_16_wide():
    """Two neighbouring 16-blocks a factor 64 apart get e4m3 scales whose
    values are a factor 64 apart (a 32-wide block would share one)."""
    x = np.zeros((1, 32))
    x[0, :16] = np.linspace(-1, 1, 16)
    x[0, 16:] = np.linspace(-1, 1, 16) / 64.0
    codes, s, g = N.quantize_rows(x, rotate=False)
    d = O.e4m3_decode(s[0])
    assert d[0] == 448.0 and d[1] == 7.0                 # 448 / 64
    assert np.array_equal(codes[0, :16], codes[0, 16:])


def test_quantize_zero_and_tiny_rows():
    x = np.zeros((3, 32))
    x[1, 5] = 1e-3
    x[2, :16] = 1.0
    codes, s, g = N.quantize_rows(x, rotate=False)
    assert g[0] == 0 and not codes[0].any() and not s[0].any()
    # one nonzero value: it gets the top code, the other block scales are 0
    assert codes[1, 5] == 7 and s[1, 0] == 0x7E and s[1, 1] == 0 and not codes[1, 16:].any()
    # a flat block: every value is the block maximum -> code 7 (6 x 1/6)
    assert np.all(codes[2, :16] == 7) and s[2, 1] == 0


def test_quantize_per_tensor_scalar():
    """Weights: one g for the whole tensor (the runbook); a row 100x smaller
    than the largest gets block scales 100x smaller, not its own g."""
    rng = np.random.default_rng(5)
    w = rng.normal(0, 1, (4, 64))
    w[1] /= 100.0
    codes, s, g = N.quantize_rows(w, rotate=False, per_row=False)
    assert np.all(g == g[0])
    assert g[0] == np.float32(np.float32(np.abs(w).max()) / np.float32(2688.0))
    ratio = O.e4m3_decode(s[0]).max() / O.e4m3_decode(s[1]).max()
    assert 60 < ratio < 160


def test_quantize_error_bound_brute_force():
    """Every value lands within one unit of the block's effective scale S
    (the widest E2M1 gap is 2, between 4 and 6, so half a gap is 1 S; the
    e4m3 rounding of the block scale can push the block maximum up to 6 x
    (1 + 1/16) / (1 - 1/16), which saturates by < 1 S), and its code is the
    nearest grid point of x / S found by search."""
    rng = np.random.default_rng(11)
    x = rng.normal(0, 1, (6, 256)) * np.exp(rng.normal(0, 2, (6, 1)))
    x[2, 17] = 40.0
    codes, s, g = N.quantize_rows(x, rotate=False)
    xr = x.astype(np.float32).astype(np.float64)
    big_s = (O.e4m3_decode(s).astype(np.float32) * g[:, None]).astype(np.float32).astype(np.float64)
    bs = np.repeat(big_s, 16, axis=1)
    deq = N.e2m1_decode(codes) * bs
    assert np.all(np.abs(xr - deq) <= bs * 1.0 + 1e-30)
    grid = np.array(E2M1_TABLE + [-v for v in E2M1_TABLE])
    q = (xr / bs)
    nearest = np.abs(q[..., None] - grid).min(axis=-1)
    assert np.allclose(np.abs(q - N.e2m1_decode(codes)), nearest, atol=1e-6)


def test_quantize_largest_block_gets_top_scale():
    """g = amax / 2688 puts the block holding the tensor's maximum at the
    largest e4m3 scale (448) and the maximum itself at code +-6."""
    rng = np.random.default_rng(2)
    for _ in range(20):
        x = rng.normal(0, 1, (3, 128)) * rng.uniform(1e-3, 1e3)
        codes, s, g = N.quantize_rows(x, rotate=False)
        for r in range(3):
            i = int(np.argmax(np.abs(x[r])))
            assert s[r, i // 16] == 0x7E
            assert codes[r, i] & 7 == 7


def test_quantize_rotates_like_the_codebook_path():
    """rotate=True quantises rotate_blocks(x) (the codebook path's basis):
    a row that rotates to a spike keeps only the spike."""
    import scipy.linalg
    x = np.zeros((1, 256))
    x[0] = scipy.linalg.hadamard(256)[9] * (3.0 / 16.0)   # rotates to 3 at k = 9
    codes, s, g = N.quantize_rows(x, rotate=True)
    assert codes[0, 9] == 7 and np.count_nonzero(codes[0] & 7) == 1


def test_gemm_brute_force_tiny():
    """Reading N6 on a 2 x 3 x 32 case with loops over hand-decoded values."""
    rng = np.random.default_rng(7)
    cx = rng.integers(0, 16, (2, 32)).astype(np.uint8)
    cw = rng.integers(0, 16, (3, 32)).astype(np.uint8)
    sx = rng.integers(0x30, 0x48, (2, 2)).astype(np.uint8)
    sw = rng.integers(0x30, 0x48, (3, 2)).astype(np.uint8)
    gx = np.array([0.5, 3.0], dtype=np.float32)
    gw = np.array([0.25, 0.25, 0.25], dtype=np.float32)

    def val(c):
        v = E2M1_TABLE[c & 7]
        return -v if c & 8 else v

    def e4m3(c):   # positive normal codes only in this test
        e, m = int(c) >> 3, int(c) & 7
        return (1 + m / 8.0) * 2.0 ** (e - 7)

    want = np.zeros((2, 3))
    for m, n in itertools.product(range(2), range(3)):
        acc = 0.0
        for k in range(32):
            acc += val(cx[m, k]) * e4m3(sx[m, k // 16]) * val(cw[n, k]) * e4m3(sw[n, k // 16])
        want[m, n] = acc * float(gx[m]) * float(gw[n])
    got = N.gemm(cx, sx, gx, cw, sw, gw)
    assert np.allclose(got, want, rtol=1e-14, atol=0)


def test_linear_exact_on_representable_inputs():
    """x and W already on the NVFP4 grid (every block holding a 6, so every
    block scale is 448 and the effective scale is 448 g; rotate=False):
    the codes are the grid's own, and the layer equals the exact product up
    to the fp32 rounding of the tensor scalar g = amax / 2688."""
    xrow = [6, 4, -3, 2, 1.5, -1, 0.5, 0, 6, 0, 0, 0, -6, 2, 1, 3]
    wrow = [1, -1, 2, 0.5, -6, 4, 3, 0, 1.5, 1, 2, 6, -2, 0, 0, 1]
    xv = np.array([xrow * 2]) / 64.0
    wv = np.array([wrow * 2, [6] * 32]) / 16.0
    cx, _, _ = N.quantize_rows(xv, rotate=False)
    cw, _, _ = N.quantize_rows(wv, rotate=False, per_row=False)
    assert np.array_equal(N.e2m1_decode(cx[0]), np.array(xrow * 2, dtype=float))
    assert np.array_equal(N.e2m1_decode(cw[1]), np.full(32, 6.0))
    y = N.linear(xv, wv, rotate=False)
    assert np.allclose(y, xv @ wv.T, rtol=1e-6, atol=0)


def test_linear_error_is_nvfp4_sized():
    """On Gaussian data the W4A4 layer is a few percent off the fp64 product
    (4-bit floats with 16-value blocks); the int8-activation codebook layer
    is well under that on the same inputs."""
    rng = np.random.default_rng(9)
    x = rng.normal(0, 1, (8, 512))
    w = rng.normal(0, 0.02, (64, 512))
    ref = x @ w.T
    y = N.linear(x, w)
    rel = np.linalg.norm(y - ref) / np.linalg.norm(ref)
    assert 0.03 < rel < 0.2
