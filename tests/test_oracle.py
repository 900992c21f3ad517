"""Pins for the CPU oracle: each test checks it against something other than
itself -- a library routine, a closed form, a published table, brute force
written another way, or an exact special case -- so that a dropped term, a
wrong sign or index, or a transposed operand fails at least one of them.

Runs without a GPU.
"""

import os
import struct

import numpy as np
import pytest
import scipy.linalg
import torch
from scipy.stats import norm

import oracle as O
import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(v: float) -> float:
    """Round a Python float to fp32 (C cast, round to nearest even)."""
    return struct.unpack("f", struct.pack("f", v))[0]


# ---------------------------------------------------------------- rotation

@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_hadamard_matches_scipy(n):
    h = O.sylvester_hadamard(n)
    assert np.array_equal(h, scipy.linalg.hadamard(n))
    assert np.array_equal(h @ h.T, n * np.eye(n, dtype=np.int64))


def test_rotation_preserves_products():
    """H/16 is orthonormal, so rotating both sides leaves x W^T unchanged."""
    rng = np.random.default_rng(1)
    x = rng.normal(size=(5, 768))
    w = rng.normal(size=(7, 768))
    got = O.rotate_blocks(x) @ O.rotate_blocks(w).T
    assert np.allclose(got, x @ w.T, rtol=0, atol=1e-11 * np.abs(x @ w.T).max())


def test_rotation_spike_is_flat_hadamard_row():
    """e_i in block b rotates to the scipy Hadamard row i / 16 in block b only."""
    hs = scipy.linalg.hadamard(256) / 16.0
    for b, i in [(0, 0), (1, 37), (2, 255)]:
        x = np.zeros((1, 768))
        x[0, 256 * b + i] = 1.0
        r = O.rotate_blocks(x)[0]
        expect = np.zeros(768)
        expect[256 * b: 256 * (b + 1)] = hs[i]
        assert np.array_equal(r, expect)


def test_rotation_is_an_involution():
    rng = np.random.default_rng(2)
    x = rng.normal(size=(3, 512))
    assert np.allclose(O.rotate_blocks(O.rotate_blocks(x)), x, atol=1e-13)


def test_rotation_rejects_ragged_k():
    with pytest.raises(ValueError):
        O.rotate_blocks(np.zeros((1, 300)))


# ---------------------------------------------------------------- e4m3

def test_e4m3_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(got), np.isnan(ref))
    ok = ~np.isnan(ref)
    assert np.array_equal(got[ok], ref[ok])


def test_e4m3_encode_matches_torch_cast():
    # every representable value, every midpoint between neighbours, and a
    # dense random sweep over [0, 448], positive and negative
    vals = O.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    mids = 0.5 * (vals[:-1] + vals[1:])
    rng = np.random.default_rng(3)
    sweep = np.concatenate([vals, mids, rng.uniform(0, 448, 20000),
                            np.exp2(rng.uniform(-12, 8.8, 20000))])
    sweep = sweep[sweep <= 448.0]
    sweep = np.concatenate([sweep, -sweep])
    ref = torch.from_numpy(sweep).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = O.e4m3_encode(sweep)
    assert np.array_equal(got, ref)


def test_e4m3_encode_saturates_and_flags_nan():
    assert O.e4m3_encode(np.array([1000.0, np.inf, 465.0]))[0] == 0x7E
    assert O.e4m3_encode(np.array([np.inf]))[0] == 0x7E
    assert O.e4m3_encode(np.array([np.nan]))[0] == 0x7F
    assert O.e4m3_decode(np.array([0x7E]))[0] == 448.0


# ---------------------------------------------------------------- Lloyd-Max

def _analytic_gaussian_lloyd(levels):
    """Continuous Lloyd-Max for N(0,1) with analytic cell centroids
    E[X | a < X < b] = (pdf(a) - pdf(b)) / (cdf(b) - cdf(a))."""
    c = norm.ppf((np.arange(levels) + 0.5) / levels)
    for _ in range(50000):
        b = np.concatenate([[-np.inf], 0.5 * (c[:-1] + c[1:]), [np.inf]])
        new = (norm.pdf(b[:-1]) - norm.pdf(b[1:])) / (norm.cdf(b[1:]) - norm.cdf(b[:-1]))
        if np.max(np.abs(new - c)) < 1e-14:
            return new
        c = new
    return c


def _max_table():
    rows = [ln.split() for ln in open(os.path.join(GOLDEN, "lloyd_max_gaussian16.txt"))
            if ln.strip() and not ln.startswith("#")]
    levels = np.array([float(r[1]) for r in rows if r[0] != "mse"])
    return np.concatenate([-levels[::-1], levels])


def test_analytic_gaussian_matches_published_table():
    assert np.allclose(_analytic_gaussian_lloyd(16), _max_table(), atol=6e-4)


def test_lloyd_16_levels_on_gaussian_sample_matches_table():
    s = np.random.default_rng(4).normal(size=2 ** 21)
    lv, rounds = O.lloyd_max(s, 16, max_iter=2000, tol=1e-10)
    assert np.allclose(lv, _max_table(), atol=0.02)
    assert np.allclose(lv, _analytic_gaussian_lloyd(16), atol=0.02)


def test_lloyd_two_levels_on_gaussian_is_closed_form():
    """2-level MMSE quantiser of N(0, s^2): levels = +-s * sqrt(2/pi)."""
    sigma = 0.7
    s = np.random.default_rng(5).normal(0, sigma, size=2 ** 21)
    s = np.concatenate([s, -s])                # exactly symmetric sample
    lv, _ = O.lloyd_max(s, 2)
    assert abs(lv[1] + lv[0]) < 1e-12
    assert abs(lv[1] - sigma * np.sqrt(2 / np.pi)) < 2e-3


@pytest.mark.parametrize("levels", [2, 4, 16])
def test_lloyd_uniform_grid_gives_cell_centres(levels):
    """Uniform on [0, 1): the optimum is the centres (2i + 1) / (2L)."""
    n = 1 << 16
    s = (np.arange(n) + 0.5) / n
    lv, _ = O.lloyd_max(s, levels)
    assert np.allclose(lv, (2 * np.arange(levels) + 1) / (2 * levels), atol=2.0 / n)


def test_lloyd_fixed_point_conditions():
    rng = np.random.default_rng(6)
    s = np.concatenate([rng.normal(size=40000), 5 * rng.standard_t(3, size=2000)])
    lv, rounds = O.lloyd_max(s, 16)
    assert rounds < 500
    worst, empty = O.lloyd_residuals(s, lv)
    assert empty == 0 and worst < 1e-9
    assert np.all(np.diff(lv) > 0)


def test_lloyd_residuals_hand_computed_non_fixed_point():
    # Worked by hand.  Two levels (-1, 3): the midpoint is 1, and the sample
    # value 1 sits on it, so it belongs to the lower cell.  Lower cell
    # {-3, -2, -1, 1}: mean -5/4, residual |-1 - (-5/4)| = 1/4.  Upper cell
    # {2, 4}: mean 3, residual 0.  (Had the tie gone up, the lower cell's mean
    # would be -2 and the residual 1.)
    s = np.array([4.0, -1.0, 2.0, -3.0, 1.0, -2.0])   # unsorted on purpose
    worst, empty = O.lloyd_residuals(s, np.array([-1.0, 3.0]))
    assert worst == 0.25 and empty == 0
    # A sign error (level + mean) or a cell taken on the wrong side of the
    # midpoint would show here: upper level 2 against a cell mean of 3.
    worst, empty = O.lloyd_residuals(s, np.array([-1.0, 2.0]))
    # midpoint 0.5: lower {-3, -2, -1} mean -2 -> 1; upper {1, 2, 4} mean 7/3 -> 1/3
    assert worst == 1.0 and empty == 0


def test_lloyd_residuals_hand_computed_empty_cell():
    # Three levels (0.5, 2, 5): midpoints 1.25 and 3.5.  Cells {0, 0.25, 0.5}
    # (mean 0.25, residual 0.25), {} (empty), {5, 5.5, 6} (mean 5.5,
    # residual 0.5).  All values are exact in binary.
    s = np.array([0.0, 0.25, 0.5, 5.0, 5.5, 6.0])
    worst, empty = O.lloyd_residuals(s, np.array([0.5, 2.0, 5.0]))
    assert worst == 0.5 and empty == 1
    # the same sample at its own fixed point: levels = cell means, one cell empty
    worst, empty = O.lloyd_residuals(s, np.array([0.25, 2.0, 5.5]))
    assert worst == 0.0 and empty == 1
    # The fit starts at the 1/6, 1/2, 5/6 quantiles (linear interpolation:
    # 5/24, 11/4, 67/12); the middle cell (1.479.., 4.166..] is empty, so one
    # round gives (1/4, 11/4, 11/2) with the empty cell's level kept, and
    # that is a fixed point with one empty cell.
    lv, rounds = O.lloyd_max(s, 3, max_iter=1, tol=0.0)
    assert rounds == 1 and np.array_equal(lv, [0.25, 2.75, 5.5])
    assert O.lloyd_residuals(s, lv) == (0.0, 1)


def test_lloyd_empty_cell_keeps_level():
    # two far clusters and 16 levels: quantile init puts levels inside the
    # clusters, so no cell is empty -- but a sample of identical values leaves
    # all but one cell empty, and those levels must not move
    s = np.full(100, 0.25)
    lv, _ = O.lloyd_max(s, 4)
    assert np.allclose(lv, 0.25)


# ---------------------------------------------------------------- nearest level / packing

def test_nearest_level_matches_argmin_and_breaks_ties_low():
    cb = np.array([-1.0, -0.3, 0.1, 0.8], dtype=np.float32)
    rng = np.random.default_rng(7)
    v = rng.uniform(-1.5, 1.5, 10000)
    brute = np.argmin(np.abs(v[:, None] - cb.astype(np.float64)[None, :]), axis=1)
    assert np.array_equal(O.nearest_level(v, cb), brute)
    mids = 0.5 * (cb[:-1].astype(np.float64) + cb[1:])
    assert np.array_equal(O.nearest_level(mids, cb), np.arange(3))


def test_pack_hand_set_bytes_and_round_trip():
    idx = np.array([[1, 2, 3, 4, 15, 0, 0, 15]])
    p = O.pack_nibbles(idx)
    assert p.tolist() == [[0x21, 0x43, 0x0F, 0xF0]]
    rng = np.random.default_rng(8)
    idx = rng.integers(0, 16, size=(9, 64))
    assert np.array_equal(O.unpack_nibbles(O.pack_nibbles(idx)), idx)
    with pytest.raises(ValueError):
        O.pack_nibbles(np.array([[16, 0]]))


# ---------------------------------------------------------------- converter

@pytest.fixture(scope="module")
def toy():
    w = synth.weights(256, 512, synth.rng_for(0, 0, "weight"))
    return w, O.convert_weight(w)


def test_converter_scales_brute_force(toy):
    w, c = toy
    hs = scipy.linalg.hadamard(256) / 16.0
    r = np.concatenate([w[:, :256].astype(np.float64) @ hs, w[:, 256:].astype(np.float64) @ hs], axis=1)
    assert np.array_equal(c["s_ch"], np.abs(r).max(axis=1).astype(np.float32))
    sr = O.e4m3_decode(c["s_rel"])
    for n in range(0, 256, 17):
        kmax = int(np.argmax(np.abs(r[n])))
        assert c["s_rel"][n, kmax // 16] == 0x38          # e4m3 code of 1.0
        for g in range(32):
            grp = r[n, 16 * g: 16 * g + 16]
            if sr[n, g] >= 2.0 ** -6:                       # normal e4m3 ratio
                vmax = np.abs(grp).max() / (sr[n, g] * float(c["s_ch"][n]))
                assert 1 / (1 + 2 ** -4) - 1e-12 <= vmax <= 1 / (1 - 2 ** -4) + 1e-12


def test_converter_fit_is_a_fixed_point(toy):
    w, c = toy
    live = np.repeat(O.e4m3_decode(c["s_rel"]), 16, axis=1) > 0
    lv, _ = O.lloyd_max(c["v"][live])
    assert np.array_equal(lv.astype(np.float32), c["cb"])
    worst, empty = O.lloyd_residuals(c["v"][live], lv)
    assert empty == 0 and worst < 1e-9


def test_converter_indices_are_nearest(toy):
    w, c = toy
    cb = c["cb"].astype(np.float64)
    d = np.abs(c["v"][..., None] - cb)
    assert np.all(np.take_along_axis(d, c["idx"][..., None].astype(np.int64), -1)[..., 0]
                  <= d.min(axis=-1) + 0.0)


def test_converter_zero_row_and_given_codebook():
    w = synth.weights(32, 256, synth.rng_for(9, 0, "weight"))
    w[3] = 0.0
    c = O.convert_weight(w)
    assert c["s_ch"][3] == 0 and np.all(c["s_rel"][3] == 0)
    assert np.all(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])[3] == 0)
    c2 = O.convert_weight(w, codebook=c["cb"])
    assert np.array_equal(c2["idx"], c["idx"]) and np.array_equal(c2["s_rel"], c["s_rel"])


def test_converter_sampling_is_seeded():
    w = synth.weights(64, 512, synth.rng_for(10, 0, "weight"))
    a = O.convert_weight(w, sample_cap=5000)
    b = O.convert_weight(w, sample_cap=5000)
    c = O.convert_weight(w, sample_cap=5000, seed=7)
    assert np.array_equal(a["cb"], b["cb"]) and not np.array_equal(a["cb"], c["cb"])


# ---------------------------------------------------------------- dequant

def test_dequant_brute_force_triple_loop(toy):
    w, c = toy
    rows = [0, 1, 100, 255]
    got = O.dequant_packed(c["packed"], c["s_rel"], c["s_ch"], c["cb"])
    srel = torch.from_numpy(c["s_rel"].copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for n in rows:
        for k in range(512):
            byte = int(c["packed"][n, k // 2])
            i = (byte >> 4) if (k & 1) else (byte & 15)
            t = f32(float(c["cb"][i]) * float(srel[n, k // 16]))
            assert got[n, k] == np.float32(f32(t * float(c["s_ch"][n])))


# ---------------------------------------------------------------- activations

def test_activation_quant_brute_force():
    bits, x, _ = synth.activations(3, 512, synth.rng_for(0, 0, "act"), 2)
    q, s_x, x_rot = O.quantize_activations(x)
    hs = scipy.linalg.hadamard(256) / 16.0
    for m in range(3):
        xr = np.concatenate([x[m, :256].astype(np.float64) @ hs, x[m, 256:].astype(np.float64) @ hs])
        xr32 = [f32(v) for v in xr]
        amax = max(abs(v) for v in xr32)
        s = np.float32(np.float32(amax) / np.float32(127))
        assert s_x[m] == s
        for k in range(512):
            quot = float(np.float32(np.float32(xr32[k]) / s))
            assert q[m, k] == max(-127, min(127, round(quot)))   # Python round: half to even


def test_activation_quant_special_cases():
    x = np.zeros((3, 256), dtype=np.float32)
    x[1] = scipy.linalg.hadamard(256)[5] * (3.0 / 16.0)  # rotates to a spike 3 at 5
    x[2, 7] = -2.0                                        # rotates to a flat row
    q, s_x, _ = O.quantize_activations(x)
    assert s_x[0] == 0 and np.all(q[0] == 0)
    assert s_x[1] == np.float32(3.0) / np.float32(127)
    assert q[1, 5] == 127 and np.count_nonzero(q[1]) == 1
    assert np.array_equal(np.abs(q[2]), np.full(256, 127))
    assert np.array_equal(np.sign(q[2]), -scipy.linalg.hadamard(256)[7])


# ---------------------------------------------------------------- linear

def test_linear_exact_integer_case():
    """Integer levels, unit scales, and activations built so that x_rot is a
    spike q_b at position i_b of each block: y[n] = sum_b q_b cb[idx[n, 256b + i_b]]."""
    rng = np.random.default_rng(11)
    n, k = 48, 768
    cb = np.arange(-8, 8).astype(np.float32)
    idx = rng.integers(0, 16, size=(n, k))
    s_rel = np.full((n, k // 16), 0x38, dtype=np.uint8)
    s_ch = np.ones(n, dtype=np.float32)
    hs = scipy.linalg.hadamard(256)
    qb, ib = [127, -45, 3], [9, 200, 0]
    x = np.concatenate([hs[i] * (q / 16.0) for q, i in zip(qb, ib)])[None, :].astype(np.float32)
    y = O.linear(x, idx, s_rel, s_ch, cb)
    expect = [sum(q * float(cb[idx[r, 256 * b + i]]) for b, (q, i) in enumerate(zip(qb, ib)))
              for r in range(n)]
    assert np.array_equal(y[0], np.array(expect))


def test_linear_equals_unrotated_product(toy):
    """Undoing the rotation on both quantised operands gives the same y."""
    w, c = toy
    bits, x, _ = synth.activations(4, 512, synth.rng_for(0, 0, "act"), 2)
    y = O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
    q, s_x, _ = O.quantize_activations(x)
    w_hat = O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"]).astype(np.float64)
    hs = scipy.linalg.hadamard(256) / 16.0
    unrot = lambda a: np.concatenate([a[:, :256] @ hs, a[:, 256:] @ hs], axis=1)
    x_deq = unrot(q.astype(np.float64) * s_x.astype(np.float64)[:, None])
    assert np.allclose(unrot(w_hat) @ x_deq.T, y.T, rtol=1e-12, atol=1e-12 * np.abs(y).max())


def test_linear_quality_band(toy):
    """W4A8 card "Accuracy": forward error against full precision is about
    1 %.  On these synthetic weights the relative mean squared error lands
    near that figure (4-bit, 16 levels: the Gaussian Lloyd-Max floor alone is
    0.95 % of the variance)."""
    w, c = toy
    bits, x, _ = synth.activations(4, 512, synth.rng_for(0, 0, "act"), 2)
    y = O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
    yt = x.astype(np.float64) @ w.astype(np.float64).T
    rel_mse = np.sum((y - yt) ** 2) / np.sum(yt ** 2)
    assert 1e-3 < rel_mse < 3e-2


def test_linear_rows_subset_matches_full(toy):
    w, c = toy
    bits, x, _ = synth.activations(2, 512, synth.rng_for(0, 1, "act"), 2)
    full = O.linear_packed(x, c["packed"], c["s_rel"], c["s_ch"], c["cb"])
    rows = np.array([3, 77, 255])
    part = O.linear_packed(x, c["packed"], c["s_rel"], c["s_ch"], c["cb"], rows=rows)
    assert np.array_equal(part, full[:, rows])


def test_round_to_bf16_matches_torch():
    a = np.random.default_rng(12).normal(size=5000) * 10.0
    ref = torch.from_numpy(a.astype(np.float32)).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(a.astype(np.float32)), ref)


# ---------------------------------------------------------------- regression fixture

def test_toy_fixture_unchanged():
    """The toy layer's converted tensors and output match the committed
    fixture written by tests/golden/make_golden.py (oracle only)."""
    import json
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(GOLDEN, "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    want = json.load(open(os.path.join(GOLDEN, "toy_oracle.json")))
    got = json.loads(json.dumps(mg.toy()))
    assert got == want
