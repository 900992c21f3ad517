"""Parity of the GPU weight converter (w4a8_convert_weight) against the
CPU oracle's converter.

Bars:
  * given the same codebook: packed indices, e4m3 group scales and fp32 row
    scales bit-exact;
  * fitting the codebook (Lloyd-Max, same sample): the fp32 levels equal to
    the oracle's within one fp32 ulp (the cell means are summed in another
    order), the fixed-point conditions hold on the sample, and where the
    levels are equal every output is bit-exact.
Inputs include an all-zero row, a row whose outlier drives most group
scales to e4m3 subnormals or zero, negative and positive outliers, and
shapes with several 256-blocks and row counts that are not multiples of 32.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def weights_with_edges(n, k, seed):
    w = synth.weights(n, k, synth.rng_for(seed, 0, "weight"))
    w[1] = 0.0                                  # all-zero row: s_ch = 0, every group dead
    w[2, 5] = 3.0e3                             # one huge value: the row's other groups go subnormal / zero
    w[3, : k // 2] = 0.0                        # half a row zero: dead groups mixed with live ones
    w[4] *= -1.0
    return w.astype(np.float32)


def gpu_convert(lib, w, **kw):
    out = lib.convert_weight(torch.from_numpy(w).cuda(), **kw)
    return {key: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for key, v in out.items()}


@pytest.mark.parametrize("n,k", [(48, 256), (592, 768), (80, 2048), (16, 32768)])
def test_convert_given_codebook_bit_exact(lib, n, k):
    w = weights_with_edges(n, k, 30 + k // 256)
    ref = O.convert_weight(w, sample_cap=2 ** 16)
    got = gpu_convert(lib, w, codebook=torch.from_numpy(ref["cb"]).cuda())
    assert np.array_equal(got["s_ch"].view(np.uint32), ref["s_ch"].view(np.uint32))
    assert np.array_equal(got["s_rel"], ref["s_rel"])
    assert np.array_equal(got["packed"], ref["packed"])
    assert np.array_equal(got["cb"].view(np.uint32), ref["cb"].view(np.uint32))
    assert int(got["fit_rounds"][0]) == 0
    assert lib.get_device_error() == 0


def check_fit(got, ref, pool):
    ulp = np.spacing(np.abs(ref["cb"]).astype(np.float32))
    assert np.all(np.abs(got["cb"].astype(np.float64) - ref["cb"].astype(np.float64)) <= ulp)
    worst, empty = O.lloyd_residuals(pool, got["cb"].astype(np.float64))
    assert worst < 1e-6 and empty == 0
    if np.array_equal(got["cb"], ref["cb"]):
        assert np.array_equal(got["packed"], ref["packed"])
    assert np.array_equal(got["s_rel"], ref["s_rel"])
    assert np.array_equal(got["s_ch"].view(np.uint32), ref["s_ch"].view(np.uint32))


def test_convert_fit_whole_pool(lib):
    """Fewer live values than the sample cap: the fit uses all of them."""
    n, k = 64, 512
    w = weights_with_edges(n, k, 41)
    ref = O.convert_weight(w)
    got = gpu_convert(lib, w)
    live = ref["v"][np.repeat((ref["s_rel"] & 0x7F) != 0, 16, axis=1) & (ref["s_ch"] > 0)[:, None]]
    check_fit(got, ref, live)
    assert abs(int(got["fit_rounds"][0]) - ref["fit_rounds"]) <= 1
    assert lib.get_device_error() == 0


def test_convert_fit_sampled_pool(lib):
    """More live values than the cap: the seeded sample, drawn by the binding,
    is the oracle's sample, so the fits agree."""
    n, k, cap = 592, 1024, 2 ** 16
    w = weights_with_edges(n, k, 42)
    ref = O.convert_weight(w, sample_cap=cap)
    out = lib.convert_weight_sampled(torch.from_numpy(w).cuda(), sample_cap=cap, seed=42)
    got = {key: (v.cpu().numpy() if isinstance(v, torch.Tensor) else v) for key, v in out.items()}
    live = ref["v"][np.repeat((ref["s_rel"] & 0x7F) != 0, 16, axis=1) & (ref["s_ch"] > 0)[:, None]]
    pool = np.random.Generator(np.random.PCG64(42)).choice(live, size=cap, replace=False)
    check_fit(got, ref, pool)
    assert lib.get_device_error() == 0


def test_convert_sample_position_out_of_range_is_reported(lib):
    """A bad sample position is caught on the device (no access is made), and
    reported as W4A8_ERR_INPUT by the error query."""
    n, k = 16, 256
    w = weights_with_edges(n, k, 43)
    pos = torch.tensor([0, 1, n * k + 5], dtype=torch.int64, device="cuda")
    lib.convert_weight(torch.from_numpy(w).cuda(), sample_pos=pos)
    assert lib.get_device_error() == 8
    assert lib.get_device_error() == 0


def test_converted_layer_runs_through_linear(lib):
    """The GPU-converted tensors pack and run like the oracle's."""
    n, k = 592, 768
    w = synth.weights(n, k, synth.rng_for(44, 0, "weight"))
    got = gpu_convert(lib, w.astype(np.float32))
    packed = lib.pack_layout(*(torch.from_numpy(np.ascontiguousarray(got[key])).cuda()
                               for key in ("packed", "s_rel", "s_ch", "cb")))
    bits, x, _ = synth.activations(3, k, synth.rng_for(44, 3, "act"), 8)
    y = lib.linear(torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16), packed, n)
    y_ref = O.linear_packed(x, got["packed"], got["s_rel"], got["s_ch"], got["cb"])
    rel = np.linalg.norm(y.float().cpu().numpy() - y_ref) / np.linalg.norm(y_ref)
    assert rel <= 2e-3
