"""Fidelity checks (w4a8_compare, w4a8_dense_reference, and the binding's
verify_layer that composes them) against the oracle.

Bars: the reductions equal numpy's fp64 sums to 1e-12 relative; the dense
reference equals the fp64 product rounded to fp32 within one fp32 ulp; a
layer converted by the oracle verifies with fidelity ~0 (at most one fp32
ulp of codebook drift, 1e-6); a layer with a dropped scale tensor row or a
zeroed codebook verifies with the oracle's own fidelity figure; the forward
error equals the oracle's figure for the same quantised outputs.  (On these
i.i.d. Gaussian synthetic weights a 16-level codebook leaves ~7 % relative
weight error, and the forward error follows it; the pages' ~1 % is a
figure for real layers, which these inputs do not stand in for.)
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def test_compare_matches_numpy(lib):
    rng = np.random.default_rng(3)
    ref = rng.standard_normal(1_000_003).astype(np.float32)
    a = (ref + 1e-3 * rng.standard_normal(ref.size)).astype(np.float32)
    got = lib.compare(cuda(a), cuda(ref)).cpu().numpy()
    d = a.astype(np.float64) - ref
    want = np.array([np.sum(d * d), np.sum(ref.astype(np.float64) ** 2), np.max(np.abs(d))])
    assert np.allclose(got, want, rtol=1e-12, atol=0)
    # bf16 left operand
    ab = torch.from_numpy(a).to(torch.bfloat16)
    got_b = lib.compare(ab.cuda(), cuda(ref)).cpu().numpy()
    d = ab.float().numpy().astype(np.float64) - ref
    assert np.allclose(got_b, [np.sum(d * d), want[1], np.max(np.abs(d))], rtol=1e-12, atol=0)
    # deterministic
    assert torch.equal(lib.compare(cuda(a), cuda(ref)), lib.compare(cuda(a), cuda(ref)))


def test_dense_reference_matches_fp64_product(lib):
    n, k, m = 300, 1280, 3
    w = synth.weights(n, k, synth.rng_for(60, 0, "weight")).astype(np.float32)
    bits, x, _ = synth.activations(m, k, synth.rng_for(60, 1, "act"), 8)
    y = lib.dense_reference(cuda(bits.view(np.int16)).view(torch.bfloat16), cuda(w)).cpu().numpy()
    want = (x.astype(np.float64) @ w.astype(np.float64).T).astype(np.float32)
    assert np.all(np.abs(y - want) <= np.spacing(np.abs(want)))


@pytest.fixture(scope="module")
def stored():
    n, k = 592, 1024
    w = synth.weights(n, k, synth.rng_for(61, 0, "weight")).astype(np.float32)
    ref = O.convert_weight(w, sample_cap=2 ** 16)
    bits, x, _ = synth.activations(4, k, synth.rng_for(61, 4, "act"), 10)
    return w, ref, bits, x


def run_verify(lib, w, q, bits):
    packed = lib.pack_layout(cuda(q["packed"]), cuda(q["s_rel"]), cuda(q["s_ch"]), cuda(q["cb"]))
    xt = cuda(bits.view(np.int16)).view(torch.bfloat16)
    return lib.verify_layer(cuda(w), packed, xt, sample_cap=2 ** 16, seed=42), packed, xt


def test_faithful_layer_verifies_near_zero(lib, stored):
    w, ref, bits, x = stored
    res, packed, xt = run_verify(lib, w, ref, bits)
    assert res["fidelity"] <= 1e-6
    # forward error: the oracle's figure for the same quantised outputs
    y_q = lib.linear(xt, packed, w.shape[0]).float().cpu().numpy().astype(np.float64)
    y_full = x.astype(np.float64) @ w.astype(np.float64).T
    want = np.linalg.norm(y_q - y_full) / np.linalg.norm(y_full)
    assert abs(res["forward"] - want) <= 1e-6 * want
    w_hat = O.dequant(ref["idx"], ref["s_rel"], ref["s_ch"], ref["cb"]).astype(np.float64)
    w_rot = O.rotate_blocks(w)
    weight_err = np.linalg.norm(w_hat - w_rot) / np.linalg.norm(w_rot)
    assert 0.7 * weight_err < res["forward"] < 1.3 * weight_err
    assert lib.get_device_error() == 0


@pytest.mark.parametrize("damage", ["row_scales_dropped", "codebook_zeroed"])
def test_damaged_layer_is_caught_with_the_oracles_figure(lib, stored, damage):
    w, ref, bits, x = stored
    q = {key: np.array(v, copy=True) for key, v in ref.items() if key in ("packed", "s_rel", "s_ch", "cb")}
    if damage == "row_scales_dropped":
        q["s_rel"][7] = 0
    else:
        q["cb"][:] = 0.0
    res, _, _ = run_verify(lib, w, q, bits)
    w_bad = O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"]).astype(np.float64)
    w_good = O.dequant_packed(ref["packed"], ref["s_rel"], ref["s_ch"], ref["cb"]).astype(np.float64)
    want = np.linalg.norm(w_bad - w_good) / np.linalg.norm(w_good)
    assert want > 1e-3
    assert abs(res["fidelity"] - want) <= 1e-6 * want
    assert abs(res["fidelity_max_abs"] - np.max(np.abs(w_bad - w_good))) <= 1e-12
