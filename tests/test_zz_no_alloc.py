"""GPU test of w4a8_linear_decode_static, the decode call that needs no
workspace.  It is for callers that cannot allocate device memory where they
run the layer: a plugin whose host application owns the device heap, a
latency-critical path that must not allocate (cudaMalloc can synchronise the
device), or a foreign-function caller with no device allocator.  It runs on
a scratch array built into the library instead.

Calls in a row on different layers, token counts and widths -- so each call
meets the previous call's leftovers in the shared scratch, and a one-token
call follows a 16-token one -- must give exactly the bits of w4a8_linear
(with a caller workspace: both run the same kernels on the same codes), and
agree with the oracle within the layer's tolerance.  K = 9216 takes the
cluster-pair path of the one-token kernel in w4a8_linear.  A call made right
after the bounded-wait self-test recorded a timeout still matches.

This file is collected last so that a failure here does not hide the other
tests; it passes alone in a fresh process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS_FACTOR = 1e-2

_LAYERS = {}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _layer(lib, n, k, seed):
    key = (n, k, seed)
    if key not in _LAYERS:
        c = O.convert_weight(synth.weights(n, k, synth.rng_for(seed, 0, "weight")))
        packed = lib.pack_layout(_dev(c["packed"]), _dev(c["s_rel"]), _dev(c["s_ch"]), _dev(c["cb"]))
        _LAYERS[key] = (c, packed)
    return _LAYERS[key]


def _call_and_check(lib, m, n, k, seed):
    c, packed = _layer(lib, n, k, seed)
    bits, x, _ = synth.activations(m, k, synth.rng_for(seed, m, "act"), max(2, k // 100))
    xt = _dev(bits.view(np.int16)).view(torch.bfloat16)
    y_static = lib.linear_decode_static(xt, packed, n)
    y_ws = lib.linear(xt, packed, n)
    # same kernels on the same codes: the same bits
    assert torch.equal(y_static.view(torch.int16), y_ws.view(torch.int16)), (m, n, k)
    # and within the layer's tolerance of the oracle
    y_ref = O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
    y = y_static.float().cpu().numpy().astype(np.float64)
    floor = np.linalg.norm(O.round_to_bf16(y_ref) - y_ref) / np.linalg.norm(y_ref)
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel <= max(REL_L2, 1.1 * floor), f"relative L2 error {rel:.3e} ({m}, {n}, {k})"
    wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
    bound = MAX_ABS_FACTOR * np.linalg.norm(x.astype(np.float64), axis=1) * wmax
    assert np.all(np.abs(y - y_ref).max(axis=1) <= bound), (m, n, k)


def test_static_scratch_matches_workspace_call_in_a_row(lib):
    # (M, N, K, seed): one token, 16 tokens on a wide layer, one token on that
    # wide layer (it meets the 16-token call's leftovers), then a few tokens
    calls = [(1, 592, 768, 60), (16, 160, 9216, 61), (1, 160, 9216, 61), (4, 592, 768, 62), (1, 592, 768, 60)]
    for m, n, k, seed in calls:
        _call_and_check(lib, m, n, k, seed)
    assert lib.get_device_error() == 0


def test_static_scratch_after_a_recorded_timeout(lib):
    lib.selftest_timeout()
    assert lib.get_device_error() == 6  # W4A8_ERR_TIMEOUT, read and cleared
    _call_and_check(lib, 1, 592, 768, 60)
    _call_and_check(lib, 8, 160, 9216, 61)
    assert lib.get_device_error() == 0


def test_static_scratch_rejects_prefill_sizes(lib):
    _, packed = _layer(lib, 64, 256, 63)
    x = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.W4A8Error) as e:
        lib.linear_decode_static(x, packed, 64)
    assert e.value.status == 2
