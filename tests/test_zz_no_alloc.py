"""GPU test of w4a8_linear_decode_static, the decode call that needs no
workspace: it runs on a scratch array built into the library, for callers
that cannot allocate device memory where they run the layer (a plugin whose
host owns the device heap, a latency-critical path that must not allocate,
a foreign-function caller with no device allocator).

Two calls in a row -- different tokens and different layers, so the second
call meets the first call's leftovers in the shared scratch -- must agree
with w4a8_linear (caller workspace) within the parity tolerance.  This file
is collected last so that a failure here does not hide the other tests; it
passes alone in a fresh process and after the rest of the suite.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _layer(lib, n, k, seed):
    c = O.convert_weight(synth.weights(n, k, synth.rng_for(seed, 0, "weight")))
    packed = lib.pack_layout(_dev(c["packed"]), _dev(c["s_rel"]), _dev(c["s_ch"]), _dev(c["cb"]))
    wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
    return packed, wmax


def _close(y_static, y_ws, x, wmax):
    a = y_static.float().cpu().numpy().astype(np.float64)
    b = y_ws.float().cpu().numpy().astype(np.float64)
    rel = np.linalg.norm(a - b) / np.linalg.norm(b)
    assert rel <= REL_L2, f"relative L2 difference {rel:.3e}"
    bound = 1e-2 * np.linalg.norm(x.astype(np.float64), axis=1) * wmax
    assert np.all(np.abs(a - b).max(axis=1) <= bound)


def test_static_scratch_matches_workspace_call_twice(lib):
    n, k = 592, 768
    calls = [(1, 60), (16, 61)]          # two calls in a row: M=1 then M=16, different layers
    for m, seed in calls:
        packed, wmax = _layer(lib, n, k, seed)
        bits, x, _ = synth.activations(m, k, synth.rng_for(seed, m, "act"), 8)
        xt = _dev(bits.view(np.int16)).view(torch.bfloat16)
        y_static = lib.linear_decode_static(xt, packed, n)
        y_ws = lib.linear(xt, packed, n)
        _close(y_static, y_ws, x, wmax)
    assert lib.get_device_error() == 0


def test_static_scratch_rejects_prefill_sizes(lib):
    packed, _ = _layer(lib, 64, 256, 62)
    x = torch.zeros((17, 256), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(lib.W4A8Error) as e:
        lib.linear_decode_static(x, packed, 64)
    assert e.value.status == 2
