"""Parity of every linear path at the edges of the stored format.

ConvRot card, "Format" (three tiers of scaling: codebook level, e4m3 group
scale, fp32 row scale) and W4A8 card, "Model Overview" (group 16, fp8 group
scales).  Two kinds of layer, each at K = 5120 and K = 17408 (the one-token
kernel's cluster-pair path):
  * converted by the oracle from weights with edge rows: an all-zero row, a
    row whose single huge entry drives its other groups' e4m3 scales to
    subnormals and zero, a half-zero row and a row with one zero group;
  * drawn directly in the stored format: subnormal and zero group scales
    inside live rows, a dead row, a row with one live group, a zero row
    scale, and a codebook with levels within 1e-4 of zero and out to -8 and
    7.5.
Each runs through the one-token kernel (activation step fused, and the
two-kernel path), the 2..16-token kernel, the sliced path (17..64 tokens),
the small-batch tensor-core kernel (65..256 tokens on a narrow layer; 256
tokens take its single-accumulator path) and
the tensor-core GEMM, against the oracle at the layer's bars.
"""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS_FACTOR = 1e-2
N_ROWS = 96

_CACHE = {}


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _layer(lib, kind, k):
    key = (kind, k)
    if key not in _CACHE:
        if kind == "converted":
            c = O.convert_weight(synth.weights_with_edges(N_ROWS, k, synth.rng_for(40, k, "weight")))
            q = {"packed": c["packed"], "s_rel": c["s_rel"], "s_ch": c["s_ch"], "cb": c["cb"]}
            # the large-entry row carries e4m3 subnormal group scales, and zero scales occur in live rows
            assert np.any((q["s_rel"][2] > 0) & (q["s_rel"][2] < 8)) and np.any(q["s_rel"][4] == 0)
        else:
            q = synth.quantized_format_edges(N_ROWS, k, synth.rng_for(41, k, "qfmt"))
        packed = lib.pack_layout(_dev(q["packed"]), _dev(q["s_rel"]), _dev(q["s_ch"]), _dev(q["cb"]))
        wmax = float(np.abs(O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"])).max())
        _CACHE[key] = (q, packed, wmax)
    return _CACHE[key]


def _check(y, y_ref, x, wmax):
    floor = np.linalg.norm(O.round_to_bf16(y_ref) - y_ref) / np.linalg.norm(y_ref)
    rel = np.linalg.norm(y - y_ref) / np.linalg.norm(y_ref)
    assert rel <= max(REL_L2, 1.1 * floor), f"relative L2 error {rel:.3e}"
    bound = MAX_ABS_FACTOR * np.linalg.norm(x.astype(np.float64), axis=1) * wmax
    worst = np.abs(y - y_ref).max(axis=1)
    assert np.all(worst <= bound), f"max abs error {worst.max():.3e} > {bound.min():.3e}"


@pytest.mark.parametrize("kind", ["converted", "stored"])
@pytest.mark.parametrize("k", [5120, 17408])
@pytest.mark.parametrize("m,path", [(1, "fused"), (1, "two_kernel"), (4, "decode"), (16, "decode"),
                                    (40, "sliced"), (100, "small_batch"), (256, "small_batch_single_acc"),
                                    (300, "gemm")])
def test_edge_layers_every_path(lib, kind, k, m, path):
    q, packed, wmax = _layer(lib, kind, k)
    bits, x, _ = synth.activations(m, k, synth.rng_for(42, m, "act"), k // 100)
    xt = _dev(bits.view(np.int16)).view(torch.bfloat16)
    if path == "two_kernel":
        ws = lib.linear_workspace(m, k, N_ROWS, "cuda")
        lib.linear_prepare(xt, N_ROWS, ws)
        y = lib.linear_run(m, k, packed, N_ROWS, ws)
        assert torch.equal(y.view(torch.int16), lib.linear(xt, packed, N_ROWS).view(torch.int16))
    else:
        y = lib.linear(xt, packed, N_ROWS)
    y = y.float().cpu().numpy().astype(np.float64)
    y_ref = O.linear_packed(x, q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    _check(y, y_ref, x, wmax)
    # the dead row and the zero-scale row give exact zeros
    dead = [1] if kind == "converted" else [0, 2]
    assert np.all(y[:, dead] == 0.0)
    assert lib.get_device_error() == 0
