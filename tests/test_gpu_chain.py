"""A chain of one-token layers in one persistent launch (w4a8_chain_plan /
w4a8_chain_run): every layer's output equals the layer-by-layer w4a8_linear
call bit for bit, and each layer matches the oracle on the input it was given
(the previous layer's bf16 output), including when a later layer overwrites a
buffer an earlier layer read."""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def cuda(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def layer(lib, n, k, seed):
    c = O.convert_weight(synth.weights(n, k, synth.rng_for(seed, 0, "weight")), sample_cap=2 ** 16)
    return c, lib.pack_layout(cuda(c["packed"]), cuda(c["s_rel"]), cuda(c["s_ch"]), cuda(c["cb"]))


def bits_to_f32(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("reuse", [False, True])
def test_chain_equals_layer_by_layer_and_oracle(lib, reuse):
    shapes = [(1024, 768), (512, 1024), (2048, 512), (768, 2048)]  # (N, K): each K is the previous N
    layers = [layer(lib, n, k, 80 + i) for i, (n, k) in enumerate(shapes)]
    bits, _, _ = synth.activations(1, 768, synth.rng_for(81, 1, "act"), 8)
    x0 = cuda(bits.view(np.int16)).view(torch.bfloat16).reshape(-1)
    ys = [torch.empty(n, dtype=torch.bfloat16, device="cuda") for n, _ in shapes]
    if reuse:  # the last layer writes into the first layer's input buffer
        ys[3] = x0
    x_in = x0.clone()
    desc, xs = [], [x0] + ys[:-1]
    for i, ((n, k), (c, pk)) in enumerate(zip(shapes, layers)):
        desc.append((pk, n, k, xs[i], ys[i]))
    plan, ws, nl = lib.chain_plan(desc)
    lib.chain_run(plan, nl, ws)
    got = [y.clone() for y in ys]
    assert lib.get_device_error() == 0
    # layer by layer through w4a8_linear
    x = x_in.reshape(1, -1)
    for i, ((n, k), (c, pk)) in enumerate(zip(shapes, layers)):
        y = lib.linear(x, pk, n)
        assert torch.equal(y.reshape(-1).view(torch.int16), got[i].view(torch.int16)), f"layer {i}"
        # oracle on the input this layer saw
        xi = bits_to_f32(x)
        ref = O.linear(xi, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
        yv = bits_to_f32(y)
        rel = np.linalg.norm(yv - ref) / np.linalg.norm(ref)
        assert rel <= 2e-3, f"layer {i}: rel {rel}"
        x = y
    # a second run of the same plan gives the same bits (workspace counters were reset)
    if not reuse:
        lib.chain_run(plan, nl, ws)
        for i in range(len(shapes)):
            assert torch.equal(ys[i].view(torch.int16), got[i].view(torch.int16))
