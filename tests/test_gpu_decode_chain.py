"""GPU tests of w4a8_decode_chain: a decode step as one launch per one-token
layer, each layer rotating the next layer's input blocks in its epilogue
(ConvRot card, "Why this exists": a decode step re-reads every layer's
weights for one token).  Every layer's output must equal the layer-by-layer
w4a8_linear calls bit for bit (the consumer quantises the same rotated
values with the same arithmetic), and the chain's last layer must match the
oracle on the input the chain gave it."""

import numpy as np
import pytest
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _layer(lib, n, k, seed):
    q = synth.quantized_format(n, k, synth.rng_for(50, seed, "qfmt"))
    return q, lib.pack_layout(_dev(q["packed"]), _dev(q["s_rel"]), _dev(q["s_ch"]), _dev(q["cb"]))


def _blocks(lib, nblocks, d, d_qkv, d_ff, seed0):
    """Layers of a hybrid-decoder-like stack: per block h -> qkv -> out (on
    the first d outputs of qkv) -> gate, up (both on out's output) -> down
    (on up's output) -> next h."""
    h0 = torch.randn((1, d), device="cuda").to(torch.bfloat16)
    qkv = torch.empty((1, d_qkv), dtype=torch.bfloat16, device="cuda")
    out = torch.empty((1, d), dtype=torch.bfloat16, device="cuda")
    gate = torch.empty((1, d_ff), dtype=torch.bfloat16, device="cuda")
    up = torch.empty((1, d_ff), dtype=torch.bfloat16, device="cuda")
    h = torch.empty((1, d), dtype=torch.bfloat16, device="cuda")
    layers, qs = [], []
    x = h0
    for b in range(nblocks):
        for j, (n, k, xin, yout) in enumerate([(d_qkv, d, x, qkv), (d, d, qkv[:, :d], out), (d_ff, d, out, gate),
                                               (d_ff, d, out, up), (d, d_ff, up, h)]):
            q, pk = _layer(lib, n, k, seed0 + 10 * b + j)
            layers.append((pk, n, k, xin.reshape(-1), yout.reshape(-1)))
            qs.append(q)
        x = h
    return layers, qs, (h0, qkv, out, gate, up, h)


def _layer_by_layer(lib, layers):
    outs = []
    for pk, n, k, x, y in layers:
        lib.linear(x.view(1, k), pk, n, out=y.view(1, n))
        outs.append(y.clone())
    return outs


@pytest.mark.parametrize("d,d_qkv,d_ff", [(512, 1024, 768), (1024, 1536, 9216)])
def test_decode_chain_equals_layer_by_layer(lib, d, d_qkv, d_ff):
    layers, qs, bufs = _blocks(lib, 3, d, d_qkv, d_ff, 7 * d)
    ref = _layer_by_layer(lib, layers)          # 15 layers, 12 of them read a fused activation
    chain = lib.DecodeChain(layers)
    for rep in range(2):                        # the workspace is reused: counters left at zero
        for t in bufs[1:]:
            t.fill_(0)
        chain.run()
        torch.cuda.synchronize()
        # the buffers hold the last block's outputs: qkv, out, gate, up, h
        for buf, r in zip(bufs[1:], ref[-5:]):
            assert torch.equal(buf.view(torch.int16), r.view(1, -1).view(torch.int16)), rep
    # every layer of the chain, one prefix at a time
    for i in range(1, len(layers) + 1):
        sub = lib.DecodeChain(layers[:i])
        sub.run()
        torch.cuda.synchronize()
        assert torch.equal(layers[i - 1][4].view(torch.int16), ref[i - 1].view(torch.int16)), i
    # the last layer against the oracle, on the input the chain gave it
    pk, n, k, x, y = layers[-1]
    q = qs[-1]
    xb = x.view(torch.int16).cpu().numpy().view(np.uint16).reshape(1, k)
    xf = synth.bf16_bits_to_f32(xb)
    y_ref = O.linear_packed(xf, q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    got = y.float().cpu().numpy().astype(np.float64).reshape(1, n)
    rel = np.linalg.norm(got - y_ref) / np.linalg.norm(y_ref)
    floor = np.linalg.norm(O.round_to_bf16(y_ref) - y_ref) / np.linalg.norm(y_ref)
    assert rel <= max(2e-3, 1.1 * floor)
    assert lib.get_device_error() == 0


def test_decode_chain_offset_slice_and_overwritten_input(lib):
    """A consumer reading y[256:768] of a producer (an offset slice), and a
    layer whose input was overwritten by a layer in between (it must rotate
    the new values itself)."""
    a = torch.randn((1, 512), device="cuda").to(torch.bfloat16)
    y1 = torch.empty((1, 1024), dtype=torch.bfloat16, device="cuda")
    y2 = torch.empty((1, 512), dtype=torch.bfloat16, device="cuda")
    y3 = torch.empty((1, 256), dtype=torch.bfloat16, device="cuda")
    _, l1 = _layer(lib, 1024, 512, 1)
    _, l2 = _layer(lib, 512, 512, 2)
    _, l3 = _layer(lib, 256, 512, 3)
    _, l4 = _layer(lib, 1024, 256, 4)
    _, l5 = _layer(lib, 512, 512, 5)
    layers = [(l1, 1024, 512, a.reshape(-1), y1.reshape(-1)),
              (l2, 512, 512, y1.reshape(-1)[256:768], y2.reshape(-1)),      # offset slice of l1's output
              (l3, 256, 512, y2.reshape(-1), y3.reshape(-1)),
              (l4, 1024, 256, y3.reshape(-1), y1.reshape(-1)),              # overwrites l1's output
              (l5, 512, 512, y1.reshape(-1)[256:768], y2.reshape(-1))]      # now fused from l4
    ref = _layer_by_layer(lib, layers)
    lib.DecodeChain(layers).run()
    torch.cuda.synchronize()
    assert torch.equal(y2.reshape(-1).view(torch.int16), ref[-1].view(torch.int16))
    assert torch.equal(y1.reshape(-1).view(torch.int16), ref[3].view(torch.int16))
    assert lib.get_device_error() == 0
