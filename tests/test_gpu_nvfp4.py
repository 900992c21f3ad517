"""GPU parity of the NVFP4 comparison layer (w4a8_nvfp4_* through the C ABI)
against the NVFP4 oracle (oracle/nvfp4_ref.py).

Format: "Qwen3.8-27B-Uncensored-NVFP4: En runbook för servering på
Blackwell-GPU:er", section "Vad NVFP4 är, och hur det skiljer sig från FP8
och från INT8/AWQ" (E2M1 values, an e4m3 scale per 16, an fp32 scalar per
tensor).

Bars:
  * quantiser without rotation: codes, scales and g bit-exact (every decision
    is an IEEE fp32 operation on the same inputs);
  * quantiser with rotation: g within 1 ulp; scales and codes equal except on
    at most 1e-3 of the blocks / values, where the rotated value (fp32
    butterflies against the fp64 rotation rounded once) sits on a rounding
    boundary: there they are one step apart;
  * product from the same quantised operands (the oracle's, uploaded): per
    element |y - ref| <= 2^-8 |ref| + 2^-16 sum_k |terms| (bf16 output
    rounding plus fp32 accumulation), relative L2 <= max(2e-3, 1.1 x the
    bf16 rounding floor);
  * the whole layer from bf16 x and fp32 W against the oracle's layer:
    relative L2 <= max(3e-3, 1.1 x floor) (the rare code flips above add a
    little to the product's bar).
Shapes: the smallest tile first, then several tiles with ragged token and
weight-row tails on each token-tile width (64, 128, 256), then the full
workload shape on sampled outputs.
"""

import numpy as np
import pytest
import torch

import synth
from oracle import nvfp4_ref as N
from oracle import w4a8_ref as O

pytestmark = pytest.mark.gpu


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def sf_rows(buf, r, k):
    """The header's tensor-core scale order -> row-major [r_padded, k/16]."""
    cols = k // 16
    rr = np.arange((r + 127) // 128 * 128)[:, None]
    cc = np.arange(cols)[None, :]
    off = ((rr >> 7) * (k // 64) + (cc >> 2)) * 512 + (rr & 31) * 16 + ((rr >> 5) & 3) * 4 + (cc & 3)
    return np.asarray(buf)[off]


def upload(lib, codes, scales, g):
    """Oracle operands (unpacked codes, row-major scales) -> device operands."""
    return dev(N.pack_codes(codes)), lib.nvfp4_pack_scales(dev(scales)), dev(g)


def check_product(y, ref, absref, rel_bar=2e-3):
    y64 = y.float().cpu().numpy().astype(np.float64)
    err = np.abs(y64 - ref)
    bound = 2.0 ** -8 * np.abs(ref) + 2.0 ** -16 * absref
    bad = err > bound
    assert not bad.any(), f"{bad.sum()} outputs off, worst {(err - bound).max():.3e}"
    floor = np.linalg.norm(O.round_to_bf16(ref) - ref) / max(np.linalg.norm(ref), 1e-300)
    rel = np.linalg.norm(y64 - ref) / max(np.linalg.norm(ref), 1e-300)
    assert rel <= max(rel_bar, 1.1 * floor), f"relative L2 {rel:.3e}"


def oracle_product(cx, sx, gx, cw, sw, gw):
    xh = N.dequant_rows(cx, sx, gx)
    wh = N.dequant_rows(cw, sw, gw)
    return xh @ wh.T, np.abs(xh) @ np.abs(wh).T


def operands(m, n, k, seed):
    x = synth.nvfp4_operands(m, k, synth.rng_for(60, seed, "act"))
    w = synth.nvfp4_operands(n, k, synth.rng_for(60, seed, "weight"))
    return x, w


def run_gemm(lib, x, w):
    xd = upload(lib, N.unpack_codes(x["codes"]), x["scales"], x["g"])
    wd = upload(lib, N.unpack_codes(w["codes"]), w["scales"], w["g"])
    return lib.nvfp4_gemm(*xd, *wd)


def test_pack_scales_layout(lib):
    rng = np.random.default_rng(1)
    for r, k in ((1, 256), (130, 512), (256, 768)):
        rows = rng.integers(0, 256, size=(r, k // 16), dtype=np.uint8)
        got = lib.nvfp4_pack_scales(dev(rows)).cpu().numpy()
        back = sf_rows(got, r, k)
        assert np.array_equal(back[:r], rows)
        assert not back[r:].any()


def test_gemm_single_tile(lib):
    """One CTA, one 256-k stage: 16 tokens x 128 weight rows."""
    x, w = operands(16, 128, 256, 0)
    y = run_gemm(lib, x, w)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref, absref = oracle_product(N.unpack_codes(x["codes"]), x["scales"], x["g"],
                                 N.unpack_codes(w["codes"]), w["scales"], w["g"])
    check_product(y, ref, absref)


@pytest.mark.parametrize("m,n,k", [
    (1, 128, 512),        # one token: 64-token tile, 63 zero-filled rows
    (64, 256, 1024),      # 64-token tile, 2 weight tiles, 4 stages
    (100, 384, 768),      # 128-token tile, ragged tokens
    (300, 200, 1280),     # 256-token tiles, ragged tokens (second tile past one scale block) and weight rows
    (513, 136, 2560),     # 3 token tiles, the last with one token; 10 stages over 4 buffers
])
def test_gemm_tiles_and_tails(lib, m, n, k):
    x, w = operands(m, n, k, m)
    y = run_gemm(lib, x, w)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref, absref = oracle_product(N.unpack_codes(x["codes"]), x["scales"], x["g"],
                                 N.unpack_codes(w["codes"]), w["scales"], w["g"])
    check_product(y, ref, absref)


def test_gemm_zero_rows_and_scales(lib):
    """A token with g = 0 and a weight row with zero scales give exact zeros;
    zero e4m3 block scales inside live rows drop just those blocks."""
    m, n, k = 40, 160, 512
    x, w = operands(m, n, k, 7)
    sub = np.random.default_rng(3).integers(0, 8, size=w["scales"][:, 1::7].shape)   # subnormal and zero scales
    w["scales"][:, 1::7] = sub
    x["scales"][:, ::5] = 0
    x["g"][3] = 0.0
    w["scales"][5] = 0
    y = run_gemm(lib, x, w)
    torch.cuda.synchronize()
    yc = y.float().cpu().numpy()
    assert not yc[3].any() and not yc[:, 5].any()
    ref, absref = oracle_product(N.unpack_codes(x["codes"]), x["scales"], x["g"],
                                 N.unpack_codes(w["codes"]), w["scales"], w["g"])
    check_product(y, ref, absref)


@pytest.mark.parametrize("f32", [False, True])
def test_quantize_without_rotation_bit_exact(lib, f32):
    r, k = 70, 768
    if f32:
        a = synth.weights(r, k, synth.rng_for(61, 0, "weight"))
        xt = dev(a)
        xa = a.astype(np.float64)
    else:
        bits, xa, _ = synth.activations(r, k, synth.rng_for(61, 1, "act"), 8)
        xt = dev(bits.view(np.int16)).view(torch.bfloat16)
    xa = np.array(xa, dtype=np.float64)
    xa[4] = 0.0                                   # a zero row: g = 0, all codes and scales 0
    xt[4] = 0
    for per_tensor in (False, True):
        codes, scales, g = lib.nvfp4_quantize(xt, rotate=False, per_tensor=per_tensor)
        c_ref, s_ref, g_ref = N.quantize_rows(xa, rotate=False, per_row=not per_tensor)
        assert np.array_equal(g.cpu().numpy().view(np.uint32), g_ref.view(np.uint32))
        sc = sf_rows(scales.cpu().numpy(), r, k)
        assert np.array_equal(sc[:r], s_ref) and not sc[r:].any()
        assert np.array_equal(codes.cpu().numpy(), N.pack_codes(c_ref))


@pytest.mark.parametrize("r,k,per_tensor,f32", [(37, 512, False, False), (16, 5120, False, False),
                                                (64, 17408, False, False), (96, 768, True, True)])
def test_quantize_with_rotation(lib, r, k, per_tensor, f32):
    if f32:
        a = synth.weights(r, k, synth.rng_for(62, r, "weight"))
        xt, xa = dev(a), a.astype(np.float64)
    else:
        bits, xa, _ = synth.activations(r, k, synth.rng_for(62, r, "act"), max(1, k // 100))
        xt = dev(bits.view(np.int16)).view(torch.bfloat16)
    codes, scales, g = lib.nvfp4_quantize(xt, rotate=True, per_tensor=per_tensor)
    c_ref, s_ref, g_ref = N.quantize_rows(xa, rotate=True, per_row=not per_tensor)
    gd = g.cpu().numpy()
    assert np.all(np.abs(gd.view(np.int32).astype(np.int64) - g_ref.view(np.int32)) <= 1)
    sc = sf_rows(scales.cpu().numpy(), r, k)[:r]
    ds = sc != s_ref
    assert ds.sum() <= max(2, 1e-3 * ds.size), f"{ds.sum()} block scales differ"
    assert np.all(np.abs(sc[ds].astype(int) - s_ref[ds].astype(int)) <= 1)
    cg = N.unpack_codes(codes.cpu().numpy())
    # compare values only where the block scale agrees (a scale flip rescales its 16 codes)
    same = np.repeat(~ds, 16, axis=1)
    vg, vr = N.e2m1_decode(cg)[same], N.e2m1_decode(c_ref)[same]
    dc = vg != vr
    assert dc.sum() <= max(4, 1e-3 * dc.size), f"{dc.sum()} codes differ"
    grid = np.array(sorted({abs(v) for v in N.E2M1_MAGNITUDES}))
    step = lambda v: np.searchsorted(grid, np.abs(v))
    assert np.all(np.abs(step(vg[dc]) - step(vr[dc])) <= 1)
    assert np.all((np.sign(vg[dc]) == np.sign(vr[dc])) | (vg[dc] == 0) | (vr[dc] == 0))


@pytest.mark.parametrize("m,n,k", [(1, 256, 512), (45, 384, 1024), (300, 256, 768)])
def test_linear_matches_oracle(lib, m, n, k):
    bits, x, _ = synth.activations(m, k, synth.rng_for(63, m, "act"), max(1, k // 100))
    w = synth.weights(n, k, synth.rng_for(63, n, "weight"))
    wc, ws, gw = lib.nvfp4_quantize(dev(w), rotate=True, per_tensor=True)
    y = lib.nvfp4_linear(dev(bits.view(np.int16)).view(torch.bfloat16), wc, ws, gw)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    ref = N.linear(x, w, rotate=True)
    y64 = y.float().cpu().numpy().astype(np.float64)
    floor = np.linalg.norm(O.round_to_bf16(ref) - ref) / np.linalg.norm(ref)
    rel = np.linalg.norm(y64 - ref) / np.linalg.norm(ref)
    assert rel <= max(3e-3, 1.1 * floor), f"relative L2 {rel:.3e}"


def test_gemm_full_size_sampled(lib):
    """The timed shape (4096 tokens, K = 5120, N = 17408), sampled outputs."""
    m, n, k = 4096, 17408, 5120
    x, w = operands(m, n, k, 99)
    y = run_gemm(lib, x, w)
    torch.cuda.synchronize()
    assert lib.get_device_error() == 0
    rng = np.random.default_rng(4)
    rows = np.sort(rng.choice(m, 48, replace=False))
    cols = np.sort(rng.choice(n, 192, replace=False))
    ref, absref = oracle_product(N.unpack_codes(x["codes"][rows]), x["scales"][rows], x["g"][rows],
                                 N.unpack_codes(w["codes"][cols]), w["scales"][cols], w["g"][cols])
    check_product(y[torch.from_numpy(rows).cuda()][:, torch.from_numpy(cols).cuda()], ref, absref)
