"""Parity of the CUDA library (through its C ABI) against the CPU oracle.

Bars (the layer's stated tolerances):
  * dequantisation and layout: bit-exact;
  * int8 activations: at most 1 LSB apart, on at most 1e-4 of the elements;
  * linear output (bf16) against the unrounded fp64 oracle: relative L2
    error <= 2e-3 and, per token m, max |error| <= 1e-2 * ||x_m||_2 * max|W_hat|
    (for outputs so small that rounding the exact result to bf16 already
    costs more than 2e-3, the L2 bar is 1.1x that rounding floor);
  * integer-valued special cases: exact.
Shapes span several tiles and ragged tails (odd tile counts, token counts
that are not multiples of 8 or 256) and the full workload shapes (sampled
outputs, computed one by one by the oracle).
"""

import math

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle as O
import synth

pytestmark = pytest.mark.gpu

REL_L2 = 2e-3
MAX_ABS_FACTOR = 1e-2


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def bf16(bits):
    return dev(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)


def pack(lib, q):
    return lib.pack_layout(dev(q["packed"]), dev(q["s_rel"]), dev(q["s_ch"]), dev(q["cb"]))


def converted(n, k, seed):
    w = synth.weights(n, k, synth.rng_for(seed, 0, "weight"))
    return O.convert_weight(w)


def rel_l2_bar(y_ref):
    """2e-3, unless rounding the exact result itself to bf16 already costs
    more (outputs of a few dozen elements, where the L2 statistic is noisy):
    then 1.1x that rounding floor."""
    floor = np.linalg.norm(O.round_to_bf16(y_ref) - y_ref) / np.linalg.norm(y_ref)
    return max(REL_L2, 1.1 * floor)


def check_linear(y_gpu, y_ref, x, w_maxabs):
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    err = y_gpu - y_ref
    rel = np.linalg.norm(err) / np.linalg.norm(y_ref)
    assert rel <= rel_l2_bar(y_ref), f"relative L2 error {rel:.3e}"
    bound = MAX_ABS_FACTOR * np.linalg.norm(np.asarray(x, dtype=np.float64), axis=1) * w_maxabs
    worst = np.max(np.abs(err), axis=1)
    assert np.all(worst <= bound), f"max abs error {worst.max():.3e} > bound {bound.min():.3e}"
    return rel


def run_linear(lib, x_bits, packed, n):
    return lib.linear(bf16(x_bits), packed, n).float().cpu().numpy()


# ------------------------------------------------------------------ dequant / layout

@pytest.mark.parametrize("n,k,seed", [(256, 512, 0), (592, 768, 1), (16, 256, 2)])
def test_dequant_bit_exact(lib, n, k, seed):
    c = converted(n, k, seed)
    got = lib.unpack_dequant(pack(lib, c), n, k).cpu().numpy()
    ref = O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_dequant_edge_scales_bit_exact(lib):
    """Subnormal and zero e4m3 scales, zero rows and extreme levels."""
    rng = np.random.default_rng(20)
    n, k = 64, 512
    q = synth.quantized_format(n, k, rng)
    q["s_rel"][:, ::3] = rng.integers(0, 8, size=q["s_rel"][:, ::3].shape)  # subnormals and zero
    q["s_rel"][5] = 0
    q["s_ch"][7] = 0.0
    q["s_ch"][9] = np.float32(1e-30)
    q["cb"] = np.array([-3.0e-8, *np.linspace(-1, 1, 14), 7.5], dtype=np.float32)
    got = lib.unpack_dequant(pack(lib, q), n, k).cpu().numpy()
    ref = O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def test_dequant_full_size_sampled_rows(lib):
    n, k = 17408, 5120
    q = synth.quantized_format(n, k, synth.rng_for(1, 0, "qfmt"))
    got = lib.unpack_dequant(pack(lib, q), n, k)
    rows = np.sort(synth.rng_for(1, 0, "sample").choice(n, 96, replace=False))
    ref = O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=rows)
    assert np.array_equal(got[torch.from_numpy(rows).cuda()].cpu().numpy().view(np.uint32), ref.view(np.uint32))


# ------------------------------------------------------------------ activations

def flips_ok(q_gpu, q_ref):
    d = np.abs(q_gpu.astype(np.int32) - q_ref.astype(np.int32))
    assert d.max() <= 1, f"int8 codes differ by {d.max()}"
    allowed = math.ceil(1e-4 * d.size)
    assert np.count_nonzero(d) <= allowed, f"{np.count_nonzero(d)} flips > {allowed}"


@pytest.mark.parametrize("m,k,outl", [(4, 512, 2), (37, 768, 8), (1, 5120, 51), (16, 17408, 174), (64, 17408, 174)])
def test_rotate_quant_matches_oracle(lib, m, k, outl):
    bits, x, _ = synth.activations(m, k, synth.rng_for(7, m, "act"), outl)
    xq, sx = lib.rotate_quant_act(bf16(bits))
    q_ref, s_ref, _ = O.quantize_activations(x)
    sx = sx.cpu().numpy()
    assert np.all(np.abs(sx.view(np.int32) - s_ref.view(np.int32)) <= 1)   # within 1 ulp
    flips_ok(xq.cpu().numpy(), q_ref)


def test_rotate_quant_special_rows(lib):
    k = 512
    x = np.zeros((3, k), dtype=np.float32)
    x[1, :256] = scipy.linalg.hadamard(256)[5] * (3.0 / 16.0)   # rotates to a spike of 3 at k = 5
    x[2, 300] = -2.0                                             # rotates to a flat block
    bits = synth.f32_to_bf16_bits(x)
    xq, sx = lib.rotate_quant_act(bf16(bits))
    q_ref, s_ref, _ = O.quantize_activations(x)
    assert np.array_equal(xq.cpu().numpy(), q_ref)
    assert np.array_equal(sx.cpu().numpy(), s_ref)
    assert sx[0].item() == 0.0


# ------------------------------------------------------------------ linear

@pytest.fixture(scope="module")
def layer592(lib):
    c = converted(592, 768, 3)          # 37 tiles of 16 rows: an odd tile count
    return c, pack(lib, c), float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())


@pytest.mark.parametrize("m", [1, 2, 3, 5, 8, 9, 13, 16])
def test_linear_decode_matches_oracle(lib, layer592, m):
    c, packed, wmax = layer592
    bits, x, _ = synth.activations(m, 768, synth.rng_for(4, m, "act"), 8)
    y = run_linear(lib, bits, packed, 592)
    check_linear(y, O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


@pytest.mark.parametrize("m", [17, 24, 33, 47, 64])
def test_linear_sliced_decode_matches_oracle(lib, layer592, m):
    """17..64 tokens run the decode kernel once per slice of 16 tokens (the
    last slice ragged); prepare-then-run gives the same bits as the one call."""
    c, packed, wmax = layer592
    bits, x, _ = synth.activations(m, 768, synth.rng_for(12, m, "act"), 8)
    y = run_linear(lib, bits, packed, 592)
    check_linear(y, O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)
    ws = lib.linear_workspace(m, 768, 592, "cuda")
    lib.linear_prepare(bf16(bits), 592, ws)
    y2 = lib.linear_run(m, 768, packed, 592, ws).float().cpu().numpy()
    assert np.array_equal(y.view(np.uint32), y2.view(np.uint32))


@pytest.mark.parametrize("m", [65, 255, 256, 300])
def test_linear_prefill_matches_oracle(lib, layer592, m):
    c, packed, wmax = layer592
    bits, x, _ = synth.activations(m, 768, synth.rng_for(5, m, "act"), 8)
    y = run_linear(lib, bits, packed, 592)
    check_linear(y, O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


@pytest.mark.parametrize("m,n,k", [(4, 256, 512), (513, 256, 512), (1, 16, 256), (40, 16, 256), (3, 4096, 1024)])
def test_linear_small_shapes(lib, m, n, k):
    c = converted(n, k, 6)
    wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
    bits, x, _ = synth.activations(m, k, synth.rng_for(6, m, "act"), 2)
    y = run_linear(lib, bits, pack(lib, c), n)
    check_linear(y, O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


def integer_case(m, n, k, seed):
    """Integer codebook, unit scales, and activations whose rotation is a
    spike per 256-block: every sum is a small integer, so y is exact."""
    rng = np.random.default_rng(seed)
    nb = k // 256
    cb = np.arange(-8, 8).astype(np.float32)
    idx = rng.integers(0, 16, size=(n, k)).astype(np.uint8)
    hs = scipy.linalg.hadamard(256)
    x = np.zeros((m, k), dtype=np.float32)
    expect = np.zeros((m, n))
    for r in range(m):
        pos = rng.integers(0, 256, size=nb)
        qv = rng.integers(-4, 5, size=nb)
        qv[0] = 127                        # sets s_x = 1 exactly
        idx[:, pos[0]] = 8                 # level 0.0 under the 127 spike, for every row
        for b in range(nb):
            x[r, 256 * b: 256 * (b + 1)] = hs[pos[b]] * (qv[b] / 16.0)
        # filled in after idx is final, below
        expect[r] = 0
    # expected values from the final index table
    for r in range(m):
        xr = O.rotate_blocks(x[r:r + 1])[0]
        nz = np.nonzero(np.rint(xr))[0]
        expect[r] = (np.rint(xr[nz])[None, :] * cb[idx[:, nz].astype(np.int64)]).sum(axis=1)
    q = {"packed": O.pack_nibbles(idx), "s_rel": np.full((n, k // 16), 0x38, np.uint8),
         "s_ch": np.ones(n, np.float32), "cb": cb}
    return q, x, expect


@pytest.mark.parametrize("m", [1, 4, 16, 300])
def test_linear_exact_integer_case(lib, m):
    n, k = 272, 768
    q, x, expect = integer_case(m, n, k, 30 + m)
    assert np.abs(expect).max() <= 256      # bf16 represents these exactly
    y = run_linear(lib, synth.f32_to_bf16_bits(x), pack(lib, q), n)
    assert np.array_equal(y.astype(np.float64), expect)


@pytest.mark.parametrize("m,k,n", [(1, 5120, 17408), (1, 17408, 5120), (4, 17408, 5120), (16, 17408, 5120),
                                   (1, 5120, 10240), (1, 5120, 5120), (64, 17408, 5120), (128, 17408, 5120),
                                   (4096, 5120, 17408), (8192, 17408, 5120)])
def test_linear_full_size_sampled(lib, m, k, n):
    """Workload shapes in the launch configuration the benchmark times (the
    decode step's four projections at one token, the down projection at 1,
    4, 16, 64 and 128 tokens, both prefill shapes); the oracle computes a
    sample of outputs (tokens x output rows)."""
    q = synth.quantized_format(n, k, synth.rng_for(11, n, "qfmt"))
    bits, x, _ = synth.activations(m, k, synth.rng_for(11, m, "act"), max(1, k // 100))
    y = lib.linear(bf16(bits), pack(lib, q), n)
    srng = synth.rng_for(11, m, "sample")
    toks = np.sort(srng.choice(m, min(m, 24), replace=False))
    rows = np.sort(srng.choice(n, 128, replace=False))
    y_s = y[torch.from_numpy(toks).cuda()][:, torch.from_numpy(rows).cuda()].float().cpu().numpy()
    ref = O.linear_packed(x[toks], q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=rows)
    wmax = float(np.abs(O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=rows)).max())
    check_linear(y_s, ref, x[toks], wmax)


@pytest.mark.parametrize("m", [1, 16, 300])
def test_linear_deterministic_and_workspace_reuse(lib, layer592, m):
    c, packed, _ = layer592
    bits, _, _ = synth.activations(m, 768, synth.rng_for(8, m, "act"), 8)
    xt = bf16(bits)
    need = max(lib.linear_workspace_bytes(mm, 768, 592) for mm in (1, 5, 16, 300))
    ws = torch.zeros(need + 4096, dtype=torch.uint8, device="cuda")
    a = lib.linear(xt, packed, 592, workspace=ws).clone()
    # other shapes through the same workspace in between (each path lays out
    # its scratch differently; the words that must start at zero stay put)
    for mm in (5, 16, 300, 1):
        other, _, _ = synth.activations(mm, 768, synth.rng_for(8, 99 + mm, "act"), 8)
        lib.linear(bf16(other), packed, 592, workspace=ws)
        b = lib.linear(xt, packed, 592, workspace=ws)
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), mm


def test_binding_refuses_bad_arguments(lib, layer592):
    c, packed, _ = layer592
    with pytest.raises(ValueError):
        lib.linear(torch.zeros(2, 768, device="cuda"), packed, 592)           # fp32 input
    with pytest.raises(Exception):
        lib.linear(torch.zeros(2, 700, dtype=torch.bfloat16, device="cuda"), packed, 592)   # K % 256
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(Exception):
        lib.linear(torch.zeros(2, 768, dtype=torch.bfloat16, device="cuda"), packed, 592, workspace=small)


def test_no_device_error_recorded(lib):
    assert lib.get_device_error() == 0


def test_bounded_waits_report_a_timeout_and_the_context_stays_usable(lib, layer592):
    """The library's bounded device waits (an mbarrier phase, a global word),
    run on things that never complete, give up, record a timeout that the
    next get_device_error returns and clears; the layer still runs and
    matches the oracle afterwards."""
    c, packed, wmax = layer592
    assert lib.get_device_error() == 0
    lib.selftest_timeout()
    assert lib.get_device_error() == 6  # W4A8_ERR_TIMEOUT
    assert lib.get_device_error() == 0  # cleared
    bits, x, _ = synth.activations(3, 768, synth.rng_for(19, 3, "act"), 8)
    y = lib.linear(bf16(bits), packed, 592).float().cpu().numpy()
    assert lib.get_device_error() == 0
    check_linear(y, O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


@pytest.mark.parametrize("m", [1, 4, 300])
def test_prepare_once_run_several_layers(lib, m):
    """One prepared activation, several layers of the same shape, each run
    equal to the fused call and to the oracle."""
    n, k = 592, 768
    layers = [converted(n, k, 40 + i) for i in range(3)]
    bits, x, _ = synth.activations(m, k, synth.rng_for(9, m, "act"), 8)
    xt = bf16(bits)
    ws = lib.linear_workspace(m, k, n, "cuda")
    lib.linear_prepare(xt, n, ws)
    for c in layers:
        packed = pack(lib, c)
        y_run = lib.linear_run(m, k, packed, n, ws)
        y_ref = lib.linear(xt, packed, n)
        assert torch.equal(y_run.view(torch.int16), y_ref.view(torch.int16))
        wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
        check_linear(y_run.float().cpu().numpy(), O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


@pytest.mark.parametrize("k", [5120, 15872, 16128, 17408, 32768])
def test_one_token_single_kernel_equals_two_kernel_path(lib, k):
    """For one token, w4a8_linear is one kernel that rotates and quantises the
    token itself (above K = 8192 as pairs of CTAs that split the rotation;
    past 64 blocks a warp rotates some blocks a second time); it must give
    the same bits as the activation kernel followed by the decode kernel,
    and match the oracle."""
    n = 592
    c = O.convert_weight(synth.weights(n, k, synth.rng_for(70, k, "weight")), sample_cap=2**16)
    packed = pack(lib, c)
    bits, x, _ = synth.activations(1, k, synth.rng_for(10, k, "act"), max(1, k // 100))
    xt = bf16(bits)
    y_one = lib.linear(xt, packed, n)
    ws = lib.linear_workspace(1, k, n, "cuda")
    lib.linear_prepare(xt, n, ws)
    y_two = lib.linear_run(1, k, packed, n, ws)
    assert torch.equal(y_one.view(torch.int16), y_two.view(torch.int16))
    # and again through the same workspace (its split-K counters were left at zero)
    assert torch.equal(lib.linear(xt, packed, n, workspace=ws).view(torch.int16), y_one.view(torch.int16))
    wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
    check_linear(y_one.float().cpu().numpy(), O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


@pytest.mark.parametrize("n,k", [(16, 8448), (48, 16640), (272, 8960), (16, 256), (1040, 8448)])
def test_one_token_small_grids_and_long_pairs(lib, n, k):
    """One token on shapes whose warp count is not a multiple of the CTA size:
    the CTA-pair launch rounds the grid up to an even count (the extra CTA
    holds no units), and with few rows and a long K a single row pair spans
    many CTAs, so its last CTA adds many workspace partials.  Same bits as
    the two-kernel path, repeatable through one workspace, and the oracle's
    values within the bars."""
    c = O.convert_weight(synth.weights(n, k, synth.rng_for(71, n + k, "weight")), sample_cap=2**16)
    packed = pack(lib, c)
    bits, x, _ = synth.activations(1, k, synth.rng_for(11, n + k, "act"), max(1, k // 100))
    xt = bf16(bits)
    ws = lib.linear_workspace(1, k, n, "cuda")
    y_one = lib.linear(xt, packed, n, workspace=ws)
    y_again = lib.linear(xt, packed, n, workspace=ws)
    assert torch.equal(y_one.view(torch.int16), y_again.view(torch.int16))
    lib.linear_prepare(xt, n, ws)
    y_two = lib.linear_run(1, k, packed, n, ws)
    assert torch.equal(y_one.view(torch.int16), y_two.view(torch.int16))
    wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
    check_linear(y_one.float().cpu().numpy(), O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"]), x, wmax)


# The words at the start of every workspace that join partial sums across
# CTAs: per CTA boundary (148) 32 eight-byte exchange words and one 4-byte
# arrival counter, rounded up to 256 bytes.
ZERO_REGION_BYTES = (148 * 32 * 8 + 148 * 4 + 255) // 256 * 256


@pytest.mark.parametrize("m,k,n", [(1, 5120, 17408), (1, 17408, 5120), (1, 8448, 16), (4, 17408, 5120),
                                   (16, 5120, 4096), (40, 768, 592), (300, 768, 592)])
def test_workspace_zero_region_left_at_zero(lib, m, k, n):
    """Every completed call, whatever its path (one-token kernel, two-kernel
    path, 2-16-token decode, slices, GEMM), leaves the exchange words and
    arrival counters at zero, which is what the next call on the workspace
    needs; and a region filled with garbage by nothing else stays so."""
    q = synth.quantized_format_device(n, k, seed=5, device="cuda")
    packed = lib.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    bits, _, _ = synth.activations(m, k, synth.rng_for(17, m + k, "act"), max(1, k // 100))
    xt = bf16(bits)
    ws = lib.linear_workspace(m, k, n, "cuda")
    assert ws.numel() > ZERO_REGION_BYTES
    y = lib.linear(xt, packed, n, workspace=ws)
    torch.cuda.synchronize()
    assert int(ws[:ZERO_REGION_BYTES].count_nonzero()) == 0
    if m <= 64:
        lib.linear_prepare(xt, n, ws)
        y_run = lib.linear_run(m, k, packed, n, ws)
        torch.cuda.synchronize()
        assert int(ws[:ZERO_REGION_BYTES].count_nonzero()) == 0
        assert torch.equal(y.view(torch.int16), y_run.view(torch.int16))


def test_one_workspace_shared_by_layers_of_different_shapes(lib):
    """A decode step shares one workspace among layers of different (K, N)
    (and token counts): each call gives the same bits as with a fresh
    workspace of its own, in any order, twice over."""
    shapes = [(768, 592), (8448, 16), (17408, 272), (5120, 2048), (256, 4096)]
    layers, xs, fresh = [], [], []
    for i, (k, n) in enumerate(shapes):
        q = synth.quantized_format_device(n, k, seed=30 + i, device="cuda")
        layers.append(lib.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"]))
        m = 1 if i % 2 == 0 else 3
        bits, _, _ = synth.activations(m, k, synth.rng_for(23, i, "act"), max(1, k // 100))
        xs.append(bf16(bits))
        fresh.append(lib.linear(xs[-1], layers[-1], n).clone())
    need = max(lib.linear_workspace_bytes(x.shape[0], k, n) for x, (k, n) in zip(xs, shapes))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    for order in (range(len(shapes)), reversed(range(len(shapes))), [0, 2, 4, 1, 3]):
        for i in order:
            k, n = shapes[i]
            y = lib.linear(xs[i], layers[i], n, workspace=ws)
            assert torch.equal(y.view(torch.int16), fresh[i].view(torch.int16)), shapes[i]


GUARD = 64  # elements of guard band on each side of an output (keeps 16-byte alignment)


@pytest.mark.parametrize("m,k,n", [(1, 768, 592), (1, 8448, 16), (1, 17408, 272), (5, 768, 592), (16, 256, 16),
                                   (40, 768, 592), (300, 768, 592)])
def test_outputs_leave_guard_bands_untouched(lib, m, k, n):
    """y written into the middle of a larger buffer filled with a canary
    pattern: every path writes exactly its [M, N] outputs (the canaries on
    both sides survive) and the same bits as into a buffer of its own; the
    same for the standalone dequant's fp32 output."""
    q = synth.quantized_format_device(n, k, seed=9, device="cuda")
    packed = lib.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    bits, _, _ = synth.activations(m, k, synth.rng_for(21, m + k, "act"), max(1, k // 100))
    xt = bf16(bits)
    canary = 0x7BAD
    buf = torch.full((m * n + 2 * GUARD,), canary, dtype=torch.int16, device="cuda")
    y = buf[GUARD:GUARD + m * n].view(torch.bfloat16).view(m, n)
    lib.linear(xt, packed, n, out=y)
    ref = lib.linear(xt, packed, n)
    torch.cuda.synchronize()
    assert bool((buf[:GUARD] == canary).all()) and bool((buf[GUARD + m * n:] == canary).all())
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    if m == 1:
        dbuf = torch.full((n * k + 2 * GUARD,), -7.25, dtype=torch.float32, device="cuda")
        st = lib.load_library().w4a8_unpack_dequant(packed.data_ptr(), n, k, dbuf[GUARD:].data_ptr(),
                                                    torch.cuda.current_stream().cuda_stream)
        assert st == 0
        torch.cuda.synchronize()
        assert bool((dbuf[:GUARD] == -7.25).all()) and bool((dbuf[GUARD + n * k:] == -7.25).all())
        assert torch.equal(dbuf[GUARD:GUARD + n * k].view(n, k), lib.unpack_dequant(packed, n, k))


@pytest.mark.parametrize("m", [1, 3, 20, 80])
def test_linear_zero_token_and_zero_rows(lib, m):
    """An all-zero token gives s_x = 0 and a zero output row; an all-zero
    weight row gives s_channel = 0 and a zero output column; every path
    (one-token kernel, decode, sliced decode, GEMM) and the oracle agree."""
    n, k = 592, 768
    w = synth.weights(n, k, synth.rng_for(13, 0, "weight"))
    w[[0, 17, 591]] = 0.0
    c = O.convert_weight(w)
    assert c["s_ch"][0] == 0 and c["s_ch"][591] == 0
    packed = pack(lib, c)
    bits, x, _ = synth.activations(m, k, synth.rng_for(13, m, "act"), 8)
    bits[m - 1] = 0
    x[m - 1] = 0.0
    y = run_linear(lib, bits, packed, n)
    assert np.all(y[m - 1] == 0.0)
    assert np.all(y[:, [0, 17, 591]] == 0.0)
    if m > 1:
        wmax = float(np.abs(O.dequant(c["idx"], c["s_rel"], c["s_ch"], c["cb"])).max())
        ref = O.linear(x, c["idx"], c["s_rel"], c["s_ch"], c["cb"])
        check_linear(y[: m - 1], ref[: m - 1], x[: m - 1], wmax)
