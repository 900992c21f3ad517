"""GPU tests of w4a8_linear_flagged: the layer waits on the GPU for a ready
word that the caller's copy writes after x, instead of a stream dependency
on that copy (which would cost the overlap of consecutive layers)."""

import numpy as np
import pytest
import torch

import synth

pytestmark = pytest.mark.gpu


def _layer(lib, n, k, seed):
    q = synth.quantized_format(n, k, synth.rng_for(60, seed, "qfmt"))
    t = {kk: torch.from_numpy(np.ascontiguousarray(v)).cuda() for kk, v in q.items()}
    return lib.pack_layout(t["packed"], t["s_rel"], t["s_ch"], t["cb"])


@pytest.mark.parametrize("m,k,n", [(1, 5120, 1024), (1, 9216, 512), (4, 768, 592), (100, 512, 256)])
def test_flagged_equals_linear_and_clears_its_flag(lib, m, k, n):
    packed = _layer(lib, n, k, k + m)
    x = torch.randn((m, k), device="cuda").to(torch.bfloat16)
    ref = lib.linear(x, packed, n)
    ws = lib.linear_workspace(m, k, n, "cuda")
    ready = torch.tensor([1, 0], dtype=torch.int32, device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    for _ in range(2):
        ready[0] = 1
        lib.linear_flagged(x, packed, n, ready, ws, y)
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
        assert ready.tolist() == [0, 0]  # cleared for the caller's next copy
    assert lib.get_device_error() == 0


def test_flagged_input_from_a_copy_on_another_stream(lib):
    """x and its ready word arrive by copies on a second stream; the layer's
    stream never waits on that stream's events."""
    m, k, n = 1, 5120, 2048
    packed = _layer(lib, n, k, 7)
    x_host = torch.randn((m, k)).to(torch.bfloat16).pin_memory()
    one = torch.tensor([1, 0], dtype=torch.int32).pin_memory()
    ref = lib.linear(x_host.cuda(), packed, n)
    x_dev = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    ready = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = lib.linear_workspace(m, k, n, "cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    copy = torch.cuda.Stream()
    torch.cuda.synchronize()
    lib.linear_flagged(x_dev, packed, n, ready, ws, y)     # launched first: waits on the GPU
    with torch.cuda.stream(copy):
        x_dev.copy_(x_host, non_blocking=True)
        ready[:1].copy_(one[:1], non_blocking=True)          # after the data, same stream
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert ready.tolist() == [0, 0]
    assert lib.get_device_error() == 0


def test_flagged_wait_runs_out_and_reports_a_timeout(lib):
    """A ready word nothing sets: the bounded wait gives up (about a second),
    the call records a timeout, and the context stays usable."""
    m, k, n = 1, 512, 256
    packed = _layer(lib, n, k, 9)
    x = torch.randn((m, k), device="cuda").to(torch.bfloat16)
    ws = lib.linear_workspace(m, k, n, "cuda")
    ready = torch.zeros(2, dtype=torch.int32, device="cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    lib.linear_flagged(x, packed, n, ready, ws, y)
    assert lib.get_device_error() == 6  # W4A8_ERR_TIMEOUT, read and cleared
    ready.zero_()
    ws.zero_()  # the workspace after a timeout, as the header asks
    ready[0] = 1
    lib.linear_flagged(x, packed, n, ready, ws, y)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), lib.linear(x, packed, n).view(torch.int16))
    assert lib.get_device_error() == 0


def test_flagged_pipeline_of_distinct_tokens(lib):
    """Consecutive one-token calls on one stream (so each may start while the
    previous one runs), each token delivered by a copy and its ready word on
    another stream into one of three buffer sets that are reused once the
    call that read them is done.  Every step's output equals the plain
    layer's on that token."""
    m, k, n, steps, nbuf = 1, 5120, 4096, 12, 3
    packed = _layer(lib, n, k, 11)
    xs_host = [torch.randn((m, k)).mul(1 + i).to(torch.bfloat16).pin_memory() for i in range(steps)]
    refs = [lib.linear(xh.cuda(), packed, n) for xh in xs_host]
    one = torch.tensor([1, 0], dtype=torch.int32).pin_memory()
    xs = [torch.zeros((m, k), dtype=torch.bfloat16, device="cuda") for _ in range(nbuf)]
    flags = [torch.zeros(2, dtype=torch.int32, device="cuda") for _ in range(nbuf)]
    ys = [torch.empty((m, n), dtype=torch.bfloat16, device="cuda") for _ in range(steps)]
    done = [torch.cuda.Event() for _ in range(nbuf)]
    ws = lib.linear_workspace(m, k, n, "cuda")
    comp, copy = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for i in range(steps):
        b = i % nbuf
        if i >= nbuf:
            copy.wait_event(done[b])  # the call that read this set is done
        with torch.cuda.stream(copy):
            xs[b].copy_(xs_host[i], non_blocking=True)
            flags[b][:1].copy_(one[:1], non_blocking=True)
        lib.linear_flagged(xs[b], packed, n, flags[b], ws, ys[i], stream=comp)
        done[b].record(comp)
    torch.cuda.synchronize()
    for i in range(steps):
        assert torch.equal(ys[i].view(torch.int16), refs[i].view(torch.int16)), i
    assert all(f.tolist() == [0, 0] for f in flags)
    assert lib.get_device_error() == 0


def test_ready_word_written_by_the_copy_stream(lib):
    """w4a8_signal_ready after the copy of x on the copy stream: the layer,
    launched first on its own stream, sees x complete."""
    m, k, n = 1, 5120, 2048
    packed = _layer(lib, n, k, 13)
    x_host = torch.randn((m, k)).to(torch.bfloat16).pin_memory()
    ref = lib.linear(x_host.cuda(), packed, n)
    x_dev = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    ready = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = lib.linear_workspace(m, k, n, "cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    comp, copy = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    lib.linear_flagged(x_dev, packed, n, ready, ws, y, stream=comp)
    with torch.cuda.stream(copy):
        x_dev.copy_(x_host, non_blocking=True)
    lib.signal_ready(ready, stream=copy)
    torch.cuda.synchronize()
    assert torch.equal(y.view(torch.int16), ref.view(torch.int16))
    assert ready.tolist() == [0, 0]
    assert lib.get_device_error() == 0


def test_ready_word_signal_in_a_captured_graph(lib):
    """The copy, the stream-written ready word and the layer captured into one
    CUDA graph (copy and layer on separate captured streams, no edge between
    them), replayed with new tokens."""
    m, k, n = 1, 5120, 2048
    packed = _layer(lib, n, k, 14)
    x_host = torch.empty((m, k), dtype=torch.bfloat16).pin_memory()
    x_dev = torch.zeros((m, k), dtype=torch.bfloat16, device="cuda")
    ready = torch.zeros(2, dtype=torch.int32, device="cuda")
    ws = lib.linear_workspace(m, k, n, "cuda")
    y = torch.empty((m, n), dtype=torch.bfloat16, device="cuda")
    side, copy = torch.cuda.Stream(), torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        copy.wait_stream(side)
        with torch.cuda.stream(copy):
            x_dev.copy_(x_host, non_blocking=True)
        lib.signal_ready(ready, stream=copy)
        lib.linear_flagged(x_dev, packed, n, ready, ws, y, stream=side)
        side.wait_stream(copy)
    torch.cuda.current_stream().wait_stream(side)
    for rep in range(3):
        x_host.copy_(torch.randn((m, k)).mul(rep + 1).to(torch.bfloat16))
        g.replay()
        torch.cuda.synchronize()
        ref = lib.linear(x_host.cuda(), packed, n)
        assert torch.equal(y.view(torch.int16), ref.view(torch.int16)), rep
        assert ready.tolist() == [0, 0]
    assert lib.get_device_error() == 0
