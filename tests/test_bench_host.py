"""Host-side pieces of the benchmark that need no GPU: the algorithmic byte
count of a layer, and the rule that a committed DRAM-traffic figure is only
reported while the kernel source it was captured from is unchanged."""

from __future__ import annotations

import json
import os

import pytest

import bench


def test_weight_bytes_is_the_packed_layer():
    # 0.5 B of index and 1/16 B of group scale per weight, 4 B per row, 64 B of codebook
    assert bench.weight_bytes(17408, 5120) == 17408 * 5120 // 2 + 17408 * 5120 // 16 + 4 * 17408 + 64
    assert bench.weight_bytes(17408, 5120) == 50204736


def test_committed_traffic_matches_its_source_hash():
    with open(os.path.join(bench.ROOT, "profiles", "traffic.json")) as f:
        d = json.load(f)
    for kernel, srcs in bench.TRAFFIC_SOURCES.items():
        if kernel not in d:
            assert bench.profiled_traffic(kernel, srcs) is None
            continue
        got = bench.profiled_traffic(kernel, srcs)
        if d[kernel]["source_sha256_16"] == bench.kernel_source_hash(srcs):
            assert got == pytest.approx(d[kernel]["dram_bytes_per_launch"])
            # every capture is of a launch that reads a whole 17408 x 5120 layer (its 4-bit codes
            # and e4m3 scales, 50.1 MB) at least once
            assert got >= 17408 * 5120 * (0.5 + 1 / 16)
        else:
            assert got is None


def test_one_token_hash_covers_the_shared_helpers_only():
    """The one-token kernel's hash takes gemv.cuh up to the multi-token body:
    the marker is there once, the part before it holds what the one-token
    kernel uses (its parameters, its wait), and the body is outside it."""
    with open(os.path.join(bench.ROOT, "w4a8_codebook_quantized_rotate_b200", "csrc", "gemv.cuh")) as f:
        text = bench.strip_comments(f.read())
    assert text.count(bench.DECODE_MULTI_BODY) == 1
    head = text[:text.find(bench.DECODE_MULTI_BODY)]
    assert "struct DecodeParams" in head and "struct DecWaitPdl" in head
    assert "decode_body" not in head and "decode_kernel" not in head
    gemv1 = open(os.path.join(bench.ROOT, "w4a8_codebook_quantized_rotate_b200", "csrc", "gemv1.cuh")).read()
    assert "decode_body" not in bench.strip_comments(gemv1)  # the one-token kernel never calls it
    with pytest.raises(ValueError):
        bench.kernel_source_hash([("gemv.cuh", "no such text")])


def test_traffic_is_withheld_when_the_source_changes(tmp_path, monkeypatch):
    (tmp_path / "profiles").mkdir()
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(
        {"k": {"source_sha256_16": "0" * 16, "dram_bytes_per_launch": 123}}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "1" * 16)
    assert bench.profiled_traffic("k", ["x"]) is None
    monkeypatch.setattr(bench, "kernel_source_hash", lambda files: "0" * 16)
    assert bench.profiled_traffic("k", ["x"]) == 123
    assert bench.profiled_traffic("missing", ["x"]) is None


def test_source_hash_ignores_comments_only():
    a = "int f(int x) {\n  return x + 1;  // one more\n}\n"
    b = "/* a block\n   comment */\nint f(int x) {\n\n  return x + 1;\n}  // trailing\n"
    c = "int f(int x) {\n  return x + 2;\n}\n"
    assert bench.strip_comments(a) == bench.strip_comments(b)
    assert bench.strip_comments(a) != bench.strip_comments(c)


def test_oracle_pool_splits_rows_over_processes():
    import numpy as np
    import synth
    q = synth.quantized_format(64, 256, synth.rng_for(9, 0, "qfmt"))
    _, x, _ = synth.activations(1, 256, synth.rng_for(9, 0, "act"), 2)
    pool = bench.OraclePool(q, x)
    try:
        assert 1 <= pool.workers <= bench.OraclePool.MAX_WORKERS
        assert pool.run(48) > 0.0
    finally:
        pool.close()
    assert np.isfinite(bench.weight_bytes(48, 256))


def test_c2_path_names_follow_the_library_rule():
    assert bench.c2_path(1, 17408, 5120).startswith("one-token")
    assert bench.c2_path(4, 17408, 5120) == "decode"
    assert bench.c2_path(16, 17408, 5120) == "decode"
    assert bench.c2_path(17, 17408, 5120) == "decode, 32-token variant"
    assert bench.c2_path(32, 17408, 5120) == "decode, 32-token variant"
    assert bench.c2_path(64, 17408, 5120) == "decode, slices of 32"
    assert bench.c2_path(65, 17408, 5120).startswith("small-batch")
    assert bench.c2_path(128, 17408, 5120).startswith("small-batch")
    assert bench.c2_path(128, 5120, 17408) == "tensor-core GEMM"
    assert bench.c2_path(256, 17408, 5120).startswith("small-batch")
    assert bench.c2_path(257, 17408, 5120) == "tensor-core GEMM"
