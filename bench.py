"""Benchmark of the asym_w4a8_int8 ConvRot linear layer on B200.

Headline workload: decode GEMV, M=1 token, K=5120, N=17408 (an MLP gate/up
projection of a 27B hybrid decoder), weights cycled over 8 distinct copies
(8 x 50.2 MB > the 126 MB L2) so every step streams its weights from HBM.
A step is one pass of the layer: w4a8_linear, which for one token is a
single kernel (every CTA rotates and quantises x, then streams its share of
the weights).  Metric: weight GB/s = weight bytes per step / time per step.

Also reported in the same line: that kernel's roofline against measured HBM
bandwidth, the decode kernel on activations prepared once (the two-kernel
path's second half, timed alone), the prefill GEMM at M=4096, K=5120,
N=17408 (TOPS against the measured dense fp16/bf16 tensor peak), an
end-to-end figure through the C ABI with host buffers, SM clocks sampled
during the timed regions, and the CPU oracle timed on a bounded sample.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

N > 1 is launched by torchrun, one process per GPU; every rank runs an
independent replica of the workload (the layer needs no exchange between
GPUs for these shapes), the timed region is bracketed by a barrier and a
device synchronisation, and the time is the maximum over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

M_DEC, K_DEC, N_DEC = 1, 5120, 17408
M_PRE, K_PRE, N_PRE = 4096, 5120, 17408
COPIES = 8
METRIC = "w4a8_linear weight GB/s at M=1 and TOPS at M=4096, % of B200 roofline"


def weight_bytes(n: int, k: int) -> int:
    """Algorithmic bytes of one layer: indices 0.5 B/weight, e4m3 scales
    1/16 B/weight, fp32 row scales, 16 fp32 levels."""
    return n * k // 2 + n * k // 16 + 4 * n + 64


def measured_peaks() -> dict:
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained"), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def strip_comments(src: str) -> str:
    """C/C++ source without its comments and blank lines, trailing spaces
    removed: what the compiler sees, so that a comment edit does not change
    the hash below.  (The kernel sources have no comment markers inside
    string literals.)"""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(ln.rstrip() for ln in src.splitlines() if ln.strip()) + "\n"


def kernel_source_hash(files) -> str:
    """Hash of the comment-stripped kernel sources a traffic figure was
    captured from.  An entry (file, marker) covers the file's stripped text
    before `marker` only: the part a kernel compiles against when the rest
    of the file holds other kernels (a missing marker is an error)."""
    h = hashlib.sha256()
    for f in files:
        name, marker = f if isinstance(f, tuple) else (f, None)
        with open(os.path.join(ROOT, "w4a8_codebook_quantized_rotate_b200", "csrc", name)) as fh:
            text = strip_comments(fh.read())
        if marker is not None:
            cut = text.find(marker)
            if cut < 0:
                raise ValueError(f"{name}: marker not found")
            text = text[:cut]
        h.update(text.encode())
    return h.hexdigest()[:16]


# The sources of each kernel with a committed traffic figure.  The one-token
# kernel includes gemv.cuh for the helpers it shares with the multi-token
# kernel, whose body (from decode_body on) it does not use.
DECODE_MULTI_BODY = "template <int NB, int D, class Wait>\n__device__ __forceinline__ void decode_body"
TRAFFIC_SOURCES = {
    "decode_one_kernel_fused": ["gemv1.cuh", ("gemv.cuh", DECODE_MULTI_BODY), "act.cuh", "common.cuh"],
    "gemm_tc_kernel": ["gemm_tc.cuh", "common.cuh"],
    "nvfp4_gemm_kernel_prefill": ["nvfp4.cuh", "act.cuh", "common.cuh"],
    "gemm_sk_kernel_m128": ["gemm_sk.cuh", "gemm_tc.cuh", "common.cuh"],
}


def profiled_traffic(kernel: str, files=None) -> float | None:
    """DRAM bytes per launch from a committed ncu capture, if the kernel
    source is unchanged since the capture."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        d = json.load(f).get(kernel)
    if not d or d.get("source_sha256_16") != kernel_source_hash(files or TRAFFIC_SOURCES[kernel]):
        return None
    return float(d["dram_bytes_per_launch"])


def graph_loop(step, k, stream, chunk=128):
    """Capture `step(i)` for i in [0, k) into CUDA graphs of at most `chunk`
    steps (one graph for the full chunks, one for the remainder) and return
    a function that replays them in order, i.e. runs exactly k steps."""
    import torch
    graphs = []
    side = torch.cuda.Stream()
    side.wait_stream(stream)
    done = 0
    full, rem = divmod(k, chunk)
    for size, reps in ((chunk, full), (rem, 1 if rem else 0)):
        if reps == 0 or size == 0:
            continue
        g = torch.cuda.CUDAGraph()
        base = done
        with torch.cuda.graph(g, stream=side):
            for i in range(size):
                step(base + i)
        graphs.append((g, reps))
        done += size * reps
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def replay():
        for g, reps in graphs:
            for _ in range(reps):
                g.replay()
    return replay


class ClockSampler:
    """Samples SM clock and clock-event reasons through NVML while running."""

    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown",
               0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, index: int, period_s: float = 0.002):
        self.samples, self.reasons, self.max_mhz = [], set(), None
        self.period, self._stop, self._ok = period_s, threading.Event(), False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            self.h = pynvml.nvmlDeviceGetHandleByIndex(index)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self._ok = True
        except Exception:
            self.nv = None

    def _reasons(self):
        try:
            return self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            return self.nv.nvmlDeviceGetCurrentClocksThrottleReasons(self.h)

    def _run(self):
        while not self._stop.is_set():
            try:
                self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
                bits = self._reasons()
                for b, name in self.REASONS.items():
                    if bits & b:
                        self.reasons.add(name)
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self._ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self._ok:
            self._stop.set()
            self._t.join()

    def summary(self) -> dict:
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": ["unavailable"]}
        return {"sm_mhz": statistics.median(self.samples), "sm_max_mhz": self.max_mhz,
                "reasons": sorted(self.reasons), "samples": len(self.samples)}


# ----------------------------------------------------------------------- CPU side (oracle)

def oracle_sample(rows: int):
    """Bounded sample of the decode workload for the CPU oracle: the first
    ``rows`` output rows of a synthetic C1 layer and one token."""
    import synth
    q = synth.quantized_format(N_DEC, K_DEC, synth.rng_for(1, 0, "qfmt"))
    bits, x, _ = synth.activations(M_DEC, K_DEC, synth.rng_for(1, 0, "act"), K_DEC // 100)
    return q, bits, x


def time_oracle(q, x, rows: int, reps: int):
    """Oracle linear on ``rows`` output rows, ``reps`` times, one BLAS thread.
    Returns (seconds per rep, weight bytes per rep, the last rep's output)."""
    import oracle as O
    from threadpoolctl import threadpool_limits
    sel = np.arange(rows)
    y = None
    with threadpool_limits(limits=1):
        O.linear_packed(x, q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=sel[: min(rows, 64)])  # warm
        t0 = time.perf_counter()
        for _ in range(reps):
            y = O.linear_packed(x, q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=sel)
        dt = (time.perf_counter() - t0) / reps
    return dt, weight_bytes(rows, K_DEC), y


_POOL = {}


def _pool_init(q, x):
    """Worker start-up: keep the sample, one BLAS thread per process."""
    from threadpoolctl import threadpool_limits
    _POOL["q"], _POOL["x"] = q, x
    _POOL["limits"] = threadpool_limits(limits=1)


def _pool_rows(lo: int, hi: int) -> int:
    import oracle as O
    q = _POOL["q"]
    O.linear_packed(_POOL["x"], q["packed"], q["s_rel"], q["s_ch"], q["cb"], rows=np.arange(lo, hi))
    return hi - lo


def host_cores() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count() or 1


class OraclePool:
    """The oracle, as it stands, run on all host cores: one spawned process
    per core, each with one BLAS thread, each taking a contiguous slice of
    the sampled output rows.  (Spawned, not forked: the parent may hold a
    CUDA context.)"""

    MAX_WORKERS = 64  # bounds the sample copies held by the workers

    def __init__(self, q, x):
        import concurrent.futures as cf
        import multiprocessing as mp
        self.workers = max(1, min(host_cores(), self.MAX_WORKERS))
        self.ex = cf.ProcessPoolExecutor(self.workers, mp_context=mp.get_context("spawn"),
                                         initializer=_pool_init, initargs=(q, x))
        # start every worker and warm it (imports, first call)
        list(self.ex.map(_pool_rows, [0] * self.workers, [16] * self.workers))

    def run(self, rows: int) -> float:
        """Seconds (wall clock) for one pass over the first `rows` rows."""
        cuts = np.linspace(0, rows, self.workers + 1).astype(int)
        t0 = time.perf_counter()
        done = sum(self.ex.map(_pool_rows, cuts[:-1].tolist(), cuts[1:].tolist()))
        dt = time.perf_counter() - t0
        assert done == rows
        return dt

    def close(self):
        self.ex.shutdown()


def blas_threads() -> int | None:
    try:
        from threadpoolctl import threadpool_info
        return max((i.get("num_threads") or 0) for i in threadpool_info() if i.get("user_api") == "blas") or None
    except Exception:
        return None


def cpu_baseline(budget_s: float = 15.0, B=None, torch=None, dev=None) -> dict:
    """The oracle timed on a bounded row sample of the C1 layer.  With the
    library at hand (B), the same layer also runs through w4a8_linear on the
    GPU and the sampled rows are compared with the oracle's (relative L2,
    and the largest per-row error over the bar 1e-2 * ||x|| * max|W_hat|)."""
    q, bits, x = oracle_sample(N_DEC)
    dt1, _, _ = time_oracle(q, x, 1024, 1)
    rows = int(min(N_DEC, max(256, 1024 * (budget_s / 3) / max(dt1, 1e-6))))
    rows -= rows % 16
    reps = max(1, int(budget_s / max(dt1 * rows / 1024, 1e-6)))
    reps = min(reps, 5)
    dt, nbytes, y_ref = time_oracle(q, x, rows, reps)
    single = {"value": nbytes / dt / 1e9, "unit": "GB/s", "cores": 1, "kind": "oracle",
              "sample": f"oracle linear (rotate+quantise x, three-tier dequant, fp64 matmul) on {rows} of "
                        f"{N_DEC} output rows of the M=1 K=5120 layer, {reps} repeats, 1 thread"}
    # all host cores: the whole layer, split by rows over one process per core
    pool = OraclePool(q, x)
    try:
        dt_all = min(pool.run(N_DEC) for _ in range(2))
    finally:
        pool.close()
    out = {"value": weight_bytes(N_DEC, K_DEC) / dt_all / 1e9, "unit": "GB/s", "cores": pool.workers,
           "kind": "oracle",
           "sample": f"oracle linear on all {N_DEC} output rows of the M=1 K=5120 layer, split by rows over "
                     f"{pool.workers} processes (one per host core, 1 BLAS thread each), best of 2 passes",
           "os_cpu_count": os.cpu_count(), "blas_threads_per_process": 1,
           "blas_threads_default": blas_threads(), "single_thread": single}
    if B is not None:
        import oracle as O
        t = {kk: torch.from_numpy(np.ascontiguousarray(v)).to(dev) for kk, v in q.items()}
        packed = B.pack_layout(t["packed"], t["s_rel"], t["s_ch"], t["cb"])
        xt = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
        y = B.linear(xt, packed, N_DEC)[:, :rows].double().cpu().numpy()
        err = y - y_ref
        wmax = float(np.abs(O.dequant_packed(q["packed"], q["s_rel"], q["s_ch"], q["cb"],
                                             rows=np.arange(rows))).max())
        bar = 1e-2 * np.linalg.norm(np.asarray(x, dtype=np.float64), axis=1) * wmax
        out["parity"] = {"rows": rows,
                         "rel_l2": float(np.linalg.norm(err) / np.linalg.norm(y_ref)),
                         "max_abs_over_bar": float((np.abs(err).max(axis=1) / bar).max()),
                         "how": "the same seeded layer and token through w4a8_linear on the GPU (one "
                                "kernel), its first rows against the oracle's; bars: rel_l2 <= 2e-3, "
                                "max_abs_over_bar <= 1"}
    return out


def max_over_ranks(v: float, world: int, device) -> float:
    """The maximum of a per-rank figure over the process group (the time of
    the slowest rank); the value itself when running alone."""
    if world == 1:
        return v
    import torch
    import torch.distributed as dist
    t = torch.tensor([v], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(bytes_per_rank_step: float, world: int, steps: int, ms: float) -> float:
    """Whole-job GB/s: every rank streams its own replica's bytes each step;
    the time is the slowest rank's."""
    return world * bytes_per_rank_step * steps / (ms * 1e-3) / 1e9


def run_reference(args) -> None:
    """The reference arm: the oracle (the only other implementation of the
    layer) on all host cores, each step one pass over a bounded row sample of
    the decode layer sized so that warm-up and timed steps take about
    ``--ref-seconds`` in all.  Rank 0 alone runs it."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    q, _, x = oracle_sample(N_DEC)
    pool = OraclePool(q, x)
    try:
        dt_full = pool.run(N_DEC)
        per_step = args.ref_seconds / max(1, args.steps + args.warmup)
        rows = N_DEC if dt_full <= per_step else int(N_DEC * per_step / dt_full)
        rows = max(16, rows - rows % 16)
        for _ in range(args.warmup):
            pool.run(rows)
        t0 = time.perf_counter()
        for _ in range(args.steps):
            pool.run(rows)
        dt = (time.perf_counter() - t0) / args.steps
    finally:
        pool.close()
    value = weight_bytes(rows, K_DEC) / dt / 1e9
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": dt * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"decode GEMV M={M_DEC} K={K_DEC} N={N_DEC} (bounded row sample per step)",
                   "rows_per_step": rows},
        "cpu_baseline": {"value": value, "unit": "GB/s", "cores": pool.workers, "kind": "oracle",
                         "sample": f"{rows} of {N_DEC} output rows per step, split over {pool.workers} "
                                   f"processes (one per host core, 1 BLAS thread each)",
                         "os_cpu_count": os.cpu_count()},
        "e2e": {"value": value, "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ----------------------------------------------------------------------- GPU side

C3_BLOCKS = 62
C3_SHAPES = (("qkv", 5120, 10240), ("out", 5120, 5120), ("gate", 5120, 17408), ("up", 5120, 17408),
             ("down", 17408, 5120))


def c2_path(m: int, k: int, n: int) -> str:
    """Which kernel w4a8_linear runs for (M, K, N) (the library's rule)."""
    if m == 1:
        return "one-token decode (activation step fused)"
    if 65 <= m <= 256 and (n + 127) // 128 < 100:
        return "small-batch tensor-core (stream-K)"
    if m <= 16:
        return "decode"
    if m <= 32:
        return "decode, 32-token variant"
    if m <= 64:
        return "decode, slices of 32"
    return "tensor-core GEMM"


def measure_c2(B, synth, torch, dev, rank, stream, steps, warmup):
    """Down-projection shape K=17408, N=5120 at several token counts, 8 weight
    copies cycled; `path` names the kernel each count takes (c2_path); the
    per-call and per-token times show the crossover from the weight-bound
    decode kernels to the tensor-core kernels."""
    k, n = 17408, 5120
    copies = []
    for c in range(COPIES):
        q = synth.quantized_format_device(n, k, seed=2000 * (rank + 1) + c, device=dev)
        copies.append(B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"]))
        del q
    wbytes = weight_bytes(n, k)
    out = {}
    for m in (1, 4, 16, 32, 64, 128, 256):
        g = torch.Generator(device=dev)
        g.manual_seed(300 + m)
        x = torch.randn((m, k), generator=g, device=dev).to(torch.bfloat16)
        ws = B.linear_workspace(m, k, n, dev)
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        st = steps if m <= 16 else max(8, steps // 8)

        def step(i):
            B.linear(x, copies[i % COPIES], n, workspace=ws, out=y)

        for i in range(warmup):
            step(i)
        replay = graph_loop(step, st, stream)
        replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay()
        e1.record(stream)
        torch.cuda.synchronize()
        us = e0.elapsed_time(e1) * 1e3 / st
        out[f"M={m}"] = {"us_per_call": us, "weight_GBs": wbytes / us / 1e3,
                         "us_per_token": us / m, "TOPS": 2.0 * m * n * k / us / 1e6,
                         "path": c2_path(m, k, n)}
        if m == 128:  # the small-batch kernel's DRAM bytes from its committed capture at this size
            out[f"M={m}"]["traffic"] = profiled_traffic("gemm_sk_kernel_m128")
        del replay
    del copies
    torch.cuda.empty_cache()
    return {"workload": f"K={k} N={n}, 8 weight copies cycled, one w4a8_linear per call", "by_m": out}


def measure_c1_rate(B, synth, torch, dev, rank, stream, steps=400, copies=4):
    """The one-token layer at K=5120 with N = 17408 x {1, 2, 4, 8} (4 weight
    copies cycled, all larger than L2 together): the time per extra 50.2 MB is
    the streaming loop's rate, and the line through the points at N = 0 is the
    per-call cost that does not scale with the weights (the wait for the
    previous grid, the activation step, the tail)."""
    k = 5120
    pts = []
    for mult in (1, 2, 4, 8):
        n = 17408 * mult
        ws_ = []
        for c in range(copies):
            q = synth.quantized_format_device(n, k, seed=5000 * (rank + 1) + 10 * mult + c, device=dev)
            ws_.append(B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"]))
            del q
        g = torch.Generator(device=dev)
        g.manual_seed(500 + mult)
        x = torch.randn((1, k), generator=g, device=dev).to(torch.bfloat16)
        ws = B.linear_workspace(1, k, n, dev)
        y = torch.empty((1, n), dtype=torch.bfloat16, device=dev)
        st = max(40, steps // mult)

        def step(i):
            B.linear(x, ws_[i % copies], n, workspace=ws, out=y)

        for i in range(5):
            step(i)
        replay = graph_loop(step, st, stream)
        replay()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay()
        e1.record(stream)
        torch.cuda.synchronize()
        pts.append((weight_bytes(n, k), e0.elapsed_time(e1) * 1e3 / st))
        del replay, ws_
        torch.cuda.empty_cache()
    xs = [b for b, _ in pts]
    ys = [t for _, t in pts]
    xm, ym = sum(xs) / len(xs), sum(ys) / len(ys)
    slope = sum((a - xm) * (b - ym) for a, b in zip(xs, ys)) / sum((a - xm) ** 2 for a in xs)  # us per byte
    return {"workload": "M=1 K=5120, N = 17408 x {1,2,4,8}, 4 weight copies cycled, one w4a8_linear per call",
            "us_per_call": {str(17408 * m): round(t, 3) for m, (_, t) in zip((1, 2, 4, 8), pts)},
            "stream_GBs": 1e-3 / slope,
            "fixed_us": ym - slope * xm,
            "how": "least-squares line of time per call against weight bytes"}


def measure_c3(B, synth, torch, dev, rank, stream, steps, warmup):
    """Decode step of a 62-block stack of projections, M=1, all weights
    distinct and resident.  Per block the projections run as a chain:
    h -> qkv (10240) -> out (its first 5120) -> gate and up (17408 each) ->
    down (from up) -> next h; every call is one w4a8_linear."""
    layers = []
    total = 0
    for b in range(C3_BLOCKS):
        blk = []
        for j, (name, k, n) in enumerate(C3_SHAPES):
            q = synth.quantized_format_device(n, k, seed=100000 * (rank + 1) + 10 * b + j, device=dev)
            blk.append((B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"]), k, n))
            del q
            total += weight_bytes(n, k)
        layers.append(blk)
    resident = sum(pk.numel() for blk in layers for pk, _, _ in blk)
    ws = B.linear_workspace(1, 17408, 17408, dev)
    need = max(B.linear_workspace_bytes(1, k, n) for _, k, n in C3_SHAPES)
    assert ws.numel() >= need
    g = torch.Generator(device=dev)
    g.manual_seed(7 + rank)
    h0 = torch.randn((1, 5120), generator=g, device=dev).to(torch.bfloat16)
    bufs = {n: torch.empty((1, n), dtype=torch.bfloat16, device=dev) for n in (5120, 10240, 17408)}
    qkv_o, out_o = torch.empty((1, 10240), dtype=torch.bfloat16, device=dev), bufs[5120]
    gate_o, up_o = torch.empty((1, 17408), dtype=torch.bfloat16, device=dev), bufs[17408]
    h = torch.empty((1, 5120), dtype=torch.bfloat16, device=dev)

    def step(_i):
        x = h0
        for blk in layers:
            (wq, _, _), (wo, _, _), (wg, _, _), (wu, _, _), (wd, _, _) = blk
            B.linear(x, wq, 10240, workspace=ws, out=qkv_o)
            B.linear(qkv_o[:, :5120], wo, 5120, workspace=ws, out=out_o)
            B.linear(out_o, wg, 17408, workspace=ws, out=gate_o)
            B.linear(out_o, wu, 17408, workspace=ws, out=up_o)
            B.linear(up_o, wd, 5120, workspace=ws, out=h)
            x = h

    for i in range(warmup):
        step(i)
    replay = graph_loop(step, steps, stream, chunk=4)
    replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_calls = e0.elapsed_time(e1) / steps
    y_calls = h.clone()
    del replay
    # the same step as one persistent launch over the 310 layers
    desc = []
    xin = h0.reshape(-1)
    for blk in layers:
        (wq, _, _), (wo, _, _), (wg, _, _), (wu, _, _), (wd, _, _) = blk
        desc += [(wq, 10240, 5120, xin, qkv_o.reshape(-1)),
                 (wo, 5120, 5120, qkv_o.reshape(-1)[:5120], out_o.reshape(-1)),
                 (wg, 17408, 5120, out_o.reshape(-1), gate_o.reshape(-1)),
                 (wu, 17408, 5120, out_o.reshape(-1), up_o.reshape(-1)),
                 (wd, 5120, 17408, up_o.reshape(-1), h.reshape(-1))]
        xin = h.reshape(-1)
    # the same step with each layer quantising the next layer's activation (one launch per layer)
    fused = B.DecodeChain(desc)
    for i in range(warmup):
        fused.run()
    replay = graph_loop(lambda i: fused.run(), steps, stream, chunk=4)
    replay()
    torch.cuda.synchronize()
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms_fused = e0.elapsed_time(e1) / steps
    same_fused = bool(torch.equal(h.view(torch.int16), y_calls.view(torch.int16)))
    del replay, fused
    plan, cws, nl = B.chain_plan(desc)
    for i in range(warmup):
        B.chain_run(plan, nl, cws)
    replay = graph_loop(lambda i: B.chain_run(plan, nl, cws), steps, stream, chunk=4)
    replay()
    torch.cuda.synchronize()
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    same = bool(torch.equal(h.view(torch.int16), y_calls.view(torch.int16)))
    finite = bool(torch.isfinite(h.float()).all().item())
    del replay, layers, plan, cws
    torch.cuda.empty_cache()
    return {"workload": f"{C3_BLOCKS} blocks x (qkv 5120->10240, out 5120->5120, gate/up 5120->17408, "
                        "down 17408->5120), M=1, chained",
            "ms_per_step": ms_calls, "weight_GBs": total / (ms_calls * 1e-3) / 1e9, "weight_bytes_per_step": total,
            "resident_bytes": resident, "kernels_per_step": C3_BLOCKS * len(C3_SHAPES), "steps": steps,
            "how": "310 w4a8_linear calls, one kernel each, replayed from CUDA graphs",
            "decode_chain": {"ms_per_step": ms_fused, "weight_GBs": total / (ms_fused * 1e-3) / 1e9,
                             "kernels_per_step": C3_BLOCKS * len(C3_SHAPES),
                             "how": "w4a8_decode_chain: one launch per layer; each layer rotates the next layer's "
                                    "input blocks in its epilogue and the next layer only quantises them",
                             "same_bits_as_layer_by_layer": same_fused},
            "persistent_chain": {"ms_per_step": ms, "weight_GBs": total / (ms * 1e-3) / 1e9, "kernels_per_step": 1,
                                 "how": "one persistent launch of the 310 layers (w4a8_chain_run), grid barrier "
                                        "between layers",
                                 "same_bits_as_layer_by_layer": same},
            "output_finite": finite}


def measure_c4b(B, synth, torch, dev, rank, stream, steps, warmup):
    """Second prefill shape: M=8192, K=17408, N=5120 (one w4a8_linear per step)."""
    m, k, n = 8192, 17408, 5120
    q = synth.quantized_format_device(n, k, seed=88 + rank, device=dev)
    pk = B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    del q
    g = torch.Generator(device=dev)
    g.manual_seed(9 + rank)
    x = torch.randn((m, k), generator=g, device=dev).to(torch.bfloat16)
    ws = B.linear_workspace(m, k, n, dev)
    y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)

    def step(_i):
        B.linear(x, pk, n, workspace=ws, out=y)

    for i in range(warmup):
        step(i)
    replay = graph_loop(step, steps, stream)
    replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1) / steps
    del replay, pk, x, ws, y
    torch.cuda.empty_cache()
    return {"workload": f"prefill GEMM M={m} K={k} N={n}", "ms_per_step": ms,
            "TOPS": 2.0 * m * n * k / (ms * 1e-3) / 1e12}


def measure_converter(B, torch, dev, rank, stream, reps=5):
    """GPU weight converter on the C1 layer's shape: fp32 W [17408, 5120] ->
    the four stored tensors.  'assign' = given codebook (rotation, scales,
    indices); 'fit' = Lloyd-Max on a 2^22-value seeded sample first."""
    import numpy as np
    n, k = N_DEC, K_DEC
    g = torch.Generator(device=dev)
    g.manual_seed(11 + rank)
    w = torch.randn((n, k), generator=g, device=dev) * 0.02
    first = B.convert_weight_sampled(w, sample_cap=2 ** 22, seed=42)
    pos = B.fit_sample_positions(first["s_rel"].cpu().numpy(), first["s_ch"].cpu().numpy(), 2 ** 22, 42)
    pos_d = None if pos is None else torch.from_numpy(np.ascontiguousarray(pos)).to(dev)
    cb = first["cb"].clone()

    def timed(fn):
        fn()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(reps):
            fn()
        e1.record(stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1) / reps

    assign_ms = timed(lambda: B.convert_weight(w, codebook=cb))
    fit_ms = timed(lambda: B.convert_weight(w, sample_pos=pos_d))
    rounds = int(first["fit_rounds"].item())
    wb = n * k * 4
    # fidelity check of the converted layer against its source (host-side sample draw included)
    packed = B.pack_layout(first["packed"], first["s_rel"], first["s_ch"], first["cb"])
    xg = torch.Generator(device=dev)
    xg.manual_seed(12 + rank)
    x = torch.randn((4, k), generator=xg, device=dev).to(torch.bfloat16)
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    ver = B.verify_layer(w, packed, x)
    torch.cuda.synchronize()
    verify_ms = (time.perf_counter() - t0) * 1e3
    del w, first, pos_d, packed
    torch.cuda.empty_cache()
    return {"workload": f"fp32 W [{n}, {k}] -> packed indices, e4m3 group scales, fp32 row scales, codebook",
            "assign_ms": assign_ms, "assign_W_GBs": wb / (assign_ms * 1e-3) / 1e9,
            "fit_ms": fit_ms, "fit_rounds": rounds, "fit_sample": 2 ** 22,
            "note": "fp64 rotation and decisions (bit-exact with the oracle given the codebook)",
            "verify": {"fidelity": ver["fidelity"], "forward_error_4_tokens": ver["forward"],
                       "wall_ms": verify_ms,
                       "note": "stored = this conversion; fresh re-conversion with the seeded fit; "
                               "wall time includes the host-side sample draw"}}


E2M1_GRID = (-6.0, -4.0, -3.0, -2.0, -1.5, -1.0, -0.5, -0.0, 0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0)


def measure_nvfp4_foil(B, torch, dev, rank, n=17408, k=5120, tokens=16):
    """Accuracy foil: the same weights quantised with the Lloyd-Max codebook
    and with the uniform E2M1 grid (the FP4 values of NVFP4, divided by 6 so
    that they span the normalised [-1, 1]), both with the format's e4m3
    per-16 and fp32 per-row scales; relative L2 error of the dequantised
    weights and of the layer's output on probe tokens, against fp32."""
    g = torch.Generator(device=dev)
    g.manual_seed(21 + rank)
    w = torch.randn((n, k), generator=g, device=dev) * 0.02
    mask = torch.rand((n, k), generator=g, device=dev) < 0.005
    w = torch.where(mask, torch.randn((n, k), generator=g, device=dev) * 0.2, w)
    x = torch.randn((tokens, k), generator=g, device=dev)
    x[:, torch.randperm(k, generator=g, device=dev)[: k // 100]] *= 20.0
    x = x.to(torch.bfloat16)
    y_ref = B.dense_reference(x, w)
    out = {}
    grid = torch.tensor([v / 6.0 for v in E2M1_GRID], dtype=torch.float32, device=dev)
    for name, conv in (("lloyd_max_codebook", lambda: B.convert_weight_sampled(w)),
                       ("e2m1_grid", lambda: B.convert_weight(w, codebook=grid))):
        q = conv()
        pk = B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
        y = B.linear(x, pk, n)
        c = B.compare(y, y_ref).cpu()
        out[name] = {"forward_rel_l2": float((c[0] / c[1]).sqrt()), "codebook": [round(float(v), 5) for v in q["cb"]]}
        del q, pk, y
    # the native NVFP4 layer: 4-bit activations too (one fp32 scalar per token), with and without the rotation
    wc, wsf, gw = B.nvfp4_quantize(w, rotate=True, per_tensor=True)
    c = B.compare(B.nvfp4_linear(x, wc, wsf, gw), y_ref).cpu()
    out["nvfp4_w4a4_rotated"] = {"forward_rel_l2": float((c[0] / c[1]).sqrt())}
    wc, wsf, gw = B.nvfp4_quantize(w, rotate=False, per_tensor=True)
    xc, xs, gx = B.nvfp4_quantize(x, rotate=False)
    c = B.compare(B.nvfp4_gemm(xc, xs, gx, wc, wsf, gw), y_ref).cpu()
    out["nvfp4_w4a4_unrotated"] = {"forward_rel_l2": float((c[0] / c[1]).sqrt())}
    del wc, wsf, gw, xc, xs, gx
    del w, x, y_ref
    torch.cuda.empty_cache()
    return {"workload": f"W [{n}, {k}] ~ N(0, 0.02^2) with 0.5% N(0, 0.2^2) outliers, {tokens} probe tokens "
                        "with 1% channels x20; forward error of w4a8_linear against fp32 x W^T",
            **out,
            "speed_note": "lloyd_max_codebook and e2m1_grid run through the codebook layer's kernels (same "
                          "bytes, same speed); nvfp4_w4a4_* run the native block-scaled FP4 layer "
                          "(other_configs.nvfp4_native has its speed)"}


def _timed_replay(replay, stream, steps):
    import torch
    replay()
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    replay()
    e1.record(stream)
    torch.cuda.synchronize()
    return e0.elapsed_time(e1) / steps


def measure_nvfp4(B, torch, dev, rank, stream, peaks, steps=30, dec_steps=2000, copies=4):
    """Native NVFP4 layer (4-bit weights AND activations, tcgen05.mma
    kind::mxf4nvf4) on the codebook layer's shape K=5120, N=17408: the weight
    conversion, the prefill step (quantise + GEMM) and the GEMM alone at
    M=4096, and decode calls at M=1 and 16 (64-token tile, no split-K) on
    `copies` weight copies cycled (each 50 MB, together more than L2)."""
    n, k = N_PRE, K_PRE
    g = torch.Generator(device=dev)
    g.manual_seed(31 + rank)
    w = torch.randn((n, k), generator=g, device=dev) * 0.02
    conv_ms = _timed_replay(lambda: [B.nvfp4_quantize(w, rotate=True, per_tensor=True) for _ in range(3)],
                            stream, 3)
    wc, wsf, gw = B.nvfp4_quantize(w, rotate=True, per_tensor=True)
    del w
    fp4_peak = 4.0 * peaks["bf16_tflops"]
    wbytes = n * k // 2 + n * k // 16 + 4 * n
    out = {"workload": f"K={k} N={n}; weights fp32 N(0, 0.02^2) -> NVFP4 (rotated, one fp32 scalar per tensor)",
           "convert_ms": conv_ms}
    for m in (4096, 1, 16):
        x = torch.randn((m, k), generator=g, device=dev).to(torch.bfloat16)
        wsp = B.nvfp4_linear_workspace(m, k, dev)
        y = torch.empty((m, n), dtype=torch.bfloat16, device=dev)
        sets = [(wc, wsf, gw)] if m > 64 else [(wc.clone(), wsf.clone(), gw.clone()) for _ in range(copies)]
        reps = steps if m > 64 else dec_steps
        step = lambda i: B.nvfp4_linear(x, *sets[i % len(sets)], workspace=wsp, out=y)
        for i in range(3):
            step(i)
        lin_ms = _timed_replay(graph_loop(step, reps, stream), stream, reps)
        xc, xs, gx = B.nvfp4_quantize(x, rotate=True)
        gstep = lambda i: B.nvfp4_gemm(xc, xs, gx, *sets[i % len(sets)], out=y)
        gemm_ms = _timed_replay(graph_loop(gstep, reps, stream), stream, reps)
        flops = 2.0 * m * n * k
        if m > 64:
            tf = flops / (gemm_ms * 1e-3) / 1e12
            out[f"prefill_M{m}"] = {
                "ms_per_step": lin_ms, "TOPS": flops / (lin_ms * 1e-3) / 1e12,
                "roofline": {"kernel": "nvfp4_gemm_kernel<128, 2>", "bound": "tensor", "achieved": tf,
                             "peak": fp4_peak, "unit": "TFLOP/s", "frac": tf / fp4_peak,
                             "peak_note": "measured dense bf16 burst peak x 4 (the nominal dense fp4/bf16 "
                                          "ratio, 9 / 2.25 PFLOP/s)",
                             "traffic": profiled_traffic("nvfp4_gemm_kernel_prefill"),
                             "ms_per_launch": gemm_ms}}
        else:
            gb = wbytes / (gemm_ms * 1e-3) / 1e9
            out[f"decode_M{m}"] = {
                "us_per_step": lin_ms * 1e3, "step_GBs": wbytes / (lin_ms * 1e-3) / 1e9,
                "roofline": {"kernel": "nvfp4_gemm_kernel<64, 1>", "bound": "hbm", "achieved": gb,
                             "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": gb / peaks["hbm_gbs"],
                             "us_per_launch": gemm_ms * 1e3,
                             "bytes": "codes 0.5 B + scales 1/16 B per weight + 4 B per row"}}
        del sets, x, wsp, y, xc, xs, gx
    del wc, wsf, gw
    torch.cuda.empty_cache()
    return out


def main() -> None:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=200)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--prefill-steps", type=int, default=30)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true", help="skip the C2/C3/second-prefill lines")
    ap.add_argument("--only", default="", help="comma-separated subset of the other configurations to run")
    ap.add_argument("--ref-seconds", type=float, default=120.0,
                    help="reference arm: about how long warm-up plus timed steps take in all")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    import torch.distributed as dist

    import synth
    from w4a8_codebook_quantized_rotate_b200 import build as _build
    from w4a8_codebook_quantized_rotate_b200 import binding as B

    _build.build()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120), device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    def ranks_max(v: float) -> float:
        return max_over_ranks(v, world, dev)

    stream = torch.cuda.current_stream()
    peaks = measured_peaks()

    # ---------------- decode workload: 8 distinct copies of the layer
    copies = []
    for c in range(COPIES):
        q = synth.quantized_format_device(N_DEC, K_DEC, seed=1000 * (rank + 1) + c, device=dev)
        copies.append(B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"]))
        del q
    bits, _, _ = synth.activations(M_DEC, K_DEC, synth.rng_for(1, rank, "act"), K_DEC // 100)
    x = torch.from_numpy(bits.view(np.int16)).to(dev).view(torch.bfloat16)
    ws = B.linear_workspace(M_DEC, K_DEC, N_DEC, dev)
    y = torch.empty((M_DEC, N_DEC), dtype=torch.bfloat16, device=dev)
    wbytes = weight_bytes(N_DEC, K_DEC)

    def step(i):
        B.linear(x, copies[i % COPIES], N_DEC, workspace=ws, out=y)

    # Steps are launched from CUDA graphs: a host loop through the Python
    # binding issues launches more slowly than the GPU finishes them.
    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    replay_steps = graph_loop(step, args.steps, stream)
    B.linear_prepare(x, N_DEC, ws)
    replay_runs = graph_loop(lambda i: B.linear_run(M_DEC, K_DEC, copies[i % COPIES], N_DEC, ws, out=y),
                             args.steps, stream)
    sampler = ClockSampler(local)
    with sampler:
        replay_steps()  # one untimed pass through the captured graphs
        torch.cuda.synchronize()
        barrier()
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        replay_steps()
        e1.record(stream)
        torch.cuda.synchronize()
        barrier()
        ms = ranks_max(e0.elapsed_time(e1))
        ms_step = ms / args.steps
        value = whole_job_rate(wbytes, world, args.steps, ms)

        # decode kernel alone: activations prepared once, then back-to-back runs
        B.linear_prepare(x, N_DEC, ws)
        replay_runs()
        torch.cuda.synchronize()
        g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        g0.record(stream)
        replay_runs()
        g1.record(stream)
        torch.cuda.synchronize()
        gemv_ms = ranks_max(g0.elapsed_time(g1)) / args.steps
    dec_clocks = sampler.summary()
    del replay_steps, replay_runs

    # ---------------- end to end through the C ABI, host buffers
    x_host = torch.empty((M_DEC, K_DEC), dtype=torch.bfloat16, pin_memory=True)
    x_host.copy_(x.cpu())
    y_host = torch.empty((M_DEC, N_DEC), dtype=torch.bfloat16, pin_memory=True)
    x_dev = torch.empty_like(x)
    e2e_steps = min(args.steps, 5000)

    def e2e_step(i):
        x_dev.copy_(x_host, non_blocking=True)
        B.linear(x_dev, copies[i % COPIES], N_DEC, workspace=ws, out=y)
        y_host.copy_(y, non_blocking=True)

    for i in range(args.warmup):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier()
    # (a) pipelined: step i's copy in, layer and copy out run on three streams
    # with four buffer sets, so the copies of the neighbouring steps overlap
    # step i's layer; every step still moves its x in from pinned host memory
    # and its y out to pinned host memory.  The layer stream holds kernels
    # only (w4a8_linear_flagged waits on the GPU for a ready word that the
    # copy stream writes after x), so consecutive layers keep their programmatic launch
    # overlap: a stream dependency on the copy event costs that overlap
    # (18.5 against 14.2 us per step, measured).  Captured in CUDA graphs of
    # 512 steps (no overlap across graph boundaries).
    NBUF = 4
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
    xs = [torch.empty_like(x) for _ in range(NBUF)]
    ys = [torch.empty_like(y) for _ in range(NBUF)]
    yh = [torch.empty((M_DEC, N_DEC), dtype=torch.bfloat16, pin_memory=True) for _ in range(NBUF)]
    flags = [torch.zeros(2, dtype=torch.int32, device=dev) for _ in range(NBUF)]
    ev_comp = [torch.cuda.Event() for _ in range(NBUF)]
    ev_out = [torch.cuda.Event() for _ in range(NBUF)]
    side = torch.cuda.Stream()
    side.wait_stream(stream)

    def capture_pipelined(n, base):
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=side):
            for i in range(n):
                b = i % NBUF
                if i >= NBUF:  # the layer that read this set and the copy that read its y are done
                    s_in.wait_event(ev_comp[b])
                    s_in.wait_event(ev_out[b])
                else:
                    s_in.wait_stream(side)
                with torch.cuda.stream(s_in):
                    xs[b].copy_(x_host, non_blocking=True)
                B.signal_ready(flags[b], stream=s_in)  # the ready word, written by the stream after x
                B.linear_flagged(xs[b], copies[(base + i) % COPIES], N_DEC, flags[b], ws, ys[b], stream=side)
                ev_comp[b].record(side)
                s_out.wait_event(ev_comp[b])
                with torch.cuda.stream(s_out):
                    yh[b].copy_(ys[b], non_blocking=True)
                    ev_out[b].record(s_out)
            side.wait_stream(s_in)
            side.wait_stream(s_out)
        return g

    chunk = 512
    pipe_graphs = [capture_pipelined(min(chunk, e2e_steps - b0), b0) for b0 in range(0, e2e_steps, chunk)]
    stream.wait_stream(side)
    torch.cuda.synchronize()

    def replay_pipe():
        for g in pipe_graphs:
            g.replay()
    replay_pipe()
    torch.cuda.synchronize()
    barrier()
    h0, h1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    h0.record(stream)
    replay_pipe()
    h1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_ms = ranks_max(h0.elapsed_time(h1)) / e2e_steps
    del pipe_graphs
    # (b) the same steps issued one by one from Python (host launch cost included)
    h0.record(stream)
    for i in range(e2e_steps):
        e2e_step(i)
    h1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e2e_loop_ms = ranks_max(h0.elapsed_time(h1)) / e2e_steps
    del copies
    torch.cuda.empty_cache()

    # ---------------- prefill GEMM, M=4096
    q = synth.quantized_format_device(N_PRE, K_PRE, seed=77 + rank, device=dev)
    packed_pre = B.pack_layout(q["packed"], q["s_rel"], q["s_ch"], q["cb"])
    del q
    g = torch.Generator(device=dev)
    g.manual_seed(5 + rank)
    xp = torch.randn((M_PRE, K_PRE), generator=g, device=dev, dtype=torch.float32).to(torch.bfloat16)
    ws_p = B.linear_workspace(M_PRE, K_PRE, N_PRE, dev)
    yp = torch.empty((M_PRE, N_PRE), dtype=torch.bfloat16, device=dev)
    flops = 2.0 * M_PRE * N_PRE * K_PRE
    for _ in range(3):
        B.linear(xp, packed_pre, N_PRE, workspace=ws_p, out=yp)
    torch.cuda.synchronize()
    replay_pre = graph_loop(lambda i: B.linear(xp, packed_pre, N_PRE, workspace=ws_p, out=yp),
                            args.prefill_steps, stream)
    B.linear_prepare(xp, N_PRE, ws_p)
    replay_gemm = graph_loop(lambda i: B.linear_run(M_PRE, K_PRE, packed_pre, N_PRE, ws_p, out=yp),
                             args.prefill_steps, stream)
    psampler = ClockSampler(local)
    with psampler:
        replay_pre()
        torch.cuda.synchronize()
        barrier()
        p0, p1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        p0.record(stream)
        replay_pre()
        p1.record(stream)
        torch.cuda.synchronize()
        pre_ms = ranks_max(p0.elapsed_time(p1)) / args.prefill_steps
        B.linear_prepare(xp, N_PRE, ws_p)
        replay_gemm()
        torch.cuda.synchronize()
        q0, q1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        q0.record(stream)
        replay_gemm()
        q1.record(stream)
        torch.cuda.synchronize()
        gemm_ms = ranks_max(q0.elapsed_time(q1)) / args.prefill_steps
    del replay_pre, replay_gemm
    pre_clocks = psampler.summary()

    # ---------------- the other configurations: C2 token sweep, C3 decode step, C4 second shape
    extra = {}
    only = {s for s in args.only.split(",") if s}
    runs = {
        "c2_down_proj": lambda: measure_c2(B, synth, torch, dev, rank, stream, min(2000, args.steps), args.warmup),
        "c1_streaming_rate": lambda: measure_c1_rate(B, synth, torch, dev, rank, stream),
        "c3_decode_step": lambda: measure_c3(B, synth, torch, dev, rank, stream, 20, 3),
        "c4_prefill_8192": lambda: measure_c4b(B, synth, torch, dev, rank, stream, max(3, args.prefill_steps // 2), 3),
        "weight_converter": lambda: measure_converter(B, torch, dev, rank, stream),
        "nvfp4_foil": lambda: measure_nvfp4_foil(B, torch, dev, rank),
        "nvfp4_native": lambda: measure_nvfp4(B, torch, dev, rank, stream, peaks, steps=max(3, args.prefill_steps),
                                              dec_steps=min(2000, args.steps)),
    }
    if not args.no_extra:
        for name, run in runs.items():
            if not only or name in only:
                extra[name] = run()
    err = B.get_device_error()

    if world > 1:
        barrier()
        dist.destroy_process_group()
    if rank != 0:
        return

    achieved = wbytes / (gemv_ms * 1e-3) / 1e9
    step_gbs = wbytes / (ms_step * 1e-3) / 1e9
    gemm_tflops = flops / (gemm_ms * 1e-3) / 1e12
    line = {
        "metric": METRIC,
        "value": value,
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f16*f16->f32 (4-bit codebook weights, int8 activations, bf16 out)",
        "data": "synthetic",
        "config": {
            "workload": f"decode GEMV M={M_DEC} K={K_DEC} N={N_DEC}, {COPIES} distinct weight copies cycled",
            "l2": f"inputs larger than L2: {COPIES} x {wbytes / 1e6:.1f} MB weights cycled > 126 MB L2",
            "weight_bytes_per_step": wbytes,
            "parallelism": f"replicas x{world}" if world > 1 else "1 GPU",
            "launch": "timed steps replayed from CUDA graphs (1 kernel per step, programmatic dependent launch)",
        },
        "roofline": {
            "kernel": "decode_one_kernel<true> (M=1, rotate + quantise fused)",
            "bound": "hbm", "achieved": step_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": step_gbs / peaks["hbm_gbs"], "peak_source": peaks["source"],
            "traffic": profiled_traffic("decode_one_kernel_fused"),
            "us_per_launch": ms_step * 1e3,
            "note": "the step is this one kernel, so its launch duration is the step time",
        },
        "decode_run_only": {
            "kernel": "decode_one_kernel<false> (activations prepared once, runs back to back)",
            "achieved": achieved, "unit": "GB/s", "frac": achieved / peaks["hbm_gbs"],
            "us_per_launch": gemv_ms * 1e3,
        },
        "prefill": {
            "workload": f"prefill GEMM M={M_PRE} K={K_PRE} N={N_PRE}",
            "value": flops / (pre_ms * 1e-3) / 1e12, "unit": "TOPS", "ms_per_step": pre_ms,
            "roofline": {"kernel": "gemm_tc_kernel", "bound": "tensor", "achieved": gemm_tflops,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": gemm_tflops / peaks["bf16_tflops"],
                         "peak_note": "measured dense bf16 burst peak; fp16 kind::f16 runs at the bf16 rate",
                         "traffic": profiled_traffic("gemm_tc_kernel"),
                         "ms_per_launch": gemm_ms},
            "clocks": pre_clocks,
        },
        "e2e": {"value": wbytes / (e2e_ms * 1e-3) / 1e9 * world, "unit": "GB/s",
                "h2d_bytes_per_step": M_DEC * K_DEC * 2, "d2h_bytes_per_step": M_DEC * N_DEC * 2,
                "ms_per_step": e2e_ms,
                "how": "per step: pinned x copied in (then the ready word, written by the copy stream "
                       "itself: w4a8_signal_ready), w4a8_linear_flagged through the "
                       "Python binding (the layer waits on the GPU for the ready word, so its stream holds "
                       "kernels only), y copied out to pinned memory; copies on their own streams overlap the "
                       "neighbouring steps' layers (four buffer sets); replayed from CUDA graphs of 512 steps",
                "host_loop": {"value": wbytes / (e2e_loop_ms * 1e-3) / 1e9 * world, "ms_per_step": e2e_loop_ms,
                              "how": "the same steps issued one by one from Python"}},
        "clocks": dec_clocks,
        "gpu_launches": args.steps,
        "other_configs": extra,
        "device_error": err,
    }
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(B=B, torch=torch, dev=dev)
    print(json.dumps(line), flush=True)


if __name__ == "__main__":
    main()
