"""Thin ctypes binding of the C ABI in ``include/w4a8.h``.

Argument marshalling only: every step of the layer runs in the CUDA library
``lib/libw4a8.so``.  PyTorch supplies device memory and the current stream.
There is no fallback: if the library or a CUDA device is missing, the calls
raise.
"""

from __future__ import annotations

import ctypes
import os

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "lib", "libw4a8.so")

STATUS = {
    0: "ok", 1: "null pointer", 2: "bad shape", 3: "misaligned pointer",
    4: "buffer too small", 5: "CUDA error", 6: "device wait timed out", 7: "device is not sm_100",
    8: "device-side input check failed",
}

EXPORTS = (
    "w4a8_packed_bytes", "w4a8_pack_layout", "w4a8_unpack_dequant", "w4a8_rotate_quant_act",
    "w4a8_linear_workspace_bytes", "w4a8_linear", "w4a8_linear_prepare", "w4a8_linear_run",
    "w4a8_linear_decode_static", "w4a8_get_device_error", "w4a8_selftest_timeout", "w4a8_status_string",
    "w4a8_convert_workspace_bytes", "w4a8_convert_weight",
    "w4a8_compare_workspace_bytes", "w4a8_compare", "w4a8_dense_reference",
    "w4a8_chain_plan_bytes", "w4a8_chain_workspace_bytes", "w4a8_chain_plan", "w4a8_chain_run",
    "w4a8_decode_chain_workspace_bytes", "w4a8_decode_chain", "w4a8_linear_flagged", "w4a8_signal_ready",
    "w4a8_nvfp4_scale_bytes", "w4a8_nvfp4_quantize", "w4a8_nvfp4_pack_scales", "w4a8_nvfp4_gemm",
    "w4a8_nvfp4_linear_workspace_bytes", "w4a8_nvfp4_linear",
)


class ChainLayer(ctypes.Structure):
    """w4a8_chain_layer: one layer of a chain (device pointers)."""
    _fields_ = [("packed", ctypes.c_void_p), ("N", ctypes.c_int64), ("K", ctypes.c_int64),
                ("x", ctypes.c_void_p), ("y", ctypes.c_void_p)]

_lib = None


class W4A8Error(RuntimeError):
    def __init__(self, call: str, status: int):
        super().__init__(f"{call}: {STATUS.get(status, 'unknown')} (status {status})")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library and declare the C signatures."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"CUDA library not built: {path} (run __graft_entry__.build())")
    lib = ctypes.CDLL(path)
    i64, sz, vp, st = ctypes.c_int64, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_int
    sigs = {
        "w4a8_packed_bytes": (sz, [i64, i64]),
        "w4a8_pack_layout": (st, [vp, vp, vp, vp, i64, i64, vp, sz, vp]),
        "w4a8_unpack_dequant": (st, [vp, i64, i64, vp, vp]),
        "w4a8_rotate_quant_act": (st, [vp, i64, i64, vp, vp, vp]),
        "w4a8_linear_workspace_bytes": (sz, [i64, i64, i64]),
        "w4a8_linear": (st, [vp, i64, i64, vp, i64, vp, vp, sz, vp]),
        "w4a8_linear_prepare": (st, [vp, i64, i64, i64, vp, sz, vp]),
        "w4a8_linear_run": (st, [i64, i64, vp, i64, vp, vp, sz, vp]),
        "w4a8_linear_decode_static": (st, [vp, i64, i64, vp, i64, vp, vp]),
        "w4a8_get_device_error": (st, [vp]),
        "w4a8_selftest_timeout": (st, [vp]),
        "w4a8_status_string": (ctypes.c_char_p, [st]),
        "w4a8_convert_workspace_bytes": (sz, [i64, i64, i64]),
        "w4a8_convert_weight": (st, [vp, i64, i64, vp, vp, i64, ctypes.c_int32, ctypes.c_double,
                                     vp, vp, vp, vp, vp, vp, sz, vp]),
        "w4a8_compare_workspace_bytes": (sz, []),
        "w4a8_compare": (st, [vp, ctypes.c_int32, vp, i64, vp, vp, sz, vp]),
        "w4a8_dense_reference": (st, [vp, i64, i64, vp, i64, vp, vp]),
        "w4a8_chain_plan_bytes": (sz, [i64]),
        "w4a8_chain_workspace_bytes": (sz, [vp, i64]),
        "w4a8_chain_plan": (st, [vp, i64, vp, sz, vp, sz, vp]),
        "w4a8_chain_run": (st, [vp, i64, vp, sz, vp]),
        "w4a8_decode_chain_workspace_bytes": (sz, [vp, i64]),
        "w4a8_decode_chain": (st, [vp, i64, vp, sz, vp]),
        "w4a8_linear_flagged": (st, [vp, i64, i64, vp, i64, vp, vp, vp, sz, vp]),
        "w4a8_signal_ready": (st, [vp, vp]),
        "w4a8_nvfp4_scale_bytes": (sz, [i64, i64]),
        "w4a8_nvfp4_quantize": (st, [vp, ctypes.c_int32, i64, i64, ctypes.c_int32, ctypes.c_int32,
                                     vp, vp, vp, vp, vp]),
        "w4a8_nvfp4_pack_scales": (st, [vp, i64, i64, vp, vp]),
        "w4a8_nvfp4_gemm": (st, [vp, vp, vp, i64, vp, vp, vp, i64, i64, vp, vp]),
        "w4a8_nvfp4_linear_workspace_bytes": (sz, [i64, i64]),
        "w4a8_nvfp4_linear": (st, [vp, i64, i64, vp, vp, vp, i64, vp, vp, sz, vp]),
    }
    for name, (res, args) in sigs.items():
        fn = getattr(lib, name)
        fn.restype, fn.argtypes = res, args
    _lib = lib
    return lib


def _check(call: str, status: int) -> None:
    if status != 0:
        raise W4A8Error(call, status)


def _stream(stream=None) -> int:
    s = torch.cuda.current_stream() if stream is None else stream
    return s.cuda_stream


def _cuda(t: torch.Tensor, dtype: torch.dtype, name: str) -> torch.Tensor:
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def packed_bytes(n: int, k: int) -> int:
    return int(load_library().w4a8_packed_bytes(n, k))


def pack_layout(idx: torch.Tensor, s_rel: torch.Tensor, s_channel: torch.Tensor, codebook: torch.Tensor,
                stream=None) -> torch.Tensor:
    """Canonical tensors (idx uint8 [N, K/2], s_rel e4m3 codes uint8 [N, K/16],
    s_channel fp32 [N], codebook fp32 [16]) -> packed device buffer (uint8)."""
    lib = load_library()
    _cuda(idx, torch.uint8, "idx")
    _cuda(s_rel, torch.uint8, "s_rel")
    _cuda(s_channel, torch.float32, "s_channel")
    _cuda(codebook, torch.float32, "codebook")
    n, k = idx.shape[0], idx.shape[1] * 2
    nbytes = lib.w4a8_packed_bytes(n, k)
    if nbytes == 0:
        raise W4A8Error("w4a8_packed_bytes", 2)
    out = torch.empty(nbytes, dtype=torch.uint8, device=idx.device)
    _check("w4a8_pack_layout", lib.w4a8_pack_layout(
        idx.data_ptr(), s_rel.data_ptr(), s_channel.data_ptr(), codebook.data_ptr(), n, k,
        out.data_ptr(), nbytes, _stream(stream)))
    return out


def unpack_dequant(packed: torch.Tensor, n: int, k: int, stream=None) -> torch.Tensor:
    lib = load_library()
    _cuda(packed, torch.uint8, "packed")
    out = torch.empty((n, k), dtype=torch.float32, device=packed.device)
    _check("w4a8_unpack_dequant", lib.w4a8_unpack_dequant(packed.data_ptr(), n, k, out.data_ptr(),
                                                          _stream(stream)))
    return out


def rotate_quant_act(x: torch.Tensor, stream=None):
    """bf16 x [M, K] -> (int8 x_q [M, K], fp32 s_x [M])."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    xq = torch.empty((m, k), dtype=torch.int8, device=x.device)
    sx = torch.empty((m,), dtype=torch.float32, device=x.device)
    _check("w4a8_rotate_quant_act", lib.w4a8_rotate_quant_act(x.data_ptr(), m, k, xq.data_ptr(),
                                                              sx.data_ptr(), _stream(stream)))
    return xq, sx


def linear_workspace_bytes(m: int, k: int, n: int) -> int:
    return int(load_library().w4a8_linear_workspace_bytes(m, k, n))


def linear_workspace(m: int, k: int, n: int, device) -> torch.Tensor:
    """A zero-filled workspace for layers of shape (M, K, N) (zero before its first use)."""
    need = linear_workspace_bytes(m, k, n)
    if need == 0:
        raise W4A8Error("w4a8_linear_workspace_bytes", 2)
    return torch.zeros(need, dtype=torch.uint8, device=device)


def linear(x: torch.Tensor, packed: torch.Tensor, n: int, workspace: torch.Tensor | None = None,
           out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """bf16 x [M, K] and a packed [N, K] layer -> bf16 y [M, N]."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    _cuda(packed, torch.uint8, "packed")
    m, k = x.shape
    need = lib.w4a8_linear_workspace_bytes(m, k, n)
    if need == 0:
        raise W4A8Error("w4a8_linear_workspace_bytes", 2)
    if workspace is None:
        workspace = torch.zeros(need, dtype=torch.uint8, device=x.device)
    _cuda(workspace, torch.uint8, "workspace")
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "out")
    _check("w4a8_linear", lib.w4a8_linear(x.data_ptr(), m, k, packed.data_ptr(), n, out.data_ptr(),
                                          workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out


def linear_prepare(x: torch.Tensor, n: int, workspace: torch.Tensor, stream=None) -> None:
    """Quantise x [M, K] into ``workspace`` for layers of N output rows."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    _cuda(workspace, torch.uint8, "workspace")
    m, k = x.shape
    _check("w4a8_linear_prepare", lib.w4a8_linear_prepare(x.data_ptr(), m, k, n, workspace.data_ptr(),
                                                          workspace.numel(), _stream(stream)))


def linear_run(m: int, k: int, packed: torch.Tensor, n: int, workspace: torch.Tensor,
               out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """Apply a packed [N, K] layer to the activations prepared in ``workspace``."""
    lib = load_library()
    _cuda(packed, torch.uint8, "packed")
    _cuda(workspace, torch.uint8, "workspace")
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=packed.device)
    _cuda(out, torch.bfloat16, "out")
    _check("w4a8_linear_run", lib.w4a8_linear_run(m, k, packed.data_ptr(), n, out.data_ptr(),
                                                  workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out


def linear_decode_static(x: torch.Tensor, packed: torch.Tensor, n: int, out: torch.Tensor | None = None,
                         stream=None) -> torch.Tensor:
    """The layer for M <= 16 using the library's built-in device scratch
    instead of a workspace (for callers that cannot allocate device memory).
    Calls on one device share that scratch, so they must not overlap on the GPU."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    _cuda(packed, torch.uint8, "packed")
    m, k = x.shape
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _cuda(out, torch.bfloat16, "out")
    _check("w4a8_linear_decode_static", lib.w4a8_linear_decode_static(
        x.data_ptr(), m, k, packed.data_ptr(), n, out.data_ptr(), _stream(stream)))
    return out


def get_device_error(stream=None) -> int:
    """Synchronise and return (and clear) the device error status (0 = ok)."""
    return int(load_library().w4a8_get_device_error(_stream(stream)))


def selftest_timeout(stream=None) -> None:
    """Run the device self-test of the bounded waits (they record a timeout
    that the next get_device_error returns)."""
    _check("w4a8_selftest_timeout", load_library().w4a8_selftest_timeout(_stream(stream)))


def convert_weight(w: torch.Tensor, codebook: torch.Tensor | None = None, sample_pos: torch.Tensor | None = None,
                   max_iter: int = 500, tol: float = 1e-12, stream=None) -> dict:
    """fp32 W [N, K] on the GPU -> the four stored tensors (``packed`` [N, K/2] uint8,
    ``s_rel`` [N, K/16] uint8 e4m3 codes, ``s_ch`` [N] fp32, ``cb`` [16] fp32) and
    ``fit_rounds``.  With ``codebook`` given its levels are used; otherwise they are
    fitted on the values at ``sample_pos`` (int64 flat positions), or on every
    value whose scales are non-zero when ``sample_pos`` is None."""
    lib = load_library()
    _cuda(w, torch.float32, "w")
    n, k = w.shape
    dev = w.device
    packed = torch.empty((n, k // 2), dtype=torch.uint8, device=dev)
    s_rel = torch.empty((n, k // 16), dtype=torch.uint8, device=dev)
    s_ch = torch.empty((n,), dtype=torch.float32, device=dev)
    cb = torch.empty((16,), dtype=torch.float32, device=dev)
    rounds = torch.zeros((1,), dtype=torch.int32, device=dev)
    ws, ws_ptr, ws_bytes = None, None, 0
    cb_ptr, pos_ptr, n_pos = None, None, 0
    if codebook is not None:
        _cuda(codebook, torch.float32, "codebook")
        cb_ptr = codebook.data_ptr()
    else:
        if sample_pos is not None:
            _cuda(sample_pos, torch.int64, "sample_pos")
            pos_ptr, n_pos = sample_pos.data_ptr(), sample_pos.numel()
        ws_bytes = lib.w4a8_convert_workspace_bytes(n, k, n_pos)
        if ws_bytes == 0:
            raise W4A8Error("w4a8_convert_workspace_bytes", 2)
        ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        ws_ptr = ws.data_ptr()
    _check("w4a8_convert_weight", lib.w4a8_convert_weight(
        w.data_ptr(), n, k, cb_ptr, pos_ptr, n_pos, int(max_iter), float(tol), packed.data_ptr(),
        s_rel.data_ptr(), s_ch.data_ptr(), cb.data_ptr(), rounds.data_ptr(), ws_ptr, ws_bytes, _stream(stream)))
    return {"packed": packed, "s_rel": s_rel, "s_ch": s_ch, "cb": cb, "fit_rounds": rounds, "workspace": ws}


def fit_sample_positions(s_rel: "np.ndarray", s_ch: "np.ndarray", cap: int, seed: int):
    """Flat positions (n K + k) of a codebook-fit sample: the values whose group
    and row scales are non-zero, in row-major order, form the pool; if it holds
    more than ``cap`` values, ``cap`` of them are drawn without replacement by
    numpy's PCG64 generator seeded with ``seed`` (Generator.choice over the pool
    size); else None (fit on the whole pool)."""
    import numpy as np
    s_rel = np.asarray(s_rel, dtype=np.uint8)
    live = ((s_rel & 0x7F) != 0) & (np.asarray(s_ch) > 0)[:, None]
    groups = np.flatnonzero(live.ravel())
    n_live = groups.size * 16
    if n_live <= cap:
        return None
    p = np.random.Generator(np.random.PCG64(seed)).choice(n_live, size=cap, replace=False)
    return groups[p // 16].astype(np.int64) * 16 + (p % 16)


def convert_weight_sampled(w: torch.Tensor, sample_cap: int = 2 ** 22, seed: int = 42, max_iter: int = 500,
                           tol: float = 1e-12, stream=None) -> dict:
    """:func:`convert_weight` with the fit sample drawn as described in
    :func:`fit_sample_positions` (the scales are computed first, with a
    provisional codebook, to find the pool)."""
    import numpy as np
    provisional = torch.linspace(-1.0, 1.0, 16, dtype=torch.float32, device=w.device)
    first = convert_weight(w, codebook=provisional, stream=stream)
    pos = fit_sample_positions(first["s_rel"].cpu().numpy(), first["s_ch"].cpu().numpy(), sample_cap, seed)
    sample = None if pos is None else torch.from_numpy(np.ascontiguousarray(pos)).to(w.device)
    return convert_weight(w, sample_pos=sample, max_iter=max_iter, tol=tol, stream=stream)


def compare(a: torch.Tensor, ref: torch.Tensor, stream=None) -> torch.Tensor:
    """fp64 device tensor [sum (a - ref)^2, sum ref^2, max |a - ref|]; a fp32 or bf16, ref fp32."""
    lib = load_library()
    if a.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("a must be fp32 or bf16")
    _cuda(a, a.dtype, "a")
    _cuda(ref, torch.float32, "ref")
    if a.numel() != ref.numel():
        raise ValueError("a and ref differ in size")
    out = torch.empty(3, dtype=torch.float64, device=a.device)
    ws = torch.empty(lib.w4a8_compare_workspace_bytes(), dtype=torch.uint8, device=a.device)
    _check("w4a8_compare", lib.w4a8_compare(a.data_ptr(), int(a.dtype == torch.bfloat16), ref.data_ptr(),
                                            a.numel(), out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def dense_reference(x: torch.Tensor, w: torch.Tensor, stream=None) -> torch.Tensor:
    """Unquantised layer: fp32 y [M, N] = bf16 x [M, K] times fp32 W [N, K]^T (fp64 sums)."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    _cuda(w, torch.float32, "w")
    m, k = x.shape
    n = w.shape[0]
    if w.shape[1] != k:
        raise ValueError("x and w disagree on K")
    y = torch.empty((m, n), dtype=torch.float32, device=x.device)
    _check("w4a8_dense_reference", lib.w4a8_dense_reference(x.data_ptr(), m, k, w.data_ptr(), n, y.data_ptr(),
                                                            _stream(stream)))
    return y


def verify_layer(w: torch.Tensor, packed: torch.Tensor, x: torch.Tensor, sample_cap: int = 2 ** 22,
                 seed: int = 42, stream=None) -> dict:
    """Fidelity of a stored layer (``packed``, from :func:`pack_layout`) to its fp32
    source ``w`` [N, K]: ``fidelity`` = relative L2 distance between the stored
    layer's dequantised weights and those of a fresh conversion of ``w`` (seeded
    fit), ~0 for a faithful file; ``forward`` = relative L2 error of the stored
    layer's output on the probe activations ``x`` [M, K] (bf16) against the
    unquantised x W^T."""
    n, k = w.shape
    fresh = convert_weight_sampled(w, sample_cap=sample_cap, seed=seed, stream=stream)
    packed_fresh = pack_layout(fresh["packed"], fresh["s_rel"], fresh["s_ch"], fresh["cb"], stream=stream)
    w_file = unpack_dequant(packed, n, k, stream=stream)
    w_fresh = unpack_dequant(packed_fresh, n, k, stream=stream)
    c1 = compare(w_file, w_fresh, stream=stream).cpu()
    y_q = linear(x, packed, n, stream=stream)
    y_ref = dense_reference(x, w, stream=stream)
    c2 = compare(y_q, y_ref, stream=stream).cpu()
    rel = lambda c: float((c[0] / c[1]).sqrt()) if c[1] > 0 else float(c[0] > 0)
    return {"fidelity": rel(c1), "fidelity_max_abs": float(c1[2]), "forward": rel(c2),
            "forward_max_abs": float(c2[2]), "fit_rounds": int(fresh["fit_rounds"].item())}


def chain_plan(layers, stream=None):
    """Plan a chain of one-token layers.  ``layers`` is a list of
    (packed, n, k, x, y): x a bf16 CUDA tensor of k values (may be a view of
    an earlier layer's y), y a bf16 CUDA tensor of n values.  Returns
    (plan, workspace, n_layers); the tensors must outlive the runs."""
    lib = load_library()
    arr = (ChainLayer * len(layers))()
    dev = None
    for i, (packed, n, k, x, y) in enumerate(layers):
        _cuda(packed, torch.uint8, "packed")
        _cuda(x, torch.bfloat16, "x")
        _cuda(y, torch.bfloat16, "y")
        if x.numel() != k or y.numel() != n:
            raise ValueError(f"layer {i}: x must hold K and y N values")
        arr[i] = ChainLayer(packed.data_ptr(), n, k, x.data_ptr(), y.data_ptr())
        dev = packed.device
    n_layers = len(layers)
    plan = torch.empty(lib.w4a8_chain_plan_bytes(n_layers), dtype=torch.uint8, device=dev)
    ws_bytes = lib.w4a8_chain_workspace_bytes(arr, n_layers)
    if ws_bytes == 0:
        raise W4A8Error("w4a8_chain_workspace_bytes", 2)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    _check("w4a8_chain_plan", lib.w4a8_chain_plan(arr, n_layers, plan.data_ptr(), plan.numel(), ws.data_ptr(),
                                                  ws.numel(), _stream(stream)))
    return plan, ws, n_layers


def chain_run(plan: torch.Tensor, n_layers: int, workspace: torch.Tensor, stream=None) -> None:
    """Run a planned chain (one persistent launch)."""
    lib = load_library()
    _check("w4a8_chain_run", lib.w4a8_chain_run(plan.data_ptr(), n_layers, workspace.data_ptr(), workspace.numel(),
                                                _stream(stream)))


class DecodeChain:
    """A decode step as one launch per one-token layer, each layer quantising
    the next one's activation (w4a8_decode_chain).  ``layers`` as for
    :func:`chain_plan`; the tensors must outlive the runs."""

    def __init__(self, layers):
        lib = load_library()
        self._arr = (ChainLayer * len(layers))()
        dev = None
        for i, (packed, n, k, x, y) in enumerate(layers):
            _cuda(packed, torch.uint8, "packed")
            _cuda(x, torch.bfloat16, "x")
            _cuda(y, torch.bfloat16, "y")
            if x.numel() != k or y.numel() != n:
                raise ValueError(f"layer {i}: x must hold K and y N values")
            self._arr[i] = ChainLayer(packed.data_ptr(), n, k, x.data_ptr(), y.data_ptr())
            dev = packed.device
        self.n_layers = len(layers)
        need = lib.w4a8_decode_chain_workspace_bytes(self._arr, self.n_layers)
        if need == 0:
            raise W4A8Error("w4a8_decode_chain_workspace_bytes", 2)
        self.workspace = torch.zeros(need, dtype=torch.uint8, device=dev)

    def run(self, stream=None) -> None:
        _check("w4a8_decode_chain", load_library().w4a8_decode_chain(
            self._arr, self.n_layers, self.workspace.data_ptr(), self.workspace.numel(), _stream(stream)))


def linear_flagged(x: torch.Tensor, packed: torch.Tensor, n: int, x_ready: torch.Tensor,
                   workspace: torch.Tensor, out: torch.Tensor, stream=None) -> torch.Tensor:
    """w4a8_linear that waits on the GPU for ``x_ready[0] != 0`` (an int32
    CUDA tensor of 2 words written by the caller's copy after x) instead of a
    stream dependency; the layer clears the flag once it has read x."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    _cuda(packed, torch.uint8, "packed")
    _cuda(x_ready, torch.int32, "x_ready")
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(out, torch.bfloat16, "out")
    m, k = x.shape
    _check("w4a8_linear_flagged", lib.w4a8_linear_flagged(
        x.data_ptr(), m, k, packed.data_ptr(), n, out.data_ptr(), x_ready.data_ptr(), workspace.data_ptr(),
        workspace.numel(), _stream(stream)))
    return out


def signal_ready(x_ready: torch.Tensor, stream=None) -> None:
    """Writes 1 to ``x_ready[0]`` in stream order (after the stream's earlier
    work, e.g. the copy of x) without a host copy: w4a8_signal_ready."""
    lib = load_library()
    _cuda(x_ready, torch.int32, "x_ready")
    _check("w4a8_signal_ready", lib.w4a8_signal_ready(x_ready.data_ptr(), _stream(stream)))


# ---------------------------------------------------------------- NVFP4 comparison layer

def nvfp4_scale_bytes(rows: int, k: int) -> int:
    return int(load_library().w4a8_nvfp4_scale_bytes(rows, k))


def nvfp4_quantize(x: torch.Tensor, rotate: bool = True, per_tensor: bool = False, stream=None):
    """x [R, K] (bf16 or fp32) -> (codes uint8 [R, K/2], scales uint8 in the
    tensor cores' order, g fp32 [R]); one g per tensor or per row."""
    lib = load_library()
    if x.dtype not in (torch.bfloat16, torch.float32):
        raise ValueError("x must be bf16 or fp32")
    _cuda(x, x.dtype, "x")
    r, k = x.shape
    nbytes = lib.w4a8_nvfp4_scale_bytes(r, k)
    if nbytes == 0:
        raise W4A8Error("w4a8_nvfp4_scale_bytes", 2)
    codes = torch.empty((r, k // 2), dtype=torch.uint8, device=x.device)
    scales = torch.empty(nbytes, dtype=torch.uint8, device=x.device)
    g = torch.empty(r, dtype=torch.float32, device=x.device)
    scratch = torch.empty(4, dtype=torch.int32, device=x.device) if per_tensor else None
    _check("w4a8_nvfp4_quantize", lib.w4a8_nvfp4_quantize(
        x.data_ptr(), int(x.dtype == torch.float32), r, k, int(rotate), int(per_tensor), codes.data_ptr(),
        scales.data_ptr(), g.data_ptr(), scratch.data_ptr() if scratch is not None else None, _stream(stream)))
    return codes, scales, g


def nvfp4_pack_scales(scales_rows: torch.Tensor, stream=None) -> torch.Tensor:
    """Row-major e4m3 scale codes uint8 [R, K/16] -> the tensor cores' order."""
    lib = load_library()
    _cuda(scales_rows, torch.uint8, "scales_rows")
    r, k = scales_rows.shape[0], scales_rows.shape[1] * 16
    nbytes = lib.w4a8_nvfp4_scale_bytes(r, k)
    if nbytes == 0:
        raise W4A8Error("w4a8_nvfp4_scale_bytes", 2)
    out = torch.empty(nbytes, dtype=torch.uint8, device=scales_rows.device)
    _check("w4a8_nvfp4_pack_scales", lib.w4a8_nvfp4_pack_scales(
        scales_rows.data_ptr(), r, k, out.data_ptr(), _stream(stream)))
    return out


def nvfp4_gemm(x_codes: torch.Tensor, x_scales: torch.Tensor, g_x: torch.Tensor, w_codes: torch.Tensor,
               w_scales: torch.Tensor, g_w: torch.Tensor, out: torch.Tensor | None = None,
               stream=None) -> torch.Tensor:
    """y [M, N] bf16 from NVFP4 operands (codes [rows, K/2], scales in the
    tensor cores' order, g fp32 [rows])."""
    lib = load_library()
    for t, name in ((x_codes, "x_codes"), (x_scales, "x_scales"), (w_codes, "w_codes"), (w_scales, "w_scales")):
        _cuda(t, torch.uint8, name)
    _cuda(g_x, torch.float32, "g_x")
    _cuda(g_w, torch.float32, "g_w")
    m, k = x_codes.shape[0], x_codes.shape[1] * 2
    n = w_codes.shape[0]
    if w_codes.shape[1] * 2 != k:
        raise ValueError("x and w differ in K")
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x_codes.device)
    _cuda(out, torch.bfloat16, "out")
    _check("w4a8_nvfp4_gemm", lib.w4a8_nvfp4_gemm(
        x_codes.data_ptr(), x_scales.data_ptr(), g_x.data_ptr(), m, w_codes.data_ptr(), w_scales.data_ptr(),
        g_w.data_ptr(), n, k, out.data_ptr(), _stream(stream)))
    return out


def nvfp4_linear_workspace(m: int, k: int, device) -> torch.Tensor:
    nbytes = int(load_library().w4a8_nvfp4_linear_workspace_bytes(m, k))
    if nbytes == 0:
        raise W4A8Error("w4a8_nvfp4_linear_workspace_bytes", 2)
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def nvfp4_linear(x: torch.Tensor, w_codes: torch.Tensor, w_scales: torch.Tensor, g_w: torch.Tensor,
                 workspace: torch.Tensor | None = None, out: torch.Tensor | None = None,
                 stream=None) -> torch.Tensor:
    """The NVFP4 layer on bf16 x [M, K] (quantised per token, rotated) against
    weights from nvfp4_quantize(w, rotate=True, per_tensor=True)."""
    lib = load_library()
    _cuda(x, torch.bfloat16, "x")
    m, k = x.shape
    n = w_codes.shape[0]
    if workspace is None:
        workspace = torch.empty(lib.w4a8_nvfp4_linear_workspace_bytes(m, k), dtype=torch.uint8, device=x.device)
    if out is None:
        out = torch.empty((m, n), dtype=torch.bfloat16, device=x.device)
    _cuda(workspace, torch.uint8, "workspace")
    _cuda(out, torch.bfloat16, "out")
    _check("w4a8_nvfp4_linear", lib.w4a8_nvfp4_linear(
        x.data_ptr(), m, k, w_codes.data_ptr(), w_scales.data_ptr(), g_w.data_ptr(), n, out.data_ptr(),
        workspace.data_ptr(), workspace.numel(), _stream(stream)))
    return out
