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
}

EXPORTS = (
    "w4a8_packed_bytes", "w4a8_pack_layout", "w4a8_unpack_dequant", "w4a8_rotate_quant_act",
    "w4a8_linear_workspace_bytes", "w4a8_linear", "w4a8_linear_prepare", "w4a8_linear_run",
    "w4a8_linear_decode_static", "w4a8_get_device_error", "w4a8_status_string",
)

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
        "w4a8_status_string": (ctypes.c_char_p, [st]),
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
