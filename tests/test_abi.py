"""Host-side checks of the C ABI that need no GPU: the library loads, it
exports every function declared in include/w4a8.h, the size functions agree
with the layout arithmetic, and bad arguments are refused before any launch."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "w4a8.h")


@pytest.fixture(scope="module")
def lib():
    import __graft_entry__
    __graft_entry__.build()
    from w4a8_codebook_quantized_rotate_b200 import binding
    return binding.load_library()


def declared_functions():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const char\*|size_t|w4a8_status)\s+(w4a8_\w+)\s*\(", text, re.M)))


def test_header_declares_the_boundary():
    assert declared_functions() == sorted([
        "w4a8_chain_plan", "w4a8_chain_plan_bytes", "w4a8_chain_run", "w4a8_chain_workspace_bytes",
        "w4a8_compare", "w4a8_compare_workspace_bytes", "w4a8_convert_weight", "w4a8_convert_workspace_bytes",
        "w4a8_decode_chain", "w4a8_decode_chain_workspace_bytes", "w4a8_dense_reference",
        "w4a8_get_device_error", "w4a8_linear", "w4a8_linear_decode_static", "w4a8_linear_flagged",
        "w4a8_linear_prepare",
        "w4a8_linear_run",
        "w4a8_linear_workspace_bytes", "w4a8_nvfp4_gemm", "w4a8_nvfp4_linear",
        "w4a8_nvfp4_linear_workspace_bytes", "w4a8_nvfp4_pack_scales", "w4a8_nvfp4_quantize",
        "w4a8_nvfp4_scale_bytes", "w4a8_pack_layout",
        "w4a8_packed_bytes", "w4a8_rotate_quant_act", "w4a8_selftest_timeout", "w4a8_signal_ready",
        "w4a8_status_string", "w4a8_unpack_dequant"])


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_packed_bytes_layout_arithmetic(lib):
    # codebook (256) | row scales (4 N, padded to 256) | 32-row blocks of 0.5625 B per weight
    def expect(n, k):
        rows = -(-n // 32) * 32
        body = rows * k // 2 + rows * k // 16
        return 256 + -(-4 * n // 256) * 256 + -(-body // 256) * 256
    n, k = 17408, 5120
    assert lib.w4a8_packed_bytes(n, k) == 256 + 4 * n + n * k // 2 + n * k // 16
    assert lib.w4a8_packed_bytes(n, k) == expect(n, k)
    assert lib.w4a8_packed_bytes(16, 256) == 256 + 256 + 32 * 128 + 32 * 16
    assert lib.w4a8_packed_bytes(48, 768) == expect(48, 768)


@pytest.mark.parametrize("n,k", [(0, 256), (8, 256), (24, 256), (16, 300), (16, 0), (16, 65536), (-16, 256)])
def test_bad_weight_shapes_have_zero_size(lib, n, k):
    assert lib.w4a8_packed_bytes(n, k) == 0
    assert lib.w4a8_linear_workspace_bytes(1, k, n) == 0


def test_nvfp4_sizes(lib):
    """Scales: rows padded to 128, one byte per 16 values; the layer's
    workspace holds the activation codes, scales and per-token scalars."""
    assert lib.w4a8_nvfp4_scale_bytes(17408, 5120) == 17408 * 5120 // 16
    assert lib.w4a8_nvfp4_scale_bytes(1, 256) == 128 * 16
    assert lib.w4a8_nvfp4_scale_bytes(129, 512) == 256 * 32
    for r, k in ((0, 256), (1, 128), (1, 300), (1, 65536), (-1, 256)):
        assert lib.w4a8_nvfp4_scale_bytes(r, k) == 0
        assert lib.w4a8_nvfp4_linear_workspace_bytes(r, k) == 0
    ws = lib.w4a8_nvfp4_linear_workspace_bytes(4096, 5120)
    assert ws >= 4096 * 5120 // 2 + 4096 * 5120 // 16 + 4096 * 4


def test_nvfp4_refuses_bad_arguments_before_any_launch(lib):
    vp = ctypes.c_void_p
    fake = vp(4096)
    assert lib.w4a8_nvfp4_gemm(None, fake, fake, 16, fake, fake, fake, 128, 256, fake, None) == 1
    assert lib.w4a8_nvfp4_gemm(fake, fake, fake, 16, fake, fake, fake, 128, 200, fake, None) == 2
    assert lib.w4a8_nvfp4_gemm(fake, fake, fake, 0, fake, fake, fake, 128, 256, fake, None) == 2
    assert lib.w4a8_nvfp4_gemm(vp(4097), fake, fake, 16, fake, fake, fake, 128, 256, fake, None) == 3
    assert lib.w4a8_nvfp4_quantize(fake, 0, 4, 256, 1, 1, fake, fake, fake, None, None) == 1
    assert lib.w4a8_nvfp4_quantize(fake, 0, 4, 100, 1, 0, fake, fake, fake, None, None) == 2
    assert lib.w4a8_nvfp4_quantize(fake, 0, 4, 256, 1, 1, fake, fake, fake, vp(4098), None) == 3
    assert lib.w4a8_nvfp4_linear(fake, 4, 256, fake, fake, fake, 128, fake, fake, 16, None) == 4
    # the GEMM's grid holds at most 65535 token tiles of 128
    assert lib.w4a8_nvfp4_gemm(fake, fake, fake, 65535 * 128 + 1, fake, fake, fake, 128, 256, fake, None) == 2


# Every workspace starts with the words that join partial sums across CTAs:
# per CTA boundary (148) 32 eight-byte exchange words and a 4-byte counter.
ZERO_REGION_BYTES = (148 * 32 * 8 + 148 * 4 + 255) // 256 * 256


def test_workspace_sizes(lib):
    assert lib.w4a8_linear_workspace_bytes(0, 256, 16) == 0
    # token counts stop at 65535 GEMM tiles of 256
    assert lib.w4a8_linear_workspace_bytes(65535 * 256, 256, 16) > 0
    assert lib.w4a8_linear_workspace_bytes(65535 * 256 + 1, 256, 16) == 0
    dec = lib.w4a8_linear_workspace_bytes(1, 5120, 17408)
    pre = lib.w4a8_linear_workspace_bytes(4096, 5120, 17408)
    assert dec > 5120 * 16 and pre >= 4096 * 5120 * 2 + 4096 * 4
    # the region is there for every shape, ahead of the activations (and, for
    # the GEMM, of s_x and the fp16 x_q)
    assert dec >= ZERO_REGION_BYTES + 256 + 5120 * 16
    assert pre >= ZERO_REGION_BYTES + 4096 * 4 + 4096 * 5120 * 2
    for m in (1, 2, 9, 16, 17, 64, 65, 300):
        assert lib.w4a8_linear_workspace_bytes(m, 768, 592) > ZERO_REGION_BYTES


def test_null_and_shape_errors_before_launch(lib):
    buf = ctypes.create_string_buffer(4096 + 16)
    p = ctypes.addressof(buf) + (-ctypes.addressof(buf)) % 16   # 16-byte aligned host address
    assert lib.w4a8_pack_layout(None, p, p, p, 16, 256, p, 4096, None) == 1
    assert lib.w4a8_pack_layout(p, p, p, p, 16, 300, p, 4096, None) == 2
    assert lib.w4a8_pack_layout(p + 1, p, p, p, 16, 256, p, 4096, None) == 3
    assert lib.w4a8_pack_layout(p, p, p, p, 16, 256, p, 16, None) == 4
    assert lib.w4a8_unpack_dequant(None, 16, 256, p, None) == 1
    assert lib.w4a8_unpack_dequant(p, 15, 256, p, None) == 2
    assert lib.w4a8_rotate_quant_act(p, 1, 255, p, p, None) == 2
    assert lib.w4a8_rotate_quant_act(p, 0, 256, p, p, None) == 2
    assert lib.w4a8_rotate_quant_act(p, 1, 256, p + 8, p, None) == 3
    assert lib.w4a8_linear(p, 1, 256, p, 16, p, None, 0, None) == 1
    assert lib.w4a8_linear(p, 1, 256, p, 17, p, p, 1 << 30, None) == 2
    assert lib.w4a8_linear(p, 1, 256, p, 16, p, p, 16, None) == 4
    assert lib.w4a8_linear_prepare(None, 1, 256, 16, p, 1 << 30, None) == 1
    assert lib.w4a8_linear_prepare(p, 1, 256, 16, p + 4, 1 << 30, None) == 3
    assert lib.w4a8_linear_run(1, 256, p, 16, p, p, 8, None) == 4
    assert lib.w4a8_linear_run(1, 512, p, 16, None, p, 1 << 30, None) == 1
    assert lib.w4a8_linear_decode_static(None, 1, 256, p, 16, p, None) == 1
    assert lib.w4a8_linear_decode_static(p, 17, 256, p, 16, p, None) == 2


def test_signal_ready_refuses_before_issuing(lib):
    """A null or misaligned ready word is refused before the driver is asked
    for anything (so this runs without a GPU)."""
    assert lib.w4a8_signal_ready(None, None) == 1     # W4A8_ERR_NULL
    assert lib.w4a8_signal_ready(4, None) == 3        # W4A8_ERR_ALIGN: not 8-byte aligned


def test_status_strings(lib):
    for s in range(8):
        assert lib.w4a8_status_string(s)
    assert b"unknown" in lib.w4a8_status_string(99)


def test_convert_workspace_sizes(lib):
    assert lib.w4a8_convert_workspace_bytes(16, 256, 0) > 16 * 256 * 8
    assert lib.w4a8_convert_workspace_bytes(16, 300, 0) == 0
    assert lib.w4a8_convert_workspace_bytes(16, 256, 16 * 256 + 1) == 0   # more positions than values
    small = lib.w4a8_convert_workspace_bytes(17408, 5120, 2 ** 22)
    whole = lib.w4a8_convert_workspace_bytes(17408, 5120, 0)
    assert 2 ** 22 * 24 < small < whole


def test_convert_refuses_bad_arguments_without_a_gpu(lib):
    # null pointers and shapes are checked before any device work
    assert lib.w4a8_convert_weight(None, 16, 256, None, None, 0, 500, 1e-12, None, None, None, None, None,
                                   None, 0, None) == 1


def test_static_scratch_holds_every_decode_plan(lib):
    # The built-in scratch of w4a8_linear_decode_static must hold the
    # workspace of every shape it accepts (M <= 16, any N, K up to the
    # maximum), and should not be much larger than the largest of them.
    size = int(re.search(r"#define W4A8_STATIC_SCRATCH_BYTES \((\d+)u << (\d+)\)", open(HEADER).read())
               .group(1)) << 20
    need = max(lib.w4a8_linear_workspace_bytes(m, k, n)
               for m in (1, 2, 8, 9, 16) for k in (256, 8192, 8448, 32768) for n in (16, 5120, 17408, 1 << 20))
    assert 0 < need <= size
    assert size <= 2 * need


def test_header_is_plain_c_and_links_against_the_library(lib):
    """include/w4a8.h is a C header: a C99 program (pedantic) that includes
    it compiles, links against the built library by the declared names, and
    runs a host-only entry (no GPU needed)."""
    import shutil
    import subprocess
    gcc = shutil.which("gcc")
    if gcc is None:
        pytest.skip("no C compiler")
    out_dir = os.path.join(ROOT, "_build", "abi_c")
    os.makedirs(out_dir, exist_ok=True)
    src = os.path.join(out_dir, "abi.c")
    exe = os.path.join(out_dir, "abi")
    with open(src, "w") as f:
        f.write('#include <stdio.h>\n#include "w4a8.h"\n'
                "int main(void) {\n"
                "  size_t b = w4a8_packed_bytes(17408, 5120);\n"
                "  size_t z = w4a8_packed_bytes(17408, 100);\n"
                '  printf("%zu %zu %s\\n", b, z, w4a8_status_string(W4A8_ERR_SHAPE));\n'
                "  return 0;\n"
                "}\n")
    from w4a8_codebook_quantized_rotate_b200 import binding
    libdir = os.path.dirname(binding.LIB_PATH)
    subprocess.run([gcc, "-std=c99", "-Wall", "-Wextra", "-pedantic", "-Werror", "-I", os.path.dirname(HEADER),
                    src, "-o", exe, "-L", libdir, "-lw4a8", "-Wl,-rpath," + libdir], check=True)
    res = subprocess.run([exe], check=True, capture_output=True, text=True)
    b, z, msg = res.stdout.split(" ", 2)
    assert int(b) == 256 + 4 * 17408 + 17408 * 5120 // 2 + 17408 * 5120 // 16
    assert int(z) == 0  # K not a multiple of 256: zero size
    assert msg.strip() == lib.w4a8_status_string(2).decode()
