"""The C ABI library loads and exports every entry point the header declares;
host-side argument checks reject bad calls before any device work (CPU only)."""
import ctypes
import os
import re

import pytest

import nvfp4_w4a4_quantized_04_b200 as nv
from nvfp4_w4a4_quantized_04_b200 import build as nvbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    src = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    names = re.findall(r"^[A-Za-z_][\w \*]*?\b((?:nvfp4|mxfp4)_\w+)\s*\(", src, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    nvbuild.build()
    return nv.load_library()


def test_header_declares_the_path(lib):
    names = _declared()
    for n in ["nvfp4_quantize", "nvfp4_dequantize", "mxfp4_to_nvfp4", "nvfp4_grouped_gemm",
              "nvfp4_swiglu_quantize", "nvfp4_kv_quantize", "nvfp4_kv_dequantize"]:
        assert n in names


def test_library_exports_every_declared_symbol(lib):
    raw = ctypes.CDLL(nv.LIB_PATH)
    for n in _declared():
        assert hasattr(raw, n), n
    assert set(nv.EXPORTS) <= set(_declared())


def test_sizes(lib):
    assert nv.nvfp4_padded_rows_bound(0, 1) == 128
    assert nv.nvfp4_padded_rows_bound(81920, 512) >= 81920 + 127 * 512
    assert nv.nvfp4_padded_rows_bound(300, 2) % 128 == 0
    assert nv.nvfp4_workspace_size(512) >= 512 * 8 and nv.nvfp4_workspace_size(512) % 256 == 0
    assert nv.status_string(nv.ERR_TIMEOUT) == "bounded wait timed out"


def test_host_validation_without_device(lib):
    P = ctypes.c_void_p
    fake = P(1 << 20)                   # never dereferenced: the checks fail first
    L = lib
    # K not a multiple of 16
    assert L.nvfp4_quantize(fake, 4, 24, 24, None, None, 1, 0, fake, fake, fake, 0, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # ld_x < K
    assert L.nvfp4_quantize(fake, 4, 32, 16, None, None, 1, 0, fake, fake, fake, 0, fake, None, None) == nv.ERR_INVALID_ARG
    # tiled scales need K % 64
    assert L.nvfp4_quantize(fake, 4, 32, 32, None, None, 1, 0, fake, fake, fake, 1, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # null output
    assert L.nvfp4_quantize(fake, 4, 32, 32, None, None, 1, 0, fake, None, fake, 0, fake, None, None) == nv.ERR_INVALID_ARG
    # misaligned x
    assert L.nvfp4_quantize(P((1 << 20) + 2), 4, 32, 32, None, None, 1, 0, fake, fake, fake, 0, fake, None, None) == nv.ERR_INVALID_ARG
    # bad enum
    assert L.nvfp4_quantize(fake, 4, 32, 32, None, None, 1, 7, fake, fake, fake, 0, fake, None, None) == nv.ERR_INVALID_ARG
    # too many groups
    assert L.nvfp4_quantize(fake, 4, 32, 32, None, fake, 5000, 0, fake, fake, fake, 0, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # GEMM shape limits
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 100, 512, fake, 0, 0, None, None, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 128, 320, fake, 0, 0, None, None, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, fake, 100000, 128, 128, 512, fake, 0, 0, None, None, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 128, 512, fake, 0, 3, None, None, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_grouped_gemm(None, fake, fake, fake, fake, fake, None, 1, 128, 128, 512, fake, 0, 0, None, None, None, None) == nv.ERR_INVALID_ARG
    # SwiGLU epilogue: bf16 output and an amax buffer are required
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 256, 512, fake, 0, 1, fake, None, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 256, 512, fake, 1, 1, None, None, None, None) == nv.ERR_INVALID_ARG
    # AMAX_GIVEN is an accepted mode, an unknown one is not
    assert L.nvfp4_quantize(fake, 4, 32, 32, None, None, 1, 3, fake, fake, fake, 0, fake, None, None) == nv.ERR_INVALID_ARG
    # empty problems are no-ops that touch nothing
    assert L.nvfp4_grouped_gemm(None, None, None, None, None, None, None, 1, 0, 128, 512, None, 0, 0, None, None, None, None) == nv.OK
    # the wait-budget switch rejects a negative budget before touching the device
    assert L.nvfp4_gemm_set_wait_budget(-1) == nv.ERR_INVALID_ARG
    # element-wise codecs: length multiple of 8 (E2M1) or 4 (E4M3), aligned pointers
    assert L.nvfp4_e2m1_encode(fake, 12, fake, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_e2m1_encode(fake, -8, fake, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_e2m1_encode(fake, 16, P((1 << 20) + 4), None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_e2m1_encode(None, 0, None, None) == nv.OK
    assert L.nvfp4_e4m3_encode(fake, 6, fake, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_e4m3_encode(None, 8, fake, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_e4m3_encode(None, 0, None, None) == nv.OK
    assert L.nvfp4_dequantize(None, None, 0, None, None, 1, 0, 32, None, 0, None) == nv.OK
    # remap shape limits
    assert L.mxfp4_to_nvfp4(fake, fake, 1, 4, 48, fake, fake, 0, fake, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.mxfp4_to_nvfp4(fake, fake, 1, 100, 64, fake, fake, 1, fake, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # swiglu
    assert L.nvfp4_swiglu_quantize(fake, 0, 4, 24, None, 1, fake, fake, fake, 0, fake, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # GEMM kernel switch: modes 0..4; CTA pairs cannot take N % 256 != 0
    assert L.nvfp4_gemm_select_kernel(5) == nv.ERR_INVALID_ARG
    assert L.nvfp4_gemm_select_kernel(-1) == nv.ERR_INVALID_ARG
    assert L.nvfp4_gemm_select_kernel(2) == nv.OK
    assert L.nvfp4_grouped_gemm(fake, fake, fake, fake, fake, fake, None, 1, 128, 384, 512, fake, 0, 0, None, None, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_gemm_select_kernel(0) == nv.OK
    # MoE dispatch quantize: topk 1..32, offsets required
    assert L.nvfp4_moe_quantize(fake, 4, 64, 64, fake, 0, fake, 2, 0, fake, fake, fake, 1, fake, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_moe_quantize(fake, 4, 64, 64, fake, 2, None, 2, 0, fake, fake, fake, 1, fake, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_moe_quantize(fake, 4, 48, 48, fake, 2, fake, 2, 0, fake, fake, fake, 1, fake, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    # W4A16: K % 256, N % 128, a workspace is required
    ws = fake
    assert L.nvfp4_grouped_gemm_w4a16(fake, 1088, 8, None, fake, fake, fake, None, 1, 8, 128, 1088, fake, 0, 0, ws, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_grouped_gemm_w4a16(fake, 1024, 8, None, fake, fake, fake, None, 1, 8, 96, 1024, fake, 0, 0, ws, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.nvfp4_grouped_gemm_w4a16(fake, 1024, 8, None, fake, fake, fake, None, 1, 8, 128, 1024, fake, 0, 0, None, None, None) == nv.ERR_INVALID_ARG
    assert L.nvfp4_w4a16_workspace_size(640, 384, 7168) >= 640 * 7168 * 2
    # MXFP4 encode: K % 32, K % 128 for tiled scales, aligned pointers, rows == 0 a no-op
    assert L.mxfp4_quantize(fake, 4, 48, 48, fake, fake, 0, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.mxfp4_quantize(fake, 4, 64, 64, fake, fake, 1, None, None) == nv.ERR_UNSUPPORTED_SHAPE
    assert L.mxfp4_quantize(fake, 4, 64, 60, fake, fake, 0, None, None) == nv.ERR_INVALID_ARG
    assert L.mxfp4_quantize(P((1 << 20) + 2), 4, 64, 64, fake, fake, 0, None, None) == nv.ERR_INVALID_ARG
    assert L.mxfp4_quantize(fake, 4, 64, 64, fake, fake, 2, None, None) == nv.ERR_INVALID_ARG
    assert L.mxfp4_quantize(None, 0, 64, 64, None, None, 0, None, None) == nv.OK


def test_product_path_has_no_oracle_or_cpu_fallback():
    """The package never imports the oracle and refuses to run without the library."""
    pkg = os.path.join(ROOT, "nvfp4_w4a4_quantized_04_b200")
    for fn in os.listdir(pkg):
        if fn.endswith(".py"):
            text = open(os.path.join(pkg, fn)).read()
            assert "import oracle" not in text and "from oracle" not in text, fn
    import subprocess, sys
    code = ("import nvfp4_w4a4_quantized_04_b200 as nv\n"
            "try:\n    nv.load_library('/nonexistent/libnvfp4.so')\nexcept nv.Nvfp4Error:\n    print('raised')\n")
    out = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, cwd=ROOT)
    assert "raised" in out.stdout
