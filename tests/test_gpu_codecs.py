"""The device's own E2M1 and E4M3 conversions over every fp32 bit pattern (GPU,
through the C ABI).

nvfp4_e2m1_encode / nvfp4_e4m3_encode run exactly the device helpers that the
quantize kernels apply to x*r (codes) and to the block-scale quotient
(scales).  Both are compared, chunk by chunk over all 2^32 inputs, with the
oracle's encoders; the CPU pins check those against ml_dtypes over the same
2^32 inputs (E2M1 value set and packing: "DeepSeek-V4.1-Flash-NVFP4", format
section; E4M3 block scales up to 448: "Qwen3.8-Flash-Next-NVFP4", two-level
scaling section).
"""
import numpy as np
import pytest

import oracle
from tests._util import to_np

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")]

CHUNK = 1 << 28


def _patterns():
    """Yield (lo, int32 device tensor of the bit patterns lo .. lo+CHUNK-1)."""
    base = torch.arange(CHUNK, dtype=torch.int32, device="cuda")
    for lo in range(0, 1 << 32, CHUNK):
        start = lo - (1 << 32) if lo >= (1 << 31) else lo      # the same bits as a signed int32
        yield lo, base + start


def test_e2m1_encode_all_fp32_patterns():
    import nvfp4_w4a4_quantized_04_b200 as nv
    q = torch.empty(CHUNK // 2, dtype=torch.uint8, device="cuda")
    for lo, bits in _patterns():
        nv.nvfp4_e2m1_encode(bits.view(torch.float32), CHUNK, q)
        got = to_np(q)
        want = oracle.e2m1_encode_bits_range(lo, lo + CHUNK)
        packed = want[0::2] | (want[1::2] << 4)
        assert np.array_equal(got, packed), hex(lo)


def test_e4m3_encode_all_fp32_patterns():
    import nvfp4_w4a4_quantized_04_b200 as nv
    out = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    for lo, bits in _patterns():
        nv.nvfp4_e4m3_encode(bits.view(torch.float32), CHUNK, out)
        got = to_np(out)
        want = oracle.e4m3_encode_bits_range(lo, lo + CHUNK)
        assert np.array_equal(got, want), hex(lo)


def test_codec_spot_values():
    """A few values by hand: ties to even, saturation, signed zero, NaN."""
    import nvfp4_w4a4_quantized_04_b200 as nv
    v = torch.tensor([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 7.0,
                      -0.0, -0.1, float("inf"), float("-inf"), float("nan"), 6.0, -6.0, 0.5],
                     dtype=torch.float32, device="cuda")
    q = torch.empty(8, dtype=torch.uint8, device="cuda")
    nv.nvfp4_e2m1_encode(v, 16, q)
    h = to_np(q)
    codes = np.stack([h & 15, h >> 4], axis=1).reshape(-1)
    assert codes.tolist() == [0, 2, 2, 4, 4, 6, 6, 7, 8, 8, 7, 15, 0, 7, 15, 1]
    s = torch.tensor([448.0, 463.9, 464.0, 2.0 ** -9, 2.0 ** -10, -1.0, float("nan"), float("inf")],
                     dtype=torch.float32, device="cuda")
    o = torch.empty(8, dtype=torch.uint8, device="cuda")
    nv.nvfp4_e4m3_encode(s, 8, o)
    assert to_np(o).tolist() == [0x7E, 0x7E, 0x7E, 0x01, 0x00, 0xB8, 0x7F, 0x7E]
