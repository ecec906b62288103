"""The allocation-free quantize entry point.

nvfp4_quantize_noalloc serves callers that cannot give the library a scratch
buffer (no cudaMalloc or caching-allocator call allowed where they run); it
keeps its scratch in a static device array inside libnvfp4.so.  This test
calls it through the C ABI and checks that it produces exactly what
nvfp4_quantize produces with a caller workspace, on two calls in a row (the
second call must not see the first call's leftover scratch).
"""
import ctypes

import numpy as np
import pytest

import synthetic

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_w4a4_quantized_04_b200 import build
    build.build()
    import nvfp4_w4a4_quantized_04_b200 as nv
    return nv.load_library()


def _dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _quantize_both(L, x_bits, row_index, offsets, G, layout):
    """Run the workspace entry point and the allocation-free one on the same input."""
    import nvfp4_w4a4_quantized_04_b200 as nv
    x = _dev(x_bits.view(np.int16)).view(torch.bfloat16)
    R = len(row_index) if row_index is not None else x.shape[0]
    K = x.shape[1]
    rows_alloc = nv.nvfp4_padded_rows_bound(R, G) if offsets is not None else (R + 127) // 128 * 128
    ri = _dev(row_index) if row_index is not None else None
    off = _dev(offsets) if offsets is not None else None
    s = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    outs = []
    for noalloc in (False, True):
        q = torch.zeros((rows_alloc, K // 2), dtype=torch.uint8, device="cuda")
        sf = torch.zeros(rows_alloc * (K // 16), dtype=torch.uint8, device="cuda")
        gs = torch.zeros(max(G, 1), dtype=torch.float32, device="cuda")
        st = torch.zeros(1, dtype=torch.int32, device="cuda")
        if noalloc:
            rc = L.nvfp4_quantize_noalloc(_p(x), R, K, K, _p(ri), _p(off), G, 0, _p(gs), _p(q), _p(sf), layout,
                                          _p(st), s)
        else:
            ws = torch.empty(nv.nvfp4_workspace_size(G), dtype=torch.uint8, device="cuda")
            rc = L.nvfp4_quantize(_p(x), R, K, K, _p(ri), _p(off), G, 0, _p(gs), _p(q), _p(sf), layout, _p(ws),
                                  _p(st), s)
        assert rc == 0
        torch.cuda.synchronize()
        assert int(st.item()) == 0
        outs.append((q.cpu().numpy(), sf.cpu().numpy(), gs.cpu().numpy()))
    return outs


def test_noalloc_matches_workspace_path_twice(lib):
    # call 1: large magnitudes, 12 gathered groups
    T, H, E = 512, 1024, 12
    x1 = synthetic.gaussian_bf16(21, synthetic.STREAMS["x"], (T, H), outlier_frac=0.01)
    r = synthetic.route_topk_softmax(21, T, E, 2)
    a, b = _quantize_both(lib, x1, r["row_index"], r["offsets"], E, 1)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    # call 2: much smaller magnitudes on the same groups; stale scratch from
    # call 1 would give the wrong (larger) global scales
    x2 = synthetic.gaussian_bf16(22, synthetic.STREAMS["x"], (T, H), sigma=1e-3)
    a, b = _quantize_both(lib, x2, r["row_index"], r["offsets"], E, 1)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)
    # and a dense tensor (one group)
    x3 = synthetic.gaussian_bf16(23, synthetic.STREAMS["x"], (200, 512))
    a, b = _quantize_both(lib, x3, None, None, 1, 0)
    for u, v in zip(a, b):
        assert np.array_equal(u, v)


def test_noalloc_at_the_group_limit(lib):
    """The static array's edge: NOALLOC_MAX_GROUPS groups, most of them empty and
    a few ragged, twice in a row with different magnitudes."""
    import nvfp4_w4a4_quantized_04_b200 as nv
    G = nv.NOALLOC_MAX_GROUPS
    rng = np.random.default_rng(5)
    counts = np.zeros(G, np.int64)
    busy = rng.choice(G, size=40, replace=False)
    busy[:2] = [0, G - 1]                        # the first and the last group hold rows
    counts[busy] = rng.integers(1, 300, size=busy.size)
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    T = 700
    ri = rng.integers(0, T, size=R).astype(np.int32)
    for seed, sigma in ((31, 1.0), (32, 1e-4)):
        x = synthetic.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, 256), sigma=sigma, outlier_frac=0.002)
        a, b = _quantize_both(lib, x, ri, offsets, G, 1)
        for u, v in zip(a, b):
            assert np.array_equal(u, v)


def test_noalloc_rejects_too_many_groups(lib):
    import nvfp4_w4a4_quantized_04_b200 as nv
    fake = ctypes.c_void_p(1 << 20)
    rc = lib.nvfp4_quantize_noalloc(fake, 4, 64, 64, None, fake, nv.NOALLOC_MAX_GROUPS + 1, 0, fake, fake, fake, 0,
                                    None, None)
    assert rc == nv.ERR_UNSUPPORTED_SHAPE
