"""CUDA path vs the oracle on small seeded inputs (bit-exact for codes/scales,
the stated tolerance for GEMM outputs).  Calls go through the C ABI."""
import numpy as np
import pytest

import oracle
import synthetic
from tests._util import bf16_dev, slot_rows, tile, to_dev, to_np, untile

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module", autouse=True)
def _setup():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from nvfp4_w4a4_quantized_04_b200 import build
    build.build()
    import synthetic.cuda as sc
    sc.build()


def nvmod():
    import nvfp4_w4a4_quantized_04_b200 as nv
    return nv


def layer():
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    return L


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


@pytest.fixture(params=[0, 1, 2, 3, 4], ids=["auto", "one_cta", "cta_pair", "deep_ring", "two_blocks"])
def gemm_kernel(request):
    """Run the test on each grouped GEMM kernel: automatic (the two-block
    kernel for bf16 outputs with N % 256 == 0 and K >= 1024, else 512-element K
    stages when K % 512 == 0, with the deep ring for decode-sized groups), one
    CTA per tile with 256-element stages, the
    CTA-pair kernel, the 512-element kernel's deep ring (tiles of at most
    64 tokens, three slots), and two weight blocks per tile (bf16 outputs with
    N % 256 == 0; other calls of that mode run the automatic choice)."""
    nv = nvmod()
    nv.nvfp4_gemm_select_kernel(request.param)
    yield request.param
    nv.nvfp4_gemm_select_kernel(0)


@pytest.fixture(params=[0, 1, 3, 4], ids=["auto", "k256", "deep_ring", "two_blocks"])
def mx_kernel(request):
    """Run an MXFP4 GEMM test on the kernels that take MXFP4 operands: 512-element
    K stages (automatic when K % 512 == 0; also with the deep ring), 256-element
    stages, and two weight blocks per tile (bf16 outputs with N % 256 == 0;
    other calls of that mode run the automatic choice)."""
    nv = nvmod()
    nv.nvfp4_gemm_select_kernel(request.param)
    yield request.param
    nv.nvfp4_gemm_select_kernel(0)


def gemm_tol(y, y_ref, s_ref):
    """|y - y_ref| <= 1e-5 * sum|a*b| + 1e-6 elementwise."""
    err = np.abs(y.astype(np.float64) - y_ref)
    bound = 1e-5 * s_ref + 1e-6
    return err <= bound, err, bound


# --------------------------------------------------------------------------- quantize
@pytest.mark.parametrize("layout", [0, 1])
def test_quantize_dense_config1_bitexact(layout):
    L = layer()
    x = synthetic.gaussian_bf16(0, synthetic.STREAMS["x"], (128, 512), outlier_frac=0.001)
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
    assert st == 0
    p = L.quantize(bf16_dev(x), layout=layout)
    torch.cuda.synchronize()
    assert to_np(p.gs)[0] == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:128], q_ref)
    sf = to_np(p.sf)
    sf = untile(sf, 128, 32) if layout == 1 else sf.reshape(128, 32)
    assert np.array_equal(sf, sf_ref)


@pytest.mark.parametrize("layout", [0, 1])
def test_quantize_dense_strided_rows_one_launch(layout):
    """The ungrouped dynamic quantize runs as one cooperative launch (amax,
    global scale and encode with a grid-wide wait in between).  Rows with
    ld_x = K + 64 and a tensor of 524,288 blocks, so every CTA of the resident
    wave takes part in the wait and warps encode several chunks each: byte-exact
    to the oracle, the global scale included; the status word stays 0."""
    L = layer()
    rows, K, pad = 8192, 1024, 64
    xw = synthetic.gaussian_bf16(41, synthetic.STREAMS["x"], (rows, K + pad), outlier_frac=0.001)
    x = np.ascontiguousarray(xw[:, :K])
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
    assert st == 0
    xd = bf16_dev(xw)[:, :K]
    assert xd.stride(0) == K + pad
    s = status_word()
    p = L.quantize(xd, layout=layout, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    assert to_np(p.gs)[0] == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:rows], q_ref)
    sf = to_np(p.sf)
    sf = untile(sf, rows, K // 16) if layout == 1 else sf.reshape(-1, K // 16)[:rows]
    assert np.array_equal(sf, sf_ref)


@pytest.mark.parametrize("layout", [0, 1])
def test_quantize_dense_16byte_aligned_input(layout):
    """A dense input that is 16-byte but not 32-byte aligned takes the 16-byte
    load forms of the amax pass and the encode; many chunks per warp and a
    ragged last chunk (rows * K/16 not a multiple of 64) in the round-robin
    deal of the encode."""
    L = layer()
    rows, K = 3001, 1088
    x = synthetic.gaussian_bf16(2, synthetic.STREAMS["x"], (rows, K), outlier_frac=0.001)
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
    assert st == 0
    buf = torch.empty(rows * K + 64, dtype=torch.bfloat16, device="cuda")
    base = (buf.data_ptr() // 2) % 16                          # elements past a 32-byte boundary
    start = (16 - base) % 16 + 8                                # 16 bytes past a 32-byte boundary
    xd = buf[start:start + rows * K].view(rows, K)
    assert xd.data_ptr() % 32 == 16
    xd.copy_(bf16_dev(x))
    p = L.quantize(xd, layout=layout)
    torch.cuda.synchronize()
    assert to_np(p.gs)[0] == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:rows], q_ref)
    sf = to_np(p.sf)
    sf = untile(sf, rows, K // 16) if layout == 1 else sf.reshape(-1, K // 16)[:rows]
    assert np.array_equal(sf, sf_ref)


@pytest.mark.parametrize("layout,H", [(0, 512), (1, 512), (1, 4096), (0, 2048), (0, 2064)])
def test_quantize_grouped_gather_bitexact(layout, H):
    L = layer()
    T, E, k = 1024, 12, 2
    x = synthetic.gaussian_bf16(1, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(1, T, E, k)
    counts = np.diff(r["offsets"])
    assert counts.max() > 128            # a group spanning two slot tiles
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x, r["row_index"], r["offsets"])
    assert st == 0
    off = to_dev(r["offsets"])
    out = L.empty_packed(T * k, H, E, off, layout)
    out.q.fill_(0xAB)                       # padding rows must keep this: they are not written
    out.sf.fill_(0xAB)
    p = L.quantize(bf16_dev(x), to_dev(r["row_index"]), off, E, layout=layout, out=out)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(p.gs), gs_ref)
    rows, starts = slot_rows(r["offsets"])
    used = int(starts[-1])
    q = to_np(p.q)
    assert np.array_equal(q[rows], q_ref)
    pad = np.setdiff1d(np.arange(used), rows)
    assert (q[pad] == 0xAB).all()
    sf = to_np(p.sf)
    sfm = untile(sf, p.q.shape[0], H // 16) if layout == 1 else sf.reshape(-1, H // 16)
    assert np.array_equal(sfm[rows], sf_ref)
    assert (sfm[pad] == 0xAB).all()


# --------------------------------------------------------------------------- token-order MoE quantize
def _moe_quantize_check(x, slot, off, E, layout, x_dev=None):
    """nvfp4_moe_quantize against the oracle's gathered per-expert quantize
    (row_index = inverse of slot): bit-exact in every routed row."""
    L = layer()
    R = int(off[-1])
    t, c = np.nonzero(slot >= 0)
    ri = np.full(R, -1, np.int64)
    ri[slot[t, c]] = t
    assert (ri >= 0).all()
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x, ri.astype(np.int32), off)
    assert st == 0
    s = status_word()
    K = x.shape[1]
    out = L.empty_packed(R, K, E, to_dev(off), layout)
    out.q.fill_(0xAB)
    out.sf.fill_(0xAB)
    p = L.moe_quantize(bf16_dev(x) if x_dev is None else x_dev, to_dev(slot.astype(np.int32)), to_dev(off), E,
                       layout=layout, out=out, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    assert np.array_equal(to_np(p.gs), gs_ref)
    rows, starts = slot_rows(off)
    q = to_np(p.q)
    assert np.array_equal(q[rows], q_ref)
    pad = np.setdiff1d(np.arange(int(starts[-1])), rows)
    assert (q[pad] == 0xAB).all()
    sf = to_np(p.sf)
    sfm = untile(sf, p.q.shape[0], K // 16) if layout == 1 else sf.reshape(-1, K // 16)
    assert np.array_equal(sfm[rows], sf_ref)
    assert (sfm[pad] == 0xAB).all()


@pytest.mark.parametrize("layout,T,H,E,k", [(1, 1024, 512, 12, 2), (0, 1024, 2064, 12, 2), (1, 300, 7168, 40, 8),
                                            (1, 2048, 4096, 64, 10), (0, 5, 64, 3, 3), (1, 8192, 4096, 512, 10),
                                            (1, 777, 1024, 9, 1), (1, 64, 10240, 16, 32)])
def test_moe_quantize_bitexact(layout, T, H, E, k):
    x = synthetic.gaussian_bf16(21, synthetic.STREAMS["x"], (T, H), outlier_frac=0.001)
    r = synthetic.route_topk_softmax(21, T, E, k)
    _moe_quantize_check(x, r["slot"], r["offsets"], E, layout)


def test_moe_quantize_strided_rows():
    """ld_x = K + 8 (rows not 32-byte aligned: the two 16-byte load path)."""
    T, H, E, k = 333, 512, 7, 3
    xw = synthetic.gaussian_bf16(22, synthetic.STREAMS["x"], (T, H + 8), outlier_frac=0.01)
    r = synthetic.route_topk_softmax(22, T, E, k)
    xd = bf16_dev(xw)[:, :H]
    _moe_quantize_check(np.ascontiguousarray(xw[:, :H]), r["slot"], r["offsets"], E, 0, x_dev=xd)


def test_moe_quantize_scale_ties_and_near_ties():
    """Blocks whose amax over 6*s_g is exactly an E4M3 rounding midpoint (ties
    to even) or one bf16 step from it.  With s_g = 2^-4 (the expert amax is
    2688 * 2^-4 = 168) each quotient is exact, so the division the kernel may
    skip in the common case must be taken here and must round like the oracle."""
    import ml_dtypes
    codes = np.arange(0, 126, dtype=np.uint8)
    v = codes.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    w = (codes + 1).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    mids = (v + w) / 2                                        # 126 midpoints, at most 5 significant bits
    a = synthetic.f32_to_bf16_bits((mids * 6 * 2.0 ** -4).astype(np.float32))
    assert np.array_equal(synthetic.bf16_bits_to_f32(a).astype(np.float64), mids * 6 * 2.0 ** -4)
    amaxes = np.concatenate([a, a + 1, a - 1])               # ties, one bf16 step above and below
    amaxes = amaxes[synthetic.bf16_bits_to_f32(amaxes) > 0]
    T, H = 64, 512
    x = np.zeros((T, H), np.uint16)
    x[0, 0] = synthetic.f32_to_bf16_bits(np.float32([168.0]))[0]            # expert amax -> s_g = 2^-4
    blocks = x.reshape(T, H // 16, 16)
    flat = blocks.reshape(-1, 16)
    n = min(len(amaxes), flat.shape[0] - 1)
    flat[1:1 + n, 3] = amaxes[:n]                                            # the block amax
    flat[1:1 + n, 7] = synthetic.f32_to_bf16_bits(-0.5 * synthetic.bf16_bits_to_f32(amaxes[:n]))  # exact halves
    x = flat.reshape(T, H)
    slot = np.arange(T, dtype=np.int64).reshape(T, 1)
    off = np.array([0, T], dtype=np.int32)
    _moe_quantize_check(x, slot, off, 1, 1)
    _, _, gs_ref, _ = oracle.quantize(x, None, off)
    assert gs_ref[0] == np.float32(2.0 ** -4)


def test_moe_quantize_dropped_choices_and_bad_index():
    """Choices with slot -1 are skipped; a slot beyond the routed rows is
    reported as an index error and skipped."""
    L = layer()
    T, H, E, k = 200, 256, 6, 3
    x = synthetic.gaussian_bf16(23, synthetic.STREAMS["x"], (T, H))
    experts = synthetic.route_topk_softmax(23, T, E, k)["experts"].astype(np.int64)
    rng = np.random.default_rng(23)
    experts[rng.random((T, k)) < 0.15] = -1
    t, c = np.nonzero(experts >= 0)
    e = experts[t, c]
    order = np.lexsort((c, t, e))
    slot = np.full((T, k), -1, np.int64)
    slot[t[order], c[order]] = np.arange(len(order))
    off = np.concatenate([[0], np.cumsum(np.bincount(e, minlength=E))]).astype(np.int32)
    _moe_quantize_check(x, slot, off, E, 1)
    bad = slot.copy()
    bad[0, np.argmax(bad[0] >= 0)] = int(off[-1]) + 3
    s = status_word()
    L.moe_quantize(bf16_dev(x), to_dev(bad.astype(np.int32)), to_dev(off), E, layout=1, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 19


def test_quantize_groups_with_empty_experts():
    L = layer()
    H = 256
    offsets = np.array([0, 0, 3, 3, 3, 200, 200, 201], dtype=np.int32)
    x = synthetic.gaussian_bf16(2, synthetic.STREAMS["x"], (201, H))
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x, None, offsets)
    p = L.quantize(bf16_dev(x), None, to_dev(offsets), 7, layout=1)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(p.gs), gs_ref)        # empty groups: s_g = 1
    rows, _ = slot_rows(offsets)
    assert np.array_equal(to_np(p.q)[rows], q_ref)
    assert np.array_equal(untile(to_np(p.sf), p.q.shape[0] // 128 * 128, H // 16)[rows], sf_ref)


def test_quantize_and_dispatch_with_4096_groups():
    """4096 groups, the most the quantizers take (their group tables sit in
    shared memory): mostly empty, a few with 1-5 rows.  The grouped quantize and
    the token-order dispatch (top-2) are both bit-exact to the oracle."""
    rng = np.random.default_rng(26)
    G, H = 4096, 256
    counts = np.where(rng.random(G) < 0.9, 0, rng.integers(1, 6, G))
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    L = layer()
    x = synthetic.gaussian_bf16(26, synthetic.STREAMS["x"], (R, H))
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x, None, offsets)
    assert st == 0
    p = L.quantize(bf16_dev(x), None, to_dev(offsets), G, layout=1)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(p.gs), gs_ref)
    rows, _ = slot_rows(offsets)
    assert np.array_equal(to_np(p.q)[rows], q_ref)
    assert np.array_equal(untile(to_np(p.sf), p.q.shape[0] // 128 * 128, H // 16)[rows], sf_ref)
    T = 700
    xt = synthetic.gaussian_bf16(27, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(27, T, G, 2)
    _moe_quantize_check(xt, r["slot"], r["offsets"], G, 1)


@pytest.mark.parametrize("shape", [(1, 16), (5, 48), (3, 208), (0, 64), (1000, 16), (7, 1040), (33, 5120),
                                   (2, 17408)])
def test_quantize_ragged_shapes(shape):
    L = layer()
    x = synthetic.gaussian_bf16(7, synthetic.STREAMS["x"], shape, outlier_frac=0.01)
    R, K = shape
    if R == 0:
        xd = torch.empty((0, K), dtype=torch.bfloat16, device="cuda")
        p = L.quantize(xd, layout=0)
        torch.cuda.synchronize()
        assert to_np(p.gs)[0] == 1.0
        return
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
    p = L.quantize(bf16_dev(x), layout=0)
    torch.cuda.synchronize()
    assert to_np(p.gs)[0] == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:R], q_ref)
    assert np.array_equal(to_np(p.sf)[:R * K // 16].reshape(R, K // 16), sf_ref)


def _special_tensor():
    """Zeros, -0, tiny and huge magnitudes, exact E2M1 midpoints after scaling."""
    f = np.zeros((8, 64), dtype=np.float32)
    f[0, :16] = 6.0 * np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5, 6, -0.25, -0.75, -1.25, -1.75, -2.5, -3.5, -5, -6]) / 6
    f[1, :] = -0.0
    f[2, :16] = np.float32(1e-30)
    f[2, 16:32] = -np.float32(3e-38)
    f[3, :] = np.linspace(-3, 3, 64)
    f[4, 5] = 1e30
    f[5, :16] = [1, 1e-5, 2e-6, 0, -0.0, 1e-7, 3e-8, 1, 0.5, 0.25, 0.125, 0.0625, 0.03125, 1e-3, 1e-4, 1e-9]
    return synthetic.f32_to_bf16_bits(f)


def test_quantize_special_values():
    L = layer()
    x = _special_tensor()
    for layout in (0, 1):
        q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
        p = L.quantize(bf16_dev(x), layout=layout)
        torch.cuda.synchronize()
        assert to_np(p.gs)[0] == gs_ref[0]
        assert np.array_equal(to_np(p.q)[:8], q_ref)
    # a tensor whose amax is tiny (subnormal global scale)
    tiny = np.zeros((2, 32), dtype=np.float32)
    tiny[0, 3] = 3e-38
    tiny[1, 9] = -1.2e-39
    tiny[1, 10] = -0.0
    xb = synthetic.f32_to_bf16_bits(tiny)
    q_ref, sf_ref, gs_ref, st = oracle.quantize(xb)
    p = L.quantize(bf16_dev(xb), layout=0)
    torch.cuda.synchronize()
    assert to_np(p.gs)[0] == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:2], q_ref)
    assert np.array_equal(to_np(p.sf)[:4].reshape(2, 2), sf_ref)


def test_quantize_all_zero_tensor():
    L = layer()
    x = np.zeros((4, 128), dtype=np.uint16)
    x[2, 7] = 0x8000
    q_ref, sf_ref, gs_ref, st = oracle.quantize(x)
    p = L.quantize(bf16_dev(x), layout=0)
    torch.cuda.synchronize()
    assert to_np(p.gs)[0] == 1.0 == gs_ref[0]
    assert np.array_equal(to_np(p.q)[:4], q_ref)
    assert (to_np(p.sf)[:32] == 0).all()


def test_quantize_given_scale_and_nonfinite_status():
    L = layer()
    x = synthetic.gaussian_bf16(3, synthetic.STREAMS["x"], (64, 256))
    gs = np.array([0.0123], dtype=np.float32)
    q_ref, sf_ref, _, st = oracle.quantize(x, global_scale=gs)
    p = L.quantize(bf16_dev(x), layout=0, global_scale=to_dev(gs))
    torch.cuda.synchronize()
    assert np.array_equal(to_np(p.q)[:64], q_ref)
    assert np.array_equal(to_np(p.sf)[:64 * 16].reshape(64, 16), sf_ref)
    for bad in (0x7FC0, 0x7F80, 0xFF80):
        xb = x.copy()
        xb[10, 100] = bad
        for given in (None, to_dev(gs)):
            s = status_word()
            L.quantize(bf16_dev(xb), layout=0, global_scale=given, dev_status=s)
            torch.cuda.synchronize()
            assert int(s.item()) == oracle.ERR_NONFINITE == 16


def test_status_word_first_error_wins():
    """The device status word keeps the first error: a word already holding an
    error (here NOT_REPRESENTABLE, as if a remap had failed) is not overwritten
    by a quantize that meets a NaN, and a word holding NONFINITE is not
    overwritten by a routing call that meets an expert id out of range."""
    L = layer()
    x = synthetic.gaussian_bf16(3, synthetic.STREAMS["x"], (64, 256))
    x[7, 9] = 0x7FC0                                       # NaN
    s = torch.full((1,), 17, dtype=torch.int32, device="cuda")
    L.quantize(bf16_dev(x), layout=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 17
    s = status_word()
    L.quantize(bf16_dev(x), layout=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 16
    L.route(to_dev(np.array([[0, 1], [2, 9]], dtype=np.int32)), 4, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 16


# --------------------------------------------------------------------------- dequantize
@pytest.mark.parametrize("layout", [0, 1])
def test_dequantize_bitexact(layout):
    L = layer()
    rng = np.random.default_rng(0)
    R, K = 256, 256
    q = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, (R, K // 16), dtype=np.uint8)
    gs = np.array([0.0371], dtype=np.float32)
    ref32 = oracle.dequantize(q, sf, np.full(R, gs[0], np.float32))
    ref16 = oracle.dequantize(q, sf, np.full(R, gs[0], np.float32), out="bf16")
    sfd = tile(sf) if layout == 1 else sf.reshape(-1)
    p = L.Packed(to_dev(q), to_dev(sfd), to_dev(gs), R, K, layout)
    y32 = L.dequantize(p, 0)
    y16 = L.dequantize(p, 1)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(y32).view(np.uint32), ref32.view(np.uint32))
    assert np.array_equal(to_np(y16), ref16)


@pytest.mark.parametrize("R,K", [(333, 1088), (1, 64), (7, 48), (4099, 256)])
@pytest.mark.parametrize("y_offset", [0, 16])
def test_dequantize_ragged_and_alignments(R, K, y_offset):
    """Ungrouped dequantize: block counts that are not a multiple of the
    kernel's per-warp step, every layout and output type, and an output that is
    16 but not 32 bytes aligned (the per-thread kernel then runs instead of the
    flat one).  Bit-exact either way."""
    nv = nvmod()
    rng = np.random.default_rng(R + K)
    q = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, (R, K // 16), dtype=np.uint8)
    gs = np.array([2.0 ** -7 * 1.375], dtype=np.float32)
    ref32 = oracle.dequantize(q, sf, np.full(R, gs[0], np.float32))
    ref16 = oracle.dequantize(q, sf, np.full(R, gs[0], np.float32), out="bf16")
    layouts = [0, 1] if K % 64 == 0 else [0]
    for layout in layouts:
        if layout == 1:
            sfa = np.zeros(((R + 127) // 128 * 128, K // 16), np.uint8)
            sfa[:R] = sf
            sfd = to_dev(tile(sfa))
        else:
            sfd = to_dev(sf.reshape(-1))
        for out_dtype, ref, esz in ((0, ref32.view(np.uint32), 4), (1, ref16, 2)):
            buf = torch.zeros(R * K * esz + 64, dtype=torch.uint8, device="cuda")
            base = (-buf.data_ptr()) % 32 + y_offset
            yv = buf[base:base + R * K * esz]
            nv.nvfp4_dequantize(to_dev(q), sfd, layout, to_dev(gs), None, 1, R, K, yv, out_dtype)
            torch.cuda.synchronize()
            got = to_np(yv).view(np.uint32 if esz == 4 else np.uint16).reshape(R, K)
            assert np.array_equal(got, ref), (layout, out_dtype)


def test_dequantize_grouped_slots():
    L = layer()
    T, H, E = 128, 256, 5
    x = synthetic.gaussian_bf16(4, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(4, T, E, 2)
    q_ref, sf_ref, gs_ref, _ = oracle.quantize(x, r["row_index"], r["offsets"])
    ref = oracle.dequantize(q_ref, sf_ref, oracle.rows_global_scale(gs_ref, r["offsets"], len(r["row_index"])))
    p = L.quantize(bf16_dev(x), to_dev(r["row_index"]), to_dev(r["offsets"]), E, layout=1)
    y = L.dequantize(p, 0)
    torch.cuda.synchronize()
    assert np.array_equal(to_np(y).view(np.uint32), ref.view(np.uint32))


# --------------------------------------------------------------------------- remap
def _mx(seed, n, rows, K, lo=-10):
    q = synthetic.mxfp4_codes(seed, synthetic.STREAMS["mx_codes"], n * rows * K // 2).reshape(n * rows, K // 2)
    e = synthetic.mxfp4_exponents(seed, synthetic.STREAMS["mx_exp"], n * rows * K // 32, lo=lo).reshape(n * rows, K // 32)
    return q, e


# Shapes for the scale pass's paths: 16-byte exponent loads with runs of 8 or
# 16 scale groups (K = 512, 1024), byte loads (K/32 not a multiple of 16:
# K = 128, 1152, 2112) with partial runs (1152: 16 + 2 groups, 2112: 16+16+1),
# and an exponent pointer that is not 16-byte aligned.
@pytest.mark.parametrize("layout", [0, 1])
@pytest.mark.parametrize("n,rows,K,e_offset", [(3, 128, 512, 0), (2, 256, 128, 0), (1, 128, 1024, 0),
                                               (2, 128, 1152, 0), (1, 256, 2112, 0), (1, 128, 1024, 1)])
def test_remap_bitexact(layout, n, rows, K, e_offset):
    L = layer()
    q, e = _mx(0, n, rows, K)
    q[5, :16] = 0x88                            # one all -0 block (exempt)
    e[5, 0] = 3
    q_ref, sf_ref, gs_ref, st = oracle.remap_mxfp4(q, e, n, rows, K)
    assert st == 0
    s = status_word()
    e_dev = to_dev(e)
    if e_offset:
        buf = torch.empty(e.size + 16, dtype=torch.uint8, device="cuda")
        e_dev = buf[e_offset:e_offset + e.size].view(e.shape)
        e_dev.copy_(to_dev(e))
    p = L.remap_mxfp4(to_dev(q), e_dev, n, rows, K, layout=layout, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    assert np.array_equal(to_np(p.gs), gs_ref)
    assert np.array_equal(to_np(p.q), q_ref)
    sf = to_np(p.sf)
    sf = untile(sf, n * rows, K // 16) if layout == 1 else sf.reshape(n * rows, K // 16)
    assert np.array_equal(sf, sf_ref)
    # lossless: the GPU's NVFP4 dequantizes to the MXFP4 values exactly
    for t in range(n):
        sl = slice(t * rows, (t + 1) * rows)
        dq = oracle.dequantize_f64(to_np(p.q)[sl], sf[sl], np.full(rows, to_np(p.gs)[t], np.float32))
        assert np.array_equal(dq, oracle.dequantize_mxfp4_f64(q[sl], e[sl]))


# --------------------------------------------------------------------------- MXFP4 encode
def _mx_input(seed, rows, K, ld=None):
    """Gaussian rows, each 32-block scaled by its own power of two over the
    bf16 range (subnormal amax to ~2^120), plus hand-placed edge blocks."""
    ld = ld or K
    lp = (ld + 31) // 32 * 32
    z = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(seed, 1, (rows, lp))).astype(np.float64)
    mag = np.ldexp(1.0, (synthetic.words(seed, 2, 0, rows * lp // 32) % 250).astype(np.int64) - 130)
    x = synthetic.f32_to_bf16_bits((z * np.repeat(mag, 32).reshape(rows, lp)).astype(np.float32))
    x = np.ascontiguousarray(x[:, :ld])
    x[0, :32] = 0                                             # all-zero block
    x[0, 32:64] = 0x8000                                      # all -0 block
    x[1, :32] = synthetic.f32_to_bf16_bits(np.float32([1e30] + [-1e-30] * 31))   # products underflow to -0
    x[1, 32:64] = synthetic.f32_to_bf16_bits(np.float32([4.0, 5.0, 2.5, -1.75, 0.25] + [0.0] * 27))  # ties
    x[2, :32] = np.arange(1, 33, dtype=np.uint16)             # subnormal-only block
    return x


@pytest.mark.parametrize("rows, K, ld, layout", [(300, 1024, 1024, 0), (300, 1024, 1024, 1),
                                                  (7, 96, 104, 0), (129, 384, 400, 1)])
def test_mxfp4_quantize_bitexact(rows, K, ld, layout):
    L = layer()
    xw = _mx_input(31, rows, K, ld)
    q_ref, e_ref, st = oracle.quantize_mxfp4(np.ascontiguousarray(xw[:, :K]))
    assert st == 0
    s = status_word()
    xd = bf16_dev(xw)[:, :K]
    q, e = L.mxfp4_quantize(xd, layout=layout, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    assert np.array_equal(to_np(q), q_ref)
    e = to_np(e)
    e = untile(e, (rows + 127) // 128 * 128, K // 32)[:rows] if layout == 1 else e
    assert np.array_equal(e, e_ref)


def test_mxfp4_quantize_nonfinite_blocks():
    L = layer()
    rows, K = 64, 256
    x = _mx_input(32, rows, K)
    x[3, 40] = 0x7F80                                        # +inf
    x[9, 200] = 0xFFC1                                       # NaN
    q_ref, e_ref, st = oracle.quantize_mxfp4(x)
    assert st == oracle.ERR_NONFINITE
    s = status_word()
    q, e = L.mxfp4_quantize(bf16_dev(x), dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == oracle.ERR_NONFINITE
    assert np.array_equal(to_np(q), q_ref) and np.array_equal(to_np(e), e_ref)
    assert to_np(e)[3, 1] == 0xFF and to_np(e)[9, 6] == 0xFF


def test_mxfp4_quantize_then_remap_lossless_on_device():
    """Both device kernels in a row: MXFP4 encode, then the NVFP4 remap, which
    must dequantize to the oracle's MXFP4 values exactly."""
    L = layer()
    rows, K = 256, 512
    x = synthetic.gaussian_bf16(33, 1, (rows, K))
    q_ref, e_ref, _ = oracle.quantize_mxfp4(x)
    q, e = L.mxfp4_quantize(bf16_dev(x))
    s = status_word()
    p = L.remap_mxfp4(q, e, 1, rows, K, layout=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    got = oracle.dequantize_f64(to_np(p.q), to_np(p.sf).reshape(rows, K // 16), np.full(rows, to_np(p.gs)[0], np.float32))
    assert np.array_equal(got, oracle.dequantize_mxfp4_f64(q_ref, e_ref))


def test_mxfp4_quantize_full_size_sampled_rows():
    """The bench's workload (65,536 x 4,096 bf16, 2^28 elements, tiled scales):
    sampled rows against the oracle."""
    import synthetic.cuda as sc
    L = layer()
    rows, K = 65536, 4096
    xd = sc.gaussian_bf16(34, 1, (rows, K))
    q, e = L.mxfp4_quantize(xd, layout=1)
    torch.cuda.synchronize()
    pick = np.array([0, 1, 127, 128, 4097, 33333, rows - 129, rows - 1])
    xs = to_np(xd[torch.from_numpy(pick).cuda()])
    q_ref, e_ref, _ = oracle.quantize_mxfp4(xs)
    assert np.array_equal(to_np(q)[pick], q_ref)
    e_rm = untile(to_np(e), rows, K // 32)
    assert np.array_equal(e_rm[pick], e_ref)


def _run_mx_gemm(x_bits, w_bits, offsets, E, N, K, out_dtype):
    """MXFP4 GEMM on oracle-encoded operands; returns (y, y_ref, s_ref)."""
    L = layer()
    nv = nvmod()
    R = x_bits.shape[0]
    qa, ea, st = oracle.quantize_mxfp4(x_bits)
    qw, ew, st2 = oracle.quantize_mxfp4(w_bits)
    assert st == 0 and st2 == 0
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qs = np.zeros((bound, K // 2), np.uint8)
    es = np.zeros((bound, K // 32), np.uint8)
    if offsets is not None:
        rows, _ = slot_rows(offsets)
    else:
        rows = np.arange(R)
    qs[rows] = qa
    es[rows] = ea
    s = status_word()
    y = L.mx_grouped_gemm(to_dev(qs), to_dev(tile(es)), to_dev(qw), to_dev(tile(ew)), N, K, R,
                          to_dev(offsets) if offsets is not None else None, E, out_dtype, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    a = oracle.dequantize_mxfp4_f64(qa, ea)
    b = oracle.dequantize_mxfp4_f64(qw, ew)
    if offsets is None:
        y_ref, s_ref = oracle.gemm_f64(a, b)
    else:
        y_ref, s_ref = oracle.grouped_gemm_f64(a, b.reshape(E, N, K), offsets)
    return to_np(y), y_ref, s_ref


def test_mx_gemm_wide_exponent_range(mx_kernel):
    """Random E2M1 codes with UE8M0 bytes spread over 2^-57 ... 2^53 on both
    operands (products stay finite in fp32), some blocks at 2^-127: the
    tensor core's reading of each exponent byte against the fp64 oracle."""
    L = layer()
    nv = nvmod()
    rng = np.random.default_rng(25)
    E, N, K = 2, 256, 1024
    counts = [90, 150]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    qa = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    ea = rng.integers(70, 181, (R, K // 32), dtype=np.uint8)
    qw = rng.integers(0, 256, (E * N, K // 2), dtype=np.uint8)
    ew = rng.integers(70, 181, (E * N, K // 32), dtype=np.uint8)
    ea[3, :5] = 0                                                   # 2^-127
    ew[7, :5] = 0
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qs = np.zeros((bound, K // 2), np.uint8)
    es = np.zeros((bound, K // 32), np.uint8)
    rows, _ = slot_rows(offsets)
    qs[rows] = qa
    es[rows] = ea
    s = status_word()
    y = L.mx_grouped_gemm(to_dev(qs), to_dev(tile(es)), to_dev(qw), to_dev(tile(ew)), N, K, R,
                          to_dev(offsets), E, 0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    a = oracle.dequantize_mxfp4_f64(qa, ea)
    b = oracle.dequantize_mxfp4_f64(qw, ew)
    y_ref, s_ref = oracle.grouped_gemm_f64(a, b.reshape(E, N, K), offsets)
    ok, err, bnd = gemm_tol(to_np(y), y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bnd).max())


def test_mx_gemm_closed_form_integer_case(mx_kernel):
    """All UE8M0 scales 1: every product is a multiple of 1/4 and the fp32 sum
    is exact, so the kind::mxf4 result must equal the oracle exactly."""
    L = layer()
    rng = np.random.default_rng(1)
    M, N, K = 128, 256, 512
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    ea = np.full((M, K // 32), 127, np.uint8)
    ew = np.full((N, K // 32), 127, np.uint8)
    ea[5, 3] = 129                                   # a few non-unit scales (still exact sums)
    ew[7, 0] = 125
    s = status_word()
    y = L.mx_grouped_gemm(to_dev(qa), to_dev(tile(ea)), to_dev(qw), to_dev(tile(ew)), N, K, M, out_dtype=0,
                          dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    y_ref, _ = oracle.gemm_f64(oracle.dequantize_mxfp4_f64(qa, ea), oracle.dequantize_mxfp4_f64(qw, ew))
    assert np.array_equal(to_np(y).astype(np.float64), y_ref)


@pytest.mark.parametrize("out_dtype", [0, 1])
def test_mx_gemm_dense_many_tiles(out_dtype, mx_kernel):
    M, N, K = 1000, 384, 1024
    x = synthetic.gaussian_bf16(41, synthetic.STREAMS["x"], (M, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(41, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    y, y_ref, s_ref = _run_mx_gemm(x, w, None, 1, N, K, 0)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max())
    if out_dtype == 1:
        y16, _, _ = _run_mx_gemm(x, w, None, 1, N, K, 1)
        assert np.array_equal(y16, synthetic.f32_to_bf16_bits(y))


def test_mx_gemm_grouped_chunk_edges(mx_kernel):
    counts = [1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 257, 385, 0, 2, 17, 33]
    E, N, K = len(counts), 256, 512
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(42, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(42, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    y, y_ref, s_ref = _run_mx_gemm(x, w, offsets, E, N, K, 0)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max(), np.argwhere(~ok)[:5])
    # bf16 Y (the two-block kernel in modes 0 and 4 at K >= 1024 or in mode 4)
    # is the round-to-nearest-even of the fp32 Y
    y16, _, _ = _run_mx_gemm(x, w, offsets, E, N, K, 1)
    assert np.array_equal(y16, synthetic.f32_to_bf16_bits(y))


def _mx_gemm_raw(qa, ea, qw, ew, offsets, E, N, K, out_dtype, mode):
    """MXFP4 GEMM of raw codes and exponent bytes on kernel mode `mode`."""
    L = layer()
    nv = nvmod()
    bound = nv.nvfp4_padded_rows_bound(qa.shape[0], E)
    qs = np.zeros((bound, K // 2), np.uint8)
    es = np.zeros((bound, K // 32), np.uint8)
    rows, _ = slot_rows(offsets)
    qs[rows] = qa
    es[rows] = ea
    s = status_word()
    nv.nvfp4_gemm_select_kernel(mode)
    try:
        y = L.mx_grouped_gemm(to_dev(qs), to_dev(tile(es)), to_dev(qw), to_dev(tile(ew)), N, K, qa.shape[0],
                              to_dev(offsets), E, out_dtype, dev_status=s)
        torch.cuda.synchronize()
    finally:
        nv.nvfp4_gemm_select_kernel(0)
    assert int(s.item()) == 0
    return to_np(y)


@pytest.mark.parametrize("counts", [[90, 150, 0, 1, 255, 257, 129, 64],
                                    [1, 63, 64, 65, 0, 2, 17] + [0] * 30 + [3]],
                         ids=["groups", "small_groups"])
def test_mx_gemm_two_blocks_bf16(counts):
    """bf16 MXFP4 GEMMs with N % 256 == 0 and K >= 1024 run on the two-block
    kernel (automatic choice; 64-token ring when M_total <= 16 E): its bf16 Y
    must be the bf16 rounding of the fp32 Y of the one-CTA 256-element kernel,
    which sits within the fp32 accumulation bound of the fp64 oracle.  UE8M0
    bytes spread over 2^-57 ... 2^53, a few at 2^-127."""
    rng = np.random.default_rng(26)
    E, N, K = len(counts), 512, 1024
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    qa = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    ea = rng.integers(70, 181, (R, K // 32), dtype=np.uint8)
    qw = rng.integers(0, 256, (E * N, K // 2), dtype=np.uint8)
    ew = rng.integers(70, 181, (E * N, K // 32), dtype=np.uint8)
    ea[3, :5] = 0
    ew[N + 7, :5] = 0
    y32 = _mx_gemm_raw(qa, ea, qw, ew, offsets, E, N, K, 0, 1)
    y16 = _mx_gemm_raw(qa, ea, qw, ew, offsets, E, N, K, 1, 0)
    a = oracle.dequantize_mxfp4_f64(qa, ea)
    b = oracle.dequantize_mxfp4_f64(qw, ew)
    y_ref, s_ref = oracle.grouped_gemm_f64(a, b.reshape(E, N, K), offsets)
    ok, err, bnd = gemm_tol(y32, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bnd).max())
    assert np.array_equal(y16, synthetic.f32_to_bf16_bits(y32))


def test_mx_gemm_matches_remapped_nvfp4_gemm():
    """The two routes for MXFP4 weights: the direct kind::mxf4 GEMM, and the
    lossless NVFP4 remap followed by the NVFP4 GEMM.  Both multiply the same
    values, so both sit within the fp32 accumulation bound of one fp64 result."""
    L = layer()
    M, N, K = 256, 256, 1024
    x = synthetic.gaussian_bf16(43, synthetic.STREAMS["x"], (M, K))
    w = synthetic.gaussian_bf16(43, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    y_mx, y_ref, s_ref = _run_mx_gemm(x, w, None, 1, N, K, 0)
    qa, ea, _ = oracle.quantize_mxfp4(x)
    qw, ew, _ = oracle.quantize_mxfp4(w)
    pa = L.remap_mxfp4(to_dev(qa), to_dev(ea), 1, M, K, layout=1)
    pw = L.remap_mxfp4(to_dev(qw), to_dev(ew), 1, N, K, layout=1)
    # the GEMM's token operand spans nvfp4_padded_rows_bound rows: pad the remapped copy
    bound = nvmod().nvfp4_padded_rows_bound(M, 1)
    qpad = torch.zeros((bound, K // 2), dtype=torch.uint8, device="cuda")
    qpad[:M] = pa.q
    spad = torch.zeros(bound * (K // 16), dtype=torch.uint8, device="cuda")
    spad[:pa.sf.numel()] = pa.sf
    a_nv = L.Packed(qpad, spad, pa.gs, M, K, 1, None, 1)
    y_nv = to_np(L.grouped_gemm(a_nv, pw, N, 0))
    for y in (y_mx, y_nv):
        ok, err, bound = gemm_tol(y, y_ref, s_ref)
        assert ok.all(), (err.max(), (err / bound).max())


def test_remap_errors_and_inplace():
    L = layer()
    rows, K = 128, 64
    q = np.full((rows, K // 2), 0x22, dtype=np.uint8)
    e = np.full((rows, K // 32), 127, dtype=np.uint8)
    e[0, 0] = 127 + 8
    e[3, 1] = 127 - 9
    q_ref, sf_ref, gs_ref, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    qd = to_dev(q)
    s = status_word()
    p = L.remap_mxfp4(qd, to_dev(e), 1, rows, K, layout=0, dev_status=s, inplace=True)
    torch.cuda.synchronize()
    assert int(s.item()) == 0 and p.q.data_ptr() == qd.data_ptr()
    assert np.array_equal(to_np(p.sf).reshape(rows, K // 16), sf_ref)
    assert to_np(p.gs)[0] == gs_ref[0]
    for bad in (127 - 10, 0xFF):
        e2 = e.copy()
        e2[3, 1] = bad
        s = status_word()
        L.remap_mxfp4(to_dev(q), to_dev(e2), 1, rows, K, layout=0, dev_status=s)
        torch.cuda.synchronize()
        assert int(s.item()) == oracle.ERR_NOT_REPRESENTABLE
    # tiny exponents: subnormal global scale 2^g with g < -126
    e3 = np.full((rows, K // 32), 2, dtype=np.uint8)
    q3, sf3, gs3, st3 = oracle.remap_mxfp4(q, e3, 1, rows, K)
    p3 = L.remap_mxfp4(to_dev(q), to_dev(e3), 1, rows, K, layout=0)
    torch.cuda.synchronize()
    assert to_np(p3.gs)[0] == gs3[0] and np.array_equal(to_np(p3.sf).reshape(rows, K // 16), sf3)


# --------------------------------------------------------------------------- GEMM
def _packed_weights(w_bits, E, N, K):
    """Oracle-quantized weights [E*N, K], one global per expert, MMA-tiled scales."""
    offs = np.arange(0, (E + 1) * N, N, dtype=np.int32)
    q, sf, gs, st = oracle.quantize(w_bits, None, offs)
    assert st == 0
    return q, sf, gs


def _packed_acts(x_bits, row_index, offsets, E):
    q, sf, gs, st = oracle.quantize(x_bits, row_index, offsets)
    assert st == 0
    R, K2 = q.shape
    rows, starts = slot_rows(offsets)
    alloc = max(int(starts[-1]), 128)
    alloc = (alloc + 127) // 128 * 128
    qs = np.zeros((alloc, K2), np.uint8)
    ss = np.zeros((alloc, K2 // 8), np.uint8)
    qs[rows] = q
    ss[rows] = sf
    return q, sf, gs, qs, ss


def _run_gemm(qs, ss, gs_a, qw, sfw, gs_w, offsets, E, R, N, K, out_dtype):
    L = layer()
    nv = nvmod()
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qa = np.zeros((bound, K // 2), np.uint8)
    qa[:qs.shape[0]] = qs
    sa = np.zeros((((bound + 127) // 128) * 128, K // 16), np.uint8)
    sa[:ss.shape[0]] = ss
    a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(gs_a), R, K, 1,
                 to_dev(offsets) if offsets is not None else None, E)
    w = L.Packed(to_dev(qw), to_dev(tile(sfw)), to_dev(gs_w), qw.shape[0], K, 1)
    s = status_word()
    y = L.grouped_gemm(a, w, N, out_dtype, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    return to_np(y)


def test_gemm_closed_form_integer_case(gemm_kernel):
    """All scales 1.0 and s_g = 1: every product is a multiple of 1/4 and the
    fp32 sum is exact, so the tensor-core result must equal the oracle exactly."""
    rng = np.random.default_rng(0)
    M, N, K = 128, 256, 512
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qw = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sa = np.full((M, K // 16), 0x38, np.uint8)
    sw = np.full((N, K // 16), 0x38, np.uint8)
    one = np.ones(1, np.float32)
    y = _run_gemm(qa, sa, one, qw, sw, one, None, 1, M, N, K, 0)
    a = oracle.dequantize_f64(qa, sa, np.ones(M, np.float32))
    b = oracle.dequantize_f64(qw, sw, np.ones(N, np.float32))
    y_ref, _ = oracle.gemm_f64(a, b)
    assert np.array_equal(y.astype(np.float64), y_ref)


@pytest.mark.parametrize("out_dtype", [0, 1])
def test_gemm_dense_config1(out_dtype, gemm_kernel):
    M, N, K = 128, 256, 512
    x = synthetic.gaussian_bf16(0, synthetic.STREAMS["x"], (M, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(0, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    qx, sx, gx, st = oracle.quantize(x)
    qw, sw, gw = _packed_weights(w, 1, N, K)
    y = _run_gemm(qx, sx, gx, qw, sw, gw, None, 1, M, N, K, out_dtype)
    a = oracle.dequantize_f64(qx, sx, np.full(M, gx[0], np.float32))
    b = oracle.dequantize_f64(qw, sw, np.full(N, gw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    if out_dtype == 0:
        ok, err, bound = gemm_tol(y, y_ref, s_ref)
        assert ok.all(), (err.max(), (err / bound).max())
    else:
        y32 = _run_gemm(qx, sx, gx, qw, sw, gw, None, 1, M, N, K, 0)
        assert np.array_equal(y, synthetic.f32_to_bf16_bits(y32))


@pytest.mark.parametrize("mode", [0, 1, 3, 4], ids=["k512", "k256", "k512_deep", "two_blocks"])
def test_gemm_wait_timeout_reports_and_recovers(mode):
    """The failure path of the one-CTA GEMM without any GPU fault: with a
    1-cycle budget on its main-loop waits, the first wait that is not already
    complete gives up, the kernel writes NVFP4_ERR_TIMEOUT to the status word
    and ends (its closing waits for copies and MMAs in flight keep the full
    budget).  With the budget restored, the same context runs the same GEMM
    again and gets the result of a run made before the timeout, bit for bit.
    The two-block kernel takes bf16 outputs only, so its case writes bf16."""
    L = layer()
    nv = nvmod()
    E, N, K = 6, 256, 1024
    od = 1 if mode == 4 else 0
    counts = [0, 5, 130, 300, 16, 257]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(21, synthetic.STREAMS["x"], (R, K))
    w = synthetic.gaussian_bf16(21, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    nv.nvfp4_gemm_select_kernel(mode)
    try:
        y_before = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, od)
        bound = nv.nvfp4_padded_rows_bound(R, E)
        qa = np.zeros((bound, K // 2), np.uint8)
        qa[:qs.shape[0]] = qs
        sa = np.zeros((((bound + 127) // 128) * 128, K // 16), np.uint8)
        sa[:ss.shape[0]] = ss
        a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(gs), R, K, 1, to_dev(offsets), E)
        wp = L.Packed(to_dev(qw), to_dev(tile(sw)), to_dev(gw), qw.shape[0], K, 1)
        nv.nvfp4_gemm_set_wait_budget(1)
        s = status_word()
        L.grouped_gemm(a, wp, N, od, dev_status=s)
        torch.cuda.synchronize()
        assert int(s.item()) == nv.ERR_TIMEOUT
        nv.nvfp4_gemm_set_wait_budget(0)
        y_after = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, od)
    finally:
        nv.nvfp4_gemm_set_wait_budget(0)
        nv.nvfp4_gemm_select_kernel(0)
    assert np.array_equal(y_after, y_before)


@pytest.mark.parametrize("bad", ["decreasing", "end_past_rows", "end_short", "nonzero_start"])
def test_gemm_rejects_bad_offsets(gemm_kernel, bad):
    """Expert offsets that do not start at 0, decrease, or end elsewhere than
    at M_total: every CTA reports NVFP4_ERR_INDEX and runs no tile, so y keeps
    its sentinel.  The buffers are sized so that even a kernel that trusted
    the offsets would stay inside them (the slots of the largest offsets fit).
    fp32 and bf16 outputs (the two-block kernel writes bf16 only)."""
    L = layer()
    nv = nvmod()
    E, N, K, M = 3, 256, 1024, 300
    offsets = {"decreasing": [0, 200, 120, 300], "end_past_rows": [0, 100, 200, 380],
               "end_short": [0, 100, 200, 250], "nonzero_start": [7, 100, 200, 300]}[bad]
    offsets = np.array(offsets, np.int32)
    rows_alloc = 2048
    rng = np.random.default_rng(1)
    qa = rng.integers(0, 256, (rows_alloc, K // 2), dtype=np.uint8)
    sa = np.full((rows_alloc, K // 16), 0x38, np.uint8)
    qw = rng.integers(0, 256, (E * N, K // 2), dtype=np.uint8)
    sw = np.full((E * N, K // 16), 0x38, np.uint8)
    one = np.ones(E, np.float32)
    a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(one), M, K, 1, to_dev(offsets), E)
    w = L.Packed(to_dev(qw), to_dev(tile(sw)), to_dev(one), E * N, K, 1)
    for od, dt in ((0, torch.float32), (1, torch.bfloat16)):
        y = torch.full((rows_alloc, N), 12345.0, dtype=dt, device="cuda")
        s = status_word()
        L.grouped_gemm(a, w, N, od, y=y[:M], dev_status=s)
        torch.cuda.synchronize()
        assert int(s.item()) == nv.ERR_INDEX
        assert (y == 12345.0).all().item()


def test_quantize_rejects_bad_group_offsets():
    """The grouped quantize and the dispatch quantize check their group offsets
    the same way: NVFP4_ERR_INDEX and no packed byte written."""
    L = layer()
    nv = nvmod()
    T, K, E = 64, 256, 4
    x = synthetic.gaussian_bf16(3, synthetic.STREAMS["x"], (T, K))
    xd = bf16_dev(x)
    for offs in ([0, 10, 5, 64], [0, 10, 20, 60], [3, 10, 20, 64]):
        off = to_dev(np.array(offs, np.int32))
        q = torch.full((2048, K // 2), 0xAB, dtype=torch.uint8, device="cuda")
        sf = torch.full((2048 * K // 16,), 0xAB, dtype=torch.uint8, device="cuda")
        gs = torch.ones(E - 1, dtype=torch.float32, device="cuda")
        ws = L.workspace(E - 1)
        for layout in (0, 1):
            s = status_word()
            nv.nvfp4_quantize(xd, T, K, K, None, off, E - 1, nv.GS_GIVEN, gs, q, sf, layout, ws, s)
            torch.cuda.synchronize()
            assert int(s.item()) == nv.ERR_INDEX, (offs, layout)
            assert (to_np(q) == 0xAB).all() and (to_np(sf) == 0xAB).all()
    # the dispatch quantize: offsets past the routed rows of T tokens x top-1
    slot = to_dev(np.arange(T, dtype=np.int32).reshape(T, 1))
    off = to_dev(np.array([0, 30, 20, 64], np.int32))
    q = torch.full((2048, K // 2), 0xAB, dtype=torch.uint8, device="cuda")
    sf = torch.full((2048 * K // 16,), 0xAB, dtype=torch.uint8, device="cuda")
    gs = torch.ones(E - 1, dtype=torch.float32, device="cuda")
    s = status_word()
    nv.nvfp4_moe_quantize(xd, T, K, K, slot, 1, off, E - 1, nv.GS_GIVEN, gs, q, sf, 1, L.workspace(E - 1), s)
    torch.cuda.synchronize()
    assert int(s.item()) == nv.ERR_INDEX
    assert (to_np(q) == 0xAB).all() and (to_np(sf) == 0xAB).all()


def test_gemm_max_experts(gemm_kernel):
    """1024 experts, the most the GEMM's shared-memory tile tables hold: mostly
    empty groups, a few with 1-3 rows and one with 200 (two token chunks)."""
    rng = np.random.default_rng(23)
    E, N, K = 1024, 256, 512
    counts = np.where(rng.random(E) < 0.8, 0, rng.integers(1, 4, E))
    counts[517] = 200
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(23, synthetic.STREAMS["x"], (R, K))
    w = synthetic.gaussian_bf16(23, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    y = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    for e in np.nonzero(counts)[0]:
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        a = oracle.dequantize_f64(q[r0:r1], sf[r0:r1], np.full(r1 - r0, gs[e], np.float32))
        b = oracle.dequantize_f64(qw[e * N:(e + 1) * N], sw[e * N:(e + 1) * N], np.full(N, gw[e], np.float32))
        y_ref, s_ref = oracle.gemm_f64(a, b)
        ok, err, bound = gemm_tol(y[r0:r1], y_ref, s_ref)
        assert ok.all(), (int(e), err.max(), (err / bound).max())


def test_gemm_scale_bytes_over_the_whole_e4m3_range(gemm_kernel):
    """Random E2M1 codes with block-scale bytes drawn from every non-negative
    finite E4M3 value (0, the subnormals 2^-9 ... 7*2^-9, up to 448) on both
    operands, and globals far from 1: the tensor core's reading of each scale
    byte is checked against the fp64 oracle of the same packed operands."""
    rng = np.random.default_rng(24)
    E, N, K = 3, 256, 1024
    counts = [130, 7, 64]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    q = rng.integers(0, 256, (R, K // 2), dtype=np.uint8)
    sf = rng.integers(0, 0x7F, (R, K // 16), dtype=np.uint8)          # 0x00 .. 0x7E
    qw = rng.integers(0, 256, (E * N, K // 2), dtype=np.uint8)
    sw = rng.integers(0, 0x7F, (E * N, K // 16), dtype=np.uint8)
    sf[0, :8] = np.arange(8)                                           # zero and every subnormal
    sw[1, :8] = 0x7E                                                   # 448
    gs = np.array([2.0 ** -20, 3.5e-3, 1.25e2], dtype=np.float32)
    gw = np.array([7.0e-4, 2.0 ** 10, 1.0], dtype=np.float32)
    rows, starts = slot_rows(offsets)
    alloc = (max(int(starts[-1]), 128) + 127) // 128 * 128
    qs = np.zeros((alloc, K // 2), np.uint8)
    ss = np.zeros((alloc, K // 16), np.uint8)
    qs[rows] = q
    ss[rows] = sf
    y = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        a = oracle.dequantize_f64(q[r0:r1], sf[r0:r1], np.full(r1 - r0, gs[e], np.float32))
        b = oracle.dequantize_f64(qw[e * N:(e + 1) * N], sw[e * N:(e + 1) * N], np.full(N, gw[e], np.float32))
        y_ref, s_ref = oracle.gemm_f64(a, b)
        ok, err, bound = gemm_tol(y[r0:r1], y_ref, s_ref)
        assert ok.all(), (e, err.max(), (err / bound).max())


def test_gemm_k_not_multiple_of_512():
    """K = 1280 (a multiple of 256, not of 512): the automatic choice falls back
    to the 256-element-stage kernel; ragged groups, fp32 out, within the bound."""
    E, N, K = 3, 256, 1280
    counts = [77, 0, 190]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(22, synthetic.STREAMS["x"], (R, K))
    w = synthetic.gaussian_bf16(22, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    y = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    for e in range(E):
        r0, r1 = int(offsets[e]), int(offsets[e + 1])
        if r0 == r1:
            continue
        a = oracle.dequantize_f64(q[r0:r1], sf[r0:r1], np.full(r1 - r0, gs[e], np.float32))
        b = oracle.dequantize_f64(qw[e * N:(e + 1) * N], sw[e * N:(e + 1) * N], np.full(N, gw[e], np.float32))
        y_ref, s_ref = oracle.gemm_f64(a, b)
        ok, err, bound = gemm_tol(y[r0:r1], y_ref, s_ref)
        assert ok.all(), (e, err.max(), (err / bound).max())


def test_gemm_grouped_ragged(gemm_kernel):
    E, N, K = 6, 256, 512
    counts = [0, 5, 130, 300, 16, 257]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(5, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(5, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    y = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    a = oracle.dequantize_f64(q, sf, oracle.rows_global_scale(gs, offsets, R))
    bw = oracle.dequantize_f64(qw, sw, np.repeat(gw, N))
    y_ref, s_ref = oracle.grouped_gemm_f64(a, bw.reshape(E, N, K), offsets)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max(), np.argwhere(~ok)[:5])


@pytest.mark.parametrize("out_dtype", [0, 1])
def test_gemm_grouped_chunk_edges(out_dtype, gemm_kernel):
    """Expert sizes around every tile and chunk boundary (64-row chunk starts,
    one or two scale row blocks, the 192-token tile limit, token-tile halves of
    8..96 rows on a CTA pair)."""
    counts = [1, 63, 64, 65, 127, 128, 129, 191, 192, 193, 255, 256, 257, 383, 384, 385, 577, 0, 2, 17, 33]
    E, N, K = len(counts), 256, 256
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(12, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(12, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    y = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    a = oracle.dequantize_f64(q, sf, oracle.rows_global_scale(gs, offsets, R))
    bw = oracle.dequantize_f64(qw, sw, np.repeat(gw, N))
    y_ref, s_ref = oracle.grouped_gemm_f64(a, bw.reshape(E, N, K), offsets)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max(), np.argwhere(~ok)[:5])
    if out_dtype == 1:
        y16 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
        assert np.array_equal(y16, synthetic.f32_to_bf16_bits(y))


@pytest.mark.parametrize("N", [384, 512])
def test_gemm_dense_many_tiles(N, gemm_kernel):
    """Dense M = 1000 rows (6 token chunks, ragged last), K = 1024; N = 384 is
    not a multiple of the pair's 256 weight rows (one-CTA kernel only)."""
    if gemm_kernel == 2 and N % 256:
        pytest.skip("CTA pairs need N % 256 == 0")
    M, K = 1000, 1024
    x = synthetic.gaussian_bf16(13, synthetic.STREAMS["x"], (M, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(13, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    qx, sx, gx, _ = oracle.quantize(x)
    qw, sw, gw = _packed_weights(w, 1, N, K)
    y = _run_gemm(qx, sx, gx, qw, sw, gw, None, 1, M, N, K, 0)
    a = oracle.dequantize_f64(qx, sx, np.full(M, gx[0], np.float32))
    b = oracle.dequantize_f64(qw, sw, np.full(N, gw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max())


def test_gemm_long_k_tolerance(gemm_kernel):
    """K = 17408 (the dense MLP's down projection) on a thin slice."""
    M, N, K = 64, 256, 17408
    x = synthetic.gaussian_bf16(9, synthetic.STREAMS["x"], (M, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(9, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    qx, sx, gx, _ = oracle.quantize(x)
    qw, sw, gw = _packed_weights(w, 1, N, K)
    y = _run_gemm(qx, sx, gx, qw, sw, gw, None, 1, M, N, K, 0)
    a = oracle.dequantize_f64(qx, sx, np.full(M, gx[0], np.float32))
    b = oracle.dequantize_f64(qw, sw, np.full(N, gw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max())


def test_gemm_two_blocks_max_experts():
    """The two-block kernel at the 1024-expert limit of the GEMM tile tables:
    mostly empty groups, a few of 1-3 rows and one of 200 (two token chunks);
    bf16 Y bit for bit that of the one-CTA kernel with 256-element stages."""
    nv = nvmod()
    rng = np.random.default_rng(29)
    E, N, K = 1024, 256, 1024
    counts = np.where(rng.random(E) < 0.8, 0, rng.integers(1, 4, E))
    counts[700] = 200
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(29, synthetic.STREAMS["x"], (R, K))
    w = synthetic.gaussian_bf16(29, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    try:
        nv.nvfp4_gemm_select_kernel(4)
        y4 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
        nv.nvfp4_gemm_select_kernel(1)
        y1 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
    finally:
        nv.nvfp4_gemm_select_kernel(0)
    assert np.array_equal(y4, y1)


@pytest.mark.parametrize("swiglu", [False, True])
def test_gemm_two_blocks_small_groups(swiglu):
    """Decode-sized groups (at most 16 routed rows per expert on average) take
    the two-block kernel's 64-token tiles in four slots with two accumulator
    pairs: expert sizes around the 64-row chunk edges among many empty ones,
    bf16 Y (or SwiGLU h and its amax) bit for bit those of the one-CTA kernel
    with 256-element stages."""
    L = layer()
    nv = nvmod()
    counts = [1, 63, 64, 65, 127, 128, 129, 0, 2, 17, 191, 193] + [0] * 60 + [3, 5]
    E, N, K = len(counts), 512, 1024
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    assert R <= 16 * E
    x = synthetic.gaussian_bf16(37, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(37, synthetic.STREAMS["w_gate_up"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    if not swiglu:
        try:
            nv.nvfp4_gemm_select_kernel(4)
            y4 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
            nv.nvfp4_gemm_select_kernel(1)
            y1 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
        finally:
            nv.nvfp4_gemm_select_kernel(0)
        assert np.array_equal(y4, y1)
        return
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qa = np.zeros((bound, K // 2), np.uint8)
    qa[:qs.shape[0]] = qs
    sa = np.zeros((bound, K // 16), np.uint8)
    sa[:ss.shape[0]] = ss
    a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(gs), R, K, 1, to_dev(offsets), E)
    wp = L.Packed(to_dev(qw), to_dev(tile(sw)), to_dev(gw), E * N, K, 1)
    out = {}
    try:
        for mode in (4, 1):
            nv.nvfp4_gemm_select_kernel(mode)
            st = status_word()
            h, amax = L.grouped_gemm_swiglu(a, wp, N, dev_status=st)
            torch.cuda.synchronize()
            assert int(st.item()) == 0
            out[mode] = (to_np(h), to_np(amax))
    finally:
        nv.nvfp4_gemm_select_kernel(0)
    assert np.array_equal(out[4][0], out[1][0]) and np.array_equal(out[4][1], out[1][1])


def test_gemm_two_blocks_long_k_bf16():
    """The two-weight-block kernel on ragged groups with K = 4096 (16 turns of
    its three-slot ring per tile) and 4 weight-block pairs per expert: bf16 Y
    within the GEMM bound plus bf16 rounding of the oracle, and bit for bit the
    bf16 Y of the one-CTA kernel with 256-element stages (same MMAs in the same
    K order)."""
    nv = nvmod()
    E, N, K = 5, 1024, 4096
    counts = [1, 70, 0, 200, 385]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(31, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(31, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    try:
        nv.nvfp4_gemm_select_kernel(4)
        y16 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
        nv.nvfp4_gemm_select_kernel(1)
        y16_k256 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 1)
    finally:
        nv.nvfp4_gemm_select_kernel(0)
    assert np.array_equal(y16, y16_k256)
    a = oracle.dequantize_f64(q, sf, oracle.rows_global_scale(gs, offsets, R))
    bw = oracle.dequantize_f64(qw, sw, np.repeat(gw, N))
    y_ref, s_ref = oracle.grouped_gemm_f64(a, bw.reshape(E, N, K), offsets)
    y = synthetic.bf16_bits_to_f32(y16).astype(np.float64)
    err = np.abs(y - y_ref)
    bound = (1e-5 * s_ref + 1e-6) * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(y_ref)
    assert (err <= bound).all(), (err.max(), (err / bound).max())


# --------------------------------------------------------------------------- fused SwiGLU epilogue
def test_gemm_swiglu_epilogue(gemm_kernel):
    """h = bf16(silu(g)*u) from the gate_up accumulators: compared with the
    oracle SwiGLU of the same GEMM's fp32 output (one bf16 ulp), amax exact."""
    L = layer()
    nv = nvmod()
    E, I, K = 5, 256, 512
    N = 2 * I
    counts = [3, 0, 200, 70, 129]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(14, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(14, synthetic.STREAMS["w_gate_up"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    qw, sw, gw = _packed_weights(w, E, N, K)
    y32 = _run_gemm(qs, ss, gs, qw, sw, gw, offsets, E, R, N, K, 0)
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qa = np.zeros((bound, K // 2), np.uint8)
    qa[:qs.shape[0]] = qs
    sa = np.zeros((bound, K // 16), np.uint8)
    sa[:ss.shape[0]] = ss
    a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(gs), R, K, 1, to_dev(offsets), E)
    il = L.gate_up_interleave_index(E, I, "cpu").numpy()
    wp = L.Packed(to_dev(qw[il]), to_dev(tile(sw[il])), to_dev(gw), E * N, K, 1)
    st = status_word()
    h, amax = L.grouped_gemm_swiglu(a, wp, N, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    h_gpu = to_np(h)
    h_ref = oracle.swiglu(y32)
    d = np.abs(h_gpu.astype(np.int32) - h_ref.astype(np.int32))
    assert (d <= 1).all() and (d == 0).mean() > 0.99
    hf = np.abs(synthetic.bf16_bits_to_f32(h_gpu))
    want = np.array([hf[offsets[e]:offsets[e + 1]].max() if counts[e] else 0.0 for e in range(E)], np.float32)
    assert np.array_equal(to_np(amax), want)


def test_gemm_swiglu_nvfp4_epilogue(gemm_kernel):
    """The epilogue that quantizes h with a given global per expert writes the
    bytes the oracle's GIVEN-mode quantize writes for the device's bf16 h
    (taken from the SwiGLU epilogue of the same GEMM); padding rows untouched.
    One expert's global is tiny, so its block scales saturate at 448."""
    L = layer()
    E, I, K = 5, 256, 512
    N = 2 * I
    counts = [3, 0, 200, 70, 129]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    x = synthetic.gaussian_bf16(16, synthetic.STREAMS["x"], (R, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(16, synthetic.STREAMS["w_gate_up"], (E * N, K), sigma=0.02)
    q, sf, gs, qs, ss = _packed_acts(x, None, offsets, E)
    il = L.gate_up_interleave_index(E, I, "cpu").numpy()
    qw, sw, gw = _packed_weights(w[il], E, N, K)
    nv = nvmod()
    bound = nv.nvfp4_padded_rows_bound(R, E)
    qa = np.zeros((bound, K // 2), np.uint8)
    qa[:qs.shape[0]] = qs
    sa = np.zeros((bound, K // 16), np.uint8)
    sa[:ss.shape[0]] = ss
    a = L.Packed(to_dev(qa), to_dev(tile(sa)), to_dev(gs), R, K, 1, to_dev(offsets), E)
    wp = L.Packed(to_dev(qw), to_dev(tile(sw)), to_dev(gw), E * N, K, 1)
    h, amax = L.grouped_gemm_swiglu(a, wp, N)
    torch.cuda.synchronize()
    h_gs = (to_np(amax) / 2688.0 * 1.3).astype(np.float32)
    h_gs[h_gs == 0] = 1.0
    h_gs[4] = np.float32(to_np(amax)[4] / 2688.0 / 50.0)        # block scales clip at 448
    out = L.empty_packed(R, I, E, to_dev(offsets), 1)
    out.q.fill_(0xAB)
    out.sf.fill_(0xAB)
    st = status_word()
    p = L.grouped_gemm_swiglu_nvfp4(a, wp, N, to_dev(h_gs), out=out, dev_status=st)
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    q_ref, sf_ref, _, ost = oracle.quantize(to_np(h), None, offsets, global_scale=h_gs)
    assert ost == 0
    rows, starts = slot_rows(offsets)
    qd = to_np(p.q)
    assert np.array_equal(qd[rows], q_ref)
    sfm = untile(to_np(p.sf), qd.shape[0], I // 16)
    assert np.array_equal(sfm[rows], sf_ref)
    assert (sfm[rows[offsets[4]:]] == 0x7E).any()                  # saturated scales on expert 4
    pad = np.setdiff1d(np.arange(int(starts[-1])), rows)
    assert (qd[pad] == 0xAB).all() and (sfm[pad] == 0xAB).all()
    bad = h_gs.copy()
    bad[2] = 0.0
    st2 = status_word()
    L.grouped_gemm_swiglu_nvfp4(a, wp, N, to_dev(bad), dev_status=st2)
    torch.cuda.synchronize()
    assert int(st2.item()) == 1


def test_moe_layer_fused_swiglu_stagewise():
    L = layer()
    T, H, I, E, k = 96, 256, 256, 8, 3
    x = synthetic.gaussian_bf16(15, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(15, T, E, k)
    off = r["offsets"]
    R = len(r["row_index"])
    wgu = synthetic.gaussian_bf16(15, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wd = synthetic.gaussian_bf16(15, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    il = L.gate_up_interleave_index(E, I, "cpu").numpy()
    qg, sg, gg = _packed_weights(wgu[il], E, 2 * I, H)
    qd, sd, gd = _packed_weights(wd, E, H, I)
    Wgu = L.Packed(to_dev(qg), to_dev(tile(sg)), to_dev(gg), E * 2 * I, H, 1)
    Wd = L.Packed(to_dev(qd), to_dev(tile(sd)), to_dev(gd), E * H, I, 1)
    moe = L.MoEExperts(Wgu, Wd, E, H, I, max_rows=R, out_dtype=0, mid_dtype=0, fused_swiglu=True)
    s = status_word()
    y2 = moe.forward(bf16_dev(x), to_dev(r["row_index"]), to_dev(off), dev_status=s,
                     slot=to_dev(r["slot"].astype(np.int32)))
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    rows, _ = slot_rows(off)
    q1_ref, _, gs1_ref, _ = oracle.quantize(x, r["row_index"], off)     # stage 1 (token-order quantize)
    assert np.array_equal(to_np(moe.a1.gs), gs1_ref) and np.array_equal(to_np(moe.a1.q)[rows], q1_ref)
    h = to_np(moe.h[:R])
    # stage 1+2: h against silu(g)*u of the fp64 gate_up GEMM on the oracle's
    # quantized operands (gate/up rows put back in source order).  Bound: the
    # GEMM tolerance on g and u carried through h (|dh/dg| <= 1.1|u|,
    # |dh/du| = |silu g|) plus one bf16 rounding on each side.
    q1, sf1, gs1, _ = oracle.quantize(x, r["row_index"], off)
    a1 = oracle.dequantize_f64(q1, sf1, oracle.rows_global_scale(gs1, off, R))
    b_il = oracle.dequantize_f64(qg, sg, np.repeat(gg, 2 * I))
    b1 = np.empty_like(b_il)
    b1[il] = b_il
    y1, s1 = oracle.grouped_gemm_f64(a1, b1.reshape(E, 2 * I, H), off)
    g, u, sg1, su1 = y1[:, :I], y1[:, I:], s1[:, :I], s1[:, I:]
    silu = g / (1.0 + np.exp(-g))
    h64 = silu * u
    tol = 1.1 * np.abs(u) * (1e-5 * sg1 + 1e-6) + np.abs(silu) * (1e-5 * su1 + 1e-6) + 2.0 ** -7 * np.abs(h64) + 1e-30
    hf = synthetic.bf16_bits_to_f32(h).astype(np.float64)
    assert (np.abs(hf - h64) <= tol).all(), (np.abs(hf - h64) / tol).max()
    q2, sf2, gs2, _ = oracle.quantize(h, None, off)          # requantize of the device's h: bit-exact
    assert np.array_equal(to_np(moe.a2.gs), gs2)
    assert np.array_equal(to_np(moe.a2.q)[rows], q2)
    a2 = oracle.dequantize_f64(q2, sf2, oracle.rows_global_scale(gs2, off, R))
    bd = oracle.dequantize_f64(qd, sd, np.repeat(gd, H)).reshape(E, H, I)
    y2_ref, s2_ref = oracle.grouped_gemm_f64(a2, bd, off)
    ok, err, bound = gemm_tol(to_np(y2), y2_ref, s2_ref)
    assert ok.all(), (err / bound).max()


def test_moe_layer_given_down_input_scale():
    """MoEExperts with a calibrated down-input global: the packed h equals the
    oracle's GIVEN-mode quantize of the dynamic path's h, and the down GEMM
    meets the tolerance on it."""
    L = layer()
    T, H, I, E, k = 96, 256, 256, 8, 3
    x = synthetic.gaussian_bf16(17, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(17, T, E, k)
    off = r["offsets"]
    R = len(r["row_index"])
    wgu = synthetic.gaussian_bf16(17, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wd = synthetic.gaussian_bf16(17, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    il = L.gate_up_interleave_index(E, I, "cpu").numpy()
    qg, sg, gg = _packed_weights(wgu[il], E, 2 * I, H)
    qd, sd, gd = _packed_weights(wd, E, H, I)
    Wgu = L.Packed(to_dev(qg), to_dev(tile(sg)), to_dev(gg), E * 2 * I, H, 1)
    Wd = L.Packed(to_dev(qd), to_dev(tile(sd)), to_dev(gd), E * H, I, 1)
    moe = L.MoEExperts(Wgu, Wd, E, H, I, max_rows=R, out_dtype=0, mid_dtype=0, fused_swiglu=True)
    xd, rid, offd, sld = bf16_dev(x), to_dev(r["row_index"]), to_dev(off), to_dev(r["slot"].astype(np.int32))
    # a dynamic forward first: its requantize leaves s_g of each expert's max |h| in moe.amax
    moe.forward(xd, rid, offd, slot=sld)
    gs_dyn = to_np(moe.amax).copy()
    h_dyn = to_np(moe.h[:R]).copy()
    # margin 1: the calibrated global is the dynamic one, bit for bit
    gs_1 = to_np(L.calibrate_h_scale(moe, xd, rid, offd, slot=sld, margin=1.0))
    assert np.array_equal(gs_1.view(np.uint32), gs_dyn.view(np.uint32))
    gs_h = to_np(L.calibrate_h_scale(moe, xd, rid, offd, slot=sld, margin=1.25))
    assert np.array_equal(to_np(moe.h[:R]), h_dyn)
    hf = synthetic.bf16_bits_to_f32(h_dyn)
    for e in range(E):
        a = float(np.abs(hf[off[e]:off[e + 1]]).max()) if off[e + 1] > off[e] else 0.0
        assert gs_1[e] == np.float32(oracle.global_scale_from_amax(a))
        assert gs_h[e] == np.float32(oracle.global_scale_from_amax(float(np.float32(a) * np.float32(1.25))))
    s = status_word()
    y2 = moe.forward(xd, rid, offd, dev_status=s, slot=sld)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    rows, _ = slot_rows(off)
    q2, sf2, _, st = oracle.quantize(h_dyn, None, off, global_scale=gs_h)
    assert st == 0
    assert np.array_equal(to_np(moe.a2.q)[rows], q2)
    # with 25 % headroom no block scale of h saturates
    assert (sf2 < 0x7E).all() and (sf2.max() >> 3) >= 14
    a2 = oracle.dequantize_f64(q2, sf2, oracle.rows_global_scale(gs_h, off, R))
    bd = oracle.dequantize_f64(qd, sd, np.repeat(gd, H)).reshape(E, H, I)
    y2_ref, s2_ref = oracle.grouped_gemm_f64(a2, bd, off)
    ok, err, bound = gemm_tol(to_np(y2), y2_ref, s2_ref)
    assert ok.all(), (err / bound).max()


def test_global_scale_from_amax_entry_point():
    """The global-scale rule as its own call equals the oracle's rule on amaxes
    over the whole fp32 range, with and without a margin; zero gives 1, a
    non-finite amax gives NaN and NVFP4_ERR_NONFINITE; negative amaxes count by
    magnitude; in place works."""
    nv = nvmod()
    rng = np.random.default_rng(9)
    vals = np.concatenate([
        [0.0, -0.0, 1.0, 2688.0, 448.0, 6.0, 3.0e38, 1e-45, 1.17549435e-38, -7.5],
        np.exp2(rng.uniform(-140, 127, 4000)),
        rng.standard_normal(1000) * 100,
    ]).astype(np.float32)
    for margin in (1.0, 1.25, 0.75):
        a = to_dev(vals)
        out = torch.empty_like(a)
        s = status_word()
        nv.nvfp4_global_scale_from_amax(a, vals.size, margin, out, s)
        torch.cuda.synchronize()
        got = to_np(out)
        m = np.float32(margin)
        want = np.array([oracle.global_scale_from_amax(float(abs(v) if margin == 1.0 else np.float32(abs(v)) * m))
                         for v in vals], np.float32)
        fin = np.isfinite(want)
        assert np.array_equal(got[fin].view(np.uint32), want[fin].view(np.uint32))
        assert np.isnan(got[~fin]).all()
        assert int(s.item()) == (16 if (~fin).any() else 0)
    bad = to_dev(np.array([1.0, np.inf, np.nan, 5.0], np.float32))
    s = status_word()
    nv.nvfp4_global_scale_from_amax(bad, 4, 1.0, bad, s)        # in place
    torch.cuda.synchronize()
    g = to_np(bad)
    assert int(s.item()) == 16 and np.isnan(g[1]) and np.isnan(g[2])
    assert g[0] == np.float32(1.0) / np.float32(2688.0) and g[3] == np.float32(5.0) / np.float32(2688.0)
    for margin in (0.0, -1.0, float("inf"), float("nan")):
        assert nv.nvfp4_global_scale_from_amax(bad, 4, margin, bad, None, check=False) == nv.ERR_INVALID_ARG


# --------------------------------------------------------------------------- SwiGLU + requantize
@pytest.mark.parametrize("ydt", [0, 1])
def test_swiglu_requantize(ydt):
    L = layer()
    E, I = 5, 256
    counts = [3, 0, 140, 17, 40]
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R = int(offsets[-1])
    yb = synthetic.gaussian_bf16(11, synthetic.STREAMS["x"], (R, 2 * I))
    yf = synthetic.bf16_bits_to_f32(yb) * np.float32(3.0)
    yd = to_dev(yf) if ydt == 0 else bf16_dev(synthetic.f32_to_bf16_bits(yf))
    yin = yf if ydt == 0 else synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(yf))
    p, h = L.swiglu_quantize(yd, to_dev(offsets), E, layout=1)
    torch.cuda.synchronize()
    h_gpu = to_np(h)
    h_ref = oracle.swiglu(yin)
    # h: within one bf16 ulp of the fp64 reference (device expf vs host exp)
    d = np.abs(h_gpu.astype(np.int32) - h_ref.astype(np.int32))
    assert (d <= 1).all() and (d == 0).mean() > 0.99
    # requantize of the GPU's h is bit-exact with the oracle's quantizer
    q_ref, sf_ref, gs_ref, st = oracle.quantize(h_gpu, None, offsets)
    assert np.array_equal(to_np(p.gs), gs_ref)
    rows, _ = slot_rows(offsets)
    assert np.array_equal(to_np(p.q)[rows], q_ref)
    assert np.array_equal(untile(to_np(p.sf), p.q.shape[0] // 128 * 128, I // 16)[rows], sf_ref)


# --------------------------------------------------------------------------- KV cache
@pytest.mark.parametrize("mode", [0, 1])
def test_kv_quantize_dequantize(mode):
    nv = nvmod()
    L = layer()
    T, Hh, D = 64, 4, 256
    k = synthetic.gaussian_bf16(0, synthetic.STREAMS["kv_k"], (T * Hh, D))
    v = synthetic.gaussian_bf16(0, synthetic.STREAMS["kv_v"], (T * Hh, D))
    if mode == 1:
        kg, vg = np.array([0.002], np.float32), np.array([0.0017], np.float32)
        rk = oracle.quantize(k, global_scale=kg)
        rv = oracle.quantize(v, global_scale=vg)
    else:
        rk, rv = oracle.quantize(k), oracle.quantize(v)
    kd, vd = bf16_dev(k), bf16_dev(v)
    kq = torch.empty((T * Hh, D // 2), dtype=torch.uint8, device="cuda")
    vq = torch.empty_like(kq)
    ks = torch.empty(T * Hh * D // 16, dtype=torch.uint8, device="cuda")
    vs = torch.empty_like(ks)
    kgs = to_dev(rk[2]) if mode == 1 else torch.empty(1, device="cuda")
    vgs = to_dev(rv[2]) if mode == 1 else torch.empty(1, device="cuda")
    s = status_word()
    nv.nvfp4_kv_quantize(kd, vd, T, Hh, D, mode, kgs, vgs, kq, ks, vq, vs, L.workspace(2), s)
    ko = torch.empty((T * Hh, D), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    nv.nvfp4_kv_dequantize(kq, ks, kgs, vq, vs, vgs, T, Hh, D, ko, vo)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    for (qr, sr, gr, _), qg, sg, gg, og in ((rk, kq, ks, kgs, ko), (rv, vq, vs, vgs, vo)):
        assert to_np(gg)[0] == gr[0]
        assert np.array_equal(to_np(qg), qr)
        assert np.array_equal(to_np(sg).reshape(-1, D // 16), sr)
        ref = oracle.dequantize(qr, sr, np.full(T * Hh, gr[0], np.float32), out="bf16")
        assert np.array_equal(to_np(og), ref)


# --------------------------------------------------------------------------- MoE layer
def test_moe_layer_small_stagewise():
    """gather-quantize -> gate_up -> SwiGLU+requant -> down, each stage against the oracle."""
    L = layer()
    T, H, I, E, k = 96, 256, 256, 8, 3
    x = synthetic.gaussian_bf16(2, synthetic.STREAMS["x"], (T, H))
    r = synthetic.route_topk_softmax(2, T, E, k)
    off = r["offsets"]
    R = len(r["row_index"])
    wgu = synthetic.gaussian_bf16(2, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wd = synthetic.gaussian_bf16(2, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    qg, sg, gg = _packed_weights(wgu, E, 2 * I, H)
    qd, sd, gd = _packed_weights(wd, E, H, I)
    Wgu = L.Packed(to_dev(qg), to_dev(tile(sg)), to_dev(gg), E * 2 * I, H, 1)
    Wd = L.Packed(to_dev(qd), to_dev(tile(sd)), to_dev(gd), E * H, I, 1)
    moe = L.MoEExperts(Wgu, Wd, E, H, I, max_rows=R, out_dtype=0, mid_dtype=0)
    s = status_word()
    y2 = moe.forward(bf16_dev(x), to_dev(r["row_index"]), to_dev(off), dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    # stage 1: gather-quantize
    q1, sf1, gs1, _ = oracle.quantize(x, r["row_index"], off)
    rows, _ = slot_rows(off)
    assert np.array_equal(to_np(moe.a1.q)[rows], q1)
    # stage 2: gate_up GEMM (fp32) against the fp64 oracle on the same operands
    a1 = oracle.dequantize_f64(q1, sf1, oracle.rows_global_scale(gs1, off, R))
    bgu = oracle.dequantize_f64(qg, sg, np.repeat(gg, 2 * I)).reshape(E, 2 * I, H)
    y1_ref, s1_ref = oracle.grouped_gemm_f64(a1, bgu, off)
    y1 = to_np(moe.y1[:R])
    ok, err, bound = gemm_tol(y1, y1_ref, s1_ref)
    assert ok.all(), (err / bound).max()
    # stage 3: SwiGLU of the GPU's y1, requantized
    h = to_np(moe.h[:R])
    d = np.abs(h.astype(np.int32) - oracle.swiglu(y1).astype(np.int32))
    assert (d <= 1).all()
    q2, sf2, gs2, _ = oracle.quantize(h, None, off)
    assert np.array_equal(to_np(moe.a2.q)[rows], q2)
    # stage 4: down GEMM on the GPU's quantized h
    a2 = oracle.dequantize_f64(q2, sf2, oracle.rows_global_scale(gs2, off, R))
    bd = oracle.dequantize_f64(qd, sd, np.repeat(gd, H)).reshape(E, H, I)
    y2_ref, s2_ref = oracle.grouped_gemm_f64(a2, bd, off)
    ok, err, bound = gemm_tol(to_np(y2), y2_ref, s2_ref)
    assert ok.all(), (err / bound).max()


# --------------------------------------------------------------------------- routing / combine
@pytest.mark.parametrize("T,E,k", [(1000, 64, 8), (8192, 512, 10), (3, 2048, 2), (257, 5, 5)])
def test_route_bitexact(T, E, k):
    L = layer()
    if (T, E, k) == (8192, 512, 10):
        ids = synthetic.route_topk_softmax(0, T, E, k)["experts"].astype(np.int32)
    else:
        rng = np.random.default_rng(T)
        ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off_ref, ri_ref, slot_ref, st = oracle.route(ids, E)
    s = status_word()
    off, ri, slot = L.route(to_dev(ids), E, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    assert np.array_equal(to_np(off), off_ref)
    assert np.array_equal(to_np(ri), ri_ref)
    assert np.array_equal(to_np(slot), slot_ref)


@pytest.mark.parametrize("T,E,k,nbad", [(3, 4, 2, 1), (1000, 64, 8, 300), (600, 2048, 3, 17), (5, 7, 2, 10)])
def test_route_bad_index_status(T, E, k, nbad):
    """Out-of-range expert ids: the device drops those choices exactly as the
    oracle's routing does (slot -1, not counted, no routed row), reports
    NVFP4_ERR_INDEX, and every other output equals the oracle's in full."""
    L = layer()
    rng = np.random.default_rng(T + nbad)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    flat = ids.reshape(-1)
    pos = rng.choice(T * k, size=nbad, replace=False)
    flat[pos] = np.where(rng.random(nbad) < 0.5, E + rng.integers(0, 1 << 20, nbad), -1 - rng.integers(0, 1 << 20, nbad))
    off_ref, ri_ref, slot_ref, st = oracle.route(ids, E)
    assert st == 1
    s = status_word()
    off, ri, slot = L.route(to_dev(ids), E, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 19
    assert np.array_equal(to_np(off), off_ref)
    assert np.array_equal(to_np(ri)[:int(off_ref[-1])], ri_ref)
    assert np.array_equal(to_np(slot), slot_ref)


@pytest.mark.parametrize("ydt", [0, 1])
def test_combine(ydt):
    L = layer()
    T, E, k, H = 300, 16, 4, 512
    rng = np.random.default_rng(5)
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, ri, slot, _ = oracle.route(ids, E)
    w = rng.random((T, k)).astype(np.float32)
    w /= w.sum(1, keepdims=True)
    yb = synthetic.gaussian_bf16(5, synthetic.STREAMS["x"], (T * k, H))
    yf = synthetic.bf16_bits_to_f32(yb)
    yd = bf16_dev(yb) if ydt == 1 else to_dev(yf)
    out32 = to_np(L.combine(yd, to_dev(slot), to_dev(w), out_dtype=0))
    out16 = to_np(L.combine(yd, to_dev(slot), to_dev(w), out_dtype=1))
    torch.cuda.synchronize()
    ref, sabs = oracle.combine(yf, slot, w)
    assert (np.abs(out32 - ref) <= 1e-6 * sabs + 1e-30).all()
    assert np.array_equal(out16, synthetic.f32_to_bf16_bits(out32))


def test_combine_out_of_range_slot():
    """A slot past y's rows is skipped (never read) and reported; -1 is skipped silently."""
    L = layer()
    T, k, H = 5, 2, 64
    yb = synthetic.gaussian_bf16(6, synthetic.STREAMS["x"], (8, H))
    yf = synthetic.bf16_bits_to_f32(yb)
    slot = np.array([[0, 1], [2, -1], [3, 4], [5, 8], [6, 7]], dtype=np.int32)
    w = np.full((T, k), 0.5, np.float32)
    s = status_word()
    out = to_np(L.combine(to_dev(yf), to_dev(slot), to_dev(w), out_dtype=0, dev_status=s))
    torch.cuda.synchronize()
    assert int(s.item()) == 19
    ok = slot.copy()
    ok[3, 1] = -1
    ref, sabs = oracle.combine(yf, ok, w)
    assert (np.abs(out - ref) <= 1e-6 * sabs + 1e-30).all()


def test_moe_layer_full_small():
    """route -> experts -> combine; the combine stage checked on the device's y."""
    L = layer()
    T, H, I, E, k = 64, 256, 256, 8, 3
    r = synthetic.route_topk_softmax(6, T, E, k)
    x = synthetic.gaussian_bf16(6, synthetic.STREAMS["x"], (T, H))
    wgu = synthetic.gaussian_bf16(6, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wd = synthetic.gaussian_bf16(6, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    qg, sg, gg = _packed_weights(wgu, E, 2 * I, H)
    qd, sd, gd = _packed_weights(wd, E, H, I)
    Wgu = L.Packed(to_dev(qg), to_dev(tile(sg)), to_dev(gg), E * 2 * I, H, 1)
    Wd = L.Packed(to_dev(qd), to_dev(tile(sd)), to_dev(gd), E * H, I, 1)
    experts = L.MoEExperts(Wgu, Wd, E, H, I, max_rows=T * k, out_dtype=1, mid_dtype=1)
    moe = L.MoELayer(experts, T, k)
    s = status_word()
    out = moe.forward(bf16_dev(x), to_dev(r["experts"].astype(np.int32)),
                      to_dev(r["weights"].astype(np.float32)), dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    off_ref, ri_ref, slot_ref, _ = oracle.route(r["experts"].astype(np.int32), E)
    assert np.array_equal(to_np(moe.ri[:T * k]), ri_ref) and np.array_equal(to_np(moe.off), off_ref)
    y2 = synthetic.bf16_bits_to_f32(to_np(experts.y2[:T * k]))
    ref, sabs = oracle.combine(y2, slot_ref, r["weights"].astype(np.float32))
    got = synthetic.bf16_bits_to_f32(to_np(out)).astype(np.float64)
    # bf16 output: within one bf16 rounding of the fp32 result
    assert (np.abs(got - ref) <= 1e-6 * sabs + np.abs(ref) * 2.0 ** -8 + 1e-30).all()


@pytest.mark.parametrize("H,I,fused", [(256, 256, False), (512, 1024, True)])
def test_moe_layer_graph_replay(H, I, fused):
    """The whole block captured as a CUDA graph: a replay gives the eager
    forward's output bit for bit.  After new inputs are copied into the same
    tensors (new tokens, new routing, new weights), a replay matches an eager
    forward on them.  K = 256 takes the 256-element-stage GEMM, K = 512 and
    1024 the 512-element one."""
    L = layer()
    T, E, k = 96, 8, 3
    wgu = synthetic.gaussian_bf16(8, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wd = synthetic.gaussian_bf16(8, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    il = L.gate_up_interleave_index(E, I, "cpu").numpy() if fused else np.arange(E * 2 * I)
    qg, sg, gg = _packed_weights(wgu, E, 2 * I, H)
    qd, sd, gd = _packed_weights(wd, E, H, I)
    Wgu = L.Packed(to_dev(qg[il]), to_dev(tile(sg[il])), to_dev(gg), E * 2 * I, H, 1)
    Wd = L.Packed(to_dev(qd), to_dev(tile(sd)), to_dev(gd), E * H, I, 1)
    experts = L.MoEExperts(Wgu, Wd, E, H, I, max_rows=T * k, out_dtype=1, mid_dtype=1, fused_swiglu=fused)
    moe = L.MoELayer(experts, T, k)

    def inputs(seed):
        r = synthetic.route_topk_softmax(seed, T, E, k)
        return (synthetic.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, H)), r["experts"].astype(np.int32),
                r["weights"].astype(np.float32))
    xb, ids, wts = inputs(9)
    x, idd, wd_ = bf16_dev(xb), to_dev(ids), to_dev(wts)
    eager = moe.forward(x, idd, wd_).clone()
    graph, out = moe.capture(x, idd, wd_)
    out.zero_()
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out, eager)
    xb2, ids2, wts2 = inputs(10)
    x.copy_(bf16_dev(xb2))
    idd.copy_(to_dev(ids2))
    wd_.copy_(to_dev(wts2))
    graph.replay()
    torch.cuda.synchronize()
    replayed = out.clone()
    eager2 = moe.forward(bf16_dev(xb2), to_dev(ids2), to_dev(wts2))
    torch.cuda.synchronize()
    assert torch.equal(replayed, eager2)
    assert not torch.equal(replayed, eager)


def test_device_generator_matches_host():
    import synthetic.cuda as sc
    g = sc.gaussian_bf16(3, 5, (1000, 64), sigma=0.02, start=12345)
    h = synthetic.gaussian_bf16(3, 5, (1000, 64), sigma=0.02, start=12345)
    assert np.array_equal(to_np(g), h)
    g = sc.gaussian_bf16(3, 5, (777,))
    assert np.array_equal(to_np(g), synthetic.gaussian_bf16(3, 5, (777,)))
    c = sc.mxfp4_codes(1, 9, 4096, start_byte=64)
    assert np.array_equal(to_np(c), synthetic.mxfp4_codes(1, 9, 4096, start_byte=64))
    e = sc.mxfp4_exponents(1, 10, 999, lo=-10, start=7)
    assert np.array_equal(to_np(e), synthetic.mxfp4_exponents(1, 10, 999, lo=-10, start=7))


# --------------------------------------------------------------------------- W4A16 grouped GEMM
@pytest.fixture(params=[1, 2], ids=["warp_mma", "tcgen05"], autouse=False)
def w4a16_kernel(request):
    """Run a W4A16 test on both kernels: the warp-MMA one (small groups) and the
    tcgen05 one (weights as the A operand in tensor memory)."""
    nv = nvmod()
    nv.nvfp4_w4a16_select_kernel(request.param)
    yield request.param
    nv.nvfp4_w4a16_select_kernel(0)


def _w4a16_case(seed, counts, N, K, T):
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R, E = int(offsets[-1]), len(counts)
    rng = np.random.default_rng(seed)
    ri = rng.integers(0, T, R).astype(np.int32)                 # gathered token rows
    x = synthetic.gaussian_bf16(seed, synthetic.STREAMS["x"], (T, K), outlier_frac=0.001)
    w = synthetic.gaussian_bf16(seed, synthetic.STREAMS["w"], (E * N, K), sigma=0.02)
    qw, sw, gw = _packed_weights(w, E, N, K)
    a = synthetic.bf16_bits_to_f32(x[ri]).astype(np.float64)
    bw = oracle.dequantize_f64(qw, sw, np.repeat(gw, N)).reshape(E, N, K)
    y_ref, s_ref = oracle.grouped_gemm_f64(a, bw, offsets)
    L = layer()
    wp = L.Packed(to_dev(qw), to_dev(sw), to_dev(gw), E * N, K, 0)
    return L, x, ri, offsets, wp, y_ref, s_ref


@pytest.mark.parametrize("K", [1024, 1280])
def test_w4a16_grouped(K, w4a16_kernel):
    """bf16 activations x NVFP4 weights per expert vs fp64 on the exact
    dequantized weights: groups of 0, 1, 3, 9, 17, 64, 65 and 200 tokens
    (several 16-token chunks for the warp-MMA kernel, several 64-token items
    and partial 16-row groups for the tcgen05 one), K an even and an odd
    number of 256-element stages."""
    counts = [0, 1, 3, 9, 17, 64, 65, 200]
    N, T = 256, 40
    L, x, ri, off, wp, y_ref, s_ref = _w4a16_case(30, counts, N, K, T)
    s = status_word()
    y = L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(ri), to_dev(off), len(counts), out_dtype=0, dev_status=s)
    y16 = L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(ri), to_dev(off), len(counts), out_dtype=1)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    ok, err, bound = gemm_tol(to_np(y), y_ref, s_ref)
    assert ok.all(), (err / bound).max()
    assert np.array_equal(to_np(y16), synthetic.f32_to_bf16_bits(to_np(y)))


def test_w4a16_scale_bytes_over_the_whole_e4m3_range(w4a16_kernel):
    """Weights with random codes and block-scale bytes over every non-negative
    finite E4M3 value (zero, the subnormals, up to 448) and globals far from 1:
    the kernel's f16 code x scale products must be exact over the whole range
    (within the fp64 oracle's bound after accumulation)."""
    L = layer()
    rng = np.random.default_rng(33)
    counts = [5, 12, 0, 30]
    N, K, T = 256, 1024, 24
    offsets = np.concatenate([[0], np.cumsum(counts)]).astype(np.int32)
    R, E = int(offsets[-1]), len(counts)
    ri = rng.integers(0, T, R).astype(np.int32)
    x = synthetic.gaussian_bf16(33, synthetic.STREAMS["x"], (T, K))
    qw = rng.integers(0, 256, (E * N, K // 2), dtype=np.uint8)
    sw = rng.integers(0, 0x7F, (E * N, K // 16), dtype=np.uint8)
    sw[0, :8] = np.arange(8)
    sw[1, :8] = 0x7E
    gw = np.array([2.0 ** -20, 3.0e-3, 1.0, 2.0 ** 9], dtype=np.float32)
    a = synthetic.bf16_bits_to_f32(x[ri]).astype(np.float64)
    bw = oracle.dequantize_f64(qw, sw, np.repeat(gw, N)).reshape(E, N, K)
    y_ref, s_ref = oracle.grouped_gemm_f64(a, bw, offsets)
    wp = L.Packed(to_dev(qw), to_dev(sw), to_dev(gw), E * N, K, 0)
    s = status_word()
    y = L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(ri), to_dev(offsets), E, out_dtype=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    ok, err, bound = gemm_tol(to_np(y), y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max())


def test_w4a16_swiglu_epilogue(w4a16_kernel):
    """h = bf16(silu(g) * u) from the same g, u as the plain kernel's fp32
    output (each output element sums its K terms in the same order in both
    variants): within one bf16 ulp of the oracle SwiGLU of that output."""
    counts = [2, 0, 5, 11]
    I, K, T = 128, 2048, 20
    N = 2 * I
    L, x, ri, off, wp, y_ref, s_ref = _w4a16_case(31, counts, N, K, T)
    y32 = L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(ri), to_dev(off), len(counts), out_dtype=0)
    h = L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(ri), to_dev(off), len(counts), out_dtype=1, swiglu=True)
    torch.cuda.synchronize()
    ok, err, bound = gemm_tol(to_np(y32), y_ref, s_ref)
    assert ok.all()
    d = np.abs(to_np(h).astype(np.int32) - oracle.swiglu(to_np(y32)).astype(np.int32))
    assert (d <= 1).all() and (d == 0).mean() > 0.99


def test_w4a16_dense_and_bad_row_index(w4a16_kernel):
    L = layer()
    M, N, K = 5, 128, 4096
    x = synthetic.gaussian_bf16(32, synthetic.STREAMS["x"], (M, K))
    w = synthetic.gaussian_bf16(32, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    qw, sw, gw = _packed_weights(w, 1, N, K)
    wp = L.Packed(to_dev(qw), to_dev(sw), to_dev(gw), N, K, 0)
    y = to_np(L.grouped_gemm_w4a16(bf16_dev(x), wp, N, out_dtype=0))
    a = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    b = oracle.dequantize_f64(qw, sw, np.full(N, gw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all()
    s = status_word()
    bad = np.array([0, 1, 7, 2], dtype=np.int32)                 # 7 is past the 5 rows of x
    L.grouped_gemm_w4a16(bf16_dev(x), wp, N, to_dev(bad), out_dtype=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 19


def test_w4a16_activation_range(w4a16_kernel):
    """Rows whose magnitudes sit far from 1 (1e30, 1e-30) and a row spanning
    about 2^40 of dynamic range: the per-row power-of-two scaling into f16
    keeps every row within the GEMM tolerance; a row holding an inf is
    reported as non-finite."""
    L = layer()
    M, N, K = 6, 128, 1024
    z = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(33, synthetic.STREAMS["x"], (M, K))).astype(np.float64)
    z[0] *= 1e30
    z[1] *= 1e-30
    z[2] *= np.ldexp(1.0, (np.arange(K) % 41) - 20)             # 2^-20 .. 2^20 across the row
    z[3, ::7] = 0.0
    x = synthetic.f32_to_bf16_bits(z.astype(np.float32))
    w = synthetic.gaussian_bf16(33, synthetic.STREAMS["w"], (N, K), sigma=0.02)
    qw, sw, gw = _packed_weights(w, 1, N, K)
    wp = L.Packed(to_dev(qw), to_dev(sw), to_dev(gw), N, K, 0)
    s = status_word()
    y = to_np(L.grouped_gemm_w4a16(bf16_dev(x), wp, N, out_dtype=0, dev_status=s))
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    a = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    b = oracle.dequantize_f64(qw, sw, np.full(N, gw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    ok, err, bound = gemm_tol(y, y_ref, s_ref)
    assert ok.all(), (err / bound).max()
    x[4, 17] = 0x7F80                                            # +inf
    s = status_word()
    L.grouped_gemm_w4a16(bf16_dev(x), wp, N, out_dtype=0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 16
