"""Parity at the benchmark configurations' full sizes (GPU, through the C ABI).

The GPU runs each configuration whole, in the launch configuration the bench
times; the oracle then checks all of it:
- GEMMs: every output element (expert by expert, or in column chunks for the
  dense MLP), in fp64 on the oracle's own quantization of the same seeded
  inputs, within |y - y_ref| <= 1e-5 * sum|a*b| + 1e-6;
- quantize, KV cache, remap: every byte.

All oracle inputs are regenerated on the host from the seeded generators
(counter-based, so any slice of a device tensor can be regenerated alone);
nothing the CUDA path computes is fed to the oracle.  The host work runs on a
thread pool over experts or column chunks (the oracle's C calls and numpy's
matmul release the GIL), with one BLAS thread per task.
"""
import contextlib
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle
import synthetic
from tests._util import bf16_dev, slot_rows, to_dev, to_np, untile

torch = pytest.importorskip("torch")
pytestmark = [pytest.mark.gpu,
              pytest.mark.skipif(not torch.cuda.is_available(), reason="no CUDA device")]


def layer():
    from nvfp4_w4a4_quantized_04_b200 import layer as L
    return L


def nvmod():
    import nvfp4_w4a4_quantized_04_b200 as nv
    return nv


def status_word():
    return torch.zeros(1, dtype=torch.int32, device="cuda")


def gemm_tol(y, y_ref, s_ref):
    err = np.abs(y.astype(np.float64) - y_ref)
    bound = 1e-5 * s_ref + 1e-6
    return err <= bound, err, bound


def tiled_rows_host(sf_flat, row0, nrows, K):
    """Row-major scales of rows [row0, row0 + nrows) of a tensor-core-tiled
    scale tensor already on the host (row0 a multiple of 128)."""
    nsf = K // 16
    per_block = (nsf // 4) * 512
    b0, nb = row0 // 128, (nrows + 127) // 128
    return untile(sf_flat.reshape(-1)[b0 * per_block:(b0 + nb) * per_block], nb * 128, nsf)[:nrows]


def tiled_rows(sf_dev, row0, nrows, K):
    """Row-major scales of rows [row0, row0 + nrows) of a tensor-core-tiled scale
    tensor (row0 and nrows multiples of 128), copied from the device."""
    nsf = K // 16
    per_block = (nsf // 4) * 512
    b0, nb = row0 // 128, (nrows + 127) // 128
    flat = to_np(sf_dev.reshape(-1)[b0 * per_block:(b0 + nb) * per_block])
    return untile(flat, nb * 128, nsf)[:nrows]


def pool_map(fn, items):
    """fn over items on a thread pool of the host's cores, one BLAS thread each."""
    try:
        from threadpoolctl import threadpool_limits
        limit = threadpool_limits(1)
    except Exception:            # without threadpoolctl: the library's own threading
        limit = contextlib.nullcontext()
    with limit, ThreadPoolExecutor(max_workers=max(1, os.cpu_count() or 1)) as ex:
        return list(ex.map(fn, items))


def check_expert_gemm(x_rows_bits, w_bits, a_gpu, w_gpu, y_gpu_rows, a_gs, w_gs):
    """Oracle-quantize both operands of one expert, check the GPU's packed bytes
    against them, then the GPU's fp32 output rows against the fp64 product."""
    qa, sfa, gsa, st = oracle.quantize(x_rows_bits)
    assert st == 0
    qw, sfw, gsw, st = oracle.quantize(w_bits)
    assert st == 0
    assert np.array_equal(a_gpu[0], qa) and np.array_equal(a_gpu[1], sfa) and a_gs == gsa[0]
    assert np.array_equal(w_gpu[0], qw) and np.array_equal(w_gpu[1], sfw) and w_gs == gsw[0]
    a = oracle.dequantize_f64(qa, sfa, np.full(qa.shape[0], gsa[0], np.float32))
    b = oracle.dequantize_f64(qw, sfw, np.full(qw.shape[0], gsw[0], np.float32))
    y_ref, s_ref = oracle.gemm_f64(a, b)
    ok, err, bound = gemm_tol(y_gpu_rows, y_ref, s_ref)
    assert ok.all(), (err.max(), (err / bound).max())


def test_config3_moe_gemms_full_size():
    """512 experts, top-10 of 8192 tokens, H 4096, I 1024: the dispatch quantize
    and both grouped GEMMs run whole; every expert is checked, bytes and rows."""
    import synthetic.cuda as sc
    L = layer()
    E, T, H, I, k = 512, 8192, 4096, 1024, 10
    r = synthetic.route_topk_softmax(0, T, E, k)
    off = r["offsets"].astype(np.int64)
    R = int(off[-1])
    counts = np.diff(off)
    _, starts = slot_rows(off)
    ws = L.workspace(E, "cuda")
    offd = to_dev(r["offsets"])
    s = status_word()
    # gate_up: token-order dispatch quantize, then the grouped GEMM (fp32 out)
    x = sc.gaussian_bf16(0, synthetic.STREAMS["x"], (T, H))
    w = sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (E * 2 * I, H), sigma=0.02)
    wp = L.pack_weights(w, E, 2 * I, None, ws)
    del w
    a1 = L.moe_quantize(x, to_dev(r["slot"].astype(np.int32)), offd, E, layout=1, ws=ws, rows=R, dev_status=s)
    y1 = L.grouped_gemm(a1, wp, 2 * I, 0, dev_status=s)
    # down: an independent seeded h [R, I] in routed order
    h = sc.gaussian_bf16(1, synthetic.STREAMS["x"], (R, I))
    wd = sc.gaussian_bf16(0, synthetic.STREAMS["w_down"], (E * H, I), sigma=0.02)
    wdp = L.pack_weights(wd, E, H, None, ws)
    del wd
    a2 = L.quantize(h, None, offd, E, layout=1, ws=ws, dev_status=s)
    y2 = L.grouped_gemm(a2, wdp, H, 0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    xh = synthetic.gaussian_bf16(0, synthetic.STREAMS["x"], (T, H))
    # device results to the host once
    a1q, a1s, a1g = to_np(a1.q), to_np(a1.sf), to_np(a1.gs)
    a2q, a2s, a2g = to_np(a2.q), to_np(a2.sf), to_np(a2.gs)
    y1h, y2h = to_np(y1), to_np(y2)
    wq, wsf, wg = to_np(wp.q), to_np(wp.sf), to_np(wp.gs)
    wdq, wdsf, wdg = to_np(wdp.q), to_np(wdp.sf), to_np(wdp.gs)

    def check(e):
        m, r0, p0 = int(counts[e]), int(off[e]), int(starts[e])
        if m == 0:
            return
        rows = r["row_index"][r0:r0 + m]
        # gate_up
        a_gpu = (a1q[p0:p0 + m], tiled_rows_host(a1s, p0, m, H))
        w_gpu = (wq[e * 2 * I:(e + 1) * 2 * I], tiled_rows_host(wsf, e * 2 * I, 2 * I, H))
        wbits = synthetic.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (2 * I, H), sigma=0.02, start=e * 2 * I * H)
        check_expert_gemm(xh[rows], wbits, a_gpu, w_gpu, y1h[r0:r0 + m], a1g[e], wg[e])
        # down
        hbits = synthetic.gaussian_bf16(1, synthetic.STREAMS["x"], (m, I), start=r0 * I)
        a_gpu = (a2q[p0:p0 + m], tiled_rows_host(a2s, p0, m, I))
        w_gpu = (wdq[e * H:(e + 1) * H], tiled_rows_host(wdsf, e * H, H, I))
        wbits = synthetic.gaussian_bf16(0, synthetic.STREAMS["w_down"], (H, I), sigma=0.02, start=e * H * I)
        check_expert_gemm(hbits, wbits, a_gpu, w_gpu, y2h[r0:r0 + m], a2g[e], wdg[e])

    pool_map(check, range(E))


def test_config4_decode_full_size():
    """384 experts, 64 tokens, top-10 Zipf routing, H 7168, I 2048, weights
    generated as MXFP4 and remapped on the device: the remap and both grouped
    GEMMs run whole; every expert's remap bytes are checked, and every touched
    expert's activation bytes and GEMM rows."""
    import synthetic.cuda as sc
    L = layer()
    nv = nvmod()
    E, T, H, I, k = 384, 64, 7168, 2048, 10
    r = synthetic.route_zipf_gumbel(7, T, E, k)
    off = r["offsets"].astype(np.int64)
    R = int(off[-1])
    counts = np.diff(off)
    _, starts = slot_rows(off)
    ws = L.workspace(E, "cuda")
    offd = to_dev(r["offsets"])
    s = status_word()
    packs = []
    for name, rows_per, K in (("gate_up", 2 * I, H), ("down", H, I)):
        n = E * rows_per * K
        q = sc.mxfp4_codes(7, synthetic.STREAMS["mx_codes_" + name], n // 2).view(E * rows_per, K // 2)
        e8 = sc.mxfp4_exponents(7, synthetic.STREAMS["mx_exp_" + name], n // 32, lo=-10)
        qn = torch.empty_like(q)
        sf = torch.empty(n // 16, dtype=torch.uint8, device="cuda")
        gs = torch.empty(E, dtype=torch.float32, device="cuda")
        nv.mxfp4_to_nvfp4(q, e8, E, rows_per, K, qn, sf, 1, gs, ws, s)
        del q, e8
        packs.append(L.Packed(qn, sf, gs, E * rows_per, K, 1))
    x = sc.gaussian_bf16(7, synthetic.STREAMS["x"], (T, H))
    a1 = L.moe_quantize(x, to_dev(r["slot"].astype(np.int32)), offd, E, layout=1, ws=ws, rows=R, dev_status=s)
    y1 = L.grouped_gemm(a1, packs[0], 2 * I, 0, dev_status=s)
    h = sc.gaussian_bf16(8, synthetic.STREAMS["x"], (R, I))
    a2 = L.quantize(h, None, offd, E, layout=1, ws=ws, dev_status=s)
    y2 = L.grouped_gemm(a2, packs[1], H, 0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    xh = synthetic.gaussian_bf16(7, synthetic.STREAMS["x"], (T, H))
    acts = [(to_np(a1.q), to_np(a1.sf), to_np(a1.gs), to_np(y1)), (to_np(a2.q), to_np(a2.sf), to_np(a2.gs), to_np(y2))]
    wgs = [to_np(packs[0].gs), to_np(packs[1].gs)]

    def check(e):
        m, r0, p0 = int(counts[e]), int(off[e]), int(starts[e])
        for proj, (rows_per, K) in enumerate(((2 * I, H), (H, I))):
            name = ("gate_up", "down")[proj]
            gpu_w = packs[proj]
            nb = rows_per * K // 2
            qm = synthetic.mxfp4_codes(7, synthetic.STREAMS["mx_codes_" + name], nb, start_byte=e * nb).reshape(rows_per, K // 2)
            em = synthetic.mxfp4_exponents(7, synthetic.STREAMS["mx_exp_" + name], rows_per * K // 32, lo=-10,
                                           start=e * rows_per * K // 32).reshape(rows_per, K // 32)
            qn, sfn, gsn, st = oracle.remap_mxfp4(qm, em, 1, rows_per, K)
            assert st == 0
            assert np.array_equal(to_np(gpu_w.q[e * rows_per:(e + 1) * rows_per]), qn), (name, e)
            assert np.array_equal(tiled_rows(gpu_w.sf, e * rows_per, rows_per, K), sfn), (name, e)
            assert wgs[proj][e] == gsn[0]
            if m == 0:
                continue
            aq, asf, ags, yh = acts[proj]
            if proj == 0:
                xr = xh[r["row_index"][r0:r0 + m]]
            else:
                xr = synthetic.gaussian_bf16(8, synthetic.STREAMS["x"], (m, I), start=r0 * I)
            qa, sfa, gsa, st = oracle.quantize(xr)
            assert st == 0
            assert np.array_equal(aq[p0:p0 + m], qa) and np.array_equal(tiled_rows_host(asf, p0, m, K), sfa)
            assert ags[e] == gsa[0]
            y_ref, s_ref = oracle.gemm_f64(oracle.dequantize_f64(qa, sfa, np.full(m, gsa[0], np.float32)),
                                           oracle.dequantize_f64(qn, sfn, np.full(rows_per, gsn[0], np.float32)))
            ok, err, bound = gemm_tol(yh[r0:r0 + m], y_ref, s_ref)
            assert ok.all(), (name, e, err.max(), (err / bound).max())

    pool_map(check, range(E))


def test_config5_kv_cache_full_size_bitexact():
    """K and V [262144 tokens x 4 heads, 256] (2^28 elements each): K with the
    global from its amax, V with a given (static) global; every code and scale
    byte, the globals and the bf16 dequantized values are compared."""
    import synthetic.cuda as sc
    L = layer()
    nv = nvmod()
    T, Hh, D = 262144, 4, 256
    rows = T * Hh
    kd = sc.gaussian_bf16(0, synthetic.STREAMS["kv_k"], (rows, D))
    vd = sc.gaussian_bf16(0, synthetic.STREAMS["kv_v"], (rows, D))
    kq = torch.empty((rows, D // 2), dtype=torch.uint8, device="cuda")
    vq = torch.empty_like(kq)
    ks = torch.empty(rows * D // 16, dtype=torch.uint8, device="cuda")
    vs = torch.empty_like(ks)
    kgs = torch.empty(1, dtype=torch.float32, device="cuda")
    vgs = torch.tensor([0.0019], dtype=torch.float32, device="cuda")
    s = status_word()
    # K: global from the amax; V: a given global
    nv.nvfp4_quantize(kd, rows, D, D, None, None, 1, 0, kgs, kq, ks, 0, L.workspace(1), s)
    nv.nvfp4_quantize(vd, rows, D, D, None, None, 1, 1, vgs, vq, vs, 0, L.workspace(1), s)
    ko = torch.empty((rows, D), dtype=torch.bfloat16, device="cuda")
    vo = torch.empty_like(ko)
    nv.nvfp4_kv_dequantize(kq, ks, kgs, vq, vs, vgs, T, Hh, D, ko, vo)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    for stream, given, qg, sg, gg, og in ((synthetic.STREAMS["kv_k"], None, kq, ks, kgs, ko),
                                          (synthetic.STREAMS["kv_v"], np.float32(0.0019), vq, vs, vgs, vo)):
        xh = synthetic.gaussian_bf16(0, stream, (rows, D))
        qr, sr, gr, st = oracle.quantize(xh, global_scale=None if given is None else np.array([given], np.float32))
        assert st == 0
        assert to_np(gg)[0] == gr[0]
        assert np.array_equal(to_np(qg), qr)
        assert np.array_equal(to_np(sg).reshape(rows, D // 16), sr)
        ref = oracle.dequantize(qr, sr, np.full(rows, gr[0], np.float32), out="bf16")
        assert np.array_equal(to_np(og), ref)
        del xh, qr, sr, ref


def test_config5_activation_quantize_full_size_bitexact():
    """The largest activation sweep point, [131072, 5120] bf16 (671 M elements),
    dynamic global, tensor-core scale layout: every byte and the global."""
    import synthetic.cuda as sc
    L = layer()
    T, H = 131072, 5120
    xd = sc.gaussian_bf16(0, synthetic.STREAMS["x_sweep"], (T, H))
    s = status_word()
    p = L.quantize(xd, layout=1, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    del xd
    xh = synthetic.gaussian_bf16(0, synthetic.STREAMS["x_sweep"], (T, H))
    qr, sr, gr, st = oracle.quantize(xh)
    assert st == 0
    del xh
    assert to_np(p.gs)[0] == gr[0]
    assert np.array_equal(to_np(p.q[:T]), qr)
    assert np.array_equal(tiled_rows(p.sf, 0, T, H), sr)


def test_config5_remap_full_size_bitexact():
    """2^28 MXFP4 elements as 1024 tensors [512, 512], remapped to NVFP4 with
    tensor-core scales: codes, scale bytes and the 1024 globals."""
    import synthetic.cuda as sc
    L = layer()
    nt, rows, K = 1024, 512, 512
    n = nt * rows * K
    q = sc.mxfp4_codes(0, synthetic.STREAMS["mx_codes"], n // 2).view(nt * rows, K // 2)
    e8 = sc.mxfp4_exponents(0, synthetic.STREAMS["mx_exp"], n // 32)
    s = status_word()
    p = L.remap_mxfp4(q, e8, nt, rows, K, layout=1, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    qh = synthetic.mxfp4_codes(0, synthetic.STREAMS["mx_codes"], n // 2).reshape(nt * rows, K // 2)
    eh = synthetic.mxfp4_exponents(0, synthetic.STREAMS["mx_exp"], n // 32).reshape(nt * rows, K // 32)
    qn, sfn, gsn, st = oracle.remap_mxfp4(qh, eh, nt, rows, K)
    assert st == 0
    assert np.array_equal(to_np(p.q), qn)
    assert np.array_equal(to_np(p.gs), gsn)
    assert np.array_equal(tiled_rows(p.sf, 0, nt * rows, K), sfn)


def test_config2_dense_mlp_full_size():
    """Dense MLP, 4096 tokens, hidden 5120, intermediate 17408, X with 0.1 %
    outliers x50: both activation quantizes and both weight packings are
    compared byte for byte, every output element of both GEMMs is checked (in
    chunks of 1024 weight rows), and the fused SwiGLU epilogue plus the
    requantize of its h are checked against the same GEMM."""
    import synthetic.cuda as sc
    L = layer()
    M, H, I = 4096, 5120, 17408
    ws = L.workspace(1, "cuda")
    s = status_word()
    wgu = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (2 * I, H), sigma=0.02), 1, 2 * I, None, ws)
    wd = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_down"], (H, I), sigma=0.02), 1, H, None, ws)
    xb = synthetic.gaussian_bf16(0, synthetic.STREAMS["x"], (M, H), outlier_frac=0.001)
    a1 = L.quantize(bf16_dev(xb), layout=1, ws=ws, dev_status=s)
    y1 = L.grouped_gemm(a1, wgu, 2 * I, 0, dev_status=s)
    hb = synthetic.gaussian_bf16(2, synthetic.STREAMS["x"], (M, I))
    a2 = L.quantize(bf16_dev(hb), layout=1, ws=ws, dev_status=s)
    y2 = L.grouped_gemm(a2, wd, H, 0, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    for (abits, a, w, N, K, stream, y) in ((xb, a1, wgu, 2 * I, H, "w_gate_up", y1), (hb, a2, wd, H, I, "w_down", y2)):
        qa, sfa, gsa, st = oracle.quantize(abits)
        assert st == 0
        assert np.array_equal(to_np(a.q[:M]), qa) and np.array_equal(tiled_rows(a.sf, 0, M, K), sfa)
        assert to_np(a.gs)[0] == gsa[0]
        wbits = synthetic.gaussian_bf16(0, synthetic.STREAMS[stream], (N, K), sigma=0.02)
        qw, sfw, gsw, st = oracle.quantize(wbits)
        del wbits
        assert st == 0 and to_np(w.gs)[0] == gsw[0]
        assert np.array_equal(to_np(w.q[:N]), qw)
        assert np.array_equal(tiled_rows(w.sf, 0, N, K), sfw)
        aref = oracle.dequantize_f64(qa, sfa, np.full(M, gsa[0], np.float32))
        yh = to_np(y)

        def check(c0, qw=qw, sfw=sfw, gsw=gsw, aref=aref, yh=yh, N=N, stream=stream):
            c1 = min(N, c0 + 1024)
            bref = oracle.dequantize_f64(qw[c0:c1], sfw[c0:c1], np.full(c1 - c0, gsw[0], np.float32))
            y_ref, s_ref = oracle.gemm_f64(aref, bref)
            ok, err, bound = gemm_tol(yh[:, c0:c1], y_ref, s_ref)
            assert ok.all(), (stream, c0, err.max(), (err / bound).max())

        pool_map(check, range(0, N, 1024))
        del aref, qw, sfw
        if stream == "w_gate_up":
            y1h = yh
        del yh
    # the fused form the bench times: SwiGLU in the gate_up epilogue (one group,
    # interleaved gate/up rows), then h requantized from the epilogue's amax.
    # The accumulators are the GEMM's above, so h is checked against the
    # oracle SwiGLU of that fp32 output (one bf16 ulp), the amax exactly, and
    # the requantized bytes against the oracle's quantize of the device's h.
    from nvfp4_w4a4_quantized_04_b200 import GS_AMAX_GIVEN, nvfp4_quantize
    wil = L.pack_weights(sc.gaussian_bf16(0, synthetic.STREAMS["w_gate_up"], (2 * I, H), sigma=0.02), 1, 2 * I,
                         L.gate_up_interleave_index(1, I, "cuda"), ws)
    h, amax = L.grouped_gemm_swiglu(a1, wil, 2 * I, dev_status=s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    h_gpu = to_np(h)
    h_ref = oracle.swiglu(y1h)
    d = np.abs(h_gpu.astype(np.int32) - h_ref.astype(np.int32))
    assert (d <= 1).all() and (d == 0).mean() > 0.99
    assert to_np(amax)[0] == np.abs(synthetic.bf16_bits_to_f32(h_gpu)).max()
    a3 = L.empty_packed(M, I, 1, None, 1, "cuda")
    nvfp4_quantize(h, M, I, I, None, None, 1, GS_AMAX_GIVEN, amax, a3.q, a3.sf, 1, ws, s)
    torch.cuda.synchronize()
    assert int(s.item()) == 0
    qh, sfh, gsh, st = oracle.quantize(h_gpu)
    assert st == 0 and to_np(amax)[0] == gsh[0]
    assert np.array_equal(to_np(a3.q[:M]), qh) and np.array_equal(tiled_rows(a3.sf, 0, M, I), sfh)
