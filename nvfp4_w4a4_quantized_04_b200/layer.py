"""Host-side orchestration of the NVFP4 routed-expert path on the C ABI.

Torch provides device memory and the stream; each step is one call into
``libnvfp4.so``.  ``MoEExperts.forward`` is the MoE layer's expert part:
gather + per-group dynamic quantize -> grouped gate_up GEMM -> SwiGLU +
per-group requantize -> grouped down GEMM (the routed-expert projections of
the "Qwen3.8-Flash-Next-NVFP4" page, quantized W4A4).
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Optional

import torch

from . import (EPI_NONE, EPI_SWIGLU, GS_AMAX_GIVEN, GS_FROM_AMAX, GS_GIVEN, OUT_BF16, OUT_F32, SF_MMA_TILED, SF_ROWMAJOR,
               mxfp4_grouped_gemm as _mxfp4_grouped_gemm, mxfp4_quantize as _mxfp4_quantize, mxfp4_to_nvfp4, nvfp4_dequantize, nvfp4_grouped_gemm, nvfp4_grouped_gemm_swiglu_nvfp4,
               nvfp4_global_scale_from_amax, nvfp4_grouped_gemm_w4a16, nvfp4_moe_combine,
               nvfp4_w4a16_workspace_size,
               nvfp4_moe_route,
               nvfp4_moe_quantize, nvfp4_moe_route_workspace_size, nvfp4_padded_rows_bound, nvfp4_quantize,
               nvfp4_swiglu_quantize,
               nvfp4_workspace_size)


@dataclass
class Packed:
    """An NVFP4 tensor in device memory.

    q: uint8 [rows_alloc, K/2]; sf: uint8 scales (``layout``); gs: fp32 [G]
    global scales.  With ``offsets`` (int32 [G+1] on the device) rows sit in
    128-aligned per-group slots.
    """
    q: torch.Tensor
    sf: torch.Tensor
    gs: torch.Tensor
    rows: int
    K: int
    layout: int
    offsets: Optional[torch.Tensor] = None
    num_groups: int = 1


def workspace(num_groups: int, device="cuda") -> torch.Tensor:
    n = nvfp4_workspace_size(max(1, num_groups))
    return torch.empty(n, dtype=torch.uint8, device=device)


def alloc_rows(rows: int, num_groups: int, grouped: bool, layout: int) -> int:
    if grouped:
        return nvfp4_padded_rows_bound(rows, num_groups)
    return (rows + 127) // 128 * 128 if layout == SF_MMA_TILED else rows


def sf_bytes(rows_alloc: int, K: int) -> int:
    return rows_alloc * (K // 16)


def empty_packed(rows: int, K: int, num_groups: int = 1, offsets=None, layout=SF_MMA_TILED,
                 device="cuda") -> Packed:
    ra = alloc_rows(rows, num_groups, offsets is not None, layout)
    q = torch.empty((max(ra, 1), K // 2), dtype=torch.uint8, device=device)
    sf = torch.empty(max(sf_bytes(ra, K), 1), dtype=torch.uint8, device=device)
    gs = torch.empty(max(1, num_groups), dtype=torch.float32, device=device)
    return Packed(q, sf, gs, rows, K, layout, offsets, num_groups if offsets is not None else 1)


def quantize(x: torch.Tensor, row_index=None, offsets=None, num_groups: int = 1, layout=SF_MMA_TILED,
             global_scale=None, out: Optional[Packed] = None, ws=None, dev_status=None, rows=None) -> Packed:
    """NVFP4-quantize bf16 rows (dynamic global scale unless ``global_scale`` is given)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2
    K = x.shape[1]
    R = rows if rows is not None else (row_index.shape[0] if row_index is not None else x.shape[0])
    G = num_groups if offsets is not None else 1
    p = out if out is not None else empty_packed(R, K, G, offsets, layout, x.device)
    p.offsets, p.num_groups, p.rows = offsets, G, R
    mode = GS_FROM_AMAX
    if global_scale is not None:
        p.gs.copy_(global_scale)
        mode = GS_GIVEN
    ws = ws if ws is not None else workspace(G, x.device)
    nvfp4_quantize(x, R, K, x.stride(0), row_index, offsets, G, mode, p.gs, p.q, p.sf, layout, ws, dev_status)
    return p


def moe_quantize(x: torch.Tensor, slot: torch.Tensor, offsets: torch.Tensor, num_groups: int, layout=SF_MMA_TILED,
                 out: Optional[Packed] = None, ws=None, dev_status=None, rows=None) -> Packed:
    """Routed-expert activations quantized in token order: the same packed rows
    as ``quantize(x, row_index, offsets, ...)`` with row_index the inverse of
    ``slot`` [T, k] (routed row of each token choice), each token read once."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and slot.dim() == 2
    T, k = slot.shape
    K = x.shape[1]
    R = rows if rows is not None else T * k
    p = out if out is not None else empty_packed(R, K, num_groups, offsets, layout, x.device)
    p.offsets, p.num_groups, p.rows = offsets, num_groups, R
    ws = ws if ws is not None else workspace(num_groups, x.device)
    nvfp4_moe_quantize(x, T, K, x.stride(0), slot, k, offsets, num_groups, GS_FROM_AMAX, p.gs, p.q, p.sf, layout,
                       ws, dev_status)
    return p


def dequantize(p: Packed, out_dtype=OUT_F32) -> torch.Tensor:
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    y = torch.empty((p.rows, p.K), dtype=dt, device=p.q.device)
    nvfp4_dequantize(p.q, p.sf, p.layout, p.gs, p.offsets, p.num_groups, p.rows, p.K, y, out_dtype)
    return y


def remap_mxfp4(q_mx: torch.Tensor, e8: torch.Tensor, n_tensors: int, rows: int, K: int, layout=SF_MMA_TILED,
                ws=None, dev_status=None, inplace: bool = False) -> Packed:
    """Lossless MXFP4 -> NVFP4 remap of n_tensors [rows, K] tensors."""
    q_nv = q_mx if inplace else torch.empty_like(q_mx)
    sf = torch.empty(n_tensors * rows * (K // 16), dtype=torch.uint8, device=q_mx.device)
    gs = torch.empty(n_tensors, dtype=torch.float32, device=q_mx.device)
    ws = ws if ws is not None else workspace(n_tensors, q_mx.device)
    mxfp4_to_nvfp4(q_mx, e8, n_tensors, rows, K, q_nv, sf, layout, gs, ws, dev_status)
    return Packed(q_nv, sf, gs, n_tensors * rows, K, layout, None, n_tensors)


def mxfp4_quantize(x: torch.Tensor, layout=SF_ROWMAJOR, dev_status=None):
    """MXFP4 encode of bf16 rows [rows, K]: (codes uint8 [rows, K/2], UE8M0
    scales, one per 32 elements, in `layout`)."""
    assert x.dtype == torch.bfloat16 and x.dim() == 2 and x.stride(1) == 1
    rows, K = x.shape
    q = torch.empty((rows, K // 2), dtype=torch.uint8, device=x.device)
    if layout == SF_MMA_TILED:
        e8 = torch.empty(((rows + 127) // 128 * 128) * (K // 32), dtype=torch.uint8, device=x.device)
    else:
        e8 = torch.empty((rows, K // 32), dtype=torch.uint8, device=x.device)
    _mxfp4_quantize(x, rows, K, x.stride(0), q, e8, layout, dev_status)
    return q, e8


def mx_grouped_gemm(a_q: torch.Tensor, a_sf: torch.Tensor, w_q: torch.Tensor, w_sf: torch.Tensor, N: int, K: int,
                    rows: int, offsets: Optional[torch.Tensor] = None, num_experts: int = 1, out_dtype=OUT_BF16,
                    y=None, dev_status=None) -> torch.Tensor:
    """MXFP4 x MXFP4 grouped GEMM: Y [rows, N] = per expert A_e W_e^T
    (activations in 128-aligned expert slots, tensor-core scale layout)."""
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if y is None:
        y = torch.empty((rows, N), dtype=dt, device=a_q.device)
    E = num_experts if offsets is not None else 1
    _mxfp4_grouped_gemm(a_q, a_sf, w_q, w_sf, offsets, E, rows, N, K, y, out_dtype, None, dev_status)
    return y


def grouped_gemm(a: Packed, w: Packed, N: int, out_dtype=OUT_BF16, y=None, dev_status=None) -> torch.Tensor:
    """Y [a.rows, N] = per expert (a_gs[e] * w_gs[e]) * A_e W_e^T."""
    assert a.layout == SF_MMA_TILED and w.layout == SF_MMA_TILED
    E = a.num_groups if a.offsets is not None else 1
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if y is None:
        y = torch.empty((a.rows, N), dtype=dt, device=a.q.device)
    nvfp4_grouped_gemm(a.q, a.sf, a.gs, w.q, w.sf, w.gs, a.offsets, E, a.rows, N, a.K, y, out_dtype, EPI_NONE,
                       None, None, dev_status)
    return y


def gate_up_interleave_index(E: int, I: int, device="cuda") -> torch.Tensor:
    """Source row of each packed row of a fused gate_up weight [E*2I, K] in the
    order the SwiGLU epilogue reads: per expert, 32-row groups holding 16 gate
    rows and then the 16 matching up rows (gate rows are 0..I-1 of the expert,
    up rows I..2I-1 in the source).  int32 [E*2I]."""
    assert I % 64 == 0
    n = torch.arange(E * 2 * I, dtype=torch.int64)
    e, m = n // (2 * I), n % (2 * I)
    j, r = m // 32, m % 32
    src = e * 2 * I + torch.where(r < 16, 16 * j + r, I + 16 * j + (r - 16))
    return src.to(torch.int32).to(device)


def pack_weights(w: torch.Tensor, E: int, rows_per: int, row_index=None, ws=None) -> Packed:
    """Static NVFP4 quantization of per-expert weights [E*rows_per, K] (one global
    scale per expert, MMA-tiled scales), optionally reordering rows within each
    expert (``row_index``, e.g. ``gate_up_interleave_index``)."""
    offs = torch.arange(0, (E + 1) * rows_per, rows_per, dtype=torch.int32, device=w.device)
    p = quantize(w, row_index, offs, E, SF_MMA_TILED, ws=ws)
    p.offsets, p.num_groups, p.rows = None, 1, E * rows_per
    return p


def grouped_gemm_swiglu(a: Packed, w_gate_up: Packed, N: int, h=None, amax=None, dev_status=None):
    """h [a.rows, N/2] = bf16(silu(g) * u) straight from the gate_up GEMM's
    accumulators, plus the per-expert amax of h (fp32 [E]).  ``w_gate_up`` is
    packed in the interleaved row order of ``gate_up_interleave_index``."""
    assert a.layout == SF_MMA_TILED and w_gate_up.layout == SF_MMA_TILED
    E = a.num_groups if a.offsets is not None else 1
    if h is None:
        h = torch.empty((a.rows, N // 2), dtype=torch.bfloat16, device=a.q.device)
    if amax is None:
        amax = torch.empty(E, dtype=torch.float32, device=a.q.device)
    nvfp4_grouped_gemm(a.q, a.sf, a.gs, w_gate_up.q, w_gate_up.sf, w_gate_up.gs, a.offsets, E, a.rows, N, a.K, h,
                       OUT_BF16, EPI_SWIGLU, amax, None, dev_status)
    return h, amax


def grouped_gemm_swiglu_nvfp4(a: Packed, w_gate_up: Packed, N: int, h_gs: torch.Tensor, out: Optional[Packed] = None,
                              dev_status=None) -> Packed:
    """gate_up GEMM + SwiGLU whose epilogue quantizes h with the given per-expert
    global ``h_gs`` (the down projection's calibrated input scale): the packed
    down-GEMM input, with no bf16 h in memory."""
    assert a.layout == SF_MMA_TILED and w_gate_up.layout == SF_MMA_TILED
    E = a.num_groups if a.offsets is not None else 1
    I = N // 2
    p = out if out is not None else empty_packed(a.rows, I, E, a.offsets, SF_MMA_TILED, a.q.device)
    p.offsets, p.num_groups, p.rows = a.offsets, E, a.rows
    p.gs = h_gs
    nvfp4_grouped_gemm_swiglu_nvfp4(a.q, a.sf, a.gs, w_gate_up.q, w_gate_up.sf, w_gate_up.gs, a.offsets, E, a.rows,
                                    N, a.K, h_gs, p.q, p.sf, None, dev_status)
    return p


def w4a16_workspace(rows: int, num_groups: int, K: int, device="cuda") -> torch.Tensor:
    return torch.empty(nvfp4_w4a16_workspace_size(rows, num_groups, K), dtype=torch.uint8, device=device)


def grouped_gemm_w4a16(x: torch.Tensor, w: Packed, N: int, row_index=None, offsets=None, num_groups: int = 1,
                       rows=None, out_dtype=OUT_BF16, swiglu=False, y=None, ws=None, dev_status=None) -> torch.Tensor:
    """Weight-only NVFP4 (row-major scales) x bf16 activations, per expert:
    Y [rows, N] (or h [rows, N/2] with ``swiglu``; gate rows first)."""
    assert x.dtype == torch.bfloat16 and w.layout == SF_ROWMAJOR
    M = rows if rows is not None else (row_index.shape[0] if row_index is not None else x.shape[0])
    G = num_groups if offsets is not None else 1
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    cols = N // 2 if swiglu else N
    if y is None:
        y = torch.empty((M, cols), dtype=dt, device=x.device)
    if ws is None:
        ws = w4a16_workspace(M, G, w.K, x.device)
    nvfp4_grouped_gemm_w4a16(x, x.stride(0), x.shape[0], row_index, w.q, w.sf, w.gs, offsets, G, M, N, w.K, y,
                             out_dtype, EPI_SWIGLU if swiglu else EPI_NONE, ws, dev_status)
    return y


def swiglu_quantize(y: torch.Tensor, offsets, num_groups: int, layout=SF_MMA_TILED, out: Optional[Packed] = None,
                    h=None, ws=None, dev_status=None):
    rows, I2 = y.shape
    I = I2 // 2
    G = num_groups if offsets is not None else 1
    p = out if out is not None else empty_packed(rows, I, G, offsets, layout, y.device)
    p.offsets, p.num_groups, p.rows = offsets, G, rows
    h = h if h is not None else torch.empty((rows, I), dtype=torch.bfloat16, device=y.device)
    ws = ws if ws is not None else workspace(G, y.device)
    ydt = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    nvfp4_swiglu_quantize(y, ydt, rows, I, offsets, G, p.gs, p.q, p.sf, layout, h, ws, dev_status)
    return p, h


class MoEExperts:
    """Routed experts of one MoE layer in NVFP4 W4A4.

    w_gate_up: packed [E*2I, H], one global scale per expert: rows 0..I-1 of
    each expert = gate, I..2I-1 = up; with ``fused_swiglu`` the rows are in the
    order of ``gate_up_interleave_index`` instead.  w_down: packed [E*H, I].
    forward(x bf16 [T, H], row_index int32 [R], offsets int32 [E+1]) -> Y bf16 [R, H]
    in routed order (the weighted combine is outside this layer).  With
    ``h_scale`` set (a given down-input global per expert, see
    ``calibrate_h_scale``) the gate_up epilogue writes NVFP4 h directly.
    """

    def __init__(self, w_gate_up: Packed, w_down: Packed, E: int, H: int, I: int, max_rows: int,
                 out_dtype=OUT_BF16, mid_dtype=OUT_BF16, device="cuda", fused_swiglu: bool = False):
        self.fused_swiglu = fused_swiglu
        self.h_scale: Optional[torch.Tensor] = None   # given down-input global per expert (fp32 [E])
        self.amax = torch.zeros(E, dtype=torch.float32, device=device)
        self.w_gate_up, self.w_down = w_gate_up, w_down
        self.E, self.H, self.I = E, H, I
        self.out_dtype, self.mid_dtype = out_dtype, mid_dtype
        self.ws = workspace(E, device)
        self.a1 = empty_packed(max_rows, H, E, torch.empty(0), SF_MMA_TILED, device)
        self.a2 = empty_packed(max_rows, I, E, torch.empty(0), SF_MMA_TILED, device)
        mdt = torch.bfloat16 if mid_dtype == OUT_BF16 else torch.float32
        odt = torch.bfloat16 if out_dtype == OUT_BF16 else torch.float32
        self.y1 = torch.empty((max_rows, 2 * I), dtype=mdt, device=device)
        self.h = torch.empty((max_rows, I), dtype=torch.bfloat16, device=device)
        self.y2 = torch.empty((max_rows, H), dtype=odt, device=device)
        self.max_rows = max_rows

    def _quantize_input(self, x, row_index, offsets, slot, dev_status):
        R = row_index.shape[0]
        if slot is not None:
            return moe_quantize(x, slot, offsets, self.E, SF_MMA_TILED, out=self.a1, ws=self.ws,
                                dev_status=dev_status, rows=R)
        return quantize(x, row_index, offsets, self.E, SF_MMA_TILED, out=self.a1, ws=self.ws,
                        dev_status=dev_status, rows=R)

    def forward(self, x: torch.Tensor, row_index: torch.Tensor, offsets: torch.Tensor, dev_status=None,
                slot: Optional[torch.Tensor] = None):
        """``slot`` [T, k] (routed row of each token choice), when given, selects
        the token-order quantize that reads each token row once."""
        R = row_index.shape[0]
        assert R <= self.max_rows
        E, H, I = self.E, self.H, self.I
        a1 = self._quantize_input(x, row_index, offsets, slot, dev_status)
        if self.h_scale is not None:
            # calibrated down-input global: the gate_up epilogue writes NVFP4 h itself
            a2 = grouped_gemm_swiglu_nvfp4(a1, self.w_gate_up, 2 * I, self.h_scale, out=self.a2,
                                           dev_status=dev_status)
        elif self.fused_swiglu:
            # SwiGLU in the gate_up epilogue; its amax feeds the requantize directly
            h, amax = grouped_gemm_swiglu(a1, self.w_gate_up, 2 * I, h=self.h[:R], amax=self.amax,
                                          dev_status=dev_status)
            a2 = self.a2
            a2.offsets, a2.num_groups, a2.rows = offsets, E, R
            nvfp4_quantize(h, R, I, I, None, offsets, E, GS_AMAX_GIVEN, amax, a2.q, a2.sf, SF_MMA_TILED, self.ws,
                           dev_status)
            a2.gs = amax
        else:
            y1 = self.y1[:R]
            grouped_gemm(a1, self.w_gate_up, 2 * I, self.mid_dtype, y=y1, dev_status=dev_status)
            a2, _ = swiglu_quantize(y1, offsets, E, SF_MMA_TILED, out=self.a2, h=self.h[:R], ws=self.ws,
                                    dev_status=dev_status)
        y2 = self.y2[:R]
        grouped_gemm(a2, self.w_down, H, self.out_dtype, y=y2, dev_status=dev_status)
        return y2


def calibrate_h_scale(experts: "MoEExperts", x, row_index, offsets, slot=None, margin: float = 1.0,
                      dev_status=None) -> torch.Tensor:
    """A down-input global per expert from one calibration batch, as a
    calibration pass would set the checkpoint's input_scale, installed on
    ``experts``: the dynamic path's first two stages give the per-expert max |h|
    (SwiGLU epilogue), and the library turns it into s_g = margin * max|h| / 2688
    (1 for an expert without tokens) with the same arithmetic as the dynamic
    global scale.  With margin 1 the result is exactly the s_g a dynamic forward
    derives for the same batch."""
    assert experts.fused_swiglu
    experts.h_scale = None
    R = row_index.shape[0]
    a1 = experts._quantize_input(x, row_index, offsets, slot, dev_status)
    _, amax = grouped_gemm_swiglu(a1, experts.w_gate_up, 2 * experts.I, h=experts.h[:R], amax=experts.amax,
                                  dev_status=dev_status)
    gs = torch.empty(experts.E, dtype=torch.float32, device=amax.device)
    nvfp4_global_scale_from_amax(amax, experts.E, margin, gs, dev_status)
    experts.h_scale = gs
    return gs


def route(topk_ids: torch.Tensor, num_experts: int, dev_status=None):
    """Expert-grouped order of routed rows: (offsets [E+1], row_index [T*k], slot [T, k])."""
    T, k = topk_ids.shape
    dev = topk_ids.device
    off = torch.empty(num_experts + 1, dtype=torch.int32, device=dev)
    ri = torch.empty(T * k, dtype=torch.int32, device=dev)
    slot = torch.empty((T, k), dtype=torch.int32, device=dev)
    ws = torch.empty(nvfp4_moe_route_workspace_size(T, num_experts), dtype=torch.uint8, device=dev)
    nvfp4_moe_route(topk_ids, T, k, num_experts, off, ri, slot, ws, dev_status)
    return off, ri, slot


def combine(y: torch.Tensor, slot: torch.Tensor, weights: torch.Tensor, out_dtype=OUT_BF16, out=None,
            dev_status=None):
    """out[t] = sum_j weights[t, j] * y[slot[t, j]] (fp32 accumulation); slots
    outside y's rows are skipped and reported in dev_status."""
    T, k = slot.shape
    H = y.shape[1]
    dt = torch.float32 if out_dtype == OUT_F32 else torch.bfloat16
    if out is None:
        out = torch.empty((T, H), dtype=dt, device=y.device)
    ydt = OUT_F32 if y.dtype == torch.float32 else OUT_BF16
    nvfp4_moe_combine(y, ydt, y.shape[0], slot, weights, T, k, H, out, out_dtype, dev_status)
    return out


class MoELayer:
    """A whole routed-expert MoE block on one GPU: routing order, the NVFP4
    W4A4 experts, and the weighted combine back to [T, H].

    forward(x bf16 [T, H], topk_ids int32 [T, k], topk_weights fp32 [T, k]) -> bf16 [T, H].
    The router itself (BF16 gate, top-k) stays outside, as on the pages.
    """

    def __init__(self, experts: MoEExperts, max_tokens: int, topk: int, device="cuda"):
        self.experts = experts
        E = experts.E
        self.off = torch.empty(E + 1, dtype=torch.int32, device=device)
        self.ri = torch.empty(max_tokens * topk, dtype=torch.int32, device=device)
        self.slot = torch.empty((max_tokens, topk), dtype=torch.int32, device=device)
        self.rws = torch.empty(nvfp4_moe_route_workspace_size(max_tokens, E), dtype=torch.uint8, device=device)
        self.out = torch.empty((max_tokens, experts.H), dtype=torch.bfloat16, device=device)

    def forward(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor, dev_status=None):
        T, k = topk_ids.shape
        E = self.experts.E
        slot = self.slot[:T]
        ri = self.ri[:T * k]
        nvfp4_moe_route(topk_ids, T, k, E, self.off, ri, slot, self.rws, dev_status)
        y = self.experts.forward(x, ri, self.off, dev_status, slot=slot)
        out = self.out[:T]
        nvfp4_moe_combine(y, OUT_F32 if y.dtype == torch.float32 else OUT_BF16, y.shape[0], slot, topk_weights, T, k,
                          self.experts.H, out, OUT_BF16, dev_status)
        return out

    def capture(self, x: torch.Tensor, topk_ids: torch.Tensor, topk_weights: torch.Tensor, dev_status=None):
        """Record forward() on these input tensors as a CUDA graph.

        Returns (graph, out): graph.replay() reruns the whole block (routing
        order, experts, combine: about ten kernel launches and memsets) on the
        current contents of x, topk_ids and topk_weights, which keep their
        shapes and addresses, and leaves the result in out.  forward() issues
        no host synchronisation and allocates nothing, so it captures as is;
        one eager call first sets the kernels' launch attributes.

        ``out`` is a view of this layer's own output buffer, not a copy: a
        later eager forward(), or the replay of another graph captured on this
        layer, overwrites it.  Copy it out (or read it) before either runs."""
        self.forward(x, topk_ids, topk_weights, dev_status)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            out = self.forward(x, topk_ids, topk_weights, dev_status)
        return graph, out
