"""NVFP4 W4A4 routed-expert hot path for B200 (sm_100a): Python binding.

A thin ctypes layer over ``libnvfp4.so`` (the C ABI declared in
``include/nvfp4.h``).  It only marshals arguments: torch tensors supply device
memory and the current CUDA stream; every step of the path runs in the
library's kernels.  There is no CPU fallback: if the library is missing or
no CUDA device is present, the calls raise.

Entry points (same names as the C ABI): ``nvfp4_quantize``,
``nvfp4_dequantize``, ``mxfp4_to_nvfp4``, ``mxfp4_quantize``, ``mxfp4_grouped_gemm``,
``nvfp4_grouped_gemm``,
``nvfp4_swiglu_quantize``, ``nvfp4_kv_quantize``, ``nvfp4_kv_dequantize``,
``nvfp4_moe_quantize``, ``nvfp4_moe_route``, ``nvfp4_moe_combine``,
``nvfp4_quantize_noalloc``, ``nvfp4_global_scale_from_amax``, plus ``nvfp4_workspace_size``,
``nvfp4_padded_rows_bound`` and ``nvfp4_moe_route_workspace_size``.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libnvfp4.so")

# status codes (include/nvfp4.h)
OK = 0
ERR_INVALID_ARG = 1
ERR_UNSUPPORTED_SHAPE = 2
ERR_CUDA = 3
ERR_NONFINITE = 16
ERR_NOT_REPRESENTABLE = 17
ERR_TIMEOUT = 18
ERR_INDEX = 19

SF_ROWMAJOR = 0
SF_MMA_TILED = 1
GS_FROM_AMAX = 0
GS_GIVEN = 1
OUT_F32 = 0
OUT_BF16 = 1
EPI_NONE = 0
EPI_SWIGLU = 1
GS_AMAX_GIVEN = 2

EXPORTS = [
    "nvfp4_status_string", "nvfp4_workspace_size", "nvfp4_padded_rows_bound",
    "nvfp4_quantize", "nvfp4_dequantize", "mxfp4_to_nvfp4", "nvfp4_grouped_gemm",
    "nvfp4_swiglu_quantize", "nvfp4_kv_quantize", "nvfp4_kv_dequantize", "nvfp4_quantize_noalloc",
    "nvfp4_moe_route_workspace_size", "nvfp4_moe_route", "nvfp4_moe_combine", "nvfp4_moe_quantize",
    "nvfp4_gemm_select_kernel", "nvfp4_grouped_gemm_w4a16", "nvfp4_grouped_gemm_swiglu_nvfp4",
    "mxfp4_quantize", "mxfp4_grouped_gemm", "nvfp4_w4a16_workspace_size",
    "nvfp4_e2m1_encode", "nvfp4_e4m3_encode", "nvfp4_gemm_set_wait_budget", "nvfp4_global_scale_from_amax",
    "nvfp4_w4a16_select_kernel",
]
NOALLOC_MAX_GROUPS = 1024

_lib = None


class Nvfp4Error(RuntimeError):
    pass


def load_library(path: str = LIB_PATH):
    """Load libnvfp4.so and declare the C signatures.  Raises if it is absent."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise Nvfp4Error(f"{path} not found: build it with `python -m nvfp4_w4a4_quantized_04_b200.build`")
    L = ctypes.CDLL(path)
    P, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
    L.nvfp4_status_string.restype = ctypes.c_char_p
    L.nvfp4_status_string.argtypes = [i32]
    L.nvfp4_workspace_size.restype = ctypes.c_size_t
    L.nvfp4_workspace_size.argtypes = [i32]
    L.nvfp4_padded_rows_bound.restype = i64
    L.nvfp4_padded_rows_bound.argtypes = [i64, i32]
    L.nvfp4_quantize.restype = i32
    L.nvfp4_quantize.argtypes = [P, i64, i64, i64, P, P, i32, i32, P, P, P, i32, P, P, P]
    L.nvfp4_grouped_gemm_swiglu_nvfp4.restype = i32
    L.nvfp4_grouped_gemm_swiglu_nvfp4.argtypes = [P, P, P, P, P, P, P, i32, i64, i64, i64, P, P, P, P, P, P]
    L.nvfp4_grouped_gemm_w4a16.restype = i32
    L.nvfp4_grouped_gemm_w4a16.argtypes = [P, i64, i64, P, P, P, P, P, i32, i64, i64, i64, P, i32, i32, P, P, P]
    L.nvfp4_w4a16_workspace_size.restype = ctypes.c_size_t
    L.nvfp4_w4a16_workspace_size.argtypes = [i64, i32, i64]
    L.nvfp4_gemm_select_kernel.restype = i32
    L.nvfp4_gemm_select_kernel.argtypes = [i32]
    L.nvfp4_w4a16_select_kernel.restype = i32
    L.nvfp4_w4a16_select_kernel.argtypes = [i32]
    L.nvfp4_moe_quantize.restype = i32
    L.nvfp4_moe_quantize.argtypes = [P, i64, i64, i64, P, i32, P, i32, i32, P, P, P, i32, P, P, P]
    L.nvfp4_dequantize.restype = i32
    L.nvfp4_dequantize.argtypes = [P, P, i32, P, P, i32, i64, i64, P, i32, P]
    L.mxfp4_to_nvfp4.restype = i32
    L.mxfp4_quantize.restype = i32
    L.mxfp4_grouped_gemm.restype = i32
    L.mxfp4_grouped_gemm.argtypes = [P, P, P, P, P, i32, i64, i64, i64, P, i32, P, P, P]
    L.mxfp4_quantize.argtypes = [P, i64, i64, i64, P, P, i32, P, P]
    L.mxfp4_to_nvfp4.argtypes = [P, P, i64, i64, i64, P, P, i32, P, P, P, P]
    L.nvfp4_grouped_gemm.restype = i32
    L.nvfp4_grouped_gemm.argtypes = [P, P, P, P, P, P, P, i32, i64, i64, i64, P, i32, i32, P, P, P, P]
    L.nvfp4_swiglu_quantize.restype = i32
    L.nvfp4_swiglu_quantize.argtypes = [P, i32, i64, i64, P, i32, P, P, P, i32, P, P, P, P]
    L.nvfp4_kv_quantize.restype = i32
    L.nvfp4_kv_quantize.argtypes = [P, P, i64, i64, i64, i32, P, P, P, P, P, P, P, P, P]
    L.nvfp4_quantize_noalloc.restype = i32
    L.nvfp4_quantize_noalloc.argtypes = [P, i64, i64, i64, P, P, i32, i32, P, P, P, i32, P, P]
    L.nvfp4_moe_route_workspace_size.restype = ctypes.c_size_t
    L.nvfp4_moe_route_workspace_size.argtypes = [i64, i32]
    L.nvfp4_moe_route.restype = i32
    L.nvfp4_moe_route.argtypes = [P, i64, i32, i32, P, P, P, P, P, P]
    L.nvfp4_moe_combine.restype = i32
    L.nvfp4_moe_combine.argtypes = [P, i32, i64, P, P, i64, i32, i64, P, i32, P, P]
    L.nvfp4_kv_dequantize.restype = i32
    L.nvfp4_kv_dequantize.argtypes = [P, P, P, P, P, P, i64, i64, i64, P, P, P]
    L.nvfp4_gemm_set_wait_budget.restype = i32
    L.nvfp4_gemm_set_wait_budget.argtypes = [i64]
    L.nvfp4_e2m1_encode.restype = i32
    L.nvfp4_e2m1_encode.argtypes = [P, i64, P, P]
    L.nvfp4_e4m3_encode.restype = i32
    L.nvfp4_e4m3_encode.argtypes = [P, i64, P, P]
    L.nvfp4_global_scale_from_amax.restype = i32
    L.nvfp4_global_scale_from_amax.argtypes = [P, i64, ctypes.c_float, P, P, P]
    _lib = L
    return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    import torch
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(status: int, what: str):
    if status != OK:
        msg = load_library().nvfp4_status_string(status).decode()
        raise Nvfp4Error(f"{what}: status {status} ({msg})")


def status_string(status: int) -> str:
    return load_library().nvfp4_status_string(status).decode()


def nvfp4_workspace_size(num_groups: int) -> int:
    return int(load_library().nvfp4_workspace_size(num_groups))


def nvfp4_padded_rows_bound(rows: int, num_groups: int) -> int:
    return int(load_library().nvfp4_padded_rows_bound(rows, num_groups))


def nvfp4_quantize(x, rows, K, ld_x, row_index, group_offsets, num_groups, gs_mode, global_scale,
                   q, sf, sf_layout, workspace, dev_status=None, stream=None, check=True) -> int:
    st = load_library().nvfp4_quantize(
        _ptr(x), rows, K, ld_x, _ptr(row_index), _ptr(group_offsets), num_groups, gs_mode,
        _ptr(global_scale), _ptr(q), _ptr(sf), sf_layout, _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_quantize")
    return st


def nvfp4_quantize_noalloc(x, rows, K, ld_x, row_index, group_offsets, num_groups, gs_mode, global_scale,
                           q, sf, sf_layout, dev_status=None, stream=None, check=True) -> int:
    """nvfp4_quantize with the library's own static scratch instead of a workspace
    (for callers that cannot allocate; at most NOALLOC_MAX_GROUPS groups)."""
    st = load_library().nvfp4_quantize_noalloc(
        _ptr(x), rows, K, ld_x, _ptr(row_index), _ptr(group_offsets), num_groups, gs_mode,
        _ptr(global_scale), _ptr(q), _ptr(sf), sf_layout, _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_quantize_noalloc")
    return st


def nvfp4_grouped_gemm_swiglu_nvfp4(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, num_experts, M_total, N, K,
                                    h_gs, h_q, h_sf, workspace=None, dev_status=None, stream=None, check=True) -> int:
    """gate_up GEMM whose SwiGLU epilogue writes NVFP4 h with a given global per expert."""
    st = load_library().nvfp4_grouped_gemm_swiglu_nvfp4(
        _ptr(a_q), _ptr(a_sf), _ptr(a_gs), _ptr(b_q), _ptr(b_sf), _ptr(b_gs), _ptr(expert_offsets), num_experts,
        M_total, N, K, _ptr(h_gs), _ptr(h_q), _ptr(h_sf), _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_grouped_gemm_swiglu_nvfp4")
    return st


def nvfp4_w4a16_workspace_size(M_total: int, num_experts: int, K: int) -> int:
    return int(load_library().nvfp4_w4a16_workspace_size(M_total, num_experts, K))


def nvfp4_grouped_gemm_w4a16(x, ld_x, x_rows, row_index, b_q, b_sf, b_gs, expert_offsets, num_experts, M_total,
                             N, K, y, out_dtype, epi, workspace, dev_status=None, stream=None, check=True) -> int:
    """Weight-only NVFP4 grouped GEMM, bf16 activations (row-major weight scales)."""
    st = load_library().nvfp4_grouped_gemm_w4a16(
        _ptr(x), ld_x, x_rows, _ptr(row_index), _ptr(b_q), _ptr(b_sf), _ptr(b_gs), _ptr(expert_offsets),
        num_experts, M_total, N, K, _ptr(y), out_dtype, epi, _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_grouped_gemm_w4a16")
    return st


def nvfp4_gemm_set_wait_budget(cycles: int) -> int:
    """Main-loop wait budget of the grouped GEMM kernels in SM cycles (0 =
    default): the one-CTA kernels (256- and 512-element stages) and the
    two-block kernel; a switch for testing the timeout path."""
    st = load_library().nvfp4_gemm_set_wait_budget(cycles)
    _check(st, "nvfp4_gemm_set_wait_budget")
    return st


def nvfp4_gemm_select_kernel(mode: int) -> int:
    """Which grouped GEMM kernel runs: 0 automatic (two weight blocks per tile for
    bf16 outputs with N % 256 == 0 and K >= 1024, else one CTA per tile), 1 one
    CTA per tile with 256-element K stages, 2 CTA pairs (N % 256 == 0), 3 the
    64-token ring of the 512-element kernel, 4 two weight blocks per tile
    whenever N % 256 == 0 and the output is bf16."""
    st = load_library().nvfp4_gemm_select_kernel(mode)
    _check(st, "nvfp4_gemm_select_kernel")
    return st


def nvfp4_w4a16_select_kernel(mode: int) -> int:
    """0 automatic, 1 the warp-MMA kernel (small groups), 2 the tcgen05 kernel."""
    st = load_library().nvfp4_w4a16_select_kernel(mode)
    _check(st, "nvfp4_w4a16_select_kernel")
    return st


def nvfp4_moe_quantize(x, tokens, K, ld_x, slot, topk, group_offsets, num_groups, gs_mode, global_scale,
                       q, sf, sf_layout, workspace, dev_status=None, stream=None, check=True) -> int:
    """Routed-expert activation quantize in token order (each token row read once)."""
    st = load_library().nvfp4_moe_quantize(
        _ptr(x), tokens, K, ld_x, _ptr(slot), topk, _ptr(group_offsets), num_groups, gs_mode,
        _ptr(global_scale), _ptr(q), _ptr(sf), sf_layout, _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_moe_quantize")
    return st


def nvfp4_dequantize(q, sf, sf_layout, global_scale, group_offsets, num_groups, rows, K, y, out_dtype,
                     stream=None, check=True) -> int:
    st = load_library().nvfp4_dequantize(
        _ptr(q), _ptr(sf), sf_layout, _ptr(global_scale), _ptr(group_offsets), num_groups, rows, K,
        _ptr(y), out_dtype, _stream(stream))
    if check:
        _check(st, "nvfp4_dequantize")
    return st


def nvfp4_global_scale_from_amax(amax, n, margin, global_scale, dev_status=None, stream=None, check=True) -> int:
    """fp32 amax [n] -> fp32 s_g [n] with the library's global-scale rule (times ``margin``)."""
    st = load_library().nvfp4_global_scale_from_amax(_ptr(amax), n, float(margin), _ptr(global_scale),
                                                     _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_global_scale_from_amax")
    return st


def nvfp4_e2m1_encode(x, n, q, stream=None, check=True) -> int:
    """fp32 [n] -> packed E2M1 codes [n/2] (the quantize kernels' code step)."""
    st = load_library().nvfp4_e2m1_encode(_ptr(x), n, _ptr(q), _stream(stream))
    if check:
        _check(st, "nvfp4_e2m1_encode")
    return st


def nvfp4_e4m3_encode(x, n, out, stream=None, check=True) -> int:
    """fp32 [n] -> E4M3 bytes [n] (the block-scale step)."""
    st = load_library().nvfp4_e4m3_encode(_ptr(x), n, _ptr(out), _stream(stream))
    if check:
        _check(st, "nvfp4_e4m3_encode")
    return st


def mxfp4_to_nvfp4(q_mx, ue8m0, n_tensors, rows, K, q_nv, sf_nv, sf_layout, global_scale, workspace,
                   dev_status=None, stream=None, check=True) -> int:
    st = load_library().mxfp4_to_nvfp4(
        _ptr(q_mx), _ptr(ue8m0), n_tensors, rows, K, _ptr(q_nv), _ptr(sf_nv), sf_layout,
        _ptr(global_scale), _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "mxfp4_to_nvfp4")
    return st


def mxfp4_quantize(x, rows, K, ld_x, q, ue8m0, sf_layout, dev_status=None, stream=None, check=True) -> int:
    st = load_library().mxfp4_quantize(_ptr(x), rows, K, ld_x, _ptr(q), _ptr(ue8m0), sf_layout, _ptr(dev_status),
                                       _stream(stream))
    if check:
        _check(st, "mxfp4_quantize")
    return st


def mxfp4_grouped_gemm(a_q, a_sf, b_q, b_sf, expert_offsets, num_experts, M_total, N, K, y, out_dtype,
                       workspace=None, dev_status=None, stream=None, check=True) -> int:
    st = load_library().mxfp4_grouped_gemm(
        _ptr(a_q), _ptr(a_sf), _ptr(b_q), _ptr(b_sf), _ptr(expert_offsets), num_experts, M_total, N, K, _ptr(y),
        out_dtype, _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "mxfp4_grouped_gemm")
    return st


def nvfp4_grouped_gemm(a_q, a_sf, a_gs, b_q, b_sf, b_gs, expert_offsets, num_experts, M_total, N, K, y,
                       out_dtype, epi=EPI_NONE, amax_out=None, workspace=None, dev_status=None, stream=None,
                       check=True) -> int:
    st = load_library().nvfp4_grouped_gemm(
        _ptr(a_q), _ptr(a_sf), _ptr(a_gs), _ptr(b_q), _ptr(b_sf), _ptr(b_gs), _ptr(expert_offsets),
        num_experts, M_total, N, K, _ptr(y), out_dtype, epi, _ptr(amax_out), _ptr(workspace), _ptr(dev_status),
        _stream(stream))
    if check:
        _check(st, "nvfp4_grouped_gemm")
    return st


def nvfp4_swiglu_quantize(y, y_dtype, rows, I, group_offsets, num_groups, global_scale, q, sf, sf_layout, h,
                          workspace, dev_status=None, stream=None, check=True) -> int:
    st = load_library().nvfp4_swiglu_quantize(
        _ptr(y), y_dtype, rows, I, _ptr(group_offsets), num_groups, _ptr(global_scale), _ptr(q), _ptr(sf),
        sf_layout, _ptr(h), _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_swiglu_quantize")
    return st


def nvfp4_kv_quantize(k, v, tokens, heads, head_dim, gs_mode, k_gs, v_gs, k_q, k_sf, v_q, v_sf, workspace,
                      dev_status=None, stream=None, check=True) -> int:
    st = load_library().nvfp4_kv_quantize(
        _ptr(k), _ptr(v), tokens, heads, head_dim, gs_mode, _ptr(k_gs), _ptr(v_gs), _ptr(k_q), _ptr(k_sf),
        _ptr(v_q), _ptr(v_sf), _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_kv_quantize")
    return st


def nvfp4_kv_dequantize(k_q, k_sf, k_gs, v_q, v_sf, v_gs, tokens, heads, head_dim, k_out, v_out,
                        stream=None, check=True) -> int:
    st = load_library().nvfp4_kv_dequantize(
        _ptr(k_q), _ptr(k_sf), _ptr(k_gs), _ptr(v_q), _ptr(v_sf), _ptr(v_gs), tokens, heads, head_dim,
        _ptr(k_out), _ptr(v_out), _stream(stream))
    if check:
        _check(st, "nvfp4_kv_dequantize")
    return st


def nvfp4_moe_route_workspace_size(tokens: int, num_experts: int) -> int:
    return int(load_library().nvfp4_moe_route_workspace_size(tokens, num_experts))


def nvfp4_moe_route(topk_ids, tokens, topk, num_experts, expert_offsets, row_index, slot, workspace,
                    dev_status=None, stream=None, check=True) -> int:
    st = load_library().nvfp4_moe_route(
        _ptr(topk_ids), tokens, topk, num_experts, _ptr(expert_offsets), _ptr(row_index), _ptr(slot),
        _ptr(workspace), _ptr(dev_status), _stream(stream))
    if check:
        _check(st, "nvfp4_moe_route")
    return st


def nvfp4_moe_combine(y, y_dtype, rows, slot, weights, tokens, topk, H, out, out_dtype, dev_status=None,
                      stream=None, check=True) -> int:
    st = load_library().nvfp4_moe_combine(
        _ptr(y), y_dtype, rows, _ptr(slot), _ptr(weights), tokens, topk, H, _ptr(out), out_dtype, _ptr(dev_status),
        _stream(stream))
    if check:
        _check(st, "nvfp4_moe_combine")
    return st
