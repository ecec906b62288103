"""NVFP4 oracle -- TEST INFRASTRUCTURE ONLY.

Plain CPU reference for the NVFP4 W4A4 path: E2M1 / E4M3 codecs, quantize,
dequantize, the MXFP4 encoder and the MXFP4 -> NVFP4 remap, SwiGLU and an fp64 GEMM of dequantized
operands.  The arithmetic lives in ``oracle.c`` (scalar C, no FMA
contraction, no fast-math); this module only loads it and adds the fp64
matrix products, for which ``numpy.matmul`` in float64 is the library step.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` use this package.  It shares no code with the CUDA library and
never imports it.

Every function cites the page passage it follows (page title and section):
  P1 = "Qwen3.8-Flash-Next-NVFP4" (lpnh.cn/news/2736522), the two-level
       scaling section; P2 = "DeepSeek-V4.1-Flash-NVFP4" (kwkr.cn/news/613851),
       the format section; P3 = "Qwen3.8-2.4T-A95B-NVFP4" (hnwysp.cn/news/107543),
       the NVFP4 KV cache section.

Parity pins: every function here is checked against something other than
itself in ``tests/test_oracle_pins.py`` (printed tables, a library codec,
closed forms, brute force).  None is "parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lib = None
_lock = threading.Lock()

OK = 0
ERR_NONFINITE = 16
ERR_NOT_REPRESENTABLE = 17


def build(force: bool = False) -> str:
    """Compile oracle.c to liboracle.so (plain C, OpenMP over rows)."""
    if force or not os.path.exists(_LIB_PATH) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC):
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call([
            "gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
            "-ffp-contract=off", "-fno-fast-math", "-Wall", "-Wno-unknown-pragmas",
            _SRC, "-o", tmp, "-lm",
        ])
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB_PATH)
            P = ctypes.c_void_p
            i64 = ctypes.c_int64
            L.orc_e2m1_decode.restype = ctypes.c_double
            L.orc_e2m1_decode.argtypes = [ctypes.c_uint8]
            L.orc_e2m1_encode.restype = ctypes.c_uint8
            L.orc_e2m1_encode.argtypes = [ctypes.c_float]
            L.orc_e4m3_decode.restype = ctypes.c_double
            L.orc_e4m3_decode.argtypes = [ctypes.c_uint8]
            L.orc_e4m3_encode.restype = ctypes.c_uint8
            L.orc_e4m3_encode.argtypes = [ctypes.c_float]
            L.orc_global_scale_from_amax.restype = ctypes.c_float
            L.orc_global_scale_from_amax.argtypes = [ctypes.c_float]
            L.orc_block_scale.restype = ctypes.c_uint8
            L.orc_block_scale.argtypes = [ctypes.c_float, ctypes.c_float]
            L.orc_encode_block.restype = None
            L.orc_encode_block.argtypes = [P, ctypes.c_uint8, ctypes.c_float, P]
            L.orc_quantize.restype = ctypes.c_int
            L.orc_quantize.argtypes = [P, i64, i64, i64, P, P, ctypes.c_int, ctypes.c_int, P, P, P]
            L.orc_dequantize.restype = None
            L.orc_dequantize.argtypes = [P, P, P, i64, i64, P, P]
            L.orc_dequantize_f64.restype = None
            L.orc_dequantize_f64.argtypes = [P, P, P, i64, i64, P]
            L.orc_remap_mxfp4.restype = ctypes.c_int
            L.orc_remap_mxfp4.argtypes = [P, P, i64, i64, i64, P, P, P]
            L.orc_quantize_mxfp4.restype = ctypes.c_int
            L.orc_quantize_mxfp4.argtypes = [P, i64, i64, i64, P, P]
            L.orc_dequantize_mxfp4_f64.restype = None
            L.orc_dequantize_mxfp4_f64.argtypes = [P, P, i64, i64, P]
            L.orc_swiglu.restype = None
            L.orc_swiglu.argtypes = [P, i64, i64, P]
            L.orc_dot_f64.restype = None
            L.orc_dot_f64.argtypes = [P, P, i64, P, P]
            L.orc_route.restype = ctypes.c_int
            L.orc_route.argtypes = [P, i64, ctypes.c_int, ctypes.c_int, P, P, P]
            L.orc_combine.restype = None
            L.orc_combine.argtypes = [P, P, P, i64, ctypes.c_int, i64, P, P]
            for name in ("orc_e2m1_encode_array", "orc_e4m3_encode_array"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [P, i64, P]
            for name in ("orc_e2m1_encode_bits_range", "orc_e4m3_encode_bits_range"):
                getattr(L, name).restype = None
                getattr(L, name).argtypes = [ctypes.c_uint64, ctypes.c_uint64, P]
            _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


# ---------------------------------------------------------------- codecs
def e2m1_decode(code: int) -> float:
    """E2M1 value of a 4-bit code (P2, format section: FP4_TABLE)."""
    return lib().orc_e2m1_decode(code)


def e2m1_encode(v: float) -> int:
    """Round-to-nearest-even E2M1 code of an fp32 value, saturating at 6 (P2 format section)."""
    return lib().orc_e2m1_encode(v)


def e4m3_decode(code: int) -> float:
    """Value of an FP8 E4M3 byte (P1 two-level scaling: scale_bits [4,3])."""
    return lib().orc_e4m3_decode(code)


def e4m3_encode(v: float) -> int:
    """Round-to-nearest-even E4M3 byte, saturating to 448 (P1: max scale 448.0)."""
    return lib().orc_e4m3_encode(v)


def e2m1_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e2m1_encode_array(_p(v), v.size, _p(out))
    return out


def e4m3_encode_array(v: np.ndarray) -> np.ndarray:
    v = np.ascontiguousarray(v, dtype=np.float32)
    out = np.empty(v.shape, dtype=np.uint8)
    lib().orc_e4m3_encode_array(_p(v), v.size, _p(out))
    return out


def e2m1_encode_bits_range(lo: int, hi: int) -> np.ndarray:
    out = np.empty(hi - lo, dtype=np.uint8)
    lib().orc_e2m1_encode_bits_range(lo, hi, _p(out))
    return out


def e4m3_encode_bits_range(lo: int, hi: int) -> np.ndarray:
    out = np.empty(hi - lo, dtype=np.uint8)
    lib().orc_e4m3_encode_bits_range(lo, hi, _p(out))
    return out


def global_scale_from_amax(amax: float) -> float:
    """s_g = amax / (6*448), the block holding the amax gets scale 448 (P1 scale audit)."""
    return lib().orc_global_scale_from_amax(amax)


def block_scale(a_b: float, s_g: float) -> int:
    """E4M3 block scale of a 16-block with amax a_b (P1 level-1 block scale)."""
    return lib().orc_block_scale(a_b, s_g)


def encode_block(x16: np.ndarray, S: int, s_g: float) -> np.ndarray:
    """Packed codes of one 16-element block for a given scale byte (P1 + P2)."""
    x16 = np.ascontiguousarray(x16, dtype=np.float32)
    assert x16.size == 16
    out = np.empty(8, dtype=np.uint8)
    lib().orc_encode_block(_p(x16), S, s_g, _p(out))
    return out


# ---------------------------------------------------------------- tensors
def quantize(x_bf16: np.ndarray, row_index=None, group_offsets=None, global_scale=None):
    """NVFP4-quantize bf16 rows (P1 two-level scaling; P2 format and packing).

    x_bf16: uint16 bf16 bits [rows_x, K].  row_index: optional int32 [R]
    gather (row r of the result is x[row_index[r]]).  group_offsets: optional
    int32 [G+1] prefix sums over result rows, one global scale per group.
    global_scale: None (computed from the amax) or fp32 [G] given scales.
    Returns (q [R, K/2] uint8, sf [R, K/16] uint8 row-major, gs [G] fp32, status).
    """
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    K = x.shape[1]
    assert K % 16 == 0
    ri = None if row_index is None else np.ascontiguousarray(row_index, dtype=np.int32)
    R = x.shape[0] if ri is None else ri.shape[0]
    go = None if group_offsets is None else np.ascontiguousarray(group_offsets, dtype=np.int32)
    G = 1 if go is None else go.shape[0] - 1
    if global_scale is None:
        gs = np.zeros(max(G, 1), dtype=np.float32)
        given = 0
    else:
        gs = np.ascontiguousarray(global_scale, dtype=np.float32).copy()
        given = 1
    q = np.zeros((R, K // 2), dtype=np.uint8)
    sf = np.zeros((R, K // 16), dtype=np.uint8)
    st = lib().orc_quantize(_p(x), R, K, K, _p(ri), _p(go), G, given, _p(gs), _p(q), _p(sf))
    return q, sf, gs, st


def rows_global_scale(gs: np.ndarray, group_offsets, rows: int) -> np.ndarray:
    """Expand per-group global scales to one per row."""
    gs = np.asarray(gs, dtype=np.float32)
    if group_offsets is None:
        return np.full(rows, gs[0], dtype=np.float32)
    counts = np.diff(np.asarray(group_offsets, dtype=np.int64))
    return np.repeat(gs, counts).astype(np.float32)


def dequantize(q: np.ndarray, sf: np.ndarray, row_gs: np.ndarray, out="f32"):
    """x_hat = (code * S) * s_g in fp32; bf16 = RNE of it (P1: dequantize with the scales)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    g = np.ascontiguousarray(row_gs, dtype=np.float32)
    R, K = q.shape[0], q.shape[1] * 2
    if out == "f32":
        y = np.empty((R, K), dtype=np.float32)
        lib().orc_dequantize(_p(q), _p(sf), _p(g), R, K, _p(y), None)
    else:
        y = np.empty((R, K), dtype=np.uint16)
        lib().orc_dequantize(_p(q), _p(sf), _p(g), R, K, None, _p(y))
    return y


def dequantize_f64(q: np.ndarray, sf: np.ndarray, row_gs: np.ndarray) -> np.ndarray:
    """Exact fp64 value code * S * s_g of every element (the GEMM operands)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    sf = np.ascontiguousarray(sf, dtype=np.uint8)
    g = np.ascontiguousarray(row_gs, dtype=np.float32)
    R, K = q.shape[0], q.shape[1] * 2
    y = np.empty((R, K), dtype=np.float64)
    lib().orc_dequantize_f64(_p(q), _p(sf), _p(g), R, K, _p(y))
    return y


def remap_mxfp4(q_mx: np.ndarray, e8: np.ndarray, n_tensors: int, rows: int, K: int):
    """Lossless MXFP4 -> NVFP4 remap (P2 format table and the remap passage).

    q_mx: uint8 [n_tensors*rows, K/2]; e8: uint8 UE8M0 [n_tensors*rows, K/32].
    Returns (q_nv, sf_nv [n*rows, K/16], gs [n], status).
    """
    q_mx = np.ascontiguousarray(q_mx, dtype=np.uint8)
    e8 = np.ascontiguousarray(e8, dtype=np.uint8)
    q_nv = np.empty_like(q_mx)
    sf = np.empty((n_tensors * rows, K // 16), dtype=np.uint8)
    gs = np.empty(n_tensors, dtype=np.float32)
    st = lib().orc_remap_mxfp4(_p(q_mx), _p(e8), n_tensors, rows, K, _p(q_nv), _p(sf), _p(gs))
    return q_nv, sf, gs, st


def quantize_mxfp4(x_bf16: np.ndarray):
    """MXFP4 encode of a bf16 matrix [rows, K] (P2, the FP8 -> MXFP4 step of
    the which-layers section; rule read as the OCP MX v1.0 conversion, see
    ``orc_quantize_mxfp4``).  Returns (q uint8 [rows, K/2], e8 uint8 UE8M0
    [rows, K/32], status)."""
    x = np.ascontiguousarray(x_bf16, dtype=np.uint16)
    R, K = x.shape
    if K % 32:
        raise ValueError("K must be a multiple of 32")
    q = np.empty((R, K // 2), dtype=np.uint8)
    e8 = np.empty((R, K // 32), dtype=np.uint8)
    st = lib().orc_quantize_mxfp4(_p(x), R, K, K, _p(q), _p(e8))
    return q, e8, st


def dequantize_mxfp4_f64(q: np.ndarray, e8: np.ndarray) -> np.ndarray:
    """fp64 value code * 2^(u-127) of an MXFP4 tensor (P2 format table)."""
    q = np.ascontiguousarray(q, dtype=np.uint8)
    e8 = np.ascontiguousarray(e8, dtype=np.uint8)
    R, K = q.shape[0], q.shape[1] * 2
    y = np.empty((R, K), dtype=np.float64)
    lib().orc_dequantize_mxfp4_f64(_p(q), _p(e8), R, K, _p(y))
    return y


def swiglu(y: np.ndarray) -> np.ndarray:
    """h = bf16(silu(g) * u) with g = y[:, :I], u = y[:, I:] (gate rows first)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    R, I2 = y.shape
    h = np.empty((R, I2 // 2), dtype=np.uint16)
    lib().orc_swiglu(_p(y), R, I2 // 2, _p(h))
    return h


def gemm_f64(a_dq: np.ndarray, b_dq: np.ndarray):
    """y = A @ B^T and s = |A| @ |B|^T in fp64 (the GEMM of P2's native FP4 path,
    on the exact dequantized operands).  numpy.matmul in float64 is the library step."""
    a = np.asarray(a_dq, dtype=np.float64)
    b = np.asarray(b_dq, dtype=np.float64)
    return a @ b.T, np.abs(a) @ np.abs(b).T


def grouped_gemm_f64(a_dq: np.ndarray, b_dq_experts, offsets: np.ndarray):
    """Per expert e: Y[offsets[e]:offsets[e+1]] = A_e @ B_e^T (fp64), plus sum |a*b|.

    a_dq: fp64 [R, K] gathered rows; b_dq_experts: callable e -> fp64 [N, K]
    (or an array [E, N, K]).
    """
    offsets = np.asarray(offsets, dtype=np.int64)
    E = len(offsets) - 1
    get = b_dq_experts if callable(b_dq_experts) else (lambda e: b_dq_experts[e])
    N = None
    ys, ss = [], []
    for e in range(E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 == r0:
            continue
        b = get(e)
        N = b.shape[0]
        y, s = gemm_f64(a_dq[r0:r1], b)
        ys.append((r0, y))
        ss.append((r0, s))
    R = offsets[-1]
    Y = np.zeros((R, N if N is not None else 0))
    S = np.zeros_like(Y)
    for (r0, y), (_, s) in zip(ys, ss):
        Y[r0:r0 + y.shape[0]] = y
        S[r0:r0 + s.shape[0]] = s
    return Y, S


def dot_f64(a: np.ndarray, b: np.ndarray):
    """One output element: (sum a*b, sum |a*b|) in fp64, by a plain loop."""
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    y = ctypes.c_double()
    s = ctypes.c_double()
    lib().orc_dot_f64(_p(a), _p(b), a.size, ctypes.byref(y), ctypes.byref(s))
    return y.value, s.value


# ---------------------------------------------------------------- MoE plumbing
def route(expert_ids: np.ndarray, num_experts: int):
    """Group (token, choice) pairs by expert, tokens ascending inside a group
    (the routed-row order the grouped GEMM consumes; P1: top-10 routing).
    expert_ids: int32 [T, k].  A choice with an id outside [0, E) is dropped:
    slot -1, not counted in the offsets, no routed row.
    Returns (offsets [E+1], row_index [offsets[E]], slot [T, k], status) with
    status 0, 1 (some choice dropped) or 2 (no routing: E or k <= 0)."""
    ids = np.ascontiguousarray(expert_ids, dtype=np.int32)
    T, k = ids.shape
    off = np.zeros(max(num_experts, 0) + 1, np.int32)
    ri = np.full(T * k, -1, np.int32)
    slot = np.full((T, k), -1, np.int32)
    st = lib().orc_route(_p(ids), T, k, num_experts, _p(off), _p(ri), _p(slot))
    return off, ri[:int(off[-1])], slot, st


def combine(y: np.ndarray, slot: np.ndarray, weights: np.ndarray):
    """out[t] = sum_j w[t,j] * y[slot[t,j]] in fp64, and sum |w*y| (the weighted
    sum of the k expert outputs of each token)."""
    y = np.ascontiguousarray(y, dtype=np.float32)
    slot = np.ascontiguousarray(slot, dtype=np.int32)
    w = np.ascontiguousarray(weights, dtype=np.float32)
    T, k = slot.shape
    H = y.shape[1]
    out = np.empty((T, H), np.float64)
    sabs = np.empty((T, H), np.float64)
    lib().orc_combine(_p(y), _p(slot), _p(w), T, k, H, _p(out), _p(sabs))
    return out, sabs
