"""Seeded synthetic inputs shared by the tests, the bench and the oracle checks.

This module holds no NVFP4 arithmetic: it only makes input tensors and
routing structures.  Every value is a pure function of (seed, stream, index),
so any slice of any tensor can be regenerated on its own, on the host (numpy,
here) or on the device (``synthetic/gen.cu``), bit for bit.

Generator definition
--------------------
* Words: the SplitMix64 sequence (Steele, Lea & Flood, "Fast splittable
  pseudorandom number generators", OOPSLA 2014).  For a (seed, stream) pair
  the key is ``mix(mix(seed + G) + (stream + 1) * G)`` and word ``i`` is
  ``mix(key + (i + 1) * G)`` with ``G = 0x9E3779B97F4A7C15`` and ``mix`` the
  SplitMix64 finaliser.  All arithmetic is mod 2^64.
* Normal deviates: the Irwin-Hall approximation (sum of twelve uniforms minus
  their mean).  Element ``j`` uses words ``3j, 3j+1, 3j+2``; the twelve 16-bit
  lanes of those words are summed to an integer ``s`` and
  ``z = (s - 393210) / 65536``.  ``z`` has mean 0, variance ~1 and is exact in
  fp64, so host and device agree to the bit.
* bf16 values: ``f = fp32(z * sigma)`` (one fp64 multiply, then one
  round-to-nearest-even to fp32), an optional outlier multiply by 50 done in
  fp32, then round-to-nearest-even to bf16.
* Uniforms (routing only, host only): ``((w >> 11) + 0.5) * 2^-53``.
"""
from __future__ import annotations

import numpy as np

G = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

# Fixed stream ids, one per logical tensor.
STREAMS = {
    "x": 1,
    "w": 2,
    "w_gate_up": 3,
    "w_down": 4,
    "router": 5,
    "outlier_pos": 6,
    "kv_k": 7,
    "kv_v": 8,
    "mx_codes_gate_up": 9,
    "mx_exp_gate_up": 10,
    "mx_codes_down": 11,
    "mx_exp_down": 12,
    "route_gumbel": 13,
    "zipf_rank": 14,
    "x_sweep": 15,
    "mx_codes": 16,
    "mx_exp": 17,
}

_OLD = np.seterr(over="ignore")  # uint64 wrap-around is intended


def _mix(z: np.ndarray) -> np.ndarray:
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, stream: int) -> np.uint64:
    with np.errstate(over="ignore"):
        s = _mix(np.array([seed], dtype=np.uint64) + G)
        k = _mix(s + np.uint64(stream + 1) * G)
    return k[0]


def words(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """SplitMix64 words ``start .. start+count-1`` of (seed, stream)."""
    key = stream_key(seed, stream)
    idx = np.arange(start + 1, start + count + 1, dtype=np.uint64)
    with np.errstate(over="ignore"):
        return _mix(key + idx * G)


def normal_z(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    """Irwin-Hall deviates ``z_j`` for j in [start, start+count), as exact fp64."""
    w = words(seed, stream, 3 * start, 3 * count)
    # the twelve 16-bit lanes of the three words (lane order does not matter for a sum)
    s = w.view(np.uint16).reshape(count, 12).sum(axis=1, dtype=np.int64)
    return (s - 393210).astype(np.float64) / 65536.0


def _normal_z_at(seed: int, stream: int, idx: np.ndarray) -> np.ndarray:
    """``normal_z`` at arbitrary element indices."""
    key = stream_key(seed, stream)
    w_idx = (3 * idx.astype(np.uint64)[:, None] + np.arange(3, dtype=np.uint64)[None, :] + np.uint64(1))
    with np.errstate(over="ignore"):
        w = _mix(key + w_idx * G)
    s = np.ascontiguousarray(w).view(np.uint16).reshape(len(idx), 12).sum(axis=1, dtype=np.int64)
    return (s - 393210).astype(np.float64) / 65536.0


def uniform(seed: int, stream: int, start: int, count: int) -> np.ndarray:
    w = words(seed, stream, start, count)
    return ((w >> np.uint64(11)).astype(np.float64) + 0.5) * (2.0 ** -53)


def f32_to_bf16_bits(f: np.ndarray) -> np.ndarray:
    """Round-to-nearest-even fp32 -> bf16 (finite inputs), as uint16 bits."""
    b = np.ascontiguousarray(f, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (b + np.uint64(0x7FFF) + ((b >> np.uint64(16)) & np.uint64(1))) >> np.uint64(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def outlier_positions(seed: int, numel: int, frac: float = 0.001) -> np.ndarray:
    """Exactly floor(frac*numel) distinct flat positions, without replacement.

    Position i is chosen when its word on the ``outlier_pos`` stream is among
    the smallest; ties are broken by the lower index.
    """
    n_out = int(np.floor(frac * numel))
    if n_out == 0:
        return np.zeros(0, dtype=np.int64)
    w = words(seed, STREAMS["outlier_pos"], 0, numel)
    thr = np.partition(w, n_out - 1)[n_out - 1]        # the n_out-th smallest word
    cand = np.nonzero(w <= thr)[0]                      # ascending index
    order = cand[np.argsort(w[cand], kind="stable")]    # by word, then lower index
    return np.sort(order[:n_out]).astype(np.int64)


_HG = None


def _hostgen():
    """The C twin of ``normal_z`` + bf16 rounding (hostgen.c), built on first use."""
    global _HG
    if _HG is None:
        import ctypes
        import os
        import subprocess
        here = os.path.dirname(os.path.abspath(__file__))
        src, so = os.path.join(here, "hostgen.c"), os.path.join(here, "libhostgen.so")
        if not os.path.exists(so) or os.path.getmtime(so) < os.path.getmtime(src):
            tmp = so + f".tmp{os.getpid()}"
            subprocess.check_call(["gcc", "-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", src,
                                   "-o", tmp])
            os.replace(tmp, so)
        L = ctypes.CDLL(so)
        L.hg_normal_bf16.restype = None
        L.hg_normal_bf16.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_int64, ctypes.c_int64,
                                     ctypes.c_double, ctypes.c_int, ctypes.c_void_p]
        _HG = L
    return _HG


def gaussian_bf16_bits_fast(seed: int, stream: int, start: int, n: int, sigma: float) -> np.ndarray:
    out = np.empty(n, dtype=np.uint16)
    _hostgen().hg_normal_bf16(seed, stream, start, n, float(sigma), int(sigma != 1.0),
                              out.ctypes.data_as(__import__("ctypes").c_void_p))
    return out


def gaussian_bf16(seed: int, stream: int, shape, sigma: float = 1.0,
                  outlier_frac: float = 0.0, outlier_mult: float = 50.0,
                  start: int = 0, reference: bool = False) -> np.ndarray:
    """bf16 bits (uint16) of N(0, sigma^2) deviates, optional outliers.

    ``start`` offsets the flat element index, so a slice of a large tensor
    can be regenerated alone.  Outliers are defined over the tensor starting
    at index 0 and are not supported together with ``start``.  Large tensors
    go through the C twin (same bits); ``reference=True`` forces numpy.
    """
    shape = tuple(int(s) for s in shape)
    n = int(np.prod(shape)) if shape else 1
    if not reference and n >= (1 << 16):
        bits = gaussian_bf16_bits_fast(seed, stream, start, n, sigma)
        if outlier_frac > 0.0:
            assert start == 0
            pos = outlier_positions(seed, n, outlier_frac)
            zp = np.concatenate([normal_z(seed, stream, int(p), 1) for p in pos]) if len(pos) < 64 else \
                _normal_z_at(seed, stream, pos)
            fp = (zp * float(sigma)).astype(np.float32) if sigma != 1.0 else zp.astype(np.float32)
            bits[pos] = f32_to_bf16_bits((fp * np.float32(outlier_mult)).astype(np.float32))
        return bits.reshape(shape)
    z = normal_z(seed, stream, start, n)
    f = (z * float(sigma)).astype(np.float32) if sigma != 1.0 else z.astype(np.float32)
    if outlier_frac > 0.0:
        assert start == 0
        pos = outlier_positions(seed, n, outlier_frac)
        f[pos] = (f[pos] * np.float32(outlier_mult)).astype(np.float32)
    return f32_to_bf16_bits(f).reshape(shape)


# --------------------------------------------------------------------------
# Routing structures (inputs to the grouped path; the router is not part of it)
# --------------------------------------------------------------------------

def _group_by_expert(experts: np.ndarray, num_experts: int):
    """experts: int [T, topk].  Returns (row_index [R], offsets [E+1], slot [T, topk]).

    Rows of expert e are the tokens that selected e, in ascending token id.
    ``slot[t, k]`` is the permuted row that holds token t's k-th choice.
    """
    T, topk = experts.shape
    flat_e = experts.reshape(-1).astype(np.int64)
    flat_t = np.repeat(np.arange(T, dtype=np.int64), topk)
    order = np.lexsort((flat_t, flat_e))  # by expert, then token id
    row_index = flat_t[order].astype(np.int32)
    counts = np.bincount(flat_e, minlength=num_experts)
    offsets = np.zeros(num_experts + 1, dtype=np.int32)
    offsets[1:] = np.cumsum(counts)
    slot = np.empty(T * topk, dtype=np.int64)
    slot[order] = np.arange(T * topk)
    return row_index, offsets, slot.reshape(T, topk)


def route_topk_softmax(seed: int, tokens: int, num_experts: int, topk: int):
    """Router logits ~ N(0,1) per (token, expert); top-k by logit, lower index wins ties.

    Returns dict(row_index, offsets, experts [T,k], weights [T,k] (softmax over
    the chosen logits), slot [T,k]).
    """
    z = normal_z(seed, STREAMS["router"], 0, tokens * num_experts).reshape(tokens, num_experts)
    experts = np.argsort(-z, axis=1, kind="stable")[:, :topk]
    chosen = np.take_along_axis(z, experts, axis=1)
    e = np.exp(chosen - chosen.max(axis=1, keepdims=True))
    weights = e / e.sum(axis=1, keepdims=True)
    row_index, offsets, slot = _group_by_expert(experts, num_experts)
    return dict(row_index=row_index, offsets=offsets, experts=experts,
                weights=weights, slot=slot)


def route_zipf_gumbel(seed: int, tokens: int, num_experts: int, topk: int, s: float = 1.1):
    """Skewed decode routing: expert popularity Zipf(s) over a seeded random rank
    permutation; each token draws ``topk`` distinct experts by weighted sampling
    without replacement (Gumbel-top-k)."""
    rank_words = words(seed, STREAMS["zipf_rank"], 0, num_experts)
    rank_of_expert = np.empty(num_experts, dtype=np.int64)
    rank_of_expert[np.argsort(rank_words, kind="stable")] = np.arange(num_experts)
    p = 1.0 / np.power(rank_of_expert + 1.0, s)
    p = p / p.sum()
    u = uniform(seed, STREAMS["route_gumbel"], 0, tokens * num_experts).reshape(tokens, num_experts)
    keys = np.log(p)[None, :] - np.log(-np.log(u))
    experts = np.argsort(-keys, axis=1, kind="stable")[:, :topk]
    w = np.take_along_axis(p[None, :].repeat(tokens, 0), experts, axis=1)
    weights = w / w.sum(axis=1, keepdims=True)
    row_index, offsets, slot = _group_by_expert(experts, num_experts)
    return dict(row_index=row_index, offsets=offsets, experts=experts,
                weights=weights, slot=slot, popularity=p)


# --------------------------------------------------------------------------
# MXFP4 weights (32-element blocks, UE8M0 exponents)
# --------------------------------------------------------------------------

def mxfp4_codes(seed: int, stream: int, nbytes: int, start_byte: int = 0) -> np.ndarray:
    """Packed E2M1 codes, uniform over all 16 codes: byte b is byte (b % 8) of word b // 8."""
    assert start_byte % 8 == 0
    nw = (nbytes + 7) // 8
    w = words(seed, stream, start_byte // 8, nw)
    return w.view(np.uint8)[:nbytes].copy()


def mxfp4_exponents(seed: int, stream: int, count: int, lo: int = -10, start: int = 0) -> np.ndarray:
    """UE8M0 bytes 127 + e with e uniform in [lo, lo+7]: ``127 + lo + (w >> 61)``."""
    w = words(seed, stream, start, count)
    return (127 + lo + (w >> np.uint64(61)).astype(np.int64)).astype(np.uint8)


def padded_rows(offsets: np.ndarray, align: int = 128) -> np.ndarray:
    """Start row of each group's slot when every group is padded to ``align`` rows."""
    counts = np.diff(offsets.astype(np.int64))
    padded = (counts + align - 1) // align * align
    starts = np.zeros(len(counts) + 1, dtype=np.int64)
    starts[1:] = np.cumsum(padded)
    return starts
