"""Device-side twin of the seeded generators (bit-identical to the numpy ones).

Used to create large seeded inputs directly in device memory; the values
equal what ``synthetic.gaussian_bf16`` / ``mxfp4_codes`` / ``mxfp4_exponents``
return on the host for the same (seed, stream, index).
"""
from __future__ import annotations

import ctypes
import os
import subprocess

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gen.cu")
LIB_PATH = os.path.join(_HERE, "libsynth.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB_PATH) or os.path.getmtime(LIB_PATH) < os.path.getmtime(_SRC):
        tmp = LIB_PATH + f".tmp{os.getpid()}"
        subprocess.check_call(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3",
                               "-Xcompiler", "-fPIC", "-shared", "-cudart", "static", _SRC, "-o", tmp])
        os.replace(tmp, LIB_PATH)
    return LIB_PATH


def lib():
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            build()
        L = ctypes.CDLL(LIB_PATH)
        P, i64, u64 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_uint64
        L.synth_normal_bf16.argtypes = [u64, u64, i64, i64, ctypes.c_double, P, P]
        L.synth_words.argtypes = [u64, u64, i64, i64, P, P]
        L.synth_mx_exponents.argtypes = [u64, u64, i64, i64, ctypes.c_int, P, P]
        for f in (L.synth_normal_bf16, L.synth_words, L.synth_mx_exponents):
            f.restype = ctypes.c_int
        _lib = L
    return _lib


def _s():
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def gaussian_bf16(seed, stream, shape, sigma=1.0, start=0, device="cuda"):
    """torch.bfloat16 tensor on the device, same bits as the host generator."""
    import torch
    n = 1
    for s in shape:
        n *= int(s)
    out = torch.empty(tuple(shape), dtype=torch.bfloat16, device=device)
    assert lib().synth_normal_bf16(seed, stream, start, n, float(sigma), ctypes.c_void_p(out.data_ptr()), _s()) == 0
    return out


def mxfp4_codes(seed, stream, nbytes, start_byte=0, device="cuda"):
    import torch
    assert start_byte % 8 == 0
    nw = (nbytes + 7) // 8
    buf = torch.empty(nw * 8, dtype=torch.uint8, device=device)
    assert lib().synth_words(seed, stream, start_byte // 8, nw, ctypes.c_void_p(buf.data_ptr()), _s()) == 0
    return buf[:nbytes]


def mxfp4_exponents(seed, stream, count, lo=-10, start=0, device="cuda"):
    import torch
    out = torch.empty(count, dtype=torch.uint8, device=device)
    assert lib().synth_mx_exponents(seed, stream, start, count, lo, ctypes.c_void_p(out.data_ptr()), _s()) == 0
    return out
