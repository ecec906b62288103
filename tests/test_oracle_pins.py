"""Pins of the oracle to things other than itself (CPU only).

Each test names what fixes the expected value: a table or number the pages
print (fixtures under tests/golden/), a library codec (ml_dtypes), a closed
form, or brute force over a small domain.
"""
import math
import os

import ml_dtypes
import numpy as np
import pytest

import oracle
import synthetic

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden_kv(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        k, v = line.split()
        out[k] = float(v)
    return out


FACTS = _golden_kv("nvfp4_format_facts.txt")


def _e2m1_table():
    rows = [l.split() for l in open(os.path.join(GOLDEN, "e2m1_magnitudes.txt"))
            if l.strip() and not l.startswith("#")]
    return {int(c): float(m) for c, m in rows}


# ------------------------------------------------------------------ E2M1
def test_e2m1_decode_matches_printed_table():
    table = _e2m1_table()
    assert len(table) == 8
    for c in range(8):
        assert oracle.e2m1_decode(c) == table[c]
        neg = oracle.e2m1_decode(c | 8)
        assert neg == -table[c] and math.copysign(1.0, neg) == -1.0


def test_e2m1_decode_matches_library():
    codes = np.arange(16, dtype=np.uint8).view(ml_dtypes.float4_e2m1fn)
    lib_vals = codes.astype(np.float64)
    for c in range(16):
        assert oracle.e2m1_decode(c) == lib_vals[c]


def _e2m1_bruteforce_nearest(v: np.ndarray) -> np.ndarray:
    """Independent encoder: nearest of the 15 signed grid values by distance;
    on a tie the candidate whose mantissa bit is 0 wins; beyond 6 saturate."""
    table = _e2m1_table()
    mags = np.array([table[c] for c in range(8)])
    a = np.abs(v.astype(np.float64))
    d = np.abs(a[:, None] - mags[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = (np.arange(8) % 2 == 0)[None, :]
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    mag = np.where(has_even, np.argmax(pick_even, axis=1), np.argmax(cand, axis=1))
    sign = np.signbit(v).astype(np.uint8) * 8
    return (sign | mag).astype(np.uint8)


def test_e2m1_encode_bruteforce_dense_and_midpoints():
    # every midpoint and grid point, one ulp either side, both signs
    pts = [0.0, 0.25, 0.5, 0.75, 1.0, 1.25, 1.5, 1.75, 2.0, 2.5, 3.0, 3.5, 4.0, 5.0, 6.0, 7.0]
    vals = []
    for p in pts:
        f = np.float32(p)
        vals += [f, np.nextafter(f, np.float32(np.inf)), np.nextafter(f, np.float32(-np.inf))]
    rng = np.random.default_rng(0)
    vals = np.concatenate([np.array(vals, dtype=np.float32),
                           rng.uniform(-8, 8, 2_000_000).astype(np.float32),
                           (rng.standard_normal(200_000) * 1e-3).astype(np.float32)])
    vals = np.concatenate([vals, -vals])
    got = oracle.e2m1_encode_array(vals)
    want = _e2m1_bruteforce_nearest(vals)
    assert np.array_equal(got, want)


def test_e2m1_encode_saturation_and_specials():
    assert oracle.e2m1_encode(float("inf")) == 7
    assert oracle.e2m1_encode(float("-inf")) == 15
    assert oracle.e2m1_encode(1e30) == 7
    assert oracle.e2m1_encode(float("nan")) == 0           # reading: NaN -> +0
    assert oracle.e2m1_encode(-0.0) == 8 and oracle.e2m1_encode(-0.1) == 8


def _exhaustive(encode_range, lib_encode, lib_hi, sat_code, nan_code):
    """Walk all 2^32 fp32 bit patterns.  Positive patterns below ``lib_hi``
    are compared with the library codec; positive finite patterns above it
    must saturate; each negative pattern must be its positive twin with the
    sign bit set; NaN patterns follow the reading ``nan_code``."""
    chunk = 1 << 25
    inf = 0x7F800000
    for lo in range(0, 1 << 31, chunk):
        hi = lo + chunk
        pos = encode_range(lo, hi)
        neg = encode_range(lo + 0x80000000, hi + 0x80000000)
        bits = np.arange(lo, hi, dtype=np.uint64)
        n_lib = int(max(0, min(hi, lib_hi) - lo))
        if n_lib:
            f = bits[:n_lib].astype(np.uint32).view(np.float32)
            assert np.array_equal(pos[:n_lib], lib_encode(f)), hex(lo)
        fin = (bits >= lib_hi) & (bits <= inf)
        assert (pos[fin] == sat_code).all(), hex(lo)
        nan = bits > inf
        assert (pos[nan] == nan_code).all() and (neg[nan] == nan_code).all()
        sign = 0x80 if sat_code == 0x7E else 0x08
        assert np.array_equal(neg[~nan], pos[~nan] | sign), hex(lo)


@pytest.mark.slow
def test_e2m1_encode_exhaustive_vs_library():
    """All 2^32 fp32 patterns; the library decides every |v| < 8 (all the
    rounding decisions); NaN -> +0 is the reading."""
    lib_hi = int(np.float32(8.0).view(np.uint32))
    _exhaustive(oracle.e2m1_encode_bits_range,
                lambda f: f.astype(ml_dtypes.float4_e2m1fn).view(np.uint8),
                lib_hi, 7, 0)


# ------------------------------------------------------------------ E4M3
def test_e4m3_decode_all_codes_vs_library_and_max():
    lib = np.arange(256, dtype=np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    for c in range(256):
        v = oracle.e4m3_decode(c)
        if np.isnan(lib[c]):
            assert math.isnan(v)
        else:
            assert v == lib[c], c
    finite = [oracle.e4m3_decode(c) for c in range(128) if not math.isnan(oracle.e4m3_decode(c))]
    assert max(finite) == FACTS["max_block_scale"]
    assert len(finite) == 127      # 0 plus 126 positive values
    # the bit split printed as scale_bits [4,3]: 4 exponent + 3 mantissa bits, bias 7
    assert FACTS["scale_exponent_bits"] == 4 and FACTS["scale_mantissa_bits"] == 3
    assert oracle.e4m3_decode(0x38) == 1.0 and oracle.e4m3_decode(0x01) == 2.0 ** -9


@pytest.mark.slow
def test_e4m3_encode_exhaustive_vs_library():
    """All 2^32 fp32 patterns: the library's RNE decides every |v| < 464
    (the midpoint above 448); beyond it the satfinite reading gives 448."""
    lib_hi = int(np.float32(464.0).view(np.uint32))
    _exhaustive(oracle.e4m3_encode_bits_range,
                lambda f: f.astype(ml_dtypes.float8_e4m3fn).view(np.uint8),
                lib_hi, 0x7E, 0x7F)


def test_e4m3_encode_nearest_bruteforce_sample():
    vals = np.array([oracle.e4m3_decode(c) for c in range(0x7F)])
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(0, 460, 200_000), rng.uniform(0, 2 ** -6, 100_000),
                        (vals[:-1] + vals[1:]) / 2]).astype(np.float32)
    got = oracle.e4m3_encode_array(x)
    d = np.abs(x.astype(np.float64)[:, None] - vals[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    even = (np.arange(0x7F) % 2 == 0)[None, :]
    pe = cand & even
    want = np.where(pe.any(axis=1), np.argmax(pe, axis=1), np.argmax(cand, axis=1))
    assert np.array_equal(got, want.astype(np.uint8))


# ------------------------------------------------------- brute force 16 x 256
@pytest.mark.parametrize("s_g", [1.0, 2.0 ** -7, 0.0371])
def test_block_roundtrip_every_code_every_scale(s_g):
    """For every finite positive E4M3 scale S and all 16 codes, quantizing the
    block {decode(c) * S * s_g} with the scale forced to S returns c."""
    s_g = float(np.float32(s_g))
    codes = np.arange(16)
    for S in range(1, 0x7F):
        Sv = oracle.e4m3_decode(S)
        x = np.array([oracle.e2m1_decode(c) * Sv * s_g for c in codes]).astype(np.float32)
        out = oracle.encode_block(x, S, s_g)
        got = np.empty(16, dtype=np.int64)
        got[0::2] = out & 15
        got[1::2] = out >> 4
        assert np.array_equal(got, codes), (S, s_g)


# ------------------------------------------------------- quantize invariants
def _quant(x, **kw):
    q, sf, gs, st = oracle.quantize(x, **kw)
    assert st == oracle.OK
    return q, sf, gs


def test_effective_bits_is_4_5():
    x = synthetic.gaussian_bf16(0, 1, (128, 512), outlier_frac=0.001)
    q, sf, gs = _quant(x)
    bits = 8 * (q.nbytes + sf.nbytes) / x.size
    assert bits == FACTS["effective_bits"] == (16 * 4 + 8) / 16


@pytest.mark.parametrize("shape,sigma,outl", [((128, 512), 1.0, 0.001), ((256, 512), 0.02, 0.0),
                                              ((64, 4096), 1.0, 0.0)])
def test_scale_audit_invariants(shape, sigma, outl):
    """P1 scale audit: every scale finite and positive, the largest 448."""
    x = synthetic.gaussian_bf16(3, 1, shape, sigma=sigma, outlier_frac=outl)
    q, sf, gs = _quant(x)
    xf = synthetic.bf16_bits_to_f32(x)
    A = float(np.abs(xf).max())
    assert gs[0] == np.float32(A) / np.float32(2688.0)
    assert ((sf & 0x7F) != 0x7F).all()            # no NaN code
    assert (sf <= 0x7E).all()                     # non-negative, <= 448
    assert sf.max() == 0x7E                       # the amax block gets 448
    ab = np.abs(xf).reshape(shape[0], -1, 16).max(axis=2)
    big = ab * 448.0 / A >= 2.0 ** -10
    assert (sf[big] > 0).all()


def _wide_range_blocks(seed, rows, K):
    """N(0,1) rows whose 16-element blocks are each scaled by their own power
    of two 2^-26 .. 2^3, plus a few all-zero blocks: beside the normal E4M3
    block scales this reaches every subnormal scale and the zero scale."""
    x = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(seed, 1, (rows, K))).reshape(rows, K // 16, 16)
    rng = np.random.default_rng(seed)
    p = rng.integers(-26, 4, size=(rows, K // 16, 1)).astype(np.float32)
    x = x * np.exp2(p)
    x[rng.random((rows, K // 16)) < 0.01] = 0.0
    return synthetic.f32_to_bf16_bits(x.reshape(rows, K).astype(np.float32))


@pytest.mark.parametrize("case", ["gauss_outliers", "weights", "wide_range"])
def test_block_scale_pulls_each_group_into_pm6(case):
    """The page's rule for the block scale: it maps the group's values back into
    [-6, 6], i.e. the group's largest |x| lands on 6, the top of the E2M1 grid
    (golden fact block_scale_target_magnitude).  With S an E4M3 value:
      - S normal: S is within half an E4M3 step of the exact quotient, at
        most 2^-4 of S (the bound is reached just below 2^-6, where the
        subnormal grid's step equals the lowest binade's), so
        max|x| / (S s_g) lies in [6 (1-2^-4), 6 (1+2^-4)] = [5.625, 6.375] and
        the block's largest code is +-6 (code 7);
      - S = m 2^-9 subnormal (m = 1..7): S is within 2^-10 of the quotient, so
        max|x| / (S s_g) lies in [6 (m - 1/2)/m, 6 (m + 1/2)/m] and the largest
        code is at least the library's E2M1 rounding of the lower end;
      - S = 0: the quotient is at most 2^-10 and every code is +-0.
    A divisor other than 6 (or a product where the rule divides) fails the
    normal-scale interval on every block but the amax one."""
    top = FACTS["block_scale_target_magnitude"]
    if case == "gauss_outliers":
        x = synthetic.gaussian_bf16(11, 1, (256, 1024), outlier_frac=0.001)
    elif case == "weights":
        x = synthetic.gaussian_bf16(12, 2, (512, 512), sigma=0.02)
    else:
        x = _wide_range_blocks(13, 256, 1024)
    q, sf, gs = _quant(x)
    s_g = float(gs[0])
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    rows, K = xf.shape
    a_b = np.abs(xf).reshape(rows, K // 16, 16).max(axis=2)
    S = ml_dtypes_e4m3(sf)
    codes = np.empty((rows, K), dtype=np.int64)
    codes[:, 0::2] = q & 15
    codes[:, 1::2] = q >> 4
    cmax = (codes & 7).reshape(rows, K // 16, 16).max(axis=2)
    exp_field = (sf >> 3) & 15
    normal = exp_field > 0
    sub = (exp_field == 0) & (sf != 0)
    zero = sf == 0
    slack = 1e-6
    ratio = np.where(S > 0, a_b / np.where(S > 0, S * s_g, 1.0), 0.0)
    assert normal.any()
    lo, hi = top * (1 - 2.0 ** -4), top * (1 + 2.0 ** -4)
    assert (ratio[normal] >= lo * (1 - slack)).all() and (ratio[normal] <= hi * (1 + slack)).all()
    assert (cmax[normal] == 7).all()
    if case == "wide_range":
        m = (sf & 7).astype(np.float64)
        assert set(np.unique(m[sub]).astype(int)) == set(range(1, 8))
        assert zero.any() and (a_b[zero] > 0).any()
    if sub.any():
        m = (sf[sub] & 7).astype(np.float64)
        r = ratio[sub]
        assert (r >= top * (m - 0.5) / m * (1 - slack)).all() and (r <= top * (m + 0.5) / m * (1 + slack)).all()
        e2m1 = np.array([oracle.e2m1_decode(c) for c in range(8)])
        least = np.abs((top * (m - 0.5) / m).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).astype(np.float64))
        assert (e2m1[cmax[sub]] >= least).all()
    if zero.any():
        assert (a_b[zero] / (6.0 * s_g) <= 2.0 ** -10 * (1 + slack)).all()
        assert (cmax[zero] == 0).all()


def ml_dtypes_e4m3(sf):
    """E4M3 bytes -> float64 through the library codec (independent of the oracle)."""
    return np.asarray(sf, np.uint8).view(ml_dtypes.float8_e4m3fn).astype(np.float64)


def test_quantize_rne_error_bound():
    """|x/(S s_g) - code| <= half the local E2M1 spacing, unless clipped at 6."""
    x = synthetic.gaussian_bf16(5, 1, (256, 1024), outlier_frac=0.001)
    q, sf, gs = _quant(x)
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    S = np.array([oracle.e4m3_decode(c) for c in range(256)])[sf]
    scale = np.repeat(S, 16, axis=1) * float(gs[0])
    codes = np.empty(xf.shape, dtype=np.int64)
    codes[:, 0::2] = q & 15
    codes[:, 1::2] = q >> 4
    table = _e2m1_table()
    val = np.array([table[c & 7] * (-1 if c & 8 else 1) for c in range(16)])[codes]
    v = xf / scale
    spacing = np.where(np.abs(val) < 2, 0.5, np.where(np.abs(val) < 4, 1.0, 2.0))
    err = np.abs(v - val)
    clipped = np.abs(v) > 6.0
    tol = spacing / 2 + 1e-5 * np.abs(v)
    assert (err[~clipped] <= tol[~clipped]).all()
    assert (np.abs(val[clipped]) == 6).all()
    assert (np.sign(val) * np.sign(xf) >= 0).all()


def test_nibble_order_low_is_even_element():
    x = np.zeros((1, 16), dtype=np.float32)
    x[0, 0] = 6.0      # element 0 -> code 7
    x[0, 1] = -1.0     # element 1 -> code 0xA at the amax-scaled grid
    xb = synthetic.f32_to_bf16_bits(x)
    q, sf, gs = _quant(xb)
    S = oracle.e4m3_decode(int(sf[0, 0])) * float(gs[0])
    assert q[0, 0] & 15 == oracle.e2m1_encode(6.0 / S)
    assert q[0, 0] >> 4 == oracle.e2m1_encode(-1.0 / S)
    assert q[0, 0] & 15 == 7


def test_zero_tensor_and_zero_blocks():
    x = np.zeros((4, 64), dtype=np.uint16)
    x[1, 5] = 0x8000                                  # -0.0
    q, sf, gs = _quant(x)
    assert gs[0] == 1.0 and (sf == 0).all()
    assert q[1, 2] == 0x80                            # element 5 -> high nibble, -0
    assert (np.delete(q.reshape(-1), 1 * 32 + 2) == 0).all()


def test_nonfinite_input_reported():
    x = synthetic.gaussian_bf16(0, 1, (8, 32))
    x[3, 7] = 0x7FC0                                  # NaN
    *_, st = oracle.quantize(x)
    assert st == oracle.ERR_NONFINITE
    x[3, 7] = 0x7F80                                  # +inf
    *_, st = oracle.quantize(x, global_scale=np.array([0.01], np.float32))
    assert st == oracle.ERR_NONFINITE


def test_grouped_gather_equals_per_group_dense():
    """A gathered group quantizes like the dense tensor of its rows."""
    x = synthetic.gaussian_bf16(2, 1, (64, 256))
    r = synthetic.route_topk_softmax(1, 64, 8, 2)
    q, sf, gs, st = oracle.quantize(x, row_index=r["row_index"], group_offsets=r["offsets"])
    assert st == 0
    off = r["offsets"]
    for g in range(8):
        rows = x[r["row_index"][off[g]:off[g + 1]]]
        if rows.shape[0] == 0:
            continue
        q2, sf2, gs2 = _quant(rows)
        assert gs2[0] == gs[g]
        assert np.array_equal(q2, q[off[g]:off[g + 1]])
        assert np.array_equal(sf2, sf[off[g]:off[g + 1]])


def test_given_scale_matches_amax_scale_when_equal():
    x = synthetic.gaussian_bf16(4, 1, (32, 128))
    q, sf, gs = _quant(x)
    q2, sf2, gs2, st = oracle.quantize(x, global_scale=gs)
    assert st == 0 and np.array_equal(q, q2) and np.array_equal(sf, sf2)


def test_dequantize_is_code_times_scales():
    x = synthetic.gaussian_bf16(6, 1, (16, 64))
    q, sf, gs = _quant(x)
    rg = oracle.rows_global_scale(gs, None, 16)
    y = oracle.dequantize(q, sf, rg)
    y64 = oracle.dequantize_f64(q, sf, rg)
    # fp32 result is the RN of the exact fp64 product (one rounding)
    assert np.array_equal(y, y64.astype(np.float32))
    yb = oracle.dequantize(q, sf, rg, out="bf16")
    assert np.array_equal(yb, synthetic.f32_to_bf16_bits(y))
    table = _e2m1_table()
    i, k = 3, 37
    code = (q[i, k // 2] >> (4 * (k % 2))) & 15
    want = table[code & 7] * (-1 if code & 8 else 1) * oracle.e4m3_decode(int(sf[i, k // 16])) * float(gs[0])
    assert y64[i, k] == want


# ------------------------------------------------------------------ remap
def _mx_tensor(seed, rows, K, lo=-10):
    q = synthetic.mxfp4_codes(seed, 16, rows * K // 2).reshape(rows, K // 2)
    e = synthetic.mxfp4_exponents(seed, 17, rows * K // 32, lo=lo).reshape(rows, K // 32)
    return q, e


def test_remap_lossless_and_ue8m0_library_decode():
    n, rows, K = 3, 64, 256
    q, e = _mx_tensor(0, n * rows, K)
    qn, sfn, gs, st = oracle.remap_mxfp4(q, e, n, rows, K)
    assert st == 0 and np.array_equal(qn, q)
    ref = oracle.dequantize_mxfp4_f64(q, e)
    # UE8M0 decode by the library agrees with 2^(u-127)
    assert np.array_equal(e.view(ml_dtypes.float8_e8m0fnu).astype(np.float64),
                          np.ldexp(1.0, e.astype(np.int64) - 127))
    for t in range(n):
        sl = slice(t * rows, (t + 1) * rows)
        got = oracle.dequantize_f64(qn[sl], sfn[sl], np.full(rows, gs[t], np.float32))
        assert np.array_equal(got, ref[sl])
        assert gs[t] == 2.0 ** (int(e[sl].max()) - 127 - 8)
        assert (sfn[sl] <= 0x7E).all() and sfn[sl].max() == 0x78   # 2^8 = 256 for the top block


def test_remap_spread_17_ok_18_not():
    rows, K = 4, 64
    q = np.full((rows, K // 2), 0x22, dtype=np.uint8)     # all codes 1.0
    e = np.full((rows, K // 32), 127, dtype=np.uint8)
    e[0, 0] = 127 + 8
    e[3, 1] = 127 - 9                                      # spread 17
    qn, sfn, gs, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    assert st == 0
    assert np.array_equal(oracle.dequantize_f64(qn, sfn, np.full(rows, gs[0], np.float32)),
                          oracle.dequantize_mxfp4_f64(q, e))
    e[3, 1] = 127 - 10                                     # spread 18
    *_, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    assert st == oracle.ERR_NOT_REPRESENTABLE
    e[3, 1] = 0xFF
    *_, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    assert st == oracle.ERR_NOT_REPRESENTABLE


def test_remap_zero_blocks_exempt():
    rows, K = 2, 64
    q = np.full((rows, K // 2), 0x33, dtype=np.uint8)
    q[1, 16:] = 0x88                                       # block (1,1): all -0
    e = np.full((rows, K // 32), 120, dtype=np.uint8)
    e[1, 1] = 10                                           # far outside the spread, but exempt
    qn, sfn, gs, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    assert st == 0
    assert np.array_equal(oracle.dequantize_f64(qn, sfn, np.full(rows, gs[0], np.float32)),
                          oracle.dequantize_mxfp4_f64(q, e))


# ------------------------------------------------------------------ MXFP4 encode
def _bf16(vals):
    return synthetic.f32_to_bf16_bits(np.asarray(vals, dtype=np.float32))


def _mx_block(vals):
    x = np.zeros(32, dtype=np.float32)
    x[:len(vals)] = vals
    return _bf16(x).reshape(1, 32)


def _codes(q):
    return np.stack([q & 15, q >> 4], axis=-1).reshape(q.shape[0], -1)


@pytest.mark.parametrize("vals, byte, first_codes", [
    # amax 6 = 1.5 * 2^2: E = 2 - 2 = 0, the block is already on the E2M1 grid
    ([6.0, -3.0, 0.5], 127, [7, 8 + 5, 1]),
    # amax 7: floor(log2 7) = 2, E = 0; 7 saturates to 6 and 5 ties to 4 (even)
    ([7.0, 5.0, -1.25], 127, [7, 6, 8 + 2]),
    # amax 8: E = 1, so every value is halved before rounding: 3 -> 1.5, and
    # 0.5 -> 0.25 ties to 0 (even)
    ([8.0, 3.0, 0.5], 128, [6, 3, 0]),
    # amax 1: E = -2, so every value is quadrupled: 0.75 -> 3, -0.25 -> -1,
    # bf16(0.3) = 0.30078125 -> 1.203 -> 1.0
    ([1.0, 0.75, -0.25, 0.3], 125, [6, 5, 8 + 2, 2]),
])
def test_mxfp4_encode_worked_blocks(vals, byte, first_codes):
    """Blocks worked by hand from the OCP MX v1.0 rule (E = floor(log2 amax) - 2)."""
    q, e, st = oracle.quantize_mxfp4(_mx_block(vals))
    assert st == oracle.OK and int(e[0, 0]) == byte
    c = _codes(q)[0]
    assert list(c[:len(first_codes)]) == first_codes
    assert (c[len(vals):] == 0).all()


def test_mxfp4_encode_vs_log2_and_library_codec():
    """Scale byte = floor(log2 amax) + 125 (numpy log2), codes = ml_dtypes E2M1
    of x / 2^E, over blocks whose amax spans the bf16 normal and subnormal range."""
    rows, K = 64, 256
    x = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(21, 1, (rows, K))).astype(np.float64)
    mag = np.ldexp(1.0, (synthetic.words(21, 2, 0, rows * K // 32) % 250).astype(np.int64) - 130)
    x = x * np.repeat(mag, 32).reshape(rows, K)
    xb = synthetic.f32_to_bf16_bits(x.astype(np.float32))
    q, e, st = oracle.quantize_mxfp4(xb)
    assert st == oracle.OK
    xf = synthetic.bf16_bits_to_f32(xb).astype(np.float64).reshape(rows, K // 32, 32)
    amax = np.abs(xf).max(axis=2)
    E = np.clip(np.floor(np.log2(np.where(amax > 0, amax, 1.0))) - 2, -127, 127).astype(np.int64)
    E = np.where(amax > 0, E, -127)
    assert np.array_equal(e.astype(np.int64), E + 127)
    scaled = (xf / np.ldexp(1.0, E)[..., None]).astype(np.float32).reshape(rows, K)
    lib = scaled.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)
    assert np.array_equal(_codes(q), lib)
    # the subnormal and clamped end of the range is exercised
    assert (e == 0).any() and (e > 200).any()


def test_mxfp4_encode_error_bound_and_exact_powers():
    """|x - deq| <= 2^E on the unsaturated grid, < 2^(E+1) where x / 2^E in (6, 8);
    a block whose amax is a power of two reproduces its amax exactly."""
    x = synthetic.gaussian_bf16(22, 1, (32, 512), sigma=3.0)
    q, e, st = oracle.quantize_mxfp4(x)
    assert st == oracle.OK
    xf = synthetic.bf16_bits_to_f32(x).astype(np.float64)
    y = oracle.dequantize_mxfp4_f64(q, e)
    X = np.repeat(np.ldexp(1.0, e.astype(np.int64) - 127), 32, axis=1)
    err = np.abs(xf - y)
    small = np.abs(xf) <= 6 * X
    assert (err[small] <= X[small]).all() and (err[~small] < 2 * X[~small]).all()
    assert (~small).any()                                   # saturation happens on Gaussian data
    xp = _mx_block([2.0 ** -5, 0.01, -0.02])
    qp, ep, _ = oracle.quantize_mxfp4(xp)
    assert oracle.dequantize_mxfp4_f64(qp, ep)[0, 0] == 2.0 ** -5


def test_mxfp4_encode_zero_and_nonfinite_blocks():
    x = np.zeros((2, 96), dtype=np.uint16)
    x[0, 40] = 0x8000                                     # -0 in block 1
    x[1, 5] = 0x7F80                                      # +inf in block 0
    x[1, 70] = _bf16([1.5])[0]                            # block 2 stays encodable
    q, e, st = oracle.quantize_mxfp4(x)
    assert st == oracle.ERR_NONFINITE
    assert list(e[0]) == [0, 0, 0]
    assert _codes(q)[0, 40] == 8 and (np.delete(_codes(q)[0], 40) == 0).all()
    assert e[1, 0] == 0xFF and (q[1, :16] == 0).all()
    assert e[1, 2] == 125 and _codes(q)[1, 70] == 7     # 1.5 / 2^-2 = 6


def test_mxfp4_encode_then_remap_is_lossless():
    """The encoder's output is a valid remap input: its NVFP4 remap dequantizes
    to the same values (the lossless remap of the format section)."""
    rows, K = 48, 512
    x = synthetic.gaussian_bf16(23, 1, (rows, K))
    q, e, _ = oracle.quantize_mxfp4(x)
    qn, sfn, gs, st = oracle.remap_mxfp4(q, e, 1, rows, K)
    assert st == oracle.OK
    assert np.array_equal(oracle.dequantize_f64(qn, sfn, np.full(rows, gs[0], np.float32)),
                          oracle.dequantize_mxfp4_f64(q, e))


def test_mxfp4_from_fp8_relative_error_matches_page():
    """FP8 (E4M3) Gaussian weights through the encoder lose about 12 % in
    relative L2, the figure the page prints for its FP8 -> MXFP4 step."""
    want = FACTS["mxfp4_from_fp8_rel_l2_error_approx"]
    x = synthetic.bf16_bits_to_f32(synthetic.gaussian_bf16(24, 1, (256, 1024)))
    x8 = x.astype(ml_dtypes.float8_e4m3fn).astype(np.float32)
    q, e, st = oracle.quantize_mxfp4(synthetic.f32_to_bf16_bits(x8))
    assert st == oracle.OK
    y = oracle.dequantize_mxfp4_f64(q, e)
    rel = np.linalg.norm(y - x8) / np.linalg.norm(x8)
    assert abs(rel - want) < 0.015


# ------------------------------------------------------------------ GEMM
def test_gemm_closed_form_integer_case():
    """All S = 1 (0x38), s_g = 1: values are multiples of 0.5, so 4*y is an
    integer matrix product, computed here exactly in int64."""
    rng = np.random.default_rng(0)
    M, N, K = 128, 256, 512
    qa = rng.integers(0, 256, (M, K // 2), dtype=np.uint8)
    qb = rng.integers(0, 256, (N, K // 2), dtype=np.uint8)
    sfa = np.full((M, K // 16), 0x38, np.uint8)
    sfb = np.full((N, K // 16), 0x38, np.uint8)
    a = oracle.dequantize_f64(qa, sfa, np.ones(M, np.float32))
    b = oracle.dequantize_f64(qb, sfb, np.ones(N, np.float32))
    y, s = oracle.gemm_f64(a, b)
    table2 = np.array([0, 1, 2, 3, 4, 6, 8, 12], dtype=np.int64)   # 2 * magnitudes

    def ints(qq):
        c = np.empty((qq.shape[0], qq.shape[1] * 2), dtype=np.int64)
        c[:, 0::2] = qq & 15
        c[:, 1::2] = qq >> 4
        return np.where(c & 8, -1, 1) * table2[c & 7]

    ia, ib = ints(qa), ints(qb)
    assert np.array_equal(4 * y, (ia @ ib.T).astype(np.float64))
    assert np.array_equal(4 * s, (np.abs(ia) @ np.abs(ib).T).astype(np.float64))


def test_gemm_matches_plain_dot_loop():
    x = synthetic.gaussian_bf16(0, 1, (8, 256), outlier_frac=0.01)
    w = synthetic.gaussian_bf16(0, 2, (12, 256), sigma=0.02)
    qa, sfa, ga = _quant(x)
    qb, sfb, gb = _quant(w)
    a = oracle.dequantize_f64(qa, sfa, np.full(8, ga[0], np.float32))
    b = oracle.dequantize_f64(qb, sfb, np.full(12, gb[0], np.float32))
    y, s = oracle.gemm_f64(a, b)
    for i in range(8):
        for j in range(12):
            yy, ss = oracle.dot_f64(a[i], b[j])
            assert abs(yy - y[i, j]) <= 1e-12 * ss and abs(ss - s[i, j]) <= 1e-12 * ss


def test_grouped_gemm_equals_dense_per_expert():
    rng = np.random.default_rng(3)
    offsets = np.array([0, 5, 5, 17, 20])
    a = rng.standard_normal((20, 64))
    b = rng.standard_normal((4, 8, 64))
    y, s = oracle.grouped_gemm_f64(a, b, offsets)
    for e in range(4):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            assert np.array_equal(y[r0:r1], a[r0:r1] @ b[e].T)


# ------------------------------------------------------------------ SwiGLU
def test_swiglu_closed_forms():
    g = np.array([0.0, 1.0, -1.0, 30.0, -30.0, 2.0], dtype=np.float32)
    u = np.array([5.0, 1.0, 1.0, 2.0, 3.0, -0.5], dtype=np.float32)
    y = np.concatenate([g, u])[None, :]
    h = synthetic.bf16_bits_to_f32(oracle.swiglu(y))[0]
    e = math.e
    want = [0.0, 1 / (1 + 1 / e), -1 / (1 + e), 60.0, -30.0 * 3.0 / (1 + math.exp(30.0)),
            -0.5 * 2 / (1 + math.exp(-2.0))]
    for hv, wv in zip(h, want):
        assert hv == synthetic.bf16_bits_to_f32(synthetic.f32_to_bf16_bits(np.float32(wv)))[()]


# ------------------------------------------------------------------ KV facts
def test_kv_cache_size_facts():
    """P3: 4 heads x 256 x 2 = 2048 elements per token per layer; NVFP4 ~ 1/4 of bf16."""
    n = FACTS["kv_heads"] * FACTS["kv_head_dim"] * 2
    assert n == FACTS["kv_elements_per_token"]
    bf16 = n * 2
    nvfp4 = n * FACTS["effective_bits"] / 8
    assert abs(nvfp4 / bf16 - FACTS["kv_nvfp4_over_bf16_approx"]) < 0.04


# ------------------------------------------------------------------ routing / combine
def test_route_matches_library_sort_and_invariants():
    """Grouping by expert equals a stable lexicographic sort on (expert, token)
    done by numpy, and every (token, choice) lands in its expert's rows."""
    rng = np.random.default_rng(0)
    T, E, k = 300, 37, 4
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    off, ri, slot, st = oracle.route(ids, E)
    assert st == 0
    flat_e = ids.reshape(-1)
    flat_t = np.repeat(np.arange(T), k)
    order = np.lexsort((flat_t, flat_e))
    assert np.array_equal(ri, flat_t[order])
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat_e, minlength=E))]))
    for t in range(T):
        for j in range(k):
            r = slot[t, j]
            e = ids[t, j]
            assert off[e] <= r < off[e + 1] and ri[r] == t
    assert sorted(slot.reshape(-1).tolist()) == list(range(T * k))


def test_route_drops_out_of_range_choices():
    """An id outside [0, E) names no expert of the model (the pages route each
    token to its top-10 of the model's 512 experts): that choice is dropped.
    The rest must be exactly numpy's stable (expert, token) sort of the valid
    pairs alone, the dropped ones get slot -1 and the offsets count only valid
    choices."""
    rng = np.random.default_rng(3)
    T, E, k = 257, 19, 5
    ids = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)]).astype(np.int32)
    bad_pos = rng.choice(T * k, size=40, replace=False)
    flat = ids.reshape(-1)
    flat[bad_pos[:20]] = E + rng.integers(0, 1000, 20)
    flat[bad_pos[20:]] = -1 - rng.integers(0, 1000, 20)
    ids = flat.reshape(T, k)
    off, ri, slot, st = oracle.route(ids, E)
    assert st == 1
    flat_t = np.repeat(np.arange(T), k)
    valid = (flat >= 0) & (flat < E)
    order = np.lexsort((flat_t[valid], flat[valid]))
    assert np.array_equal(ri, flat_t[valid][order])
    assert np.array_equal(off, np.concatenate([[0], np.cumsum(np.bincount(flat[valid], minlength=E))]))
    sl = slot.reshape(-1)
    assert (sl[~valid] == -1).all()
    want = np.empty(valid.sum(), np.int64)
    want[order] = np.arange(valid.sum())
    assert np.array_equal(sl[valid], want)
    # all choices dropped: empty routing, every slot -1
    off0, ri0, slot0, st0 = oracle.route(np.full((4, 2), E, np.int32), E)
    assert st0 == 1 and (off0 == 0).all() and ri0.size == 0 and (slot0 == -1).all()
    # no routing at all
    assert oracle.route(ids, 0)[3] == 2


def test_combine_closed_forms():
    rng = np.random.default_rng(1)
    T, k, H = 5, 3, 16
    y = rng.standard_normal((T * k, H)).astype(np.float32)
    slot = np.arange(T * k, dtype=np.int32).reshape(T, k)
    onehot = np.zeros((T, k), np.float32)
    onehot[:, 1] = 1.0
    out, s = oracle.combine(y, slot, onehot)
    assert np.array_equal(out, y[slot[:, 1]].astype(np.float64))
    w = np.full((T, k), 0.25, np.float32)
    out, s = oracle.combine(y, slot, w)
    for t in range(T):
        want = sum(0.25 * y[slot[t, j]].astype(np.float64) for j in range(k))
        assert np.allclose(out[t], want, rtol=0, atol=1e-12)
        assert np.allclose(s[t], sum(np.abs(0.25 * y[slot[t, j]].astype(np.float64)) for j in range(k)))
    # a dropped choice (slot -1) contributes nothing: same as weight 0 on a real row
    dropped = slot.copy()
    dropped[:, 2] = -1
    w0 = w.copy()
    w0[:, 2] = 0.0
    out_d, s_d = oracle.combine(y, dropped, w)
    out_0, s_0 = oracle.combine(y, slot, w0)
    assert np.array_equal(out_d, out_0) and np.array_equal(s_d, s_0)
