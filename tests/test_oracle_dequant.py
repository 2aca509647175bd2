"""Pins of the oracle's dequantisation: hand-built blocks with hand-written
expected values, exhaustive scale x code sweeps against exact rational
rounding, and mutation checks showing the golden comparison catches a swapped
nibble convention, a reversed scale byte order, a flipped nibble and a scale
off by one ulp."""
import math
from fractions import Fraction

import numpy as np
import pytest

import oracle
from conftest import golden_lines, parse_value


def _to_bits(vals):
    return np.array(vals, dtype=np.float64).astype(np.float16).view(np.uint16)


def _iq4_cases():
    lines = golden_lines("iq4nl_blocks_handmade.txt")
    cases = []
    for i in range(0, len(lines), 2):
        blk = bytes(int(t, 16) for t in lines[i].split()[1:])
        exp = [parse_value(t) for t in lines[i + 1].split()[1:]]
        assert len(blk) == 18 and len(exp) == 32
        cases.append((np.frombuffer(blk, dtype=np.uint8).copy(), exp))
    return cases


def _fp4_cases():
    lines = golden_lines("fp4g16_rows_handmade.txt")
    cases = []
    for i in range(0, len(lines), 3):
        codes = np.array([int(t, 16) for t in lines[i].split()[1:]], dtype=np.uint8)
        sc = lines[i + 1].split()
        if sc[0] == "scales_f16":
            fmt = oracle.FMT_FP4G16_F16
            s16 = np.array([int(t, 16) for t in sc[1:3]], dtype=np.uint16)
            scales, g = s16.view(np.uint8), 1.0
        else:
            fmt = oracle.FMT_FP4G16_E4M3
            scales, g = np.array([int(t, 16) for t in sc[1:3]], dtype=np.uint8), float(sc[4])
        exp = [parse_value(t) for t in lines[i + 2].split()[1:]]
        assert len(codes) == 16 and len(exp) == 32
        cases.append((fmt, codes, scales, np.float32(g), exp))
    return cases


def test_iq4nl_handmade_blocks():
    for blk, exp in _iq4_cases():
        got = oracle.dequant(oracle.FMT_IQ4_NL, 1, 32, blk)
        assert np.array_equal(got[0], _to_bits(exp)), (blk, got)


def test_fp4g16_handmade_rows():
    for fmt, codes, scales, g, exp in _fp4_cases():
        got = oracle.dequant(fmt, 1, 32, codes, scales, g)
        assert np.array_equal(got[0], _to_bits(exp)), (fmt, got)


def test_mutations_are_caught():
    blk, exp = _iq4_cases()[3]      # the rounding block: distinct values per nibble
    ref = _to_bits(exp)
    muts = []
    m = blk.copy(); m[2:] = ((m[2:] & 0x0F) << 4) | (m[2:] >> 4); muts.append(m)   # swapped nibble convention
    m = blk.copy(); m[0], m[1] = blk[1], blk[0]; muts.append(m)                      # reversed scale byte order
    m = blk.copy(); m[3] ^= 0x01; muts.append(m)                                     # one flipped nibble bit
    m = blk.copy(); m[0] += 1; muts.append(m)                                        # scale off by one ulp
    for mut in muts:
        assert not np.array_equal(oracle.dequant(oracle.FMT_IQ4_NL, 1, 32, mut)[0], ref)
    fmt, codes, scales, g, exp = _fp4_cases()[0]
    ref = _to_bits(exp)
    c2 = ((codes & 0x0F) << 4) | (codes >> 4)
    assert not np.array_equal(oracle.dequant(fmt, 1, 32, c2, scales, g)[0], ref)
    s2 = scales.copy(); s2[0] += 1
    assert not np.array_equal(oracle.dequant(fmt, 1, 32, codes, s2, g)[0], ref)


def _exact_round_f16(fr: Fraction) -> float:
    """Round an exact rational to fp16 (nearest, ties to even), written from
    the binary16 definition with integer arithmetic only (finite range)."""
    if fr == 0:
        return 0.0
    sign = -1.0 if fr < 0 else 1.0
    a = abs(fr)
    e = a.numerator.bit_length() - a.denominator.bit_length()
    if Fraction(2) ** e > a:
        e -= 1                               # now 2^e <= a < 2^(e+1)
    e = max(e, -14)                          # subnormal spacing below 2^-14
    q = a / Fraction(2) ** (e - 10)          # units of the fp16 spacing
    fl = q.numerator // q.denominator
    rem = q - fl
    r = fl + (1 if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1) else 0)
    v = r * Fraction(2) ** (e - 10)
    if v > 65504:
        return sign * math.inf
    return sign * float(v)


@pytest.mark.parametrize("stride", [97])
def test_exact_rational_rounding_sample(stride):
    """A sample of d patterns x all 16 codes against exact rational rounding."""
    kv = [oracle.iq4nl_value(i) for i in range(16)]
    dbits = np.arange(1, 0x7C00, stride, dtype=np.uint16)
    blocks = np.zeros((dbits.size, 18), dtype=np.uint8)
    blocks[:, 0] = dbits & 0xFF
    blocks[:, 1] = dbits >> 8
    blocks[:, 2:] = (np.arange(16) | ((15 - np.arange(16)) << 4)).astype(np.uint8)
    got = oracle.dequant(oracle.FMT_IQ4_NL, 1, 32 * dbits.size, blocks.reshape(-1))[0].reshape(-1, 32)
    for i, db in enumerate(dbits):
        d = Fraction(float(np.uint16(db).view(np.float16)))
        for j in range(32):
            idx = j if j < 16 else 15 - (j - 16)
            exp = _exact_round_f16(d * kv[idx])
            g = float(np.uint16(got[i, j]).view(np.float16))
            assert g == exp or (math.isinf(g) and math.isinf(exp) and (g > 0) == (exp > 0)), (db, j, g, exp)


def test_iq4nl_exhaustive_scales_vs_numpy_rounding():
    """Every finite and non-finite fp16 d x all 16 codes: the exact product
    d*kv (exact in float64) rounded by numpy's float64->float16 conversion."""
    kv = np.array([oracle.iq4nl_value(i) for i in range(16)], dtype=np.float64)
    dbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blocks = np.zeros((65536, 18), dtype=np.uint8)
    blocks[:, 0] = dbits & 0xFF
    blocks[:, 1] = dbits >> 8
    blocks[:, 2:] = (np.arange(16) | ((15 - np.arange(16)) << 4)).astype(np.uint8)
    got = oracle.dequant(oracle.FMT_IQ4_NL, 1, 32 * 65536, blocks.reshape(-1))[0].reshape(65536, 32)
    idx = np.concatenate([np.arange(16), 15 - np.arange(16)])
    d = dbits.view(np.float16).astype(np.float64)
    with np.errstate(all="ignore"):
        exp = (d[:, None] * kv[idx][None, :]).astype(np.float16).view(np.uint16)
    nan_g = (got & 0x7C00) == 0x7C00
    nan_g &= (got & 0x3FF) != 0
    nan_e = ((exp & 0x7C00) == 0x7C00) & ((exp & 0x3FF) != 0)
    assert np.array_equal(nan_g, nan_e)
    assert np.array_equal(got[~nan_g], exp[~nan_e])


def test_fp4_f16_exhaustive_scales_vs_numpy_rounding():
    e2m1 = np.array([oracle.e2m1_to_f64(c) for c in range(16)], dtype=np.float64)
    sbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    n = 65536
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8), (n, 1))
    got = oracle.dequant(oracle.FMT_FP4G16_F16, n, 16, codes.reshape(-1), sbits.view(np.uint8))
    s = sbits.view(np.float16).astype(np.float64)
    with np.errstate(all="ignore"):
        exp = (s[:, None] * e2m1[None, :]).astype(np.float16).view(np.uint16)
    nan_g = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
    nan_e = ((exp & 0x7C00) == 0x7C00) & ((exp & 0x3FF) != 0)
    assert np.array_equal(nan_g, nan_e)
    assert np.array_equal(got[~nan_g], exp[~nan_e])


@pytest.mark.parametrize("g", [1.0, 0.5, 0.1, 3.0e-5, 1.7e3, 0.013671875, 2.0 ** -20, 123.456])
def test_fp4_e4m3_all_scale_bytes_vs_numpy_rounding(g):
    e2m1 = np.array([oracle.e2m1_to_f64(c) for c in range(16)], dtype=np.float64)
    e4 = np.array([oracle.e4m3_to_f64(b) for b in range(256)], dtype=np.float64)
    n = 256
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8), (n, 1))
    g32 = np.float32(g)
    got = oracle.dequant(oracle.FMT_FP4G16_E4M3, n, 16, codes.reshape(-1), np.arange(256, dtype=np.uint8), g32)
    with np.errstate(all="ignore"):
        p = (e4[:, None] * e2m1[None, :]) * np.float64(g32)   # exact in float64
        exp = p.astype(np.float32).astype(np.float16).view(np.uint16)
    nan_g = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
    nan_e = ((exp & 0x7C00) == 0x7C00) & ((exp & 0x3FF) != 0)
    assert np.array_equal(nan_g, nan_e)
    assert np.array_equal(got[~nan_g], exp[~nan_e])


# -- MXFP4 (E2M1 codes, one E8M0 scale byte per 32) ---------------------------
def _mx_cases():
    lines = golden_lines("mxfp4_rows_handmade.txt")
    cases = []
    for i in range(0, len(lines), 3):
        codes = np.array([int(t, 16) for t in lines[i].split()[1:]], dtype=np.uint8)
        scale = np.array([int(lines[i + 1].split()[1], 16)], dtype=np.uint8)
        exp = [parse_value(t) for t in lines[i + 2].split()[1:]]
        assert len(codes) == 16 and len(exp) == 32
        cases.append((codes, scale, exp))
    return cases


def test_mxfp4_handmade_rows():
    cases = _mx_cases()
    assert len(cases) == 6
    for codes, scale, exp in cases:
        got = oracle.dequant(oracle.FMT_MXFP4, 1, 32, codes, scale)
        assert np.array_equal(got[0], _to_bits(exp)), (scale, got)


def test_mxfp4_nan_scale():
    """E8M0 0xFF is NaN: every weight of its group is NaN, zeros included."""
    codes = np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE] * 2, dtype=np.uint8)
    got = oracle.dequant(oracle.FMT_MXFP4, 1, 32, codes, np.array([0xFF], dtype=np.uint8))[0]
    assert np.all(((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0))


def test_mxfp4_mutations_are_caught():
    """A swapped nibble convention, a reversed code pair order, a flipped
    nibble and a scale off by one are each visible in the golden rows."""
    codes, scale, exp = _mx_cases()[5]
    ref = _to_bits(exp)
    muts = [(((codes & 0x0F) << 4) | (codes >> 4), scale),                  # swapped nibble convention
            (np.concatenate([codes[1::-1], codes[2:]]), scale),             # reversed byte (pair) order
            (codes ^ np.array([0x01] + [0] * 15, dtype=np.uint8), scale),   # one flipped nibble bit
            (codes, scale + 1), (codes, scale - 1)]                          # scale off by one
    for c, s in muts:
        assert not np.array_equal(oracle.dequant(oracle.FMT_MXFP4, 1, 32, c, s)[0], ref)


def test_mxfp4_all_scale_bytes_vs_numpy_rounding():
    """Every E8M0 byte x every code: fp16(code * 2^(e-127)) rounded by numpy
    from the exact double product."""
    e2m1 = np.array([oracle.e2m1_to_f64(c) for c in range(16)], dtype=np.float64)
    n = 256
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE] * 2, dtype=np.uint8), (n, 1))
    got = oracle.dequant(oracle.FMT_MXFP4, n, 32, codes.reshape(-1), np.arange(256, dtype=np.uint8))
    with np.errstate(all="ignore"):
        scale = np.where(np.arange(256) == 255, np.nan, np.ldexp(1.0, np.arange(256) - 127))
        exp = (scale[:, None] * np.tile(e2m1, 2)[None, :]).astype(np.float16).view(np.uint16)
    nan_g = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
    nan_e = ((exp & 0x7C00) == 0x7C00) & ((exp & 0x3FF) != 0)
    assert np.array_equal(nan_g, nan_e) and nan_g[255].all() and not nan_g[:255].any()
    assert np.array_equal(got[~nan_g], exp[~nan_e])
