"""Pins of the oracle's encoders (fp16 weights -> packed bytes).  The pages
fix the formats, not the quantiser, so the choice of scale is a reading
(parity unpinned); the nearest-value step and the byte layout are pinned:
hand-worked rows, exact recovery of the codes of weights built from
power-of-two scales, an error bound, and optimality against candidates
rounded by numpy."""
import numpy as np
import pytest

import oracle
from conftest import golden_lines, parse_value

FMT = {"fp4g16_f16": oracle.FMT_FP4G16_F16, "mxfp4": oracle.FMT_MXFP4, "iq4_nl": oracle.FMT_IQ4_NL}
E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
KV = np.array([int(t) for t in golden_lines("iq4nl_codebook.txt")[-1].split()])


def _f16(vals):
    return np.array(vals, dtype=np.float64).astype(np.float16).view(np.uint16)


def test_quantize_handmade_rows():
    lines = golden_lines("quantize_handmade.txt")
    assert len(lines) == 20
    for i in range(0, len(lines), 4):
        fmt = FMT[lines[i].split()[1]]
        w = [parse_value(t) for t in lines[i + 1].split()[1:]]
        sc = bytes(int(t, 16) for t in lines[i + 2].split()[1:])
        data = bytes(int(t, 16) for t in lines[i + 3].split()[1:])
        k = len(w)
        d, s = oracle.quantize(fmt, 1, k, _f16(w))
        assert bytes(d) == data, (lines[i], bytes(d).hex(" "))
        assert (b"" if s is None else bytes(s)) == sc, (lines[i], bytes(s).hex(" "))


@pytest.mark.parametrize("fmt", [oracle.FMT_FP4G16_F16, oracle.FMT_MXFP4])
def test_fp4_codes_recovered_from_power_of_two_scales(fmt):
    """Weights = code * 2^j with a +-6 in every group: the encoder's scale is
    2^j again and every code comes back (code 8, -0, decodes like +0 and is
    left out)."""
    rng = np.random.default_rng(1)
    n, k = 64, 256
    g = 32 if fmt == oracle.FMT_MXFP4 else 16
    codes = rng.choice([c for c in range(16) if c != 8], size=(n, k))
    codes[:, ::g] = rng.choice([7, 15], size=(n, k // g))
    j = rng.integers(-12, 4, size=(n, k // g))
    w = E2M1[codes] * np.ldexp(1.0, np.repeat(j, g, axis=1))
    d, s = oracle.quantize(fmt, n, k, _f16(w))
    assert np.array_equal(d.reshape(n, k // 2) & 15, codes[:, 0::2])
    assert np.array_equal(d.reshape(n, k // 2) >> 4, codes[:, 1::2])
    if fmt == oracle.FMT_MXFP4:
        assert np.array_equal(s.reshape(n, k // 32).astype(int), j + 127 + 0)
    else:
        assert np.array_equal(s.view(np.uint16).reshape(n, k // 16), _f16(np.ldexp(1.0, j)))


def test_iq4nl_codes_recovered_from_power_of_two_scales():
    """Block = kv[idx] * (-2^j) with index 0 (the -127 entry) present and
    every other |kv| below 127: d = -2^j and the indices come back."""
    rng = np.random.default_rng(2)
    n, k = 32, 256
    idx = rng.integers(1, 16, size=(n, k))
    idx[:, ::32] = 0
    j = rng.integers(-12, -2, size=(n, k // 32))
    w = KV[idx] * -np.ldexp(1.0, np.repeat(j, 32, axis=1))
    d, _ = oracle.quantize(oracle.FMT_IQ4_NL, n, k, _f16(w))
    blk = d.reshape(n, k // 32, 18)
    assert np.array_equal(blk[..., 2:] & 15, idx.reshape(n, k // 32, 32)[..., :16])
    assert np.array_equal(blk[..., 2:] >> 4, idx.reshape(n, k // 32, 32)[..., 16:])
    dbits = blk[..., 0].astype(np.uint16) | (blk[..., 1].astype(np.uint16) << 8)
    assert np.array_equal(dbits, _f16(-np.ldexp(1.0, j)))


@pytest.mark.parametrize("fmt", [oracle.FMT_FP4G16_F16, oracle.FMT_MXFP4, oracle.FMT_IQ4_NL])
def test_quantize_is_nearest_and_bounded(fmt):
    """Random fp16 weights: no other code of the group's scale decodes closer
    (candidates rounded by numpy), and the error is within half the largest
    gap between neighbouring values (plus the rounding of the candidates)."""
    rng = np.random.default_rng(3 + fmt)
    n, k = 24, 128
    w16 = _f16(rng.standard_normal((n, k)) * np.exp(rng.uniform(-6, 3, size=(n, 1))))
    w = w16.view(np.float16).astype(np.float64)
    d, s = oracle.quantize(fmt, n, k, w16)
    deq = oracle.dequant(fmt, n, k, d, s).view(np.float16).astype(np.float64)
    err = np.abs(w - deq)
    if fmt == oracle.FMT_IQ4_NL:
        blk = d.reshape(n, k // 32, 18)
        dd = (blk[..., 0].astype(np.uint16) | (blk[..., 1].astype(np.uint16) << 8)).view(np.float16).astype(np.float64)
        cand = (dd[..., None] * KV[None, None, :]).astype(np.float16).astype(np.float64)   # [n][blocks][16]
        cand = np.repeat(cand, 32, axis=1)
        # half the largest table gap (24: 89 -> 113) or the clipped end of the
        # asymmetric table (|m| = 127 |d| on one side, 113 |d| on the other)
        gap = 14.0 * np.abs(np.repeat(dd, 32, axis=1))
    else:
        g = 32 if fmt == oracle.FMT_MXFP4 else 16
        if fmt == oracle.FMT_MXFP4:
            sc = np.ldexp(1.0, s.reshape(n, k // 32).astype(int) - 127)
        else:
            sc = s.view(np.uint16).reshape(n, k // 16).view(np.float16).astype(np.float64)
        cand = (sc[..., None] * E2M1[None, None, :]).astype(np.float16).astype(np.float64)
        cand = np.repeat(cand, g, axis=1)
        gap = np.repeat(sc, g, axis=1) * 1.0   # largest gap 2 (4 -> 6)
        if fmt == oracle.FMT_MXFP4:            # MX saturates values above 6 * scale (up to 8 * scale)
            gap = np.repeat(sc, g, axis=1) * 2.0
    best = np.min(np.abs(w[..., None] - cand), axis=-1)
    assert np.array_equal(err, best)
    assert np.all(err <= gap * (1 + 2.0 ** -10) + 2.0 ** -24)
