"""Pins of the oracle's own number codecs against independent libraries and
the values printed on the pages."""
import math

import numpy as np
import pytest
import torch

import oracle
from conftest import golden_lines


def _same(a: float, b: float) -> bool:
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


def test_f16_decode_all_patterns_match_numpy():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = bits.view(np.float16).astype(np.float64)
    L = oracle.lib()
    got = np.array([L.orc_f16_to_f64(int(b)) for b in bits])
    assert all(_same(g, r) for g, r in zip(got, ref))


def _encode_many(vals):
    L = oracle.lib()
    return np.array([L.orc_f64_to_f16(float(v)) for v in vals], dtype=np.uint16)


def test_f16_encode_exact_values_and_ties():
    finite = np.arange(0, 0x7C00, dtype=np.uint32).astype(np.uint16)  # +0 .. 65504
    vals = finite.view(np.float16).astype(np.float64)
    # every finite fp16 value encodes to itself (both signs)
    assert np.array_equal(_encode_many(vals), finite)
    assert np.array_equal(_encode_many(-vals), finite | 0x8000)
    # halfway points between neighbours: ties go to the even pattern
    mids = (vals[:-1] + vals[1:]) / 2.0
    exp_even = np.where(finite[:-1] % 2 == 0, finite[:-1], finite[1:]).astype(np.uint16)
    assert np.array_equal(_encode_many(mids), exp_even)
    # just above / below a tie go up / down
    up = np.nextafter(mids, np.inf)
    dn = np.nextafter(mids, -np.inf)
    assert np.array_equal(_encode_many(up), finite[1:])
    assert np.array_equal(_encode_many(dn), finite[:-1])


def test_f16_encode_random_and_special_vs_numpy():
    rng = np.random.default_rng(1234)
    v = np.concatenate([
        rng.standard_normal(20000) * 10.0 ** rng.integers(-9, 6, 20000),
        np.array([65504.0, 65519.999, 65520.0, 1e9, -1e9, 2.0 ** -25, 2.0 ** -25 * 1.0000001,
                  2.0 ** -26, 3 * 2.0 ** -26, 0.0, -0.0, np.inf, -np.inf]),
    ])
    got = _encode_many(v)
    ref = v.astype(np.float16).view(np.uint16)
    assert np.array_equal(got, ref)
    assert oracle.f64_to_f16(float("nan")) & 0x7C00 == 0x7C00 and oracle.f64_to_f16(float("nan")) & 0x3FF


def test_e4m3_all_bytes_match_torch():
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = allb.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = np.array([oracle.e4m3_to_f64(b) for b in range(256)])
    assert all(_same(g, r) for g, r in zip(got, ref))
    # OCP E4M3FN extremes: max normal 448 (0x7e), min subnormal 2^-9 (0x01), NaN only at 0x7f/0xff
    assert got[0x7E] == 448.0 and got[0x01] == 2.0 ** -9 and math.isnan(got[0x7F]) and math.isnan(got[0xFF])
    assert sum(math.isnan(g) for g in got) == 2


def test_e8m0_all_bytes_match_torch():
    """OCP E8M0 (the MXFP4 scale): all 256 bytes against torch's
    float8_e8m0fnu; 0x7f is 1, 0x00 is 2^-127, 0xff the only NaN."""
    allb = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = allb.view(torch.float8_e8m0fnu).to(torch.float64).numpy()
    got = np.array([oracle.e8m0_to_f64(b) for b in range(256)])
    assert all(_same(g, r) for g, r in zip(got, ref))
    assert got[0x7F] == 1.0 and got[0x00] == 2.0 ** -127 and got[0xFE] == 2.0 ** 127 and math.isnan(got[0xFF])
    assert sum(math.isnan(g) for g in got) == 1


def test_e2m1_matches_printed_magnitudes():
    mags = [float(t) for t in golden_lines("e2m1_magnitudes.txt")[0].split()]
    assert mags == sorted(mags) and len(mags) == 8
    for code in range(8):
        assert _same(oracle.e2m1_to_f64(code), mags[code])
        assert _same(oracle.e2m1_to_f64(code + 8), -mags[code])   # code 8 is -0


def test_iq4nl_codebook_matches_page_and_round_trips():
    kv = [int(t) for t in golden_lines("iq4nl_codebook.txt")[0].split()]
    assert len(kv) == 16 and all(a < b for a, b in zip(kv, kv[1:]))
    assert [oracle.iq4nl_value(i) for i in range(16)] == kv
    # nearest-code round trip: decoding index i with d = 1 and picking the
    # nearest table entry gives back i
    for i in range(16):
        v = oracle.iq4nl_value(i)
        assert min(range(16), key=lambda j: abs(kv[j] - v)) == i
    # for a generic d the scaled entries stay distinct in fp16, so the round
    # trip holds through fp16 as well
    for dbits in (0x3C00, 0x1400, 0x2A8F, 0x0200):
        d = oracle.f16_to_f64(dbits)
        w = [oracle.f16_to_f64(oracle.f64_to_f16(d * kv[i])) for i in range(16)]
        assert len(set(w)) == 16
        for i in range(16):
            assert min(range(16), key=lambda j: abs(d * kv[j] - w[i])) == i
