"""GPU parity: qmm_dequant is bit-exact against the oracle (NaN by class)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import dev, from_dev_u16, nan_class_equal
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu

FMTS = [synth.FMT_IQ4_NL, synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4]


def _deq(w):
    out = torch.empty((w.n, w.k), dtype=torch.int16, device="cuda")
    qmm.qmm_dequant(w, out)
    assert qmm.qmm_sync_check() == 0
    return from_dev_u16(out)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k", [(1, 32), (7, 64), (256, 512), (33, 2560), (100, 896), (18560, 4096)])
def test_dequant_random(fmt, n, k):
    rng = np.random.default_rng(100 + n + k + fmt)
    p = synth.gen_weights(rng, fmt, n, k)
    got = _deq(dev(p))
    exp = oracle.dequant(fmt, n, k, p.data, p.scales, p.global_scale)
    assert np.array_equal(got, exp)


def test_dequant_iq4nl_every_scale_and_code():
    dbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    blocks = np.zeros((65536, 18), dtype=np.uint8)
    blocks[:, 0] = dbits & 0xFF
    blocks[:, 1] = dbits >> 8
    blocks[:, 2:] = (np.arange(16) | ((15 - np.arange(16)) << 4)).astype(np.uint8)
    p = synth.Packed(synth.FMT_IQ4_NL, 1024, 32 * 64, blocks.reshape(-1), None)
    got = _deq(dev(p))
    exp = oracle.dequant(p.fmt, p.n, p.k, p.data, None)
    assert nan_class_equal(got, exp)


def test_dequant_fp4_f16_every_scale_and_code():
    sbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8), 65536)
    p = synth.Packed(synth.FMT_FP4G16_F16, 65536, 16, codes, sbits.view(np.uint8).copy())
    got = _deq(dev(p))
    exp = oracle.dequant(p.fmt, p.n, p.k, p.data, p.scales)
    assert nan_class_equal(got, exp)


@pytest.mark.parametrize("g", [1.0, 0.1, 3.0e-5, 1.7e3, 2.0 ** -20, 123.456, 0.013671875])
def test_dequant_fp4_e4m3_every_scale_byte_and_code(g):
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE], dtype=np.uint8), 256)
    p = synth.Packed(synth.FMT_FP4G16_E4M3, 256, 16, codes, np.arange(256, dtype=np.uint8), float(np.float32(g)))
    got = _deq(dev(p))
    exp = oracle.dequant(p.fmt, p.n, p.k, p.data, p.scales, np.float32(g))
    assert nan_class_equal(got, exp)


def test_dequant_empty_and_errors():
    p = synth.gen_fp4(np.random.default_rng(0), 4, 32)
    w = dev(p)
    w0 = qmm.PackedWeights(w.fmt, 0, 32, w.data, w.scales)
    qmm.qmm_dequant(w0, torch.empty((0, 32), dtype=torch.int16, device="cuda"))
    bad = qmm.PackedWeights(w.fmt, 4, 24, w.data, w.scales)          # k not a multiple of 16
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_dequant(bad, torch.empty((4, 24), dtype=torch.int16, device="cuda"))
    assert e.value.status == 2
    out = torch.empty((4 * 32 + 8,), dtype=torch.int16, device="cuda")
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_dequant(w, out[1:129])                                   # 2-byte offset: misaligned
    assert e.value.status == 3
    assert qmm.qmm_sync_check() == 0


def test_dequant_mxfp4_every_scale_byte_and_code():
    """All 256 E8M0 bytes x all 16 codes: the bytes whose power of two is an
    fp16 value take one f16x2 multiply, the others the fp32 path."""
    codes = np.tile(np.array([0x10, 0x32, 0x54, 0x76, 0x98, 0xBA, 0xDC, 0xFE] * 2, dtype=np.uint8), 256)
    p = synth.Packed(synth.FMT_MXFP4, 256, 32, codes, np.arange(256, dtype=np.uint8))
    got = _deq(dev(p))
    exp = oracle.dequant(p.fmt, p.n, p.k, p.data, p.scales)
    assert nan_class_equal(got, exp)
