"""GPU parity: qmm_quantize (fp16 weights -> packed bytes) is byte-identical
to the oracle's encoder: random weights over many magnitudes, the
hand-worked rows, zeros, fp16 subnormals and ties, for every encoded format;
quantize then dequantize gives the oracle's decoded weights."""
import numpy as np
import pytest
import torch

import oracle
from conftest import golden_lines, parse_value
from gpu_util import from_dev_u16, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu

FMTS = [synth.FMT_FP4G16_F16, synth.FMT_MXFP4, synth.FMT_IQ4_NL]
NAMES = {"fp4g16_f16": synth.FMT_FP4G16_F16, "mxfp4": synth.FMT_MXFP4, "iq4_nl": synth.FMT_IQ4_NL}


def _gpu_quantize(fmt, w_bits):
    n, k = w_bits.shape
    w = to_dev_u16(w_bits).view(n, k)
    data = torch.full((max(qmm.qmm_data_bytes(fmt, n, k), 1),), 0xA5, dtype=torch.uint8, device="cuda")
    sb = qmm.qmm_scale_bytes(fmt, n, k)
    scales = torch.full((sb,), 0xA5, dtype=torch.uint8, device="cuda") if sb else None
    qmm.qmm_quantize(fmt, w, data, scales)
    assert qmm.qmm_sync_check() == 0
    return data.cpu().numpy()[: qmm.qmm_data_bytes(fmt, n, k)], (scales.cpu().numpy() if sb else None)


def _weights(rng, n, k):
    """fp16 weights over many magnitudes per row, with zeros, subnormals,
    exact E2M1 multiples and a negative zero sprinkled in."""
    w = rng.standard_normal((n, k)) * np.exp(rng.uniform(-12, 6, size=(n, 1)))
    w[rng.random((n, k)) < 0.05] = 0.0
    w[rng.random((n, k)) < 0.02] = rng.choice([0.25, 0.75, 1.25, 2.5, 5.0, -0.75, -5.0], size=1)[0]
    bits = w.astype(np.float16).view(np.uint16).copy()
    bits[rng.random((n, k)) < 0.01] = 0x8000
    bits[rng.random((n, k)) < 0.01] = rng.integers(1, 0x400, size=1)[0]   # subnormal
    return bits


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k", [(1, 32), (7, 64), (100, 512), (33, 2560), (257, 4096)])
def test_quantize_matches_oracle(fmt, n, k):
    rng = np.random.default_rng(900 + n + k + fmt)
    w = _weights(rng, n, k)
    d, s = _gpu_quantize(fmt, w)
    od, os_ = oracle.quantize(fmt, n, k, w)
    assert np.array_equal(d, od), qmm.qmm_last_variant()
    if os_ is not None:
        assert np.array_equal(s, os_)
    # and the round trip decodes like the oracle's decoder
    pw = qmm.PackedWeights(fmt, n, k, torch.from_numpy(d).cuda(), None if s is None else torch.from_numpy(s).cuda())
    out = torch.empty((n, k), dtype=torch.int16, device="cuda")
    qmm.qmm_dequant(pw, out)
    assert np.array_equal(from_dev_u16(out), oracle.dequant(fmt, n, k, od, os_))


def test_quantize_handmade_rows():
    lines = golden_lines("quantize_handmade.txt")
    for i in range(0, len(lines), 4):
        fmt = NAMES[lines[i].split()[1]]
        w = np.array([parse_value(t) for t in lines[i + 1].split()[1:]], dtype=np.float64)
        bits = w.astype(np.float16).view(np.uint16)[None, :]
        d, s = _gpu_quantize(fmt, bits)
        assert bytes(d) == bytes(int(t, 16) for t in lines[i + 3].split()[1:]), lines[i]
        assert (b"" if s is None else bytes(s)) == bytes(int(t, 16) for t in lines[i + 2].split()[1:]), lines[i]


def test_quantize_special_values():
    """All-zero groups, infinities and NaNs: the oracle's reading (code 0 for
    NaN, the largest MX scale for an infinite amax)."""
    n, k = 4, 64
    w = np.zeros((n, k), dtype=np.uint16)
    w[1, 3] = 0x7C00            # +inf
    w[2, 40] = 0xFC00           # -inf
    w[3, 7] = 0x7E00            # NaN
    w[3, 8] = 0x3C00            # 1.0
    for fmt in FMTS:
        d, s = _gpu_quantize(fmt, w)
        od, os_ = oracle.quantize(fmt, n, k, w)
        assert np.array_equal(d, od), fmt
        if os_ is not None:
            assert np.array_equal(s, os_), fmt


def test_quantize_rejects_e4m3_and_ragged_k():
    w = torch.zeros((2, 32), dtype=torch.int16, device="cuda")
    data = torch.zeros((64,), dtype=torch.uint8, device="cuda")
    sc = torch.zeros((64,), dtype=torch.uint8, device="cuda")
    with pytest.raises(qmm.QmmError):
        qmm.qmm_quantize(synth.FMT_FP4G16_E4M3, w, data, sc)
    w2 = torch.zeros((2, 48), dtype=torch.int16, device="cuda")
    with pytest.raises(qmm.QmmError):
        qmm.qmm_quantize(synth.FMT_MXFP4, w2, data, sc)


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_MXFP4])
def test_quantize_then_gemv_back_to_back_on_one_stream(fmt):
    """qmm_quantize writes packed W and qmm_gemv, next on the same stream
    with nothing in between, reads W before its dependency wait: the GEMV
    must see the encoded bytes (the oracle's product of the oracle's
    encoding), also when the same buffers held other weights just before."""
    from gpu_util import check_tol
    rng = np.random.default_rng(77 + fmt)
    n, k, m = 4096, 4096, 2
    # moderate weights, so that every sum stays inside the fp16 range
    w_old, w_new = [(rng.standard_normal((n, k)) * 0.02).astype(np.float16).view(np.uint16) for _ in range(2)]
    x_bits = synth.gen_x(rng, m, k)
    data = torch.empty((qmm.qmm_data_bytes(fmt, n, k),), dtype=torch.uint8, device="cuda")
    scales = torch.empty((qmm.qmm_scale_bytes(fmt, n, k),), dtype=torch.uint8, device="cuda")
    x = to_dev_u16(x_bits)
    y = torch.empty((m, n), dtype=torch.int16, device="cuda")
    pw = qmm.PackedWeights(fmt, n, k, data, scales)
    st = torch.cuda.current_stream()
    qmm.qmm_quantize(fmt, to_dev_u16(w_old).view(n, k), data, scales, stream=st)
    wd = to_dev_u16(w_new).view(n, k)
    torch.cuda.synchronize()
    for _ in range(3):
        qmm.qmm_quantize(fmt, wd, data, scales, stream=st)
        qmm.qmm_gemv(pw, x, y, stream=st)
    assert qmm.qmm_sync_check() == 0
    od, os_ = oracle.quantize(fmt, n, k, w_new)
    yref, absy = oracle.matmul(fmt, n, k, od, os_, 1.0, x_bits)
    check_tol(from_dev_u16(y), yref, absy, "quantize->gemv " + qmm.qmm_last_variant())
