"""GPU parity: qmm_gemm (tcgen05 prefill GEMM) against the oracle within
|y - y_ref| <= 1e-3 * sum_k |w_k x_k| (+2^-24), plus exact special cases."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_tol, dev, from_dev_u16, nz, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu


def run_gemm(w, x_bits, canary=64):
    m = x_bits.shape[0]
    x = to_dev_u16(x_bits)
    yb = torch.full((m * w.n + canary,), 0x5A5A, dtype=torch.int16, device="cuda")
    y = yb[: m * w.n].view(m, w.n)
    qmm.qmm_gemm(w, x, y)
    st = qmm.qmm_sync_check()
    assert st == 0, "qmm_sync_check -> %s" % qmm.STATUS.get(st, st)
    assert bool((yb[m * w.n:] == 0x5A5A).all()), "write past the end of y"
    return from_dev_u16(y)


@pytest.mark.parametrize("variant", ["persistent", "tile"])
@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("m,n,k", [(128, 256, 64), (128, 256, 256), (256, 384, 512), (200, 300, 1024),
                                   (64, 128, 128), (384, 1000, 2048), (2560, 2048, 64), (2048, 2560, 256)])
def test_gemm_vs_oracle(variant, fmt, m, n, k, monkeypatch):
    monkeypatch.setenv("QMM_GEMM_VARIANT", variant)
    rng = np.random.default_rng(500 + m + n + k + fmt)
    p = synth.gen_fp4(rng, n, k, fmt)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    v = qmm.qmm_last_variant()
    # the persistent kernel stages packed weights in 256-wide k chunks; MXFP4
    # has only that tensor-core kernel (other k: the decode kernel per row block)
    if fmt == synth.FMT_MXFP4:
        want = "gemm_fp4_tc_persistent" if (variant == "persistent" and k % 256 == 0) else "gemm_by_gemv"
    else:
        want = "gemm_fp4_tc_persistent" if (variant == "persistent" and k % 256 == 0) else "gemm_fp4_tc<"
    assert v.startswith(want), v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, "gemm m=%d n=%d k=%d" % (m, n, k))


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
def test_gemm_identity_rows_give_decoded_weights(fmt):
    """X = [I | 0]: row i of Y is column i of the decoded W, bit-exactly."""
    rng = np.random.default_rng(9)
    m, n, k = 128, 512, 256
    p = synth.gen_fp4(rng, n, k, fmt)
    x = np.zeros((m, k), dtype=np.uint16)
    x[np.arange(m), np.arange(m)] = 0x3C00
    y = run_gemm(dev(p), x)
    deq = oracle.dequant(fmt, n, k, p.data, p.scales, p.global_scale)
    # a sum that starts from +0 returns +0 for a -0 weight: compare values
    # bit-exactly with the sign of zero normalised
    assert np.array_equal(nz(y), nz(deq[:, :m].T))


def test_gemm_small_m_uses_decode_kernel_and_agrees():
    rng = np.random.default_rng(4)
    p = synth.gen_fp4(rng, 300, 512)
    x = synth.gen_x(rng, 20, 512)
    y = run_gemm(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemm_by_gemv")
    yref, absy = oracle.matmul(p.fmt, p.n, p.k, p.data, p.scales, 1.0, x)
    check_tol(y, yref, absy, "small m")


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4, synth.FMT_IQ4_NL])
@pytest.mark.parametrize("m", [17, 32, 33, 48, 63])
@pytest.mark.parametrize("variant", [None, "tc", "gemv"])
def test_gemm_decode_batches_17_to_63(fmt, m, variant, monkeypatch):
    """Batches between the decode GEMV's 16 tokens and the tensor-core
    tiles: the default (16-token GEMV slices), the tensor-core kernel forced
    at small m (rows past m masked), and the slices forced; 16-row tiles with
    a ragged tail of rows (n = 1000), k spanning several 128-wide segments."""
    if variant:
        monkeypatch.setenv("QMM_GEMM_VARIANT", variant)
    rng = np.random.default_rng(700 + m + 10 * fmt)
    n, k = 1000, 1024
    p = synth.gen_weights(rng, fmt, n, k)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemm_fp4_tc_persistent" if variant == "tc" else
                        "gemm_by_gemv[slices=%d]:" % ((m + 15) // 16)), v
    yref, absy = oracle.matmul(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, "gemm m=%d fmt=%d %s" % (m, fmt, variant))


def test_gemm_iq4nl():
    rng = np.random.default_rng(6)
    p = synth.gen_iq4nl(rng, 100, 256)
    x = synth.gen_x(rng, 40, 256)
    y = run_gemm(dev(p), x)
    yref, absy = oracle.matmul(p.fmt, p.n, p.k, p.data, None, 1.0, x)
    check_tol(y, yref, absy, "iq4 gemm")


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3])
def test_config5_prefill_full_size_sampled(fmt):
    p, x = synth.make_prefill(fmt)
    w = dev(p)
    y = run_gemm(w, x)
    assert qmm.qmm_last_variant().startswith("gemm_fp4_tc")
    rng = np.random.default_rng(44)
    mi = np.concatenate([[0, 0, p.k and 2047, 2047], rng.integers(0, 2048, 1500)])
    ri = np.concatenate([[0, p.n - 1, 0, p.n - 1], rng.integers(0, p.n, 1500)])
    # plus one full row and one full column of the output
    ys, as_ = oracle.matmul_sampled(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x, mi, ri)
    check_tol(y[mi, ri], ys, as_, "prefill sampled")
    col = np.full(2048, 18559)
    ys, as_ = oracle.matmul_sampled(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x, np.arange(2048), col)
    check_tol(y[np.arange(2048), col], ys, as_, "prefill last column")
    y2 = run_gemm(w, x)
    assert np.array_equal(y, y2)  # deterministic


@pytest.mark.parametrize("m,path", [(32, "gemm_by_gemv[slices=2]:"), (48, "gemm_fp4_tc_persistent")])
def test_in_proj_decode_batches_sampled(m, path):
    """The in_proj matrix (18560 x 4096) at decode batches of 32 and 48: the
    dispatch takes the GEMV slices at 32 tokens and the tensor-core GEMM at
    48 (the measured crossover); sampled outputs against the oracle, every
    token of the first and last rows."""
    p, _ = synth.make_gemv(synth.FP4_IN_PROJ)
    x = synth.gen_x(np.random.default_rng(90 + m), m, p.k)
    y = run_gemm(dev(p), x)
    assert qmm.qmm_last_variant().startswith(path), qmm.qmm_last_variant()
    rng = np.random.default_rng(91)
    mi = np.concatenate([np.arange(m), np.arange(m), rng.integers(0, m, 1000)])
    ri = np.concatenate([np.zeros(m, np.int64), np.full(m, p.n - 1), rng.integers(0, p.n, 1000)])
    ys, as_ = oracle.matmul_sampled(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x, mi, ri)
    check_tol(y[mi, ri], ys, as_, "in_proj m=%d sampled" % m)


def test_gemm_mxfp4_small_and_normal_scales():
    """The tensor-core decode of MXFP4 groups through f16x2 (E8M0 103..142)
    and through fp32 (0..102) in one tile."""
    rng = np.random.default_rng(31)
    m, n, k = 256, 512, 1024
    p = synth.gen_fp4(rng, n, k, synth.FMT_MXFP4)
    sc = p.scales.copy()
    sc[::5] = rng.integers(0, 131, size=sc[::5].size)
    p = synth.Packed(p.fmt, n, k, p.data, sc)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemm_fp4_tc_persistent<fmt=4")
    yref, absy = oracle.matmul(p.fmt, n, k, p.data, p.scales, 1.0, x)
    check_tol(y, yref, absy, "gemm mxfp4 scales")


@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (200, 300, 1024), (384, 1000, 2048), (64, 17, 512),
                                   (2048, 1792, 2560), (256, 512, 384)])
def test_gemm_iq4nl_tensor_cores(m, n, k):
    """IQ4_NL prefill on the persistent tcgen05 kernel (k % 256 == 0; other k
    take the decode kernel per 16-row slice): ragged m and n tiles, one
    routed expert's gate+up shape."""
    rng = np.random.default_rng(600 + m + n + k)
    p = synth.gen_iq4nl(rng, n, k)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemm_fp4_tc_persistent<fmt=1" if k % 256 == 0 else "gemm_by_gemv"), v
    if m * n * k > 2 ** 31:
        rows = rng.integers(0, m, 48)
        cols = rng.integers(0, n, 48)
        ys, as_ = oracle.matmul_sampled(p.fmt, n, k, p.data, None, 1.0, x, rows, cols)
        check_tol(y[rows, cols], ys, as_, v)
    else:
        yref, absy = oracle.matmul(p.fmt, n, k, p.data, None, 1.0, x)
        check_tol(y, yref, absy, v)


def test_gemm_iq4nl_identity_rows_give_decoded_weights():
    """X = [I | 0]: row i of Y is column i of the decoded IQ4_NL W, bit-exactly."""
    rng = np.random.default_rng(10)
    m, n, k = 128, 512, 256
    p = synth.gen_iq4nl(rng, n, k)
    x = np.zeros((m, k), dtype=np.uint16)
    x[np.arange(m), np.arange(m)] = 0x3C00
    y = run_gemm(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemm_fp4_tc_persistent<fmt=1")
    deq = oracle.dequant(p.fmt, n, k, p.data, None)
    assert np.array_equal(nz(y), nz(deq[:, :m].T))


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4, synth.FMT_IQ4_NL])
@pytest.mark.parametrize("m,n,k", [(256, 128, 256), (200, 300, 1024), (300, 1000, 512), (64, 17, 512),
                                   (2048, 640, 2560), (520, 200, 768)])
def test_gemm_256_token_tiles(fmt, m, n, k, monkeypatch):
    """The persistent kernel with 256-token x 128-row tiles (two M=128 MMAs
    per k16 step on the same decoded weights, two accumulator halves): ragged
    m (the second half partly or wholly past m) and n (64-row last tiles)."""
    monkeypatch.setenv("QMM_GEMM_MH", "2")
    rng = np.random.default_rng(700 + m + n + k + fmt)
    p = synth.gen_weights(rng, fmt, n, k)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemm_fp4_tc_persistent<fmt=%d,bm=256,bn=128" % fmt), v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_MXFP4, synth.FMT_IQ4_NL])
def test_gemm_256_token_tiles_identity_rows(fmt, monkeypatch):
    """X = [I | 0] over 256 tokens: both accumulator halves return the decoded
    weight columns bit-exactly."""
    monkeypatch.setenv("QMM_GEMM_MH", "2")
    rng = np.random.default_rng(11 + fmt)
    m, n, k = 256, 384, 512
    p = synth.gen_weights(rng, fmt, n, k)
    x = np.zeros((m, k), dtype=np.uint16)
    x[np.arange(m), np.arange(m)] = 0x3C00
    y = run_gemm(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemm_fp4_tc_persistent<fmt=%d,bm=256" % fmt)
    deq = oracle.dequant(fmt, n, k, p.data, p.scales, p.global_scale)
    assert np.array_equal(nz(y), nz(deq[:, :m].T))


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_IQ4_NL])
@pytest.mark.parametrize("m,n,k", [(128, 256, 256), (200, 300, 1024)])
def test_gemm_128_token_tiles_forced(fmt, m, n, k, monkeypatch):
    """The 128-token x 256-row tiles (the default below m = 256), forced."""
    monkeypatch.setenv("QMM_GEMM_MH", "1")
    rng = np.random.default_rng(800 + m + n + k + fmt)
    p = synth.gen_weights(rng, fmt, n, k)
    x = synth.gen_x(rng, m, k)
    y = run_gemm(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemm_fp4_tc_persistent<fmt=%d,bm=128,bn=256" % fmt), v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)
