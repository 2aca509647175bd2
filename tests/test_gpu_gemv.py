"""GPU parity: qmm_gemv against the oracle within |y - y_ref| <= 1e-3 *
sum_k |w_k x_k| (+2^-24), plus exact special cases and edge cases."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_tol, dev, f16, from_dev_u16, nz, run_gemv, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu

FMTS = [synth.FMT_IQ4_NL, synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4]


def _case(fmt, n, k, m, seed):
    rng = np.random.default_rng(seed)
    p = synth.gen_weights(rng, fmt, n, k)
    x = synth.gen_x(rng, m, k)
    return p, x


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("n,k,m", [(1, 32, 1), (37, 64, 1), (256, 512, 1), (100, 160, 3), (64, 1024, 8),
                                   (45, 2048, 9), (1000, 2048, 1), (1000, 2048, 5), (999, 4096, 16),
                                   (2000, 4096, 4)])
def test_gemv_vs_oracle(fmt, n, k, m):
    p, x = _case(fmt, n, k, m, 1000 + n + k + m + fmt)
    w = dev(p)
    y = run_gemv(w, x)
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, "%s n=%d k=%d m=%d [%s]" % (fmt, n, k, m, qmm.qmm_last_variant()))


def test_fast_path_is_used_for_streaming_shapes():
    p, x = _case(synth.FMT_FP4G16_F16, 1000, 4096, 1, 5)
    run_gemv(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemv_fp4_splitk")   # 63 tiles: split across clusters
    p, x = _case(synth.FMT_FP4G16_F16, 18560, 4096, 1, 5)
    run_gemv(dev(p), x)
    assert qmm.qmm_last_variant().startswith("gemv_fp4_ldg")      # 1160 tiles: one CTA per tile


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("k,spw,wpc", [(512, 1, 4), (1024, 2, 4), (1536, 3, 4), (2048, 4, 4), (2560, 5, 4),
                                       (3072, 6, 4), (3584, 7, 4), (4096, 8, 4), (5120, 5, 8), (6144, 6, 8),
                                       (7168, 7, 8), (8192, 8, 8)])
@pytest.mark.parametrize("m", [9, 16])
def test_every_two_n_tile_configuration(fmt, k, spw, wpc, m, monkeypatch):
    """Every configuration of the register kernel at 9..16 tokens (two
    n-tiles): 4 warps of 1..8 segments for k <= 4096, 8 warps of 5..8 for
    k = 5120..8192; 40 rows (a ragged tile), m = 9 (a half-empty second
    n-tile) and 16."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "ldg")
    p, x = _case(fmt, 40, k, m, 2600 + k + m + fmt)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_ldg<fmt=%d,nt=2,spw=%d,wpc=%d," % (fmt, spw, wpc)), v
    yref, absy = oracle.matmul(fmt, p.n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("variant", ["ldg", "generic"])
@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3])
@pytest.mark.parametrize("n,k,m", [(1000, 4096, 1), (333, 8192, 3), (64, 2048, 16), (517, 3072, 9)])
def test_every_streaming_variant_vs_oracle(variant, fmt, n, k, m, monkeypatch):
    monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    p, x = _case(fmt, n, k, m, 2000 + n + k + m + fmt)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    want = {"ldg": "gemv_fp4_ldg", "generic": "gemv_generic"}[variant]
    assert v.startswith(want), v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("wide", ["0", "1"])
@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("n,k,m", [(1000, 4096, 1), (333, 8192, 3), (517, 3072, 9), (64, 2048, 16),
                                   (77, 1536, 5), (40, 1024, 1), (129, 2048, 8)])
def test_register_kernel_both_load_layouts(wide, fmt, n, k, m, monkeypatch):
    """The register GEMV with 128-bit loads and with 256-bit loads (segment
    pairs; taken when k % 256 == 0, the warp's segment count is even and the
    codes are 32-byte aligned)."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "ldg")
    monkeypatch.setenv("QMM_GEMV_WIDE", wide)
    p, x = _case(fmt, n, k, m, 3000 + n + k + m + fmt)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_ldg"), v
    spw = int(v.split("spw=")[1].split(",")[0])
    expect_wide = wide == "1" and k % 256 == 0 and spw % 2 == 0
    assert ("wide=1" in v) == expect_wide, v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_MXFP4])
def test_codes_16_byte_aligned_take_the_128_bit_layout(fmt, monkeypatch):
    """Codes that are 16- but not 32-byte aligned (legal in the ABI) must not
    reach the 256-bit loads."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "ldg")
    n, k, m = 300, 4096, 2
    p, x = _case(fmt, n, k, m, 91 + fmt)
    w = dev(p)
    buf = torch.zeros(w.data.numel() + 48, dtype=torch.uint8, device="cuda")
    off = 16 if (buf.data_ptr() + 16) % 32 else 48
    shifted = buf[off:off + w.data.numel()]
    shifted.copy_(w.data.view(torch.uint8).reshape(-1))
    assert shifted.data_ptr() % 32 == 16
    w2 = qmm.PackedWeights(w.fmt, w.n, w.k, shifted, w.scales, w.global_scale)
    y = run_gemv(w2, x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_ldg") and "wide=0" in v, v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("fmt", FMTS)
def test_one_hot_gives_the_decoded_column_bit_exactly(fmt):
    n, k = 300, 4096
    p, _ = _case(fmt, n, k, 1, 77)
    w = dev(p)
    deq = oracle.dequant(fmt, n, k, p.data, p.scales, p.global_scale)
    for col in (0, 1, 777, 4095):
        x = np.zeros((1, k), dtype=np.uint16)
        x[0, col] = 0x3C00
        y = run_gemv(w, x)
        assert np.array_equal(nz(y[0]), nz(deq[:, col])), (fmt, col, qmm.qmm_last_variant())


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3])
def test_config2_in_proj_full(fmt):
    p, x = synth.make_gemv(synth.FP4_IN_PROJ, fmt)
    w = dev(p)
    y = run_gemv(w, x)
    assert qmm.qmm_last_variant().startswith("gemv_fp4_ldg")
    yref, absy = oracle.matmul(fmt, p.n, p.k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, "in_proj")
    y2 = run_gemv(w, x)
    assert np.array_equal(y, y2)                      # deterministic


def test_config1_iq4nl_tiny():
    p, x = synth.make_gemv(synth.IQ4_TINY)
    y = run_gemv(dev(p), x)
    yref, absy = oracle.matmul(p.fmt, p.n, p.k, p.data, None, 1.0, x)
    check_tol(y, yref, absy, "iq4 tiny")


@pytest.mark.parametrize("m", [1, 4, 16])
def test_config3_sweep(m):
    mats = synth.make_sweep()
    rng = np.random.default_rng(31 + m)
    for name, (p, xall) in mats.items():
        x = xall[:m]
        w = dev(p)
        y = run_gemv(w, x)
        if p.n <= 4096:
            yref, absy = oracle.matmul(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x)
            check_tol(y, yref, absy, name)
        else:  # LM head: sampled outputs, first and last rows included
            ri = np.concatenate([[0, p.n - 1], rng.integers(0, p.n, 600)])
            mi = rng.integers(0, m, ri.size)
            ys, as_ = oracle.matmul_sampled(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x, mi, ri)
            check_tol(y[mi, ri], ys, as_, name)
        del w


@pytest.mark.parametrize("m", [1, 16])
def test_lm_head_full_output(m):
    """The whole 256000 x 4096 LM head output at m = 1 and 16 against the
    oracle, element by element (the oracle over row blocks on the host's
    cores)."""
    from gpu_util import oracle_matmul_rows
    mats = synth.make_sweep(mats=[("lm_head", 256000, 4096)])
    p, xall = mats["lm_head"]
    x = np.ascontiguousarray(xall[:m])
    y = run_gemv(dev(p), x)
    yref, absy = oracle_matmul_rows(p.fmt, p.n, p.k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, "lm_head m=%d %s" % (m, qmm.qmm_last_variant()))


def test_gemv_edge_cases():
    p, x = _case(synth.FMT_FP4G16_F16, 64, 256, 2, 3)
    w = dev(p)
    xd = to_dev_u16(x)
    y = torch.zeros((2, 64), dtype=torch.int16, device="cuda")
    qmm.qmm_gemv(w, xd[:0], y[:0])                                    # m = 0: no-op
    with pytest.raises(qmm.QmmError) as e:                              # m = 17
        qmm.qmm_gemv(w, torch.zeros((17, 256), dtype=torch.int16, device="cuda"),
                     torch.zeros((17, 64), dtype=torch.int16, device="cuda"))
    assert e.value.status == 2
    wk0 = qmm.PackedWeights(w.fmt, 64, 0, w.data, w.scales)            # k = 0: y = 0
    y.fill_(77)
    qmm.qmm_gemv(wk0, xd[:, :0].contiguous(), y)
    assert qmm.qmm_sync_check() == 0 and bool((y == 0).all())
    yb = torch.zeros((2 * 64 + 8,), dtype=torch.int16, device="cuda")
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_gemv(w, xd, yb[1:129].view(2, 64))                      # misaligned y
    assert e.value.status == 3


@pytest.mark.parametrize("variant", [None, "iq4t", "generic"])
@pytest.mark.parametrize("n,k,m", [(256, 512, 1), (2000, 4096, 5), (48, 2560, 16), (4096, 8192, 2),
                                   (17600, 1024, 1), (300, 896, 12), (256, 512, 16)])
def test_iq4nl_kernels_vs_oracle(variant, n, k, m, monkeypatch):
    """Each IQ4_NL GEMV kernel: the default choice between the tile-resident
    and the streaming kernel, the tile-resident one forced (k <= 5376 in
    steps of 256, or k <= 2048; a shape it does not take goes to the generic
    kernel) and the generic one."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    p, x = _case(synth.FMT_IQ4_NL, n, k, m, 3000 + n + k + m)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    # default: the tile kernel where it takes the shape (k <= 4096), except
    # very tall matrices at small m and short rows at m > 8
    tiles = (n + 15) // 16
    stream_first = (m > 8 and k < 2048) or (tiles >= 4096 and m <= 8) or (tiles >= 1024 and m == 1)
    tile_ok = (k % 256 == 0 and k <= 5376) or (k % 128 == 0 and k <= 2048)
    default = ("iq4_tile",) if tile_ok and not stream_first else ("gemv_iq4_stream",)
    want = {None: default, "iq4t": ("iq4_tile",) if tile_ok else ("gemv_generic",),
            "generic": ("gemv_generic",)}[variant]
    assert v.startswith(want), v
    yref, absy = oracle.matmul(synth.FMT_IQ4_NL, n, k, p.data, None, 1.0, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("variant", [None, "generic"])
@pytest.mark.parametrize("m", [1, 5, 16])
def test_mxfp4_small_and_normal_scales(variant, m, monkeypatch):
    """MXFP4 groups scaled by one f16x2 multiply (E8M0 103..142) and groups
    scaled through fp32 (0..102: subnormal and zero weights) in the same
    warp."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    rng = np.random.default_rng(77 + m)
    n, k = 96, 4096
    p = synth.gen_fp4(rng, n, k, synth.FMT_MXFP4)
    sc = p.scales.copy()
    sc[::7] = rng.integers(0, 131, size=sc[::7].size)
    sc[:103] = np.arange(103)
    p = synth.Packed(p.fmt, n, k, p.data, sc)
    x = synth.gen_x(rng, m, k)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith(("gemv_generic",) if variant else ("gemv_fp4_ldg", "gemv_fp4_splitk")), v
    yref, absy = oracle.matmul(p.fmt, n, k, p.data, p.scales, 1.0, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("m", [1, 4, 16])
def test_mxfp4_one_multiply_path_gives_the_two_factor_bits(m, monkeypatch):
    """A warp whose scales are all fp16 values multiplies once, a warp with
    any other scale multiplies by both factors; the two give the same bits.
    One tile, two versions of the scales that differ in one group of row 0
    (in range / out of range): rows 1..15 come out bit-identical, although
    the warp holding that group switches paths, and both versions agree
    with the oracle."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "ldg")
    rng = np.random.default_rng(4321 + m)
    n, k = 16, 4096
    p = synth.gen_fp4(rng, n, k, synth.FMT_MXFP4)
    sc = rng.integers(118, 136, size=p.scales.size).astype(np.uint8)  # every group an fp16 value
    sc_b = sc.copy()
    sc_b[5] = 60                                                        # row 0, group 5: 2^-67
    x = synth.gen_x(rng, m, k)
    ys = []
    for scales in (sc, sc_b):
        q = synth.Packed(p.fmt, n, k, p.data, scales)
        y = run_gemv(dev(q), x)
        assert qmm.qmm_last_variant().startswith("gemv_fp4_ldg<fmt=4"), qmm.qmm_last_variant()
        yref, absy = oracle.matmul(q.fmt, n, k, q.data, q.scales, 1.0, x)
        check_tol(y, yref, absy, "mxfp4 one-multiply m=%d" % m)
        ys.append(y)
    assert np.array_equal(ys[0][:, 1:], ys[1][:, 1:])


@pytest.mark.parametrize("variant", [None, "generic"])
def test_mxfp4_huge_scales_overflow_like_the_oracle(variant, monkeypatch):
    """E8M0 bytes 143..254 turn codes >= 1 into fp16 infinities; 0xFF is NaN.
    The outputs of those rows are infinite or NaN exactly where the oracle's
    are, with the same sign."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    rng = np.random.default_rng(5)
    n, k, m = 32, 512, 2
    p = synth.gen_fp4(rng, n, k, synth.FMT_MXFP4)
    sc = p.scales.copy().reshape(n, k // 32)
    sc[0:8, 3] = [143, 150, 160, 180, 200, 220, 240, 254]   # one huge group in rows 0..7
    sc[8, :] = 0xFF                            # a NaN row
    p = synth.Packed(p.fmt, n, k, p.data, sc.reshape(-1))
    x = synth.gen_x(rng, m, k)
    y = f16(run_gemv(dev(p), x))
    with np.errstate(all="ignore"):
        yref, _ = oracle.matmul(p.fmt, n, k, p.data, p.scales, 1.0, x)
    big = ~np.isfinite(yref)
    assert big[:, :9].all() and not big[:, 9:].any()
    assert np.array_equal(np.isnan(y[big]), np.isnan(yref[big]))
    nn = big & ~np.isnan(yref)
    assert np.array_equal(y[nn], yref[nn])      # +-inf, same sign


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_IQ4_NL, synth.FMT_MXFP4])
@pytest.mark.parametrize("pinned", [True, False])
def test_gemv_host_round_trip(fmt, pinned):
    """qmm_gemv_host: host x in, host y out in one call, the same result as
    qmm_gemv on device buffers (bit-exact) and within tolerance of the
    oracle."""
    n, k, m = 1000, 4096, 3
    p, x = _case(fmt, n, k, m, 5000 + fmt)
    w = dev(p)
    xh = torch.from_numpy(x.view(np.int16).copy())
    yh = torch.full((m, n), 0x5A5A, dtype=torch.int16)
    if pinned:
        xh, yh = xh.pin_memory(), yh.pin_memory()
    xd = torch.empty((m, k), dtype=torch.int16, device="cuda")
    yd = torch.empty((m, n), dtype=torch.int16, device="cuda")
    qmm.qmm_gemv_host(w, xh, yh, xd, yd)
    torch.cuda.synchronize()
    assert qmm.qmm_sync_check() == 0
    got = yh.numpy().view(np.uint16)
    yref_dev = run_gemv(w, x)
    assert np.array_equal(got, yref_dev)
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(got, yref, absy, "gemv_host %d" % fmt)


def test_gemv_host_argument_errors():
    p, x = _case(synth.FMT_FP4G16_F16, 64, 256, 2, 9)
    w = dev(p)
    xh = torch.from_numpy(x.view(np.int16).copy())
    yh = torch.empty((2, 64), dtype=torch.int16)
    xd = torch.empty((2, 256), dtype=torch.int16, device="cuda")
    yd = torch.empty((2, 64), dtype=torch.int16, device="cuda")
    with pytest.raises(ValueError):
        qmm.qmm_gemv_host(w, xd, yh, xd, yd)                  # device tensor as the host input
    with pytest.raises(ValueError):
        qmm.qmm_gemv_host(w, xh, yh, xh, yd)                  # host tensor as the device staging buffer
    big = torch.zeros((17, 256), dtype=torch.int16)
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_gemv_host(w, big, torch.empty((17, 64), dtype=torch.int16), torch.empty((17, 256), dtype=torch.int16,
                          device="cuda"), torch.empty((17, 64), dtype=torch.int16, device="cuda"))
    assert e.value.status == 2                                  # m > 16: UNSUPPORTED_SHAPE
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_gemv_host(w, xh, yh, xd, torch.zeros((2 * 64 + 8,), dtype=torch.int16, device="cuda")[1:129])
    assert e.value.status == 3                                  # misaligned y staging buffer



@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("n,k,m", [(1000, 4096, 1), (333, 8192, 4), (517, 2048, 16)])
@pytest.mark.parametrize("how", ["knob", "x16"])
def test_register_kernel_128_bit_activation_loads(fmt, n, k, m, how, monkeypatch):
    """The 16-byte activation loads: forced by QMM_GEMV_XW=0, or taken
    because x is 16- but not 32-byte aligned (legal in the ABI)."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "ldg")
    p, xb = _case(fmt, n, k, m, 7000 + n + k + m + fmt)
    w = dev(p)
    if how == "knob":
        monkeypatch.setenv("QMM_GEMV_XW", "0")
        y = run_gemv(w, xb)
    else:
        buf = torch.zeros(m * k + 32, dtype=torch.int16, device="cuda")
        off = 8 if buf.data_ptr() % 32 == 0 else 0  # elements: x starts 16 bytes past a 32-byte boundary
        xs = buf[off:off + m * k].view(m, k)
        assert xs.data_ptr() % 32 == 16
        xs.copy_(to_dev_u16(xb))
        yd = torch.empty((m, n), dtype=torch.int16, device="cuda")
        qmm.qmm_gemv(w, xs, yd)
        assert qmm.qmm_sync_check() == 0
        y = from_dev_u16(yd)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_ldg") and "xw=0" in v, v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, xb)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("n,k,m,cs", [(100, 4096, 1, 2), (100, 4096, 1, 4), (100, 4096, 1, 8), (333, 8192, 3, 2),
                                      (333, 8192, 3, 8), (77, 2048, 16, 2), (77, 2048, 16, 4), (30, 1024, 9, 2),
                                      (77, 2048, 16, 8), (50, 1536, 5, 4), (40, 3072, 2, 2), (17, 512, 1, 2)])
def test_split_k_clusters_vs_oracle(fmt, n, k, m, cs, monkeypatch):
    """Split-K over a cluster of cs CTAs per 16-row tile (ragged n, m = 1..16),
    reduced through distributed shared memory; split counts that do not
    divide the shape into whole 4-warp CTAs (k = 2048 at cs = 8, k = 1536,
    3072, 512) fall back to the unsplit kernel.  Deterministic: two calls
    give the same bits."""
    monkeypatch.setenv("QMM_GEMV_SPLITK", str(cs))
    p, x = _case(fmt, n, k, m, 8000 + n + k + m + cs + fmt)
    w = dev(p)
    y = run_gemv(w, x)
    v = qmm.qmm_last_variant()
    segs = k // 128
    spw = segs // (4 * cs)
    split = segs % (4 * cs) == 0 and spw in ((1, 2, 4, 8) if m <= 8 else (1, 2, 4))
    assert v.startswith("gemv_fp4_splitk" if split else "gemv_fp4_ldg"), v
    if split:
        assert "cs=%d" % cs in v, v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)
    assert np.array_equal(run_gemv(w, x), y)


@pytest.mark.parametrize("n,k,m,split", [(256, 8192, 1, True), (1000, 4096, 3, True), (2000, 4096, 1, True),
                                         (4096, 8192, 1, False), (4096, 8192, 16, False), (256, 4096, 16, False),
                                         (128, 16384, 16, True), (64, 32768, 2, True)])
def test_split_k_default_dispatch(n, k, m, split):
    """Narrow matrices at m <= 8 take split-K by default, out_proj (256
    tiles) and m > 8 do not, except where the unsplit kernel has no
    configuration for k (k = 16384 at m = 16, k = 32768)."""
    p, x = _case(synth.FMT_FP4G16_F16, n, k, m, 8500 + n + k + m)
    y = run_gemv(dev(p), x)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_splitk" if split else "gemv_fp4_ldg"), v
    yref, absy = oracle.matmul(p.fmt, n, k, p.data, p.scales, p.global_scale, x)
    check_tol(y, yref, absy, v)


@pytest.mark.parametrize("fmt", [synth.FMT_FP4G16_F16, synth.FMT_MXFP4])
@pytest.mark.parametrize("m", [1, 12])
def test_split_k_with_16_byte_aligned_activations(fmt, m, monkeypatch):
    """x 16- but not 32-byte aligned: the split-K kernel takes the 128-bit
    activation loads (xw=0)."""
    monkeypatch.setenv("QMM_GEMV_SPLITK", "4")
    n, k = 200, 4096
    p, xb = _case(fmt, n, k, m, 9100 + m + fmt)
    w = dev(p)
    buf = torch.zeros(m * k + 32, dtype=torch.int16, device="cuda")
    off = 8 if buf.data_ptr() % 32 == 0 else 0
    xs = buf[off:off + m * k].view(m, k)
    assert xs.data_ptr() % 32 == 16
    xs.copy_(to_dev_u16(xb))
    yd = torch.empty((m, n), dtype=torch.int16, device="cuda")
    qmm.qmm_gemv(w, xs, yd)
    assert qmm.qmm_sync_check() == 0
    v = qmm.qmm_last_variant()
    assert v.startswith("gemv_fp4_splitk") and "xw=0" in v, v
    yref, absy = oracle.matmul(fmt, n, k, p.data, p.scales, p.global_scale, xb)
    check_tol(from_dev_u16(yd), yref, absy, v)
