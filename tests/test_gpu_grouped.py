"""GPU parity: routing bucket sort (exact) and the routed-expert grouped GEMV
against the oracle (tolerance as for the GEMV)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_tol, dev, from_dev_u16, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu


def _route_gpu(ids, E):
    t, topk = ids.shape
    d_ids = torch.from_numpy(ids).cuda()
    off = torch.full((E + 1,), -7, dtype=torch.int32, device="cuda")
    perm = torch.full((max(1, t * topk),), -7, dtype=torch.int32, device="cuda")
    qmm.qmm_route(d_ids, E, off, perm)
    st = qmm.qmm_sync_check()
    return off.cpu().numpy(), perm.cpu().numpy()[: t * topk], st


@pytest.mark.parametrize("t,topk,E", [(64, 4, 32), (1, 1, 1), (7, 3, 5), (3000, 4, 32), (1024, 8, 256), (5, 2, 200)])
def test_route_matches_oracle(t, topk, E):
    rng = np.random.default_rng(t * 7 + E)
    ids = synth.gen_topk(rng, t, topk, E)
    off, perm, st = _route_gpu(ids, E)
    assert st == 0
    ooff, operm, bad = oracle.route(ids, E)
    assert bad == 0
    assert np.array_equal(off, ooff)
    assert np.array_equal(perm, operm)        # the GPU sort is stable too


def test_route_flags_out_of_range_ids():
    ids = synth.gen_topk(np.random.default_rng(1), 16, 2, 8)
    ids[3, 1] = 8
    ids[0, 0] = -2
    off, perm, st = _route_gpu(ids, 8)
    assert st == 7  # QMM_ERR_DEVICE_FAULT
    ooff, operm, bad = oracle.route(ids, 8)
    assert bad == 2 and np.array_equal(off, ooff) and np.array_equal(perm[: off[8]], operm[: ooff[8]])


def _grouped(w, x_bits, ids, x_per_pair):
    t, topk = ids.shape
    x = to_dev_u16(x_bits)
    d_ids = torch.from_numpy(ids).cuda()
    y = torch.full((t, topk, w.n), 0x5A5A, dtype=torch.int16, device="cuda")
    nb = qmm.qmm_workspace_bytes(qmm.OP_GROUPED, w, 0, t, topk)
    ws = torch.empty((nb,), dtype=torch.uint8, device="cuda")
    qmm.qmm_grouped_gemv(w, x, d_ids, y, x_per_pair=x_per_pair, ws=ws)
    st = qmm.qmm_sync_check()
    return from_dev_u16(y), st


@pytest.mark.parametrize("fmt", [synth.FMT_IQ4_NL, synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
@pytest.mark.parametrize("E,n,k,t,topk,per_pair", [(6, 40, 64, 9, 2, False), (4, 33, 256, 70, 3, True),
                                                    (8, 128, 512, 3, 4, False)])
def test_grouped_vs_oracle(fmt, E, n, k, t, topk, per_pair):
    rng = np.random.default_rng(E * 100 + n + k + fmt)
    p = synth.gen_weights(rng, fmt, n, k, experts=E)
    x = synth.gen_x(rng, t, topk, k) if per_pair else synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    y, st = _grouped(dev(p), x, ids, per_pair)
    assert st == 0
    if per_pair:
        yref = np.empty((t, topk, n)); absy = np.empty((t, topk, n))
        for s in range(topk):
            for tok in range(t):
                e = ids[tok, s]
                de = p.data[e * p.data_stride:(e + 1) * p.data_stride]
                se = None if p.scales is None else p.scales[e * p.scale_stride:(e + 1) * p.scale_stride]
                yy, aa = oracle.matmul(fmt, n, k, de, se, p.global_scale, x[tok, s][None])
                yref[tok, s], absy[tok, s] = yy[0], aa[0]
    else:
        yref, absy = oracle.grouped_gemv(fmt, n, k, p.data, p.data_stride, p.scales, p.scale_stride,
                                         p.global_scale, E, x, ids)
    check_tol(y, yref, absy, "grouped %s" % qmm.qmm_last_variant())


def test_config4_experts_sampled():
    wgu, wdn, x_gu, x_dn, ids = synth.make_experts()
    for w, x, per_pair in ((wgu, x_gu, False), (wdn, x_dn, True)):
        y, st = _grouped(dev(w), x, ids, per_pair)
        assert st == 0
        rng = np.random.default_rng(8)
        for tok in rng.integers(0, 64, 6):
            for s in range(4):
                e = ids[tok, s]
                de = w.data[e * w.data_stride:(e + 1) * w.data_stride]
                xr = x[tok, s][None] if per_pair else x[tok][None]
                rows = rng.integers(0, w.n, 64)
                ys, as_ = oracle.matmul_sampled(w.fmt, w.n, w.k, de, None, 1.0, xr, np.zeros(64, np.int64), rows)
                check_tol(y[tok, s, rows], ys, as_, "config4")


def test_config4_experts_full_output():
    """Every (token, slot, row) of the routed-expert workload (32 experts,
    gate+up 1792 x 2560 and down 2560 x 896, 64 tokens top-4) against the
    oracle element by element."""
    from gpu_util import oracle_grouped_full
    wgu, wdn, x_gu, x_dn, ids = synth.make_experts()
    for w, x, per_pair in ((wgu, x_gu, False), (wdn, x_dn, True)):
        y, st = _grouped(dev(w), x, ids, per_pair)
        assert st == 0
        yref, absy = oracle_grouped_full(w, x, ids, per_pair)
        check_tol(y, yref, absy, "config4 full %s" % qmm.qmm_last_variant())


def test_grouped_rejects_small_workspace():
    rng = np.random.default_rng(2)
    p = synth.gen_iq4nl(rng, 32, 64, experts=4)
    w = dev(p)
    ids = torch.from_numpy(synth.gen_topk(rng, 8, 2, 4)).cuda()
    x = to_dev_u16(synth.gen_x(rng, 8, 64))
    y = torch.empty((8, 2, 32), dtype=torch.int16, device="cuda")
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_grouped_gemv(w, x, ids, y, ws=torch.empty((16,), dtype=torch.uint8, device="cuda"))
    assert e.value.status == 8


@pytest.mark.parametrize("variant", [None, "iq4", "iq4t"])
@pytest.mark.parametrize("E,n,k,t,topk,per_pair", [(3, 64, 256, 50, 2, False), (5, 48, 384, 200, 3, True),
                                                    (2, 16, 128, 2100, 2, False), (32, 32, 128, 1, 4, True)])
def test_grouped_iq4_many_pairs_per_expert(variant, E, n, k, t, topk, per_pair, monkeypatch):
    """IQ4_NL experts with more than 16 pairs each (several token groups per
    expert, whose row tiles land on different CTAs), with the default
    (tile-resident) kernel and the streaming one."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    rng = np.random.default_rng(E * 1000 + n + k + t)
    p = synth.gen_weights(rng, synth.FMT_IQ4_NL, n, k, experts=E)
    x = synth.gen_x(rng, t, topk, k) if per_pair else synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    y, st = _grouped(dev(p), x, ids, per_pair)
    v = qmm.qmm_last_variant()
    assert st == 0, v
    if variant == "iq4t":
        assert "grouped_iq4_tile" in v, v
    elif variant == "iq4":
        assert v.startswith("route+grouped_iq4_stream"), v
    else:
        assert "iq4_tile" in v, v  # default: the tile-resident kernel
    if per_pair:
        xs = x.reshape(t * topk, k)
        yref = np.empty((t * topk, n)); absy = np.empty((t * topk, n))
        for e in range(E):
            sel = np.flatnonzero(ids.reshape(-1) == e)
            if len(sel):
                de = p.data[e * p.data_stride:(e + 1) * p.data_stride]
                yref[sel], absy[sel] = oracle.matmul(synth.FMT_IQ4_NL, n, k, de, None, 1.0, xs[sel])
        yref, absy = yref.reshape(t, topk, n), absy.reshape(t, topk, n)
    else:
        yref, absy = oracle.grouped_gemv(synth.FMT_IQ4_NL, n, k, p.data, p.data_stride, None, 0, 1.0, E, x, ids)
    check_tol(y, yref, absy, "grouped iq4 %s" % v)


@pytest.mark.parametrize("stage", ["0", "1"])
@pytest.mark.parametrize("spec", ["0", "1"])
@pytest.mark.parametrize("E,n,k,t,topk,per_pair", [(32, 1792, 2560, 64, 4, False), (32, 2560, 896, 64, 4, True),
                                                    (32, 2560, 896, 1, 4, True), (7, 1000, 1152, 37, 3, False),
                                                    (4, 72, 4096, 20, 2, False), (2, 72, 4096, 16, 2, False),
                                                    (3, 100, 896, 10, 3, True), (3, 99, 896, 10, 3, False),
                                                    (5, 83, 2560, 12, 2, False)])
def test_grouped_iq4_tile_kernel(stage, spec, E, n, k, t, topk, per_pair, monkeypatch):
    """The tile-resident IQ4_NL kernel with its weight loads before and after
    the dependency wait, its windows read from global memory or from the
    tiles' shared-memory copy (stage; a last tile whose bytes are not whole
    16-byte units, 99 rows at k = 896, stays on global loads), items of two
    tiles (two super-steps per warp, k % 256 == 0) or four (one super-step
    per warp: k = 896, 1152), ragged last items (n = 1000, 72, 99, 83), the
    routed-expert shapes (gate+up 1792 x 2560, down 2560 x 896 at 64 and 1
    tokens), and routing inside the kernel (at most 32 pairs; 16 tokens x 2
    over 2 experts puts more than one token group on an expert)."""
    monkeypatch.setenv("QMM_GEMV_VARIANT", "iq4t")
    monkeypatch.setenv("QMM_IQ4T_SPEC", spec)
    monkeypatch.setenv("QMM_IQ4T_STAGE", stage)
    rng = np.random.default_rng(E * 7 + n + k + t)
    p = synth.gen_weights(rng, synth.FMT_IQ4_NL, n, k, experts=E)
    x = synth.gen_x(rng, t, topk, k) if per_pair else synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    y, st = _grouped(dev(p), x, ids, per_pair)
    v = qmm.qmm_last_variant()
    assert st == 0 and "grouped_iq4_tile" in v, v
    fits = n % 16 == 0 or (k // 128) % 2 == 0 or (n % 16) % 2 == 0
    assert ("stg=1" in v) == (stage == "1" and fits), v
    if per_pair:
        xs = x.reshape(t * topk, k)
        yref = np.empty((t * topk, n)); absy = np.empty((t * topk, n))
        for e in range(E):
            sel = np.flatnonzero(ids.reshape(-1) == e)
            if len(sel):
                de = p.data[e * p.data_stride:(e + 1) * p.data_stride]
                yref[sel], absy[sel] = oracle.matmul(synth.FMT_IQ4_NL, n, k, de, None, 1.0, xs[sel])
        yref, absy = yref.reshape(t, topk, n), absy.reshape(t, topk, n)
    else:
        yref, absy = oracle.grouped_gemv(synth.FMT_IQ4_NL, n, k, p.data, p.data_stride, None, 0, 1.0, E, x, ids)
    check_tol(y, yref, absy, "grouped iq4 tile %s" % v)



@pytest.mark.parametrize("E,n,k,t,topk,per_pair,bad", [(32, 100, 512, 3, 4, False, False),
                                                        (64, 48, 256, 5, 6, True, False),
                                                        (32, 1792, 2560, 1, 4, False, False),
                                                        (40, 64, 896, 3, 4, False, True),
                                                        (33, 16, 256, 8, 4, False, False)])
def test_grouped_iq4_compact_in_kernel_routing(E, n, k, t, topk, per_pair, bad):
    """Fewer pairs than experts (decode): the tile kernel launches CTAs for
    as many experts as there are pairs, slot j taking the j-th distinct id in
    order of first occurrence; tokens that share experts (3 tokens x 4 of 32)
    leave slots empty; an id outside [0, E) is flagged and its row left
    unwritten while every other pair is computed."""
    rng = np.random.default_rng(E * 11 + n + k + t)
    p = synth.gen_weights(rng, synth.FMT_IQ4_NL, n, k, experts=E)
    x = synth.gen_x(rng, t, topk, k) if per_pair else synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    if t >= 3:
        ids[2] = ids[0]  # a token with the same experts as another
    if bad:
        ids[1, 2] = E + 3
    y, st = _grouped(dev(p), x, ids, per_pair)
    v = qmm.qmm_last_variant()
    assert "in_kernel_compact" in v, v
    assert st == (7 if bad else 0), v
    valid = (ids >= 0) & (ids < E)
    assert np.all(y[~valid] == 0x5A5A), v
    safe = np.where(valid, ids, 0)
    if per_pair:
        xs = x.reshape(t * topk, k)
        yref = np.empty((t * topk, n)); absy = np.empty((t * topk, n))
        for e in range(E):
            sel = np.flatnonzero(safe.reshape(-1) == e)
            if len(sel):
                de = p.data[e * p.data_stride:(e + 1) * p.data_stride]
                yref[sel], absy[sel] = oracle.matmul(synth.FMT_IQ4_NL, n, k, de, None, 1.0, xs[sel])
        yref, absy = yref.reshape(t, topk, n), absy.reshape(t, topk, n)
    else:
        yref, absy = oracle.grouped_gemv(synth.FMT_IQ4_NL, n, k, p.data, p.data_stride, None, 0, 1.0, E, x, safe)
    check_tol(y[valid], yref[valid], absy[valid], "compact %s" % v)


@pytest.mark.parametrize("variant", [None, "iq4"])
def test_grouped_iq4_out_of_range_ids_are_left_out_and_flagged(variant, monkeypatch):
    """IQ4_NL experts with ids outside [0, E): the default kernel routes in
    the kernel (no routing pass), the streaming one after the routing sort;
    both flag QMM_ERR_DEVICE_FAULT, leave those pairs' rows unwritten and
    compute every other pair."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    rng = np.random.default_rng(1234)
    E, n, k, t, topk = 6, 64, 256, 12, 2  # 24 pairs: routed inside the kernel by default
    p = synth.gen_weights(rng, synth.FMT_IQ4_NL, n, k, experts=E)
    x = synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    ids[3, 1] = E
    ids[7, 0] = -1
    y, st = _grouped(dev(p), x, ids, False)
    v = qmm.qmm_last_variant()
    assert st == 7, v  # QMM_ERR_DEVICE_FAULT
    valid = (ids >= 0) & (ids < E)
    assert np.all(y[~valid] == 0x5A5A), v
    yref, absy = oracle.grouped_gemv(synth.FMT_IQ4_NL, n, k, p.data, p.data_stride, None, 0, 1.0, E, x,
                                     np.where(valid, ids, 0))
    check_tol(y[valid], yref[valid], absy[valid], "bad ids %s" % v)
