"""GPU parity for the routed-expert block of a mixture-of-experts layer
("Mark-Experimental-V3-8B", section "Mixture-of-Experts (MoE)"): the router
(fp32 logits, softmax, top-k) and the fused gate/up + SiLU, down and weighted
combine, each stage against the oracle on the GPU's own input to it."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import REL, check_tol, dev, f16, from_dev_u16, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu


def _router_gpu(x, w, b, topk, with_logits=True):
    t, E = x.shape[0], w.shape[0]
    ids = torch.full((t, topk), -9, dtype=torch.int32, device="cuda")
    g = torch.full((t, topk), -1.0, dtype=torch.float32, device="cuda")
    z = torch.full((t, E), float("nan"), dtype=torch.float32, device="cuda") if with_logits else None
    qmm.qmm_router_topk(to_dev_u16(x), to_dev_u16(w), torch.from_numpy(b).cuda(), topk, ids, g, z)
    assert qmm.qmm_sync_check() == 0
    return ids.cpu().numpy(), g.cpu().numpy(), None if z is None else z.cpu().numpy()


def _check_router(x, w, b, topk):
    ids, g, z = _router_gpu(x, w, b, topk)
    zr, idr, gr, pr = oracle.router_topk(x, w, b, topk)
    # logits: the same fp64 sum rounded once; summation order may move the
    # fp32 rounding by one unit in the last place at most
    assert np.all(np.abs(z.astype(np.float64) - zr) <= np.spacing(np.abs(zr)).astype(np.float64))
    t = x.shape[0]
    for i in range(t):
        # the GPU's choice is the exact top-k of its own logits (ties to the lower index)
        order = sorted(range(w.shape[0]), key=lambda e: (-float(z[i, e]), e))[:topk]
        assert list(ids[i]) == order, (i, ids[i], order)
        if list(ids[i]) != list(idr[i]):
            # only a near tie may differ from the oracle's choice
            j = int(np.argmax(ids[i] != idr[i]))
            za, zb = float(zr[i, ids[i][j]]), float(zr[i, idr[i][j]])
            assert abs(za - zb) <= 2 * float(np.spacing(np.float32(max(abs(za), abs(zb))))), (i, ids[i], idr[i])
    # weights: the softmax score of each chosen expert (fp32 vs fp64)
    ref = np.take_along_axis(pr, ids.astype(np.int64), axis=1)
    assert np.all(np.abs(g - ref) <= 4e-6 * ref + 1e-30), np.abs(g - ref).max()
    return ids, g


@pytest.mark.parametrize("t,k,E,topk", [(64, 2560, 32, 4), (5, 64, 7, 3), (1, 8, 256, 16), (17, 520, 1, 1),
                                        (3, 24, 40, 40), (300, 128, 32, 4)])
def test_router_vs_oracle(t, k, E, topk):
    rng = np.random.default_rng(t * 1000 + k + E)
    x = synth.gen_x(rng, t, k)
    w, b = synth.gen_router(rng, E, k)
    _check_router(x, w, b, topk)


@pytest.mark.parametrize("cs", ["1", "2", "4", "8"])
@pytest.mark.parametrize("t,k,E,topk", [(1, 2560, 32, 4), (6, 520, 7, 3), (3, 24, 40, 40)])
def test_router_every_cluster_size(cs, t, k, E, topk, monkeypatch):
    """The router's k split over 1, 2, 4 or 8 CTAs per token (k = 24 leaves
    most CTAs of a cluster without a chunk; k = 520 a ragged last chunk)."""
    monkeypatch.setenv("QMM_ROUTER_CS", cs)
    rng = np.random.default_rng(t * 1000 + k + E + int(cs))
    x = synth.gen_x(rng, t, k)
    w, b = synth.gen_router(rng, E, k)
    _check_router(x, w, b, topk)
    assert qmm.qmm_last_variant() == "router_topk<cs=%s>" % cs


def test_router_ties_go_to_the_lower_index():
    rng = np.random.default_rng(5)
    x = synth.gen_x(rng, 4, 256)
    w, b = synth.gen_router(rng, 32, 256)
    w[21] = w[6]
    b[21] = b[6] = np.float32(40.0)   # experts 6 and 21: equal logits, far above the rest
    ids, g = _check_router(x, w, b, 4)
    assert np.all(ids[:, 0] == 6) and np.all(ids[:, 1] == 21)
    assert np.all(g[:, 0] == g[:, 1])


def test_router_empty_k_uses_the_bias():
    b = np.array([0.5, -1.0, 2.0, 2.0], dtype=np.float32)
    x = np.zeros((2, 0), dtype=np.uint16)
    w = np.zeros((4, 0), dtype=np.uint16)
    ids = torch.full((2, 2), -9, dtype=torch.int32, device="cuda")
    g = torch.zeros((2, 2), dtype=torch.float32, device="cuda")
    z = torch.zeros((2, 4), dtype=torch.float32, device="cuda")
    xe = torch.empty((2, 0), dtype=torch.int16, device="cuda")
    we = torch.empty((4, 0), dtype=torch.int16, device="cuda")
    qmm.qmm_router_topk(xe, we, torch.from_numpy(b).cuda(), 2, ids, g, z)
    assert qmm.qmm_sync_check() == 0
    assert np.array_equal(z.cpu().numpy(), np.stack([b, b]))
    assert np.array_equal(ids.cpu().numpy(), [[2, 3], [2, 3]])
    _, _, _, pr = oracle.router_topk(x, w, b, 2)
    assert np.allclose(g.cpu().numpy(), pr[:, [2, 3]], rtol=4e-6, atol=0)


def _ws_parts(E, P, f):
    a = lambda v: (v + 255) // 256 * 256
    h0 = a(4 * (E + 1)) + a(4 * P)
    return h0, h0 + a(2 * P * f)


def _moe_gpu(wgu, wdn, x, ids, g, f):
    t, topk = ids.shape
    E = wgu.experts
    gu = dev(wgu)
    gate, up = gu.rows(0, f), gu.rows(f, 2 * f)
    down = dev(wdn)
    out = torch.full((t, wdn.n), 0x5A5A, dtype=torch.int16, device="cuda")
    nb = qmm.qmm_workspace_bytes(qmm.OP_MOE, gate, 0, t, topk)
    ws = torch.zeros((nb,), dtype=torch.uint8, device="cuda")
    qmm.qmm_moe_routed(gate, up, down, to_dev_u16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(g).cuda(),
                       out, ws=ws)
    st = qmm.qmm_sync_check()
    variant = qmm.qmm_last_variant()
    h0, h1 = _ws_parts(E, t * topk, f)
    h = ws[h0:h0 + 2 * t * topk * f].view(torch.int16).view(t, topk, f)
    return from_dev_u16(out), from_dev_u16(h), st, variant


def _moe_reference_stages(wgu, wdn, x, ids, g, f, h_gpu):
    """(h_ref, h_bound) from the oracle's gate/up products, and (out_ref,
    out_abs) from the oracle's down product of the GPU's own h."""
    d = wgu.k
    E = wgu.experts
    rowb = oracle.data_bytes(1, 1, d)
    yg, ag = oracle.grouped_gemv(1, f, d, wgu.data, wgu.data_stride, None, 0, 1.0, E, x, ids)
    yu, au = oracle.grouped_gemv(1, f, d, wgu.data[f * rowb:], wgu.data_stride, None, 0, 1.0, E, x, ids)
    t, topk = ids.shape
    h_ref = oracle.swiglu(np.concatenate([yg, yu], axis=2).reshape(t * topk, 2 * f)).reshape(t, topk, f)
    with np.errstate(over="ignore"):
        silu_g = yg / (1.0 + np.exp(-yg))
    dg, du = REL * ag, REL * au
    h_bound = 1.1 * dg * (np.abs(yu) + du) + np.abs(silu_g) * du
    h_bound += 2.0 ** -11 * (np.abs(h_ref) + h_bound) + 2.0 ** -24
    # down product of each pair's own h row, one oracle call per expert
    yd = np.zeros((t, topk, wdn.n))
    ad = np.zeros((t, topk, wdn.n))
    for e in range(E):
        sel = np.argwhere(ids == e)
        if len(sel) == 0:
            continue
        de = wdn.data[e * wdn.data_stride:(e + 1) * wdn.data_stride]
        yy, aa = oracle.matmul(1, wdn.n, f, de, None, 1.0, h_gpu[sel[:, 0], sel[:, 1]])
        yd[sel[:, 0], sel[:, 1]] = yy
        ad[sel[:, 0], sel[:, 1]] = aa
    valid = (ids >= 0) & (ids < E)
    gg = np.where(valid, g.astype(np.float64), 0.0)
    yd = np.where(valid[..., None], yd, 0.0)
    ad = np.where(valid[..., None], ad, 0.0)
    out_ref = oracle.combine(yd, gg)
    out_abs = oracle.combine(ad, np.abs(gg))
    return h_ref, h_bound, out_ref, out_abs


@pytest.mark.parametrize("variant", [None, "iq4", "iq4t"])
@pytest.mark.parametrize("E,f,d,t,topk", [(6, 128, 256, 9, 2), (4, 256, 128, 40, 4), (2, 128, 384, 5, 2),
                                          (32, 896, 2560, 64, 4), (32, 896, 2560, 1, 4)])
def test_moe_routed_vs_oracle(E, f, d, t, topk, variant, monkeypatch):
    """Default (and iq4t): tile-resident kernels (routing inside the kernel
    up to 32 pairs, after the routing sort above); iq4: route + streaming
    kernels."""
    if variant:
        monkeypatch.setenv("QMM_GEMV_VARIANT", variant)
    rng = np.random.default_rng(E * 31 + f + d + t)
    wgu = synth.gen_iq4nl(rng, 2 * f, d, E)
    wdn = synth.gen_iq4nl(rng, d, f, E)
    x = synth.gen_x(rng, t, d)
    wr, br = synth.gen_router(rng, E, d)
    ids, g = _check_router(x, wr, br, topk)
    out, h, st, used = _moe_gpu(wgu, wdn, x, ids, g, f)
    assert st == 0, used
    assert ("iq4_tile" in used) == (variant in ("iq4t", None)), used
    variant = used
    h_ref, h_bound, out_ref, out_abs = _moe_reference_stages(wgu, wdn, x, ids, g, f, h)
    err = np.abs(f16(h) - h_ref)
    assert np.all(err <= h_bound), ("h", float((err / h_bound).max()), variant)
    check_tol(out, out_ref, out_abs, "moe out %s" % variant)


def test_moe_shared_experts_as_two_always_on_experts():
    """F_shared: the same call with ids {0, 1} and unit weights."""
    rng = np.random.default_rng(77)
    f, d, t = 128, 256, 12
    wgu = synth.gen_iq4nl(rng, 2 * f, d, 2)
    wdn = synth.gen_iq4nl(rng, d, f, 2)
    x = synth.gen_x(rng, t, d)
    ids = np.tile(np.array([[0, 1]], dtype=np.int32), (t, 1))
    g = np.ones((t, 2), dtype=np.float32)
    out, h, st, variant = _moe_gpu(wgu, wdn, x, ids, g, f)
    assert st == 0
    h_ref, h_bound, out_ref, out_abs = _moe_reference_stages(wgu, wdn, x, ids, g, f, h)
    assert np.all(np.abs(f16(h) - h_ref) <= h_bound)
    check_tol(out, out_ref, out_abs, "shared experts")


def test_moe_out_of_range_ids_are_left_out_and_flagged():
    rng = np.random.default_rng(78)
    E, f, d, t, topk = 4, 128, 128, 6, 2
    wgu = synth.gen_iq4nl(rng, 2 * f, d, E)
    wdn = synth.gen_iq4nl(rng, d, f, E)
    x = synth.gen_x(rng, t, d)
    ids = synth.gen_topk(rng, t, topk, E)
    ids[2, 1] = E
    ids[4, 0] = -1
    g = rng.random((t, topk), dtype=np.float32)
    out, h, st, _ = _moe_gpu(wgu, wdn, x, ids, g, f)
    assert st == 7  # QMM_ERR_DEVICE_FAULT
    _, _, out_ref, out_abs = _moe_reference_stages(wgu, wdn, x, ids, g, f, h)
    check_tol(out, out_ref, out_abs, "moe with bad ids")


def test_moe_rejects_unsupported_shapes():
    rng = np.random.default_rng(79)
    wgu = dev(synth.gen_iq4nl(rng, 2 * 96, 256, 2))       # f = 96: not a multiple of 128
    wdn = dev(synth.gen_iq4nl(rng, 256, 96, 2))
    x = torch.zeros((3, 256), dtype=torch.int16, device="cuda")
    ids = torch.zeros((3, 1), dtype=torch.int32, device="cuda")
    g = torch.ones((3, 1), dtype=torch.float32, device="cuda")
    out = torch.zeros((3, 256), dtype=torch.int16, device="cuda")
    ws = torch.zeros((1 << 20,), dtype=torch.uint8, device="cuda")
    with pytest.raises(qmm.QmmError) as ei:
        qmm.qmm_moe_routed(wgu.rows(0, 96), wgu.rows(96, 192), wdn, x, ids, g, out, ws=ws)
    assert ei.value.status == 2  # QMM_ERR_UNSUPPORTED_SHAPE
    fp4 = dev(synth.gen_fp4(rng, 256, 256, experts=2))
    with pytest.raises(qmm.QmmError) as ei:
        qmm.qmm_moe_routed(fp4.rows(0, 128), fp4.rows(128, 256), dev(synth.gen_iq4nl(rng, 256, 128, 2)),
                           x, ids, g, out, ws=ws)
    assert ei.value.status == 2
