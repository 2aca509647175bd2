"""Pins of the oracle's mixture-of-experts pieces ("Mark-Experimental-V3-8B",
section "Mixture-of-Experts (MoE)"): router softmax and top-k, SiLU /
SwiGLU, and the weighted combine."""
import math

import numpy as np
import pytest

import oracle
from packed_bit_weight_b200 import synth


def _router_case(seed, t=9, k=64, E=32):
    rng = np.random.default_rng(seed)
    x = synth.gen_x(rng, t, k)
    w = synth.gen_x(rng, E, k)
    b = (rng.standard_normal(E) * 0.5).astype(np.float32)
    return x, w, b


def test_router_softmax_and_topk_brute_force():
    x, w, b = _router_case(1)
    logits, ids, g, probs = oracle.router_topk(x, w, b, 4)
    assert np.allclose(probs.sum(axis=1), 1.0, atol=1e-15)
    xf = x.view(np.float16).astype(np.float64)
    wf = w.view(np.float16).astype(np.float64)
    z = (xf @ wf.T + b.astype(np.float64)).astype(np.float32)     # independent evaluation, fp32 rounding
    assert np.array_equal(z, logits)
    for i in range(x.shape[0]):
        order = sorted(range(w.shape[0]), key=lambda e: (-float(z[i, e]), e))[:4]
        assert list(ids[i]) == order
        ez = np.exp(z[i].astype(np.float64) - z[i].max())
        assert np.allclose(g[i], (ez / ez.sum())[order], rtol=1e-14)


def test_router_zero_weights_reduce_to_bias_order():
    x, w, b = _router_case(2)
    w[:] = 0
    b = np.array([0.5, 3.0, -1.0, 3.0, 2.0, 0.1], dtype=np.float32)
    logits, ids, g, probs = oracle.router_topk(x, w[:6], b, 3)
    for i in range(x.shape[0]):
        assert list(ids[i]) == [1, 3, 4]                              # tie 3.0: lower index first
        e = np.exp(b.astype(np.float64) - 3.0)
        assert np.allclose(g[i], (e / e.sum())[[1, 3, 4]], rtol=1e-14)


def test_router_one_hot_reads_one_weight_column():
    _, w, b = _router_case(3)
    x = np.zeros((1, w.shape[1]), dtype=np.uint16)
    x[0, 5] = 0x3C00
    logits, _, _, _ = oracle.router_topk(x, w, b, 2)
    exp = (w[:, 5].view(np.float16).astype(np.float64) + b).astype(np.float32)
    assert np.array_equal(logits[0], exp)


def test_silu_closed_forms():
    assert oracle.silu(0.0) == 0.0
    assert math.isclose(oracle.silu(math.log(3.0)), 0.75 * math.log(3.0), rel_tol=1e-15)   # sigma(ln 3) = 3/4
    assert math.isclose(oracle.silu(-math.log(3.0)), -0.25 * math.log(3.0), rel_tol=1e-15)
    for z in (0.3, 1.7, 5.0):                       # silu(z) - silu(-z) = z
        assert math.isclose(oracle.silu(z) - oracle.silu(-z), z, rel_tol=1e-14)
    assert oracle.silu(60.0) == pytest.approx(60.0, rel=1e-20)
    assert abs(oracle.silu(-60.0)) < 1e-24


def test_swiglu_halves_and_combine_linearity():
    rng = np.random.default_rng(4)
    gu = rng.standard_normal((5, 8))
    h = oracle.swiglu(gu)
    for p in range(5):
        for j in range(4):
            assert h[p, j] == pytest.approx(oracle.silu(gu[p, j]) * gu[p, 4 + j], rel=1e-15)
    y = rng.standard_normal((3, 2, 7))
    g = rng.random((3, 2))
    out = oracle.combine(y, g)
    assert np.allclose(out, np.einsum("ts,tsn->tn", g, y), rtol=1e-14)
    g1 = np.zeros((3, 2)); g1[:, 1] = 1.0           # one slot with weight 1 returns that slot
    assert np.array_equal(oracle.combine(y, g1), y[:, 1, :])
