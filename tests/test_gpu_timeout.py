"""The bounded-wait failure path of the tensor-core GEMMs (and of the
routed-expert tile kernel's copy wait, last test), made to run out
without faulting anything: with the activation tile loads withheld (a test
switch of the library), the MMA issuer's wait for the first stage never
completes; after the wait limit (lowered to 1 ms for the test) every role of
the kernel gives up, the kernel raises QMM_ERR_TIMEOUT in the device error
word, drains its own copies and MMAs, frees its tensor memory and returns.
qmm_sync_check reports the timeout once and clears it; the next normal call
on the same device (which allocates tensor memory again) gives the oracle's
result, so the context stayed usable and nothing leaked."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import check_tol, dev, from_dev_u16, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu

QMM_ERR_TIMEOUT = 6


@pytest.fixture
def debug_reset():
    yield
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_X_TILES, 0)
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_TILE_COPIES, 0)
    qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 2_000_000_000)


@pytest.mark.parametrize("variant,k", [("persistent", 512), ("tile", 320)])
def test_gemm_wait_runs_out_reports_timeout_and_recovers(variant, k, monkeypatch, debug_reset):
    monkeypatch.setenv("QMM_GEMM_VARIANT", variant)
    rng = np.random.default_rng(4242 + k)
    m, n = 256, 384
    p = synth.gen_weights(rng, synth.FMT_FP4G16_F16, n, k)
    x_bits = synth.gen_x(rng, m, k)
    w = dev(p)
    x = to_dev_u16(x_bits)
    y = torch.full((m, n), 0x5A5A, dtype=torch.int16, device="cuda")
    assert qmm.qmm_sync_check() == 0
    qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 1_000_000)
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_X_TILES, 1)
    qmm.qmm_gemm(w, x, y)
    v = qmm.qmm_last_variant()
    assert v.startswith("gemm_fp4_tc_persistent" if variant == "persistent" else "gemm_fp4_tc<"), v
    assert qmm.qmm_sync_check() == QMM_ERR_TIMEOUT
    assert qmm.qmm_sync_check() == 0                      # reported once, then cleared
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_X_TILES, 0)
    qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 2_000_000_000)
    for _ in range(2):                                     # tensor memory is allocated again and again
        qmm.qmm_gemm(w, x, y)
        assert qmm.qmm_sync_check() == 0
    yref, absy = oracle.matmul(p.fmt, n, k, p.data, p.scales, p.global_scale, x_bits)
    check_tol(from_dev_u16(y), yref, absy, "after timeout " + v)


def test_expert_tile_copy_wait_runs_out_reports_timeout_and_recovers(debug_reset):
    """The routed-expert tile kernel's wait for its bulk copies (tiles and
    pair table, announced on its mbarrier) runs out when the copies are
    withheld: QMM_ERR_TIMEOUT once, then a normal call gives the oracle's
    result."""
    rng = np.random.default_rng(4343)
    E, n, k, t, topk = 4, 64, 512, 8, 2  # 16 pairs: routed inside the kernel, tiles staged
    p = synth.gen_weights(rng, synth.FMT_IQ4_NL, n, k, experts=E)
    x_bits = synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    w = dev(p)
    x = to_dev_u16(x_bits)
    d_ids = torch.from_numpy(ids).cuda()
    y = torch.full((t, topk, n), 0x5A5A, dtype=torch.int16, device="cuda")
    ws = torch.empty((qmm.qmm_workspace_bytes(qmm.OP_GROUPED, w, 0, t, topk),), dtype=torch.uint8, device="cuda")
    assert qmm.qmm_sync_check() == 0
    qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 1_000_000)
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_TILE_COPIES, 1)
    qmm.qmm_grouped_gemv(w, x, d_ids, y, ws=ws)
    v = qmm.qmm_last_variant()
    assert "iq4_tile" in v and "stg=1" in v, v
    assert qmm.qmm_sync_check() == QMM_ERR_TIMEOUT
    assert qmm.qmm_sync_check() == 0
    qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_TILE_COPIES, 0)
    qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 2_000_000_000)
    qmm.qmm_grouped_gemv(w, x, d_ids, y, ws=ws)
    assert qmm.qmm_sync_check() == 0
    yref, absy = oracle.grouped_gemv(p.fmt, n, k, p.data, p.data_stride, None, 0, 1.0, E, x_bits, ids)
    check_tol(from_dev_u16(y), yref, absy, "after timeout " + v)


def test_debug_hook_rejects_bad_values():
    with pytest.raises(qmm.QmmError):
        qmm.qmm_debug_set(qmm.DEBUG_WAIT_LIMIT_NS, 10)     # below 1 us
    with pytest.raises(qmm.QmmError):
        qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_X_TILES, 7)
    with pytest.raises(qmm.QmmError):
        qmm.qmm_debug_set(qmm.DEBUG_WITHHOLD_TILE_COPIES, 2)
    with pytest.raises(qmm.QmmError):
        qmm.qmm_debug_set(99, 0)
