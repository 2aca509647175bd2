"""The allocation-free grouped GEMV entry point.

qmm_grouped_gemv_noalloc serves callers that cannot allocate device memory
(a runtime that hands out all device memory from its own fixed pool, or a
serving loop that must not block in the allocator) and therefore cannot pass
the routing workspace that qmm_grouped_gemv takes.  Its routing scratch is a
fixed array inside the library.  This file checks, through the C ABI, that
two calls in a row give the oracle's results and the workspace entry point's,
within the tolerance the other parity tests use, that further calls take no
device memory, and that calls beyond the array's limit are refused.  It is
collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import REL, ABS, dev, f16, from_dev_u16, to_dev_u16
from packed_bit_weight_b200 import qmm, synth

pytestmark = pytest.mark.gpu


def _case(seed, fmt, E, n, k, t, topk, per_pair):
    rng = np.random.default_rng(seed)
    p = synth.gen_weights(rng, fmt, n, k, experts=E)
    x = synth.gen_x(rng, t, topk, k) if per_pair else synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    return p, x, ids


def _oracle_y(p, fmt, n, k, x_bits, ids_np, per_pair):
    """The oracle's product for every (token, slot) and its tolerance scale
    sum_k |w_k x_k|."""
    t, topk = ids_np.shape
    yref, absy = np.empty((t, topk, n)), np.empty((t, topk, n))
    for tok in range(t):
        for s in range(topk):
            e = ids_np[tok, s]
            de = p.data[e * p.data_stride:(e + 1) * p.data_stride]
            se = None if p.scales is None else p.scales[e * p.scale_stride:(e + 1) * p.scale_stride]
            xr = x_bits[tok, s][None] if per_pair else x_bits[tok][None]
            yr, ar = oracle.matmul(fmt, n, k, de, se, p.global_scale, xr)
            yref[tok, s], absy[tok, s] = yr[0], ar[0]
    return yref, absy


def test_noalloc_matches_oracle_and_workspace_entry_point_on_two_calls():
    # two different calls in a row: the second reuses the library's scratch
    # array after the first and must not see anything left over from it
    cases = [(71, synth.FMT_IQ4_NL, 8, 96, 256, 40, 4, False),
             (72, synth.FMT_FP4G16_F16, 5, 64, 512, 300, 2, True)]
    for seed, fmt, E, n, k, t, topk, per_pair in cases:
        p, x_bits, ids_np = _case(seed, fmt, E, n, k, t, topk, per_pair)
        w = dev(p)
        x = to_dev_u16(x_bits)
        ids = torch.from_numpy(ids_np).cuda()
        y_ws = torch.zeros((t, topk, n), dtype=torch.int16, device="cuda")
        ws = torch.empty((qmm.qmm_workspace_bytes(qmm.OP_GROUPED, w, 0, t, topk),), dtype=torch.uint8, device="cuda")
        qmm.qmm_grouped_gemv(w, x, ids, y_ws, x_per_pair=per_pair, ws=ws)
        y_na = torch.full((t, topk, n), 0x5A5A, dtype=torch.int16, device="cuda")
        qmm.qmm_grouped_gemv_noalloc(w, x, ids, y_na, x_per_pair=per_pair)
        assert qmm.qmm_sync_check() == 0
        assert qmm.qmm_last_variant().startswith("noalloc:")
        yref, absy = _oracle_y(p, fmt, n, k, x_bits, ids_np, per_pair)
        got = f16(from_dev_u16(y_na))
        assert (np.abs(got - yref) <= REL * absy + ABS).all()            # against the oracle
        assert (np.abs(got - f16(from_dev_u16(y_ws))) <= REL * absy + ABS).all()  # and the workspace call


def test_noalloc_call_takes_no_device_memory():
    """After a first call (which may load the kernels' code), further calls
    leave the device's free memory unchanged."""
    p, x_bits, ids_np = _case(73, synth.FMT_IQ4_NL, 8, 96, 256, 40, 4, False)
    w = dev(p)
    x = to_dev_u16(x_bits)
    ids = torch.from_numpy(ids_np).cuda()
    y = torch.zeros((40, 4, 96), dtype=torch.int16, device="cuda")
    qmm.qmm_grouped_gemv_noalloc(w, x, ids, y)
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    for _ in range(3):
        qmm.qmm_grouped_gemv_noalloc(w, x, ids, y)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert qmm.qmm_sync_check() == 0
    assert free1 == free0


def test_noalloc_refuses_more_pairs_than_its_array_holds():
    rng = np.random.default_rng(3)
    p = synth.gen_iq4nl(rng, 16, 64, experts=4)
    w = dev(p)
    t, topk = 16385, 4                         # 65540 pairs > 65536
    ids = torch.zeros((t, topk), dtype=torch.int32, device="cuda")
    x = torch.zeros((t, 64), dtype=torch.int16, device="cuda")
    y = torch.zeros((t, topk, 16), dtype=torch.int16, device="cuda")
    with pytest.raises(qmm.QmmError) as e:
        qmm.qmm_grouped_gemv_noalloc(w, x, ids, y)
    assert e.value.status == 2                 # QMM_ERR_UNSUPPORTED_SHAPE, nothing launched
    assert qmm.qmm_sync_check() == 0
