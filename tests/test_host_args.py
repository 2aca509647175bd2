"""Host-side argument checks, run without a GPU.

The C entry points (qmm_gemv_host, qmm_gemm, qmm_grouped_gemv, qmm_route,
qmm_moe_routed, qmm_router_topk, qmm_quantize, qmm_workspace_bytes) check
descriptors, sizes, null pointers and alignment before they touch CUDA; the
cases here all return there, with fake device addresses that are never
dereferenced.  The Python binding's own checks (host vs device tensors,
contiguity, and that every tensor holds the bytes its call touches) run on
CPU tensors, which reach them before the device check."""
import ctypes

import numpy as np
import pytest

from packed_bit_weight_b200 import qmm

OK, INVALID, UNSUPPORTED, MISALIGNED = 0, 1, 2, 3
FAKE = 1 << 40  # a 16-byte-aligned address that is never dereferenced


def _desc(fmt=2, n=64, k=256, data=FAKE, scales=FAKE + (1 << 20)):
    d = qmm.qmm_weights()
    d.fmt, d.reserved, d.n, d.k = fmt, 0, n, k
    d.data = ctypes.c_void_p(data) if data else None
    d.scales = ctypes.c_void_p(scales) if scales else None
    d.global_scale, d.reserved2, d.num_experts = 1.0, 0, 1
    d.expert_data_stride, d.expert_scale_stride = 0, 0
    return d


def _call(d, m=1, xh=True, yh=True, xd=FAKE + (2 << 20), yd=FAKE + (3 << 20)):
    L = qmm._lib()
    xbuf = np.zeros(max(m, 1) * 256 + 16, dtype=np.uint16)
    ybuf = np.zeros(max(m, 1) * 64 + 16, dtype=np.uint16)
    xp = ctypes.c_void_p(xbuf.ctypes.data) if xh else None
    yp = ctypes.c_void_p(ybuf.ctypes.data) if yh else None
    return L.qmm_gemv_host(ctypes.byref(d) if d is not None else None, xp, m, yp,
                           ctypes.c_void_p(xd) if xd else None, ctypes.c_void_p(yd) if yd else None, None)


def test_descriptor_errors():
    assert _call(None) == INVALID
    assert _call(_desc(fmt=9)) == INVALID                  # unknown format
    assert _call(_desc(k=250)) == UNSUPPORTED              # k not a multiple of the group
    assert _call(_desc(data=None)) == INVALID              # packed codes missing
    assert _call(_desc(scales=None)) == INVALID            # FP4-G16 needs its scales
    assert _call(_desc(data=FAKE + 8)) == MISALIGNED       # codes not 16-byte aligned


def test_batch_and_buffer_errors():
    d = _desc()
    assert _call(d, m=-1) == INVALID
    assert _call(d, m=17) == UNSUPPORTED                   # decode batches are 1..16
    assert _call(d, m=0) == OK                             # nothing to do
    assert _call(_desc(n=0)) == OK
    assert _call(d, yh=False) == INVALID                   # no host output
    assert _call(d, xh=False) == INVALID                   # no host input (k > 0)
    assert _call(d, yd=None) == INVALID                    # no device staging for y
    assert _call(d, yd=FAKE + 4) == MISALIGNED
    assert _call(d, xd=FAKE + 8) == MISALIGNED


def test_binding_rejects_device_tensors_as_host_buffers():
    torch = pytest.importorskip("torch")
    w = qmm.PackedWeights(2, 64, 256, torch.zeros(64 * 128, dtype=torch.uint8),
                          torch.zeros(64 * 16, dtype=torch.float16))
    xh = torch.zeros((1, 256), dtype=torch.int16)
    yh = torch.zeros((1, 64), dtype=torch.int16)
    with pytest.raises(ValueError):                        # staging buffers must be CUDA tensors
        qmm.qmm_gemv_host(w, xh, yh, xh, yh)
    with pytest.raises(ValueError):                        # host buffers must be contiguous
        qmm.qmm_gemv_host(w, xh.view(-1)[:128].view(1, 128).t(), yh, xh, yh)


def _stack(fmt=1, n=64, k=256, experts=4, data_stride=None, scale_stride=None):
    d = _desc(fmt=fmt, n=n, k=k, scales=None if fmt == 1 else FAKE + (1 << 20))
    d.num_experts = experts
    db, sb = qmm.qmm_data_bytes(fmt, n, k), qmm.qmm_scale_bytes(fmt, n, k)
    d.expert_data_stride = db if data_stride is None else data_stride
    d.expert_scale_stride = sb if scale_stride is None else scale_stride
    return d


def _vp(a):
    return ctypes.c_void_p(a) if a else None


def test_gemm_argument_errors():
    L = qmm._lib()
    assert L.qmm_gemm(None, _vp(FAKE), 4, _vp(FAKE), None, 0, None) == INVALID
    assert L.qmm_gemm(ctypes.byref(_desc()), _vp(FAKE), -1, _vp(FAKE), None, 0, None) == INVALID
    assert L.qmm_gemm(ctypes.byref(_desc(k=250)), _vp(FAKE), 4, _vp(FAKE), None, 0, None) == UNSUPPORTED


def test_grouped_argument_errors():
    L = qmm._lib()
    ids = _vp(FAKE + (4 << 20))

    def call(d, t=8, topk=2, per_pair=0, ids=ids):
        return L.qmm_grouped_gemv(ctypes.byref(d), _vp(FAKE), per_pair, ids, t, topk, _vp(FAKE), None, 0, None)

    assert call(_stack(data_stride=100)) == INVALID                        # stride below one matrix
    assert call(_stack(data_stride=qmm.qmm_data_bytes(1, 64, 256) + 8)) == MISALIGNED
    assert call(_stack(), t=-1) == INVALID
    assert call(_stack(experts=257)) == UNSUPPORTED                         # at most 256 experts
    assert call(_stack(), ids=None) == INVALID                              # pairs but no ids
    assert call(_stack(), ids=_vp(FAKE + 4)) == MISALIGNED
    assert call(_stack(), per_pair=2) == INVALID
    assert call(_stack(fmt=2, scale_stride=4)) == INVALID                  # FP4 scale stride below one matrix
    # t * topk would overflow int64: refused on the bounds, before any product
    assert call(_stack(), t=1 << 62, topk=1 << 40) == UNSUPPORTED
    assert call(_stack(), t=(1 << 30), topk=2) == UNSUPPORTED               # more pairs than INT32_MAX / 2
    assert L.qmm_grouped_gemv_noalloc(ctypes.byref(_stack()), _vp(FAKE), 0, ids, 1 << 62, 1 << 40, _vp(FAKE),
                                      None) == UNSUPPORTED


def test_route_argument_errors():
    L = qmm._lib()
    ids = _vp(FAKE)
    assert L.qmm_route(ids, 8, 2, 4, None, _vp(FAKE + 256), None, 0, None) == INVALID   # no offsets
    assert L.qmm_route(ids, 8, 2, 4, _vp(FAKE + 256), None, None, 0, None) == INVALID   # no permutation
    assert L.qmm_route(ids, 8, 2, 4, _vp(FAKE + 8), _vp(FAKE + 256), None, 0, None) == MISALIGNED
    assert L.qmm_route(ids, 8, 2, 0, _vp(FAKE + 256), _vp(FAKE + 512), None, 0, None) == INVALID  # no experts


def test_moe_argument_errors():
    L = qmm._lib()
    E, f, d = 4, 128, 256
    gate, up, down = _stack(n=f, k=d, experts=E), _stack(n=f, k=d, experts=E), _stack(n=d, k=f, experts=E)

    def call(g=gate, u=up, dn=down, t=8, topk=2):
        return L.qmm_moe_routed(ctypes.byref(g), ctypes.byref(u), ctypes.byref(dn), _vp(FAKE), _vp(FAKE + 4096),
                                _vp(FAKE + 8192), t, topk, _vp(FAKE), None, 0, None)

    assert call(g=_stack(fmt=2, n=f, k=d, experts=E)) == UNSUPPORTED       # the expert kernels are IQ4_NL
    assert call(u=_stack(n=f + 16, k=d, experts=E)) == INVALID             # gate and up differ
    assert call(dn=_stack(n=d, k=f, experts=E + 1)) == INVALID             # expert counts differ
    assert call(t=-1) == INVALID
    g2, u2 = _stack(n=f, k=160, experts=E), _stack(n=f, k=160, experts=E)
    assert call(g=g2, u=u2, dn=_stack(n=160, k=f, experts=E)) == UNSUPPORTED  # d % 128 != 0


def test_router_and_quantize_argument_errors():
    L = qmm._lib()
    p = _vp(FAKE)
    # x, w_router, bias, t, k, E, topk, ids, weights, logits, stream
    assert L.qmm_router_topk(p, p, p, 4, 256, 8, 9, p, p, None, None) == INVALID        # topk > E
    assert L.qmm_router_topk(p, p, p, 4, 250, 8, 2, p, p, None, None) == UNSUPPORTED    # k % 8
    assert L.qmm_router_topk(p, p, p, 4, 256, 300, 2, p, p, None, None) == UNSUPPORTED  # too many experts
    assert L.qmm_router_topk(p, p, p, -1, 256, 8, 2, p, p, None, None) == INVALID
    # fmt, w, n, k, data, scales, stream
    assert L.qmm_quantize(9, p, 4, 256, p, p, None) == INVALID
    assert L.qmm_quantize(3, p, 4, 256, p, p, None) == UNSUPPORTED      # E4M3 needs a matrix-wide scale
    assert L.qmm_quantize(2, p, 4, 250, p, p, None) == UNSUPPORTED
    assert L.qmm_quantize(2, p, -1, 256, p, p, None) == INVALID


def test_workspace_size_rejects_bad_descriptors():
    L = qmm._lib()
    assert L.qmm_workspace_bytes(qmm.OP_GROUPED, None, 0, 8, 2) == 0
    assert L.qmm_workspace_bytes(qmm.OP_GROUPED, ctypes.byref(_stack()), 0, -1, 2) == 0
    assert L.qmm_workspace_bytes(qmm.OP_GROUPED, ctypes.byref(_stack()), 0, 8, 2) > 0
    assert L.qmm_workspace_bytes(qmm.OP_GROUPED, ctypes.byref(_stack()), 0, 1 << 62, 1 << 40) == 0  # no overflow


def _pw(fmt=2, n=64, k=256, experts=1, short=0, scales_short=0):
    torch = pytest.importorskip("torch")
    db, sb = qmm.qmm_data_bytes(fmt, n, k) * experts, qmm.qmm_scale_bytes(fmt, n, k) * experts
    sc = torch.zeros(sb - scales_short, dtype=torch.uint8) if sb else None
    return qmm.PackedWeights(fmt, n, k, torch.zeros(db - short, dtype=torch.uint8), sc, 1.0, experts)


def _short(fn, *a, **kw):
    with pytest.raises(ValueError, match="holds"):
        fn(*a, **kw)


def test_binding_refuses_undersized_weight_tensors():
    _short(lambda: _pw(short=16).desc())
    _short(lambda: _pw(scales_short=2).desc())
    _short(lambda: _pw(fmt=1, experts=3, short=18).desc())          # last expert's last block missing
    _pw(fmt=1, experts=3).desc()                                     # exact sizes pass
    _pw(fmt=2, k=250).desc()                                         # bad shape: left to the C checks


def test_binding_refuses_undersized_buffers():
    torch = pytest.importorskip("torch")
    i16, i32, f32 = torch.int16, torch.int32, torch.float32
    w = _pw()
    z = lambda *s, dt=i16: torch.zeros(*s, dtype=dt)
    _short(qmm.qmm_gemv, w, z(2, 256), z(2 * 64 - 1))                # y one element short
    _short(qmm.qmm_gemv, w, z(2, 255), z(2, 64))                     # x rows shorter than k
    _short(qmm.qmm_gemm, w, z(300, 256), z(299, 64))
    _short(qmm.qmm_dequant, w, z(64 * 256 - 8))
    _short(qmm.qmm_gemv_host, w, z(2, 256), z(2, 64), z(2, 256), z(2, 63))
    _short(qmm.qmm_quantize, 2, z(64, 256), torch.zeros(64 * 128 - 1, dtype=torch.uint8),
           torch.zeros(64 * 16 * 2, dtype=torch.uint8))
    _short(qmm.qmm_quantize, 2, z(64, 256), torch.zeros(64 * 128, dtype=torch.uint8),
           torch.zeros(64 * 16 * 2 - 1, dtype=torch.uint8))
    ids = z(8, 2, dt=i32)
    _short(qmm.qmm_route, ids, 4, z(4, dt=i32), z(16, dt=i32))       # offsets need E + 1
    _short(qmm.qmm_route, ids, 4, z(5, dt=i32), z(15, dt=i32))       # perm needs t * topk
    e = _pw(fmt=1, experts=4)
    _short(qmm.qmm_grouped_gemv, e, z(8, 256), ids, z(8, 2, 63))
    _short(qmm.qmm_grouped_gemv, e, z(8, 256), ids, z(8, 2, 64), x_per_pair=True)   # one x row per pair
    _short(qmm.qmm_grouped_gemv_noalloc, e, z(7, 256), ids, z(8, 2, 64))
    _short(qmm.qmm_router_topk, z(8, 256), z(4, 255), z(4, dt=f32), 2, ids, z(8, 2, dt=f32))
    _short(qmm.qmm_router_topk, z(8, 256), z(4, 256), z(4, dt=f32), 2, ids, z(8, 2, dt=f32), z(8, 3, dt=f32))
    g, u, d = _pw(fmt=1, n=128, k=256, experts=4), _pw(fmt=1, n=128, k=256, experts=4), _pw(fmt=1, n=256, k=128,
                                                                                            experts=4)
    _short(qmm.qmm_moe_routed, g, u, d, z(8, 256), ids, z(8, 1, dt=f32), z(8, 256))
    _short(qmm.qmm_moe_routed, g, u, d, z(8, 256), ids, z(8, 2, dt=f32), z(8, 255))


def test_binding_size_checks_pass_exact_buffers_on_to_the_device_check():
    """Exactly sized buffers pass the size checks and are refused only
    because they are host tensors (the device check that follows)."""
    torch = pytest.importorskip("torch")
    w = _pw()
    with pytest.raises(ValueError, match="CUDA"):
        qmm.qmm_gemv(w, torch.zeros(2, 256, dtype=torch.int16), torch.zeros(2, 64, dtype=torch.int16))
    with pytest.raises(ValueError, match="CUDA"):
        qmm.qmm_gemv(w, torch.zeros(0, 256, dtype=torch.int16), torch.zeros(0, 64, dtype=torch.int16))
