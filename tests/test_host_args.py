"""Host-side argument checks of qmm_gemv_host, run without a GPU: every case
here returns before the library touches CUDA (descriptor, batch size, null
and alignment checks come first), with fake device addresses that are never
dereferenced."""
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
