"""ctypes binding of libqmm.so (include/qmm.h).

Argument marshalling only: every function here takes torch tensors, checks
that they are CUDA tensors of the right element size and that each holds at
least the bytes the call will read or write (the C ABI takes bare pointers
and cannot see a buffer's extent), passes raw device pointers and the current
CUDA stream to the C ABI, and raises ``QmmError`` on a non-OK status.  No arithmetic of the path happens in Python, and there is
no fallback: if the library is missing the first call raises.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import numpy as np
import torch

from . import _build

FMT_IQ4_NL = 1
FMT_FP4G16_F16 = 2
FMT_FP4G16_E4M3 = 3
FMT_MXFP4 = 4

OP_DEQUANT, OP_GEMV, OP_GEMM, OP_ROUTE, OP_GROUPED, OP_MOE = 0, 1, 2, 3, 4, 5

STATUS = {0: "QMM_OK", 1: "QMM_ERR_INVALID_ARG", 2: "QMM_ERR_UNSUPPORTED_SHAPE", 3: "QMM_ERR_MISALIGNED",
          4: "QMM_ERR_NOT_SM100", 5: "QMM_ERR_CUDA", 6: "QMM_ERR_TIMEOUT", 7: "QMM_ERR_DEVICE_FAULT",
          8: "QMM_ERR_WORKSPACE"}


class QmmError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__("%s: %s (%s)" % (where, STATUS.get(status, status), _lib().qmm_status_string(status).decode()))


class qmm_weights(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("reserved", ctypes.c_int32), ("n", ctypes.c_int64), ("k", ctypes.c_int64),
                ("data", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_float),
                ("reserved2", ctypes.c_int32), ("num_experts", ctypes.c_int64),
                ("expert_data_stride", ctypes.c_int64), ("expert_scale_stride", ctypes.c_int64)]


_L = None
LIB_PATH = _build.LIB


def _lib():
    global _L
    if _L is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError("libqmm.so is not built (expected at %s); run __graft_entry__.build()" % LIB_PATH)
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        W = ctypes.POINTER(qmm_weights)
        sigs = {
            "qmm_data_bytes": (sz, [i32, i64, i64]),
            "qmm_scale_bytes": (sz, [i32, i64, i64]),
            "qmm_packed_bytes": (sz, [i32, i64, i64]),
            "qmm_dequant": (i32, [W, vp, vp]),
            "qmm_quantize": (i32, [i32, vp, i64, i64, vp, vp, vp]),
            "qmm_gemv": (i32, [W, vp, i64, vp, vp, sz, vp]),
            "qmm_gemv_host": (i32, [W, vp, i64, vp, vp, vp, vp]),
            "qmm_gemm": (i32, [W, vp, i64, vp, vp, sz, vp]),
            "qmm_route": (i32, [vp, i64, i64, i64, vp, vp, vp, sz, vp]),
            "qmm_grouped_gemv": (i32, [W, vp, i32, vp, i64, i64, vp, vp, sz, vp]),
            "qmm_grouped_gemv_noalloc": (i32, [W, vp, i32, vp, i64, i64, vp, vp]),
            "qmm_router_topk": (i32, [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, vp]),
            "qmm_moe_routed": (i32, [W, W, W, vp, vp, vp, i64, i64, vp, vp, sz, vp]),
            "qmm_workspace_bytes": (sz, [i32, W, i64, i64, i64]),
            "qmm_sync_check": (i32, [vp]),
            "qmm_debug_set": (i32, [i32, i64]),
            "qmm_status_string": (ctypes.c_char_p, [i32]),
            "qmm_last_variant": (ctypes.c_char_p, []),
            "qmm_version": (ctypes.c_char_p, []),
        }
        for name, (res, args) in sigs.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _L = L
    return _L


def lib():
    return _lib()


def _check(status: int, where: str):
    if status != 0:
        raise QmmError(status, where)


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor | None, nbytes: int, name: str) -> None:
    """Refuse a tensor smaller than the bytes the C call touches through its
    pointer: an undersized buffer would otherwise be an out-of-bounds access
    on the device instead of an error here.  None is left to the C checks."""
    if t is not None and t.nbytes < nbytes:
        raise ValueError("%s holds %d bytes; the call reads or writes %d" % (name, t.nbytes, nbytes))


def _ptr(t: torch.Tensor | None, esize: int | None = None, name: str = "tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if esize is not None and t.element_size() != esize:
        raise ValueError("%s must have %d-byte elements" % (name, esize))
    return ctypes.c_void_p(t.data_ptr())


@dataclass
class PackedWeights:
    """Device tensors of one packed matrix (or expert stack) plus its C descriptor."""
    fmt: int
    n: int
    k: int
    data: torch.Tensor
    scales: torch.Tensor | None
    global_scale: float = 1.0
    experts: int = 1
    data_stride: int | None = None    # bytes between experts (default: data split evenly)
    scale_stride: int | None = None

    def desc(self) -> qmm_weights:
        """The C descriptor, rebuilt only when a field or a buffer changed."""
        key = (self.fmt, self.n, self.k, None if self.data is None else (self.data.data_ptr(), self.data.numel()),
               None if self.scales is None else (self.scales.data_ptr(), self.scales.numel()), self.global_scale,
               self.experts, self.data_stride, self.scale_stride)
        cached = self.__dict__.get("_desc")
        if cached is not None and cached[0] == key:
            return cached[1]
        d = self._build_desc()
        self.__dict__["_desc"] = (key, d)
        return d

    def _build_desc(self) -> qmm_weights:
        d = qmm_weights()
        d.fmt, d.reserved, d.n, d.k = self.fmt, 0, self.n, self.k
        d.data = ctypes.c_void_p(self.data.data_ptr()) if self.data is not None else None
        d.scales = ctypes.c_void_p(self.scales.data_ptr()) if self.scales is not None else None
        d.global_scale, d.reserved2, d.num_experts = float(self.global_scale), 0, self.experts
        if self.data_stride is not None:
            d.expert_data_stride = self.data_stride
        else:
            d.expert_data_stride = self.data.numel() // self.experts if self.data is not None else 0
        if self.scale_stride is not None:
            d.expert_scale_stride = self.scale_stride
        else:
            d.expert_scale_stride = (self.scales.numel() * self.scales.element_size() // self.experts
                                     if self.scales is not None else 0)
        # every expert's codes and scales must lie inside the tensors (the
        # sizes are 0 for a shape the C checks reject anyway)
        last = max(int(self.experts), 1) - 1
        db, sb = qmm_data_bytes(self.fmt, self.n, self.k), qmm_scale_bytes(self.fmt, self.n, self.k)
        _need(self.data, last * d.expert_data_stride + db if db else 0, "data")
        _need(self.scales, last * d.expert_scale_stride + sb if sb else 0, "scales")
        return d

    def rows(self, r0: int, r1: int) -> "PackedWeights":
        """View of rows [r0, r1) of every matrix of the stack (no copy): e.g.
        the gate and up halves of an expert stack stored as [E][2f][k]."""
        db, sb = qmm_data_bytes(self.fmt, 1, self.k), qmm_scale_bytes(self.fmt, 1, self.k)
        d = self.desc()
        data = self.data.view(torch.uint8).reshape(-1)[r0 * db:]
        scales = None if self.scales is None else self.scales.view(torch.uint8).reshape(-1)[r0 * sb:]
        return PackedWeights(self.fmt, r1 - r0, self.k, data, scales, self.global_scale, self.experts,
                             d.expert_data_stride, d.expert_scale_stride)

    @property
    def nbytes(self) -> int:
        return self.data.numel() + (0 if self.scales is None else self.scales.numel() * self.scales.element_size())

    @staticmethod
    def from_host(p, device="cuda") -> "PackedWeights":
        """From a ``synth.Packed`` (numpy bytes) to device tensors.  An expert
        stack whose per-expert byte counts are not multiples of 16 (e.g.
        MXFP4 scales of an odd row count) is copied with each expert padded
        to 16 bytes, as the expert strides of the C ABI require."""
        ds, ss = p.data_stride, p.scale_stride
        if p.experts > 1 and (ds % 16 or ss % 16):
            pd, ps = -(-ds // 16) * 16, -(-ss // 16) * 16
            d = np.zeros((p.experts, pd), dtype=np.uint8)
            d[:, :ds] = p.data.reshape(p.experts, ds)
            sc = None
            if p.scales is not None:
                sc = np.zeros((p.experts, ps), dtype=np.uint8)
                sc[:, :ss] = p.scales.reshape(p.experts, ss)
                sc = torch.from_numpy(sc.reshape(-1)).to(device)
            return PackedWeights(p.fmt, p.n, p.k, torch.from_numpy(d.reshape(-1)).to(device), sc, p.global_scale,
                                 p.experts, pd, ps if p.scales is not None else None)
        data = torch.from_numpy(p.data).to(device)
        scales = None if p.scales is None else torch.from_numpy(p.scales).to(device)
        return PackedWeights(p.fmt, p.n, p.k, data, scales, p.global_scale, p.experts)


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------
def qmm_data_bytes(fmt: int, n: int, k: int) -> int:
    return _lib().qmm_data_bytes(fmt, n, k)


def qmm_scale_bytes(fmt: int, n: int, k: int) -> int:
    return _lib().qmm_scale_bytes(fmt, n, k)


def qmm_packed_bytes(fmt: int, n: int, k: int) -> int:
    return _lib().qmm_packed_bytes(fmt, n, k)


def qmm_workspace_bytes(op: int, w: PackedWeights | None, m: int = 0, t: int = 0, topk: int = 0) -> int:
    d = w.desc() if w is not None else None
    return _lib().qmm_workspace_bytes(op, ctypes.byref(d) if d is not None else None, m, t, topk)


def qmm_dequant(w: PackedWeights, out: torch.Tensor, stream=None) -> torch.Tensor:
    d = w.desc()
    _need(out, 2 * w.n * w.k, "out")
    _check(_lib().qmm_dequant(ctypes.byref(d), _ptr(out, 2, "out"), _stream(stream)), "qmm_dequant")
    return out


def qmm_quantize(fmt: int, w: torch.Tensor, data: torch.Tensor, scales: torch.Tensor | None = None,
                 stream=None) -> None:
    """fp16 weights w [n][k] (2-byte elements) -> packed data / scales."""
    n, k = w.shape
    _need(data, qmm_data_bytes(fmt, n, k), "data")
    _need(scales, qmm_scale_bytes(fmt, n, k), "scales")
    _check(_lib().qmm_quantize(fmt, _ptr(w, 2, "w"), n, k, _ptr(data, None, "data"), _ptr(scales, None, "scales"),
                               _stream(stream)), "qmm_quantize")


def _ws(ws):
    return (_ptr(ws, None, "ws"), 0 if ws is None else ws.numel() * ws.element_size())


def qmm_gemv(w: PackedWeights, x: torch.Tensor, y: torch.Tensor, ws: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    d = w.desc()
    wp, wb = _ws(ws)
    m = x.shape[0] if x.dim() == 2 else 1
    _need(x, 2 * m * w.k, "x")
    _need(y, 2 * m * w.n, "y")
    _check(_lib().qmm_gemv(ctypes.byref(d), _ptr(x, 2, "x"), m, _ptr(y, 2, "y"), wp, wb, _stream(stream)), "qmm_gemv")
    return y


def _host_ptr(t: torch.Tensor, esize: int, name: str):
    if t.is_cuda:
        raise ValueError("%s must be a host tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if t.element_size() != esize:
        raise ValueError("%s must have %d-byte elements" % (name, esize))
    return ctypes.c_void_p(t.data_ptr())


def qmm_gemv_host(w: PackedWeights, x_host: torch.Tensor, y_host: torch.Tensor, x_dev: torch.Tensor,
                  y_dev: torch.Tensor, stream=None) -> torch.Tensor:
    """qmm_gemv on host tensors in one library call: x_host -> x_dev, the
    product into y_dev, y_dev -> y_host, enqueued on the stream (asynchronous
    when the host tensors are pinned)."""
    d = w.desc()
    m = x_host.shape[0] if x_host.dim() == 2 else 1
    xb, yb = 2 * m * w.k, 2 * m * w.n
    _need(x_host, xb, "x_host")
    _need(x_dev, xb, "x_dev")
    _need(y_host, yb, "y_host")
    _need(y_dev, yb, "y_dev")
    _check(_lib().qmm_gemv_host(ctypes.byref(d), _host_ptr(x_host, 2, "x_host"), m, _host_ptr(y_host, 2, "y_host"),
                                _ptr(x_dev, 2, "x_dev"), _ptr(y_dev, 2, "y_dev"), _stream(stream)), "qmm_gemv_host")
    return y_host


def qmm_gemm(w: PackedWeights, x: torch.Tensor, y: torch.Tensor, ws: torch.Tensor | None = None,
             stream=None) -> torch.Tensor:
    d = w.desc()
    wp, wb = _ws(ws)
    _need(x, 2 * x.shape[0] * w.k, "x")
    _need(y, 2 * x.shape[0] * w.n, "y")
    _check(_lib().qmm_gemm(ctypes.byref(d), _ptr(x, 2, "x"), x.shape[0], _ptr(y, 2, "y"), wp, wb, _stream(stream)),
           "qmm_gemm")
    return y


def qmm_route(topk_ids: torch.Tensor, num_experts: int, offsets: torch.Tensor, perm: torch.Tensor,
              ws: torch.Tensor | None = None, stream=None):
    t, topk = topk_ids.shape
    wp, wb = _ws(ws)
    _need(offsets, 4 * (num_experts + 1), "offsets")
    _need(perm, 4 * t * topk, "perm")
    _check(_lib().qmm_route(_ptr(topk_ids, 4, "topk_ids"), t, topk, num_experts, _ptr(offsets, 4, "offsets"),
                            _ptr(perm, 4, "perm"), wp, wb, _stream(stream)), "qmm_route")
    return offsets, perm


def _need_grouped(w: PackedWeights, x, topk_ids, y, x_per_pair):
    t, topk = topk_ids.shape
    _need(x, 2 * w.k * (t * topk if x_per_pair else t), "x")
    _need(y, 2 * t * topk * w.n, "y")
    return t, topk


def qmm_grouped_gemv(w: PackedWeights, x: torch.Tensor, topk_ids: torch.Tensor, y: torch.Tensor,
                     x_per_pair: bool = False, ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    d = w.desc()
    t, topk = _need_grouped(w, x, topk_ids, y, x_per_pair)
    wp, wb = _ws(ws)
    _check(_lib().qmm_grouped_gemv(ctypes.byref(d), _ptr(x, 2, "x"), int(bool(x_per_pair)),
                                   _ptr(topk_ids, 4, "topk_ids"), t, topk, _ptr(y, 2, "y"), wp, wb,
                                   _stream(stream)), "qmm_grouped_gemv")
    return y


def qmm_grouped_gemv_noalloc(w: PackedWeights, x: torch.Tensor, topk_ids: torch.Tensor, y: torch.Tensor,
                             x_per_pair: bool = False, stream=None) -> torch.Tensor:
    """qmm_grouped_gemv without a workspace: the routing scratch is the
    library's own fixed device array (at most 65536 pairs, 256 experts; calls
    that overlap on the GPU race on it)."""
    d = w.desc()
    t, topk = _need_grouped(w, x, topk_ids, y, x_per_pair)
    _check(_lib().qmm_grouped_gemv_noalloc(ctypes.byref(d), _ptr(x, 2, "x"), int(bool(x_per_pair)),
                                           _ptr(topk_ids, 4, "topk_ids"), t, topk, _ptr(y, 2, "y"),
                                           _stream(stream)), "qmm_grouped_gemv_noalloc")
    return y


def qmm_router_topk(x: torch.Tensor, w_router: torch.Tensor, bias: torch.Tensor, topk: int,
                    topk_ids: torch.Tensor, topk_weights: torch.Tensor, logits: torch.Tensor | None = None,
                    stream=None):
    """Router logits (fp64 sums rounded once to fp32), fp32 softmax and the
    top-k experts with their softmax weights."""
    t, k = x.shape
    E = w_router.shape[0]
    for tt, nb, name in ((w_router, 2 * E * k, "w_router"), (bias, 4 * E, "bias"),
                         (topk_ids, 4 * t * topk, "topk_ids"), (topk_weights, 4 * t * topk, "topk_weights"),
                         (logits, 4 * t * E, "logits")):
        _need(tt, nb, name)
    _check(_lib().qmm_router_topk(_ptr(x, 2, "x"), _ptr(w_router, 2, "w_router"), _ptr(bias, 4, "bias"), t, k, E,
                                  topk, _ptr(topk_ids, 4, "topk_ids"), _ptr(topk_weights, 4, "topk_weights"),
                                  _ptr(logits, 4, "logits"), _stream(stream)), "qmm_router_topk")
    return topk_ids, topk_weights


def qmm_moe_routed(gate: PackedWeights, up: PackedWeights, down: PackedWeights, x: torch.Tensor,
                   topk_ids: torch.Tensor, topk_weights: torch.Tensor, out: torch.Tensor,
                   ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """out[t] = sum_s g[t][s] * W_down,e (SiLU(W_gate,e x_t) * W_up,e x_t)."""
    dg, du, dd = gate.desc(), up.desc(), down.desc()
    t, topk = topk_ids.shape
    wp, wb = _ws(ws)
    _need(x, 2 * t * gate.k, "x")
    _need(topk_weights, 4 * t * topk, "topk_weights")
    _need(out, 2 * t * down.n, "out")
    _check(_lib().qmm_moe_routed(ctypes.byref(dg), ctypes.byref(du), ctypes.byref(dd), _ptr(x, 2, "x"),
                                 _ptr(topk_ids, 4, "topk_ids"), _ptr(topk_weights, 4, "topk_weights"), t, topk,
                                 _ptr(out, 2, "out"), wp, wb, _stream(stream)), "qmm_moe_routed")
    return out


DEBUG_WAIT_LIMIT_NS = 1
DEBUG_WITHHOLD_X_TILES = 2
DEBUG_WITHHOLD_TILE_COPIES = 3


def qmm_debug_set(what: int, value: int) -> None:
    """Test hooks of the bounded pipeline waits (include/qmm.h)."""
    _check(_lib().qmm_debug_set(int(what), int(value)), "qmm_debug_set")


def qmm_sync_check(stream=None) -> int:
    return _lib().qmm_sync_check(_stream(stream))


def qmm_last_variant() -> str:
    return _lib().qmm_last_variant().decode()


def qmm_version() -> str:
    return _lib().qmm_version().decode()
