"""ctypes wrapper around ``qmm_oracle.c`` (the plain CPU definition).

TEST INFRASTRUCTURE ONLY -- see the package docstring.  Arrays are numpy;
fp16 values travel as uint16 bit patterns so that no library conversion sits
between the oracle's own codec and the caller.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

FMT_IQ4_NL = 1
FMT_FP4G16_F16 = 2
FMT_FP4G16_E4M3 = 3
FMT_MXFP4 = 4

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "qmm_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

# What pins each oracle function to something other than itself (tests named).
PINS = {
    "f16_to_f64": "all 65536 patterns vs numpy float16 (tests/test_oracle_codecs.py)",
    "f64_to_f16": "every fp16 value, every halfway point and its neighbours, random doubles vs "
                  "numpy float16 (tests/test_oracle_codecs.py)",
    "e4m3_to_f64": "all 256 bytes vs torch float8_e4m3fn and the printed OCP extremes "
                   "(tests/test_oracle_codecs.py)",
    "e2m1_to_f64": "printed magnitude list (tests/golden/e2m1_magnitudes.txt)",
    "iq4nl_value": "printed codebook (tests/golden/iq4nl_codebook.txt)",
    "e8m0_to_f64": "all 256 bytes vs torch float8_e8m0fnu (tests/test_oracle_codecs.py)",
    "data_bytes/scale_bytes": "byte identities from the model-card storage table "
                              "(tests/test_oracle_sizes.py)",
    "dequant": "hand-built blocks with hand-written expected values (tests/golden/*.txt), "
               "exhaustive scale x code sweeps vs exact rationals (tests/test_oracle_dequant.py)",
    "matmul": "exact-rational brute force, one-hot identity, integer special case "
              "(tests/test_oracle_matmul.py)",
    "matmul_sampled": "equals matmul on every sampled coordinate (tests/test_oracle_matmul.py)",
    "route": "brute-force bucket check (tests/test_oracle_matmul.py)",
    "grouped_gemv": "per-pair loop of the plain product (tests/test_oracle_matmul.py)",
    "router_topk": "softmax sums to 1, brute-force top-k, zero-weight and one-hot special cases "
                   "(tests/test_oracle_moe.py)",
    "silu/swiglu": "closed forms: silu(0)=0, silu(ln 3)=0.75 ln 3, odd/even split, limits (tests/test_oracle_moe.py)",
    "combine": "linearity and the one-slot special case (tests/test_oracle_moe.py)",
    "quantize": "exact recovery of codes from power-of-two scaled weights, hand-written rows "
                "(tests/golden/quantize_handmade.txt), error bound, optimality against numpy-rounded "
                "candidates (tests/test_oracle_quantize.py); the scale choice itself is parity unpinned",
}


def build(force: bool = False) -> str:
    """Compile ``liboracle.so`` with gcc (no fast-math, no fp contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


_lib = None


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i64, i32, f32, vp = ctypes.c_int64, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
        L.orc_f16_to_f64.argtypes = [ctypes.c_uint16]
        L.orc_f16_to_f64.restype = ctypes.c_double
        L.orc_f64_to_f16.argtypes = [ctypes.c_double]
        L.orc_f64_to_f16.restype = ctypes.c_uint16
        L.orc_e4m3_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_f64.restype = ctypes.c_double
        L.orc_e8m0_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e8m0_to_f64.restype = ctypes.c_double
        L.orc_e2m1_to_f64.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_to_f64.restype = ctypes.c_double
        L.orc_iq4nl_value.argtypes = [i32]
        L.orc_iq4nl_value.restype = i32
        L.orc_data_bytes.argtypes = [i32, i64, i64]
        L.orc_data_bytes.restype = i64
        L.orc_scale_bytes.argtypes = [i32, i64, i64]
        L.orc_scale_bytes.restype = i64
        L.orc_dequant_row.argtypes = [i32, i64, i64, vp, vp, f32, i64, vp]
        L.orc_dequant.argtypes = [i32, i64, i64, vp, vp, f32, vp]
        L.orc_matmul.argtypes = [i32, i64, i64, vp, vp, f32, vp, i64, vp, vp]
        L.orc_quantize.argtypes = [i32, i64, i64, vp, vp, vp]
        L.orc_matmul_sampled.argtypes = [i32, i64, i64, vp, vp, f32, vp, i64, vp, vp, i64, vp, vp]
        L.orc_route.argtypes = [vp, i64, i64, i64, vp, vp]
        L.orc_route.restype = i64
        L.orc_grouped_gemv.argtypes = [i32, i64, i64, vp, i64, vp, i64, f32, i64, vp, vp, i64, i64, vp, vp]
        L.orc_router_topk.argtypes = [vp, vp, vp, i64, i64, i64, i64, vp, vp, vp, vp]
        L.orc_silu.argtypes = [ctypes.c_double]
        L.orc_silu.restype = ctypes.c_double
        L.orc_swiglu.argtypes = [vp, i64, i64, vp]
        L.orc_combine.argtypes = [vp, vp, i64, i64, i64, vp]
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


# -- codecs ------------------------------------------------------------------
def f16_to_f64(bits: int) -> float:
    return lib().orc_f16_to_f64(int(bits))


def f64_to_f16(v: float) -> int:
    return lib().orc_f64_to_f16(float(v))


def e4m3_to_f64(b: int) -> float:
    return lib().orc_e4m3_to_f64(int(b))


def e8m0_to_f64(b: int) -> float:
    return lib().orc_e8m0_to_f64(int(b))


def e2m1_to_f64(nib: int) -> float:
    return lib().orc_e2m1_to_f64(int(nib))


def iq4nl_value(i: int) -> int:
    return lib().orc_iq4nl_value(int(i))


def data_bytes(fmt: int, n: int, k: int) -> int:
    return lib().orc_data_bytes(fmt, n, k)


def scale_bytes(fmt: int, n: int, k: int) -> int:
    return lib().orc_scale_bytes(fmt, n, k)


# -- dequantisation ------------------------------------------------------------
def dequant(fmt, n, k, data, scales=None, global_scale=1.0):
    """[n][k] fp16 bit patterns (uint16) of the decoded matrix."""
    data = _c(data, np.uint8)
    scales = _c(scales, np.uint8) if scales is not None else None
    out = np.empty((n, k), dtype=np.uint16)
    lib().orc_dequant(fmt, n, k, _p(data), _p(scales), float(global_scale), _p(out))
    return out


def dequant_row(fmt, n, k, data, scales, global_scale, row):
    data = _c(data, np.uint8)
    scales = _c(scales, np.uint8) if scales is not None else None
    out = np.empty((k,), dtype=np.uint16)
    lib().orc_dequant_row(fmt, n, k, _p(data), _p(scales), float(global_scale), int(row), _p(out))
    return out


# -- products --------------------------------------------------------------------
def quantize(fmt, n, k, w_bits):
    """fp16 weights [n][k] (bit patterns) -> (data, scales) packed bytes:
    FP4G16_F16 (fp16 scale amax/6), MXFP4 (E8M0 exponent floor(log2 amax) - 2)
    or IQ4_NL (d = m / -127); each weight the nearest decoded value, ties to
    the lowest code."""
    if fmt not in (FMT_FP4G16_F16, FMT_MXFP4, FMT_IQ4_NL):
        raise ValueError("no encoder for this format")
    w_bits = _c(w_bits, np.uint16).reshape(n, k)
    data = np.zeros(data_bytes(fmt, n, k), dtype=np.uint8)
    sb = scale_bytes(fmt, n, k)
    scales = np.zeros(max(sb, 1), dtype=np.uint8)
    lib().orc_quantize(fmt, n, k, _p(w_bits), _p(data), _p(scales))
    return data, (scales[:sb] if sb else None)


def matmul(fmt, n, k, data, scales, global_scale, x_bits):
    """(y, absy): y[m][n] = sum_k w16[n][k] x[m][k] in double, absy = sum |w x|."""
    data = _c(data, np.uint8)
    scales = _c(scales, np.uint8) if scales is not None else None
    x_bits = _c(x_bits, np.uint16).reshape(-1, k)
    m = x_bits.shape[0]
    y = np.empty((m, n), dtype=np.float64)
    a = np.empty((m, n), dtype=np.float64)
    lib().orc_matmul(fmt, n, k, _p(data), _p(scales), float(global_scale), _p(x_bits), m, _p(y), _p(a))
    return y, a


def matmul_sampled(fmt, n, k, data, scales, global_scale, x_bits, mi, ri):
    data = _c(data, np.uint8)
    scales = _c(scales, np.uint8) if scales is not None else None
    x_bits = _c(x_bits, np.uint16).reshape(-1, k)
    mi = _c(mi, np.int64)
    ri = _c(ri, np.int64)
    out = np.empty(mi.shape[0], dtype=np.float64)
    a = np.empty(mi.shape[0], dtype=np.float64)
    lib().orc_matmul_sampled(fmt, n, k, _p(data), _p(scales), float(global_scale), _p(x_bits),
                             x_bits.shape[0], _p(mi), _p(ri), mi.shape[0], _p(out), _p(a))
    return out, a


def route(ids, num_experts):
    """(offsets[E+1], perm[t*topk], n_bad): counting sort of pairs by expert."""
    ids = _c(ids, np.int32)
    t, topk = ids.shape
    off = np.empty(num_experts + 1, dtype=np.int32)
    perm = np.full(t * topk, -1, dtype=np.int32)
    bad = lib().orc_route(_p(ids), t, topk, num_experts, _p(off), _p(perm))
    return off, perm, bad


def grouped_gemv(fmt, n, k, data, data_stride, scales, scale_stride, global_scale, num_experts,
                 x_bits, ids):
    """(y, absy), both [t][topk][n]: y[t][s] = W_{ids[t][s]} x_t."""
    data = _c(data, np.uint8)
    scales = _c(scales, np.uint8) if scales is not None else None
    x_bits = _c(x_bits, np.uint16).reshape(-1, k)
    ids = _c(ids, np.int32)
    t, topk = ids.shape
    y = np.full((t, topk, n), np.nan, dtype=np.float64)
    a = np.full((t, topk, n), np.nan, dtype=np.float64)
    lib().orc_grouped_gemv(fmt, n, k, _p(data), int(data_stride), _p(scales), int(scale_stride),
                           float(global_scale), num_experts, _p(x_bits), _p(ids), t, topk, _p(y), _p(a))
    return y, a


# -- mixture-of-experts block ---------------------------------------------------
def router_topk(x_bits, w_bits, bias, topk):
    """(logits fp32 [t][E], ids [t][topk], g [t][topk] double, probs [t][E])."""
    x_bits = _c(x_bits, np.uint16)
    w_bits = _c(w_bits, np.uint16)
    bias = _c(bias, np.float32)
    t, k = x_bits.shape
    E = w_bits.shape[0]
    logits = np.empty((t, E), dtype=np.float32)
    ids = np.empty((t, topk), dtype=np.int32)
    g = np.empty((t, topk), dtype=np.float64)
    probs = np.empty((t, E), dtype=np.float64)
    lib().orc_router_topk(_p(x_bits), _p(w_bits), _p(bias), t, k, E, topk, _p(logits), _p(ids), _p(g), _p(probs))
    return logits, ids, g, probs


def silu(z: float) -> float:
    return lib().orc_silu(float(z))


def swiglu(gu):
    """gu [pairs][2f] double -> h [pairs][f] = SiLU(gate) * up."""
    gu = _c(gu, np.float64)
    pairs, f2 = gu.shape
    h = np.empty((pairs, f2 // 2), dtype=np.float64)
    lib().orc_swiglu(_p(gu), pairs, f2 // 2, _p(h))
    return h


def combine(y, g):
    """y [t][topk][n], g [t][topk] -> out [t][n] = sum_s g y."""
    y = _c(y, np.float64)
    g = _c(g, np.float64)
    t, topk, n = y.shape
    out = np.empty((t, n), dtype=np.float64)
    lib().orc_combine(_p(y), _p(g), t, topk, n, _p(out))
    return out
