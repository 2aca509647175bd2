"""Helpers shared by the GPU parity tests (test code: may use the oracle)."""
import numpy as np
import torch

import oracle
from packed_bit_weight_b200 import qmm, synth

# Output tolerance: |y - y_ref| <= REL * sum_k |w_k x_k| per element, plus the
# fp16 output's smallest spacing (2^-24) for sums that land in the fp16
# subnormal range.
REL = 1e-3
ABS = 2.0 ** -24


def dev(p: synth.Packed) -> qmm.PackedWeights:
    return qmm.PackedWeights.from_host(p, "cuda")


def to_dev_u16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).cuda()


def from_dev_u16(t: torch.Tensor) -> np.ndarray:
    return t.cpu().numpy().view(np.uint16)


def f16(bits: np.ndarray) -> np.ndarray:
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def nan_class_equal(got: np.ndarray, exp: np.ndarray) -> bool:
    """Bit-exact, except that NaN payloads compare by class."""
    ng = ((got & 0x7C00) == 0x7C00) & ((got & 0x3FF) != 0)
    ne = ((exp & 0x7C00) == 0x7C00) & ((exp & 0x3FF) != 0)
    return bool(np.array_equal(ng, ne) and np.array_equal(got[~ng], exp[~ne]))


def nz(bits: np.ndarray) -> np.ndarray:
    """fp16 bit patterns with -0 (0x8000) mapped to +0."""
    b = np.asarray(bits, dtype=np.uint16).copy()
    b[b == 0x8000] = 0
    return b


def check_tol(y_bits: np.ndarray, y_ref: np.ndarray, absy: np.ndarray, what: str = ""):
    y = f16(y_bits)
    err = np.abs(y - y_ref)
    bound = REL * absy + ABS
    bad = ~(err <= bound)
    if bad.any():
        i = np.argwhere(bad)[0]
        raise AssertionError("%s: %d/%d outside tolerance; first %s: got %r ref %r bound %r" %
                             (what, bad.sum(), bad.size, tuple(i), y[tuple(i)], y_ref[tuple(i)], bound[tuple(i)]))
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0


def run_gemv(w: qmm.PackedWeights, x_bits: np.ndarray, canary: int = 64) -> np.ndarray:
    """GEMV through the C ABI with a canary region after y; returns y bits."""
    m = x_bits.shape[0]
    x = to_dev_u16(x_bits)
    yb = torch.full((m * w.n + canary,), 0x5A5A, dtype=torch.int16, device="cuda")
    y = yb[: m * w.n].view(m, w.n)
    qmm.qmm_gemv(w, x, y)
    assert qmm.qmm_sync_check() == 0
    tail = yb[m * w.n:].cpu()
    assert bool((tail == 0x5A5A).all()), "write past the end of y"
    return from_dev_u16(y)


def oracle_matmul_rows(fmt, n, k, data, scales, global_scale, x_bits, threads=None):
    """oracle.matmul over row blocks on several host threads (each ctypes call
    releases the interpreter lock): the same per-row definition, for full
    outputs of the large matrices.  Returns (y, absy), [m][n]."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or max(1, len(os.sched_getaffinity(0)))
    db, sb = oracle.data_bytes(fmt, 1, k), oracle.scale_bytes(fmt, 1, k)
    cuts = np.linspace(0, n, threads + 1).astype(np.int64)

    def part(i):
        r0, r1 = int(cuts[i]), int(cuts[i + 1])
        if r1 <= r0:
            return r0, None, None
        sc = None if scales is None else scales[r0 * sb:r1 * sb]
        y, a = oracle.matmul(fmt, r1 - r0, k, data[r0 * db:r1 * db], sc, global_scale, x_bits)
        return r0, y, a

    m = x_bits.shape[0]
    y, a = np.empty((m, n)), np.empty((m, n))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for r0, yy, aa in ex.map(part, range(threads)):
            if yy is not None:
                y[:, r0:r0 + yy.shape[1]], a[:, r0:r0 + aa.shape[1]] = yy, aa
    return y, a


def oracle_grouped_full(w, x_bits, ids, per_pair, threads=None):
    """The oracle's grouped product for every (token, slot, row), over
    tokens on several host threads.  Returns (y, absy), [t][topk][n]."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    threads = threads or max(1, len(os.sched_getaffinity(0)))
    t, topk = ids.shape

    def one(tok):
        if per_pair:   # one activation row per pair: pairs as tokens of one slot
            xs = np.ascontiguousarray(x_bits[tok])
            ii = np.ascontiguousarray(ids[tok].reshape(topk, 1))
        else:
            xs = np.ascontiguousarray(x_bits[tok][None])
            ii = np.ascontiguousarray(ids[tok][None])
        yy, aa = oracle.grouped_gemv(w.fmt, w.n, w.k, w.data, w.data_stride, w.scales,
                                     0 if w.scales is None else w.scale_stride, w.global_scale, w.experts, xs, ii)
        return tok, yy.reshape(topk, w.n), aa.reshape(topk, w.n)

    y, a = np.empty((t, topk, w.n)), np.empty((t, topk, w.n))
    with ThreadPoolExecutor(max_workers=threads) as ex:
        for tok, yy, aa in ex.map(one, range(t)):
            y[tok], a[tok] = yy, aa
    return y, a
