"""Pins of the oracle's products: exact-rational brute force on tiny inputs,
one-hot and integer special cases, the sampled form, and the routed-expert
bucket and per-pair definitions."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from packed_bit_weight_b200 import synth


def _f16(bits):
    return np.asarray(bits, dtype=np.uint16).view(np.float16).astype(np.float64)


def _weights_exact(w):
    """Decoded weights of a Packed matrix as exact Fractions, rounded by
    numpy (independent of the oracle's codec): fp16(code * scale)."""
    n, k = w.n, w.k
    out = np.empty((n, k), dtype=object)
    if w.fmt == synth.FMT_IQ4_NL:
        kv = [int(t) for t in open(__file__.replace("test_oracle_matmul.py", "golden/iq4nl_codebook.txt"))
              .read().splitlines()[-1].split()]
        blocks = w.data.reshape(n, k // 32, 18)
        for r in range(n):
            for b in range(k // 32):
                d = float(np.uint16(int(blocks[r, b, 0]) | (int(blocks[r, b, 1]) << 8)).view(np.float16))
                for j in range(16):
                    lo, hi = blocks[r, b, 2 + j] & 15, blocks[r, b, 2 + j] >> 4
                    out[r, 32 * b + j] = Fraction(float(np.float16(d * kv[lo])))
                    out[r, 32 * b + j + 16] = Fraction(float(np.float16(d * kv[hi])))
        return out
    mags = [0, 0.5, 1, 1.5, 2, 3, 4, 6]
    codes = w.data.reshape(n, k // 2)
    for r in range(n):
        for kk in range(k):
            byte = codes[r, kk // 2]
            nib = (byte & 15) if kk % 2 == 0 else (byte >> 4)
            c = mags[nib & 7] * (-1 if nib & 8 else 1)
            if w.fmt == synth.FMT_FP4G16_F16:
                s = float(w.scales.view(np.uint16).reshape(n, k // 16)[r, kk // 16].view(np.float16))
                out[r, kk] = Fraction(float(np.float16(c * s)))
            elif w.fmt == synth.FMT_MXFP4:
                import torch
                e = float(torch.tensor([w.scales.reshape(n, k // 32)[r, kk // 32]], dtype=torch.uint8)
                          .view(torch.float8_e8m0fnu).double())
                out[r, kk] = Fraction(float(np.float16(c * e)))
            else:
                import torch
                e = float(torch.tensor([w.scales.reshape(n, k // 16)[r, kk // 16]], dtype=torch.uint8)
                          .view(torch.float8_e4m3fn).float())
                out[r, kk] = Fraction(float(np.float16(np.float32(c * e * np.float64(np.float32(w.global_scale))))))
    return out


@pytest.mark.parametrize("fmt,n,k,m", [(synth.FMT_IQ4_NL, 8, 64, 3), (synth.FMT_IQ4_NL, 5, 32, 1),
                                       (synth.FMT_FP4G16_F16, 8, 32, 2), (synth.FMT_FP4G16_F16, 3, 64, 4),
                                       (synth.FMT_FP4G16_E4M3, 6, 48, 2), (synth.FMT_MXFP4, 4, 64, 3)])
def test_brute_force_exact(fmt, n, k, m):
    rng = np.random.default_rng(7 + n + k)
    w = synth.gen_weights(rng, fmt, n, k)
    x = synth.gen_x(rng, m, k)
    y, a = oracle.matmul(fmt, n, k, w.data, w.scales, w.global_scale, x)
    W = _weights_exact(w)
    X = [[Fraction(float(v)) for v in row] for row in _f16(x)]
    for i in range(m):
        for r in range(n):
            exact = sum(W[r, kk] * X[i][kk] for kk in range(k))
            absum = sum(abs(W[r, kk] * X[i][kk]) for kk in range(k))
            assert abs(Fraction(y[i, r]) - exact) <= Fraction(2 * k, 2 ** 53) * absum
            assert abs(Fraction(a[i, r]) - absum) <= Fraction(2 * k, 2 ** 53) * absum


@pytest.mark.parametrize("fmt", [synth.FMT_IQ4_NL, synth.FMT_FP4G16_F16, synth.FMT_FP4G16_E4M3, synth.FMT_MXFP4])
def test_one_hot_gives_decoded_column(fmt):
    rng = np.random.default_rng(11)
    n, k = 16, 64
    w = synth.gen_weights(rng, fmt, n, k)
    deq = oracle.dequant(fmt, n, k, w.data, w.scales, w.global_scale)
    for col in (0, 17, 63):
        x = np.zeros((1, k), dtype=np.uint16)
        x[0, col] = 0x3C00                        # 1.0
        y, _ = oracle.matmul(fmt, n, k, w.data, w.scales, w.global_scale, x)
        assert np.array_equal(y[0].astype(np.float16).view(np.uint16) & 0x7FFF, deq[:, col] & 0x7FFF)
        assert np.array_equal(y[0], _f16(deq[:, col]))


def test_integer_special_case_is_exact():
    """d = 1 and small integer x: every product and sum is an integer well
    inside 2^53, so the double result equals the integer dot product."""
    rng = np.random.default_rng(5)
    n, k = 12, 128
    w = synth.gen_iq4nl(rng, n, k)
    blk = w.data.reshape(n, k // 32, 18)
    blk[..., 0], blk[..., 1] = 0x00, 0x3C               # d = 1.0
    xi = rng.integers(-8, 9, size=(3, k))
    x = xi.astype(np.float16).view(np.uint16)
    y, _ = oracle.matmul(synth.FMT_IQ4_NL, n, k, blk.reshape(-1), None, 1.0, x)
    kv = np.array([int(t) for t in open(__file__.replace("test_oracle_matmul.py", "golden/iq4nl_codebook.txt"))
                   .read().splitlines()[-1].split()])
    q = blk[..., 2:]
    idx = np.concatenate([q & 15, q >> 4], axis=-1).reshape(n, k)      # per block: lows then highs
    wi = kv[idx]
    assert np.array_equal(y, (xi @ wi.T).astype(np.float64))


def test_gemm_rows_equal_gemv_and_sampled_equals_full():
    rng = np.random.default_rng(3)
    n, k, m = 40, 96, 9
    w = synth.gen_fp4(rng, n, k)
    x = synth.gen_x(rng, m, k)
    y, a = oracle.matmul(w.fmt, n, k, w.data, w.scales, 1.0, x)
    for i in range(m):
        yi, ai = oracle.matmul(w.fmt, n, k, w.data, w.scales, 1.0, x[i:i + 1])
        assert np.array_equal(yi[0], y[i]) and np.array_equal(ai[0], a[i])
    mi = rng.integers(0, m, 50)
    ri = rng.integers(0, n, 50)
    ys, as_ = oracle.matmul_sampled(w.fmt, n, k, w.data, w.scales, 1.0, x, mi, ri)
    assert np.array_equal(ys, y[mi, ri]) and np.array_equal(as_, a[mi, ri])


def test_route_buckets_brute_force():
    rng = np.random.default_rng(9)
    ids = synth.gen_topk(rng, 64, 4, 32)
    ids[3, 1] = 40          # out of range: left out of every bucket
    ids[5, 0] = -1
    off, perm, bad = oracle.route(ids, 32)
    assert bad == 2
    flat = ids.reshape(-1)
    for e in range(32):
        want = [p for p in range(flat.size) if flat[p] == e]
        assert list(perm[off[e]:off[e + 1]]) == want
    assert off[0] == 0 and off[32] == flat.size - 2


def test_grouped_equals_per_pair_loop():
    rng = np.random.default_rng(4)
    E, n, k, t, topk = 6, 24, 64, 7, 2
    w = synth.gen_iq4nl(rng, n, k, experts=E)
    x = synth.gen_x(rng, t, k)
    ids = synth.gen_topk(rng, t, topk, E)
    y, a = oracle.grouped_gemv(w.fmt, n, k, w.data, w.data_stride, None, 0, 1.0, E, x, ids)
    for tok in range(t):
        for s in range(topk):
            e = ids[tok, s]
            de = w.data[e * w.data_stride:(e + 1) * w.data_stride]
            yy, aa = oracle.matmul(w.fmt, n, k, de, None, 1.0, x[tok:tok + 1])
            assert np.array_equal(y[tok, s], yy[0]) and np.array_equal(a[tok, s], aa[0])
