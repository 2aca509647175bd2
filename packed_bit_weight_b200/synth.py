"""Seeded synthetic inputs of the pages' workload shapes.

This module only draws random numbers and packs them into the byte layouts;
it holds none of the decode or product arithmetic, and both the CUDA path
and the CPU oracle take their inputs from it.

Distributions (one numpy PCG64 generator per workload, seeded by the
workload's seed, draws taken in the order codes, scales, activations,
routing):

* FP4-G16: every 4-bit E2M1 code uniform over its 16 values (so every code
  byte is uniform over 0..255); one scale per 16 consecutive K elements,
  ``|N(0,1)| * 0.05`` rounded to fp16 (config-literal variant) or, for the
  E4M3FN variant of the model card, ``s = |N(0,1)| * 0.05`` in fp32,
  ``g = max(s) / 448`` and block scale ``e4m3(s / g)`` (round to nearest even,
  by torch's float8_e4m3fn cast).
* MXFP4: the same codes and one E8M0 byte per 32 consecutive K elements,
  ``127 + floor(log2(|N(0,1)| * 0.05))`` (the power of two at or below the
  draw, clipped to 0..254).
* IQ4_NL: per 32-weight block a scale ``d = fp16(|N(0,1)| * 0.002)`` and 16
  bytes of uniform random nibble pairs.
* Activations: ``fp16(N(0,1))``.
* Routing: each token picks ``topk`` distinct experts uniformly at random.

Shapes follow the Mamba-2 8B projections and LM head (d_model 4096,
d_inner 8192, in_proj N = 2*8192 + 2*8*128 + 128 = 18560, vocab 256000) and
the 32-expert MoE of the IQ4_NL model card (hidden 2560, expert FFN 896).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np

FMT_IQ4_NL = 1
FMT_FP4G16_F16 = 2
FMT_FP4G16_E4M3 = 3
FMT_MXFP4 = 4
FMT_NAMES = {FMT_IQ4_NL: "iq4_nl", FMT_FP4G16_F16: "fp4g16_f16", FMT_FP4G16_E4M3: "fp4g16_e4m3",
             FMT_MXFP4: "mxfp4"}


@dataclass
class Packed:
    """One packed [n][k] matrix (or a stack of ``experts`` of them)."""
    fmt: int
    n: int
    k: int
    data: np.ndarray            # uint8, IQ4_NL blocks or FP4 codes (stacked over experts)
    scales: np.ndarray | None   # uint8 view of fp16 or e4m3 scales; None for IQ4_NL
    global_scale: float = 1.0
    experts: int = 1

    @property
    def data_stride(self) -> int:
        return self.data.size // self.experts

    @property
    def scale_stride(self) -> int:
        return 0 if self.scales is None else self.scales.size // self.experts

    @property
    def nbytes(self) -> int:
        return self.data.nbytes + (0 if self.scales is None else self.scales.nbytes)


def _fp16_bits(a: np.ndarray) -> np.ndarray:
    return np.asarray(a, dtype=np.float16).view(np.uint16)


def gen_fp4(rng: np.random.Generator, n: int, k: int, fmt: int = FMT_FP4G16_F16, experts: int = 1) -> Packed:
    if k % 16 or (fmt == FMT_MXFP4 and k % 32):
        raise ValueError("FP4-G16 needs k % 16 == 0, MXFP4 k % 32 == 0")
    codes = rng.integers(0, 256, size=(experts, n, k // 2), dtype=np.uint8)
    if fmt == FMT_MXFP4:
        s = np.abs(rng.standard_normal((experts, n, k // 32), dtype=np.float32)) * np.float32(0.05)
        with np.errstate(divide="ignore"):
            e = np.clip(127.0 + np.floor(np.log2(s.astype(np.float64))), 0, 254).astype(np.uint8)
        return Packed(fmt, n, k, codes.reshape(-1), e.reshape(-1), 1.0, experts)
    s = np.abs(rng.standard_normal((experts, n, k // 16), dtype=np.float32)) * np.float32(0.05)
    if fmt == FMT_FP4G16_F16:
        return Packed(fmt, n, k, codes.reshape(-1), _fp16_bits(s).view(np.uint8).reshape(-1), 1.0, experts)
    if fmt != FMT_FP4G16_E4M3:
        raise ValueError("not an FP4 format")
    import torch
    g = np.float32(s.max() / np.float32(448.0)) if s.size else np.float32(1.0)
    e = torch.from_numpy(np.ascontiguousarray(s / g)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    return Packed(fmt, n, k, codes.reshape(-1), e.reshape(-1).copy(), float(g), experts)


def gen_iq4nl(rng: np.random.Generator, n: int, k: int, experts: int = 1) -> Packed:
    if k % 32:
        raise ValueError("IQ4_NL needs k % 32 == 0")
    nb = k // 32
    qs = rng.integers(0, 256, size=(experts, n, nb, 16), dtype=np.uint8)
    d = _fp16_bits(np.abs(rng.standard_normal((experts, n, nb), dtype=np.float32)) * np.float32(0.002))
    blocks = np.empty((experts, n, nb, 18), dtype=np.uint8)
    blocks[..., 0] = (d & 0xFF).astype(np.uint8)        # little-endian fp16 scale first
    blocks[..., 1] = (d >> 8).astype(np.uint8)
    blocks[..., 2:] = qs
    return Packed(FMT_IQ4_NL, n, k, blocks.reshape(-1), None, 1.0, experts)


def gen_weights(rng, fmt, n, k, experts=1) -> Packed:
    if fmt == FMT_IQ4_NL:
        return gen_iq4nl(rng, n, k, experts)
    return gen_fp4(rng, n, k, fmt, experts)


def gen_x(rng: np.random.Generator, *shape: int) -> np.ndarray:
    """fp16 N(0,1) activations as uint16 bit patterns."""
    return _fp16_bits(rng.standard_normal(shape, dtype=np.float32))


def gen_topk(rng: np.random.Generator, t: int, topk: int, experts: int) -> np.ndarray:
    ids = np.empty((t, topk), dtype=np.int32)
    for i in range(t):
        ids[i] = rng.choice(experts, size=topk, replace=False)
    return ids


def gen_router(rng: np.random.Generator, experts: int, k: int):
    """Router weights [experts][k] as fp16 bits, N(0, 1/k) so that the logits
    of N(0,1) activations are about N(0,1), and an fp32 bias N(0, 0.1^2)."""
    w = _fp16_bits(rng.standard_normal((experts, k), dtype=np.float32) / np.float32(np.sqrt(max(k, 1))))
    b = (rng.standard_normal(experts, dtype=np.float32) * np.float32(0.1)).astype(np.float32)
    return w, b


# ---------------------------------------------------------------------------
# The five workloads
# ---------------------------------------------------------------------------
@dataclass
class Workload:
    name: str
    seed: int
    fmt: int
    shapes: dict = field(default_factory=dict)


IQ4_TINY = Workload("iq4nl_gemv_tiny_256x512", 0, FMT_IQ4_NL, dict(n=256, k=512, m=1))
FP4_IN_PROJ = Workload("fp4g16_gemv_mamba2_8b_in_proj_18560x4096_m1", 1, FMT_FP4G16_F16,
                       dict(n=18560, k=4096, m=1))
FP4_SWEEP = Workload("fp4g16_gemv_sweep_out_proj_4096x8192_lm_head_256000x4096", 2, FMT_FP4G16_F16,
                     dict(mats=[("out_proj", 4096, 8192), ("lm_head", 256000, 4096)], ms=[1, 4, 16]))
IQ4_EXPERTS = Workload("iq4nl_grouped_gemv_32x(1792x2560,2560x896)_t64_top4", 3, FMT_IQ4_NL,
                       dict(experts=32, gate_up=(1792, 2560), down=(2560, 896), t=64, topk=4))
FP4_PREFILL = Workload("fp4g16_prefill_gemm_2048x18560x4096", 4, FMT_FP4G16_F16, dict(m=2048, n=18560, k=4096))


def make_gemv(wl: Workload, fmt: int | None = None, n=None, k=None, m=None):
    """(Packed W, x bits [m][k]) for a single-matrix workload, drawn in order
    codes, scales, activations.  n/k/m override the workload's sizes."""
    fmt = wl.fmt if fmt is None else fmt
    n = wl.shapes["n"] if n is None else n
    k = wl.shapes["k"] if k is None else k
    m = wl.shapes["m"] if m is None else m
    rng = np.random.default_rng(wl.seed)
    w = gen_weights(rng, fmt, n, k)
    x = gen_x(rng, m, k)
    return w, x


def make_sweep(fmt: int = FMT_FP4G16_F16, mats=None):
    """{name: (Packed W, x bits [16][k])}: matrices drawn in listed order,
    then one [16][k] activation block per matrix (M=1 and M=4 use its first
    rows)."""
    rng = np.random.default_rng(FP4_SWEEP.seed)
    mats = FP4_SWEEP.shapes["mats"] if mats is None else mats
    ws = {name: gen_weights(rng, fmt, n, k) for name, n, k in mats}
    return {name: (ws[name], gen_x(rng, 16, k)) for name, n, k in mats}


def make_experts(experts=32, gate_up=(1792, 2560), down=(2560, 896), t=64, topk=4, seed=None):
    """Expert stacks and routing for the grouped GEMV: gate+up weights
    (gate rows then up rows, one [1792][2560] matrix per expert), down
    weights ([2560][896] per expert), per-token activations [t][2560],
    per-pair activations [t][topk][896], routing ids [t][topk]."""
    rng = np.random.default_rng(IQ4_EXPERTS.seed if seed is None else seed)
    wgu = gen_iq4nl(rng, gate_up[0], gate_up[1], experts)
    wdn = gen_iq4nl(rng, down[0], down[1], experts)
    x_gu = gen_x(rng, t, gate_up[1])
    x_dn = gen_x(rng, t, topk, down[1])
    ids = gen_topk(rng, t, topk, experts)
    return wgu, wdn, x_gu, x_dn, ids


def make_moe(experts=32, f=896, d=2560, t=64, topk=4, seed=None):
    """Routed-expert block inputs: gate+up stack [E][2f][d] (gate rows, then
    up rows, as the grouped GEMV's stack), down stack [E][d][f], activations
    [t][d], router weights [E][d] fp16 and bias [E] fp32."""
    rng = np.random.default_rng(IQ4_EXPERTS.seed + 100 if seed is None else seed)
    wgu = gen_iq4nl(rng, 2 * f, d, experts)
    wdn = gen_iq4nl(rng, d, f, experts)
    x = gen_x(rng, t, d)
    wr, br = gen_router(rng, experts, d)
    return wgu, wdn, x, wr, br


def make_prefill(fmt: int = FMT_FP4G16_F16, m=None, n=None, k=None):
    s = FP4_PREFILL.shapes
    return make_gemv(FP4_PREFILL, fmt, n or s["n"], k or s["k"], m or s["m"])
