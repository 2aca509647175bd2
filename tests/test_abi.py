"""The C-ABI library loads and exports every entry point include/qmm.h
declares (no GPU needed: no compute call is made)."""
import ctypes
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(qmm_[a-z_0-9]+)\s*\(", src))
    return names


def test_header_declares_the_boundary():
    names = _declared()
    for want in ("qmm_dequant", "qmm_gemv", "qmm_gemm", "qmm_route", "qmm_grouped_gemv", "qmm_router_topk",
                 "qmm_moe_routed", "qmm_sync_check", "qmm_quantize"):
        assert want in names


def test_library_exports_every_declared_symbol():
    from packed_bit_weight_b200 import _build
    path = _build.build()
    L = ctypes.CDLL(path)
    missing = [n for n in sorted(_declared()) if not hasattr(L, n)]
    assert not missing, missing


def test_size_functions_match_the_oracle():
    import oracle
    from packed_bit_weight_b200 import qmm
    for fmt in (1, 2, 3, 4):
        for n, k in ((256, 512), (18560, 4096), (1792, 2560), (2560, 896), (3, 64), (0, 32)):
            assert qmm.qmm_data_bytes(fmt, n, k) == oracle.data_bytes(fmt, n, k)
            assert qmm.qmm_scale_bytes(fmt, n, k) == oracle.scale_bytes(fmt, n, k)
    assert qmm.qmm_packed_bytes(2, 18560, 4096) == 47513600
    assert qmm.qmm_packed_bytes(3, 18560, 4096) == 42762244
    assert qmm.qmm_data_bytes(1, 1, 48) == 0          # k not a multiple of 32: invalid
    assert qmm.qmm_data_bytes(9, 1, 32) == 0          # bad format


def test_moe_workspace_size():
    """Host-side size rule of the routed-expert block's workspace: routing
    offsets and permutation, h in fp16 and the fp32 slot outputs, each
    rounded up to 256 bytes."""
    from packed_bit_weight_b200 import qmm
    import torch
    a = lambda v: (v + 255) // 256 * 256
    E, f, d, t, topk = 32, 896, 2560, 64, 4
    gate = qmm.PackedWeights(1, f, d, torch.zeros(E * qmm.qmm_data_bytes(1, f, d), dtype=torch.uint8), None,
                             1.0, E)
    P = t * topk
    want = a(4 * (E + 1)) + a(4 * P) + a(2 * P * f) + a(4 * P * d)
    assert qmm.qmm_workspace_bytes(qmm.OP_MOE, gate, 0, t, topk) == want
    assert qmm.qmm_workspace_bytes(qmm.OP_GROUPED, gate, 0, t, topk) == a(4 * (E + 1)) + a(4 * P)
    view = gate.rows(f // 2, f)
    assert view.desc().expert_data_stride == gate.desc().expert_data_stride
    assert view.data.data_ptr() - gate.data.data_ptr() == (f // 2) * qmm.qmm_data_bytes(1, 1, d)


def test_product_path_does_not_import_the_oracle():
    """The package and its C sources never reference the oracle."""
    pkg = os.path.join(ROOT, "packed_bit_weight_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src and "qmm_oracle" not in src, fn


C_CLIENT = r"""
#include <stdio.h>
#include <string.h>
#include "qmm.h"

int main(void) {
  qmm_weights w;
  memset(&w, 0, sizeof w);
  w.fmt = QMM_FMT_FP4G16_F16;
  w.n = 18560;
  w.k = 4096;
  w.num_experts = 1;
  w.data = (const void*)(uintptr_t)0x10000;
  w.scales = (const void*)(uintptr_t)0x20000;
  /* in_proj at fp16 scales: 47,513,600 packed bytes */
  if (qmm_packed_bytes(QMM_FMT_FP4G16_F16, 18560, 4096) != 47513600u) return 1;
  if (qmm_data_bytes(QMM_FMT_IQ4_NL, 256, 512) != 73728u) return 2;
  if (qmm_scale_bytes(QMM_FMT_MXFP4, 4, 64) != 8u) return 3;
  if (qmm_packed_bytes(99, 4, 64) != 0u) return 4;
  /* argument errors return before any device call */
  w.fmt = 99;
  if (qmm_gemv(&w, (const uint16_t*)(uintptr_t)0x30000, 1, (uint16_t*)(uintptr_t)0x40000, NULL, 0, NULL)
      != QMM_ERR_INVALID_ARG) return 5;
  if (qmm_gemv(NULL, NULL, 1, NULL, NULL, 0, NULL) != QMM_ERR_INVALID_ARG) return 6;
  if (strlen(qmm_status_string(QMM_ERR_MISALIGNED)) == 0) return 7;
  printf("ok\n");
  return 0;
}
"""


@pytest.mark.parametrize("lang", ["c", "c++"])
def test_plain_c_client_links_and_calls_the_library(tmp_path, lang):
    """The header is valid C99 and C++ (no C++ or torch types cross the
    boundary), and a C program linked against libqmm.so alone reaches the
    size queries and the host-side argument checks."""
    from packed_bit_weight_b200 import _build
    lib = _build.build()
    src = tmp_path / ("client.c" if lang == "c" else "client.cpp")
    src.write_text(C_CLIENT)
    exe = tmp_path / "client"
    cc = ["gcc", "-std=c99"] if lang == "c" else ["g++", "-std=c++17"]
    cmd = cc + ["-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe),
                lib, "-Wl,-rpath," + os.path.dirname(lib)]
    r = subprocess.run(cmd, capture_output=True, text=True)
    assert r.returncode == 0, r.stderr
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", (r.returncode, r.stdout, r.stderr)
