"""The C-ABI library loads and exports every entry point include/qmm.h
declares (no GPU needed: no compute call is made)."""
import ctypes
import os
import re

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
    for want in ("qmm_dequant", "qmm_gemv", "qmm_gemm", "qmm_route", "qmm_grouped_gemv", "qmm_sync_check"):
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
    for fmt in (1, 2, 3):
        for n, k in ((256, 512), (18560, 4096), (1792, 2560), (2560, 896), (3, 64), (0, 32)):
            assert qmm.qmm_data_bytes(fmt, n, k) == oracle.data_bytes(fmt, n, k)
            assert qmm.qmm_scale_bytes(fmt, n, k) == oracle.scale_bytes(fmt, n, k)
    assert qmm.qmm_packed_bytes(2, 18560, 4096) == 47513600
    assert qmm.qmm_packed_bytes(3, 18560, 4096) == 42762244
    assert qmm.qmm_data_bytes(1, 1, 48) == 0          # k not a multiple of 32: invalid
    assert qmm.qmm_data_bytes(9, 1, 32) == 0          # bad format


def test_product_path_does_not_import_the_oracle():
    """The package and its C sources never reference the oracle."""
    pkg = os.path.join(ROOT, "packed_bit_weight_b200")
    for dirpath, _, files in os.walk(pkg):
        for fn in files:
            if fn.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, fn)).read()
                assert "import oracle" not in src and "from oracle" not in src and "qmm_oracle" not in src, fn
