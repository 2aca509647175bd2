import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a B200 (sm_100a) and the built CUDA library")


def golden_lines(name):
    """Non-comment, non-empty lines of a golden fixture."""
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.strip() for ln in f if ln.strip() and not ln.lstrip().startswith("#")]


def parse_value(tok: str) -> float:
    """Decimal, 'inf'/'-inf', or '<int>p<exp>' meaning int * 2^exp (exact)."""
    if tok in ("inf", "-inf"):
        return float(tok)
    if "p" in tok:
        mant, ex = tok.split("p")
        return float(int(mant)) * 2.0 ** int(ex)
    return float(tok)
