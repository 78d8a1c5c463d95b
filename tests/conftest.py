import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def pytest_configure(config):
    config.addinivalue_line("markers", "gpu: needs a CUDA device (B200, sm_100a)")


def f64(inp):
    """Float64 views of a ssd_synth input dict (the exact values of the stored bits)."""
    return {k: (v[1] if isinstance(v, tuple) else v) for k, v in inp.items()}


def oracle_args(f):
    return (f["x"], f["dt"], f["A_log"], f["Bm"], f["Cm"], f["D"], f["dt_bias"],
            f["dt_min"], f["dt_max"], f["h0"])
