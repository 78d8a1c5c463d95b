"""The oracle and the seeded generator still reproduce the stored snapshot
(tests/golden/tiny_f32_seed0.json, written by tests/golden/make_golden.py from the
oracle alone)."""
import json
import os

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))


def test_tiny_snapshot_reproduces():
    import importlib.util
    spec = importlib.util.spec_from_file_location("make_golden",
                                                  os.path.join(HERE, "golden", "make_golden.py"))
    mg = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mg)
    want = json.load(open(os.path.join(HERE, "golden", "tiny_f32_seed0.json")))
    got = mg.snapshot()
    for k in ("y_sum", "y_abs_sum", "h_sum", "h_abs_sum"):
        assert np.isclose(got[k], want[k], rtol=1e-12, atol=1e-12), k
    np.testing.assert_allclose(got["y_at"], want["y_at"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(got["h_at"], want["h_at"], rtol=1e-12, atol=1e-14)
