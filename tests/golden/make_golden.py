"""Write tests/golden/tiny_f32_seed0.json from the fp64 oracle alone.

The pages print no worked example, so this fixture is a regression snapshot of the
oracle on the tiny fp32 workload (batch 1, L=512, H=4, P=64, G=1, N=16, seed 0; the
value distributions of "Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching for Inference" as restated in ssd_synth).  It calls only
oracle/ and the seeded generator; nothing here comes from the CUDA path.
Run: python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import ssd_synth as S  # noqa: E402

# flat indices sampled from y and h_final (fixed, spread over chunks, heads and the tail)
Y_IDX = [0, 1, 63, 64, 255 * 256 + 17, 256 * 256 + 5, 511 * 256 + 255, 300 * 256 + 130]
H_IDX = [0, 15, 16 * 64 - 1, 2 * 1024 + 77, 4 * 1024 - 1]


def snapshot():
    w = S.PREFILL_WORKLOADS["tiny_f32"]
    inp = S.prefill_inputs(w.B, w.L, w.H, w.P, w.G, w.N, dtype=w.dtype, seed=w.seed, h0=w.h0)
    f = {k: (v[1] if isinstance(v, tuple) else v) for k, v in inp.items()}
    y, hf = oracle.ssd_scan_sequential(f["x"], f["dt"], f["A_log"], f["Bm"], f["Cm"], f["D"],
                                       f["dt_bias"], f["dt_min"], f["dt_max"], f["h0"])
    return {
        "workload": "tiny_f32 (B1 L512 H4 P64 G1 N16, fp32 storage, seed 0)",
        "source": "oracle.ssd_scan_sequential via tests/golden/make_golden.py",
        "y_sum": float(y.sum()), "y_abs_sum": float(np.abs(y).sum()),
        "h_sum": float(hf.sum()), "h_abs_sum": float(np.abs(hf).sum()),
        "y_idx": Y_IDX, "y_at": [float(v) for v in y.ravel()[Y_IDX]],
        "h_idx": H_IDX, "h_at": [float(v) for v in hf.ravel()[H_IDX]],
    }


if __name__ == "__main__":
    with open(os.path.join(HERE, "tiny_f32_seed0.json"), "w") as fh:
        json.dump(snapshot(), fh, indent=1)
        fh.write("\n")
