"""GPU parity of ssd_gated_rmsnorm_fwd (through the C ABI) against the fp64 oracle.

Shapes: the 2.7B-shaped block output (4096 tokens x 5120 channels, one norm group, and
eight groups of 640), small ragged ones (8 channels, three groups of 8, 33 tokens), groups
that the warp-per-row form takes with 1 to 4 vectors of 16 bytes per lane (up to 1024 bf16 /
512 float32 channels, the largest rows it takes), groups of 1032 channels (the last thread of a row holds part of its 16 elements), both sides of the
streaming form's limit (10240 bf16 / 5120 float32 channels per group streamed; 10248 / 5128
staged), the largest group supported (32768 channels, past the default shared-memory limit),
zero gates, eps = 0, and the empty call.  Tolerances are those of tests/parity.py ("norm").
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_synth as S
from parity import check_close, dev, host64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mamba_ssd_b200 as ssd


def run(inp, n_groups, eps):
    y, z, w = dev(inp["y"][0]), dev(inp["z"][0]), dev(inp["w"][0])
    out = ssd.ssd_gated_rmsnorm_fwd(y, z, w, n_groups=n_groups, eps=eps)
    torch.cuda.synchronize()
    return host64(out)


@pytest.mark.parametrize("dtype,T,C,n_groups,eps", [
    ("bf16", 4096, 5120, 1, 1e-5),
    ("bf16", 4096, 5120, 8, 1e-5),
    ("f32", 512, 5120, 1, 1e-5),
    ("f32", 33, 64, 2, 1e-6),
    ("bf16", 7, 8, 1, 1e-5),
    ("f32", 5, 24, 3, 0.0),
    ("bf16", 64, 4096, 8, 1e-5),
    ("bf16", 21, 3072, 3, 1e-5),
    ("f32", 40, 1024, 2, 1e-5),
    ("bf16", 37, 2064, 2, 1e-5),
    ("f32", 19, 1032, 1, 1e-5),
    ("bf16", 9, 10240, 1, 1e-5),
    ("bf16", 9, 10248, 1, 1e-5),
    ("f32", 6, 5128, 1, 1e-5),
    ("bf16", 3, 32768, 1, 1e-5),
    ("f32", 2, 65536, 2, 1e-5),
])
def test_norm_matches_oracle(dtype, T, C, n_groups, eps):
    inp = S.norm_inputs(T, C, dtype=dtype, seed=T + C + n_groups)
    got = run(inp, n_groups, eps)
    ref = oracle.gated_rmsnorm(inp["y"][1], inp["z"][1], inp["w"][1], eps=eps, n_groups=n_groups)
    check_close(got, ref, dtype, "norm", f"norm {dtype} T{T} C{C} G{n_groups}")


def test_zero_gate_is_exactly_zero():
    inp = S.norm_inputs(16, 256, dtype="bf16", seed=9)
    zb = inp["z"][0].copy()
    zb[:, ::3] = 0  # bf16 bits of +0.0
    inp["z"] = (zb, S.bf16_bits_to_f64(zb))
    got = run(inp, 2, 1e-5)
    assert np.all(got[:, ::3] == 0.0)
    ref = oracle.gated_rmsnorm(inp["y"][1], inp["z"][1], inp["w"][1], eps=1e-5, n_groups=2)
    check_close(got, ref, "bf16", "norm", "zero gates")


def test_empty_and_unsupported():
    y = torch.empty((0, 64), device="cuda", dtype=torch.bfloat16)
    w = torch.ones(64, device="cuda")
    out = ssd.ssd_gated_rmsnorm_fwd(y, y, w)
    assert out.shape == (0, 64)
    y = torch.zeros((2, 12), device="cuda", dtype=torch.bfloat16)  # group of 12: not a multiple of 8
    with pytest.raises(ssd.SSDError):
        ssd.ssd_gated_rmsnorm_fwd(y, y, torch.ones(12, device="cuda"))
