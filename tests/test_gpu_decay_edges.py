"""GPU parity of the prefill on the decay edge cases, against the fp64 oracle.

The workload distributions (dt clipped to [1e-3, 0.1], exp(A_log) in [1, 16]) keep the decay
inside one 32-token sub-block below 2^96, so on their own they never reach the tensor-core
chunk scan's unfactored diagonal branch (a diagonal 32 x 32 sub-block whose cumulative decay
falls by more than 96 in base 2 takes its decay factors one by one instead of through its
middle token).  These cases drive that branch and the special cases of the recurrence:

  no_decay       A_log = -30: exp(dt A) = 1 to fp32 rounding, the state only accumulates
                 (causal linear attention)
  full_decay     A_log = 40: exp(dt A) = 0, each output keeps only its own token's term
  steep_unit_dt  dt = 1, A = -33: the decay falls by ~48 (base 2) per token
  steep_partial  dt in [0.075, 0.125], A = -40: 3 to 5 nats per token, so the previous few
                 tokens still count while every diagonal sub-block is unfactored
  mixed_heads    exp(A_log) from 1 to 60 across the heads of one call: factored and
                 unfactored diagonal sub-blocks side by side in the same CTAs

Every case runs on bf16 storage with P = 64, N = 128 (the tensor-core kernels) and on fp32
storage (the CUDA-core kernels); tests/test_gpu_switches.py runs this file again with every
shape sent to the CUDA-core kernels.
"""
import math

import numpy as np
import pytest
import torch

import ssd_synth as S
from test_gpu_prefill import compare

pytestmark = pytest.mark.gpu

H = 8
EDGES = {
    "no_decay": dict(a_log=-30.0, dt_clip=(1e-3, 0.1)),
    "full_decay": dict(a_log=40.0, dt_clip=(1e-3, 0.1)),
    "steep_unit_dt": dict(a_log=3.5, dt_clip=(1.0, 1.0)),
    "steep_partial": dict(a_log=math.log(40.0), dt_clip=(0.075, 0.125)),
    "mixed_heads": dict(a_log=np.log(np.linspace(1.0, 60.0, H)), dt_clip=(1e-3, 0.1)),
}


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("case", sorted(EDGES))
def test_decay_edge_case(case, dtype):
    # two sequences of 1000 tokens (seven full 128-token blocks and a ragged one), two groups,
    # a nonzero h0 and dt_bias, so the carried-in state meets every decay regime too
    inp = S.prefill_inputs(2, 1000, H, 64, 2, 128, dtype=dtype, seed=900 + sorted(EDGES).index(case),
                           h0=True, dt_bias_zero=False, **EDGES[case])
    compare(inp, 256, dtype, f"{case} {dtype}")


def test_steep_decay_reaches_the_unfactored_branch():
    # the cases above are only meaningful if they cross the threshold: check on the host that
    # the steep cases' decay over one 32-token sub-block exceeds 96 in base 2, and that the
    # mixed case has heads on both sides of it
    def drop32(a_log, dt):
        return 31.0 * dt * math.exp(a_log) / math.log(2.0)

    assert drop32(3.5, 1.0) > 96.0
    assert drop32(math.log(40.0), 0.075) > 96.0
    drops = [drop32(a, 0.1) for a in EDGES["mixed_heads"]["a_log"]]
    assert min(drops) < 96.0 < max(drops)
