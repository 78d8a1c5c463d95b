"""Failure detection on the GPU without a fault: the bounded waits of the tensor-core
kernels give up, report SSD_ERR_TIMEOUT through a status word, and leave the context usable.

The self-test entry point makes one warp wait, with the same bounded-wait helper the prefill
kernels use, on an mbarrier that no thread ever arrives at (a flag that nothing sets).
"""
import time

import pytest
import torch

import ssd_synth as S
from test_gpu_prefill import compare

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mamba_ssd_b200 as ssd

SSD_OK, SSD_ERR_TIMEOUT = 0, 5


@pytest.mark.parametrize("limit_us", [1000, 20000])
def test_bounded_wait_gives_up_and_reports(limit_us):
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    status = ssd.ssd_selftest_wait_timeout(limit_us)  # synchronises through .item()
    elapsed = time.perf_counter() - t0
    assert status == SSD_ERR_TIMEOUT
    assert elapsed >= limit_us * 1e-6, "the wait gave up before its limit"
    assert elapsed < limit_us * 1e-6 + 5.0, "the wait did not give up"


def test_context_usable_after_timeout():
    assert ssd.ssd_selftest_wait_timeout(1000) == SSD_ERR_TIMEOUT
    # the same process, stream and library: a tensor-core prefill still matches the oracle and
    # its own status word reads SSD_OK
    inp = S.prefill_inputs(1, 300, 4, 64, 1, 128, dtype="bf16", seed=7, h0=True)
    compare(inp, 256, "bf16", "prefill after a timed-out self-test")
    ws = torch.zeros(ssd.ssd_chunk_scan_workspace_size(1, 300, 4, 64, 1, 128, 256, torch.bfloat16),
                     device="cuda", dtype=torch.uint8)
    x = torch.zeros(1, 300, 4, 64, device="cuda", dtype=torch.bfloat16)
    bm = torch.zeros(1, 300, 1, 128, device="cuda", dtype=torch.bfloat16)
    ssd.ssd_chunk_scan_fwd(x, torch.zeros(1, 300, 4, device="cuda", dtype=torch.bfloat16),
                           torch.zeros(4, device="cuda"), bm, bm.clone(), workspace=ws)
    assert ssd.ssd_chunk_scan_status(ws) == SSD_OK
