"""ssd_chunk_scan_fwd_noalloc, the prefill variant whose scratch is the library's built-in
device array, for callers that cannot allocate device memory (engines that own all device
memory, latency-critical paths that must not trigger an allocation).

Called through the C ABI on two calls in a row (the second on different inputs, so stale
scratch contents must not matter), it must give y and h_final within the parity tolerances of
tests/parity.py of both the fp64 oracle and ssd_chunk_scan_fwd on the same inputs; the second
call must leave the device's free memory unchanged (the first call on a device may commit the
array, when the library's device code is loaded lazily); its status word, read through
ssd_chunk_scan_status(NULL), must be SSD_OK; and a shape whose scratch would not fit must be
refused.  This file is collected last on purpose.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_synth as S
from conftest import f64, oracle_args
from parity import check_close, dev, host64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mamba_ssd_b200 as ssd
    from mamba_ssd_b200 import _lib


@pytest.mark.parametrize("dtype,B,L,H,N,chunk,h0", [
    ("bf16", 1, 4096, 24, 128, 256, False),   # a 130M-shaped layer (38.5 MB of scratch)
    ("f32", 2, 700, 4, 16, 128, True),
])
def test_noalloc_matches_oracle_and_workspace_entry_twice(dtype, B, L, H, N, chunk, h0):
    free_after = []
    for call in range(2):
        inp = S.prefill_inputs(B, L, H, 64, 1, N, dtype=dtype, seed=40 + call, h0=h0)
        args = (dev(inp["x"][0]), dev(inp["dt"][0]), dev(inp["A_log"][0]), dev(inp["Bm"][0]),
                dev(inp["Cm"][0]))
        kw = dict(D=dev(inp["D"][0]), chunk=chunk, h0=None if inp["h0"] is None else dev(inp["h0"][0]),
                  dt_bias=dev(inp["dt_bias"][0]), dt_min=inp["dt_min"], dt_max=inp["dt_max"])
        y_ref, h_ref = ssd.ssd_chunk_scan_fwd(*args, **kw)
        y = torch.empty_like(args[0])
        h = torch.empty((B, H, 64, N), device="cuda", dtype=torch.float32)
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        ssd.ssd_chunk_scan_fwd_noalloc(*args, y=y, h_final=h, **kw)
        torch.cuda.synchronize()
        free_after.append((free_before, torch.cuda.mem_get_info()[0]))
        assert ssd.ssd_chunk_scan_status(None) == _lib.SSD_OK
        yo, ho = oracle.ssd_scan_sequential(*oracle_args(f64(inp)))
        check_close(host64(y), yo, dtype, "y", f"noalloc call {call} y against the oracle")
        check_close(host64(h), ho, dtype, "h", f"noalloc call {call} h_final against the oracle")
        check_close(host64(y), host64(y_ref), dtype, "y", f"noalloc call {call} y against the workspace entry")
        check_close(host64(h), host64(h_ref), dtype, "h", f"noalloc call {call} h_final against the workspace entry")
    # the second call committed no device memory
    assert free_after[1][0] == free_after[1][1], free_after


def test_noalloc_rejects_shapes_beyond_its_scratch():
    # 16 sequences of the 2.7B head count: beyond the 48 MiB scratch on either tensor-core path
    # (128 MB of block states, or 52.4 MB of run states with the fused kernels)
    B, L, H, P, G, N, chunk = 16, 256, 80, 64, 1, 128, 256
    need = _lib.lib().ssd_chunk_scan_workspace_size(B, L, H, P, G, N, chunk, _lib.SSD_DTYPE_BF16)
    assert need > _lib.SSD_NOALLOC_SCRATCH_BYTES
    x = torch.empty((B, L, H, P), device="cuda", dtype=torch.bfloat16)
    dt = torch.empty((B, L, H), device="cuda", dtype=torch.bfloat16)
    Bm = torch.empty((B, L, G, N), device="cuda", dtype=torch.bfloat16)
    A_log = torch.zeros(H, device="cuda")
    with pytest.raises(_lib.SSDError) as err:
        ssd.ssd_chunk_scan_fwd_noalloc(x, dt, A_log, Bm, Bm)
    assert err.value.status == _lib.SSD_ERR_WORKSPACE
