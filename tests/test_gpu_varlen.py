"""GPU parity of ssd_chunk_scan_varlen_fwd (through the C ABI) against the fp64 varlen oracle:
sequences of different lengths packed into one token stream, each with its own initial and
final state.  Lengths include empty sequences, a single token, block edges (127, 128, 129)
and a full 2.7B-shaped 4096-token sequence beside short ones; both kernel paths.
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


def _case(lengths, H, G, N, dtype, seed, with_h0=True):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(int)
    T, n = int(cu[-1]), len(lengths)
    inp = S.prefill_inputs(1, T, H, 64, G, N, dtype=dtype, seed=seed, dt_bias_zero=False)
    h0 = S.prefill_inputs(n, 1, H, 64, G, N, dtype="f32", seed=seed + 1, h0=True)["h0"] if with_h0 else None
    return cu, inp, h0


@pytest.mark.parametrize("lengths,H,G,N,dtype,chunk,with_h0", [
    ([0, 1, 127, 128, 129, 300, 2000], 8, 2, 128, "bf16", 256, True),   # tensor cores
    ([5, 0, 256, 257, 64], 4, 1, 64, "f32", 128, True),                 # CUDA cores
    ([4096, 1000, 3, 0], 80, 1, 128, "bf16", 256, False),               # 2.7B heads
    ([700, 33], 8, 1, 32, "bf16", 512, True),                           # CUDA cores, chunk 512
])
def test_varlen_matches_oracle(lengths, H, G, N, dtype, chunk, with_h0):
    cu, inp, h0 = _case(lengths, H, G, N, dtype, seed=sum(lengths) + H, with_h0=with_h0)
    y, hf = ssd.ssd_chunk_scan_varlen_fwd(
        dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]), dev(inp["Bm"][0][0]),
        dev(inp["Cm"][0][0]), cu, D=dev(inp["D"][0]), chunk=chunk, h0=None if h0 is None else dev(h0[0]),
        dt_bias=dev(inp["dt_bias"][0]), dt_min=inp["dt_min"], dt_max=inp["dt_max"])
    torch.cuda.synchronize()
    y_ref, h_ref = oracle.ssd_scan_varlen(
        inp["x"][1][0], inp["dt"][1][0], inp["A_log"][1], inp["Bm"][1][0], inp["Cm"][1][0], cu,
        D=inp["D"][1], dt_bias=inp["dt_bias"][1], dt_min=inp["dt_min"], dt_max=inp["dt_max"],
        h0=None if h0 is None else h0[1])
    check_close(host64(y), y_ref, dtype, "y", f"varlen y {lengths}")
    check_close(host64(hf), h_ref, dtype, "h", f"varlen h_final {lengths}")
    for i, L in enumerate(lengths):  # an empty sequence hands its initial state straight through
        if L == 0:
            want = np.zeros_like(h_ref[i]) if h0 is None else h0[1][i]
            np.testing.assert_array_equal(host64(hf)[i], want)


def test_varlen_rejects_misaligned_dt_rows():
    cu, inp, _ = _case([1, 3], 4, 1, 128, "bf16", seed=3, with_h0=False)
    with pytest.raises(ssd.SSDError):
        ssd.ssd_chunk_scan_varlen_fwd(dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]),
                                      dev(inp["Bm"][0][0]), dev(inp["Cm"][0][0]), cu)


@pytest.mark.parametrize("lengths", [[300, 0], [0, 0], [129, 5]])
def test_varlen_status_reset_once_per_call(lengths):
    # the call resets the workspace status word itself (stale contents do not survive), also
    # when its last sequence, or every sequence, is empty and launches no kernel that would
    cu, inp, _ = _case(lengths, 8, 1, 128, "bf16", seed=11, with_h0=False)
    T = int(cu[-1])
    need = ssd.ssd_chunk_scan_workspace_size(1, max(lengths), 8, 64, 1, 128, 256, torch.bfloat16)
    ws = torch.full((max(need, 256),), 0xFF, device="cuda", dtype=torch.uint8)
    ssd.ssd_chunk_scan_varlen_fwd(dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]),
                                  dev(inp["Bm"][0][0]), dev(inp["Cm"][0][0]), cu, workspace=ws)
    assert ssd.ssd_chunk_scan_status(ws) == 0, T
