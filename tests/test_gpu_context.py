"""The multi-GPU prefill's kernels on one GPU, against the fp64 oracle.

Context parallelism: a sequence is cut into W consecutive segments, and the ranks are played
one after another in this process through the same functions the distributed path uses
(mamba_ssd_b200.parallel.segment_summary, then segment_output with every summary stacked in
rank order, as the all-gather would deliver them).  The segments' y, concatenated, and the
state after the whole sequence must match oracle.ssd_scan_sequential over the whole sequence.
The pieces are checked on their own too: the state-only prefill (y = NULL) gives the same
h_final bits as the full prefill; the segment decay against the oracle's discretisation; the
combine with r = 0 returns h0.

Head sharding: each rank's heads, run on their own (head_sharded_prefill), against the
oracle's slice.
"""
import math

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
    from mamba_ssd_b200 import parallel


def _dev_inputs(inp):
    d = {k: dev(inp[k][0]) for k in ("x", "dt", "Bm", "Cm", "A_log", "D", "dt_bias")}
    d["h0"] = None if inp["h0"] is None else dev(inp["h0"][0])
    return d


@pytest.mark.parametrize("dtype,B,L,H,G,N,W,h0", [
    ("bf16", 1, 4096, 80, 1, 128, 2, True),    # 2.7B-shaped, two segments
    ("bf16", 1, 4096, 80, 1, 128, 3, False),   # three uneven segments
    ("bf16", 2, 1000, 8, 2, 128, 4, True),     # ragged segments of 250 tokens
    ("f32", 2, 700, 4, 1, 16, 2, True),        # CUDA-core kernels
])
def test_context_parallel_segments(dtype, B, L, H, G, N, W, h0):
    inp = S.prefill_inputs(B, L, H, 64, G, N, dtype=dtype, seed=6000 + L + W, h0=h0, dt_bias_zero=False)
    d = _dev_inputs(inp)
    cuts = [L * i // W for i in range(W + 1)]
    segs = [{k: d[k][:, cuts[r]:cuts[r + 1]].contiguous() for k in ("x", "dt", "Bm", "Cm")} for r in range(W)]
    kw = dict(chunk=256, dt_bias=d["dt_bias"], dt_min=inp["dt_min"], dt_max=inp["dt_max"])
    summaries = [parallel.segment_summary(s["x"], s["dt"], d["A_log"], s["Bm"], s["Cm"], **kw) for s in segs]
    states = torch.stack([sm[0] for sm in summaries])
    decays = torch.stack([sm[1] for sm in summaries])
    ys, h_fin = [], None
    for r, s in enumerate(segs):
        y, h_fin_r = parallel.segment_output(r, states, decays, s["x"], s["dt"], d["A_log"], s["Bm"], s["Cm"],
                                             D=d["D"], h0=d["h0"], **kw)
        ys.append(y)
        if h_fin is not None:  # every rank computes the same state after the sequence
            assert torch.equal(h_fin, h_fin_r)
        h_fin = h_fin_r
    torch.cuda.synchronize()
    y_ref, h_ref = oracle.ssd_scan_sequential(*oracle_args(f64(inp)))
    check_close(host64(torch.cat(ys, dim=1)), y_ref, dtype, "y", f"{W} segments y")
    check_close(host64(h_fin), h_ref, dtype, "h", f"{W} segments h_final")


def test_state_only_prefill_matches_full():
    inp = S.prefill_inputs(1, 1500, 8, 64, 1, 128, dtype="bf16", seed=6100, h0=True)
    d = _dev_inputs(inp)
    _, h_full = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A_log"], d["Bm"], d["Cm"], D=d["D"], h0=d["h0"],
                                       dt_min=inp["dt_min"], dt_max=inp["dt_max"])
    y_none, h_only = ssd.ssd_chunk_scan_fwd(d["x"], d["dt"], d["A_log"], d["Bm"], None, h0=d["h0"],
                                            dt_min=inp["dt_min"], dt_max=inp["dt_max"], want_y=False)
    torch.cuda.synchronize()
    assert y_none is None
    assert torch.equal(h_full, h_only)


@pytest.mark.parametrize("dtype,L,unclipped", [("bf16", 4096, False), ("f32", 333, True), ("bf16", 0, False)])
def test_segment_decay(dtype, L, unclipped):
    inp = S.prefill_inputs(3, L, 80, 64, 1, 16, dtype=dtype, seed=6200 + L, dt_bias_zero=False, unclipped=unclipped)
    ld = ssd.ssd_segment_decay(dev(inp["dt"][0]), dev(inp["A_log"][0]), dt_bias=dev(inp["dt_bias"][0]),
                               dt_min=inp["dt_min"], dt_max=inp["dt_max"])
    torch.cuda.synchronize()
    _, dA = oracle.discretise(inp["dt"][1], inp["A_log"][1], inp["dt_bias"][1], inp["dt_min"], inp["dt_max"])
    ref = dA.sum(axis=1) / math.log(2.0)
    np.testing.assert_allclose(host64(ld), ref, rtol=2e-5, atol=1e-6)


def test_state_combine_recurrence():
    g = torch.Generator(device="cuda").manual_seed(3)
    W, B, H, P, N = 4, 2, 3, 64, 16
    states = torch.randn((W, B, H, P, N), generator=g, device="cuda")
    decays = -torch.rand((W, B, H), generator=g, device="cuda") * 4
    h0 = torch.randn((B, H, P, N), generator=g, device="cuda")
    assert torch.equal(ssd.ssd_state_combine(states, decays, 0, h0=h0), h0)
    assert torch.count_nonzero(ssd.ssd_state_combine(states, decays, 0)) == 0
    for r in range(1, W + 1):
        h = h0.double()
        for j in range(r):
            h = torch.exp2(decays[j].double())[:, :, None, None] * h + states[j].double()
        got = ssd.ssd_state_combine(states, decays, r, h0=h0)
        torch.testing.assert_close(got.double(), h, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("W", [2, 4])
def test_head_sharded_prefill(W):
    inp = S.prefill_inputs(1, 2000, 16, 64, 2, 128, dtype="bf16", seed=6300 + W, h0=True)
    d = _dev_inputs(inp)
    y_ref, h_ref = oracle.ssd_scan_sequential(*oracle_args(f64(inp)))
    for r in range(W):
        a, b, _, _ = parallel.head_range(16, 2, W, r)
        y, h = parallel.head_sharded_prefill(d["x"], d["dt"], d["A_log"], d["Bm"], d["Cm"], D=d["D"], h0=d["h0"],
                                             dt_bias=d["dt_bias"], dt_min=inp["dt_min"], dt_max=inp["dt_max"],
                                             rank=r, world=W)
        torch.cuda.synchronize()
        check_close(host64(y), y_ref[:, :, a:b], "bf16", "y", f"heads {a}..{b} y")
        check_close(host64(h), h_ref[:, a:b], "bf16", "h", f"heads {a}..{b} h_final")
