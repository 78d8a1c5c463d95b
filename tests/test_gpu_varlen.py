"""GPU parity of ssd_chunk_scan_varlen_fwd (through the C ABI) against the fp64 varlen oracle:
sequences of different lengths packed into one token stream, each with its own initial and
final state.  Lengths include empty sequences, a single token, block edges (127, 128, 129)
and a full 2.7B-shaped 4096-token sequence beside short ones; both kernel paths.  The
tensor-core path runs the packed batch in one pass from a table of its sequences: 300
sequences (more than one table launch carries), the 64-sequence 2.7B-shaped batch the bench
times (checked on sampled heads), sequences starting at odd tokens, and the call captured in
a CUDA graph and replayed on new contents.
"""
import os

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


def _run(cu, inp, h0, chunk=256, workspace=None):
    return ssd.ssd_chunk_scan_varlen_fwd(
        dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]), dev(inp["Bm"][0][0]),
        dev(inp["Cm"][0][0]), cu, D=dev(inp["D"][0]), chunk=chunk, h0=None if h0 is None else dev(h0[0]),
        dt_bias=dev(inp["dt_bias"][0]), dt_min=inp["dt_min"], dt_max=inp["dt_max"], workspace=workspace)


def _oracle(cu, inp, h0, heads=None):
    hs = slice(None) if heads is None else heads
    gsel = slice(None)
    return oracle.ssd_scan_varlen(
        np.ascontiguousarray(inp["x"][1][0][:, hs]), np.ascontiguousarray(inp["dt"][1][0][:, hs]),
        inp["A_log"][1][hs], inp["Bm"][1][0][:, gsel], inp["Cm"][1][0][:, gsel], cu, D=inp["D"][1][hs],
        dt_bias=inp["dt_bias"][1][hs], dt_min=inp["dt_min"], dt_max=inp["dt_max"],
        h0=None if h0 is None else np.ascontiguousarray(h0[1][:, hs]))


def test_varlen_many_sequences_one_pass():
    # 300 sequences, a quarter of them empty: more entries than one table launch carries
    rng = np.random.default_rng(5)
    lengths = [int(v) if rng.random() > 0.25 else 0 for v in rng.integers(1, 400, 300)]
    cu, inp, h0 = _case(lengths, 8, 2, 128, "bf16", seed=77)
    y, hf = _run(cu, inp, h0)
    torch.cuda.synchronize()
    y_ref, h_ref = _oracle(cu, inp, h0)
    check_close(host64(y), y_ref, "bf16", "y", "300 sequences y")
    check_close(host64(hf), h_ref, "bf16", "h", "300 sequences h_final")
    for i, L in enumerate(lengths):
        if L == 0:
            np.testing.assert_array_equal(host64(hf)[i], h0[1][i])


def test_varlen_bench_batch_sampled_heads():
    lengths = S.varlen_lengths()  # the batch the bench's varlen leg times
    cu, inp, h0 = _case(lengths, 80, 1, 128, "bf16", seed=91)
    y, hf = _run(cu, inp, h0)
    torch.cuda.synchronize()
    heads = [0, 37, 79]  # the oracle on three heads of the 80 (heads never interact)
    y_ref, h_ref = _oracle(cu, inp, h0, heads)
    check_close(host64(y)[:, heads], y_ref, "bf16", "y", "bench batch y, sampled heads")
    check_close(host64(hf)[:, heads], h_ref, "bf16", "h", "bench batch h_final, sampled heads")


@pytest.mark.skipif(os.environ.get("SSD_PREFILL_KERNELS") in ("simt", "fused"),
                    reason="the per-sequence path these switches select rejects unaligned starts (tested below)")
def test_varlen_odd_starts_one_pass():
    # H = 4 bf16: dt rows are 8 bytes, so sequences start off 16-byte boundaries; the one-pass
    # path reads the packed tensors from their bases and takes any start
    lengths = [1, 3, 130, 7, 257]
    cu, inp, h0 = _case(lengths, 4, 1, 128, "bf16", seed=3)
    y, hf = _run(cu, inp, h0)
    torch.cuda.synchronize()
    y_ref, h_ref = _oracle(cu, inp, h0)
    check_close(host64(y), y_ref, "bf16", "y", "odd starts y")
    check_close(host64(hf), h_ref, "bf16", "h", "odd starts h_final")


def test_varlen_rejects_misaligned_dt_rows_per_sequence_path():
    # the CUDA-core path hands each sequence to the prefill as its own arrays: H = 2 f32 dt rows
    # are 8 bytes, so the second sequence's would start off a 16-byte boundary
    cu, inp, _ = _case([1, 3], 2, 1, 16, "f32", seed=3, with_h0=False)
    with pytest.raises(ssd.SSDError):
        ssd.ssd_chunk_scan_varlen_fwd(dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]),
                                      dev(inp["Bm"][0][0]), dev(inp["Cm"][0][0]), cu)


def test_varlen_in_a_graph():
    # the call captured once (its table kernel carries the lengths as launch parameters) and
    # replayed over new contents of the same buffers
    lengths = [200, 0, 1000, 129, 64]
    cu, inp, h0 = _case(lengths, 8, 1, 128, "bf16", seed=13)
    x, dt, Bm, Cm = (dev(inp[k][0][0]) for k in ("x", "dt", "Bm", "Cm"))
    A_log, D, dt_bias = (dev(inp[k][0]) for k in ("A_log", "D", "dt_bias"))
    h0d = dev(h0[0])
    y = torch.empty_like(x)
    hf = torch.empty_like(h0d)
    ws = torch.empty(ssd.ssd_chunk_scan_varlen_workspace_size(cu, 8, 64, 1, 128), device="cuda", dtype=torch.uint8)
    kw = dict(D=D, h0=h0d, dt_bias=dt_bias, dt_min=inp["dt_min"], dt_max=inp["dt_max"], y=y, h_final=hf, workspace=ws)
    stream = torch.cuda.Stream()
    with torch.cuda.stream(stream):
        ssd.ssd_chunk_scan_varlen_fwd(x, dt, A_log, Bm, Cm, cu, **kw)  # warm-up outside the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        ssd.ssd_chunk_scan_varlen_fwd(x, dt, A_log, Bm, Cm, cu, **kw)
    for seed in (21, 22):
        new = S.prefill_inputs(1, int(cu[-1]), 8, 64, 1, 128, dtype="bf16", seed=seed, dt_bias_zero=False)
        for dst, k in ((x, "x"), (dt, "dt"), (Bm, "Bm"), (Cm, "Cm")):
            dst.copy_(dev(new[k][0][0]))
        graph.replay()
        torch.cuda.synchronize()
        new["A_log"], new["D"], new["dt_bias"] = inp["A_log"], inp["D"], inp["dt_bias"]
        y_ref, h_ref = _oracle(cu, new, h0)
        check_close(host64(y), y_ref, "bf16", "y", f"graph replay {seed} y")
        check_close(host64(hf), h_ref, "bf16", "h", f"graph replay {seed} h_final")
    del graph


@pytest.mark.parametrize("lengths", [[300, 0], [0, 0], [129, 5]])
def test_varlen_status_reset_once_per_call(lengths):
    # the call resets the workspace status word itself (stale contents do not survive), also
    # when its last sequence, or every sequence, is empty and launches no kernel that would
    cu, inp, _ = _case(lengths, 8, 1, 128, "bf16", seed=11, with_h0=False)
    T = int(cu[-1])
    need = ssd.ssd_chunk_scan_varlen_workspace_size(cu, 8, 64, 1, 128, 256, torch.bfloat16)
    ws = torch.full((max(need, 256),), 0xFF, device="cuda", dtype=torch.uint8)
    ssd.ssd_chunk_scan_varlen_fwd(dev(inp["x"][0][0]), dev(inp["dt"][0][0]), dev(inp["A_log"][0]),
                                  dev(inp["Bm"][0][0]), dev(inp["Cm"][0][0]), cu, workspace=ws)
    assert ssd.ssd_chunk_scan_status(ws) == 0, T
