"""GPU parity of ssd_chunk_scan_fwd (through the C ABI) against the fp64 oracle.

Every case feeds the same seeded input bits to both sides and compares y and h_final
element by element with the tolerances of tests/parity.py.  Sizes: the four prefill
workloads at full size (the 64-layer stack on three of its layers) and a sweep of small
shapes that covers several chunks, a ragged tail, L = 1, empty inputs, both storage
types, 1 and 2 groups, zero and nonzero h0 and dt_bias, and guard bands around every
output.
"""
import itertools

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


def run_gpu(inp, chunk, want_h=True):
    y, hf = ssd.ssd_chunk_scan_fwd(
        dev(inp["x"][0]), dev(inp["dt"][0]), dev(inp["A_log"][0]), dev(inp["Bm"][0]),
        dev(inp["Cm"][0]), D=dev(inp["D"][0]), chunk=chunk,
        h0=None if inp["h0"] is None else dev(inp["h0"][0]),
        dt_bias=dev(inp["dt_bias"][0]), dt_min=inp["dt_min"], dt_max=inp["dt_max"],
        want_h_final=want_h)
    torch.cuda.synchronize()
    return host64(y), (None if hf is None else host64(hf))


def compare(inp, chunk, dtype, what):
    f = f64(inp)
    y_ref, h_ref = oracle.ssd_scan_sequential(*oracle_args(f))
    y, h = run_gpu(inp, chunk)
    check_close(y, y_ref, dtype, "y", f"{what} y")
    check_close(h, h_ref, dtype, "h", f"{what} h_final")


@pytest.mark.parametrize("name", ["tiny_f32", "m130m", "m1p3b_b8"])
def test_workload_full(name):
    w = S.PREFILL_WORKLOADS[name]
    inp = S.prefill_inputs(w.B, w.L, w.H, w.P, w.G, w.N, dtype=w.dtype, seed=w.seed, h0=w.h0)
    compare(inp, w.chunk, w.dtype, name)


@pytest.mark.parametrize("layer", [0, 31, 63])
def test_m2p7b_stack_layers(layer):
    w = S.PREFILL_WORKLOADS["m2p7b"]
    inp = S.prefill_inputs(w.B, w.L, w.H, w.P, w.G, w.N, dtype=w.dtype,
                           seed=S.layer_seed(w.seed, layer), h0=w.h0)
    compare(inp, w.chunk, w.dtype, f"m2p7b layer {layer}")


_SWEEP = []
for i, (dtype, L, chunk) in enumerate(itertools.product(["f32", "bf16"], [1, 7, 255, 256, 257, 1000],
                                                         [64, 128, 256])):
    G = 1 + (i % 2)
    N = (16, 128, 32, 64)[i % 4]
    h0 = (i // 2) % 2 == 1
    bias = (i // 3) % 2 == 1
    _SWEEP.append((dtype, L, chunk, G, N, h0, bias))


@pytest.mark.parametrize("dtype,L,chunk,G,N,h0,bias", _SWEEP)
def test_small_sweep(dtype, L, chunk, G, N, h0, bias):
    inp = S.prefill_inputs(2, L, 4, 64, G, N, dtype=dtype, seed=100 + L + chunk, h0=h0,
                           dt_bias_zero=not bias)
    compare(inp, chunk, dtype, f"sweep {dtype} L{L} Q{chunk} G{G} N{N}")


@pytest.mark.parametrize("dtype,L,G,N,h0", [
    ("f32", 1, 1, 16, False), ("f32", 511, 2, 64, True), ("bf16", 513, 1, 32, False),
    ("bf16", 1500, 2, 16, True), ("f32", 9000, 1, 64, True), ("bf16", 9000, 1, 128, False),
])
def test_chunk_512(dtype, L, G, N, h0):
    # chunk 512, the size suggested beyond 8k tokens: one and several chunks, ragged tails.
    # bf16 N = 128 runs on the tensor cores (128-token blocks whatever the chunk); the others
    # run the CUDA-core kernels with 512-token chunks.
    inp = S.prefill_inputs(1, L, 4, 64, G, N, dtype=dtype, seed=500 + L + N, h0=h0)
    compare(inp, 512, dtype, f"chunk 512 {dtype} L{L} G{G} N{N}")


@pytest.mark.parametrize("B,L,H,G,h0", [(1, 32768, 8, 1, False), (2, 20000, 4, 2, True)])
def test_long_sequence_tensor_cores(B, L, H, G, h0):
    # hundreds of 128-token blocks: the state pass walks them all, the TMA coordinates and the
    # per-CTA item ranges reach far into the workspace; the last block is ragged in the second
    inp = S.prefill_inputs(B, L, H, 64, G, 128, dtype="bf16", seed=500 + L, h0=h0)
    compare(inp, 256, "bf16", f"long sequence B{B} L{L} H{H} G{G}")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_unclipped_dt_exercises_softplus(dtype):
    inp = S.prefill_inputs(1, 600, 8, 64, 2, 64, dtype=dtype, seed=77, h0=True,
                           dt_bias_zero=False, unclipped=True)
    compare(inp, 256, dtype, "unclipped")


def test_empty_sequence_returns_h0():
    inp = S.prefill_inputs(2, 0, 4, 64, 1, 16, dtype="bf16", seed=1, h0=True)
    y, h = run_gpu(inp, 256)
    assert y.shape == (2, 0, 4, 64)
    np.testing.assert_array_equal(h, inp["h0"][1])
    inp["h0"] = None
    _, h = run_gpu(inp, 256)
    np.testing.assert_array_equal(h, 0.0)


def test_empty_batch_is_a_no_op():
    inp = S.prefill_inputs(0, 64, 4, 64, 1, 16, dtype="bf16", seed=1)
    y, h = run_gpu(inp, 64)
    assert y.shape == (0, 64, 4, 64) and h.shape == (0, 4, 64, 16)


def _guarded(shape, dtype, pad=64):
    """A buffer with `pad` sentinel elements on each side; returns (full, view)."""
    n = int(np.prod(shape))
    full = torch.full((n + 2 * pad,), 12288.0, device="cuda", dtype=dtype)  # exact in bf16
    return full, full[pad:pad + n].view(shape)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_guard_bands_untouched(dtype):
    B, L, H, P, G, N = 2, 300, 4, 64, 2, 32
    inp = S.prefill_inputs(B, L, H, P, G, N, dtype=dtype, seed=5, h0=True)
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    yfull, y = _guarded((B, L, H, P), tdt)
    hfull, h = _guarded((B, H, P, N), torch.float32)
    ws_need = ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, 128, tdt)
    ssd.ssd_chunk_scan_fwd(dev(inp["x"][0]), dev(inp["dt"][0]), dev(inp["A_log"][0]),
                           dev(inp["Bm"][0]), dev(inp["Cm"][0]), D=dev(inp["D"][0]), chunk=128,
                           h0=dev(inp["h0"][0]), dt_min=1e-3, dt_max=0.1, y=y, h_final=h,
                           workspace=torch.empty(ws_need, device="cuda", dtype=torch.uint8))
    torch.cuda.synchronize()
    for full in (yfull, hfull):
        assert torch.all(full[:64] == 12288.0) and torch.all(full[-64:] == 12288.0)
    f = f64(inp)
    y_ref, h_ref = oracle.ssd_scan_sequential(*oracle_args(f))
    check_close(host64(y), y_ref, dtype, "y", "guarded y")
    check_close(host64(h), h_ref, dtype, "h", "guarded h")


def test_deterministic_and_h_final_optional():
    inp = S.prefill_inputs(1, 1000, 8, 64, 1, 128, dtype="bf16", seed=9, h0=True)
    y1, h1 = run_gpu(inp, 256)
    y2, h2 = run_gpu(inp, 256, want_h=False)
    assert h2 is None
    np.testing.assert_array_equal(y1, y2)


def test_split_resume_on_gpu():
    # prefill(L1 + L2) == prefill(L2, h0 = h_final(L1)), both on the GPU
    inp = S.prefill_inputs(1, 900, 8, 64, 1, 128, dtype="f32", seed=21, h0=True)
    y, h = run_gpu(inp, 256)
    cut = 389
    a = dict(inp)
    b = dict(inp)
    for k in ("x", "dt", "Bm", "Cm"):
        a[k] = (np.ascontiguousarray(inp[k][0][:, :cut]), None)
        b[k] = (np.ascontiguousarray(inp[k][0][:, cut:]), None)
    ya, ha = run_gpu(a, 256)
    b["h0"] = (ha.astype(np.float32), None)
    yb, hb = run_gpu(b, 256)
    check_close(np.concatenate([ya, yb], axis=1), y, "f32", "y", "resume y")
    check_close(hb, h, "f32", "h", "resume h")
