"""GPU parity of ssd_conv_chunk_scan_fwd (the causal conv and the chunked prefill in one call,
through the C ABI) against the fp64 oracle.

The call keeps the conv output u = SiLU(conv(xBC) + b) in its workspace, after the prefill's
own part (the documented layout), in the storage type.  The GPU rounds its own fp32 conv sums
there, which can differ from the rounded fp64 sums by one storage unit on rare elements, so
the check has two halves, both through the same bits:
  - u against oracle.causal_conv1d, within the storage type's tolerance;
  - y and h_final against oracle.ssd_scan_sequential run on the GPU's own u bits, split into
    x, B and C;
and the conv cache, which only moves raw inputs, exactly.  Cases: the 2.7B-shaped layer
(L = 4096, Cc = 5376, K = 4); the batch-16 decode workload's 4096-token prefix, continued by
decode steps from the cache the call leaves; small shapes (fp32 on the CUDA-core kernels,
N = 16 / 64, two groups, ragged lengths, L < K - 1, no conv bias, a nonzero h0, three heads per
group); the empty prefix.
"""
import numpy as np
import pytest
import torch

import oracle
import ssd_synth as S
from conftest import f64
from parity import check_close, dev, host64

pytestmark = pytest.mark.gpu

if torch.cuda.is_available():
    import mamba_ssd_b200 as ssd


def _split(u, H, P, G, N):
    x = u[..., :H * P].reshape(*u.shape[:-1], H, P)
    Bm = u[..., H * P:H * P + G * N].reshape(*u.shape[:-1], G, N)
    Cm = u[..., H * P + G * N:].reshape(*u.shape[:-1], G, N)
    return x, Bm, Cm


def _run(B, L, H, P, G, N, K, dtype, seed, h0=False, bias=True, chunk=256):
    prm = S.decode_params(H, P, G, N, K, seed=seed)
    if dtype == "f32":
        for k in ("conv_w", "conv_b"):
            v = prm[k][1].astype(np.float32)
            prm[k] = (v, v.astype(np.float64))
    seq = S.raw_xbc_sequence(B, L, H, P, G, N, dtype=dtype, seed=seed + 1)
    h0v = S.prefill_inputs(B, 1, H, P, G, N, dtype="f32", seed=seed + 2, h0=True)["h0"] if h0 else None
    tdt = torch.float32 if dtype == "f32" else torch.bfloat16
    Cc = H * P + 2 * G * N
    ws = torch.empty(ssd.ssd_conv_chunk_scan_workspace_size(B, L, H, P, G, N, K, chunk, tdt), device="cuda",
                     dtype=torch.uint8)
    y, hf, cs = ssd.ssd_conv_chunk_scan_fwd(
        dev(seq["xBC"][0]), dev(prm["conv_w"][0]), dev(prm["conv_b"][0]) if bias else None, dev(seq["dt"][0]),
        dev(prm["A_log"][0]), H, P, G, N, D=dev(prm["D"][0]), chunk=chunk, h0=None if h0v is None else dev(h0v[0]),
        dt_bias=dev(prm["dt_bias"][0]), dt_min=prm["dt_min"], dt_max=prm["dt_max"], workspace=ws)
    torch.cuda.synchronize()
    # the conv output the prefill read: after the prefill's own part of the workspace
    pre = ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, chunk, tdt)
    esz = 4 if dtype == "f32" else 2
    u_gpu = host64(ws[pre:pre + B * L * Cc * esz].view(tdt).view(B, L, Cc))
    pf = f64(prm)
    u64, cs_ref = oracle.causal_conv1d(seq["xBC"][1], pf["conv_w"], pf["conv_b"] if bias else None)
    check_close(u_gpu, u64, dtype, "y", "conv output")
    x, Bm, Cm = (np.ascontiguousarray(t) for t in _split(u_gpu, H, P, G, N))
    y_ref, h_ref = oracle.ssd_scan_sequential(x, seq["dt"][1], pf["A_log"], Bm, Cm, pf["D"], pf["dt_bias"],
                                              pf["dt_min"], pf["dt_max"], None if h0v is None else h0v[1])
    return (y, hf, cs), (y_ref, h_ref, cs_ref), (prm, seq)


def test_conv_prefill_m2p7b_layer():
    (y, hf, cs), (y_ref, h_ref, cs_ref), _ = _run(1, 4096, 80, 64, 1, 128, 4, "bf16", seed=4000)
    check_close(host64(y), y_ref, "bf16", "y", "conv+prefill y")
    check_close(host64(hf), h_ref, "bf16", "h", "conv+prefill h_final")
    np.testing.assert_array_equal(host64(cs), cs_ref)


def test_conv_prefill_then_decode_b16():
    # the batch-16 decode workload: a 4096-token prefix through the one-call conv + prefill, then
    # decode steps from the SSM state and conv cache it leaves, against the oracle's chain
    B, L, H, P, G, N, K, steps = 16, 4096, 80, 64, 1, 128, 4, 3
    (y, hf, cs), (y_ref, h_ref, cs_ref), (prm, _) = _run(B, L, H, P, G, N, K, "bf16", seed=4100)
    check_close(host64(y), y_ref, "bf16", "y", "b16 prefix y")
    check_close(host64(hf), h_ref, "bf16", "h", "b16 prefix state")
    np.testing.assert_array_equal(host64(cs), cs_ref)
    pf = f64(prm)
    ssm = hf.clone()
    ws = ssd.decode_workspace(B, H, P, G, N)
    h64, cs64 = h_ref, cs_ref
    for j in range(steps):
        tok = S.raw_xbc_sequence(B, 1, H, P, G, N, dtype="bf16", seed=4200 + j)
        yt = ssd.ssd_decode_step(ssm, cs, dev(tok["xBC"][0][:, 0]), dev(tok["dt"][0][:, 0]), dev(prm["A_log"][0]),
                                 dev(prm["D"][0]), dev(prm["dt_bias"][0]), dev(prm["conv_w"][0]),
                                 dev(prm["conv_b"][0]), H, P, G, N, dt_min=prm["dt_min"], dt_max=prm["dt_max"],
                                 workspace=ws)
        torch.cuda.synchronize()
        y_t, h64, cs64 = oracle.decode_step(h64, cs64, tok["xBC"][1][:, 0], tok["dt"][1][:, 0], pf["A_log"], pf["D"],
                                            pf["dt_bias"], pf["dt_min"], pf["dt_max"], pf["conv_w"], pf["conv_b"],
                                            H, P, G, N)
        check_close(host64(yt), y_t, "bf16", "y", f"decode step {j} after conv+prefill")
        np.testing.assert_array_equal(host64(cs), cs64)
    check_close(host64(ssm), h64, "bf16", "h", "state after the decode steps")


@pytest.mark.parametrize("B,L,H,G,N,K,dtype,h0,bias,chunk", [
    (2, 300, 4, 2, 16, 4, "f32", True, True, 64),
    (1, 1000, 8, 1, 64, 3, "f32", False, False, 256),
    (2, 2, 4, 1, 16, 4, "f32", True, True, 64),          # L < K - 1: the cache is zero-padded
    (1, 257, 8, 2, 128, 2, "bf16", True, True, 128),     # tensor cores, ragged, two groups
    (2, 130, 6, 2, 128, 4, "bf16", False, True, 256),    # three heads per group
])
def test_conv_prefill_small(B, L, H, G, N, K, dtype, h0, bias, chunk):
    (y, hf, cs), (y_ref, h_ref, cs_ref), _ = _run(B, L, H, 64, G, N, K, dtype, seed=4300 + L, h0=h0, bias=bias,
                                                  chunk=chunk)
    check_close(host64(y), y_ref, dtype, "y", "conv+prefill y")
    check_close(host64(hf), h_ref, dtype, "h", "conv+prefill h_final")
    np.testing.assert_array_equal(host64(cs), cs_ref)


def test_conv_prefill_empty_prefix():
    H, P, G, N, K = 4, 64, 1, 16, 4
    Cc = H * P + 2 * G * N
    xbc = torch.empty((2, 0, Cc), device="cuda", dtype=torch.bfloat16)
    dt = torch.empty((2, 0, H), device="cuda", dtype=torch.bfloat16)
    w = torch.ones((Cc, K), device="cuda", dtype=torch.bfloat16)
    h0 = torch.randn((2, H, P, N), device="cuda")
    y, hf, cs = ssd.ssd_conv_chunk_scan_fwd(xbc, w, None, dt, torch.zeros(H, device="cuda"), H, P, G, N, h0=h0)
    torch.cuda.synchronize()
    assert y.shape == (2, 0, H, P) and torch.count_nonzero(cs) == 0
    assert torch.equal(hf, h0)
