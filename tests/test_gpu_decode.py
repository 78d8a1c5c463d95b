"""GPU parity of ssd_decode_step and ssd_causal_conv1d_fwd (through the C ABI) against
the fp64 oracle, and the cached-decode pipeline of the 2.7B-shaped decode workload:
conv prefix + prefill over 4096 tokens, then decode steps, checked against the oracle
and against a full-prefix recompute on the GPU."""
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


def gpu_decode(state, prm, tok, H, P, G, N, ws=None):
    y = ssd.ssd_decode_step(state["ssm"], state["conv"], dev(tok["xBC_t"][0]), dev(tok["dt_t"][0]),
                            dev(prm["A_log"][0]), dev(prm["D"][0]), dev(prm["dt_bias"][0]),
                            dev(prm["conv_w"][0]), dev(prm["conv_b"][0]), H, P, G, N,
                            dt_min=prm["dt_min"], dt_max=prm["dt_max"], workspace=ws)
    return y


def _conv_params(H, P, G, N, K, dtype, seed):
    prm = S.decode_params(H, P, G, N, K, seed=seed)
    if dtype == "f32":
        for k in ("conv_w", "conv_b"):
            v = prm[k][1].astype(np.float32)
            prm[k] = (v, v.astype(np.float64))
    return prm


@pytest.mark.parametrize("dtype,B,H,G,N,K", [
    ("bf16", 1, 80, 1, 128, 4), ("bf16", 3, 8, 2, 64, 4), ("f32", 2, 4, 1, 16, 4),
    ("f32", 1, 8, 2, 256, 3), ("bf16", 2, 6, 3, 32, 2), ("bf16", 16, 80, 1, 128, 4),
])
def test_decode_steps_match_oracle(dtype, B, H, G, N, K):
    P = 64
    prm = _conv_params(H, P, G, N, K, dtype, seed=3)
    tok0 = S.decode_token_inputs(B, H, P, G, N, K, dtype=dtype, seed=4)
    state = {"ssm": dev(tok0["ssm_state"][0]).clone(), "conv": dev(tok0["conv_state"][0]).clone()}
    ref_ssm, ref_conv = tok0["ssm_state"][1], tok0["conv_state"][1]
    ws = ssd.decode_workspace(B, H, P, G, N)
    ws.fill_(0xA5)  # the workspace needs no initialisation: every call writes what it reads
    pf = f64(prm)
    for step in range(3):  # consecutive steps reuse one workspace
        tok = S.decode_token_inputs(B, H, P, G, N, K, dtype=dtype, seed=10 + step)
        y = gpu_decode(state, prm, tok, H, P, G, N, ws)
        torch.cuda.synchronize()
        ft = f64(tok)
        y_ref, ref_ssm, ref_conv = oracle.decode_step(
            ref_ssm, ref_conv, ft["xBC_t"], ft["dt_t"], pf["A_log"], pf["D"], pf["dt_bias"],
            pf["dt_min"], pf["dt_max"], pf["conv_w"], pf["conv_b"], H, P, G, N)
        check_close(host64(y), y_ref, dtype, "y", f"step {step} y")
        check_close(host64(state["ssm"]), ref_ssm, dtype, "h", f"step {step} state")
        # the conv cache only moves raw inputs: exact
        np.testing.assert_array_equal(host64(state["conv"]), ref_conv)
    assert ssd.ssd_decode_status(ws) == 0, "the decode kernels must leave the status word at SSD_OK"


@pytest.mark.parametrize("dtype,B,L,Cc,K", [
    ("bf16", 1, 1, 64, 4), ("bf16", 2, 2, 72, 4), ("f32", 1, 3, 16, 4), ("f32", 2, 70, 40, 3),
    ("bf16", 1, 4096, 5376, 4), ("bf16", 3, 130, 128, 2),
    # 32-token strips and 8-token request batches: lengths around both, every K up to 8
    ("bf16", 2, 33, 64, 8), ("f32", 1, 65, 24, 5), ("bf16", 1, 31, 8, 6), ("bf16", 1, 32, 16, 7),
    ("f32", 2, 9, 32, 2),
    # several 128-thread channel blocks with a partial last one, several sequences over several
    # strips, odd K in bf16
    ("bf16", 2, 100, 520, 5), ("bf16", 3, 70, 264, 3),
])
def test_causal_conv_matches_oracle(dtype, B, L, Cc, K):
    rng = np.random.default_rng(L + Cc)
    xbc = S.to_storage(rng.standard_normal((B, L, Cc), dtype=np.float32), dtype)
    w = S.to_storage(rng.uniform(-0.5, 0.5, (Cc, K)).astype(np.float32), dtype)
    b = S.to_storage(rng.uniform(-0.5, 0.5, Cc).astype(np.float32), dtype)
    out, cs = ssd.ssd_causal_conv1d_fwd(dev(xbc[0]), dev(w[0]), dev(b[0]))
    torch.cuda.synchronize()
    out_ref, cs_ref = oracle.causal_conv1d(xbc[1], w[1], b[1])
    check_close(host64(out), out_ref, dtype, "y", "conv out")
    np.testing.assert_array_equal(host64(cs), cs_ref)


def test_causal_conv_without_bias():
    rng = np.random.default_rng(5)
    B, L, Cc, K = 2, 40, 48, 4
    xbc = S.to_storage(rng.standard_normal((B, L, Cc), dtype=np.float32), "bf16")
    w = S.to_storage(rng.uniform(-0.5, 0.5, (Cc, K)).astype(np.float32), "bf16")
    out, cs = ssd.ssd_causal_conv1d_fwd(dev(xbc[0]), dev(w[0]), None)
    torch.cuda.synchronize()
    out_ref, cs_ref = oracle.causal_conv1d(xbc[1], w[1], None)
    check_close(host64(out), out_ref, "bf16", "y", "conv out, no bias")
    np.testing.assert_array_equal(host64(cs), cs_ref)


def test_conv_empty_prefix_gives_zero_cache():
    xbc = torch.empty((2, 0, 64), device="cuda", dtype=torch.bfloat16)
    w = torch.ones((64, 4), device="cuda", dtype=torch.bfloat16)
    _, cs = ssd.ssd_causal_conv1d_fwd(xbc, w, None)
    torch.cuda.synchronize()
    assert cs.shape == (2, 64, 3) and torch.count_nonzero(cs) == 0


def _split(u, H, P, G, N):
    Bsz, L, _ = u.shape
    x = u[..., :H * P].reshape(Bsz, L, H, P)
    Bm = u[..., H * P:H * P + G * N].reshape(Bsz, L, G, N)
    Cm = u[..., H * P + G * N:].reshape(Bsz, L, G, N)
    return x, Bm, Cm


@pytest.mark.parametrize("B,steps", [(1, 8), (16, 3)])
def test_prefill_then_decode_pipeline(B, steps):
    """2.7B-shaped cached decode on one layer: a 4096-token prefix through the conv and the
    prefill, then decode steps.

    The prefix conv output is stored as bf16 between the conv and the prefill (the
    interface's storage type).  GPU and oracle round their own conv sums, which can differ
    by one bf16 ulp on a few elements, so both prefills are fed the same bits: the oracle's
    conv output rounded to bf16.  The GPU conv is checked against those bits separately.
    Then y_t and the state after every decode step are compared with the oracle, and y_t
    with a full-prefix recompute on the GPU.
    """
    w = S.DECODE_WORKLOAD
    H, P, G, N, K, L = w.H, w.P, w.G, w.N, w.K, w.prefix_len
    prm = S.decode_params(H, P, G, N, K, seed=S.layer_seed(w.seed, 0))
    seq = S.raw_xbc_sequence(B, L + steps, H, P, G, N, dtype="bf16", seed=S.layer_seed(w.seed, 500))
    xbc_dev = dev(seq["xBC"][0])
    dt_dev = dev(seq["dt"][0])
    A_log, D, dt_bias = dev(prm["A_log"][0]), dev(prm["D"][0]), dev(prm["dt_bias"][0])
    cw, cb = dev(prm["conv_w"][0]), dev(prm["conv_b"][0])
    pf = f64(prm)
    xbc64, dt64 = seq["xBC"][1], seq["dt"][1]
    # oracle conv of the prefix, rounded to the bf16 interface
    u64, cs64 = oracle.causal_conv1d(xbc64[:, :L], pf["conv_w"], pf["conv_b"])
    u_bits, u_q = S.to_storage(u64, "bf16")
    # the GPU conv agrees with those bits to within one bf16 rounding
    u_gpu, conv_state = ssd.ssd_causal_conv1d_fwd(xbc_dev[:, :L].contiguous(), cw, cb)
    torch.cuda.synchronize()
    check_close(host64(u_gpu), u64, "bf16", "y", "prefix conv")
    np.testing.assert_array_equal(host64(conv_state), cs64)
    # prefill on identical bits, GPU and oracle
    x, Bm, Cm = (t.contiguous() for t in _split(dev(u_bits), H, P, G, N))
    _, ssm = ssd.ssd_chunk_scan_fwd(x, dt_dev[:, :L].contiguous(), A_log, Bm, Cm, D=D, chunk=256,
                                    dt_bias=dt_bias, dt_min=prm["dt_min"], dt_max=prm["dt_max"])
    xo, Bo, Co = _split(u_q, H, P, G, N)
    _, h64 = oracle.ssd_scan_sequential(xo, dt64[:, :L], pf["A_log"], Bo, Co, pf["D"],
                                        pf["dt_bias"], pf["dt_min"], pf["dt_max"], None)
    torch.cuda.synchronize()
    check_close(host64(ssm), h64, "bf16", "h", "state after prefill")
    ws = ssd.decode_workspace(B, H, P, G, N)
    ys = []
    for j in range(steps):
        t = L + j
        y = ssd.ssd_decode_step(ssm, conv_state, xbc_dev[:, t].contiguous(), dt_dev[:, t].contiguous(),
                                A_log, D, dt_bias, cw, cb, H, P, G, N, dt_min=prm["dt_min"],
                                dt_max=prm["dt_max"], workspace=ws)
        torch.cuda.synchronize()
        ys.append(host64(y))
        y_ref, h64, cs64 = oracle.decode_step(h64, cs64, xbc64[:, t], dt64[:, t], pf["A_log"],
                                              pf["D"], pf["dt_bias"], pf["dt_min"], pf["dt_max"],
                                              pf["conv_w"], pf["conv_b"], H, P, G, N)
        check_close(ys[j], y_ref, "bf16", "y", f"decode step {j}")
        check_close(host64(ssm), h64, "bf16", "h", f"state after decode step {j}")
        np.testing.assert_array_equal(host64(conv_state), cs64)
    # GPU full-prefix recompute over L + steps tokens: same outputs within bf16 tolerance
    u2, _ = ssd.ssd_causal_conv1d_fwd(xbc_dev, cw, cb, want_state=False)
    x2, B2, C2 = (t.contiguous() for t in _split(u2, H, P, G, N))
    y_full, _ = ssd.ssd_chunk_scan_fwd(x2, dt_dev, A_log, B2, C2, D=D, chunk=256, dt_bias=dt_bias,
                                       dt_min=prm["dt_min"], dt_max=prm["dt_max"], want_h_final=False)
    yf = host64(y_full)
    for j in range(steps):
        check_close(ys[j], yf[:, L + j], "bf16", "y", f"recompute step {j}")
