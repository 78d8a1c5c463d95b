"""The 2.7B-shaped cached-decode workload at its stated size, in the launch configuration
bench.py times, against the fp64 oracle.

Per layer (H = 80, P = 64, G = 1, N = 128, conv width K = 4): a 4096-token prefix goes
through the prefix conv and the prefill, which leave the conv cache and the SSM state; then
64 decode steps run for every layer.  The 64 steps x every layer are captured into ONE CUDA
graph on one stream with one decode workspace shared by all calls and programmatic
dependent launch between consecutive kernels -- exactly the bench's decode graph -- and the
graph is replayed once.

Checked (the 64-step horizon of the abstract's token-for-token validation, and of blog
§4.3):
  - y_t of every step of every layer against the oracle's chain of decode steps;
  - the SSM state after the 64th step against the oracle, and the conv cache bit-exact;
  - y_t at steps 0, 31 and 63 against a full-prefix recompute on the GPU (the conv and the
    prefill over the 4096 + 64 tokens), the equivalence blog §5.1 states.

Batch 1 runs all 64 layers; batch 16 runs 4 layers (each of its layers costs the oracle a
16-sequence prefill of 4096 tokens).

As in tests/test_gpu_decode.py, the oracle's prefix conv output, rounded to bf16, feeds both
prefills, so the two sides start decoding from states built from the same bits; the GPU conv
is checked against the oracle's conv separately.
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
    Bsz, L, _ = u.shape
    x = u[..., :H * P].reshape(Bsz, L, H, P)
    Bm = u[..., H * P:H * P + G * N].reshape(Bsz, L, G, N)
    Cm = u[..., H * P + G * N:].reshape(Bsz, L, G, N)
    return x, Bm, Cm


@pytest.mark.parametrize("B,n_layers", [(1, 64), (16, 4)])
def test_decode_workload_full_size(B, n_layers):
    w = S.DECODE_WORKLOAD
    H, P, G, N, K, L, steps = w.H, w.P, w.G, w.N, w.K, w.prefix_len, w.steps
    pre_ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, 256, torch.bfloat16),
                         device="cuda", dtype=torch.uint8)
    layers = []
    for layer in range(n_layers):
        prm = S.decode_params(H, P, G, N, K, seed=S.layer_seed(w.seed, layer))
        seq = S.raw_xbc_sequence(B, L + steps, H, P, G, N, dtype="bf16", seed=S.layer_seed(w.seed, 500 + layer))
        pf = f64(prm)
        xbc64, dt64 = seq["xBC"][1], seq["dt"][1]
        d = dict(prm=prm, xbc=dev(seq["xBC"][0]), dt=dev(seq["dt"][0]),
                 A_log=dev(prm["A_log"][0]), D=dev(prm["D"][0]), dt_bias=dev(prm["dt_bias"][0]),
                 cw=dev(prm["conv_w"][0]), cb=dev(prm["conv_b"][0]))
        # prefix: the oracle conv, rounded to the bf16 interface, feeds both prefills
        u64, cs64 = oracle.causal_conv1d(xbc64[:, :L], pf["conv_w"], pf["conv_b"])
        u_bits, u_q = S.to_storage(u64, "bf16")
        u_gpu, conv_state = ssd.ssd_causal_conv1d_fwd(d["xbc"][:, :L].contiguous(), d["cw"], d["cb"])
        torch.cuda.synchronize()
        if layer in (0, n_layers - 1):
            check_close(host64(u_gpu), u64, "bf16", "y", f"layer {layer} prefix conv")
        np.testing.assert_array_equal(host64(conv_state), cs64)
        del u_gpu
        x, Bm, Cm = (t.contiguous() for t in _split(dev(u_bits), H, P, G, N))
        _, ssm = ssd.ssd_chunk_scan_fwd(x, d["dt"][:, :L].contiguous(), d["A_log"], Bm, Cm, D=d["D"], chunk=256,
                                        dt_bias=d["dt_bias"], dt_min=prm["dt_min"], dt_max=prm["dt_max"],
                                        workspace=pre_ws)
        del x, Bm, Cm
        xo, Bo, Co = _split(u_q, H, P, G, N)
        _, h64 = oracle.ssd_scan_sequential(xo, dt64[:, :L], pf["A_log"], Bo, Co, pf["D"], pf["dt_bias"],
                                            pf["dt_min"], pf["dt_max"], None)
        torch.cuda.synchronize()
        check_close(host64(ssm), h64, "bf16", "h", f"layer {layer} state after prefill")
        d.update(ssm=ssm, conv=conv_state,
                 xs=[d["xbc"][:, L + j].contiguous() for j in range(steps)],
                 dts=[d["dt"][:, L + j].contiguous() for j in range(steps)],
                 y=torch.empty((steps, B, H, P), device="cuda", dtype=torch.bfloat16),
                 ref=(h64, cs64, xbc64[:, L:].copy(), dt64[:, L:].copy(), pf))
        layers.append(d)
        del seq, xbc64, dt64, u64, u_bits, u_q, xo, Bo, Co
    del pre_ws

    ws = ssd.decode_workspace(B, H, P, G, N)  # one workspace for every call, as in the bench
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):  # no eager pass: it would advance the states
        for j in range(steps):
            for d in layers:
                prm = d["prm"]
                ssd.ssd_decode_step(d["ssm"], d["conv"], d["xs"][j], d["dts"][j], d["A_log"], d["D"], d["dt_bias"],
                                    d["cw"], d["cb"], H, P, G, N, dt_min=prm["dt_min"], dt_max=prm["dt_max"],
                                    y_t=d["y"][j], workspace=ws, stream=stream)
    graph.replay()
    torch.cuda.synchronize()
    assert ssd.ssd_decode_status(ws) == 0
    del graph

    for layer, d in enumerate(layers):
        h64, cs64, xs64, dts64, pf = d["ref"]
        ys = host64(d["y"])
        for j in range(steps):
            y_ref, h64, cs64 = oracle.decode_step(h64, cs64, xs64[:, j], dts64[:, j], pf["A_log"], pf["D"],
                                                  pf["dt_bias"], pf["dt_min"], pf["dt_max"], pf["conv_w"],
                                                  pf["conv_b"], H, P, G, N)
            check_close(ys[j], y_ref, "bf16", "y", f"layer {layer} decode step {j}")
        check_close(host64(d["ssm"]), h64, "bf16", "h", f"layer {layer} state after {steps} steps")
        np.testing.assert_array_equal(host64(d["conv"]), cs64)
        # the GPU's own full-prefix recompute over L + steps tokens
        u2, _ = ssd.ssd_causal_conv1d_fwd(d["xbc"], d["cw"], d["cb"], want_state=False)
        x2, B2, C2 = (t.contiguous() for t in _split(u2, H, P, G, N))
        y_full, _ = ssd.ssd_chunk_scan_fwd(x2, d["dt"], d["A_log"], B2, C2, D=d["D"], chunk=256,
                                           dt_bias=d["dt_bias"], dt_min=d["prm"]["dt_min"],
                                           dt_max=d["prm"]["dt_max"], want_h_final=False)
        yf = host64(y_full)
        del u2, x2, B2, C2, y_full
        for j in (0, steps // 2 - 1, steps - 1):
            check_close(ys[j], yf[:, L + j], "bf16", "y", f"layer {layer} step {j} against recompute")
