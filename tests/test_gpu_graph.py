"""GPU parity in the launch configuration bench.py times: several layers captured into one
CUDA graph on one stream, one workspace shared by every call, programmatic dependent launch
between consecutive kernels, the graph replayed more than once.  Full 2.7B-shaped sizes,
every output compared with the fp64 oracle.
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


def test_prefill_stack_in_a_graph():
    w = S.PREFILL_WORKLOADS["m2p7b"]
    n_layers = 4
    inps, lay = [], []
    for layer in range(n_layers):
        inp = S.prefill_inputs(w.B, w.L, w.H, w.P, w.G, w.N, dtype=w.dtype,
                               seed=S.layer_seed(w.seed, layer), h0=w.h0)
        inps.append(inp)
        x = dev(inp["x"][0])
        lay.append(dict(x=x, dt=dev(inp["dt"][0]), A_log=dev(inp["A_log"][0]), Bm=dev(inp["Bm"][0]),
                        Cm=dev(inp["Cm"][0]), D=dev(inp["D"][0]), dt_bias=dev(inp["dt_bias"][0]),
                        y=torch.empty_like(x),
                        hf=torch.empty((w.B, w.H, w.P, w.N), device="cuda", dtype=torch.float32)))
    ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(w.B, w.L, w.H, w.P, w.G, w.N, w.chunk, torch.bfloat16),
                     device="cuda", dtype=torch.uint8)
    stream = torch.cuda.Stream()

    def step():
        for l, inp in zip(lay, inps):
            ssd.ssd_chunk_scan_fwd(l["x"], l["dt"], l["A_log"], l["Bm"], l["Cm"], D=l["D"], chunk=w.chunk,
                                   dt_bias=l["dt_bias"], dt_min=inp["dt_min"], dt_max=inp["dt_max"],
                                   y=l["y"], h_final=l["hf"], workspace=ws, stream=stream)

    with torch.cuda.stream(stream):
        step()  # eager once (kernel attributes), then capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step()
    for l in lay:  # the replays must produce every output themselves
        l["y"].fill_(float("nan"))
        l["hf"].fill_(float("nan"))
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    assert ssd.ssd_chunk_scan_status(ws) == 0
    for layer, (l, inp) in enumerate(zip(lay, inps)):
        y_ref, h_ref = oracle.ssd_scan_sequential(*oracle_args(f64(inp)))
        check_close(host64(l["y"]), y_ref, w.dtype, "y", f"graph layer {layer} y")
        check_close(host64(l["hf"]), h_ref, w.dtype, "h", f"graph layer {layer} h_final")
    del graph


def test_decode_steps_in_a_graph():
    B, H, P, G, N, K = 16, 80, 64, 1, 128, 4
    n_layers, n_steps = 2, 3
    prms, states, refs = [], [], []
    for layer in range(n_layers):
        prm = S.decode_params(H, P, G, N, K, seed=20 + layer)
        tok0 = S.decode_token_inputs(B, H, P, G, N, K, dtype="bf16", seed=30 + layer)
        prms.append(prm)
        states.append({"ssm": dev(tok0["ssm_state"][0]).clone(), "conv": dev(tok0["conv_state"][0]).clone()})
        refs.append([tok0["ssm_state"][1], tok0["conv_state"][1]])
    toks = [[S.decode_token_inputs(B, H, P, G, N, K, dtype="bf16", seed=100 + 10 * layer + t)
             for t in range(n_steps)] for layer in range(n_layers)]
    dev_tok = [[(dev(tk["xBC_t"][0]), dev(tk["dt_t"][0])) for tk in row] for row in toks]
    dev_prm = [{k: dev(p[k][0]) for k in ("A_log", "D", "dt_bias", "conv_w", "conv_b")} for p in prms]
    ys = [[torch.empty((B, H, P), device="cuda", dtype=torch.bfloat16) for _ in range(n_steps)]
          for _ in range(n_layers)]
    ws = ssd.decode_workspace(B, H, P, G, N)  # one workspace for every layer, as in the bench
    stream = torch.cuda.Stream()

    def run():
        for t in range(n_steps):
            for layer in range(n_layers):
                p, st = dev_prm[layer], states[layer]
                ssd.ssd_decode_step(st["ssm"], st["conv"], dev_tok[layer][t][0], dev_tok[layer][t][1],
                                    p["A_log"], p["D"], p["dt_bias"], p["conv_w"], p["conv_b"], H, P, G, N,
                                    dt_min=prms[layer]["dt_min"], dt_max=prms[layer]["dt_max"],
                                    y_t=ys[layer][t], workspace=ws, stream=stream)

    # capture first (no eager pass: it would advance the states); the graph runs once
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    graph.replay()
    torch.cuda.synchronize()
    assert ssd.ssd_decode_status(ws) == 0
    for layer in range(n_layers):
        pf = f64(prms[layer])
        ssm_ref, conv_ref = refs[layer]
        for t in range(n_steps):
            ft = f64(toks[layer][t])
            y_ref, ssm_ref, conv_ref = oracle.decode_step(
                ssm_ref, conv_ref, ft["xBC_t"], ft["dt_t"], pf["A_log"], pf["D"], pf["dt_bias"],
                pf["dt_min"], pf["dt_max"], pf["conv_w"], pf["conv_b"], H, P, G, N)
            check_close(host64(ys[layer][t]), y_ref, "bf16", "y", f"graph layer {layer} step {t} y")
        check_close(host64(states[layer]["ssm"]), ssm_ref, "bf16", "h", f"graph layer {layer} state")
        np.testing.assert_array_equal(host64(states[layer]["conv"]), conv_ref)
    del graph
