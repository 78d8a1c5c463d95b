#!/usr/bin/env python
"""Benchmark of the Mamba-2 SSD scan library on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl mine|reference]

One step = one chunked-SSD prefill pass (decay factors and block states, state pass, chunk
scan with output correction) over a Mamba-2-2.7B-shaped stack of 64 independent random
layers (batch 1, 4096 tokens, H=80, P=64, G=1, N=128, chunk 256, bf16 storage, fp32
state).  `value` is prefill tokens/s of the whole stack: B*L / (time of one step).  The
same run also measures the cached decode step of the 2.7B-shaped decode workload (64
layers, ssm_state [B,80,64,128] fp32 + conv_state [B,5376,3] bf16, B in {1, 16}, 64
steps from a state built by a 4096-token prefill) and reports it under "decode";
"decode_vs_recompute" divides the prefill of a 1024-, 4096- and 16384-token prefix through
the stack by one batch-1 decode step of it; "block_steps" times the prefix conv, the gated
RMS norm and the conv-fed prefill on one 2.7B layer; "varlen" times a packed batch of 64
sequences of 64 .. 4096 tokens in one varlen call against one prefill call per sequence.

Timing: W untimed warm-up steps, then exactly K steps bracketed by a barrier and
torch.cuda.synchronize(), timed with CUDA events on the launching stream; the step is
captured once in a CUDA graph and replayed.  Each step reads 2.8 GB of distinct layer
inputs, far larger than the 126 MB L2, so no flush is needed between steps.  Multi-GPU
(torchrun): every rank runs its own replica (the scan has no data-path collective);
rank 0 prints the max time over ranks and the summed work.

--impl reference times the fp64 CPU oracle (the only reference implementation there
is), on rank 0, each step one layer of the same workload.
"""
from __future__ import annotations

import argparse
import datetime
import json
import math
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SSD prefill tokens/s (TFLOPS, % tensor peak); decode steps/s (GB/s, % HBM)"

# prefill workload: 2.7B-shaped layer, 64-layer stack
PF = dict(B=1, L=4096, H=80, P=64, G=1, N=128, chunk=256, layers=64, seed=2)
# decode workload: 2.7B-shaped cache, 64 layers, 64 steps after a 4096-token prefill
DEC = dict(H=80, P=64, G=1, N=128, K=4, layers=64, steps=64, prefix=4096, seed=4)


# ---------------------------------------------------------------------------------------
# work accounting (algorithmic: the inputs and outputs the method must touch)
# ---------------------------------------------------------------------------------------
def prefill_flops(B, L, H, P, G, N, chunk):
    """Dense-tile flops of one prefill: per padded token 2GQN + 2HQP + 4HNP."""
    Lp = -(-L // chunk) * chunk
    return B * Lp * (2 * G * chunk * N + 2 * H * chunk * P + 4 * H * N * P)


def prefill_flops_causal(B, L, H, P, G, N, chunk):
    nc = -(-L // chunk)
    tri = chunk * (chunk + 1)  # 2 * (Q(Q+1)/2)
    return B * nc * (G * tri * N + H * tri * P + 4 * H * N * P * chunk)


def chunk_scan_flops(B, L, H, P, G, N, chunk):
    """The chunk-scan kernel's share: C.B^T once per group, the masked product, C h_prev."""
    Lp = -(-L // chunk) * chunk
    return B * Lp * (2 * G * chunk * N + 2 * H * chunk * P + 2 * H * N * P)


def chunk_state_flops(B, L, H, P, G, N, chunk):
    Lp = -(-L // chunk) * chunk
    return B * Lp * 2 * H * N * P


def prefill_bytes(B, L, H, P, G, N, e=2, h0=False):
    return B * L * (2 * H * P * e + 2 * G * N * e + H * e) + (2 if h0 else 1) * B * H * P * N * 4


# Per-kernel bytes the tensor-core prefill (128-token blocks) must move: every tensor a kernel
# reads or writes once, the workspace tensors passed between the kernels included.  These are
# design costs, not algorithmic work: the algorithmic (method-level) work of the prefill is
# prefill_flops / prefill_bytes above, and each kernel's share of it is KERNEL_METHOD_FLOPS.
TC_BLOCK = 128


def _tc_blocks(L):
    return -(-L // TC_BLOCK)


def chunk_state_bytes(B, L, H, P, G, N, e=2):
    """x, B, dt in; fp32 block states S^T and the two fp32 factor rows out."""
    nk = _tc_blocks(L)
    return B * L * (H * P * e + G * N * e + H * e) + B * nk * H * P * N * 4 + 2 * B * H * nk * TC_BLOCK * 4


def state_pass_bytes(B, L, H, P, G, N, h0=False):
    """fp32 block states and each block's decay in; bf16 h_prev^T and h_final (h0) out (in)."""
    nk = _tc_blocks(L)
    return B * nk * H * P * N * 4 + B * H * nk * 4 + B * nk * H * N * P * 2 + (2 if h0 else 1) * B * H * P * N * 4


def chunk_scan_bytes(B, L, H, P, G, N, e=2):
    """x, B, C, bf16 h_prev^T and the factor rows in; y out."""
    nk = _tc_blocks(L)
    return B * L * (2 * H * P * e + 2 * G * N * e) + B * nk * H * N * P * 2 + 2 * B * H * nk * TC_BLOCK * 4


# The fused tensor-core prefill (the default for these shapes): work in units of (head pair,
# 128-token block), CTA ranges cut into runs per head pair; each run leaves one [N][P] fp32
# state per head in a slot (chains + CTAs slots at most).
N_SMS = 148


def _run_slots(B, L, H):
    nch = B * (H // 2)
    return (nch + min(nch * _tc_blocks(L), N_SMS)) * 2  # one state per head of each slot


def run_state_bytes(B, L, H, P, G, N, e=2):
    """x, B, dt in; each run's state (and its decay) out."""
    return B * L * (H * P * e + G * N * e + H * e) + _run_slots(B, L, H) * (N * P * 4 + 4)


def run_pass_bytes(B, L, H, P, G, N, h0=False):
    """The run states read and overwritten by the carry-ins; h_final (and h0)."""
    return 2 * _run_slots(B, L, H) * N * P * 4 + (2 if h0 else 1) * B * H * P * N * 4


def chunk_scan_fused_bytes(B, L, H, P, G, N, e=2):
    """x, B, C, dt and the carry-ins in; y out."""
    return B * L * (2 * H * P * e + 2 * G * N * e + H * e) + _run_slots(B, L, H) * N * P * 4


KERNEL_BYTES = {"chunk_state": chunk_state_bytes, "state_pass": state_pass_bytes, "chunk_scan": chunk_scan_bytes,
                "run_state": run_state_bytes, "run_pass": run_pass_bytes, "chunk_scan_fused": chunk_scan_fused_bytes}
# Each kernel's share of the method-level flops (the dense-tile count of prefill_flops at the
# caller's chunk): the block state is step a3 (2HNP per token), the chunk scan steps a2 + a5 (CB once
# per group, the masked product, C h_prev); the state pass is step a4, a scan with no
# contraction.
KERNEL_METHOD_FLOPS = {"chunk_state": chunk_state_flops, "chunk_scan": chunk_scan_flops,
                       "run_state": chunk_state_flops, "chunk_scan_fused": chunk_scan_flops}
# The sources a kernel's DRAM-traffic capture depends on: a capture is used only while these
# files are byte-identical to the ones it was taken with.
KERNEL_SOURCES = {"chunk_state": ["chunk_state_tc.cu", "items.cuh"], "state_pass": ["state_pass.cu", "items.cuh"],
                  "chunk_scan": ["chunk_scan_tc.cu", "items.cuh"], "run_state": ["run_state_tc.cu", "runs.cuh"],
                  "run_pass": ["run_pass.cu", "runs.cuh"], "chunk_scan_fused": ["chunk_scan_fused.cu", "runs.cuh"]}
SHARED_SOURCES = ["common.cuh", "tc.cuh", "launch.h", "tmap.cu"]
PREFILL_KERNELS = ["decay_prep", "chunk_state", "state_pass", "chunk_scan", "run_state", "run_pass",
                   "chunk_scan_fused"]
TRAFFIC_FILE = os.path.join("profiles", "prefill_traffic_m2p7b_layer.json")


def kernel_source_sha(name):
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[name] + SHARED_SOURCES:
        with open(os.path.join(ROOT, "mamba_ssd_b200", "csrc", f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()


def measured_traffic(name):
    """DRAM bytes per launch (read + write) from the committed ncu capture of the 2.7B-shaped
    layer, or None if there is none or the kernel's sources changed since it was taken."""
    try:
        d = json.load(open(os.path.join(ROOT, TRAFFIC_FILE)))[name]
    except (OSError, KeyError, ValueError):
        return None
    return d["dram_bytes"] if d.get("source_sha256") == kernel_source_sha(name) else None


def decode_bytes(B, H, P, G, N, K, e=2):
    Cc = H * P + 2 * G * N
    return (8 * B * H * P * N + 2 * B * Cc * (K - 1) * e + B * Cc * e + Cc * K * e + Cc * e
            + B * H * P * e + B * H * e + 3 * H * 4)


# ---------------------------------------------------------------------------------------
# environment helpers
# ---------------------------------------------------------------------------------------
def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        d = json.load(open(p))
        return {"hbm_gbs": float(d["hbm_gbs"]), "bf16_tflops": float(d["bf16_tflops"]),
                "bf16_tflops_sustained": float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0,
                "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 100 ms while active."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.f = None

    def __enter__(self):
        self.f = tempfile.NamedTemporaryFile("w+", suffix=".csv", delete=False)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
        return False

    def summary(self):
        rows = []
        try:
            self.f.seek(0)
            for line in open(self.f.name):
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 9:
                    continue
                try:
                    rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
                except ValueError:
                    continue
        finally:
            try:
                os.unlink(self.f.name)
            except OSError:
                pass
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        loaded = [r for r in rows if r[2] > 250.0] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3]) if v.lower() == "active"})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(loaded), "power_w_max": max(r[2] for r in rows)}


def gpu_smi_id(torch):
    """nvidia-smi -i selector of the current device (its UUID, robust to device remapping)."""
    try:
        u = str(torch.cuda.get_device_properties(torch.cuda.current_device()).uuid)
        return u if u.startswith("GPU-") else "GPU-" + u
    except Exception:
        return str(torch.cuda.current_device())


def dist_env():
    return (int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)),
            int(os.environ.get("LOCAL_RANK", 0)))


def max_over_ranks(value, world, device=None):
    """Max of a float over all ranks (identity at world size 1)."""
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def sum_over_ranks(value, world, device=None):
    if world == 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------------------------------
# CPU oracle timing (the cpu_baseline leg and --impl reference)
# ---------------------------------------------------------------------------------------
def oracle_layer_inputs():
    import ssd_synth as S
    inp = S.prefill_inputs(PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], dtype="bf16",
                           seed=S.layer_seed(PF["seed"], 0))
    return {k: (v[1] if isinstance(v, tuple) else v) for k, v in inp.items()}


def oracle_step(f):
    import oracle
    t0 = time.perf_counter()
    oracle.ssd_scan_sequential(f["x"], f["dt"], f["A_log"], f["Bm"], f["Cm"], f["D"], f["dt_bias"],
                               f["dt_min"], f["dt_max"], None)
    return time.perf_counter() - t0


def _timed_reps(fn, min_seconds, max_reps, min_reps=1):
    times = []
    t_start = time.perf_counter()
    while len(times) < max_reps and (len(times) < min_reps or (time.perf_counter() - t_start) < min_seconds):
        times.append(fn())
    return statistics.median(times), len(times)


def oracle_decode_inputs(Bsz):
    """One 2.7B-shaped decode layer's cache and token (seeded), as the oracle consumes them."""
    import ssd_synth as S
    H, P, G, N, K = DEC["H"], DEC["P"], DEC["G"], DEC["N"], DEC["K"]
    prm = S.decode_params(H, P, G, N, K, seed=S.layer_seed(DEC["seed"], 0))
    tok = S.decode_token_inputs(Bsz, H, P, G, N, K, dtype="bf16", seed=S.layer_seed(DEC["seed"], 900))
    f = {k: (v[1] if isinstance(v, tuple) else v) for k, v in {**prm, **tok}.items()}
    return f


def oracle_decode_layer(f):
    import oracle
    H, P, G, N = DEC["H"], DEC["P"], DEC["G"], DEC["N"]
    t0 = time.perf_counter()
    oracle.decode_step(f["ssm_state"], f["conv_state"], f["xBC_t"], f["dt_t"], f["A_log"], f["D"], f["dt_bias"],
                       f["dt_min"], f["dt_max"], f["conv_w"], f["conv_b"], H, P, G, N)
    return time.perf_counter() - t0


def cpu_baseline(min_seconds=10.0, max_reps=50):
    """The fp64 oracle on this host's cores: the prefill recurrence (the headline leg) on all
    cores and on one core, and the cached decode step at batch 1 and 16 on all cores and on one
    core.  Each is timed on one layer of its workload and scaled to the 64-layer stack."""
    import oracle
    f = oracle_layer_inputs()
    cores = oracle.max_threads()
    per_layer, reps = _timed_reps(lambda: oracle_step(f), min_seconds, max_reps)
    tok_s = PF["B"] * PF["L"] / (per_layer * PF["layers"])
    legs = {}
    try:
        oracle.set_threads(1)
        t1, r1 = _timed_reps(lambda: oracle_step(f), 3.0, 3)
        legs["prefill_1core"] = {"tokens_per_s": PF["B"] * PF["L"] / (t1 * PF["layers"]), "cores": 1,
                                 "s_per_layer": t1, "runs": r1}
        for bsz in (1, 16):
            fd = oracle_decode_inputs(bsz)
            for n_threads in (cores, 1):
                oracle.set_threads(n_threads)
                td, rd = _timed_reps(lambda: oracle_decode_layer(fd), 2.0, 200, min_reps=3)
                legs[f"decode_b{bsz}_{'1core' if n_threads == 1 else 'all_cores'}"] = {
                    "steps_per_s": 1.0 / (td * DEC["layers"]), "cores": n_threads, "s_per_layer": td,
                    "runs": rd}
    finally:
        oracle.set_threads(cores)
    return {"value": tok_s, "unit": "tokens/s", "cores": cores, "kind": "oracle",
            "sample": (f"fp64 sequential recurrence on 1 of the 64 layers (all {PF['L']} tokens, "
                       f"{PF['H']} heads), {reps} runs, median {per_layer:.3f} s per layer; "
                       f"stack rate = per-layer rate / 64 (an extrapolation from one layer)"),
            "legs": legs,
            "legs_note": ("each leg times one layer of its workload and divides by 64 layers: prefill "
                          "tokens/s of the 2.7B-shaped stack, decode steps/s of the 64-layer 2.7B-shaped "
                          "cache at batch 1 and 16 (one fp64 decode step per layer)"),
            "host_cpu": _cpu_model(), "nproc": os.cpu_count()}


def _cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return None


def run_reference(args):
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import oracle
    f = oracle_layer_inputs()
    for _ in range(args.warmup):
        oracle_step(f)
    times = [oracle_step(f) for _ in range(args.steps)]
    per_layer = statistics.mean(times)
    value = PF["B"] * PF["L"] / (per_layer * PF["layers"])
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": per_layer * 1e3, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": workload_config(),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle.max_threads(),
                         "kind": "oracle",
                         "sample": "each step: fp64 sequential recurrence over 1 of the 64 layers "
                                   "(4096 tokens, 80 heads); stack rate = per-layer rate / 64"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def workload_config():
    return {"workload": (f"m2p7b_stack: Mamba-2-2.7B-shaped SSD prefill, batch {PF['B']}, "
                         f"L={PF['L']}, H={PF['H']}, P={PF['P']}, G={PF['G']}, N={PF['N']}, "
                         f"chunk {PF['chunk']}, {PF['layers']} independent random layers"),
            "global_batch": PF["B"], "seq_len": PF["L"], "layers": PF["layers"],
            "decode_workload": ("m2p7b_decode: 64 layers x ssm_state[B,80,64,128] fp32 + "
                                "conv_state[B,5376,3] bf16, K=4, 64 steps after a 4096-token prefill"),
            "l2": "inputs larger than L2 (each step reads 2.8 GB of distinct layer inputs); no flush",
            "parallelism": "replicas (no data-path collective)"}


# ---------------------------------------------------------------------------------------
# GPU legs
# ---------------------------------------------------------------------------------------
def make_prefill_layers(torch, device, layers, rank, L=None):
    H, P, G, N, B = PF["H"], PF["P"], PF["G"], PF["N"], PF["B"]
    L = PF["L"] if L is None else L
    out = []
    for layer in range(layers):
        g = torch.Generator(device=device)
        g.manual_seed(PF["seed"] * 1000 + layer + 100_000 * rank)
        bf = torch.bfloat16
        x = torch.randn((B, L, H, P), generator=g, device=device).to(bf)
        dt = (torch.randn((B, L, H), generator=g, device=device) - 2.0).to(bf)
        s = 1.0 / math.sqrt(N)
        Bm = (torch.randn((B, L, G, N), generator=g, device=device) * s).to(bf)
        Cm = (torch.randn((B, L, G, N), generator=g, device=device) * s).to(bf)
        A_log = torch.log(torch.rand((H,), generator=g, device=device) * 15.0 + 1.0)
        D = torch.randn((H,), generator=g, device=device)
        dt_bias = torch.zeros((H,), device=device)
        y = torch.empty_like(x)
        hf = torch.empty((B, H, P, N), device=device, dtype=torch.float32)
        out.append(dict(x=x, dt=dt, Bm=Bm, Cm=Cm, A_log=A_log, D=D, dt_bias=dt_bias, y=y, hf=hf))
    return out


def prefill_call(ssd, lay, ws, stream=None):
    ssd.ssd_chunk_scan_fwd(lay["x"], lay["dt"], lay["A_log"], lay["Bm"], lay["Cm"], D=lay["D"],
                           chunk=PF["chunk"], h0=None, dt_bias=lay["dt_bias"], dt_min=1e-3,
                           dt_max=0.1, y=lay["y"], h_final=lay["hf"], workspace=ws, stream=stream)


def kernel_times(torch, ssd_lib, run_eager, names):
    """Per-kernel CUDA-event durations of one eager pass of the step.  A long sleep kernel
    is queued first so that every launch is enqueued before the GPU reaches it: the events
    then time the kernels, not the host."""
    torch.cuda.synchronize()
    ssd_lib.ssd_kernel_timer_enable(1)
    for n in names:  # drop stale records
        ssd_lib.ssd_kernel_timer_read(n.encode(), None, None)
    torch.cuda._sleep(200_000_000)
    run_eager()
    torch.cuda.synchronize()
    ssd_lib.ssd_kernel_timer_enable(0)
    import ctypes
    res = {}
    for n in names:
        ms = ctypes.c_double(0)
        cnt = ctypes.c_longlong(0)
        ssd_lib.ssd_kernel_timer_read(n.encode(), ctypes.byref(ms), ctypes.byref(cnt))
        res[n] = (ms.value, cnt.value)
    return res


def bench_prefill(args, torch, ssd, device, rank, world):
    from mamba_ssd_b200 import _lib
    lib = _lib.lib()
    layers = make_prefill_layers(torch, device, PF["layers"], rank)
    B, L, H, P, G, N, Q = PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], PF["chunk"]
    ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, Q, torch.bfloat16),
                     device=device, dtype=torch.uint8)
    stream = torch.cuda.Stream(device=device)

    def step_eager():
        for lay in layers:
            prefill_call(ssd, lay, ws)

    # one eager pass (sets kernel attributes before capture), then capture the step
    with torch.cuda.stream(stream):
        step_eager()
    torch.cuda.synchronize()
    n0 = lib.ssd_kernel_launch_count()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        step_eager()
    launches_per_step = lib.ssd_kernel_launch_count() - n0
    torch.cuda.synchronize()

    for _ in range(args.warmup):
        graph.replay()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_smi_id(torch)) as clocks:
        with torch.cuda.stream(stream):
            start.record(stream)
            for _ in range(args.steps):
                graph.replay()
            end.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    ms_max = max_over_ranks(ms, world, device)

    with torch.cuda.stream(stream):
        kt = kernel_times(torch, lib, step_eager, PREFILL_KERNELS)
    kt = {n: v for n, v in kt.items() if v[1] > 0}  # only the kernels of the path that ran
    del graph
    return dict(ms_total=ms_max, launches_per_step=launches_per_step, kernel_times=kt,
                clocks=clocks.summary())


def bench_decode(args, torch, ssd, device, rank, Bsz, steps):
    """64-layer cached decode at batch Bsz: state built by conv + prefill over 4096 tokens,
    then `steps` decode steps captured in one CUDA graph and timed."""
    from mamba_ssd_b200 import _lib
    lib = _lib.lib()
    H, P, G, N, K = DEC["H"], DEC["P"], DEC["G"], DEC["N"], DEC["K"]
    Cc = H * P + 2 * G * N
    bf = torch.bfloat16
    layers = []
    pre_ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(Bsz, DEC["prefix"], H, P, G, N, 256, bf),
                         device=device, dtype=torch.uint8)
    for layer in range(DEC["layers"]):
        g = torch.Generator(device=device)
        g.manual_seed(DEC["seed"] * 1000 + layer + 100_000 * rank)
        bound = 1.0 / math.sqrt(K)
        conv_w = ((torch.rand((Cc, K), generator=g, device=device) * 2 - 1) * bound).to(bf)
        conv_b = ((torch.rand((Cc,), generator=g, device=device) * 2 - 1) * bound).to(bf)
        A_log = torch.log(torch.rand((H,), generator=g, device=device) * 15.0 + 1.0)
        D = torch.randn((H,), generator=g, device=device)
        dt_bias = torch.zeros((H,), device=device)
        scale = torch.ones(Cc, device=device)
        scale[H * P:] = 1.0 / math.sqrt(N)
        xbc = (torch.randn((Bsz, DEC["prefix"], Cc), generator=g, device=device) * scale).to(bf)
        dtp = (torch.randn((Bsz, DEC["prefix"], H), generator=g, device=device) - 2.0).to(bf)
        u, conv_state = ssd.ssd_causal_conv1d_fwd(xbc, conv_w, conv_b)
        x = u[..., :H * P].reshape(Bsz, DEC["prefix"], H, P).contiguous()
        Bm = u[..., H * P:H * P + G * N].reshape(Bsz, DEC["prefix"], G, N).contiguous()
        Cm = u[..., H * P + G * N:].reshape(Bsz, DEC["prefix"], G, N).contiguous()
        _, ssm = ssd.ssd_chunk_scan_fwd(x, dtp, A_log, Bm, Cm, D=D, chunk=256, dt_bias=dt_bias,
                                        dt_min=1e-3, dt_max=0.1, workspace=pre_ws)
        del xbc, dtp, u, x, Bm, Cm
        xs = (torch.randn((steps, Bsz, Cc), generator=g, device=device) * scale).to(bf)
        dts = (torch.randn((steps, Bsz, H), generator=g, device=device) - 2.0).to(bf)
        y = torch.empty((steps, Bsz, H, P), device=device, dtype=bf)
        layers.append(dict(ssm=ssm, conv=conv_state, w=conv_w, b=conv_b, A_log=A_log, D=D,
                           dt_bias=dt_bias, xs=xs, dts=dts, y=y))
    del pre_ws
    ws = ssd.decode_workspace(Bsz, H, P, G, N, device)
    torch.cuda.synchronize()

    def run(step_range):
        for s in step_range:
            for lay in layers:
                ssd.ssd_decode_step(lay["ssm"], lay["conv"], lay["xs"][s], lay["dts"][s], lay["A_log"],
                                    lay["D"], lay["dt_bias"], lay["w"], lay["b"], H, P, G, N,
                                    dt_min=1e-3, dt_max=0.1, y_t=lay["y"][s], workspace=ws)

    stream = torch.cuda.Stream(device=device)
    with torch.cuda.stream(stream):
        run(range(1))
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    n0 = lib.ssd_kernel_launch_count()
    with torch.cuda.graph(graph, stream=stream):
        run(range(steps))
    launches = lib.ssd_kernel_launch_count() - n0
    for _ in range(2):
        graph.replay()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        start.record(stream)
        graph.replay()
        end.record(stream)
    torch.cuda.synchronize()
    ms = start.elapsed_time(end)
    with torch.cuda.stream(stream):
        kt = kernel_times(torch, lib, lambda: run(range(min(steps, 8))), ["decode_conv", "decode_step"])
    del graph
    bytes_step = DEC["layers"] * decode_bytes(Bsz, H, P, G, N, K)
    steps_s = steps / (ms / 1e3)
    # one layer-step is two launches: the conv kernel, then the state update ("decode_step")
    cms, ccnt = kt["decode_conv"]
    kms, kcnt = kt["decode_step"]
    conv_s = cms / max(ccnt, 1) / 1e3
    state_s = kms / max(kcnt, 1) / 1e3
    k_avg_s = conv_s + state_s
    return {"batch": Bsz, "steps": steps, "layers": DEC["layers"], "ms": ms,
            "steps_per_s": steps_s, "gbs": bytes_step * steps_s / 1e9,
            "bytes_per_step": bytes_step, "launches": launches,
            "conv_kernel_avg_us": conv_s * 1e6, "state_kernel_avg_us": state_s * 1e6,
            "kernel_avg_us": k_avg_s * 1e6,
            "kernel_gbs": decode_bytes(Bsz, H, P, G, N, K) / k_avg_s / 1e9 if kcnt else None}


def bench_context_sweep(torch, ssd, device, rank, contexts=(1024, 4096, 16384), dec_steps=16):
    """Cached decode against recomputing the prefix, by context length L.  For each L: the
    64-layer stack's prefill over L tokens (what a model without the cache recomputes for
    every generated token), then B = 1 decode steps of the same stack starting from the
    states that prefill left.  A decode step reads and writes the fixed-size state only, so
    its time must not grow with L while the recompute grows linearly."""
    H, P, G, N, K = PF["H"], PF["P"], PF["G"], PF["N"], DEC["K"]
    Cc = H * P + 2 * G * N
    bf = torch.bfloat16
    stream = torch.cuda.Stream(device=device)
    rows = []
    for L in contexts:
        layers = make_prefill_layers(torch, device, PF["layers"], rank, L=L)
        ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(1, L, H, P, G, N, PF["chunk"], bf),
                         device=device, dtype=torch.uint8)
        with torch.cuda.stream(stream):
            for lay in layers:
                prefill_call(ssd, lay, ws)
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for lay in layers:
                prefill_call(ssd, lay, ws)
        pre_ms = time_graph(torch, graph, stream, reps=3)
        del graph
        # decode from the states the prefill left; per-layer conv taps, cache and tokens
        g = torch.Generator(device=device)
        g.manual_seed(DEC["seed"] * 7 + L)
        scale = torch.ones(Cc, device=device)
        scale[H * P:] = 1.0 / math.sqrt(N)
        dec = []
        for lay in layers:
            dec.append(dict(
                ssm=lay["hf"], A_log=lay["A_log"], D=lay["D"], dt_bias=lay["dt_bias"],
                conv=(torch.randn((1, Cc, K - 1), generator=g, device=device) * scale[:, None]).to(bf),
                w=((torch.rand((Cc, K), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf),
                b=((torch.rand((Cc,), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf),
                xs=(torch.randn((dec_steps, 1, Cc), generator=g, device=device) * scale).to(bf),
                dts=(torch.randn((dec_steps, 1, H), generator=g, device=device) - 2.0).to(bf),
                y=torch.empty((dec_steps, 1, H, P), device=device, dtype=bf)))
            for k in ("x", "dt", "Bm", "Cm", "y"):
                del lay[k]
        del ws
        dws = ssd.decode_workspace(1, H, P, G, N, device)
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            for s in range(dec_steps):
                for d in dec:
                    ssd.ssd_decode_step(d["ssm"], d["conv"], d["xs"][s], d["dts"][s], d["A_log"], d["D"],
                                        d["dt_bias"], d["w"], d["b"], H, P, G, N, dt_min=1e-3, dt_max=0.1,
                                        y_t=d["y"][s], workspace=dws)
        dec_ms = time_graph(torch, graph, stream, reps=3) / dec_steps
        del graph, dec, layers
        torch.cuda.synchronize()
        rows.append({"L": L, "recompute_ms": pre_ms, "decode_step_ms": dec_ms, "speedup": pre_ms / dec_ms})
    return rows


def bench_block_norm(torch, ssd, device, peaks, launches=64, buffers=8):
    """The block step after the scan on the 2.7B shape: gated RMS norm of one layer's scan
    output (4096 tokens x 5120 channels, bf16, one norm group).  `launches` calls cycle over
    `buffers` distinct (y, z, out) sets (1 GB in all, far above L2), captured in one graph;
    reported per launch against the measured copy bandwidth."""
    T, C = PF["B"] * PF["L"], PF["H"] * PF["P"]
    bf = torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(PF["seed"] + 77)
    sets = [dict(y=torch.randn((T, C), generator=g, device=device).to(bf),
                 z=torch.randn((T, C), generator=g, device=device).to(bf),
                 out=torch.empty((T, C), device=device, dtype=bf)) for _ in range(buffers)]
    w = torch.rand((C,), generator=g, device=device) + 0.5
    stream = torch.cuda.Stream(device=device)

    def run():
        for i in range(launches):
            st = sets[i % buffers]
            ssd.ssd_gated_rmsnorm_fwd(st["y"], st["z"], w, n_groups=1, eps=1e-5, out=st["out"])

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    ms = time_graph(torch, graph, stream, reps=5)
    del graph, sets
    per_launch_s = ms / launches / 1e3
    nbytes = 3 * T * C * 2 + C * 4
    return {"kernel": "gated_rmsnorm", "workload": f"{T} tokens x {C} channels, bf16, 1 norm group",
            "avg_us": per_launch_s * 1e6, "algorithmic_bytes": nbytes, "gbs": nbytes / per_launch_s / 1e9,
            "frac": nbytes / per_launch_s / 1e9 / peaks["hbm_gbs"], "launches_timed": launches}


def bench_block_conv(torch, ssd, device, peaks, launches=64, buffers=8):
    """The block step before the scan on the 2.7B shape: causal depthwise conv1d + SiLU of
    one layer's raw xBC (4096 tokens x 5376 channels, K = 4, bf16) and the conv cache it
    leaves.  `launches` calls cycle over `buffers` distinct input/output sets (700 MB in all,
    far above L2), captured in one graph; reported per launch against the measured copy
    bandwidth."""
    B, L, H, P, G, N, K = PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], DEC["K"]
    Cc = H * P + 2 * G * N
    bf = torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(PF["seed"] + 78)
    sets = [dict(x=torch.randn((B, L, Cc), generator=g, device=device).to(bf),
                 out=torch.empty((B, L, Cc), device=device, dtype=bf),
                 cs=torch.empty((B, Cc, K - 1), device=device, dtype=bf)) for _ in range(buffers)]
    w = ((torch.rand((Cc, K), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf)
    bias = ((torch.rand((Cc,), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf)
    stream = torch.cuda.Stream(device=device)

    def run():
        for i in range(launches):
            st = sets[i % buffers]
            ssd.ssd_causal_conv1d_fwd(st["x"], w, bias, out=st["out"], conv_state_out=st["cs"])

    with torch.cuda.stream(stream):
        run()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        run()
    ms = time_graph(torch, graph, stream, reps=5)
    del graph, sets
    per_launch_s = ms / launches / 1e3
    nbytes = 2 * B * L * Cc * 2 + B * Cc * (K - 1) * 2 + Cc * (K + 1) * 2
    return {"kernel": "causal_conv1d", "workload": f"B={B}, L={L}, {Cc} channels, K={K}, bf16",
            "avg_us": per_launch_s * 1e6, "algorithmic_bytes": nbytes, "gbs": nbytes / per_launch_s / 1e9,
            "frac": nbytes / per_launch_s / 1e9 / peaks["hbm_gbs"], "launches_timed": launches}


def bench_block_conv_prefill(torch, ssd, device, peaks, launches=16, buffers=8):
    """The conv before the scan and the prefill in one call (ssd_conv_chunk_scan_fwd) on the 2.7B
    layer -- raw xBC [1, 4096, 5376], K = 4 -- against the same work as separate calls: the conv
    kernel, torch copies splitting its output into contiguous x, B and C, then the prefill.
    `launches` layers cycle over `buffers` input sets (≈ 0.9 GB each way, above L2), each variant
    captured in one graph; per-layer times.  Algorithmic bytes of the one-call path: xBC and dt
    read, y written, the conv cache and h_final written."""
    B, L, H, P, G, N, K = PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], DEC["K"]
    Cc = H * P + 2 * G * N
    bf = torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(PF["seed"] + 79)
    scale = torch.ones(Cc, device=device)
    scale[H * P:] = 1.0 / math.sqrt(N)
    sets = [dict(xbc=(torch.randn((B, L, Cc), generator=g, device=device) * scale).to(bf),
                 dt=(torch.randn((B, L, H), generator=g, device=device) - 2.0).to(bf),
                 y=torch.empty((B, L, H, P), device=device, dtype=bf),
                 hf=torch.empty((B, H, P, N), device=device, dtype=torch.float32),
                 cs=torch.empty((B, Cc, K - 1), device=device, dtype=bf)) for _ in range(buffers)]
    w = ((torch.rand((Cc, K), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf)
    bias = ((torch.rand((Cc,), generator=g, device=device) * 2 - 1) / math.sqrt(K)).to(bf)
    A_log = torch.log(torch.rand((H,), generator=g, device=device) * 15.0 + 1.0)
    D = torch.randn((H,), generator=g, device=device)
    ws1 = torch.empty(ssd.ssd_conv_chunk_scan_workspace_size(B, L, H, P, G, N, K, PF["chunk"], bf),
                      device=device, dtype=torch.uint8)
    ws2 = torch.empty(ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, PF["chunk"], bf), device=device,
                      dtype=torch.uint8)
    u = torch.empty((B, L, Cc), device=device, dtype=bf)
    xs, Bs, Cs = (torch.empty((B, L, H, P), device=device, dtype=bf), torch.empty((B, L, G, N), device=device, dtype=bf),
                  torch.empty((B, L, G, N), device=device, dtype=bf))
    stream = torch.cuda.Stream(device=device)

    def one_call():
        for i in range(launches):
            st = sets[i % buffers]
            ssd.ssd_conv_chunk_scan_fwd(st["xbc"], w, bias, st["dt"], A_log, H, P, G, N, D=D, chunk=PF["chunk"],
                                        dt_min=1e-3, dt_max=0.1, y=st["y"], h_final=st["hf"], conv_state_out=st["cs"],
                                        workspace=ws1)

    def separate():
        for i in range(launches):
            st = sets[i % buffers]
            ssd.ssd_causal_conv1d_fwd(st["xbc"], w, bias, out=u, conv_state_out=st["cs"])
            xs.copy_(u[..., :H * P].view(B, L, H, P))
            Bs.copy_(u[..., H * P:H * P + G * N].view(B, L, G, N))
            Cs.copy_(u[..., H * P + G * N:].view(B, L, G, N))
            ssd.ssd_chunk_scan_fwd(xs, st["dt"], A_log, Bs, Cs, D=D, chunk=PF["chunk"], dt_min=1e-3, dt_max=0.1,
                                   y=st["y"], h_final=st["hf"], workspace=ws2)

    res = {}
    for name, fn in (("one_call", one_call), ("separate", separate)):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            fn()
        res[name] = time_graph(torch, graph, stream, reps=5) / launches * 1e3  # us per layer
        del graph
    del sets
    nbytes = B * L * Cc * 2 + B * L * H * 2 + B * L * H * P * 2 + B * Cc * (K - 1) * 2 + B * H * P * N * 4
    return {"kernel": "ssd_conv_chunk_scan_fwd",
            "workload": f"B={B}, L={L}, {Cc} channels, K={K}, H={H}, P={P}, N={N}, bf16, one layer per launch",
            "one_call_us": res["one_call"], "separate_us": res["separate"],
            "speedup": res["separate"] / res["one_call"], "algorithmic_bytes": nbytes,
            "gbs": nbytes / (res["one_call"] * 1e-6) / 1e9,
            "frac": nbytes / (res["one_call"] * 1e-6) / 1e9 / peaks["hbm_gbs"],
            "separate_note": "conv kernel, three torch copies splitting its output into x, B, C, then the prefill"}


def bench_varlen(torch, ssd, device, reps=5):
    """A packed varlen batch on the 2.7B layer shape (H = 80, P = 64, N = 128, bf16): the 64
    sequences of 64 .. 4096 tokens of ssd_synth.varlen_lengths, each with its own h0, through
    ssd_chunk_scan_varlen_fwd (one pass over all sequences' blocks), against the same work as
    one ssd_chunk_scan_fwd call per sequence.  Each is captured in one graph and timed over
    `reps` replays; the packed batch (0.5 GB of x in, 0.5 GB of y out) is larger than L2."""
    import ssd_synth as S
    H, P, G, N = PF["H"], PF["P"], PF["G"], PF["N"]
    lengths = S.varlen_lengths()
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + n)
    T, n_seq = cu[-1], len(lengths)
    bf = torch.bfloat16
    g = torch.Generator(device=device)
    g.manual_seed(PF["seed"] + 83)
    x = torch.randn((T, H, P), generator=g, device=device).to(bf)
    dt = (torch.randn((T, H), generator=g, device=device) - 2.0).to(bf)
    Bm = (torch.randn((T, G, N), generator=g, device=device) / math.sqrt(N)).to(bf)
    Cm = (torch.randn((T, G, N), generator=g, device=device) / math.sqrt(N)).to(bf)
    A_log = torch.log(torch.rand((H,), generator=g, device=device) * 15.0 + 1.0)
    D = torch.randn((H,), generator=g, device=device)
    h0 = torch.randn((n_seq, H, P, N), generator=g, device=device) * math.sqrt(0.1)
    y = torch.empty_like(x)
    hf = torch.empty_like(h0)
    ws1 = torch.empty(ssd.ssd_chunk_scan_varlen_workspace_size(cu, H, P, G, N, PF["chunk"], bf), device=device,
                      dtype=torch.uint8)
    ws2 = torch.empty(ssd.ssd_chunk_scan_workspace_size(1, max(lengths), H, P, G, N, PF["chunk"], bf),
                      device=device, dtype=torch.uint8)
    kw = dict(D=D, chunk=PF["chunk"], dt_min=1e-3, dt_max=0.1)
    stream = torch.cuda.Stream(device=device)
    from mamba_ssd_b200 import _lib
    lib = _lib.lib()

    def one_pass():
        ssd.ssd_chunk_scan_varlen_fwd(x, dt, A_log, Bm, Cm, cu, h0=h0, y=y, h_final=hf, workspace=ws1, **kw)

    def per_sequence():
        for i in range(n_seq):
            a, b = cu[i], cu[i + 1]
            ssd.ssd_chunk_scan_fwd(x[None, a:b], dt[None, a:b], A_log, Bm[None, a:b], Cm[None, a:b], h0=h0[i:i + 1],
                                   y=y[None, a:b], h_final=hf[i:i + 1], workspace=ws2, **kw)

    res = {}
    for name, fn in (("one_pass", one_pass), ("per_sequence", per_sequence)):
        with torch.cuda.stream(stream):
            fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        n0 = lib.ssd_kernel_launch_count()
        with torch.cuda.graph(graph, stream=stream):
            fn()
        launches = lib.ssd_kernel_launch_count() - n0
        ms = time_graph(torch, graph, stream, reps)
        res[name] = {"ms": ms, "tokens_per_s": T / (ms / 1e3), "launches": launches}
        del graph
    del x, dt, Bm, Cm, y
    return {"workload": f"{n_seq} sequences of {min(lengths)}..{max(lengths)} tokens (log-uniform), {T} tokens, "
                        f"H={H}, P={P}, N={N}, bf16, h0 per sequence",
            "tokens": T, "sequences": n_seq, **res,
            "speedup": res["per_sequence"]["ms"] / res["one_pass"]["ms"],
            "per_sequence_note": "one ssd_chunk_scan_fwd call (three launches) per sequence, in one graph"}


def time_graph(torch, graph, stream, reps):
    """Median CUDA-event time of `reps` replays of a captured graph, after one warm-up."""
    graph.replay()
    torch.cuda.synchronize()
    times = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(stream):
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize()
        times.append(a.elapsed_time(b))
    return sorted(times)[len(times) // 2]


def bench_e2e(args, torch, ssd, device, rank, world, steps):
    """Prefill tokens/s through the public API with host buffers: every step copies each
    layer's inputs (x, dt, B, C) from pinned host memory to the device and reads y back.

    The copies and the prefill of different layers are pipelined the way a caller of the
    stream-ordered API would: host-to-device copies on one stream, the prefill calls on a
    second, device-to-host copies on a third, over three device buffer sets, ordered by
    events.  The two copy directions and the kernels then run at the same time; the step
    time is bounded by the slower PCIe direction.  Every rank runs its own replica; the value
    is the tokens of all ranks over the slowest rank's time."""
    B, L, H, P, G, N, Q = PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], PF["chunk"]
    n_layers = PF["layers"]
    nbuf = 3
    slots = make_prefill_layers(torch, device, nbuf, 0)  # device buffers (and the layer weights)
    host = []
    for layer in range(n_layers):
        g = torch.Generator()
        g.manual_seed(PF["seed"] * 1000 + layer)
        bf = torch.bfloat16
        host.append(dict(
            x=torch.randn((B, L, H, P), generator=g).to(bf).pin_memory(),
            dt=(torch.randn((B, L, H), generator=g) - 2.0).to(bf).pin_memory(),
            Bm=(torch.randn((B, L, G, N), generator=g) / math.sqrt(N)).to(bf).pin_memory(),
            Cm=(torch.randn((B, L, G, N), generator=g) / math.sqrt(N)).to(bf).pin_memory(),
            y=torch.empty((B, L, H, P), dtype=bf).pin_memory()))
    ws = torch.empty(ssd.ssd_chunk_scan_workspace_size(B, L, H, P, G, N, Q, torch.bfloat16),
                     device=device, dtype=torch.uint8)
    h2d = sum(h[k].numel() * h[k].element_size() for h in host for k in ("x", "dt", "Bm", "Cm"))
    d2h = sum(h["y"].numel() * h["y"].element_size() for h in host)
    s_up, s_run, s_down = (torch.cuda.Stream(device=device) for _ in range(3))
    ev_up = [torch.cuda.Event() for _ in range(nbuf)]
    ev_run = [torch.cuda.Event() for _ in range(nbuf)]
    ev_down = [None] * nbuf  # the last read of each slot's y, once there is one

    def step():
        for layer, h in enumerate(host):
            i = layer % nbuf
            d = slots[i]
            with torch.cuda.stream(s_up):
                if ev_down[i] is not None:  # slot i's previous layer is computed and read back
                    s_up.wait_event(ev_down[i])
                for k in ("x", "dt", "Bm", "Cm"):
                    d[k].copy_(h[k], non_blocking=True)
                ev_up[i].record(s_up)
            with torch.cuda.stream(s_run):
                s_run.wait_event(ev_up[i])
                prefill_call(ssd, d, ws, stream=s_run)
                ev_run[i].record(s_run)
            with torch.cuda.stream(s_down):
                s_down.wait_event(ev_run[i])
                h["y"].copy_(d["y"], non_blocking=True)
                if ev_down[i] is None:
                    ev_down[i] = torch.cuda.Event()
                ev_down[i].record(s_down)

    step()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    start.record(s_up)
    for _ in range(steps):
        step()
    end.record(s_down)  # the last read-back is the last operation of the timed steps
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms = max_over_ranks(start.elapsed_time(end) / steps, world, device)
    tokens = sum_over_ranks(B * L, world, device)
    return {"value": tokens / (ms / 1e3), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "ms_per_step": ms, "steps": steps,
            "h2d_gbs": h2d / (ms / 1e3) / 1e9, "d2h_gbs": d2h / (ms / 1e3) / 1e9,
            "note": ("per layer H2D of x, dt, B, C from pinned memory, prefill, D2H of y; "
                     "copies up, prefill and copies down on three streams over three buffer sets")}


def decode_vs_recompute(prefill_ms, decode, by_context=None):
    """The pages' headline comparison on this GPU: one cached decode step of the 64-layer
    2.7B-shaped stack at batch 1 against recomputing the 4096-token prefix (the same stack's
    prefill step, one batch row of 4096 tokens).  Both come from this run's measurements."""
    b1 = decode.get("b1")
    if not b1:
        return None
    step_ms = 1e3 / b1["steps_per_s"]
    return {"context": PF["L"], "recompute_prefix_ms": prefill_ms, "cached_decode_step_ms": step_ms,
            "speedup": prefill_ms / step_ms, "by_context": by_context}


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["mine", "reference"], default="mine")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-decode", action="store_true")
    ap.add_argument("--layers", type=int, default=PF["layers"],
                    help="prefill stack depth (64 = the workload; smaller only for profiling)")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")

    PF["layers"] = args.layers
    if args.impl == "reference":
        run_reference(args)
        return

    import torch
    rank, world, local_rank = dist_env()
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)
    import mamba_ssd_b200 as ssd
    from mamba_ssd_b200 import _lib
    lib = _lib.lib()
    peaks = load_peaks()

    pf = bench_prefill(args, torch, ssd, device, rank, world)
    B, L, H, P, G, N, Q = PF["B"], PF["L"], PF["H"], PF["P"], PF["G"], PF["N"], PF["chunk"]
    ms_step = pf["ms_total"] / args.steps
    tokens_all = sum_over_ranks(B * L * args.steps, world, device)
    value = tokens_all / (pf["ms_total"] / 1e3)
    flops_layer = prefill_flops(B, L, H, P, G, N, Q)
    tflops = flops_layer * PF["layers"] * world / (ms_step / 1e3) / 1e12

    # roofline of the dominant kernel (largest summed device time), in algorithmic work: its
    # share of the method-level flops (the tensor-core kernels' target is a fraction of the
    # bf16 tensor peak), else the method-level bytes it is responsible for against HBM
    kt = pf["kernel_times"]
    dom = max(kt, key=lambda n: kt[n][0])
    dms, dcnt = kt[dom]
    avg_s = dms / max(dcnt, 1) / 1e3
    method_bytes = prefill_bytes(B, L, H, P, G, N)
    traffic = measured_traffic(dom)
    if dom in KERNEL_METHOD_FLOPS:
        fl = KERNEL_METHOD_FLOPS[dom](B, L, H, P, G, N, Q)
        ach = fl / avg_s / 1e12
        roof = {"kernel": dom, "bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"], "traffic": traffic,
                "algorithmic_flops": fl, "peak_source": f"{peaks['source']} bf16 matmul (burst)"}
    else:
        ach = method_bytes / avg_s / 1e9
        roof = {"kernel": dom, "bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": ach / peaks["hbm_gbs"], "traffic": traffic, "algorithmic_bytes": method_bytes,
                "peak_source": f"{peaks['source']} copy"}
    roof.update(avg_launch_us=avg_s * 1e6, launches_timed=dcnt)
    # the whole layer against both roofs, and the DRAM bytes the kernels really move per layer
    # (the ncu capture) over the method's own bytes
    layer_s = ms_step / 1e3 / PF["layers"]
    roof["method_frac_hbm"] = method_bytes / layer_s / 1e9 / peaks["hbm_gbs"]
    roof["method_tensor_frac"] = flops_layer / layer_s / 1e12 / peaks["bf16_tflops"]
    roof["method_bytes_per_layer"] = method_bytes
    tr = [measured_traffic(n) for n in kt]
    roof["traffic_ratio"] = sum(tr) / method_bytes if tr and all(t is not None for t in tr) else None
    kernels = {}
    for n, v in kt.items():
        avg = v[0] / max(v[1], 1) / 1e3
        kernels[n] = {"total_ms": v[0], "launches": v[1], "avg_us": avg * 1e6, "traffic": measured_traffic(n)}
        if n in KERNEL_BYTES:
            mb = KERNEL_BYTES[n](B, L, H, P, G, N)
            kernels[n].update(moved_bytes=mb, moved_gbs=mb / avg / 1e9, moved_frac=mb / avg / 1e9 / peaks["hbm_gbs"])
        if n in KERNEL_METHOD_FLOPS:
            fl = KERNEL_METHOD_FLOPS[n](B, L, H, P, G, N, Q)
            kernels[n].update(method_flops=fl, tflops=fl / avg / 1e12,
                              tensor_frac=fl / avg / 1e12 / peaks["bf16_tflops"])

    decode, by_context = {}, None
    if not args.no_decode:
        for bsz in (1, 16):
            r = bench_decode(args, torch, ssd, device, rank, bsz, DEC["steps"])
            r["gbs_frac"] = r["gbs"] / peaks["hbm_gbs"]
            if r.get("kernel_gbs"):
                r["kernel_gbs_frac"] = r["kernel_gbs"] / peaks["hbm_gbs"]
            decode[f"b{bsz}"] = r
            torch.cuda.empty_cache()
        by_context = bench_context_sweep(torch, ssd, device, rank)
        torch.cuda.empty_cache()
    block_steps = {"causal_conv1d": bench_block_conv(torch, ssd, device, peaks),
                   "gated_rmsnorm": bench_block_norm(torch, ssd, device, peaks),
                   "conv_prefill": bench_block_conv_prefill(torch, ssd, device, peaks)}
    torch.cuda.empty_cache()
    varlen = bench_varlen(torch, ssd, device)
    torch.cuda.empty_cache()

    e2e = None
    if not args.no_e2e:  # every rank, the same collective steps in the same order
        e2e = bench_e2e(args, torch, ssd, device, rank, world, steps=max(1, min(args.steps, 3)))
        torch.cuda.empty_cache()

    cpu = None
    if not args.no_cpu_baseline and rank == 0 and world == 1:
        cpu = cpu_baseline()

    if world > 1:
        torch.distributed.barrier()
    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic", "config": workload_config(),
            # method-level count at the caller's chunk (256); the tensor-core path blocks the
            # sequence in 128 tokens, which does fewer flops: both are reported
            "tflops": tflops, "tflops_frac": tflops * 1e12 / (peaks["bf16_tflops"] * 1e12) / world,
            "flops_per_layer_dense": flops_layer,
            "tflops_executed_block128": prefill_flops(B, L, H, P, G, N, TC_BLOCK) * PF["layers"] * world
                                        / (ms_step / 1e3) / 1e12,
            "flops_per_layer_causal": prefill_flops_causal(B, L, H, P, G, N, Q),
            "roofline": roof, "kernels": kernels, "decode": decode, "e2e": e2e,
            "decode_vs_recompute": decode_vs_recompute(ms_step, decode, by_context),
            "block_steps": block_steps, "varlen": varlen,
            "cpu_baseline": cpu, "clocks": pf["clocks"],
            "gpu_launches": pf["launches_per_step"] * args.steps,
            "peaks": peaks,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
