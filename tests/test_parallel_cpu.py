"""Host logic of the multi-GPU prefill (mamba_ssd_b200/parallel.py) on CPU processes over gloo,
world size 2 and 3, with the per-rank steps given by the fp64 oracle.

Context parallelism: each rank passes its consecutive segment of one sequence; the ranks
exchange (segment state from zero, segment decay) by all-gather, combine them into each rank's
carry-in, and run their segment from it.  The segments' y, concatenated in rank order, and the
state after the whole sequence (on every rank) must equal oracle.ssd_scan_sequential over the
whole sequence.  Head sharding: each rank's heads and groups, run on their own, must give the
full result's slice; head_range is checked on its own as well.

The CUDA kernels of the same steps are checked on the GPU in tests/test_gpu_context.py.
"""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


class OracleOps:
    """The per-rank steps in fp64 on the host (torch float64 CPU tensors in and out)."""

    @staticmethod
    def segment_state(x, dt, A_log, Bm, Cm, chunk, dt_bias, dt_min, dt_max):
        import oracle
        _, h = oracle.ssd_scan_sequential(x.numpy(), dt.numpy(), A_log.numpy(), Bm.numpy(), Cm.numpy(), None,
                                          None if dt_bias is None else dt_bias.numpy(), dt_min, dt_max, None)
        return torch.from_numpy(h)

    @staticmethod
    def segment_decay(dt, A_log, dt_bias, dt_min, dt_max):
        import oracle
        d, dA = oracle.discretise(dt.numpy(), A_log.numpy(), None if dt_bias is None else dt_bias.numpy(), dt_min,
                                  dt_max)
        return torch.from_numpy(dA.sum(axis=1) / math.log(2.0))  # [B, H], log2 of the decay

    @staticmethod
    def combine(states, log2_decays, r, h0):
        h = torch.zeros_like(states[0]) if h0 is None else h0.clone()
        for j in range(r):
            h = torch.exp2(log2_decays[j])[:, :, None, None] * h + states[j]
        return h

    @staticmethod
    def prefill(x, dt, A_log, Bm, Cm, D, chunk, h0, dt_bias, dt_min, dt_max):
        import oracle
        y, _ = oracle.ssd_scan_sequential(x.numpy(), dt.numpy(), A_log.numpy(), Bm.numpy(), Cm.numpy(),
                                          None if D is None else D.numpy(),
                                          None if dt_bias is None else dt_bias.numpy(), dt_min, dt_max,
                                          None if h0 is None else h0.numpy())
        return torch.from_numpy(y)


def _inputs(seed):
    import sys
    sys.path.insert(0, ROOT)
    import ssd_synth as S
    inp = S.prefill_inputs(2, 301, 4, 64, 2, 16, dtype="f32", seed=seed, h0=True, dt_bias_zero=False)
    return {k: (torch.from_numpy(np.ascontiguousarray(v[1])) if isinstance(v, tuple) else v) for k, v in inp.items()}


def _worker(rank, world, port, seed, q):
    import sys
    sys.path.insert(0, ROOT)
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from mamba_ssd_b200 import parallel
        f = _inputs(seed)
        L = f["x"].shape[1]
        cuts = [L * i // world for i in range(world + 1)]  # uneven segments when L % world
        a, b = cuts[rank], cuts[rank + 1]
        seg = {k: f[k][:, a:b].contiguous() for k in ("x", "dt", "Bm", "Cm")}
        y, h = parallel.context_parallel_prefill(seg["x"], seg["dt"], f["A_log"], seg["Bm"], seg["Cm"], D=f["D"],
                                                 chunk=64, h0=f["h0"], dt_bias=f["dt_bias"], dt_min=f["dt_min"],
                                                 dt_max=f["dt_max"], ops=OracleOps)
        q.put((rank, y.numpy(), h.numpy()))
    finally:
        dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("world", [2, 3])
def test_context_parallel_matches_whole_sequence(world):
    import oracle
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, 7, q)) for r in range(world)]
    for p in procs:
        p.start()
    got = dict()
    for _ in range(world):
        r, y, h = q.get(timeout=300)
        got[r] = (y, h)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    f = _inputs(7)
    y_ref, h_ref = oracle.ssd_scan_sequential(f["x"].numpy(), f["dt"].numpy(), f["A_log"].numpy(), f["Bm"].numpy(),
                                              f["Cm"].numpy(), f["D"].numpy(), f["dt_bias"].numpy(), f["dt_min"],
                                              f["dt_max"], f["h0"].numpy())
    y = np.concatenate([got[r][0] for r in range(world)], axis=1)
    np.testing.assert_allclose(y, y_ref, rtol=1e-10, atol=1e-12)
    for r in range(world):  # every rank holds the state after the whole sequence
        np.testing.assert_allclose(got[r][1], h_ref, rtol=1e-10, atol=1e-12)


def test_head_range():
    import sys
    sys.path.insert(0, ROOT)
    from mamba_ssd_b200.parallel import head_range
    assert head_range(80, 1, 4, 2) == (40, 60, 0, 1)
    assert head_range(8, 4, 2, 1) == (4, 8, 2, 4)       # two whole groups per rank
    assert head_range(8, 2, 4, 3) == (6, 8, 1, 2)       # inside one group
    with pytest.raises(ValueError):
        head_range(6, 1, 4, 0)
    assert head_range(12, 4, 4, 1) == (3, 6, 1, 2)      # exactly one group per rank
    with pytest.raises(ValueError):
        head_range(12, 3, 2, 0)                          # 6 heads per rank, groups of 4
    # every rank's heads tile [0, H), and its groups hold exactly its heads' groups
    for H, G, W in [(80, 1, 8), (64, 8, 4), (64, 8, 16), (24, 2, 4)]:
        seen = []
        for r in range(W):
            a, b, ga, gb = head_range(H, G, W, r)
            seen.extend(range(a, b))
            assert {h // (H // G) for h in range(a, b)} == set(range(ga, gb))
        assert seen == list(range(H))


def test_head_sharding_slices_compose():
    # each rank's heads on their own (the oracle) give exactly the full result's slice: the
    # recurrences of different heads never meet
    import sys
    sys.path.insert(0, ROOT)
    import oracle
    from mamba_ssd_b200.parallel import head_range
    f = _inputs(9)
    H, G = f["x"].shape[2], f["Bm"].shape[2]
    y_ref, h_ref = oracle.ssd_scan_sequential(f["x"].numpy(), f["dt"].numpy(), f["A_log"].numpy(), f["Bm"].numpy(),
                                              f["Cm"].numpy(), f["D"].numpy(), f["dt_bias"].numpy(), f["dt_min"],
                                              f["dt_max"], f["h0"].numpy())
    for W in (2, 4):
        for r in range(W):
            a, b, ga, gb = head_range(H, G, W, r)
            y, h = oracle.ssd_scan_sequential(f["x"].numpy()[:, :, a:b], f["dt"].numpy()[:, :, a:b],
                                              f["A_log"].numpy()[a:b], f["Bm"].numpy()[:, :, ga:gb],
                                              f["Cm"].numpy()[:, :, ga:gb], f["D"].numpy()[a:b],
                                              f["dt_bias"].numpy()[a:b], f["dt_min"], f["dt_max"],
                                              f["h0"].numpy()[:, a:b])
            np.testing.assert_allclose(y, y_ref[:, :, a:b], rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(h, h_ref[:, a:b], rtol=1e-12, atol=1e-14)
