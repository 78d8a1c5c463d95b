"""Multi-GPU prefill, one process per GPU: head sharding and context (sequence) parallelism.

Head sharding.  Every (batch, head) recurrence is independent, so a GPU that owns a contiguous
range of heads runs the prefill on those heads alone, reading the B/C groups they map to
(heads map to groups in contiguous blocks); nothing crosses GPUs inside the scan.
`head_range` computes a rank's heads and groups; `head_sharded_prefill` runs them.

Context parallelism.  The sequence is split into W consecutive segments, segment r on rank r.
The recurrence is linear in the state, so segment r maps the state it receives, h_in, to
exp(sum_{t in segment} dt_t A) h_in + S_r, with S_r the state it leaves from zero.  Per rank:
  1. S_r (the prefill with no output, from a zero state) and the segment's decay (log2);
  2. one all-gather of (S_r, decay_r) over the ranks (NCCL on GPUs);
  3. the carry-in h_in = combine(S_0 .. S_{r-1}, decays, h0), and the state after the whole
     sequence = combine(all W segments) on every rank;
  4. the prefill of the segment from h_in, which gives the segment's y.
This is the state passing between chunks of the pages' chunked scan, with whole segments as
the chunks (blog walk-through of "Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching for Inference", bqwf.cn, §1.1).  The exchange is one small all-gather
per layer (2 x B*H*P*N floats + B*H per rank), issued by torch.distributed.

Every step of the scan runs in the library's kernels (`LibraryOps`).  The functions take the
per-rank steps as an `ops` object so that the host logic (which rank computes what, in which
order, what is gathered and combined) can be tested on CPU processes with a reference
implementation of the steps.
"""
from __future__ import annotations

import math

import torch

from . import api


class LibraryOps:
    """The per-rank steps of a context-parallel prefill, as calls into the CUDA library."""

    @staticmethod
    def segment_state(x, dt, A_log, Bm, Cm, chunk, dt_bias, dt_min, dt_max):
        _, h = api.ssd_chunk_scan_fwd(x, dt, A_log, Bm, Cm, chunk=chunk, dt_bias=dt_bias, dt_min=dt_min,
                                      dt_max=dt_max, want_y=False)
        return h

    @staticmethod
    def segment_decay(dt, A_log, dt_bias, dt_min, dt_max):
        return api.ssd_segment_decay(dt, A_log, dt_bias=dt_bias, dt_min=dt_min, dt_max=dt_max)

    @staticmethod
    def combine(states, log2_decays, r, h0):
        return api.ssd_state_combine(states, log2_decays, r, h0=h0)

    @staticmethod
    def prefill(x, dt, A_log, Bm, Cm, D, chunk, h0, dt_bias, dt_min, dt_max):
        y, _ = api.ssd_chunk_scan_fwd(x, dt, A_log, Bm, Cm, D=D, chunk=chunk, h0=h0, dt_bias=dt_bias,
                                      dt_min=dt_min, dt_max=dt_max, want_h_final=False)
        return y


def segment_summary(x, dt, A_log, Bm, Cm, chunk=256, dt_bias=None, dt_min=0.0, dt_max=math.inf, ops=LibraryOps):
    """Step 1 on one rank: (S_r [B, H, P, N], log2 decay_r [B, H]) of its segment."""
    S = ops.segment_state(x, dt, A_log, Bm, Cm, chunk, dt_bias, dt_min, dt_max)
    ld = ops.segment_decay(dt, A_log, dt_bias, dt_min, dt_max)
    return S, ld


def segment_output(r, states, log2_decays, x, dt, A_log, Bm, Cm, D=None, chunk=256, h0=None, dt_bias=None,
                   dt_min=0.0, dt_max=math.inf, ops=LibraryOps):
    """Steps 3 and 4 on rank r, given every segment's summary stacked in rank order
    (states [W, B, H, P, N], log2_decays [W, B, H]): the segment's y, and the state after the
    whole sequence."""
    W = states.shape[0]
    h_in = ops.combine(states, log2_decays, r, h0)
    y = ops.prefill(x, dt, A_log, Bm, Cm, D, chunk, h_in, dt_bias, dt_min, dt_max)
    h_final = ops.combine(states, log2_decays, W, h0)
    return y, h_final


def context_parallel_prefill(x, dt, A_log, Bm, Cm, D=None, chunk=256, h0=None, dt_bias=None, dt_min=0.0,
                             dt_max=math.inf, group=None, ops=LibraryOps):
    """The prefill of a sequence split over the ranks of `group`: this rank passes its segment
    (x [B, Ls, H, P], dt [B, Ls, H], Bm/Cm [B, Ls, G, N], consecutive segments on consecutive
    ranks) and the sequence's h0 (the same on every rank, or None).  Returns (y of the segment,
    the state after the whole sequence)."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    r = dist.get_rank(group)
    S, ld = segment_summary(x, dt, A_log, Bm, Cm, chunk, dt_bias, dt_min, dt_max, ops)
    all_S = [torch.empty_like(S) for _ in range(W)]
    all_ld = [torch.empty_like(ld) for _ in range(W)]
    dist.all_gather(all_S, S.contiguous(), group=group)
    dist.all_gather(all_ld, ld.contiguous(), group=group)
    return segment_output(r, torch.stack(all_S), torch.stack(all_ld), x, dt, A_log, Bm, Cm, D, chunk, h0, dt_bias,
                          dt_min, dt_max, ops)


def head_range(H, G, world, rank):
    """Heads [h0, h1) and groups [g0, g1) of `rank` when H heads (G groups, contiguous blocks of
    H / G heads) are split evenly over `world` ranks.  Each rank's heads must cover whole groups,
    or lie inside one group."""
    if H % world:
        raise ValueError(f"{H} heads do not split evenly over {world} ranks")
    hpr, hpg = H // world, H // G
    if hpr % hpg and hpg % hpr:
        raise ValueError(f"{hpr} heads per rank neither cover whole groups of {hpg} nor lie inside one")
    h0, h1 = rank * hpr, (rank + 1) * hpr
    return h0, h1, h0 // hpg, (h1 - 1) // hpg + 1


def head_sharded_prefill(x, dt, A_log, Bm, Cm, D=None, chunk=256, h0=None, dt_bias=None, dt_min=0.0,
                         dt_max=math.inf, rank=0, world=1):
    """The prefill of this rank's heads: the full-width inputs are sliced to the rank's heads and
    groups (in a model the projections would produce the rank's heads directly).  No collective.
    Returns (y [B, L, H/world, P], h_final [B, H/world, P, N])."""
    H, G = x.shape[2], Bm.shape[2]
    a, b, ga, gb = head_range(H, G, world, rank)
    sl = lambda t, lo, hi, dim: None if t is None else t.narrow(dim, lo, hi - lo).contiguous()
    return api.ssd_chunk_scan_fwd(sl(x, a, b, 2), sl(dt, a, b, 2), sl(A_log, a, b, 0), sl(Bm, ga, gb, 2),
                                  sl(Cm, ga, gb, 2), D=sl(D, a, b, 0), chunk=chunk, h0=sl(h0, a, b, 1),
                                  dt_bias=sl(dt_bias, a, b, 0), dt_min=dt_min, dt_max=dt_max)
