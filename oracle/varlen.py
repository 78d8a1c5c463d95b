"""Varlen batches for the fp64 oracle: several sequences of different lengths packed into one
token stream, each scanned on its own.  Test infrastructure only.

Source: the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §1.1: the state is passed
along one sequence; nothing crosses from one sequence to the next.  Packing is the usual
cumulative-length layout: sequence i owns tokens cu_seqlens[i] .. cu_seqlens[i+1]-1 of the
packed [T_total, ...] arrays, and has its own initial and final state.
"""
from __future__ import annotations

import numpy as np

from .native import ssd_scan_sequential


def ssd_scan_varlen(x, dt_raw, A_log, Bm, Cm, cu_seqlens, D=None, dt_bias=None, dt_min=0.0,
                    dt_max=float("inf"), h0=None):
    """x [T, H, P], dt_raw [T, H], Bm/Cm [T, G, N] packed; cu_seqlens [n+1] with
    cu_seqlens[0] = 0 and non-decreasing; h0 [n, H, P, N] or None.
    Returns (y [T, H, P], h_final [n, H, P, N]), each sequence by the sequential recurrence."""
    x = np.asarray(x, dtype=np.float64)
    cu = [int(v) for v in cu_seqlens]
    n = len(cu) - 1
    if n < 0 or cu[0] != 0 or any(b < a for a, b in zip(cu, cu[1:])) or cu[-1] != x.shape[0]:
        raise ValueError("cu_seqlens must start at 0, never decrease and end at the token count")
    T, H, P = x.shape
    N = np.asarray(Bm).shape[-1]
    y = np.zeros_like(x)
    hf = np.zeros((n, H, P, N))
    for i in range(n):
        a, b = cu[i], cu[i + 1]
        h0_i = None if h0 is None else np.asarray(h0, dtype=np.float64)[i:i + 1]
        yi, hi = ssd_scan_sequential(x[None, a:b], np.asarray(dt_raw)[None, a:b], A_log,
                                     np.asarray(Bm)[None, a:b], np.asarray(Cm)[None, a:b], D, dt_bias,
                                     dt_min, dt_max, h0_i)
        y[a:b] = yi[0]
        hf[i] = hi[0]
    return y, hf
