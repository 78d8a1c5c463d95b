"""Second and third forms of the SSD scan, in numpy float64, written independently of
the sequential C recurrence.  Test infrastructure only.

Sources: the paper "Compiler-First State Space Duality and Portable O(1) Autoregressive
Caching for Inference" (abstract) and the article "Mamba-2状态空间模型的编译器优先实现"
(bqwf.cn), cited as [blog §x.y]:
  §1.1: fixed-size chunks (default 256 tokens); parallel matrix products inside a chunk,
        a light sequential scan passing the state between chunks; the decay mask
        L = tril(exp(segsum(log A))).
  §1.2: the intra-chunk contraction Y = einsum('bclhn,bcshn,bhcls,bcshp->bclhp', C, B, L, X).
  §3.1: layout [batch, chunk, seq, head, dim].

``ssd_chunked`` takes those steps in that order.  The blog prints only the intra-chunk
einsum; the per-chunk state (decay-weighted B^T X "passed between chunks"), the
inter-chunk recurrence and the output correction C h_prev exp(cumsum) + D x are the
plain reading of §1.1 and are written out below.

``ssd_dense`` is the quadratic "dual" form: y = M x + D x + (carry-in of h0), with
M[t,s] = (C_t . B_s) * exp(sum_{k=s+1..t} dA_k) * dt_s for s <= t, each segment sum
added up term by term (cubic cost; tiny inputs only).
"""
from __future__ import annotations

import math

import numpy as np


def softplus(z):
    """log(1 + e^z), as the library's stable log(e^0 + e^z)."""
    return np.logaddexp(0.0, np.asarray(z, dtype=np.float64))


def discretise(dt_raw, A_log, dt_bias, dt_min, dt_max):
    """dt = clip(softplus(dt_raw + dt_bias), dt_min, dt_max); dA = dt * (-exp(A_log)).

    [blog §1.1, §4.1], with the sign of the exponent restored (A = -exp(A_log)).
    """
    dt_raw = np.asarray(dt_raw, dtype=np.float64)
    H = dt_raw.shape[-1]
    bias = np.zeros(H) if dt_bias is None else np.asarray(dt_bias, dtype=np.float64)
    dt = np.clip(softplus(dt_raw + bias), dt_min, dt_max)
    A = -np.exp(np.asarray(A_log, dtype=np.float64))
    return dt, dt * A


def _heads_from_groups(M, H):
    """[B,L,G,N] -> [B,L,H,N] with head h reading group h // (H/G)."""
    G = M.shape[2]
    return np.repeat(M, H // G, axis=2)


def ssd_chunked(x, dt_raw, A_log, Bm, Cm, D=None, dt_bias=None, dt_min=0.0,
                dt_max=float("inf"), h0=None, chunk=256):
    """Chunked SSD in float64.  Returns (y [B,L,H,P], h_final [B,H,P,N])."""
    x = np.asarray(x, dtype=np.float64)
    Bsz, L, H, P = x.shape
    N = Bm.shape[3]
    Q = int(chunk)
    nc = -(-L // Q)
    Lp = nc * Q
    # a1: discretisation; tokens past L get dt = 0 (decay 1, no input).
    dt, dA = discretise(dt_raw, A_log, dt_bias, dt_min, dt_max)
    pad = Lp - L

    def padL(a):
        if pad == 0:
            return a
        w = [(0, 0)] * a.ndim
        w[1] = (0, pad)
        return np.pad(a, w)

    dt, dA = padL(dt), padL(dA)
    X = padL(x) * dt[..., None]                                    # dt * x  [B,Lp,H,P]
    Bh = padL(_heads_from_groups(np.asarray(Bm, np.float64), H))   # [B,Lp,H,N]
    Ch = padL(_heads_from_groups(np.asarray(Cm, np.float64), H))
    # [batch, chunk, seq, head, dim] layout of §3.1
    X = X.reshape(Bsz, nc, Q, H, P)
    Bh = Bh.reshape(Bsz, nc, Q, H, N)
    Ch = Ch.reshape(Bsz, nc, Q, H, N)
    Acs = np.cumsum(dA.reshape(Bsz, nc, Q, H).transpose(0, 3, 1, 2), axis=-1)  # [b,h,c,l]

    # a2: decay mask L = tril(exp(segsum)) and the intra-chunk contraction of §1.2
    seg = Acs[..., :, None] - Acs[..., None, :]                    # [b,h,c,l,s]
    lower = np.tril(np.ones((Q, Q), dtype=bool))
    Lmask = np.where(lower, np.exp(np.where(lower, seg, 0.0)), 0.0)
    Y_diag = np.einsum("bclhn,bcshn,bhcls,bcshp->bclhp", Ch, Bh, Lmask, X, optimize=True)

    # a3: per-chunk state, the decay-weighted B^T X carried to the chunk's last token
    to_end = np.exp(Acs[..., -1:] - Acs)                           # [b,h,c,s]
    S = np.einsum("bcshn,bhcs,bcshp->bchpn", Bh, to_end, X, optimize=True)

    # a4: inter-chunk sequential pass
    h = np.zeros((Bsz, H, P, N)) if h0 is None else np.array(h0, dtype=np.float64)
    h_prev = np.empty((Bsz, nc, H, P, N))
    for c in range(nc):
        h_prev[:, c] = h
        h = np.exp(Acs[:, :, c, -1])[..., None, None] * h + S[:, c]

    # a5: output correction from the carried-in state, plus the D skip
    Y_off = np.einsum("bclhn,bchpn,bhcl->bclhp", Ch, h_prev, np.exp(Acs), optimize=True)
    y = (Y_diag + Y_off).reshape(Bsz, Lp, H, P)[:, :L]
    if D is not None:
        y = y + np.asarray(D, np.float64)[None, None, :, None] * x
    return y, h


def ssd_dense(x, dt_raw, A_log, Bm, Cm, D=None, dt_bias=None, dt_min=0.0,
              dt_max=float("inf"), h0=None):
    """Quadratic dual form, per (batch, head), every segment sum added term by term."""
    x = np.asarray(x, dtype=np.float64)
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    dt, dA = discretise(dt_raw, A_log, dt_bias, dt_min, dt_max)
    y = np.zeros_like(x)
    hf = np.zeros((Bsz, H, P, N))
    for b in range(Bsz):
        for h in range(H):
            g = h // (H // G)
            Bs = np.asarray(Bm[b, :, g], np.float64)                 # [L,N]
            Cs = np.asarray(Cm[b, :, g], np.float64)
            M = np.zeros((L, L))
            for t in range(L):
                for s in range(t + 1):
                    seg = 0.0
                    for k in range(s + 1, t + 1):
                        seg += dA[b, k, h]
                    M[t, s] = float(Cs[t] @ Bs[s]) * math.exp(seg) * dt[b, s, h]
            y[b, :, h] = M @ x[b, :, h]
            # state after the last token, same segment sums to L-1
            for s in range(L):
                seg = 0.0
                for k in range(s + 1, L):
                    seg += dA[b, k, h]
                hf[b, h] += math.exp(seg) * dt[b, s, h] * np.outer(x[b, s, h], Bs[s])
            if h0 is not None:
                h0bh = np.asarray(h0[b, h], np.float64)              # [P,N]
                run = 0.0
                for t in range(L):
                    run += dA[b, t, h]
                    y[b, t, h] += math.exp(run) * (h0bh @ Cs[t])
                hf[b, h] += math.exp(run) * h0bh
            if D is not None:
                y[b, :, h] += float(D[h]) * x[b, :, h]
    return y, hf
