"""The block step after the SSD: gated RMS normalisation of the scan output, in numpy
float64.  Test infrastructure only.

Sources: the article "Mamba-2状态空间模型的编译器优先实现" (bqwf.cn) §4.1 (numerical
safeguards: a normalisation takes its variance in float32 even when its inputs are
bf16) and §3.2 (normalisations sit next to the SSD and are fused with their neighbours).
The pages do not spell the normalisation out.  The reading taken here is the one of the
Mamba-2 block that the pages' checkpoints come from: the scan output y is gated by the
SiLU of the second input projection z, then RMS-normalised per token over groups of
consecutive channels, then scaled per channel:

    g   = y * SiLU(z)                               (SiLU(z) = z / (1 + exp(-z)))
    out = g / sqrt(mean_{channels of the group}(g^2) + eps) * w

with the token's H*P channels split into n_groups groups of equal size.
"""
from __future__ import annotations

import numpy as np


def silu(z):
    """z * sigmoid(z), with the sigmoid written as 1 / (1 + exp(-z))."""
    z = np.asarray(z, dtype=np.float64)
    return z / (1.0 + np.exp(-z))


def gated_rmsnorm(y, z, w, eps=1e-5, n_groups=1):
    """Gated RMS norm over the last axis.

    y, z : [..., C] the scan output and the gate input (any float dtype; used in fp64)
    w    : [C] per-channel scale
    eps  : added to the mean square before the square root
    n_groups : C is split into n_groups consecutive groups of C / n_groups channels; each
               group of each token is normalised on its own
    Returns float64 [..., C].
    """
    y = np.asarray(y, dtype=np.float64)
    z = np.asarray(z, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    C = y.shape[-1]
    if C % n_groups != 0:
        raise ValueError("channels must split evenly into the norm groups")
    g = y * silu(z)
    grouped = g.reshape(g.shape[:-1] + (n_groups, C // n_groups))
    ms = np.mean(grouped * grouped, axis=-1, keepdims=True)
    normed = grouped / np.sqrt(ms + eps)
    return normed.reshape(g.shape) * w
