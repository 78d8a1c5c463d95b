"""Seeded synthetic inputs for the Mamba-2 SSD scan (prefill and cached decode).

This module holds no arithmetic of the method itself: it draws random tensors with
the value distributions of the five benchmark workloads and rounds them to the
storage type of the interface (bf16 by round-to-nearest-even on the bit pattern,
or fp32).  Both the fp64 oracle and the CUDA path are fed from here, so they see
exactly the same input bits; neither side imports the other.

Distributions (the workload descriptions; N(mu, var) is mean and *variance*):
  x ~ N(0, 1); B, C ~ N(0, 1/N); raw dt ~ N(0, 1) - 2 (softplus and the [1e-3, 0.1]
  clip happen inside the method, dt_bias = 0); A_log = log U(1, 16); D ~ N(0, 1);
  h0 = 0, or N(0, 0.1) for the batched workload that exercises state carry-in.
Decode (2.7B-shaped): raw xBC with the x channels N(0, 1) and the B/C channels
N(0, 1/N); depthwise conv weight and bias ~ U(-1/sqrt(K), 1/sqrt(K)).
Gated norm after the scan: y ~ N(0, 1) (the scale of the scan output), gate input
z ~ N(0, 1), per-channel weight w ~ U(0.5, 1.5) in fp32.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

__all__ = [
    "PrefillShape", "DecodeShape", "PREFILL_WORKLOADS", "DECODE_WORKLOAD",
    "bf16_bits", "bf16_bits_to_f64", "to_storage", "prefill_inputs",
    "decode_params", "decode_token_inputs", "raw_xbc_sequence", "layer_seed", "norm_inputs",
]


@dataclasses.dataclass(frozen=True)
class PrefillShape:
    name: str
    B: int
    L: int
    H: int
    P: int
    G: int
    N: int
    chunk: int
    dtype: str          # "f32" or "bf16": storage type of x, dt, B, C, y
    h0: bool            # nonzero initial state
    seed: int
    layers: int = 1


@dataclasses.dataclass(frozen=True)
class DecodeShape:
    name: str
    B: int
    H: int
    P: int
    G: int
    N: int
    K: int
    layers: int
    steps: int
    prefix_len: int
    dtype: str
    seed: int

    @property
    def Cc(self) -> int:
        return self.H * self.P + 2 * self.G * self.N


# The five workloads, in order (tiny fp32, 130M-, 2.7B-, batched 1.3B-shaped prefill,
# 2.7B-shaped cached decode).  Seed = workload index.
PREFILL_WORKLOADS = {
    "tiny_f32": PrefillShape("tiny_f32", 1, 512, 4, 64, 1, 16, 256, "f32", False, 0),
    "m130m": PrefillShape("m130m", 1, 4096, 24, 64, 1, 128, 256, "bf16", False, 1),
    "m2p7b": PrefillShape("m2p7b", 1, 4096, 80, 64, 1, 128, 256, "bf16", False, 2, layers=64),
    "m1p3b_b8": PrefillShape("m1p3b_b8", 8, 2048, 64, 64, 1, 128, 256, "bf16", True, 3),
}
DECODE_WORKLOAD = DecodeShape("m2p7b_decode", 1, 80, 64, 1, 128, 4, 64, 64, 4096, "bf16", 4)


def layer_seed(seed: int, layer: int) -> int:
    """Each layer of a stack draws from its own stream: seed * 1000 + layer."""
    return seed * 1000 + layer


# ----------------------------------------------------------------------------------
# storage rounding
# ----------------------------------------------------------------------------------
def bf16_bits(a) -> np.ndarray:
    """Round float values to bf16 (round to nearest, ties to even); return uint16 bits."""
    f = np.ascontiguousarray(np.asarray(a, dtype=np.float32))
    u = f.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    out = ((u + rounding) >> 16).astype(np.uint16)
    nan = np.isnan(f)
    if nan.any():
        out[nan] = 0x7FC0
    return out


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    u = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16
    return u.view(np.float32).astype(np.float64)


def to_storage(a, dtype: str):
    """Return (storage array, exact float64 value of that storage).

    dtype "bf16": storage is uint16 bf16 bits; "f32": storage is float32.
    """
    if dtype == "bf16":
        bits = bf16_bits(a)
        return bits, bf16_bits_to_f64(bits)
    if dtype == "f32":
        f = np.asarray(a, dtype=np.float32)
        return f, f.astype(np.float64)
    raise ValueError(f"unknown storage dtype {dtype!r}")


def _f32(a):
    f = np.asarray(a, dtype=np.float32)
    return f, f.astype(np.float64)


# ----------------------------------------------------------------------------------
# prefill inputs
# ----------------------------------------------------------------------------------
def prefill_inputs(B, L, H, P, G, N, dtype="bf16", seed=0, h0=False,
                   dt_bias_zero=True, unclipped=False, a_log=None, dt_clip=None):
    """Seeded prefill inputs.

    Returns a dict whose entries are pairs (storage, f64) for
    x[B,L,H,P], dt[B,L,H] (raw, before softplus), Bm[B,L,G,N], Cm[B,L,G,N] in the
    storage dtype, and A_log[H], D[H], dt_bias[H], h0[B,H,P,N] (or None) in fp32,
    plus dt_min / dt_max.  ``unclipped`` widens the clip so the softplus branch is
    exercised over its whole range (the workload clip saturates ~60% of dt at 0.1).
    ``a_log`` replaces the drawn A_log (a scalar for every head, or one value per head)
    and ``dt_clip`` = (dt_min, dt_max) replaces the clip range: the decay edge cases
    (no decay, full decay, steep decay inside one block) are made from these.
    """
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, L, H, P), dtype=np.float32)
    dt = rng.standard_normal((B, L, H), dtype=np.float32) - 2.0
    s = np.float32(1.0 / math.sqrt(N))
    Bm = rng.standard_normal((B, L, G, N), dtype=np.float32) * s
    Cm = rng.standard_normal((B, L, G, N), dtype=np.float32) * s
    A_log = np.log(rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    if dt_bias_zero:
        dt_bias = np.zeros(H, dtype=np.float32)
    else:
        dt_bias = (rng.standard_normal(H) * 0.5).astype(np.float32)
    out = {
        "x": to_storage(x, dtype), "dt": to_storage(dt, dtype),
        "Bm": to_storage(Bm, dtype), "Cm": to_storage(Cm, dtype),
        "A_log": _f32(A_log), "D": _f32(D), "dt_bias": _f32(dt_bias),
        "h0": None,
        "dt_min": 1e-3, "dt_max": 0.1,
    }
    if unclipped:
        out["dt_min"], out["dt_max"] = 0.0, float("inf")
    if a_log is not None:
        out["A_log"] = _f32(np.broadcast_to(np.asarray(a_log, dtype=np.float32), (H,)).copy())
    if dt_clip is not None:
        out["dt_min"], out["dt_max"] = float(dt_clip[0]), float(dt_clip[1])
    if h0:
        out["h0"] = _f32(rng.standard_normal((B, H, P, N), dtype=np.float32)
                         * np.float32(math.sqrt(0.1)))
    return out


# ----------------------------------------------------------------------------------
# decode inputs
# ----------------------------------------------------------------------------------
def decode_params(H, P, G, N, K, seed=0):
    """Per-layer decode parameters: A_log, D, dt_bias (fp32) and conv weight/bias (bf16)."""
    rng = np.random.default_rng(seed)
    Cc = H * P + 2 * G * N
    bound = 1.0 / math.sqrt(K)
    A_log = np.log(rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    dt_bias = np.zeros(H, dtype=np.float32)
    conv_w = rng.uniform(-bound, bound, size=(Cc, K)).astype(np.float32)
    conv_b = rng.uniform(-bound, bound, size=Cc).astype(np.float32)
    return {
        "A_log": _f32(A_log), "D": _f32(D), "dt_bias": _f32(dt_bias),
        "conv_w": to_storage(conv_w, "bf16"), "conv_b": to_storage(conv_b, "bf16"),
        "dt_min": 1e-3, "dt_max": 0.1,
    }


def raw_xbc_sequence(B, L, H, P, G, N, dtype="bf16", seed=0):
    """Raw (pre-conv) xBC[B,L,Cc] and raw dt[B,L,H] for a token sequence."""
    rng = np.random.default_rng(seed)
    Cc = H * P + 2 * G * N
    xbc = rng.standard_normal((B, L, Cc), dtype=np.float32)
    xbc[..., H * P:] *= np.float32(1.0 / math.sqrt(N))
    dt = rng.standard_normal((B, L, H), dtype=np.float32) - 2.0
    return {"xBC": to_storage(xbc, dtype), "dt": to_storage(dt, dtype)}


def decode_token_inputs(B, H, P, G, N, K, dtype="bf16", seed=0, state_std=0.1):
    """One decode step's inputs with a random (not prefilled) starting cache."""
    rng = np.random.default_rng(seed)
    Cc = H * P + 2 * G * N
    ssm = rng.standard_normal((B, H, P, N), dtype=np.float32) * np.float32(state_std)
    conv_state = rng.standard_normal((B, Cc, K - 1), dtype=np.float32)
    conv_state[:, H * P:, :] *= np.float32(1.0 / math.sqrt(N))
    xbc = rng.standard_normal((B, Cc), dtype=np.float32)
    xbc[:, H * P:] *= np.float32(1.0 / math.sqrt(N))
    dt = rng.standard_normal((B, H), dtype=np.float32) - 2.0
    return {
        "ssm_state": _f32(ssm), "conv_state": to_storage(conv_state, dtype),
        "xBC_t": to_storage(xbc, dtype), "dt_t": to_storage(dt, dtype),
    }


# ----------------------------------------------------------------------------------
# gated norm inputs
# ----------------------------------------------------------------------------------
def norm_inputs(T, C, dtype="bf16", seed=0):
    """y[T, C] and z[T, C] in the storage dtype, w[C] fp32."""
    rng = np.random.default_rng(seed)
    y = rng.standard_normal((T, C), dtype=np.float32)
    z = rng.standard_normal((T, C), dtype=np.float32)
    w = rng.uniform(0.5, 1.5, size=C).astype(np.float32)
    return {"y": to_storage(y, dtype), "z": to_storage(z, dtype), "w": _f32(w)}


def varlen_lengths(n=64, lo=64, hi=4096, seed=2024):
    """Lengths of a packed varlen batch: n sequences of lo .. hi tokens, log-uniform (many short
    sequences beside a few long ones, as in a serving batch of prompts).  The default is the
    batch the varlen bench leg times: 64 sequences, 51908 tokens, 439 blocks of 128."""
    rng = np.random.default_rng(seed)
    return [int(v) for v in np.exp(rng.uniform(np.log(lo), np.log(hi), n)).round()]
