"""ctypes bindings of the fp64 C oracle (ssd_oracle.c).

Test infrastructure only.  All arrays are float64, C-contiguous, row-major, with the
layouts documented in ssd_oracle.c.
"""
from __future__ import annotations

import ctypes
import threading

import numpy as np

from . import build as _build

_lib = None
_lock = threading.Lock()
_dp = ctypes.POINTER(ctypes.c_double)


def _bind(lib):
    i, d = ctypes.c_int, ctypes.c_double
    lib.oracle_ssd_scan_seq.argtypes = [i] * 6 + [_dp] * 7 + [d, d, _dp, _dp, _dp]
    lib.oracle_ssd_scan_seq.restype = None
    lib.oracle_causal_conv1d.argtypes = [i] * 4 + [_dp] * 5
    lib.oracle_causal_conv1d.restype = None
    lib.oracle_decode_step.argtypes = [i] * 6 + [_dp] * 7 + [d, d, _dp, _dp, _dp]
    lib.oracle_decode_step.restype = None
    lib.oracle_dt.argtypes = [d, d, d, d]
    lib.oracle_dt.restype = d
    lib.oracle_max_threads.restype = i
    lib.oracle_set_threads.argtypes = [i]
    return lib


def _load():
    global _lib
    with _lock:
        if _lib is None:
            _lib = _bind(ctypes.CDLL(_build.build()))
    return _lib


class use_library:
    """Context manager: route every call to another build of ssd_oracle.c (a path to a
    shared object).  The mutation tests use it to check that the pins catch planted
    mistakes; nothing else should."""

    def __init__(self, path):
        self._new = _bind(ctypes.CDLL(path))

    def __enter__(self):
        global _lib
        _load()
        self._old, _lib = _lib, self._new
        return self

    def __exit__(self, *exc):
        global _lib
        _lib = self._old
        return False


def _p(a):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags.c_contiguous
    return a.ctypes.data_as(_dp)


def _f64(a):
    return None if a is None else np.ascontiguousarray(a, dtype=np.float64)


def max_threads() -> int:
    return _load().oracle_max_threads()


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def dt_value(dt_raw: float, bias: float, dt_min: float, dt_max: float) -> float:
    return _load().oracle_dt(dt_raw, bias, dt_min, dt_max)


def ssd_scan_sequential(x, dt_raw, A_log, Bm, Cm, D=None, dt_bias=None,
                        dt_min=0.0, dt_max=float("inf"), h0=None):
    """Token-by-token recurrence.  Returns (y [B,L,H,P], h_final [B,H,P,N])."""
    x, dt_raw, A_log, Bm, Cm, D, dt_bias, h0 = map(_f64, (x, dt_raw, A_log, Bm, Cm, D, dt_bias, h0))
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    assert dt_raw.shape == (Bsz, L, H) and Bm.shape == Cm.shape == (Bsz, L, G, N)
    assert H % G == 0
    y = np.empty_like(x)
    hf = np.empty((Bsz, H, P, N))
    _load().oracle_ssd_scan_seq(Bsz, L, H, P, G, N, _p(x), _p(dt_raw), _p(A_log), _p(Bm), _p(Cm),
                                _p(D), _p(dt_bias), float(dt_min), float(dt_max), _p(h0),
                                _p(y), _p(hf))
    return y, hf


def causal_conv1d(xBC, w, bias=None):
    """Prefix causal conv + SiLU.  Returns (out [B,L,Cc], conv_state [B,Cc,K-1])."""
    xBC, w, bias = map(_f64, (xBC, w, bias))
    Bsz, L, Cc = xBC.shape
    K = w.shape[1]
    out = np.empty_like(xBC)
    cs = np.empty((Bsz, Cc, max(K - 1, 0)))
    _load().oracle_causal_conv1d(Bsz, L, Cc, K, _p(xBC), _p(w), _p(bias), _p(out),
                                 _p(cs) if K > 1 else None)
    return out, cs


def decode_step(ssm_state, conv_state, xBC_t, dt_t, A_log, D, dt_bias, dt_min, dt_max,
                conv_w, conv_b, H, P, G, N):
    """One decode step on copies of the caches.  Returns (y_t, ssm_state', conv_state')."""
    ssm = np.array(ssm_state, dtype=np.float64, copy=True, order="C")
    cs = np.array(conv_state, dtype=np.float64, copy=True, order="C")
    xBC_t, dt_t, A_log, D, dt_bias, conv_w, conv_b = map(
        _f64, (xBC_t, dt_t, A_log, D, dt_bias, conv_w, conv_b))
    Bsz = ssm.shape[0]
    K = conv_w.shape[1]
    assert ssm.shape == (Bsz, H, P, N)
    assert cs.shape == (Bsz, H * P + 2 * G * N, K - 1)
    y = np.empty((Bsz, H, P))
    _load().oracle_decode_step(Bsz, H, P, G, N, K, _p(ssm), _p(cs), _p(xBC_t), _p(dt_t),
                               _p(A_log), _p(D), _p(dt_bias), float(dt_min), float(dt_max),
                               _p(conv_w), _p(conv_b), _p(y))
    return y, ssm, cs
