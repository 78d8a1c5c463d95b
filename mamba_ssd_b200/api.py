"""Python binding of the C ABI, with the same names.  Argument marshalling only: torch
tensors supply device memory and the current CUDA stream; every step of the SSD runs in
the library's kernels.

Shapes and dtypes follow include/mamba_ssd.h:
  activations (x, dt, Bm, Cm, y, xBC, conv_state, conv_w, conv_b) are float32 or bfloat16,
  all the same; A_log, D, dt_bias, h0, h_final, ssm_state are float32.
"""
from __future__ import annotations

import math

import torch

from . import _lib
from ._lib import SSD_DTYPE_BF16, SSD_DTYPE_F32, check

_DTYPES = {torch.float32: SSD_DTYPE_F32, torch.bfloat16: SSD_DTYPE_BF16}


def _ptr(t):
    return None if t is None else t.data_ptr()


def _dtype_code(t):
    try:
        return _DTYPES[t.dtype]
    except KeyError:
        raise TypeError(f"unsupported activation dtype {t.dtype}") from None


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _need(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def ssd_chunk_scan_workspace_size(B, L, H, P, G, N, chunk=256, dtype=torch.bfloat16):
    return int(_lib.lib().ssd_chunk_scan_workspace_size(B, L, H, P, G, N, chunk, _DTYPES[dtype]))


def ssd_chunk_scan_fwd(x, dt, A_log, Bm, Cm, D=None, chunk=256, h0=None, dt_bias=None,
                       dt_min=0.0, dt_max=math.inf, y=None, h_final=None, workspace=None,
                       want_h_final=True, want_y=True, stream=None):
    """Chunked SSD prefill.  Returns (y, h_final); h_final is None if not wanted, y is None
    when want_y is False (then only the state the sequence leaves is computed)."""
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    dt_code = _dtype_code(x)
    _need(x, "x")
    _need(dt, "dt", x.dtype, (Bsz, L, H))
    _need(Bm, "Bm", x.dtype, (Bsz, L, G, N))
    _need(Cm, "Cm", x.dtype, (Bsz, L, G, N))
    _need(A_log, "A_log", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(h0, "h0", torch.float32, (Bsz, H, P, N))
    if y is None and want_y:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, x.shape)
    if h_final is None and want_h_final:
        h_final = torch.empty((Bsz, H, P, N), device=x.device, dtype=torch.float32)
    _need(h_final, "h_final", torch.float32, (Bsz, H, P, N))
    need = _lib.lib().ssd_chunk_scan_workspace_size(Bsz, L, H, P, G, N, chunk, dt_code)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=x.device, dtype=torch.uint8)
    s = _lib.lib().ssd_chunk_scan_fwd(
        _ptr(x), _ptr(dt), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(dt_bias),
        float(dt_min), float(dt_max), _ptr(h0), _ptr(y), _ptr(h_final),
        Bsz, L, H, P, G, N, int(chunk), dt_code, _ptr(workspace), workspace.numel(),
        _stream(stream))
    check(s, "ssd_chunk_scan_fwd")
    return y, h_final


def ssd_conv_chunk_scan_workspace_size(B, L, H, P, G, N, K, chunk=256, dtype=torch.bfloat16):
    return int(_lib.lib().ssd_conv_chunk_scan_workspace_size(B, L, H, P, G, N, K, chunk, _DTYPES[dtype]))


def ssd_conv_chunk_scan_fwd(xBC, conv_w, conv_b, dt, A_log, H, P, G, N, D=None, chunk=256, h0=None,
                            dt_bias=None, dt_min=0.0, dt_max=math.inf, y=None, h_final=None,
                            conv_state_out=None, want_h_final=True, want_state=True, workspace=None,
                            stream=None):
    """Causal conv + SiLU of the raw xBC [B, L, Cc] (channels [x | B | C]) and the chunked SSD
    prefill over its output, in one call.  Returns (y [B,L,H,P], h_final [B,H,P,N] or None,
    conv_state_out [B,Cc,K-1] or None)."""
    Bsz, L, Cc = xBC.shape
    K = conv_w.shape[1]
    code = _dtype_code(xBC)
    if Cc != H * P + 2 * G * N:
        raise ValueError(f"xBC has {Cc} channels, expected H*P + 2*G*N = {H * P + 2 * G * N}")
    _need(xBC, "xBC")
    _need(conv_w, "conv_w", xBC.dtype, (Cc, K))
    _need(conv_b, "conv_b", xBC.dtype, (Cc,))
    _need(dt, "dt", xBC.dtype, (Bsz, L, H))
    _need(A_log, "A_log", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(h0, "h0", torch.float32, (Bsz, H, P, N))
    if y is None:
        y = torch.empty((Bsz, L, H, P), device=xBC.device, dtype=xBC.dtype)
    _need(y, "y", xBC.dtype, (Bsz, L, H, P))
    if h_final is None and want_h_final:
        h_final = torch.empty((Bsz, H, P, N), device=xBC.device, dtype=torch.float32)
    _need(h_final, "h_final", torch.float32, (Bsz, H, P, N))
    if conv_state_out is None and want_state:
        conv_state_out = torch.empty((Bsz, Cc, K - 1), device=xBC.device, dtype=xBC.dtype)
    _need(conv_state_out, "conv_state_out", xBC.dtype, (Bsz, Cc, K - 1))
    need = _lib.lib().ssd_conv_chunk_scan_workspace_size(Bsz, L, H, P, G, N, K, chunk, code)
    if workspace is None:
        workspace = torch.empty(max(need, 256), device=xBC.device, dtype=torch.uint8)
    s = _lib.lib().ssd_conv_chunk_scan_fwd(
        _ptr(xBC), _ptr(conv_w), _ptr(conv_b), _ptr(dt), _ptr(A_log), _ptr(D), _ptr(dt_bias),
        float(dt_min), float(dt_max), _ptr(h0), _ptr(y), _ptr(h_final), _ptr(conv_state_out),
        Bsz, L, H, P, G, N, K, int(chunk), code, _ptr(workspace), workspace.numel(), _stream(stream))
    check(s, "ssd_conv_chunk_scan_fwd")
    return y, h_final, conv_state_out


def ssd_segment_decay(dt, A_log, dt_bias=None, dt_min=0.0, dt_max=math.inf, out=None, stream=None):
    """log2 of each (batch, head) segment's total decay, A_h * sum_t dt_t * log2(e), for dt
    [B, L, H] (raw).  Returns out [B, H] float32."""
    Bsz, L, H = dt.shape
    code = _dtype_code(dt)
    _need(dt, "dt")
    _need(A_log, "A_log", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    if out is None:
        out = torch.empty((Bsz, H), device=dt.device, dtype=torch.float32)
    _need(out, "out", torch.float32, (Bsz, H))
    check(_lib.lib().ssd_segment_decay(_ptr(dt), _ptr(A_log), _ptr(dt_bias), float(dt_min), float(dt_max),
                                       _ptr(out), Bsz, L, H, code, _stream(stream)), "ssd_segment_decay")
    return out


def ssd_state_combine(states, log2_decays, r, h0=None, out=None, stream=None):
    """The state entering segment r of a split sequence: h = h0 (or 0), then
    h = exp2(log2_decays[j]) h + states[j] for j < r.  states [W, B, H, P, N] and log2_decays
    [W, B, H] float32 hold every segment's own final state and decay; r = W gives the state
    after the whole sequence.  Returns out [B, H, P, N]."""
    W, Bsz, H, P, N = states.shape
    if not 0 <= r <= W:
        raise ValueError(f"r = {r} outside 0 .. {W}")
    _need(states, "states", torch.float32)
    _need(log2_decays, "log2_decays", torch.float32, (W, Bsz, H))
    _need(h0, "h0", torch.float32, (Bsz, H, P, N))
    if out is None:
        out = torch.empty((Bsz, H, P, N), device=states.device, dtype=torch.float32)
    _need(out, "out", torch.float32, (Bsz, H, P, N))
    check(_lib.lib().ssd_state_combine(_ptr(states), _ptr(log2_decays), _ptr(h0), _ptr(out), int(r), Bsz, H, P,
                                       N, _stream(stream)), "ssd_state_combine")
    return out


def ssd_chunk_scan_varlen_workspace_size(cu_seqlens, H, P, G, N, chunk=256, dtype=torch.bfloat16):
    """Bytes of workspace ssd_chunk_scan_varlen_fwd needs for the batch cu_seqlens describes."""
    import ctypes
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    cu_arr = (ctypes.c_int * len(cu))(*cu)
    return int(_lib.lib().ssd_chunk_scan_varlen_workspace_size(ctypes.cast(cu_arr, ctypes.c_void_p), len(cu) - 1,
                                                               H, P, G, N, int(chunk), _DTYPES[dtype]))


def ssd_chunk_scan_varlen_fwd(x, dt, A_log, Bm, Cm, cu_seqlens, D=None, chunk=256, h0=None,
                              dt_bias=None, dt_min=0.0, dt_max=math.inf, y=None, h_final=None,
                              workspace=None, want_h_final=True, stream=None):
    """Varlen SSD prefill: x [T,H,P], dt [T,H], Bm/Cm [T,G,N] hold n sequences packed by the
    cumulative lengths cu_seqlens (n+1 ints on the host: a list, numpy array or CPU tensor).
    Returns (y [T,H,P], h_final [n,H,P,N] or None)."""
    import ctypes
    cu = [int(v) for v in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    n = len(cu) - 1
    T, H, P = x.shape
    G, N = Bm.shape[1], Bm.shape[2]
    code = _dtype_code(x)
    _need(x, "x")
    _need(dt, "dt", x.dtype, (T, H))
    _need(Bm, "Bm", x.dtype, (T, G, N))
    _need(Cm, "Cm", x.dtype, (T, G, N))
    _need(A_log, "A_log", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(h0, "h0", torch.float32, (n, H, P, N))
    if n < 0 or cu[-1] != T:
        raise ValueError(f"cu_seqlens must end at the token count {T}")
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", x.dtype, x.shape)
    if h_final is None and want_h_final:
        h_final = torch.empty((n, H, P, N), device=x.device, dtype=torch.float32)
    _need(h_final, "h_final", torch.float32, (n, H, P, N))
    cu_arr = (ctypes.c_int * len(cu))(*cu)
    if workspace is None:
        need = ssd_chunk_scan_varlen_workspace_size(cu, H, P, G, N, chunk, x.dtype)
        workspace = torch.empty(max(need, 256), device=x.device, dtype=torch.uint8)
    s = _lib.lib().ssd_chunk_scan_varlen_fwd(
        _ptr(x), _ptr(dt), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(dt_bias),
        float(dt_min), float(dt_max), _ptr(h0), _ptr(y), _ptr(h_final), ctypes.cast(cu_arr, ctypes.c_void_p),
        n, H, P, G, N, int(chunk), code, _ptr(workspace), workspace.numel(), _stream(stream))
    check(s, "ssd_chunk_scan_varlen_fwd")
    return y, h_final


def ssd_chunk_scan_fwd_noalloc(x, dt, A_log, Bm, Cm, D=None, chunk=256, h0=None, dt_bias=None,
                               dt_min=0.0, dt_max=math.inf, y=None, h_final=None, stream=None):
    """ssd_chunk_scan_fwd whose scratch is the library's built-in device array (no workspace
    argument; for callers that cannot allocate).  Outputs y and h_final are still supplied by
    the caller, or allocated here by torch when omitted.  Returns (y, h_final)."""
    Bsz, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    code = _dtype_code(x)
    _need(x, "x")
    _need(dt, "dt", x.dtype, (Bsz, L, H))
    _need(Bm, "Bm", x.dtype, (Bsz, L, G, N))
    _need(Cm, "Cm", x.dtype, (Bsz, L, G, N))
    _need(A_log, "A_log", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(h0, "h0", torch.float32, (Bsz, H, P, N))
    if y is None:
        y = torch.empty_like(x)
    if h_final is None:
        h_final = torch.empty((Bsz, H, P, N), device=x.device, dtype=torch.float32)
    _need(y, "y", x.dtype, x.shape)
    _need(h_final, "h_final", torch.float32, (Bsz, H, P, N))
    s = _lib.lib().ssd_chunk_scan_fwd_noalloc(
        _ptr(x), _ptr(dt), _ptr(A_log), _ptr(Bm), _ptr(Cm), _ptr(D), _ptr(dt_bias),
        float(dt_min), float(dt_max), _ptr(h0), _ptr(y), _ptr(h_final),
        Bsz, L, H, P, G, N, int(chunk), code, _stream(stream))
    check(s, "ssd_chunk_scan_fwd_noalloc")
    return y, h_final


def ssd_chunk_scan_status(workspace, stream=None):
    """Synchronises the stream and returns the status word the last prefill on `workspace`
    left: SSD_OK (0), or SSD_ERR_TIMEOUT (5) if a bounded wait in a kernel gave up.
    workspace=None reads the built-in scratch of ssd_chunk_scan_fwd_noalloc on the current
    device."""
    return _lib.lib().ssd_chunk_scan_status(_ptr(workspace), _stream(stream))


def ssd_decode_status(workspace, stream=None):
    """Synchronises the stream and returns the status word the last decode step on
    `workspace` left: SSD_OK (0), or SSD_ERR_TIMEOUT (5)."""
    return _lib.lib().ssd_decode_status(_ptr(workspace), _stream(stream))


def ssd_selftest_wait_timeout(limit_us, device="cuda", stream=None):
    """Runs the bounded-wait self-test (a wait on an mbarrier that nothing arrives at, given
    up after `limit_us` microseconds) and returns the status it recorded: SSD_ERR_TIMEOUT."""
    status = torch.zeros(1, device=device, dtype=torch.int32)
    check(_lib.lib().ssd_selftest_wait_timeout(_ptr(status), int(limit_us), _stream(stream)),
          "ssd_selftest_wait_timeout")
    return int(status.item())


def ssd_decode_workspace_size(B, H, P, G, N):
    return int(_lib.lib().ssd_decode_workspace_size(B, H, P, G, N))


def decode_workspace(B, H, P, G, N, device="cuda"):
    """A decode workspace (status word, the step's conv outputs and (dt, a) pairs), reusable
    across calls of this shape or smaller on one stream.  Zero-filled only so that the status
    word reads SSD_OK before the first call; the kernels need no initialisation."""
    return torch.zeros(max(ssd_decode_workspace_size(B, H, P, G, N), 256), device=device, dtype=torch.uint8)


def ssd_decode_step(ssm_state, conv_state, xBC_t, dt_t, A_log, D, dt_bias, conv_w, conv_b,
                    H, P, G, N, dt_min=0.0, dt_max=math.inf, y_t=None, workspace=None,
                    stream=None):
    """One cached decode step; updates ssm_state and conv_state in place.  Returns y_t."""
    Bsz = ssm_state.shape[0]
    K = conv_w.shape[1]
    Cc = H * P + 2 * G * N
    code = _dtype_code(xBC_t)
    _need(ssm_state, "ssm_state", torch.float32, (Bsz, H, P, N))
    _need(conv_state, "conv_state", xBC_t.dtype, (Bsz, Cc, K - 1))
    _need(xBC_t, "xBC_t", None, (Bsz, Cc))
    _need(dt_t, "dt_t", xBC_t.dtype, (Bsz, H))
    _need(A_log, "A_log", torch.float32, (H,))
    _need(D, "D", torch.float32, (H,))
    _need(dt_bias, "dt_bias", torch.float32, (H,))
    _need(conv_w, "conv_w", xBC_t.dtype, (Cc, K))
    _need(conv_b, "conv_b", xBC_t.dtype, (Cc,))
    if y_t is None:
        y_t = torch.empty((Bsz, H, P), device=xBC_t.device, dtype=xBC_t.dtype)
    _need(y_t, "y_t", xBC_t.dtype, (Bsz, H, P))
    if workspace is None:
        workspace = decode_workspace(Bsz, H, P, G, N, xBC_t.device)
    s = _lib.lib().ssd_decode_step(
        _ptr(ssm_state), _ptr(conv_state), _ptr(xBC_t), _ptr(dt_t), _ptr(A_log), _ptr(D),
        _ptr(dt_bias), float(dt_min), float(dt_max), _ptr(conv_w), _ptr(conv_b), _ptr(y_t),
        Bsz, H, P, G, N, K, code, _ptr(workspace), workspace.numel(), _stream(stream))
    check(s, "ssd_decode_step")
    return y_t


def ssd_causal_conv1d_fwd(xBC, conv_w, conv_b=None, out=None, conv_state_out=None,
                          want_state=True, stream=None):
    """Prefix causal conv + SiLU.  Returns (out, conv_state_out)."""
    Bsz, L, Cc = xBC.shape
    K = conv_w.shape[1]
    code = _dtype_code(xBC)
    _need(xBC, "xBC")
    _need(conv_w, "conv_w", xBC.dtype, (Cc, K))
    _need(conv_b, "conv_b", xBC.dtype, (Cc,))
    if out is None:
        out = torch.empty_like(xBC)
    if conv_state_out is None and want_state:
        conv_state_out = torch.empty((Bsz, Cc, K - 1), device=xBC.device, dtype=xBC.dtype)
    s = _lib.lib().ssd_causal_conv1d_fwd(
        _ptr(xBC), _ptr(conv_w), _ptr(conv_b), _ptr(out), _ptr(conv_state_out), Bsz, L, Cc, K,
        code, _stream(stream))
    check(s, "ssd_causal_conv1d_fwd")
    return out, conv_state_out


def ssd_gated_rmsnorm_fwd(y, z, w, n_groups=1, eps=1e-5, out=None, stream=None):
    """Gated RMS norm over the last axis: y * SiLU(z), RMS-normalised per token and norm
    group (fp32 mean square), times w.  y and z share shape [..., C] and dtype; w is [C]
    float32.  Returns out (same shape and dtype as y)."""
    C = y.shape[-1]
    code = _dtype_code(y)
    _need(y, "y")
    _need(z, "z", y.dtype, tuple(y.shape))
    _need(w, "w", torch.float32, (C,))
    if out is None:
        out = torch.empty_like(y)
    _need(out, "out", y.dtype, tuple(y.shape))
    T = y.numel() // C if C else 0
    s = _lib.lib().ssd_gated_rmsnorm_fwd(_ptr(y), _ptr(z), _ptr(w), _ptr(out), T, C, int(n_groups),
                                         float(eps), code, _stream(stream))
    check(s, "ssd_gated_rmsnorm_fwd")
    return out
