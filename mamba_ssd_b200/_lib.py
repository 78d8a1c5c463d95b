"""ctypes loader of the in-tree libmamba_ssd.so (the C ABI of include/mamba_ssd.h).

There is no fallback: if the shared library is missing or does not load, importing the
package raises, and every call goes through the CUDA kernels.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmamba_ssd.so")

SSD_OK = 0
SSD_ERR_INVALID_ARG = 1
SSD_ERR_UNSUPPORTED = 2
SSD_ERR_WORKSPACE = 3
SSD_ERR_CUDA = 4
SSD_ERR_TIMEOUT = 5
SSD_DTYPE_F32 = 0
SSD_DTYPE_BF16 = 1
SSD_NOALLOC_SCRATCH_BYTES = 48 * 1024 * 1024

# name -> (restype, argtypes); must match include/mamba_ssd.h
_vp, _fp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
SIGNATURES = {
    "ssd_status_string": (ctypes.c_char_p, [_i]),
    "ssd_last_cuda_error": (_i, []),
    "ssd_abi_version": (_i, []),
    "ssd_chunk_scan_workspace_size": (_sz, [_i] * 8),
    "ssd_chunk_scan_varlen_workspace_size": (_sz, [_vp] + [_i] * 7),
    "ssd_chunk_scan_fwd": (_i, [_vp, _vp, _fp, _vp, _vp, _fp, _fp, _f, _f, _fp, _vp, _fp]
                           + [_i] * 8 + [_vp, _sz, _vp]),
    "ssd_chunk_scan_status": (_i, [_vp, _vp]),
    "ssd_conv_chunk_scan_workspace_size": (_sz, [_i] * 9),
    "ssd_segment_decay": (_i, [_vp, _fp, _fp, _f, _f, _fp, _i, _i, _i, _i, _vp]),
    "ssd_state_combine": (_i, [_fp, _fp, _fp, _fp, _i, _i, _i, _i, _i, _vp]),
    "ssd_conv_chunk_scan_fwd": (_i, [_vp, _vp, _vp, _vp, _fp, _fp, _fp, _f, _f, _fp, _vp, _fp, _vp]
                                + [_i] * 9 + [_vp, _sz, _vp]),
    "ssd_chunk_scan_varlen_fwd": (_i, [_vp, _vp, _fp, _vp, _vp, _fp, _fp, _f, _f, _fp, _vp, _fp, _vp]
                                  + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_chunk_scan_fwd_noalloc": (_i, [_vp, _vp, _fp, _vp, _vp, _fp, _fp, _f, _f, _fp, _vp, _fp]
                                   + [_i] * 8 + [_vp]),
    "ssd_decode_workspace_size": (_sz, [_i, _i, _i, _i, _i]),
    "ssd_decode_status": (_i, [_vp, _vp]),
    "ssd_decode_step": (_i, [_fp, _vp, _vp, _vp, _fp, _fp, _fp, _f, _f, _vp, _vp, _vp]
                        + [_i] * 7 + [_vp, _sz, _vp]),
    "ssd_causal_conv1d_fwd": (_i, [_vp] * 5 + [_i] * 5 + [_vp]),
    "ssd_selftest_wait_timeout": (_i, [_vp, _i, _vp]),
    "ssd_gated_rmsnorm_fwd": (_i, [_vp, _vp, _fp, _vp, _i, _i, _i, _f, _i, _vp]),
    "ssd_kernel_launch_count": (ctypes.c_longlong, []),
    "ssd_kernel_timer_enable": (_i, [_i]),
    "ssd_kernel_timer_read": (_i, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double),
                                   ctypes.POINTER(ctypes.c_longlong)]),
}


class SSDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        msg = lib().ssd_status_string(status).decode()
        if status == SSD_ERR_CUDA:
            msg += f" (cudaError {lib().ssd_last_cuda_error()})"
        super().__init__(f"{where}: status {status}: {msg}")


_lib = None


def lib():
    """The loaded shared library (loaded once)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m mamba_ssd_b200.build`")
        handle = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(handle, name)
            fn.restype = res
            fn.argtypes = args
        _lib = handle
    return _lib


def check(status: int, where: str) -> None:
    if status != SSD_OK:
        raise SSDError(status, where)
