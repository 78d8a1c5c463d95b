"""Mamba-2 SSD selective scan for NVIDIA B200 (sm_100a): chunked prefill and the O(1)
cached decode step, as CUDA kernels behind the C ABI of include/mamba_ssd.h.

Every call goes through libmamba_ssd.so (loaded on first use); if the library is missing
the call raises ImportError.  There is no CPU or PyTorch fallback.  Build it with
`python -m mamba_ssd_b200.build`.
"""
from ._lib import SSDError, lib as load_library
from .api import (decode_workspace, ssd_causal_conv1d_fwd, ssd_chunk_scan_fwd,
                  ssd_chunk_scan_fwd_noalloc, ssd_chunk_scan_status, ssd_chunk_scan_varlen_fwd,
                  ssd_chunk_scan_varlen_workspace_size, ssd_chunk_scan_workspace_size, ssd_conv_chunk_scan_fwd,
                  ssd_conv_chunk_scan_workspace_size,
                  ssd_decode_status, ssd_decode_step, ssd_decode_workspace_size,
                  ssd_gated_rmsnorm_fwd, ssd_segment_decay, ssd_selftest_wait_timeout, ssd_state_combine)

__all__ = ["SSDError", "load_library", "ssd_chunk_scan_fwd", "ssd_chunk_scan_fwd_noalloc",
           "ssd_chunk_scan_workspace_size", "ssd_chunk_scan_varlen_workspace_size", "ssd_chunk_scan_status",
           "ssd_decode_step",
           "ssd_decode_workspace_size", "ssd_decode_status", "decode_workspace", "ssd_causal_conv1d_fwd",
           "ssd_gated_rmsnorm_fwd", "ssd_selftest_wait_timeout", "ssd_chunk_scan_varlen_fwd",
           "ssd_conv_chunk_scan_fwd", "ssd_conv_chunk_scan_workspace_size", "ssd_segment_decay",
           "ssd_state_combine"]
