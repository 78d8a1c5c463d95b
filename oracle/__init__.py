"""fp64 CPU oracle of the Mamba-2 SSD selective scan (prefill and cached decode).

TEST INFRASTRUCTURE.  Only the test suite, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import, call or run anything in this package.
The CUDA library (``mamba_ssd_b200``) never imports it and shares no code with it.

Forms:
  native.ssd_scan_sequential  token-by-token recurrence (C, the definition)
  forms.ssd_chunked           chunk / segsum / einsum form of the pages (numpy)
  forms.ssd_dense             quadratic dual form M x (numpy, tiny inputs)
  native.causal_conv1d        prefix depthwise conv + SiLU and the cache it leaves (C)
  native.decode_step          one cached decode step (C)
  block.gated_rmsnorm         the block step after the scan: y * SiLU(z), RMS-normalised per
                              token and norm group, scaled per channel (numpy)
  varlen.ssd_scan_varlen      sequences of different lengths packed into one token stream,
                              each scanned on its own (a loop over native.ssd_scan_sequential)

Parity status: every function here is pinned by closed forms, invariants or
brute force in tests/test_oracle_pins.py and tests/test_oracle_norm.py; none is
"parity unpinned".
"""
from .native import (ssd_scan_sequential, causal_conv1d, decode_step, dt_value,
                     max_threads, set_threads)
from .forms import ssd_chunked, ssd_dense, discretise, softplus
from .block import gated_rmsnorm, silu
from .varlen import ssd_scan_varlen

__all__ = ["ssd_scan_sequential", "causal_conv1d", "decode_step", "dt_value", "max_threads",
           "set_threads", "ssd_chunked", "ssd_dense", "discretise", "softplus", "gated_rmsnorm", "silu",
           "ssd_scan_varlen"]
