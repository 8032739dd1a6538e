"""B200-native selective scan (Mamba S6): forward, backward and decode step,
with state passing and packed documents, the causal depthwise conv1d that
feeds the scan, and the Mamba-2 SSD forward.

The compute lives in libss.so (hand-written sm_100a CUDA behind the C ABI of
include/ss.h); ``ops`` is its ctypes binding.
"""
from .ops import (SSError, causal_conv1d_fn, conv1d_bwd, conv1d_fwd,  # noqa: F401
                  conv1d_step, fwd_path, lib, selective_scan_fn, ss_bwd, ss_fwd,
                  ss_state_update, ssd_fwd)
