"""B200-native selective scan (Mamba S6): forward, backward and decode step.

The compute lives in libss.so (hand-written sm_100a CUDA behind the C ABI of
include/ss.h); ``ops`` is its ctypes binding.
"""
from .ops import (SSError, fwd_path, lib, selective_scan_fn, ss_bwd, ss_fwd,  # noqa: F401
                  ss_state_update)
