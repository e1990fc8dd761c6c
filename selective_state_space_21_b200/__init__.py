"""B200-native fused selective scan (S6).

The CUDA library ``lib/libmambascan.so`` (built from ``csrc/`` by
``selective_state_space_21_b200.build``) does all the work; ``scan`` is its
ctypes binding and ``inputs`` draws seeded synthetic inputs.
"""
from .scan import (MambaScanError, load_library, mamba_scan_bwd, mamba_scan_bwd_saved,
                   mamba_scan_fwd, mamba_scan_fwd_save, mamba_scan_stream_status, saved_bytes,
                   selective_scan_bwd, selective_scan_bwd_saved, selective_scan_fwd,
                   selective_scan_fwd_save)

__all__ = ["MambaScanError", "load_library", "mamba_scan_fwd", "mamba_scan_bwd",
           "mamba_scan_fwd_save", "mamba_scan_bwd_saved", "saved_bytes",
           "mamba_scan_stream_status", "selective_scan_fwd", "selective_scan_bwd",
           "selective_scan_fwd_save", "selective_scan_bwd_saved"]
