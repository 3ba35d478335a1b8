"""B200-native SSD chunked scan and decode state update (sm_100a CUDA behind a C ABI).

    from state_space_model_07_b200 import chunk_scan_fwd, chunk_scan_bwd, state_update

Both calls go straight to libssd.so (include/ssd.h); there is no CPU path.
"""
from .ops import SsdError, chunk_scan_bwd, chunk_scan_fwd, state_update  # noqa: F401
