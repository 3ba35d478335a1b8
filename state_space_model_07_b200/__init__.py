"""B200-native SSD chunked scan and decode state update (sm_100a CUDA behind a C ABI)."""
