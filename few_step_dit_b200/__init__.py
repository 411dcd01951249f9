"""B200-native few-step Flash DiT hot path (sm_100a CUDA behind a C ABI)."""
