"""B200-native compensated sparse attention forward (sm_100a CUDA behind a C ABI)."""
