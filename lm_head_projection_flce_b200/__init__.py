"""B200-native fused LM-head projection + cross-entropy (sm_100a CUDA behind a C ABI)."""
