"""B200-native paged-KV decode / prefill attention (sm_100a)."""
