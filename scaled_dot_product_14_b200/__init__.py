"""B200-native fused scaled-dot-product attention forward (sm_100a)."""
