"""B200-native (sm_100a) fused scaled dot-product attention forward."""
