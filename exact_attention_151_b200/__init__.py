"""B200-native exact attention forward (fused, online softmax, per-row LSE)."""
