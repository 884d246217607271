"""B200-native LongFlow fused decode step (attention + zero-cost score + eviction)."""
