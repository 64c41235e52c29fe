"""B200-native Sparse-BitNet BitLinear path (placeholder; binding added below)."""
