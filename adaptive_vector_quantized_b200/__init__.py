"""B200-native AVQ-Attention forward (placeholder; binding added with the library)."""
