"""B200-native Flux-style DiT block forward (placeholder; binding added below)."""
