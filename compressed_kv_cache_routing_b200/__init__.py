"""B200-native BasisKV decode attention over a compressed, paged KV cache."""
