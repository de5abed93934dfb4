"""B200-native Sparse Delta Memory recurrent core (placeholder during bring-up)."""
