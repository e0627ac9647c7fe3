"""B200-native SparsePR per-call sparse attention (placeholder; binding added with the library)."""
