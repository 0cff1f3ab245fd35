"""B200-native SparsePR per-call sparse attention operator (sm_100a CUDA behind a C ABI)."""
__all__ = ["configs", "gen"]
