"""Paged-KV decode attention for B200 (sm_100a)."""
