"""Prism Attention decode hot path for B200 (sm_100a)."""
