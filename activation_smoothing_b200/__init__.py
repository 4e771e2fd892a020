"""Rotated Runtime Smooth W4A4 linear layer for B200 (sm_100a)."""
