"""Blockwise-E4M3 FP8 linear layer for B200 (sm_100a)."""
