"""Packed low-bit, Hadamard-rotated linears on B200 (sm_100a)."""
