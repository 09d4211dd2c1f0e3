"""Fused randomized Hadamard rotation + 4-bit quantization of activations (B200)."""
