"""Throughput accounting of a streamed training step.

The MegaTrain pages report "sustained TFLOPS" with the model-FLOPs formula
6ND + 12LHT^2 (Table 7 caption): N parameters, D tokens per step, L layers,
H hidden size, T sequence length; the attention term is counted per
sequence, so it is multiplied by the number of sequences B (Table 7's 256K
and 512K rows agree with their step times only that way). Tokens/s is
D / step time (Table 9).
"""
from __future__ import annotations


def model_flops(N: float, L: int, H: int, B: int, T: int) -> float:
    """6ND + 12 L H T^2 per sequence, with D = B*T tokens."""
    D = float(B) * float(T)
    return 6.0 * float(N) * D + 12.0 * float(L) * float(H) * float(T) ** 2 * float(B)


def sustained_tflops(N: float, L: int, H: int, B: int, T: int, step_s: float) -> float:
    return model_flops(N, L, H, B, T) / step_s / 1e12


def tokens_per_s(B: int, T: int, step_s: float) -> float:
    return float(B) * float(T) / step_s
