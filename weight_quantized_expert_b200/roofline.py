"""Algorithmic byte and flop counts of one MoE layer forward (what the method must move).

Bytes = weights of the experts actually selected (union over the batch) + the shared
expert + the router + activations in (fp32 x) and out (fp32 y).  Scales are counted
once per group.  Flops count 2 per multiply-add of the dense contractions.
"""
from __future__ import annotations

H, E, TOPK, I, IS = 1280, 64, 6, 896, 1792
VOCAB, DENSE_I = 129280, 6848
W_BF16, W_INT8, W_INT4 = 0, 1, 2


def matrix_bytes(rows: int, cols: int, wtype: int, group: int) -> int:
    n = rows * cols
    if wtype == W_BF16:
        return 2 * n
    codes = n // 2 if wtype == W_INT4 else n
    groups = rows * ((cols + group - 1) // group)
    return codes + 4 * groups


def swiglu_bytes(inter: int, wtype: int, group: int) -> int:
    return 2 * matrix_bytes(inter, H, wtype, group) + matrix_bytes(H, inter, wtype, group)


def moe_layer_bytes(T: int, routed_type: int, shared_type: int, group: int, experts_hit: int) -> int:
    return (experts_hit * swiglu_bytes(I, routed_type, group)
            + swiglu_bytes(IS, shared_type, group)
            + E * H * 2
            + T * H * 4 * 2)


def moe_layer_flops(T: int) -> int:
    # router + 6 routed experts + shared expert per token
    return T * 2 * (E * H + TOPK * 3 * I * H + 3 * IS * H)
