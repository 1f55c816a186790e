"""Packed-sequence metadata in the form the C ABI takes (include/csa.h)."""
from __future__ import annotations

import torch


def cu_from_lengths(seqlens, m: int):
    """cu_seqlens and cu_blocks (int32 CPU tensors) of packed sequences.

    Sequence b of L_b tokens owns floor(L_b / m) compressed entries; cu_blocks
    holds the running offsets of those entries, cu_seqlens those of the tokens.
    """
    cu, cb = [0], [0]
    for L in seqlens:
        cu.append(cu[-1] + int(L))
        cb.append(cb[-1] + int(L) // m)
    return torch.tensor(cu, dtype=torch.int32), torch.tensor(cb, dtype=torch.int32)
